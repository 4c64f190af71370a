// fwd_d128.cu -- the forward kernel's d = 128 instantiations.
#include "fwd_launch.cuh"

namespace attn_host {

int launch_fwd_d128(DeviceState* st, bool bf16, bool f32, int uk, const CUtensorMap& mq,
                    const CUtensorMap& mk, const CUtensorMap& mv, const CUtensorMap& mo,
                    const attn::KernelParams& kp, cudaStream_t stream) {
  return launch_d<128>(st, bf16, f32, uk, mq, mk, mv, mo, kp, stream);
}

}  // namespace attn_host

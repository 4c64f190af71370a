// fwd_launch.cuh -- launch of one forward kernel instantiation (shared by the
// translation units that instantiate the forward for different head dims).
#pragma once

#include "host.h"
#include "attn_kernel.cuh"

namespace attn_host {

template <int D, bool BF16, bool F32, bool ALIBI, int UK>
int launch_one(DeviceState* st, int bit, const CUtensorMap& mq, const CUtensorMap& mk,
               const CUtensorMap& mv, const CUtensorMap& mo, const attn::KernelParams& kp,
               cudaStream_t stream) {
  auto kern = attn::attn_fwd_kernel<D, BF16, F32, ALIBI, UK>;
  // At least half of the SM's shared memory, so that two CTAs can never share
  // an SM (each allocates all 512 TMEM columns).
  const int smem_need = attn::Geo<D>::SMEM_BYTES + 1024;
  const int smem = smem_need > 120 * 1024 ? smem_need : 120 * 1024;
  {
    std::lock_guard<std::mutex> lock(g_mu);
    if (!(st->attr_set & (1ull << bit))) {
      // The kernel re-splits its registers between warpgroups after launch;
      // that only works when every thread starts with LAUNCH_REGS registers.
      cudaFuncAttributes fa;
      if (cudaFuncGetAttributes(&fa, kern) != cudaSuccess) return ATTN_ERR_CUDA;
      if (fa.numRegs < attn::LAUNCH_REGS) return ATTN_ERR_UNSUPPORTED;
      if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, smem) != cudaSuccess)
        return ATTN_ERR_CUDA;
      st->attr_set |= 1ull << bit;
    }
  }
  const int grid = kp.num_units < st->sm_count ? kp.num_units : st->sm_count;
  const cudaError_t e = launch_overlapped(kern, grid, attn::NUM_THREADS, smem, stream, mq, mk, mv, mo, kp);
  g_launches.fetch_add(1, std::memory_order_relaxed);
  return e == cudaSuccess && cudaGetLastError() == cudaSuccess ? ATTN_OK : ATTN_ERR_CUDA;
}

template <int D, bool ALIBI, int UK>
int launch_da(DeviceState* st, bool bf16, bool f32, const CUtensorMap& mq, const CUtensorMap& mk,
              const CUtensorMap& mv, const CUtensorMap& mo, const attn::KernelParams& kp,
              cudaStream_t stream) {
  const int dbit = D == 16 ? 0 : D == 32 ? 1 : D == 64 ? 2 : 3;
  const int bit = UK * 32 + dbit * 8 + (ALIBI ? 4 : 0) + (bf16 ? 2 : 0) + (f32 ? 1 : 0);
  if (bf16)
    return f32 ? launch_one<D, true, true, ALIBI, UK>(st, bit, mq, mk, mv, mo, kp, stream)
               : launch_one<D, true, false, ALIBI, UK>(st, bit, mq, mk, mv, mo, kp, stream);
  return f32 ? launch_one<D, false, true, ALIBI, UK>(st, bit, mq, mk, mv, mo, kp, stream)
             : launch_one<D, false, false, ALIBI, UK>(st, bit, mq, mk, mv, mo, kp, stream);
}

// `uk`: the work-unit kind (attn::UK_PAIR, UK_SPLIT or UK_HEADS); launches
// with a position bias always use pairs.
template <int D>
int launch_d(DeviceState* st, bool bf16, bool f32, int uk, const CUtensorMap& mq,
             const CUtensorMap& mk, const CUtensorMap& mv, const CUtensorMap& mo,
             const attn::KernelParams& kp, cudaStream_t stream) {
  if (kp.alibi != nullptr)
    return launch_da<D, true, attn::UK_PAIR>(st, bf16, f32, mq, mk, mv, mo, kp, stream);
  if (uk == attn::UK_SPLIT)
    return launch_da<D, false, attn::UK_SPLIT>(st, bf16, f32, mq, mk, mv, mo, kp, stream);
  if (uk == attn::UK_HEADS)
    return launch_da<D, false, attn::UK_HEADS>(st, bf16, f32, mq, mk, mv, mo, kp, stream);
  return launch_da<D, false, attn::UK_PAIR>(st, bf16, f32, mq, mk, mv, mo, kp, stream);
}

// The d = 128 instantiations (compiled in their own translation unit).
int launch_fwd_d128(DeviceState* st, bool bf16, bool f32, int uk, const CUtensorMap& mq,
                    const CUtensorMap& mk, const CUtensorMap& mv, const CUtensorMap& mo,
                    const attn::KernelParams& kp, cudaStream_t stream);

}  // namespace attn_host

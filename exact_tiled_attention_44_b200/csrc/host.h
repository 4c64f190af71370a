// host.h -- host-side pieces shared by the translation units of libattn.so:
// per-device state, argument checks, TMA descriptor encoding and the process
// wide counters.  Internal to the library (not part of the C ABI).
#pragma once

#include <cuda.h>
#include <cuda_runtime.h>
#include <cudaTypedefs.h>

#include <atomic>
#include <cstddef>
#include <cstdint>
#include <mutex>
#include <utility>

#include "attn.h"

namespace attn_host {

constexpr int kMaxDevices = 64;
// attn_fwd_host overlaps its copies with the forward over at most this many
// chunks of the problem.
constexpr int kHostChunks = 16;

struct DeviceState {
  bool ready = false;
  int sm_count = 0;
  int cc_major = 0, cc_minor = 0;
  int* status = nullptr;           // device address of the status word
  uint64_t attr_set = 0;           // one bit per forward kernel instantiation
  uint32_t dec_attr_set = 0;       // one bit per decode kernel instantiation
  uint32_t bwd_attr_set = 0;       // one bit per backward kernel instantiation
  // attn_fwd_host: two copy streams and the events that order its chunks,
  // created on its first call on the device and kept (guarded by g_host_mu)
  bool host_ready = false;
  cudaStream_t copy_in = nullptr, copy_out = nullptr;
  cudaEvent_t ev[2 * kHostChunks + 2] = {};
};

// Guards DeviceState initialisation and the per-kernel attribute bits.
extern std::mutex g_mu;
extern std::atomic<unsigned long long> g_watchdog_ns;
extern std::atomic<unsigned long long> g_launches;
extern std::atomic<int> g_withhold;     // launches left that withhold their loads (test hook)
extern std::atomic<unsigned long long*> g_block_count;   // block-count test hook (or nullptr)
extern std::atomic<int> g_force_units;  // work-unit kind test hook: -1 automatic, else attn::UK_*
extern std::mutex g_host_mu;            // attn_fwd_host's streams and events
extern PFN_cuTensorMapEncodeTiled_v12000 g_encode;

inline bool overlaps(const void* a, size_t na, const void* b, size_t nb) {
  const uintptr_t x = reinterpret_cast<uintptr_t>(a), y = reinterpret_cast<uintptr_t>(b);
  return x < y + nb && y < x + na;
}

inline bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

inline size_t round_up(size_t x, size_t a) { return (x + a - 1) / a * a; }

struct Sizes {
  size_t q_bytes, kv_bytes, o_bytes, lse_bytes;
  int elem, d;
};

// Pure argument validation of the forward's arguments: touches no CUDA API,
// so it can be tested on a machine without a GPU.  Returns ATTN_OK and fills
// `sz` when the call is well formed; `*empty` is set when there is nothing to
// compute.
int validate(const void* q, const void* k, const void* v, const void* o, const float* lse,
             int B, int H, int H_kv, int N, int d, int causal, int window, int n_sink,
             float scale, int dtype, Sizes* sz, bool* empty);

// State of the current device, initialised on first use (an sm_100 device is
// required; anything else is ATTN_ERR_UNSUPPORTED).
int device_state(DeviceState** out);

// 3-D view [z][rows][d] of a contiguous [.., n, d] 16-bit tensor; box =
// (min(d, 64), 128, 1) with the swizzle span equal to the box's row bytes.
int encode_map(CUtensorMap* map, const void* base, bool bf16, int d, int n, int z);

// Launches `kern` with programmatic stream serialisation: its CTAs may be
// scheduled while the previous grid of the stream drains, run their set-up
// (barriers, TMEM, descriptor prefetch) and then wait for that grid in
// grid_dependency_wait before their first memory access.
template <typename... Params, typename... Args>
cudaError_t launch_overlapped(void (*kern)(Params...), int grid, int block, size_t smem,
                              cudaStream_t stream, Args&&... args) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(grid);
  cfg.blockDim = dim3(block);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, kern, std::forward<Args>(args)...);
}

// Takes one launch from the withhold-loads test hook, if any is pending.
int take_withhold();

// The forward's work-unit kind (attn::UK_*): split units (one Q tile, its
// key blocks shared out between the two softmax warpgroups) when pairs of Q
// tiles would leave SMs idle and single tiles still fit about two waves; head
// pairs for grouped heads whose rows see at most 4096 keys; pairs otherwise
// and under a position bias.
int fwd_unit_kind(int B, int H, int H_kv, int N, int window, bool alibi, int sm_count);

// attn_fwd with an optional slope array (NULL: no position bias).  uk: the
// work-unit kind, or -1 for the test hook's choice, else fwd_unit_kind's
// (callers that cut one problem into several launches pass the whole
// problem's kind, so that every row is computed as the uncut call computes it).
int fwd_impl(const void* q, const void* k, const void* v, void* o, float* lse,
             const float* slopes, int B, int H, int H_kv, int N, int d, int causal, int window,
             int n_sink, float scale, int dtype, void* stream, int uk = -1);

}  // namespace attn_host

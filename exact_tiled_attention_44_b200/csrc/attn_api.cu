// attn_api.cu -- host side of libattn.so: argument checks, TMA descriptors,
// persistent-grid launch, and the small host-only helpers of include/attn.h.
#include <cuda.h>
#include <cuda_runtime.h>
#include <cudaTypedefs.h>

#include <atomic>
#include <cmath>
#include <cstdint>
#include <cstring>
#include <mutex>

#include "attn.h"
#include "attn_kernel.cuh"
#include "bwd_kernel.cuh"
#include "decode_kernel.cuh"

namespace {

// Device status word: written by a CTA whose wait timed out, read and cleared
// by attn_get_status().
__device__ int g_device_status = 0;

constexpr int kMaxDevices = 64;

struct DeviceState {
  bool ready = false;
  int sm_count = 0;
  int cc_major = 0, cc_minor = 0;
  int* status = nullptr;           // device address of g_device_status
  uint32_t attr_set = 0;           // one bit per forward kernel instantiation
  uint32_t dec_attr_set = 0;       // one bit per decode kernel instantiation
  uint32_t dec_small_attr_set = 0; // one bit per small-group decode kernel instantiation
  uint32_t bwd_attr_set = 0;       // one bit per backward kernel instantiation
};

DeviceState g_dev[kMaxDevices];
std::mutex g_mu;
std::atomic<unsigned long long> g_watchdog_ns{2000000000ull};
std::atomic<unsigned long long> g_launches{0};
std::atomic<int> g_withhold{0};     // launches left that withhold their loads (test hook)
PFN_cuTensorMapEncodeTiled_v12000 g_encode = nullptr;

bool overlaps(const void* a, size_t na, const void* b, size_t nb) {
  const uintptr_t x = reinterpret_cast<uintptr_t>(a), y = reinterpret_cast<uintptr_t>(b);
  return x < y + nb && y < x + na;
}

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

struct Sizes {
  size_t q_bytes, kv_bytes, o_bytes, lse_bytes;
  int elem, d;
};

// Pure argument validation: touches no CUDA API, so it can be tested on a
// machine without a GPU.  Returns ATTN_OK and fills `sz` when the call is
// well formed; `*empty` is set when there is nothing to compute.
int validate(const void* q, const void* k, const void* v, const void* o, const float* lse,
             int B, int H, int H_kv, int N, int d, int causal, int window, int n_sink,
             float scale, int dtype, Sizes* sz, bool* empty) {
  *empty = false;
  if ((dtype & ~(ATTN_OUT_F32 | 0xF)) != 0) return ATTN_ERR_INVALID_ARG;
  const int base = dtype & 0xF;
  if (base != ATTN_BF16 && base != ATTN_FP16) return ATTN_ERR_INVALID_ARG;
  if (B < 0 || H < 0 || N < 0 || H_kv < 1 || d <= 0) return ATTN_ERR_INVALID_ARG;
  if (causal != 0 && causal != 1) return ATTN_ERR_INVALID_ARG;
  if (window < 0 || n_sink < 0) return ATTN_ERR_INVALID_ARG;
  if (!std::isfinite(scale)) return ATTN_ERR_INVALID_ARG;
  if (B == 0 || H == 0 || N == 0) {
    *empty = true;
    return ATTN_OK;
  }
  if (H % H_kv != 0) return ATTN_ERR_INVALID_ARG;
  if (d != 16 && d != 32 && d != 64 && d != 128) return ATTN_ERR_UNSUPPORTED;
  if (window > 0 && !causal) return ATTN_ERR_UNSUPPORTED;
  // index ranges: B*H (TMA z extent, unit count) and per-head element counts
  const long long bh = static_cast<long long>(B) * H;
  const long long n_pairs = (static_cast<long long>(N) + 2 * attn::BM - 1) / (2 * attn::BM);
  if (bh > INT32_MAX || bh * n_pairs > INT32_MAX) return ATTN_ERR_UNSUPPORTED;
  if (q == nullptr || k == nullptr || v == nullptr || o == nullptr) return ATTN_ERR_INVALID_ARG;
  if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(o) ||
      (lse != nullptr && !aligned16(lse)))
    return ATTN_ERR_MISALIGNED;
  const int elem = 2;
  const size_t rows_q = static_cast<size_t>(B) * H * N;
  const size_t rows_kv = static_cast<size_t>(B) * H_kv * N;
  sz->elem = elem;
  sz->d = d;
  sz->q_bytes = rows_q * d * elem;
  sz->kv_bytes = rows_kv * d * elem;
  sz->o_bytes = rows_q * d * ((dtype & ATTN_OUT_F32) ? 4 : elem);
  sz->lse_bytes = rows_q * sizeof(float);
  if (overlaps(o, sz->o_bytes, q, sz->q_bytes) || overlaps(o, sz->o_bytes, k, sz->kv_bytes) ||
      overlaps(o, sz->o_bytes, v, sz->kv_bytes))
    return ATTN_ERR_INVALID_ARG;
  if (lse != nullptr &&
      (overlaps(lse, sz->lse_bytes, q, sz->q_bytes) || overlaps(lse, sz->lse_bytes, k, sz->kv_bytes) ||
       overlaps(lse, sz->lse_bytes, v, sz->kv_bytes) || overlaps(lse, sz->lse_bytes, o, sz->o_bytes)))
    return ATTN_ERR_INVALID_ARG;
  return ATTN_OK;
}

int device_state(DeviceState** out) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return ATTN_ERR_CUDA;
  if (dev < 0 || dev >= kMaxDevices) return ATTN_ERR_UNSUPPORTED;
  std::lock_guard<std::mutex> lock(g_mu);
  DeviceState& st = g_dev[dev];
  if (!st.ready) {
    if (cudaDeviceGetAttribute(&st.sm_count, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess ||
        cudaDeviceGetAttribute(&st.cc_major, cudaDevAttrComputeCapabilityMajor, dev) != cudaSuccess ||
        cudaDeviceGetAttribute(&st.cc_minor, cudaDevAttrComputeCapabilityMinor, dev) != cudaSuccess)
      return ATTN_ERR_CUDA;
    if (st.cc_major != 10 || st.cc_minor != 0) return ATTN_ERR_UNSUPPORTED;
    void* addr = nullptr;
    if (cudaGetSymbolAddress(&addr, g_device_status) != cudaSuccess) return ATTN_ERR_CUDA;
    st.status = static_cast<int*>(addr);
    if (g_encode == nullptr) {
      cudaDriverEntryPointQueryResult qres;
      void* fn = nullptr;
      if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &fn, cudaEnableDefault, &qres) !=
              cudaSuccess ||
          qres != cudaDriverEntryPointSuccess || fn == nullptr)
        return ATTN_ERR_CUDA;
      g_encode = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(fn);
    }
    st.ready = true;
  }
  *out = &st;
  return ATTN_OK;
}

// 3-D view [z][rows][d] of a contiguous [.., N, d] tensor; box = (cw, 128, 1)
// with the swizzle span equal to the box's row bytes.
int encode_map(CUtensorMap* map, const void* base, bool bf16, int d, int n, int z) {
  const int cw = d < 64 ? d : 64;
  const cuuint64_t dims[3] = {static_cast<cuuint64_t>(d), static_cast<cuuint64_t>(n),
                              static_cast<cuuint64_t>(z)};
  const cuuint64_t strides[2] = {static_cast<cuuint64_t>(d) * 2,
                                 static_cast<cuuint64_t>(n) * d * 2};
  const cuuint32_t box[3] = {static_cast<cuuint32_t>(cw), 128u, 1u};
  const cuuint32_t estr[3] = {1u, 1u, 1u};
  const CUtensorMapSwizzle sw = cw * 2 == 128  ? CU_TENSOR_MAP_SWIZZLE_128B
                                : cw * 2 == 64 ? CU_TENSOR_MAP_SWIZZLE_64B
                                               : CU_TENSOR_MAP_SWIZZLE_32B;
  const CUresult r = g_encode(map, bf16 ? CU_TENSOR_MAP_DATA_TYPE_BFLOAT16 : CU_TENSOR_MAP_DATA_TYPE_FLOAT16,
                              3, const_cast<void*>(base), dims, strides, box, estr,
                              CU_TENSOR_MAP_INTERLEAVE_NONE, sw, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                              CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS ? ATTN_OK : ATTN_ERR_CUDA;
}

template <int D, bool BF16, bool F32, bool ALIBI>
int launch_one(DeviceState* st, int bit, const CUtensorMap& mq, const CUtensorMap& mk,
               const CUtensorMap& mv, const attn::KernelParams& kp, cudaStream_t stream) {
  auto kern = attn::attn_fwd_kernel<D, BF16, F32, ALIBI>;
  // At least half of the SM's shared memory, so that two CTAs can never share
  // an SM (each allocates all 512 TMEM columns).
  const int smem_need = attn::Geo<D>::SMEM_BYTES + 1024;
  const int smem = smem_need > 120 * 1024 ? smem_need : 120 * 1024;
  {
    std::lock_guard<std::mutex> lock(g_mu);
    if (!(st->attr_set & (1u << bit))) {
      // The kernel re-splits its registers between warpgroups after launch;
      // that only works when every thread starts with LAUNCH_REGS registers.
      cudaFuncAttributes fa;
      if (cudaFuncGetAttributes(&fa, kern) != cudaSuccess) return ATTN_ERR_CUDA;
      if (fa.numRegs < attn::LAUNCH_REGS) return ATTN_ERR_UNSUPPORTED;
      if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, smem) != cudaSuccess)
        return ATTN_ERR_CUDA;
      st->attr_set |= 1u << bit;
    }
  }
  const int grid = kp.num_units < st->sm_count ? kp.num_units : st->sm_count;
  kern<<<grid, attn::NUM_THREADS, smem, stream>>>(mq, mk, mv, kp);
  g_launches.fetch_add(1, std::memory_order_relaxed);
  return cudaGetLastError() == cudaSuccess ? ATTN_OK : ATTN_ERR_CUDA;
}

template <int D, bool ALIBI>
int launch_da(DeviceState* st, bool bf16, bool f32, const CUtensorMap& mq, const CUtensorMap& mk,
              const CUtensorMap& mv, const attn::KernelParams& kp, cudaStream_t stream) {
  const int dbit = D == 16 ? 0 : D == 32 ? 1 : D == 64 ? 2 : 3;
  const int bit = dbit * 8 + (ALIBI ? 4 : 0) + (bf16 ? 2 : 0) + (f32 ? 1 : 0);
  if (bf16)
    return f32 ? launch_one<D, true, true, ALIBI>(st, bit, mq, mk, mv, kp, stream)
               : launch_one<D, true, false, ALIBI>(st, bit, mq, mk, mv, kp, stream);
  return f32 ? launch_one<D, false, true, ALIBI>(st, bit, mq, mk, mv, kp, stream)
             : launch_one<D, false, false, ALIBI>(st, bit, mq, mk, mv, kp, stream);
}

template <int D>
int launch_d(DeviceState* st, bool bf16, bool f32, const CUtensorMap& mq, const CUtensorMap& mk,
             const CUtensorMap& mv, const attn::KernelParams& kp, cudaStream_t stream) {
  return kp.alibi != nullptr ? launch_da<D, true>(st, bf16, f32, mq, mk, mv, kp, stream)
                             : launch_da<D, false>(st, bf16, f32, mq, mk, mv, kp, stream);
}

// attn_fwd with an optional slope array (NULL: no position bias).
int fwd_impl(const void* q, const void* k, const void* v, void* o, float* lse,
             const float* slopes, int B, int H, int H_kv, int N, int d, int causal, int window,
             int n_sink, float scale, int dtype, void* stream) {
  Sizes sz;
  bool empty = false;
  int rc = validate(q, k, v, o, lse, B, H, H_kv, N, d, causal, window, n_sink, scale, dtype, &sz,
                    &empty);
  if (rc != ATTN_OK || empty) return rc;
  DeviceState* st = nullptr;
  rc = device_state(&st);
  if (rc != ATTN_OK) return rc;

  const bool bf16 = (dtype & 0xF) == ATTN_BF16;
  const bool f32 = (dtype & ATTN_OUT_F32) != 0;
  alignas(64) CUtensorMap mq, mk, mv;
  if (encode_map(&mq, q, bf16, d, N, B * H) != ATTN_OK ||
      encode_map(&mk, k, bf16, d, N, B * H_kv) != ATTN_OK ||
      encode_map(&mv, v, bf16, d, N, B * H_kv) != ATTN_OK)
    return ATTN_ERR_CUDA;

  attn::KernelParams kp;
  kp.o = o;
  kp.lse = lse;
  kp.status = st->status;
  kp.watchdog_ns = g_watchdog_ns.load(std::memory_order_relaxed);
  kp.B = B;
  kp.H = H;
  kp.H_kv = H_kv;
  kp.N = N;
  kp.causal = causal;
  // A window at least as long as the sequence keeps every causal key.
  kp.window = (window >= N) ? 0 : window;
  kp.n_sink = kp.window > 0 ? (n_sink < N ? n_sink : N) : 0;
  kp.scale_log2 = scale * 1.4426950408889634f;
  kp.n_qpairs = (N + 2 * attn::BM - 1) / (2 * attn::BM);
  kp.n_kblocks = (N + attn::BN - 1) / attn::BN;
  kp.num_units = B * H * kp.n_qpairs;
  kp.alibi = slopes;
  kp.withhold_loads = 0;
  for (int n = g_withhold.load(); n > 0;) {
    if (g_withhold.compare_exchange_weak(n, n - 1)) {
      kp.withhold_loads = 1;
      break;
    }
  }

  cudaStream_t s = static_cast<cudaStream_t>(stream);
  switch (d) {
    case 16: return launch_d<16>(st, bf16, f32, mq, mk, mv, kp, s);
    case 32: return launch_d<32>(st, bf16, f32, mq, mk, mv, kp, s);
    case 64: return launch_d<64>(st, bf16, f32, mq, mk, mv, kp, s);
    case 128: return launch_d<128>(st, bf16, f32, mq, mk, mv, kp, s);
    default: return ATTN_ERR_UNSUPPORTED;
  }
}

// ------------------------------------------------------------ decode

// Split rule (device independent, so that the workspace size can be queried
// without a device): at most two CTAs per SM of a 148-SM part in total (one
// wave; rounding the split count up would leave a short second wave), each
// split at least 256 keys long and a whole number of 64-key tiles.
struct DecodePlan {
  int n_splits, split_keys;
  size_t counters_off, lse_off, o_off, bytes;
};

size_t round_up(size_t x, size_t a) { return (x + a - 1) / a * a; }

DecodePlan decode_plan(int B, int H, int H_kv, int N_q, int N_kv, int d) {
  DecodePlan pl{};
  const long long groups = static_cast<long long>(B) * H_kv;
  const long long want = groups < 296 ? 296 / groups : 1;
  const long long max_splits = (static_cast<long long>(N_kv) + 255) / 256;
  long long s = want < max_splits ? want : max_splits;
  if (s < 1) s = 1;
  const long long per = (N_kv + s - 1) / s;
  pl.split_keys = static_cast<int>((per + attn::DEC_T - 1) / attn::DEC_T * attn::DEC_T);
  pl.n_splits = static_cast<int>((N_kv + pl.split_keys - 1) / pl.split_keys);
  if (pl.n_splits <= 1) {
    pl.n_splits = 1;
    pl.bytes = 0;
    return pl;
  }
  const size_t rows = static_cast<size_t>(pl.n_splits) * B * H * N_q;
  pl.counters_off = 0;
  pl.lse_off = round_up(static_cast<size_t>(groups) * sizeof(int), 256);
  pl.o_off = round_up(pl.lse_off + rows * sizeof(float), 256);
  pl.bytes = pl.o_off + rows * d * sizeof(float);
  return pl;
}

int validate_decode(const void* q, const void* k, const void* v, const void* o, const float* lse,
                    int B, int H, int H_kv, int N_q, int N_kv, int d, int causal, int window,
                    int n_sink, float scale, int dtype, bool* empty) {
  *empty = false;
  if ((dtype & ~(ATTN_OUT_F32 | 0xF)) != 0) return ATTN_ERR_INVALID_ARG;
  const int base = dtype & 0xF;
  if (base != ATTN_BF16 && base != ATTN_FP16) return ATTN_ERR_INVALID_ARG;
  if (B < 0 || H < 0 || N_q < 0 || N_kv < 0 || H_kv < 1 || d <= 0) return ATTN_ERR_INVALID_ARG;
  if (causal != 0 && causal != 1) return ATTN_ERR_INVALID_ARG;
  if (window < 0 || n_sink < 0) return ATTN_ERR_INVALID_ARG;
  if (!std::isfinite(scale)) return ATTN_ERR_INVALID_ARG;
  if (N_q > N_kv) return ATTN_ERR_INVALID_ARG;
  if (B == 0 || H == 0 || N_q == 0) {
    *empty = true;
    return ATTN_OK;
  }
  if (H % H_kv != 0) return ATTN_ERR_INVALID_ARG;
  if (d != 64 && d != 128) return ATTN_ERR_UNSUPPORTED;
  if (window > 0 && !causal) return ATTN_ERR_UNSUPPORTED;
  if (static_cast<long long>(H / H_kv) * N_q > attn::DEC_MAX_ROWS) return ATTN_ERR_UNSUPPORTED;
  if (static_cast<long long>(B) * H_kv > 65535) return ATTN_ERR_UNSUPPORTED;
  if (q == nullptr || k == nullptr || v == nullptr || o == nullptr) return ATTN_ERR_INVALID_ARG;
  if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(o) ||
      (lse != nullptr && !aligned16(lse)))
    return ATTN_ERR_MISALIGNED;
  const size_t q_bytes = static_cast<size_t>(B) * H * N_q * d * 2;
  const size_t kv_bytes = static_cast<size_t>(B) * H_kv * N_kv * d * 2;
  const size_t o_bytes = static_cast<size_t>(B) * H * N_q * d * ((dtype & ATTN_OUT_F32) ? 4 : 2);
  if (overlaps(o, o_bytes, q, q_bytes) || overlaps(o, o_bytes, k, kv_bytes) ||
      overlaps(o, o_bytes, v, kv_bytes))
    return ATTN_ERR_INVALID_ARG;
  return ATTN_OK;
}

// 3-D view [B*H_kv][N_kv][d] of the cache with 64 x 64 boxes, 128-byte swizzle.
int encode_cache_map(CUtensorMap* map, const void* base, bool bf16, int d, int n, int z) {
  const cuuint64_t dims[3] = {static_cast<cuuint64_t>(d), static_cast<cuuint64_t>(n),
                              static_cast<cuuint64_t>(z)};
  const cuuint64_t strides[2] = {static_cast<cuuint64_t>(d) * 2,
                                 static_cast<cuuint64_t>(n) * d * 2};
  const cuuint32_t box[3] = {64u, static_cast<cuuint32_t>(attn::DEC_T), 1u};
  const cuuint32_t estr[3] = {1u, 1u, 1u};
  const CUresult r = g_encode(map, bf16 ? CU_TENSOR_MAP_DATA_TYPE_BFLOAT16 : CU_TENSOR_MAP_DATA_TYPE_FLOAT16,
                              3, const_cast<void*>(base), dims, strides, box, estr,
                              CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                              CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS ? ATTN_OK : ATTN_ERR_CUDA;
}

template <int D, bool BF16, bool F32, int RW>
int launch_decode_rw(DeviceState* st, const attn::DecodeParams& dp, const CUtensorMap& mk,
                     const CUtensorMap& mv, cudaStream_t stream) {
  auto kern = attn::attn_decode_kernel<D, BF16, F32, RW>;
  const int smem = attn::DecGeo<D>::SMEM_BYTES + 1024;
  const int bit = (RW == 1 ? 0 : RW == 4 ? 8 : 16) + (D == 128 ? 4 : 0) + (BF16 ? 2 : 0) + (F32 ? 1 : 0);
  {
    std::lock_guard<std::mutex> lock(g_mu);
    if (!(st->dec_attr_set & (1u << bit))) {
      if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, smem) != cudaSuccess)
        return ATTN_ERR_CUDA;
      st->dec_attr_set |= 1u << bit;
    }
  }
  const dim3 grid(dp.n_splits, dp.B * dp.H_kv);
  kern<<<grid, attn::DEC_THREADS, smem, stream>>>(mk, mv, dp);
  g_launches.fetch_add(1, std::memory_order_relaxed);
  return cudaGetLastError() == cudaSuccess ? ATTN_OK : ATTN_ERR_CUDA;
}

template <int D, bool BF16, bool F32, int RMAX, int NW>
int launch_decode_small(DeviceState* st, const attn::DecodeParams& dp, const CUtensorMap& mk,
                        const CUtensorMap& mv, cudaStream_t stream) {
  auto kern = attn::attn_decode_small_kernel<D, BF16, F32, RMAX, NW>;
  const int smem = attn::DecSmallGeo<D, RMAX, NW>::SMEM_BYTES + 1024;
  const int bit = (RMAX == 4 ? 0 : 8) + (D == 128 ? 4 : 0) + (BF16 ? 2 : 0) + (F32 ? 1 : 0);
  {
    std::lock_guard<std::mutex> lock(g_mu);
    if (!(st->dec_small_attr_set & (1u << bit))) {
      if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, smem) != cudaSuccess)
        return ATTN_ERR_CUDA;
      st->dec_small_attr_set |= 1u << bit;
    }
  }
  const dim3 grid(dp.n_splits, dp.B * dp.H_kv);
  kern<<<grid, NW * 32, smem, stream>>>(mk, mv, dp);
  g_launches.fetch_add(1, std::memory_order_relaxed);
  return cudaGetLastError() == cudaSuccess ? ATTN_OK : ATTN_ERR_CUDA;
}

// Kernel by the group's query rows G * N_q: up to 4 and up to 16 rows use the
// warp-sliced kernel, larger groups (up to 64) the row-per-warp kernel.
template <int D, bool BF16, bool F32>
int launch_decode(DeviceState* st, const attn::DecodeParams& dp, const CUtensorMap& mk,
                  const CUtensorMap& mv, cudaStream_t stream) {
  const int rows = (dp.H / dp.H_kv) * dp.N_q;
  if (rows <= 4) return launch_decode_small<D, BF16, F32, 4, 8>(st, dp, mk, mv, stream);
  if (rows <= 16) return launch_decode_small<D, BF16, F32, 16, 4>(st, dp, mk, mv, stream);
  return launch_decode_rw<D, BF16, F32, 16>(st, dp, mk, mv, stream);
}

// Static decode scratch for attn_decode_noalloc: part of the module image on
// every device, so that entry point allocates nothing.  Its address is looked
// up once per device.
constexpr size_t kDecodeScratchBytes = size_t(4) << 20;
static __device__ __align__(256) unsigned char g_decode_scratch[kDecodeScratchBytes];

std::mutex g_scratch_mu;
void* g_scratch_addr[kMaxDevices] = {};

int decode_scratch(void** out) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return ATTN_ERR_CUDA;
  if (dev < 0 || dev >= kMaxDevices) return ATTN_ERR_UNSUPPORTED;
  std::lock_guard<std::mutex> lock(g_scratch_mu);
  if (g_scratch_addr[dev] == nullptr) {
    void* addr = nullptr;
    if (cudaGetSymbolAddress(&addr, g_decode_scratch) != cudaSuccess) return ATTN_ERR_CUDA;
    g_scratch_addr[dev] = addr;
  }
  *out = g_scratch_addr[dev];
  return ATTN_OK;
}

// attn_decode with an explicit workspace (base + size in bytes).
int decode_impl(const void* q, const void* k, const void* v, void* o, float* lse, void* ws,
                size_t ws_bytes, int B, int H, int H_kv, int N_q, int N_kv, int d, int causal,
                int window, int n_sink, float scale, int dtype, void* stream) {
  bool empty = false;
  int rc = validate_decode(q, k, v, o, lse, B, H, H_kv, N_q, N_kv, d, causal, window, n_sink,
                           scale, dtype, &empty);
  if (rc != ATTN_OK || empty) return rc;
  const DecodePlan pl = decode_plan(B, H, H_kv, N_q, N_kv, d);
  if (pl.n_splits > 1) {
    if (ws == nullptr || ws_bytes < pl.bytes) return ATTN_ERR_INVALID_ARG;
    if ((reinterpret_cast<uintptr_t>(ws) & 255u) != 0) return ATTN_ERR_MISALIGNED;
    const size_t o_bytes = static_cast<size_t>(B) * H * N_q * d * ((dtype & ATTN_OUT_F32) ? 4 : 2);
    const size_t q_bytes = static_cast<size_t>(B) * H * N_q * d * 2;
    const size_t kv_bytes = static_cast<size_t>(B) * H_kv * N_kv * d * 2;
    if (overlaps(ws, pl.bytes, o, o_bytes) || overlaps(ws, pl.bytes, q, q_bytes) ||
        overlaps(ws, pl.bytes, k, kv_bytes) || overlaps(ws, pl.bytes, v, kv_bytes) ||
        (lse != nullptr && overlaps(ws, pl.bytes, lse, static_cast<size_t>(B) * H * N_q * 4)))
      return ATTN_ERR_INVALID_ARG;
  }
  DeviceState* st = nullptr;
  rc = device_state(&st);
  if (rc != ATTN_OK) return rc;
  const bool bf16 = (dtype & 0xF) == ATTN_BF16;
  const bool f32 = (dtype & ATTN_OUT_F32) != 0;
  alignas(64) CUtensorMap mk, mv;
  if (encode_cache_map(&mk, k, bf16, d, N_kv, B * H_kv) != ATTN_OK ||
      encode_cache_map(&mv, v, bf16, d, N_kv, B * H_kv) != ATTN_OK)
    return ATTN_ERR_CUDA;
  attn::DecodeParams dp{};
  dp.q = q;
  dp.o = o;
  dp.lse = lse;
  uint8_t* w = static_cast<uint8_t*>(ws);
  dp.counters = pl.n_splits > 1 ? reinterpret_cast<int*>(w + pl.counters_off) : nullptr;
  dp.ws_lse = pl.n_splits > 1 ? reinterpret_cast<float*>(w + pl.lse_off) : nullptr;
  dp.ws_o = pl.n_splits > 1 ? reinterpret_cast<float*>(w + pl.o_off) : nullptr;
  dp.status = st->status;
  dp.watchdog_ns = g_watchdog_ns.load(std::memory_order_relaxed);
  dp.B = B;
  dp.H = H;
  dp.H_kv = H_kv;
  dp.N_q = N_q;
  dp.N_kv = N_kv;
  dp.causal = causal;
  dp.window = (window >= N_kv) ? 0 : window;
  dp.n_sink = dp.window > 0 ? (n_sink < N_kv ? n_sink : N_kv) : 0;
  dp.scale_log2 = scale * 1.4426950408889634f;
  dp.n_splits = pl.n_splits;
  dp.split_keys = pl.split_keys;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  // the per-group split counters start at zero on every call
  if (pl.n_splits > 1 &&
      cudaMemsetAsync(dp.counters, 0, static_cast<size_t>(B) * H_kv * sizeof(int), s) != cudaSuccess)
    return ATTN_ERR_CUDA;
  if (d == 128) {
    if (bf16) return f32 ? launch_decode<128, true, true>(st, dp, mk, mv, s) : launch_decode<128, true, false>(st, dp, mk, mv, s);
    return f32 ? launch_decode<128, false, true>(st, dp, mk, mv, s) : launch_decode<128, false, false>(st, dp, mk, mv, s);
  }
  if (bf16) return f32 ? launch_decode<64, true, true>(st, dp, mk, mv, s) : launch_decode<64, true, false>(st, dp, mk, mv, s);
  return f32 ? launch_decode<64, false, true>(st, dp, mk, mv, s) : launch_decode<64, false, false>(st, dp, mk, mv, s);
}

// ------------------------------------------------------------ backward

// Workspace of attn_bwd: D (one float per query row), then, unless the
// gradients are written in fp32, the fp32 dQ accumulator.
struct BwdPlan {
  size_t dq_off, bytes;
};

BwdPlan bwd_plan(int B, int H, int N, int d, bool out_f32) {
  BwdPlan pl{};
  const size_t rows = static_cast<size_t>(B) * H * N;
  pl.dq_off = round_up(rows * sizeof(float), 256);
  pl.bytes = out_f32 ? pl.dq_off : pl.dq_off + rows * d * sizeof(float);
  return pl;
}

// Pure argument validation for attn_bwd (no CUDA calls).
int validate_bwd(const void* q, const void* k, const void* v, const void* o, const void* dout,
                 const float* lse, const float* slopes, const void* dq, const void* dk,
                 const void* dv, const void* ws, size_t ws_bytes, int B, int H, int H_kv, int N,
                 int d, int causal, int window, int n_sink, float scale, int dtype, bool* empty) {
  Sizes sz;
  int rc = validate(q, k, v, dq, nullptr, B, H, H_kv, N, d, causal, window, n_sink, scale, dtype,
                    &sz, empty);
  if (rc != ATTN_OK || *empty) return rc;
  if (o == nullptr || dout == nullptr || lse == nullptr || dk == nullptr || dv == nullptr ||
      ws == nullptr)
    return ATTN_ERR_INVALID_ARG;
  if (!aligned16(o) || !aligned16(dout) || !aligned16(lse) || !aligned16(dk) || !aligned16(dv))
    return ATTN_ERR_MISALIGNED;
  if ((reinterpret_cast<uintptr_t>(ws) & 255u) != 0) return ATTN_ERR_MISALIGNED;
  if (slopes != nullptr && (reinterpret_cast<uintptr_t>(slopes) & 3u) != 0) return ATTN_ERR_MISALIGNED;
  const bool f32 = (dtype & ATTN_OUT_F32) != 0;
  const BwdPlan pl = bwd_plan(B, H, N, d, f32);
  if (ws_bytes < pl.bytes) return ATTN_ERR_INVALID_ARG;
  const size_t dq_bytes = sz.o_bytes;
  const size_t dkv_bytes = sz.kv_bytes / 2 * (f32 ? 4 : 2);
  // outputs and workspace: disjoint from each other and from every input
  struct Span { const void* p; size_t n; };
  const Span outs[4] = {{dq, dq_bytes}, {dk, dkv_bytes}, {dv, dkv_bytes}, {ws, pl.bytes}};
  const Span ins[7] = {{q, sz.q_bytes}, {k, sz.kv_bytes}, {v, sz.kv_bytes}, {o, sz.q_bytes},
                       {dout, sz.q_bytes}, {lse, sz.lse_bytes},
                       {slopes, slopes ? static_cast<size_t>(H) * sizeof(float) : 0}};
  for (int a = 0; a < 4; ++a) {
    for (int b = a + 1; b < 4; ++b)
      if (overlaps(outs[a].p, outs[a].n, outs[b].p, outs[b].n)) return ATTN_ERR_INVALID_ARG;
    for (int b = 0; b < 7; ++b)
      if (ins[b].p != nullptr && overlaps(outs[a].p, outs[a].n, ins[b].p, ins[b].n))
        return ATTN_ERR_INVALID_ARG;
  }
  return ATTN_OK;
}

// 3-D view [B*H][N][d] of the fp32 dQ buffer for the backward's bulk
// reductions: 32 x 32 boxes, 128-byte swizzle (d >= 64 only).
int encode_dq_map(CUtensorMap* map, void* base, int d, int n, int z) {
  const cuuint64_t dims[3] = {static_cast<cuuint64_t>(d), static_cast<cuuint64_t>(n),
                              static_cast<cuuint64_t>(z)};
  const cuuint64_t strides[2] = {static_cast<cuuint64_t>(d) * 4,
                                 static_cast<cuuint64_t>(n) * d * 4};
  const cuuint32_t box[3] = {32u, 32u, 1u};
  const cuuint32_t estr[3] = {1u, 1u, 1u};
  const CUresult r = g_encode(map, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 3, base, dims, strides, box,
                              estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                              CU_TENSOR_MAP_L2_PROMOTION_NONE, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS ? ATTN_OK : ATTN_ERR_CUDA;
}

template <int D, bool BF16, bool F32, bool ALIBI>
int launch_bwd_main(DeviceState* st, const CUtensorMap& mq, const CUtensorMap& mk,
                    const CUtensorMap& mv, const CUtensorMap& mdo, const CUtensorMap& mdq,
                    attn::BwdParams bp, cudaStream_t stream) {
  auto kern = attn::attn_bwd_kernel<D, BF16, F32, ALIBI>;
  const int need = attn::BwGeo<D>::SMEM_BYTES;
  // room for aligning the base to 1024 bytes where it fits; at least half of
  // the SM's shared memory so that two CTAs never share an SM (each allocates
  // all 512 TMEM columns)
  int smem = need + 1024 <= 232448 ? need + 1024 : 232448;
  if (smem < 120 * 1024) smem = 120 * 1024;
  const int dbit = D == 16 ? 0 : D == 32 ? 1 : D == 64 ? 2 : 3;
  const int bit = dbit * 8 + (ALIBI ? 4 : 0) + (BF16 ? 2 : 0) + (F32 ? 1 : 0);
  {
    std::lock_guard<std::mutex> lock(g_mu);
    if (!(st->bwd_attr_set & (1u << bit))) {
      // the kernel re-splits its registers after launch; that needs every
      // thread to start with BW_LAUNCH_REGS
      cudaFuncAttributes fa;
      if (cudaFuncGetAttributes(&fa, kern) != cudaSuccess) return ATTN_ERR_CUDA;
      if (fa.numRegs < attn::BW_LAUNCH_REGS) return ATTN_ERR_UNSUPPORTED;
      if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, smem) != cudaSuccess)
        return ATTN_ERR_CUDA;
      st->bwd_attr_set |= 1u << bit;
    }
  }
  bp.smem_alloc = smem;
  const int grid = bp.num_units < st->sm_count ? bp.num_units : st->sm_count;
  kern<<<grid, attn::BW_THREADS, smem, stream>>>(mq, mk, mv, mdo, mdq, bp);
  g_launches.fetch_add(1, std::memory_order_relaxed);
  return cudaGetLastError() == cudaSuccess ? ATTN_OK : ATTN_ERR_CUDA;
}

template <int D, bool BF16>
int launch_bwd_d(DeviceState* st, bool f32, bool alibi, const void* o, const void* dout,
                 void* dq, const CUtensorMap& mq, const CUtensorMap& mk, const CUtensorMap& mv,
                 const CUtensorMap& mdo, const CUtensorMap& mdq, attn::BwdParams bp,
                 long long rows, cudaStream_t s) {
  // 1. D = rowsum(dO * O); zero the fp32 dQ accumulator
  const long long blocks = (rows + 7) / 8;
  if (blocks > INT32_MAX) return ATTN_ERR_UNSUPPORTED;
  attn::attn_bwd_prep_kernel<D, BF16><<<static_cast<unsigned>(blocks), 256, 0, s>>>(
      o, dout, const_cast<float*>(bp.dsum), bp.dq_acc, rows);
  g_launches.fetch_add(1, std::memory_order_relaxed);
  if (cudaGetLastError() != cudaSuccess) return ATTN_ERR_CUDA;
  // 2. the tiled backward
  int rc;
  if (f32) rc = alibi ? launch_bwd_main<D, BF16, true, true>(st, mq, mk, mv, mdo, mdq, bp, s)
                      : launch_bwd_main<D, BF16, true, false>(st, mq, mk, mv, mdo, mdq, bp, s);
  else rc = alibi ? launch_bwd_main<D, BF16, false, true>(st, mq, mk, mv, mdo, mdq, bp, s)
                  : launch_bwd_main<D, BF16, false, false>(st, mq, mk, mv, mdo, mdq, bp, s);
  if (rc != ATTN_OK || f32) return rc;
  // 3. dQ to the 16-bit output
  const long long n4 = rows * D / 4;
  long long g = (n4 + 255) / 256;
  if (g > 8LL * st->sm_count) g = 8LL * st->sm_count;
  attn::attn_bwd_dq_convert_kernel<BF16><<<static_cast<unsigned>(g), 256, 0, s>>>(bp.dq_acc, dq, n4);
  g_launches.fetch_add(1, std::memory_order_relaxed);
  return cudaGetLastError() == cudaSuccess ? ATTN_OK : ATTN_ERR_CUDA;
}

int bwd_impl(const void* q, const void* k, const void* v, const void* o, const void* dout,
             const float* lse, const float* slopes, void* dq, void* dk, void* dv, void* ws,
             size_t ws_bytes, int B, int H, int H_kv, int N, int d, int causal, int window,
             int n_sink, float scale, int dtype, void* stream) {
  bool empty = false;
  int rc = validate_bwd(q, k, v, o, dout, lse, slopes, dq, dk, dv, ws, ws_bytes, B, H, H_kv, N, d,
                        causal, window, n_sink, scale, dtype, &empty);
  if (rc != ATTN_OK || empty) return rc;
  DeviceState* st = nullptr;
  rc = device_state(&st);
  if (rc != ATTN_OK) return rc;
  const bool bf16 = (dtype & 0xF) == ATTN_BF16;
  const bool f32 = (dtype & ATTN_OUT_F32) != 0;
  alignas(64) CUtensorMap mq, mk, mv, mdo;
  if (encode_map(&mq, q, bf16, d, N, B * H) != ATTN_OK ||
      encode_map(&mk, k, bf16, d, N, B * H_kv) != ATTN_OK ||
      encode_map(&mv, v, bf16, d, N, B * H_kv) != ATTN_OK ||
      encode_map(&mdo, dout, bf16, d, N, B * H) != ATTN_OK)
    return ATTN_ERR_CUDA;
  const BwdPlan pl = bwd_plan(B, H, N, d, f32);
  uint8_t* w = static_cast<uint8_t*>(ws);
  attn::BwdParams bp{};
  bp.lse = lse;
  bp.dsum = reinterpret_cast<float*>(w);
  bp.dq_acc = f32 ? static_cast<float*>(dq) : reinterpret_cast<float*>(w + pl.dq_off);
  alignas(64) CUtensorMap mdq;
  std::memset(&mdq, 0, sizeof(mdq));   // unused below d = 64 (atomics path)
  if (d >= 64 && encode_dq_map(&mdq, bp.dq_acc, d, N, B * H) != ATTN_OK) return ATTN_ERR_CUDA;
  bp.dk = dk;
  bp.dv = dv;
  bp.status = st->status;
  bp.watchdog_ns = g_watchdog_ns.load(std::memory_order_relaxed);
  bp.B = B;
  bp.H = H;
  bp.H_kv = H_kv;
  bp.N = N;
  bp.causal = causal;
  bp.window = (window >= N) ? 0 : window;
  bp.n_sink = bp.window > 0 ? (n_sink < N ? n_sink : N) : 0;
  bp.scale_log2 = scale * 1.4426950408889634f;
  bp.scale = scale;
  bp.n_tiles = (N + attn::BN - 1) / attn::BN;
  const long long units = static_cast<long long>(B) * H_kv * ((bp.n_tiles + 1) / 2);
  if (units > INT32_MAX) return ATTN_ERR_UNSUPPORTED;
  bp.num_units = static_cast<int>(units);
  bp.alibi = slopes;
  const long long rows = static_cast<long long>(B) * H * N;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  const bool al = slopes != nullptr;
  switch (d) {
    case 16: return bf16 ? launch_bwd_d<16, true>(st, f32, al, o, dout, dq, mq, mk, mv, mdo, mdq, bp, rows, s)
                         : launch_bwd_d<16, false>(st, f32, al, o, dout, dq, mq, mk, mv, mdo, mdq, bp, rows, s);
    case 32: return bf16 ? launch_bwd_d<32, true>(st, f32, al, o, dout, dq, mq, mk, mv, mdo, mdq, bp, rows, s)
                         : launch_bwd_d<32, false>(st, f32, al, o, dout, dq, mq, mk, mv, mdo, mdq, bp, rows, s);
    case 64: return bf16 ? launch_bwd_d<64, true>(st, f32, al, o, dout, dq, mq, mk, mv, mdo, mdq, bp, rows, s)
                         : launch_bwd_d<64, false>(st, f32, al, o, dout, dq, mq, mk, mv, mdo, mdq, bp, rows, s);
    case 128: return bf16 ? launch_bwd_d<128, true>(st, f32, al, o, dout, dq, mq, mk, mv, mdo, mdq, bp, rows, s)
                          : launch_bwd_d<128, false>(st, f32, al, o, dout, dq, mq, mk, mv, mdo, mdq, bp, rows, s);
    default: return ATTN_ERR_UNSUPPORTED;
  }
}

}  // namespace

extern "C" {

long long attn_decode_workspace_bytes(int B, int H, int H_kv, int N_q, int N_kv, int d) {
  if (B < 0 || H < 0 || H_kv < 1 || N_q < 0 || N_kv < 0 || d <= 0 || N_q > N_kv) return -1;
  if (B == 0 || H == 0 || N_q == 0) return 0;
  return static_cast<long long>(decode_plan(B, H, H_kv, N_q, N_kv, d).bytes);
}

int attn_decode_noalloc(const void* q, const void* k, const void* v, void* o, float* lse, int B,
                        int H, int H_kv, int N_q, int N_kv, int d, int causal, int window,
                        int n_sink, float scale, int dtype, void* stream) {
  bool empty = false;
  int rc = validate_decode(q, k, v, o, lse, B, H, H_kv, N_q, N_kv, d, causal, window, n_sink,
                           scale, dtype, &empty);
  if (rc != ATTN_OK || empty) return rc;
  if (decode_plan(B, H, H_kv, N_q, N_kv, d).bytes > kDecodeScratchBytes) return ATTN_ERR_UNSUPPORTED;
  void* scratch = nullptr;
  rc = decode_scratch(&scratch);
  if (rc != ATTN_OK) return rc;
  return decode_impl(q, k, v, o, lse, scratch, kDecodeScratchBytes, B, H, H_kv, N_q, N_kv, d,
                     causal, window, n_sink, scale, dtype, stream);
}

int attn_decode(const void* q, const void* k, const void* v, void* o, float* lse, void* workspace,
                long long workspace_bytes, int B, int H, int H_kv, int N_q, int N_kv, int d,
                int causal, int window, int n_sink, float scale, int dtype, void* stream) {
  if (workspace_bytes < 0) return ATTN_ERR_INVALID_ARG;
  return decode_impl(q, k, v, o, lse, workspace, static_cast<size_t>(workspace_bytes), B, H, H_kv,
                     N_q, N_kv, d, causal, window, n_sink, scale, dtype, stream);
}


long long attn_bwd_workspace_bytes(int B, int H, int N, int d, int dtype) {
  if (B < 0 || H < 0 || N < 0 || d <= 0) return -1;
  if ((dtype & ~(ATTN_OUT_F32 | 0xF)) != 0) return -1;
  if (B == 0 || H == 0 || N == 0) return 0;
  return static_cast<long long>(bwd_plan(B, H, N, d, (dtype & ATTN_OUT_F32) != 0).bytes);
}

int attn_bwd(const void* q, const void* k, const void* v, const void* o, const void* dout,
             const float* lse, const float* slopes, void* dq, void* dk, void* dv,
             void* workspace, long long workspace_bytes, int B, int H, int H_kv, int N, int d,
             int causal, int window, int n_sink, float scale, int dtype, void* stream) {
  if (workspace_bytes < 0) return ATTN_ERR_INVALID_ARG;
  return bwd_impl(q, k, v, o, dout, lse, slopes, dq, dk, dv, workspace,
                  static_cast<size_t>(workspace_bytes), B, H, H_kv, N, d, causal, window, n_sink,
                  scale, dtype, stream);
}


int attn_fwd(const void* q, const void* k, const void* v, void* o, float* lse, int B, int H,
             int H_kv, int N, int d, int causal, int window, int n_sink, float scale, int dtype,
             void* stream) {
  return fwd_impl(q, k, v, o, lse, nullptr, B, H, H_kv, N, d, causal, window, n_sink, scale,
                  dtype, stream);
}

int attn_fwd_alibi(const void* q, const void* k, const void* v, void* o, float* lse,
                   const float* slopes, int B, int H, int H_kv, int N, int d, int causal,
                   int window, int n_sink, float scale, int dtype, void* stream) {
  Sizes sz;
  bool empty = false;
  const int rc = validate(q, k, v, o, lse, B, H, H_kv, N, d, causal, window, n_sink, scale, dtype,
                          &sz, &empty);
  if (rc != ATTN_OK || empty) return rc;
  if (slopes == nullptr) return ATTN_ERR_INVALID_ARG;
  if ((reinterpret_cast<uintptr_t>(slopes) & 3u) != 0) return ATTN_ERR_MISALIGNED;
  if (overlaps(slopes, static_cast<size_t>(H) * sizeof(float), o, sz.o_bytes) ||
      (lse != nullptr && overlaps(slopes, static_cast<size_t>(H) * sizeof(float), lse, sz.lse_bytes)))
    return ATTN_ERR_INVALID_ARG;
  return fwd_impl(q, k, v, o, lse, slopes, B, H, H_kv, N, d, causal, window, n_sink, scale, dtype,
                  stream);
}

int attn_alibi_slopes(int H, float* slopes) {
  if (H < 1 || slopes == nullptr) return ATTN_ERR_INVALID_ARG;
  for (int h = 1; h <= H; ++h)
    slopes[h - 1] = static_cast<float>(std::exp2(-8.0 * h / H));
  return ATTN_OK;
}

int attn_fwd_host(const void* q, const void* k, const void* v, void* o, float* lse, void* dq,
                  void* dk, void* dv, void* dout, float* dlse, int B, int H, int H_kv, int N,
                  int d, int causal, int window, int n_sink, float scale, int dtype,
                  void* stream) {
  Sizes sz;
  bool empty = false;
  int rc = validate(dq, dk, dv, dout, dlse, B, H, H_kv, N, d, causal, window, n_sink, scale, dtype,
                    &sz, &empty);
  if (rc != ATTN_OK || empty) return rc;
  if (q == nullptr || k == nullptr || v == nullptr || o == nullptr) return ATTN_ERR_INVALID_ARG;
  if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(o) ||
      (lse != nullptr && !aligned16(lse)))
    return ATTN_ERR_MISALIGNED;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  if (cudaMemcpyAsync(dq, q, sz.q_bytes, cudaMemcpyHostToDevice, s) != cudaSuccess ||
      cudaMemcpyAsync(dk, k, sz.kv_bytes, cudaMemcpyHostToDevice, s) != cudaSuccess ||
      cudaMemcpyAsync(dv, v, sz.kv_bytes, cudaMemcpyHostToDevice, s) != cudaSuccess)
    return ATTN_ERR_CUDA;
  rc = attn_fwd(dq, dk, dv, dout, dlse, B, H, H_kv, N, d, causal, window, n_sink, scale, dtype,
                stream);
  if (rc != ATTN_OK) return rc;
  if (cudaMemcpyAsync(o, dout, sz.o_bytes, cudaMemcpyDeviceToHost, s) != cudaSuccess)
    return ATTN_ERR_CUDA;
  if (lse != nullptr && dlse != nullptr &&
      cudaMemcpyAsync(lse, dlse, sz.lse_bytes, cudaMemcpyDeviceToHost, s) != cudaSuccess)
    return ATTN_ERR_CUDA;
  return ATTN_OK;
}

const char* attn_error_string(int status) {
  switch (status) {
    case ATTN_OK: return "ok";
    case ATTN_ERR_INVALID_ARG: return "invalid argument";
    case ATTN_ERR_UNSUPPORTED: return "unsupported configuration or device";
    case ATTN_ERR_MISALIGNED: return "tensor pointer not 16-byte aligned";
    case ATTN_ERR_CUDA: return "CUDA runtime or driver error";
    case ATTN_ERR_DEVICE_TIMEOUT: return "kernel wait exceeded the watchdog limit";
    default: return "unknown status";
  }
}

long long attn_unmasked_pairs(int N, int causal, int window, int n_sink) {
  if (N < 0 || window < 0 || n_sink < 0 || (causal != 0 && causal != 1)) return -1;
  if (window > 0 && !causal) return -1;
  const long long n = N;
  if (!causal) return n * n;
  if (window == 0 || window >= N) return n * (n + 1) / 2;
  // Row i keeps min(i+1, W) window keys plus the sinks left of its window:
  // max(0, min(S, i - W + 1)).
  const long long W = window, S = n_sink;
  long long total = 0;
  // window part: rows 0..W-1 keep i+1, rows W..N-1 keep W
  total += W * (W + 1) / 2 + (n - W) * W;
  // sink part: rows i >= W contribute min(S, i - W + 1)
  const long long rows = n - W;                   // i - W + 1 runs over 1..rows
  const long long full = rows > S ? rows - S : 0; // rows where the count is S
  const long long ramp = rows - full;             // counts 1..ramp
  total += ramp * (ramp + 1) / 2 + full * S;
  return total;
}

long long attn_visited_blocks(int N, int causal, int window, int n_sink) {
  if (N < 0 || window < 0 || n_sink < 0 || (causal != 0 && causal != 1)) return -1;
  if (window > 0 && !causal) return -1;
  if (N == 0) return 0;
  const int W = (window >= N) ? 0 : window;
  const int S = W > 0 ? (n_sink < N ? n_sink : N) : 0;
  const int nkb = (N + attn::BN - 1) / attn::BN;
  const int sink_blocks = W > 0 ? (S + attn::BN - 1) / attn::BN : 0;
  long long total = 0;
  for (int r0 = 0; r0 < N; r0 += attn::BM) {
    const int r_last = (r0 + attn::BM - 1 < N - 1) ? r0 + attn::BM - 1 : N - 1;
    int lo = 0, hi = nkb;
    if (causal) hi = (r_last / attn::BN + 1 < nkb) ? r_last / attn::BN + 1 : nkb;
    if (W > 0) {
      const int k_min = r0 - W + 1;
      lo = k_min > 0 ? k_min / attn::BN : 0;
    }
    const int tsb = sink_blocks < hi ? sink_blocks : hi;
    const int win_start = lo > tsb ? lo : tsb;
    total += tsb + (hi > win_start ? hi - win_start : 0);
  }
  return total;
}

int attn_get_status(void) {
  DeviceState* st = nullptr;
  int rc = device_state(&st);
  if (rc != ATTN_OK) return rc;
  if (cudaDeviceSynchronize() != cudaSuccess) return ATTN_ERR_CUDA;
  int value = 0;
  const int zero = 0;
  if (cudaMemcpy(&value, st->status, sizeof(int), cudaMemcpyDeviceToHost) != cudaSuccess ||
      cudaMemcpy(st->status, &zero, sizeof(int), cudaMemcpyHostToDevice) != cudaSuccess)
    return ATTN_ERR_CUDA;
  return value;
}

unsigned long long attn_set_watchdog_ns(unsigned long long ns) {
  if (ns < 1000000ull) ns = 1000000ull;
  if (ns > 60000000000ull) ns = 60000000000ull;
  return g_watchdog_ns.exchange(ns);
}

int attn_test_withhold_loads(int n_launches) {
  if (n_launches < 0) return ATTN_ERR_INVALID_ARG;
  g_withhold.store(n_launches);
  return ATTN_OK;
}

unsigned long long attn_launch_count(void) { return g_launches.load(std::memory_order_relaxed); }

}  // extern "C"

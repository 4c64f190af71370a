// decode_api.cu -- the split-KV decoding step: attn_decode, its workspace
// query and attn_decode_noalloc.
#include "host.h"
#include "decode_kernel.cuh"

namespace attn_host {

namespace {

// ------------------------------------------------------------ decode

// Split rule (device independent, so that the workspace size can be queried
// without a device): at most two CTAs per SM of a 148-SM part in total (one
// wave; rounding the split count up would leave a short second wave), each
// split at least 256 keys long and a whole number of 64-key tiles.
struct DecodePlan {
  int n_splits, split_keys;
  size_t counters_off, lse_off, o_off, bytes;
};

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
  dp.withhold_loads = take_withhold();
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


}  // namespace

}  // namespace attn_host

using namespace attn_host;

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

}  // extern "C"

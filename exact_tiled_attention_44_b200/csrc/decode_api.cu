// decode_api.cu -- the split-KV decoding step: attn_decode, its workspace
// query and attn_decode_noalloc.
#include "host.h"
#include "decode_tc_kernel.cuh"

namespace attn_host {

namespace {

// ------------------------------------------------------------ decode

// Workspace of attn_decode (device independent, so that its size can be
// queried without a device, and independent of the mask): the kernel cuts
// the kept 128-key tiles of all (batch, K/V head) groups into at most
// DT_GRID equal ranges, so a group spans at most ceil(DT_GRID / groups) + 1
// of them, each writing one partial result per query row.
struct DecodePlan {
  int max_parts;
  size_t lse_off, o_off, bytes;
};

DecodePlan decode_plan(int B, int H, int H_kv, int N_q, int N_kv, int d) {
  (void)N_kv;
  DecodePlan pl{};
  const long long groups = static_cast<long long>(B) * H_kv;
  const long long R = static_cast<long long>(H / H_kv) * N_q;
  pl.max_parts = static_cast<int>((attn::DT_GRID + groups - 1) / groups + 1);
  const size_t rows = static_cast<size_t>(groups) * pl.max_parts * R;
  pl.lse_off = 0;
  pl.o_off = round_up(rows * sizeof(float), 256);
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
  if (static_cast<long long>(H / H_kv) * N_q > attn::DT_MAX_ROWS) return ATTN_ERR_UNSUPPORTED;
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

template <int D, bool BF16, bool F32>
int launch_decode(DeviceState* st, const attn::DecTcParams& dp, const CUtensorMap& mk,
                  const CUtensorMap& mv, bool merge, cudaStream_t stream) {
  auto kern = attn::attn_decode_tc_kernel<D, BF16, F32>;
  const int smem = attn::DtGeo<D>::SMEM_BYTES + 1024;
  const int bit = (D == 128 ? 4 : 0) + (BF16 ? 2 : 0) + (F32 ? 1 : 0);
  {
    std::lock_guard<std::mutex> lock(g_mu);
    if (!(st->dec_attr_set & (1u << bit))) {
      // the kernel re-splits its registers after launch (as the forward does)
      cudaFuncAttributes fa;
      if (cudaFuncGetAttributes(&fa, kern) != cudaSuccess) return ATTN_ERR_CUDA;
      if (fa.numRegs < attn::LAUNCH_REGS) return ATTN_ERR_UNSUPPORTED;
      if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, smem) != cudaSuccess)
        return ATTN_ERR_CUDA;
      st->dec_attr_set |= 1u << bit;
    }
  }
  cudaError_t e = launch_overlapped(kern, dp.grid, attn::NUM_THREADS, smem, stream, mk, mv, dp);
  g_launches.fetch_add(1, std::memory_order_relaxed);
  if (e != cudaSuccess || cudaGetLastError() != cudaSuccess) return ATTN_ERR_CUDA;
  if (!merge) return ATTN_OK;
  e = launch_overlapped(attn::attn_decode_tc_merge<D, BF16, F32>, dp.n_groups, 256, 0, stream, dp);
  g_launches.fetch_add(1, std::memory_order_relaxed);
  return e == cudaSuccess && cudaGetLastError() == cudaSuccess ? ATTN_OK : ATTN_ERR_CUDA;
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
  attn::DecTcParams dp{};
  dp.B = B;
  dp.H = H;
  dp.H_kv = H_kv;
  dp.N_q = N_q;
  dp.N_kv = N_kv;
  dp.causal = causal;
  dp.window = (window >= N_kv) ? 0 : window;
  dp.n_sink = dp.window > 0 ? (n_sink < N_kv ? n_sink : N_kv) : 0;
  dp.scale_log2 = scale * 1.4426950408889634f;
  dp.R = (H / H_kv) * N_q;
  dp.n_groups = B * H_kv;
  // kept 128-key tiles of every group: the sink tiles, then the tiles from the
  // first query row's window start to the end of the cache
  dp.nt = (N_kv + attn::DT_TILE - 1) / attn::DT_TILE;
  if (dp.window > 0) {
    const int first = N_kv - N_q - dp.window + 1;
    dp.wlo = first > 0 ? first / attn::DT_TILE : 0;
    const int sb = (dp.n_sink + attn::DT_TILE - 1) / attn::DT_TILE;
    dp.sb = sb < dp.nt ? sb : dp.nt;
  } else {
    dp.wlo = 0;
    dp.sb = 0;
  }
  const int w0 = dp.wlo > dp.sb ? dp.wlo : dp.sb;
  dp.tiles = dp.sb + (dp.nt > w0 ? dp.nt - w0 : 0);
  const long long F = static_cast<long long>(dp.n_groups) * dp.tiles;
  dp.grid = static_cast<int>(F < attn::DT_GRID ? F : attn::DT_GRID);
  dp.max_parts = pl.max_parts;
  // does any group span more than one range?
  bool merge = false;
  for (int g = 0; g < dp.n_groups && !merge; ++g)
    merge = attn::dt_cta_of(static_cast<long long>(g) * dp.tiles, F, dp.grid) !=
            attn::dt_cta_of(static_cast<long long>(g + 1) * dp.tiles - 1, F, dp.grid);
  if (merge) {
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
  if (encode_map(&mk, k, bf16, d, N_kv, B * H_kv) != ATTN_OK ||
      encode_map(&mv, v, bf16, d, N_kv, B * H_kv) != ATTN_OK)
    return ATTN_ERR_CUDA;
  dp.q = q;
  dp.o = o;
  dp.lse = lse;
  uint8_t* w = static_cast<uint8_t*>(ws);
  dp.ws_lse = merge ? reinterpret_cast<float*>(w + pl.lse_off) : nullptr;
  dp.ws_o = merge ? reinterpret_cast<float*>(w + pl.o_off) : nullptr;
  dp.status = st->status;
  dp.watchdog_ns = g_watchdog_ns.load(std::memory_order_relaxed);
  dp.withhold_loads = take_withhold();
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  if (d == 128) {
    if (bf16) return f32 ? launch_decode<128, true, true>(st, dp, mk, mv, merge, s)
                         : launch_decode<128, true, false>(st, dp, mk, mv, merge, s);
    return f32 ? launch_decode<128, false, true>(st, dp, mk, mv, merge, s)
               : launch_decode<128, false, false>(st, dp, mk, mv, merge, s);
  }
  if (bf16) return f32 ? launch_decode<64, true, true>(st, dp, mk, mv, merge, s)
                       : launch_decode<64, true, false>(st, dp, mk, mv, merge, s);
  return f32 ? launch_decode<64, false, true>(st, dp, mk, mv, merge, s)
             : launch_decode<64, false, false>(st, dp, mk, mv, merge, s);
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

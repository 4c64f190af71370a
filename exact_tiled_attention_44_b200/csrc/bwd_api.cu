// bwd_api.cu -- the backward's launches: attn_bwd and its workspace query.
#include <cstring>

#include "host.h"
#include "bwd_kernel.cuh"

namespace attn_host {

namespace {

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
  bp.withhold_loads = take_withhold();
  bp.block_count = g_block_count.load();
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

}  // namespace attn_host

using namespace attn_host;

extern "C" {

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

}  // extern "C"

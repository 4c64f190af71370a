// fwd_api.cu -- the forward's entry points attn_fwd and attn_fwd_alibi, and
// the head dims 16, 32 and 64 (d = 128 is in fwd_d128.cu).
#include "fwd_launch.cuh"

namespace attn_host {

int fwd_unit_kind(int B, int H, int H_kv, int N, int window, bool alibi, int sm_count) {
  if (alibi) return attn::UK_PAIR;
  const long long bh = static_cast<long long>(B) * H;
  const long long pairs = bh * ((N + 2 * attn::BM - 1) / (2 * attn::BM));
  const long long tiles = bh * ((N + attn::BM - 1) / attn::BM);
  if (pairs < sm_count && tiles <= 2LL * sm_count) return attn::UK_SPLIT;
  // Query heads sharing a K/V head: when a row sees at most 4096 keys (a
  // window, or a short sequence), a pair of consecutive Q tiles iterates the
  // union of two key ranges one block apart, a visible share of short units;
  // two heads at the same rows visit exactly the same blocks (measured on
  // B200: MQA with a 1024 window +7%, G = 4 at N = 4096 +1.5%; G = 8 causal at
  // N = 16384 -1.5%, where pairs finish tile 0 a block early).
  const int span = (window > 0 && window < N) ? window : N;
  if (H / H_kv >= 2 && span <= 4096) return attn::UK_HEADS;
  return attn::UK_PAIR;
}

int fwd_impl(const void* q, const void* k, const void* v, void* o, float* lse,
             const float* slopes, int B, int H, int H_kv, int N, int d, int causal, int window,
             int n_sink, float scale, int dtype, void* stream, int uk) {
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
  alignas(64) CUtensorMap mq, mk, mv, mo;
  if (encode_map(&mq, q, bf16, d, N, B * H) != ATTN_OK ||
      encode_map(&mk, k, bf16, d, N, B * H_kv) != ATTN_OK ||
      encode_map(&mv, v, bf16, d, N, B * H_kv) != ATTN_OK)
    return ATTN_ERR_CUDA;
  // the output's map (16-bit outputs are written by TMA stores; an fp32
  // output is stored from registers and the map is not read)
  if (f32)
    mo = mq;
  else if (encode_map(&mo, o, bf16, d, N, B * H) != ATTN_OK)
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
  if (uk < 0) uk = g_force_units.load();
  if (uk < 0) uk = fwd_unit_kind(B, H, H_kv, N, window, false, st->sm_count);
  if (slopes != nullptr) uk = attn::UK_PAIR;
  kp.n_qpairs = (N + 2 * attn::BM - 1) / (2 * attn::BM);
  kp.n_qtiles = (N + attn::BM - 1) / attn::BM;
  kp.n_kblocks = (N + attn::BN - 1) / attn::BN;
  kp.n_hpairs = (H / H_kv + 1) / 2;
  kp.num_units = uk == attn::UK_SPLIT   ? B * H * kp.n_qtiles
                 : uk == attn::UK_HEADS ? B * H_kv * kp.n_hpairs * kp.n_qtiles
                                        : B * H * kp.n_qpairs;
  kp.alibi = slopes;
  kp.withhold_loads = take_withhold();
  kp.block_count = g_block_count.load();

  cudaStream_t s = static_cast<cudaStream_t>(stream);
  switch (d) {
    case 16: return launch_d<16>(st, bf16, f32, uk, mq, mk, mv, mo, kp, s);
    case 32: return launch_d<32>(st, bf16, f32, uk, mq, mk, mv, mo, kp, s);
    case 64: return launch_d<64>(st, bf16, f32, uk, mq, mk, mv, mo, kp, s);
    case 128: return launch_fwd_d128(st, bf16, f32, uk, mq, mk, mv, mo, kp, s);
    default: return ATTN_ERR_UNSUPPORTED;
  }
}

}  // namespace attn_host

using namespace attn_host;

extern "C" {

int attn_fwd_unit_kind(int B, int H, int H_kv, int N, int window, int alibi, int sm_count) {
  if (B < 0 || H < 1 || H_kv < 1 || H % H_kv != 0 || N < 0 || window < 0 || sm_count < 0)
    return ATTN_ERR_INVALID_ARG;
  if (sm_count == 0) {
    DeviceState* st = nullptr;
    const int rc = device_state(&st);
    if (rc != ATTN_OK) return rc;
    sm_count = st->sm_count;
  }
  return fwd_unit_kind(B, H, H_kv, N, window, alibi != 0, sm_count);
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

}  // extern "C"

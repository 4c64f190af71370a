// decode_kernel.cuh -- split-KV attention of a few new query rows against a
// K/V cache, for sm_100a.
//
// What it computes (per batch b, query head h, kv head g = h / (H / H_kv)):
// the N_q new query rows of the head sit at cache positions N_kv - N_q + i
// ("USAAIO Lesson 91", slide 31: every decoding step re-reads the whole K/V
// cache; slide 32: query heads share K/V heads), and attend to the cache under
// the mask rule of the forward with that position as the query index.
//
// The K/V range is split across CTAs ("Building a FlashAttention-style tiled
// self-attention block in pure NumPy", "Extending It", item 6: split the
// sequence, each worker handling a subset of tiles, then reduce the partial
// outputs).  Each CTA owns one (b, g, split): all G * N_q query rows of the
// kv head's group read each K/V tile once.  A split writes its partial
// (O_s normalised over its own keys, LSE_s) to the caller's workspace; the
// last CTA of a (b, g) to finish, found with a per-group counter, merges the
// splits in split order:
//     LSE = ln sum_s exp(LSE_s),   O = sum_s exp(LSE_s - LSE) O_s.
// The merge order does not depend on which CTA finishes last, so results are
// deterministic.
//
// The work is bound by HBM (the cache bytes; about 2 * G * N_q flops per byte
// for 16-bit K/V), so the arithmetic runs on the FP32 pipes: K and V tiles of
// 64 keys arrive by TMA in the 128-byte swizzle (which makes the lane-per-key
// shared-memory reads conflict-free), S and P V are FFMA loops, the row max is
// a warp shuffle reduction, and the online softmax keeps the lazy rescale of
// the forward.
#pragma once

#include "attn_kernel.cuh"

namespace attn {

constexpr int DEC_T = 64;            // keys per K/V tile
constexpr int DEC_WARPS = 4;
constexpr int DEC_THREADS = 32 * DEC_WARPS;
constexpr int DEC_MAX_ROWS = 64;     // query rows of one (b, g): G * N_q
// Row capacity per warp is a template parameter RW (1, 4 or 16) chosen from
// G * N_q, so that small groups do not carry the register arrays of large ones.

struct DecodeParams {
  const void* q;
  void* o;
  float* lse;
  float* ws_o;        // [n_splits][B][H][N_q][D] partial outputs (n_splits > 1)
  float* ws_lse;      // [n_splits][B][H][N_q] partial LSE, natural log (n_splits > 1)
  int* counters;      // [B][H_kv] finished splits per group, zero at launch
  int* status;
  unsigned long long watchdog_ns;
  int B, H, H_kv, N_q, N_kv;
  int causal, window, n_sink;
  float scale_log2;   // scale * log2(e)
  int n_splits;       // split s covers keys [s * split_keys, min(N_kv, (s + 1) * split_keys))
  int split_keys;     // a multiple of DEC_T
  int withhold_loads; // test hook: no tile is loaded, so every wait on a tile runs out
};

template <int D>
struct DecGeo {
  static_assert(D == 64 || D == 128, "decode supports d = 64 and 128");
  static constexpr int NBOX = D / 64;                 // 64-column boxes per tile
  static constexpr int BOX_BYTES = DEC_T * 128;       // 64 rows x 128 bytes
  static constexpr int TILE_BYTES = NBOX * BOX_BYTES;
  static constexpr int Q_OFF = 0;                     // fp32 [DEC_MAX_ROWS][D], pre-scaled
  static constexpr int K_OFF = DEC_MAX_ROWS * D * 4;  // two K stages
  static constexpr int V_OFF = K_OFF + 2 * TILE_BYTES;  // two V stages
  static constexpr int BAR_OFF = V_OFF + 2 * TILE_BYTES;
  static constexpr int SMEM_BYTES = BAR_OFF + 64;
  static_assert(K_OFF % 1024 == 0 && TILE_BYTES % 1024 == 0, "swizzle atoms need 1 KB alignment");
};

// barrier slots: FULL[2], EMPTY[2]; then the abort flag and the last-CTA flag
enum DecBar : int { DB_FULL = 0, DB_EMPTY = 2, DB_COUNT = 4 };

// Keys [j0, j0 + DEC_T) hold a kept key for some query row of the group.
__device__ __forceinline__ bool dec_tile_kept(const DecodeParams& p, int j0) {
  if (p.window == 0) return true;
  const int pos_min = p.N_kv - p.N_q;
  return j0 < p.n_sink || j0 + DEC_T - 1 >= pos_min - p.window + 1;
}

// Next kept tile start at or after j in [.., hi); returns hi when none.
__device__ __forceinline__ int dec_next_tile(const DecodeParams& p, int j, int hi) {
  while (j < hi && !dec_tile_kept(p, j)) j += DEC_T;
  return j < hi ? j : hi;
}

// Byte offset of 16-byte chunk c (0..7) of row t inside a 128-byte-swizzled box.
__device__ __forceinline__ uint32_t sw128(int t, int c) {
  return static_cast<uint32_t>(t * 128 + ((c ^ (t & 7)) << 4));
}

template <bool BF16>
__device__ __forceinline__ float2 unpack2f(uint32_t w) {
  if constexpr (BF16) {
    return make_float2(__uint_as_float(w << 16), __uint_as_float(w & 0xFFFF0000u));
  } else {
    __half2 h = *reinterpret_cast<__half2*>(&w);
    return __half22float2(h);
  }
}

__device__ __forceinline__ float warp_max(float x) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) x = fmaxf(x, __shfl_xor_sync(0xffffffffu, x, o));
  return x;
}

__device__ __forceinline__ float warp_sum(float x) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) x += __shfl_xor_sync(0xffffffffu, x, o);
  return x;
}

template <int D, bool BF16, bool OUT_F32, int RW>
__global__ void __launch_bounds__(DEC_THREADS, 1)
attn_decode_kernel(const __grid_constant__ CUtensorMap tmK, const __grid_constant__ CUtensorMap tmV,
                   const DecodeParams p) {
  using G = DecGeo<D>;
  constexpr int CPL = D / 32;            // O columns per lane
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~static_cast<uintptr_t>(1023));
  const uint32_t sbase = smem_addr(smem);
  const uint32_t bars = sbase + G::BAR_OFF;
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + G::BAR_OFF + 8 * DB_COUNT);
  volatile int* last_flag = abort_flag + 1;
  float* qs = reinterpret_cast<float*>(smem + G::Q_OFF);

  const int warp = threadIdx.x / 32;
  const int lane = threadIdx.x % 32;
  const int split = blockIdx.x;
  const int bg = blockIdx.y;                  // b * H_kv + g
  const int b = bg / p.H_kv, g = bg % p.H_kv;
  const int G_heads = p.H / p.H_kv;
  const int R = G_heads * p.N_q;              // query rows of this group (<= DEC_MAX_ROWS)
  const int lo = split * p.split_keys;
  const int hi = min(p.N_kv, lo + p.split_keys);

  if (threadIdx.x == 0) {
    for (int s = 0; s < 2; ++s) {
      mbar_init(bars + 8 * (DB_FULL + s), 1);
      mbar_init(bars + 8 * (DB_EMPTY + s), DEC_WARPS);
    }
    *abort_flag = 0;
    *last_flag = 0;
    fence_barrier_init();
    tma_prefetch_desc(&tmK);
    tma_prefetch_desc(&tmV);
  }
  // Query rows of the group, fp32 and pre-scaled into log2 units.  Row r is
  // query head g * G + r / N_q, query i = r % N_q.
  for (int e = threadIdx.x; e < R * (D / 2); e += DEC_THREADS) {
    const int r = e / (D / 2), c2 = e % (D / 2);
    const int h = g * G_heads + r / p.N_q, i = r % p.N_q;
    const size_t off = ((static_cast<size_t>(b) * p.H + h) * p.N_q + i) * D + 2 * c2;
    const uint32_t w = *reinterpret_cast<const uint32_t*>(static_cast<const uint16_t*>(p.q) + off);
    const float2 f = unpack2f<BF16>(w);
    qs[r * D + 2 * c2] = f.x * p.scale_log2;
    qs[r * D + 2 * c2 + 1] = f.y * p.scale_log2;
  }
  __syncthreads();

  // ---- tile pipeline: warp 0 (one elected lane) loads tile n+1 while all
  // warps work on tile n; a stage is reused once every warp has released it.
  const int j_first = dec_next_tile(p, lo, hi);
  bool ok = true;
  int issued_last[2] = {-1, -1};        // parity of the last load into each stage (warp 0)
  auto issue = [&](int j0, int n) {
    // failure-detection test: nothing is loaded (and nothing is left to drain)
    if (p.withhold_loads) return true;
    const int st = n & 1;
    const uint32_t ph = (static_cast<uint32_t>(n) >> 1) & 1u;
    if (!mbar_try_wait(bars + 8 * (DB_EMPTY + st), ph ^ 1u) &&
        !wait_slow(bars + 8 * (DB_EMPTY + st), ph ^ 1u, abort_flag, p.status, p.watchdog_ns))
      return false;
    if (elect_one()) {
      mbar_arrive_expect_tx(bars + 8 * (DB_FULL + st), 2 * G::TILE_BYTES);
      for (int c = 0; c < G::NBOX; ++c) {
        tma_load_3d(sbase + G::K_OFF + st * G::TILE_BYTES + c * G::BOX_BYTES, &tmK,
                    bars + 8 * (DB_FULL + st), c * 64, j0, bg);
        tma_load_3d(sbase + G::V_OFF + st * G::TILE_BYTES + c * G::BOX_BYTES, &tmV,
                    bars + 8 * (DB_FULL + st), c * 64, j0, bg);
      }
    }
    __syncwarp();
    issued_last[st] = static_cast<int>(ph);
    return true;
  };
  if (warp == 0 && j_first < hi) ok = __all_sync(0xffffffffu, issue(j_first, 0));

  // per-row state of this warp's rows r = warp + 4 rr
  const int nr = (R > warp) ? (R - warp + DEC_WARPS - 1) / DEC_WARPS : 0;
  float m[RW], l[RW], acc[RW][CPL];
#pragma unroll
  for (int rr = 0; rr < RW; ++rr) {
    m[rr] = -INFINITY;
    l[rr] = 0.f;
#pragma unroll
    for (int c = 0; c < CPL; ++c) acc[rr][c] = 0.f;
  }

  int n = 0;
  for (int j0 = j_first; j0 < hi && ok; j0 = dec_next_tile(p, j0 + DEC_T, hi), ++n) {
    const int st = n & 1;
    if (warp == 0) {
      const int jn = dec_next_tile(p, j0 + DEC_T, hi);
      if (jn < hi) ok = __all_sync(0xffffffffu, issue(jn, n + 1));
      if (!ok) break;
    }
    {
      const uint32_t full = bars + 8 * (DB_FULL + st), ph = (static_cast<uint32_t>(n) >> 1) & 1u;
      ok = __all_sync(0xffffffffu, mbar_try_wait(full, ph) ||
                                       wait_slow(full, ph, abort_flag, p.status, p.watchdog_ns));
    }
    if (!ok) break;
    const uint32_t ks = sbase + G::K_OFF + st * G::TILE_BYTES;
    const uint32_t vs = sbase + G::V_OFF + st * G::TILE_BYTES;
    const int j_end = min(j0 + DEC_T, hi);

    // S for keys j0 + lane and j0 + 32 + lane, every row of this warp
    float s0[RW], s1[RW];
#pragma unroll
    for (int rr = 0; rr < RW; ++rr) s0[rr] = s1[rr] = 0.f;
#pragma unroll 2
    for (int c8 = 0; c8 < D / 8; ++c8) {
      const uint32_t box = static_cast<uint32_t>((c8 / 8) * G::BOX_BYTES);
      uint32_t ka[4], kb[4];
      asm volatile("ld.shared.v4.b32 {%0, %1, %2, %3}, [%4];"
                   : "=r"(ka[0]), "=r"(ka[1]), "=r"(ka[2]), "=r"(ka[3])
                   : "r"(ks + box + sw128(lane, c8 % 8)));
      asm volatile("ld.shared.v4.b32 {%0, %1, %2, %3}, [%4];"
                   : "=r"(kb[0]), "=r"(kb[1]), "=r"(kb[2]), "=r"(kb[3])
                   : "r"(ks + box + sw128(lane + 32, c8 % 8)));
      float fa[8], fb[8];
#pragma unroll
      for (int u = 0; u < 4; ++u) {
        const float2 x = unpack2f<BF16>(ka[u]), y = unpack2f<BF16>(kb[u]);
        fa[2 * u] = x.x; fa[2 * u + 1] = x.y;
        fb[2 * u] = y.x; fb[2 * u + 1] = y.y;
      }
#pragma unroll
      for (int rr = 0; rr < RW; ++rr) {
        if (rr < nr) {
          const float4* qr = reinterpret_cast<const float4*>(qs + (warp + DEC_WARPS * rr) * D + c8 * 8);
          const float4 q0 = qr[0], q1 = qr[1];
          float a = s0[rr], bb = s1[rr];
          a = fmaf(q0.x, fa[0], a); a = fmaf(q0.y, fa[1], a); a = fmaf(q0.z, fa[2], a); a = fmaf(q0.w, fa[3], a);
          a = fmaf(q1.x, fa[4], a); a = fmaf(q1.y, fa[5], a); a = fmaf(q1.z, fa[6], a); a = fmaf(q1.w, fa[7], a);
          bb = fmaf(q0.x, fb[0], bb); bb = fmaf(q0.y, fb[1], bb); bb = fmaf(q0.z, fb[2], bb); bb = fmaf(q0.w, fb[3], bb);
          bb = fmaf(q1.x, fb[4], bb); bb = fmaf(q1.y, fb[5], bb); bb = fmaf(q1.z, fb[6], bb); bb = fmaf(q1.w, fb[7], bb);
          s0[rr] = a;
          s1[rr] = bb;
        }
      }
    }

    // mask, online softmax (log2 units, lazy rescale), probabilities
    float pa[RW], pb[RW];
    const int ja = j0 + lane, jb = j0 + 32 + lane;
#pragma unroll
    for (int rr = 0; rr < RW; ++rr) {
      pa[rr] = pb[rr] = 0.f;
      if (rr < nr) {
        const int r = warp + DEC_WARPS * rr;
        const int pos = p.N_kv - p.N_q + r % p.N_q;
        const bool ka_ = ja < j_end && (!p.causal || ja <= pos) &&
                         (p.window == 0 || pos - ja < p.window || ja < p.n_sink);
        const bool kb_ = jb < j_end && (!p.causal || jb <= pos) &&
                         (p.window == 0 || pos - jb < p.window || jb < p.n_sink);
        const float xa = ka_ ? s0[rr] : -INFINITY, xb = kb_ ? s1[rr] : -INFINITY;
        const float bmax = warp_max(fmaxf(xa, xb));
        const float m_new = fmaxf(m[rr], bmax);
        if (m_new > m[rr] + RESCALE_THRESHOLD) {
          const float alpha = (m[rr] == -INFINITY) ? 0.f : fast_exp2(m[rr] - m_new);
          l[rr] *= alpha;
#pragma unroll
          for (int c = 0; c < CPL; ++c) acc[rr][c] *= alpha;
          m[rr] = m_new;
        }
        const float mref = (m[rr] == -INFINITY) ? 0.f : m[rr];
        pa[rr] = fast_exp2(xa - mref);
        pb[rr] = fast_exp2(xb - mref);
        l[rr] += pa[rr] + pb[rr];
      }
    }

    // O += P V: lane owns columns CPL * lane .. + CPL - 1
#pragma unroll 4
    for (int t = 0; t < DEC_T; ++t) {
      float vf[CPL];
      if constexpr (D == 128) {
        uint32_t w0, w1;
        const uint32_t a = vs + (lane / 16) * G::BOX_BYTES + sw128(t, (lane % 16) / 2) + (lane & 1) * 8;
        asm volatile("ld.shared.v2.b32 {%0, %1}, [%2];" : "=r"(w0), "=r"(w1) : "r"(a));
        const float2 x = unpack2f<BF16>(w0), y = unpack2f<BF16>(w1);
        vf[0] = x.x; vf[1] = x.y; vf[2] = y.x; vf[3] = y.y;
      } else {
        uint32_t w0;
        const uint32_t a = vs + sw128(t, lane / 4) + (lane & 3) * 4;
        asm volatile("ld.shared.b32 %0, [%1];" : "=r"(w0) : "r"(a));
        const float2 x = unpack2f<BF16>(w0);
        vf[0] = x.x; vf[1] = x.y;
      }
#pragma unroll
      for (int rr = 0; rr < RW; ++rr) {
        if (rr < nr) {
          const float pt = __shfl_sync(0xffffffffu, t < 32 ? pa[rr] : pb[rr], t & 31);
#pragma unroll
          for (int c = 0; c < CPL; ++c) acc[rr][c] = fmaf(pt, vf[c], acc[rr][c]);
        }
      }
    }
    __syncwarp();
    if (lane == 0) mbar_arrive(bars + 8 * (DB_EMPTY + st));
  }

  // Every warp leaves the loop: either all tiles done, or a bounded wait gave
  // up (the status word then holds ATTN_ERR_DEVICE_TIMEOUT and the abort flag
  // makes the other warps give up too).  The verdict is made CTA-wide.
  if (!__syncthreads_and(ok ? 1 : 0)) {
    // let this CTA's copies land before it exits; no result is written
    if (warp == 0) {
      for (int s = 0; s < 2; ++s)
        if (issued_last[s] >= 0) drain_wait(bars + 8 * (DB_FULL + s), issued_last[s], p.watchdog_ns);
    }
    return;
  }

  // ---- this split's result for each row of the warp
#pragma unroll
  for (int rr = 0; rr < RW; ++rr) {
    if (rr < nr) {
      const int r = warp + DEC_WARPS * rr;
      const int h = g * G_heads + r / p.N_q, i = r % p.N_q;
      const float lt = warp_sum(l[rr]);
      const bool has = lt > 0.f;
      const float inv = has ? 1.f / lt : 0.f;
      const float lse_nat = has ? (m[rr] + __log2f(lt)) * 0.69314718055994531f : -INFINITY;
      const size_t row_idx = (static_cast<size_t>(b) * p.H + h) * p.N_q + i;
      if (p.n_splits == 1) {
        if constexpr (OUT_F32) {
          float* dst = static_cast<float*>(p.o) + row_idx * D + CPL * lane;
#pragma unroll
          for (int c = 0; c < CPL; ++c) dst[c] = acc[rr][c] * inv;
        } else {
          uint32_t w[CPL / 2];
#pragma unroll
          for (int c = 0; c < CPL / 2; ++c)
            w[c] = pack2<BF16>(acc[rr][2 * c] * inv, acc[rr][2 * c + 1] * inv);
          uint32_t* dst = reinterpret_cast<uint32_t*>(static_cast<uint16_t*>(p.o) + row_idx * D + CPL * lane);
#pragma unroll
          for (int c = 0; c < CPL / 2; ++c) dst[c] = w[c];
        }
        if (lane == 0 && p.lse != nullptr) p.lse[row_idx] = lse_nat;
      } else {
        const size_t ws_row = static_cast<size_t>(split) * p.B * p.H * p.N_q + row_idx;
        float* dst = p.ws_o + ws_row * D + CPL * lane;
#pragma unroll
        for (int c = 0; c < CPL; ++c) dst[c] = acc[rr][c] * inv;
        if (lane == 0) p.ws_lse[ws_row] = lse_nat;
      }
    }
  }
  if (p.n_splits == 1) return;

  // ---- the last split of this (b, g) to finish merges all of them
  __threadfence();
  __syncthreads();
  if (threadIdx.x == 0) {
    const int prev = atomicAdd(p.counters + bg, 1);
    *last_flag = (prev == p.n_splits - 1) ? 1 : 0;
  }
  __syncthreads();
  if (!*last_flag) return;
  __threadfence();
  const size_t split_stride = static_cast<size_t>(p.B) * p.H * p.N_q;
  for (int r = 0; r < R; ++r) {
    const int h = g * G_heads + r / p.N_q, i = r % p.N_q;
    const size_t row_idx = (static_cast<size_t>(b) * p.H + h) * p.N_q + i;
    float mx = -INFINITY;
    for (int s = 0; s < p.n_splits; ++s) mx = fmaxf(mx, __ldcg(p.ws_lse + s * split_stride + row_idx));
    float tot = 0.f;
    for (int s = 0; s < p.n_splits; ++s) {
      const float ls = __ldcg(p.ws_lse + s * split_stride + row_idx);
      tot += (ls == -INFINITY) ? 0.f : __expf(ls - mx);
    }
    const float lse_nat = mx + __logf(tot);
    for (int c = threadIdx.x; c < D; c += DEC_THREADS) {
      float o = 0.f;
      for (int s = 0; s < p.n_splits; ++s) {
        const float ls = __ldcg(p.ws_lse + s * split_stride + row_idx);
        if (ls == -INFINITY) continue;
        o = fmaf(__expf(ls - lse_nat), __ldcg(p.ws_o + (s * split_stride + row_idx) * D + c), o);
      }
      if constexpr (OUT_F32) {
        static_cast<float*>(p.o)[row_idx * D + c] = o;
      } else if constexpr (BF16) {
        static_cast<__nv_bfloat16*>(p.o)[row_idx * D + c] = __float2bfloat16_rn(o);
      } else {
        static_cast<__half*>(p.o)[row_idx * D + c] = __float2half_rn(o);
      }
    }
    if (threadIdx.x == 0 && p.lse != nullptr) p.lse[row_idx] = lse_nat;
  }
  if (threadIdx.x == 0) p.counters[bg] = 0;
}


// ------------------------------------------------------------ small groups
//
// Groups of at most 16 query rows (typical decoding: one or a few new tokens,
// GQA groups up to 16) use a leaner kernel.  Each of the NW warps takes its
// own slice of KPW = 64 / NW keys of every 64-key tile for all rows of the
// group and keeps its own running (m, l, O): the warps are sub-splits of the
// split, merged once at its end, so every K/V element is converted once and
// no per-tile exchange between warps is needed.  Lane (key lane % KPW, row
// group lane / KPW) forms the dot products of its key with its rows (four
// partial sums each, to keep the dependency chains short); the probabilities
// go through shared memory to the P V loop, where each lane owns D / 32
// output columns of every row.  Three pipeline stages.  More warps per CTA
// (NW = 8 for groups of up to 4 rows) hide more latency per scheduler.

constexpr int DEC_SMALL_STAGES = 3;

template <int D, int RMAX, int NW>
struct DecSmallGeo {
  static_assert(D == 64 || D == 128, "decode supports d = 64 and 128");
  static constexpr int NBOX = D / 64;
  static constexpr int BOX_BYTES = DEC_T * 128;
  static constexpr int TILE_BYTES = NBOX * BOX_BYTES;
  static constexpr int K_OFF = 0;                                   // stages, then reused for the merge
  static constexpr int V_OFF = K_OFF + DEC_SMALL_STAGES * TILE_BYTES;
  static constexpr int Q_OFF = V_OFF + DEC_SMALL_STAGES * TILE_BYTES;   // fp32 [RMAX][D]
  static constexpr int KPW = DEC_T / NW;                           // keys per warp per tile
  static constexpr int P_OFF = Q_OFF + RMAX * D * 4;                // fp32 [warp][RMAX][KPW]
  static constexpr int A_OFF = P_OFF + NW * RMAX * KPW * 4;         // fp32 [warp][RMAX] rescale
  static constexpr int BAR_OFF = A_OFF + NW * RMAX * 4;
  static constexpr int SMEM_BYTES = BAR_OFF + 8 * 2 * DEC_SMALL_STAGES + 16;
  // end-of-split merge buffers, over the K stages: m, l [warp][RMAX], O [warp][RMAX][D]
  static constexpr int MM_OFF = K_OFF;
  static constexpr int ML_OFF = MM_OFF + NW * RMAX * 4;
  static constexpr int MO_OFF = ML_OFF + NW * RMAX * 4;
  static_assert(MO_OFF + NW * RMAX * D * 4 <= V_OFF, "merge buffers fit the K stages");
  static_assert(KPW % 4 == 0 && 32 % KPW == 0, "key slice per warp");
};

template <int D, bool BF16, bool OUT_F32, int RMAX, int NW>
__global__ void __launch_bounds__(NW * 32, 1)
attn_decode_small_kernel(const __grid_constant__ CUtensorMap tmK,
                         const __grid_constant__ CUtensorMap tmV, const DecodeParams p) {
  using G = DecSmallGeo<D, RMAX, NW>;
  constexpr int NT = NW * 32;
  constexpr int KPW = G::KPW;
  constexpr int RQ = 32 / KPW;         // row groups per warp in the S phase
  constexpr int CPL = D / 32;          // output columns per lane
  constexpr int RH = RMAX / RQ;        // rows per lane in the S phase
  static_assert(RH >= 1, "row capacity");
  constexpr int NS = DEC_SMALL_STAGES;
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~static_cast<uintptr_t>(1023));
  const uint32_t sbase = smem_addr(smem);
  const uint32_t bars = sbase + G::BAR_OFF;          // FULL[NS], EMPTY[NS]
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + G::BAR_OFF + 8 * 2 * NS);
  volatile int* last_flag = abort_flag + 1;
  float* qs = reinterpret_cast<float*>(smem + G::Q_OFF);

  const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
  const int kl = lane % KPW, hf = lane / KPW;
  const int split = blockIdx.x, bg = blockIdx.y;
  const int b = bg / p.H_kv, g = bg % p.H_kv;
  const int G_heads = p.H / p.H_kv;
  const int R = G_heads * p.N_q;
  const int lo = split * p.split_keys, hi = min(p.N_kv, lo + p.split_keys);
  float* ps = reinterpret_cast<float*>(smem + G::P_OFF) + warp * RMAX * KPW;
  float* as = reinterpret_cast<float*>(smem + G::A_OFF) + warp * RMAX;

  if (threadIdx.x == 0) {
    for (int s = 0; s < NS; ++s) {
      mbar_init(bars + 8 * s, 1);
      mbar_init(bars + 8 * (NS + s), NW);
    }
    *abort_flag = 0;
    *last_flag = 0;
    fence_barrier_init();
    tma_prefetch_desc(&tmK);
    tma_prefetch_desc(&tmV);
  }
  for (int e = threadIdx.x; e < RMAX * (D / 2); e += NT) {
    const int r = e / (D / 2), c2 = e % (D / 2);
    float2 f = make_float2(0.f, 0.f);
    if (r < R) {
      const int h = g * G_heads + r / p.N_q, i = r % p.N_q;
      const size_t off = ((static_cast<size_t>(b) * p.H + h) * p.N_q + i) * D + 2 * c2;
      f = unpack2f<BF16>(*reinterpret_cast<const uint32_t*>(static_cast<const uint16_t*>(p.q) + off));
    }
    qs[r * D + 2 * c2] = f.x * p.scale_log2;
    qs[r * D + 2 * c2 + 1] = f.y * p.scale_log2;
  }
  __syncthreads();

  const int j_first = dec_next_tile(p, lo, hi);
  bool ok = true;
  int issued_last[NS];
#pragma unroll
  for (int s = 0; s < NS; ++s) issued_last[s] = -1;
  auto issue = [&](int j0, int n) {
    // failure-detection test: nothing is loaded (and nothing is left to drain)
    if (p.withhold_loads) return true;
    const int st = n % NS;
    const uint32_t ph = static_cast<uint32_t>(n / NS) & 1u;
    const uint32_t empty = bars + 8 * (NS + st);
    if (!mbar_try_wait(empty, ph ^ 1u) &&
        !wait_slow(empty, ph ^ 1u, abort_flag, p.status, p.watchdog_ns))
      return false;
    if (elect_one()) {
      mbar_arrive_expect_tx(bars + 8 * st, 2 * G::TILE_BYTES);
      for (int c = 0; c < G::NBOX; ++c) {
        tma_load_3d(sbase + G::K_OFF + st * G::TILE_BYTES + c * G::BOX_BYTES, &tmK, bars + 8 * st,
                    c * 64, j0, bg);
        tma_load_3d(sbase + G::V_OFF + st * G::TILE_BYTES + c * G::BOX_BYTES, &tmV, bars + 8 * st,
                    c * 64, j0, bg);
      }
    }
    __syncwarp();
    issued_last[st] = static_cast<int>(ph);
    return true;
  };
  // prologue: the first NS - 1 tiles
  int j_pre = j_first;
  if (warp == 0) {
    for (int n = 0; n < NS - 1 && j_pre < hi && ok; ++n) {
      ok = __all_sync(0xffffffffu, issue(j_pre, n));
      j_pre = dec_next_tile(p, j_pre + DEC_T, hi);
    }
  }

  float m[RH], l[RH], acc[RMAX][CPL];
#pragma unroll
  for (int rr = 0; rr < RH; ++rr) {
    m[rr] = -INFINITY;
    l[rr] = 0.f;
  }
#pragma unroll
  for (int r = 0; r < RMAX; ++r)
#pragma unroll
    for (int c = 0; c < CPL; ++c) acc[r][c] = 0.f;

  int n = 0;
  for (int j0 = j_first; j0 < hi && ok; j0 = dec_next_tile(p, j0 + DEC_T, hi), ++n) {
    const int st = n % NS;
    if (warp == 0) {
      if (j_pre < hi) {
        ok = __all_sync(0xffffffffu, issue(j_pre, n + NS - 1));
        j_pre = dec_next_tile(p, j_pre + DEC_T, hi);
      }
      if (!ok) break;
    }
    {
      const uint32_t full = bars + 8 * st, ph = static_cast<uint32_t>(n / NS) & 1u;
      ok = __all_sync(0xffffffffu, mbar_try_wait(full, ph) ||
                                       wait_slow(full, ph, abort_flag, p.status, p.watchdog_ns));
    }
    if (!ok) break;
    const uint32_t ks = sbase + G::K_OFF + st * G::TILE_BYTES;
    const uint32_t vs = sbase + G::V_OFF + st * G::TILE_BYTES;
    const int t = warp * KPW + kl;                 // this lane's key within the tile
    const int j = j0 + t;

    // S for key j and rows r = hf + RQ rr, four partial sums each
    float sa[RH][4];
#pragma unroll
    for (int rr = 0; rr < RH; ++rr)
#pragma unroll
      for (int u = 0; u < 4; ++u) sa[rr][u] = 0.f;
#pragma unroll 4
    for (int c8 = 0; c8 < D / 8; ++c8) {
      uint32_t kw[4];
      asm volatile("ld.shared.v4.b32 {%0, %1, %2, %3}, [%4];"
                   : "=r"(kw[0]), "=r"(kw[1]), "=r"(kw[2]), "=r"(kw[3])
                   : "r"(ks + (c8 / 8) * G::BOX_BYTES + sw128(t, c8 % 8)));
      float kf[8];
#pragma unroll
      for (int u = 0; u < 4; ++u) {
        const float2 x = unpack2f<BF16>(kw[u]);
        kf[2 * u] = x.x;
        kf[2 * u + 1] = x.y;
      }
#pragma unroll
      for (int rr = 0; rr < RH; ++rr) {
        const int r = hf + RQ * rr;
        if (r < R) {
          const float4* qr = reinterpret_cast<const float4*>(qs + r * D + c8 * 8);
          const float4 q0 = qr[0], q1 = qr[1];
          sa[rr][0] = fmaf(q0.x, kf[0], sa[rr][0]);
          sa[rr][1] = fmaf(q0.y, kf[1], sa[rr][1]);
          sa[rr][2] = fmaf(q0.z, kf[2], sa[rr][2]);
          sa[rr][3] = fmaf(q0.w, kf[3], sa[rr][3]);
          sa[rr][0] = fmaf(q1.x, kf[4], sa[rr][0]);
          sa[rr][1] = fmaf(q1.y, kf[5], sa[rr][1]);
          sa[rr][2] = fmaf(q1.z, kf[6], sa[rr][2]);
          sa[rr][3] = fmaf(q1.w, kf[7], sa[rr][3]);
        }
      }
    }

    // masking and online softmax over this warp's KPW keys (one lane group per
    // row group); P and the rescale factors go to shared memory
    const int j_end = min(j0 + DEC_T, hi);
#pragma unroll
    for (int rr = 0; rr < RH; ++rr) {
      const int r = hf + RQ * rr;                  // rows >= R carry -inf and stay inert
      const int pos = p.N_kv - p.N_q + r % p.N_q;
      const bool keep = r < R && j < j_end && (!p.causal || j <= pos) &&
                        (p.window == 0 || pos - j < p.window || j < p.n_sink);
      const float x = keep ? (sa[rr][0] + sa[rr][1]) + (sa[rr][2] + sa[rr][3]) : -INFINITY;
      // row max over the KPW keys of this lane group (all 32 lanes shuffle)
      float bmax = x;
#pragma unroll
      for (int o = KPW / 2; o > 0; o >>= 1) bmax = fmaxf(bmax, __shfl_xor_sync(0xffffffffu, bmax, o));
      float alpha = 1.f;
      const float m_new = fmaxf(m[rr], bmax);
      if (m_new > m[rr] + RESCALE_THRESHOLD) {
        alpha = (m[rr] == -INFINITY) ? 0.f : fast_exp2(m[rr] - m_new);
        l[rr] *= alpha;
        m[rr] = m_new;
      }
      const float pj = fast_exp2(x - ((m[rr] == -INFINITY) ? 0.f : m[rr]));
      l[rr] += pj;
      ps[r * KPW + kl] = pj;
      if (kl == 0) as[r] = alpha;
    }
    __syncwarp();

    // O += P V over this warp's KPW keys; lane owns columns CPL * lane ..
#pragma unroll
    for (int r = 0; r < RMAX; ++r) {
      if (r < R) {
        const float a = as[r];
#pragma unroll
        for (int c = 0; c < CPL; ++c) acc[r][c] *= a;
      }
    }
#pragma unroll
    for (int k4 = 0; k4 < KPW; k4 += 4) {
      float vf[4][CPL];
#pragma unroll
      for (int kk = 0; kk < 4; ++kk) {
        const int tv = warp * KPW + k4 + kk;
        if constexpr (D == 128) {
          uint32_t w0, w1;
          const uint32_t a = vs + (lane / 16) * G::BOX_BYTES + sw128(tv, (lane % 16) / 2) + (lane & 1) * 8;
          asm volatile("ld.shared.v2.b32 {%0, %1}, [%2];" : "=r"(w0), "=r"(w1) : "r"(a));
          const float2 x = unpack2f<BF16>(w0), y = unpack2f<BF16>(w1);
          vf[kk][0] = x.x; vf[kk][1] = x.y; vf[kk][2] = y.x; vf[kk][3] = y.y;
        } else {
          uint32_t w0;
          const uint32_t a = vs + sw128(tv, lane / 4) + (lane & 3) * 4;
          asm volatile("ld.shared.b32 %0, [%1];" : "=r"(w0) : "r"(a));
          const float2 x = unpack2f<BF16>(w0);
          vf[kk][0] = x.x; vf[kk][1] = x.y;
        }
      }
#pragma unroll
      for (int r = 0; r < RMAX; ++r) {
        if (r < R) {
          const float4 p4 = *reinterpret_cast<const float4*>(ps + r * KPW + k4);
#pragma unroll
          for (int c = 0; c < CPL; ++c) {
            float o = acc[r][c];
            o = fmaf(p4.x, vf[0][c], o);
            o = fmaf(p4.y, vf[1][c], o);
            o = fmaf(p4.z, vf[2][c], o);
            o = fmaf(p4.w, vf[3][c], o);
            acc[r][c] = o;
          }
        }
      }
    }
    __syncwarp();
    if (lane == 0) mbar_arrive(bars + 8 * (NS + st));
  }

  if (!__syncthreads_and(ok ? 1 : 0)) {
    if (warp == 0) {
      for (int s = 0; s < NS; ++s)
        if (issued_last[s] >= 0) drain_wait(bars + 8 * s, issued_last[s], p.watchdog_ns);
    }
    return;
  }

  // ---- merge the four warps' sub-splits (buffers over the now idle K stages)
  float* mm = reinterpret_cast<float*>(smem + G::MM_OFF);
  float* ml = reinterpret_cast<float*>(smem + G::ML_OFF);
  float* mo = reinterpret_cast<float*>(smem + G::MO_OFF);
#pragma unroll
  for (int rr = 0; rr < RH; ++rr) {
    const int r = hf + RQ * rr;
    float lt = l[rr];
#pragma unroll
    for (int o = KPW / 2; o > 0; o >>= 1) lt += __shfl_xor_sync(0xffffffffu, lt, o);
    if (r < RMAX && kl == 0) {
      mm[warp * RMAX + r] = (r < R) ? m[rr] : -INFINITY;
      ml[warp * RMAX + r] = (r < R) ? lt : 0.f;
    }
  }
#pragma unroll
  for (int r = 0; r < RMAX; ++r)
#pragma unroll
    for (int c = 0; c < CPL; ++c) mo[(warp * RMAX + r) * D + CPL * lane + c] = acc[r][c];
  __syncthreads();

  const size_t split_stride = static_cast<size_t>(p.B) * p.H * p.N_q;
  for (int e = threadIdx.x; e < R * D; e += NT) {
    const int r = e / D, c = e % D;
    float M = -INFINITY;
#pragma unroll
    for (int w = 0; w < NW; ++w) M = fmaxf(M, mm[w * RMAX + r]);
    float lt = 0.f, o = 0.f;
    if (M != -INFINITY) {
#pragma unroll
      for (int w = 0; w < NW; ++w) {
        const float mw = mm[w * RMAX + r];
        if (mw == -INFINITY) continue;
        const float s = fast_exp2(mw - M);
        lt = fmaf(s, ml[w * RMAX + r], lt);
        o = fmaf(s, mo[(w * RMAX + r) * D + c], o);
      }
    }
    const bool has = lt > 0.f;
    const float ov = has ? o / lt : 0.f;
    const float lse_nat = has ? (M + __log2f(lt)) * 0.69314718055994531f : -INFINITY;
    const int h = g * G_heads + r / p.N_q, i = r % p.N_q;
    const size_t row_idx = (static_cast<size_t>(b) * p.H + h) * p.N_q + i;
    if (p.n_splits == 1) {
      if constexpr (OUT_F32) {
        static_cast<float*>(p.o)[row_idx * D + c] = ov;
      } else if constexpr (BF16) {
        static_cast<__nv_bfloat16*>(p.o)[row_idx * D + c] = __float2bfloat16_rn(ov);
      } else {
        static_cast<__half*>(p.o)[row_idx * D + c] = __float2half_rn(ov);
      }
      if (c == 0 && p.lse != nullptr) p.lse[row_idx] = lse_nat;
    } else {
      const size_t ws_row = static_cast<size_t>(split) * split_stride + row_idx;
      p.ws_o[ws_row * D + c] = ov;
      if (c == 0) p.ws_lse[ws_row] = lse_nat;
    }
  }
  if (p.n_splits == 1) return;

  // ---- the last split of this (b, g) to finish merges all of them
  __threadfence();
  __syncthreads();
  if (threadIdx.x == 0) {
    const int prev = atomicAdd(p.counters + bg, 1);
    *last_flag = (prev == p.n_splits - 1) ? 1 : 0;
  }
  __syncthreads();
  if (!*last_flag) return;
  __threadfence();
  for (int e = threadIdx.x; e < R * D; e += NT) {
    const int r = e / D, c = e % D;
    const int h = g * G_heads + r / p.N_q, i = r % p.N_q;
    const size_t row_idx = (static_cast<size_t>(b) * p.H + h) * p.N_q + i;
    float mx = -INFINITY;
    for (int s = 0; s < p.n_splits; ++s) mx = fmaxf(mx, __ldcg(p.ws_lse + s * split_stride + row_idx));
    float tot = 0.f;
    for (int s = 0; s < p.n_splits; ++s) {
      const float ls = __ldcg(p.ws_lse + s * split_stride + row_idx);
      tot += (ls == -INFINITY) ? 0.f : __expf(ls - mx);
    }
    const float lse_nat = mx + __logf(tot);
    float o = 0.f;
    for (int s = 0; s < p.n_splits; ++s) {
      const float ls = __ldcg(p.ws_lse + s * split_stride + row_idx);
      if (ls == -INFINITY) continue;
      o = fmaf(__expf(ls - lse_nat), __ldcg(p.ws_o + (s * split_stride + row_idx) * D + c), o);
    }
    if constexpr (OUT_F32) {
      static_cast<float*>(p.o)[row_idx * D + c] = o;
    } else if constexpr (BF16) {
      static_cast<__nv_bfloat16*>(p.o)[row_idx * D + c] = __float2bfloat16_rn(o);
    } else {
      static_cast<__half*>(p.o)[row_idx * D + c] = __float2half_rn(o);
    }
    if (c == 0 && p.lse != nullptr) p.lse[row_idx] = lse_nat;
  }
  if (threadIdx.x == 0) p.counters[bg] = 0;
}

}  // namespace attn

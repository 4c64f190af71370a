// decode_tc_kernel.cuh -- split-KV decoding step on the tensor cores (sm_100a).
//
// What it computes: the N_q new query rows of every query head attend to a
// K/V cache of N_kv positions under the forward's mask rule, the query row i
// of a head sitting at cache position N_kv - N_q + i ("USAAIO Lesson 91", slide 31: every decoding step re-reads
// the whole cache; slide 32: the query heads of a group share one K/V head).
//
// How: the R = (H / H_kv) * N_q query rows of one (batch, K/V head) group form
// the A operand of S = Q K^T on the tensor core, placed on TMEM lanes
// 32 (r % 4) + r / 4 of a 128-row tile whose other rows are zero, so that the
// rows are spread over the four lane quarters and the four softmax warps of a
// warpgroup share them.  Each 128-key K/V tile of the cache is read from HBM
// once, by TMA, into a ring of shared-memory stages.  Two softmax warpgroups
// take the even and the odd tiles of a run, each with its own S buffer, its
// own running (m, l) and its own O accumulator in TMEM (the same two-tile
// ping-pong as the forward kernel, over keys instead of queries), and the two
// halves are combined when the run ends.  P is written over S in TMEM and
// O += P V reads it from there.
//
// Work split ("Building a FlashAttention-style tiled self-attention block in
// pure NumPy", "Extending It", item 6: split the sequence, then reduce the
// partial outputs): the kept tiles of all groups are laid end to end and cut
// into DT_GRID equal ranges, one per CTA.  A CTA's range covers one or more
// runs (the part of a range inside one group).  A group covered by one run
// gets its output written directly; otherwise every run writes its partial
// (O_s normalised over its own keys, LSE_s) to the workspace, and a second,
// small kernel merges the parts of each group in part order:
//     LSE = ln sum_s exp(LSE_s),   O = sum_s exp(LSE_s - LSE) O_s,
// so the result does not depend on which CTA finishes first.
#pragma once

#include "attn_kernel.cuh"

namespace attn {

constexpr int DT_TILE = 128;        // keys per K/V tile
constexpr int DT_GRID = 148;        // ranges of the tile space (one CTA per SM of a B200)
constexpr int DT_MAX_ROWS = 64;     // query rows of one group: (H / H_kv) * N_q

struct DecTcParams {
  const void* q;
  void* o;
  float* lse;
  float* ws_o;        // [n_groups][max_parts][R][D] partial outputs
  float* ws_lse;      // [n_groups][max_parts][R] partial LSE (natural log)
  int* status;
  unsigned long long watchdog_ns;
  int B, H, H_kv, N_q, N_kv;
  int causal, window, n_sink;
  float scale_log2;   // scale * log2(e)
  int R;              // query rows per group
  int n_groups;       // B * H_kv
  int sb, wlo, nt;    // kept tiles of every group: [0, sb), then [max(wlo, sb), nt)
  int tiles;          // kept tiles per group
  int grid;           // ranges of the tile space (= CTAs)
  int max_parts;      // workspace slots per group
  int withhold_loads; // test hook: no tile is loaded, so every wait runs out
};

// Shared-memory layout for head dimension D (64 or 128): the Q tile, then the
// K and V stages, the second warpgroup's row statistics and the barriers.
template <int D>
struct DtGeo {
  static_assert(D == 64 || D == 128, "the decoding kernel supports d = 64 and 128");
  using G = Geo<D>;                                    // 64-column chunks, 128-byte swizzle
  static constexpr int NST = D == 128 ? 3 : 4;         // K/V ring stages
  static constexpr int Q_OFF = 0;
  static constexpr int K_OFF = Q_OFF + G::TILE_BYTES;
  static constexpr int V_OFF = K_OFF + NST * G::TILE_BYTES;
  static constexpr int STAT_OFF = V_OFF + NST * G::TILE_BYTES;   // float [3][128]
  static constexpr int BAR_OFF = STAT_OFF + 3 * 128 * 4;
  static constexpr int SMEM_BYTES = BAR_OFF + 256;
  static constexpr uint32_t S_COL0 = 0;                // S_h at column 128 h
  static constexpr uint32_t O_COL0 = 256;              // O_h at column 256 + D h
  static_assert(SMEM_BYTES + 1024 <= 232448, "shared memory budget");
};

enum DtBar : int {
  T_K_FULL = 0, T_K_EMPTY = 4, T_V_FULL = 8, T_V_EMPTY = 12,   // [NST] each (at most 4)
  T_S_FULL = 16, T_P_FULL = 18, T_O_FULL = 20,                // [2] each
  T_Q_FULL = 22, T_HALF = 23, T_DRAIN = 24, T_COUNT = 25
};
constexpr int DT_TMEM_SLOT_OFF = 8 * T_COUNT;
constexpr int DT_ABORT_OFF = DT_TMEM_SLOT_OFF + 4;

// ------------------------------------------------------------ partition

__host__ __device__ inline long long dt_range_start(int c, long long F, int grid) {
  return static_cast<long long>(c) * F / grid;
}

// The range (CTA) that holds flattened tile f.
__host__ __device__ inline int dt_cta_of(long long f, long long F, int grid) {
  int c = static_cast<int>(f * grid / F);
  while (c + 1 < grid && dt_range_start(c + 1, F, grid) <= f) ++c;
  while (c > 0 && dt_range_start(c, F, grid) > f) --c;
  return c;
}

// Block index of kept tile i of a group.
__device__ __forceinline__ int dt_block(const DecTcParams& p, int i) {
  return i < p.sb ? i : max(p.wlo, p.sb) + (i - p.sb);
}

// True when some (row, key) of the tile starting at key c0 is masked.
__device__ __forceinline__ bool dt_needs_mask(const DecTcParams& p, int c0) {
  if (c0 + DT_TILE > p.N_kv) return true;
  const int pos_min = p.N_kv - p.N_q, pos_max = p.N_kv - 1;
  if (p.causal && c0 + DT_TILE - 1 > pos_min) return true;
  if (p.window > 0 && pos_max - p.window + 1 > c0 && !(c0 + DT_TILE <= p.n_sink)) return true;
  return false;
}

// One run: tiles [i0, i0 + n) of group g, part `part` of `n_parts`.
struct DtRun {
  int g, i0, n, part, n_parts;
};

// The run that starts at flattened tile x of a CTA range ending at e.
__device__ __forceinline__ DtRun dt_run_at(const DecTcParams& p, long long x, long long e) {
  const long long FT = static_cast<long long>(p.n_groups) * p.tiles;
  DtRun r;
  r.g = static_cast<int>(x / p.tiles);
  r.i0 = static_cast<int>(x - static_cast<long long>(r.g) * p.tiles);
  const long long g_end = static_cast<long long>(r.g + 1) * p.tiles;
  r.n = static_cast<int>((e < g_end ? e : g_end) - x);
  const int c_first = dt_cta_of(static_cast<long long>(r.g) * p.tiles, FT, p.grid);
  r.part = static_cast<int>(blockIdx.x) - c_first;
  r.n_parts = dt_cta_of(g_end - 1, FT, p.grid) - c_first + 1;
  return r;
}

// Runs of CTA `cta`, in order; calls f(run) for each.
template <class F>
__device__ __forceinline__ void dt_for_runs(const DecTcParams& p, int cta, F&& f) {
  const long long FT = static_cast<long long>(p.n_groups) * p.tiles;
  const long long a = dt_range_start(cta, FT, p.grid), e = dt_range_start(cta + 1, FT, p.grid);
  long long x = a;
  while (x < e) {
    DtRun r;
    r.g = static_cast<int>(x / p.tiles);
    r.i0 = static_cast<int>(x % p.tiles);
    const long long g_end = static_cast<long long>(r.g + 1) * p.tiles;
    const long long y = e < g_end ? e : g_end;
    r.n = static_cast<int>(y - x);
    const int c_first = dt_cta_of(static_cast<long long>(r.g) * p.tiles, FT, p.grid);
    const int c_last = dt_cta_of(g_end - 1, FT, p.grid);
    r.part = cta - c_first;
    r.n_parts = c_last - c_first + 1;
    f(r);
    x = y;
  }
}

// ------------------------------------------------------------ roles

template <int D>
__device__ void dt_tma_role(const DecTcParams& p, const CUtensorMap* tmK, const CUtensorMap* tmV,
                            uint32_t sbase, uint32_t bars, volatile int* abort_flag) {
  using T = DtGeo<D>;
  using G = Geo<D>;
  if (p.withhold_loads) return;   // failure-detection test: every wait on a tile runs out
  uint32_t it = 0;
  int k_last[T::NST], v_last[T::NST];
  for (int s = 0; s < T::NST; ++s) k_last[s] = v_last[s] = -1;
  bool ok = true;
  auto wait = [&](uint32_t bar, uint32_t par) {
    const bool w = mbar_try_wait(bar, par) || wait_slow(bar, par, abort_flag, p.status, p.watchdog_ns);
    return __all_sync(0xffffffffu, w);
  };
  dt_for_runs(p, blockIdx.x, [&](const DtRun& r) {
    for (int k = 0; k < r.n && ok; ++k, ++it) {
      const int s = it % T::NST;
      const uint32_t ph = (it / T::NST) & 1u;
      const int j = dt_block(p, r.i0 + k);
      ok = wait(bars + 8 * (T_K_EMPTY + s), ph ^ 1u);
      if (!ok) break;
      if (elect_one()) {
        mbar_arrive_expect_tx(bars + 8 * (T_K_FULL + s), G::TILE_BYTES);
        for (int c = 0; c < G::NCH; ++c)
          tma_load_3d(sbase + T::K_OFF + s * G::TILE_BYTES + c * G::CHUNK_BYTES, tmK,
                      bars + 8 * (T_K_FULL + s), c * G::CW, j * DT_TILE, r.g);
      }
      __syncwarp();
      k_last[s] = static_cast<int>(ph);
      ok = wait(bars + 8 * (T_V_EMPTY + s), ph ^ 1u);
      if (!ok) break;
      if (elect_one()) {
        mbar_arrive_expect_tx(bars + 8 * (T_V_FULL + s), G::TILE_BYTES);
        for (int c = 0; c < G::NCH; ++c)
          tma_load_3d(sbase + T::V_OFF + s * G::TILE_BYTES + c * G::CHUNK_BYTES, tmV,
                      bars + 8 * (T_V_FULL + s), c * G::CW, j * DT_TILE, r.g);
      }
      __syncwarp();
      v_last[s] = static_cast<int>(ph);
    }
  });
  if (!ok) {
    for (int s = 0; s < T::NST; ++s) {
      if (k_last[s] >= 0) drain_wait(bars + 8 * (T_K_FULL + s), k_last[s], p.watchdog_ns);
      if (v_last[s] >= 0) drain_wait(bars + 8 * (T_V_FULL + s), v_last[s], p.watchdog_ns);
    }
  }
}

template <int D, bool BF16>
__device__ void dt_mma_role(const DecTcParams& p, uint32_t tmem, uint32_t sbase, uint32_t bars,
                            volatile int* abort_flag) {
  using T = DtGeo<D>;
  using G = Geo<D>;
  constexpr uint32_t idesc_qk = instr_desc(BF16, BM, DT_TILE, false);
  constexpr uint32_t idesc_pv = instr_desc(BF16, BM, D, true);
  uint32_t it = 0, q_ph = 0, p_ph[2] = {0, 0};
  bool ok = true;
  auto wait = [&](uint32_t bar, uint32_t par) {
    const bool w = mbar_try_wait(bar, par) || wait_slow(bar, par, abort_flag, p.status, p.watchdog_ns);
    return __all_sync(0xffffffffu, w);
  };
  // S_h = Q K^T of the tile in stage s
  auto issue_s = [&](int h, int s) {
    const uint32_t qa = sbase + T::Q_OFF;
    const uint32_t ka = sbase + T::K_OFF + s * G::TILE_BYTES;
#pragma unroll
    for (int kk = 0; kk < D / 16; ++kk) {
      const uint32_t off = (kk * 16 / G::CW) * G::CHUNK_BYTES + ((kk * 16) % G::CW) * 2;
      mma_ss(tmem + T::S_COL0 + h * DT_TILE, smem_desc(qa + off, 16, 8 * G::CB, G::LAYOUT),
             smem_desc(ka + off, 16, 8 * G::CB, G::LAYOUT), idesc_qk, kk > 0 ? 1u : 0u);
    }
  };
  // O_h (+)= P_h V of the tile in stage s
  auto issue_o = [&](int h, int s, bool acc) {
    const uint32_t va = sbase + T::V_OFF + s * G::TILE_BYTES;
#pragma unroll
    for (int kk = 0; kk < DT_TILE / 16; ++kk)
      mma_ts(tmem + T::O_COL0 + h * D, tmem + T::S_COL0 + h * DT_TILE + kk * 8,
             smem_desc(va + kk * 16 * G::CB, G::CHUNK_BYTES, 8 * G::CB, G::LAYOUT), idesc_pv,
             (acc || kk > 0) ? 1u : 0u);
  };
  dt_for_runs(p, blockIdx.x, [&](const DtRun& r) {
    if (!ok) return;
    // the run's query rows are in the Q tile
    ok = wait(bars + 8 * T_Q_FULL, q_ph);
    if (!ok) return;
    q_ph ^= 1u;
    tc_fence_after_sync();
    // S for the first two tiles
    for (int k = 0; k < r.n && k < 2; ++k) {
      const int s = (it + k) % T::NST;
      ok = wait(bars + 8 * (T_K_FULL + s), ((it + k) / T::NST) & 1u);
      if (!ok) return;
      tc_fence_after_sync();
      if (elect_one()) {
        issue_s(k, s);
        mma_commit(bars + 8 * (T_S_FULL + k));
        mma_commit(bars + 8 * (T_K_EMPTY + s));
      }
      __syncwarp();
    }
    for (int k = 0; k < r.n; ++k) {
      const int h = k & 1;
      const uint32_t itk = it + k;
      const int s = itk % T::NST;
      ok = wait(bars + 8 * (T_V_FULL + s), (itk / T::NST) & 1u);
      if (!ok) return;
      ok = wait(bars + 8 * (T_P_FULL + h), p_ph[h]);
      if (!ok) return;
      p_ph[h] ^= 1u;
      tc_fence_after_sync();
      if (elect_one()) {
        issue_o(h, s, k >= 2);
        if (k + 2 >= r.n) mma_commit(bars + 8 * (T_O_FULL + h));
        mma_commit(bars + 8 * (T_V_EMPTY + s));
      }
      __syncwarp();
      if (k + 2 < r.n) {
        // S_h for tile k + 2 overwrites P_h only after the P_h V just issued
        const uint32_t itn = itk + 2;
        const int sn = itn % T::NST;
        ok = wait(bars + 8 * (T_K_FULL + sn), (itn / T::NST) & 1u);
        if (!ok) return;
        tc_fence_after_sync();
        if (elect_one()) {
          issue_s(h, sn);
          mma_commit(bars + 8 * (T_S_FULL + h));
          mma_commit(bars + 8 * (T_K_EMPTY + sn));
        }
        __syncwarp();
      }
    }
    it += r.n;
  });
  if (elect_one()) mma_commit(bars + 8 * T_DRAIN);
  __syncwarp();
  drain_wait(bars + 8 * T_DRAIN, 0, p.watchdog_ns);
}

template <int D, bool BF16, bool OUT_F32>
__device__ void dt_softmax_role(const DecTcParams& p, uint32_t tmem, uint8_t* smem, uint32_t sbase,
                                uint32_t bars, int h, int w, int lane, volatile int* abort_flag) {
  using T = DtGeo<D>;
  using G = Geo<D>;
  const uint32_t lane_base = static_cast<uint32_t>(w * 32) << 16;
  const uint32_t s_tmem = tmem + lane_base + T::S_COL0 + h * DT_TILE;
  const int L = w * 32 + lane;            // TMEM lane (row of the tile)
  const int r = 4 * lane + w;             // query row of the group on this lane
  const bool real = r < p.R;
  const int pos = p.N_kv - p.N_q + (real ? r % p.N_q : p.N_q - 1);
  // A scale of 0 (every kept logit 0) is run as 1e-30: the logits then stay
  // within 1e-25 of 0, every weight rounds to exactly 1 in fp32 as for 0,
  // and masked keys still give -inf (not 0 * inf).
  const float c = p.scale_log2 != 0.f ? p.scale_log2 : 1e-30f;
  float* stat = reinterpret_cast<float*>(smem + T::STAT_OFF);
  uint32_t s_ph = 0, o_ph[2] = {0, 0}, half_ph = 0;
  bool ok = true;
  auto wait = [&](uint32_t bar, uint32_t par) {
    const bool w2 = mbar_try_wait(bar, par) || wait_slow(bar, par, abort_flag, p.status, p.watchdog_ns);
    return __all_sync(0xffffffffu, w2);
  };
  const long long FT = static_cast<long long>(p.n_groups) * p.tiles;
  const long long x_end = dt_range_start(blockIdx.x + 1, FT, p.grid);
  for (long long x = dt_range_start(blockIdx.x, FT, p.grid); x < x_end && ok;) {
    const DtRun run = dt_run_at(p, x, x_end);
    x += run.n;
    const int b = run.g / p.H_kv, gk = run.g % p.H_kv;
    const int G_heads = p.H / p.H_kv;
    const int hq = gk * G_heads + (real ? r / p.N_q : 0);
    const size_t row_idx = ((static_cast<size_t>(b) * p.H + hq) * p.N_q) + (real ? r % p.N_q : 0);
    if (h == 0) {
      // this lane's query row (zeros for lanes without one) into the Q tile, in
      // the K-major 128-byte swizzle of the S = Q K^T operand; the previous
      // run's MMAs have all completed (its epilogue waited for the last P V)
      const uint32_t row_addr = sbase + T::Q_OFF + L * 128;
      const uint4* src = reinterpret_cast<const uint4*>(static_cast<const uint16_t*>(p.q) + row_idx * D);
#pragma unroll
      for (int u = 0; u < D / 8; ++u) {
        const uint4 v4 = real ? src[u] : make_uint4(0u, 0u, 0u, 0u);
        st_shared_v4(row_addr + (u / 8) * G::CHUNK_BYTES + (((u % 8) ^ (L & 7)) << 4), v4.x, v4.y,
                     v4.z, v4.w);
      }
      fence_proxy_async_smem();
      __syncwarp();
      if (lane == 0) mbar_arrive(bars + 8 * T_Q_FULL);
    }
    float m_run = -INFINITY, l_exact = 0.f, l_round = 0.f;
    bool first = true;
    for (int k = h; k < run.n; k += 2) {
      const int c0 = dt_block(p, run.i0 + k) * DT_TILE;
      ok = wait(bars + 8 * (T_S_FULL + h), s_ph);
      if (!ok) break;
      s_ph ^= 1u;
      tc_fence_after_sync();
      uint32_t sr[128];
      tmem_ld_32x32b_x128(s_tmem, sr);
      const bool masked = dt_needs_mask(p, c0);
      if (masked) {
        // masked keys get the raw score -inf (+inf for a negative scale, which
        // the scale turns into -inf); kept keys of this row in tile columns e:
        // e <= hi and (e >= lo or e < sk)
        const uint32_t gone = c >= 0.f ? 0xff800000u : 0x7f800000u;
        const int hi = (p.causal ? pos : p.N_kv - 1) - c0;
        const int lo = p.window > 0 ? pos - p.window + 1 - c0 : -(1 << 30);
        const int sk = p.window > 0 ? p.n_sink - c0 : -(1 << 30);
#pragma unroll
        for (int e = 0; e < 128; ++e) {
          const bool keep = (e <= hi) && (e >= lo || e < sk);
          sr[e] = keep ? sr[e] : gone;
        }
      }
      // raw-score extreme, then one multiply: max of s*c is c*max(s) for
      // c >= 0 and c*min(s) for c < 0
      float m_blk;
      {
        float m0 = __uint_as_float(sr[0]), m1 = __uint_as_float(sr[1]);
        if (c >= 0.f) {
#pragma unroll
          for (int e = 2; e < 126; e += 4) {
            m0 = max3(m0, __uint_as_float(sr[e]), __uint_as_float(sr[e + 1]));
            m1 = max3(m1, __uint_as_float(sr[e + 2]), __uint_as_float(sr[e + 3]));
          }
          m0 = max3(m0, __uint_as_float(sr[126]), __uint_as_float(sr[127]));
          m_blk = fmaxf(m0, m1) * c;
        } else {
#pragma unroll
          for (int e = 2; e < 126; e += 4) {
            m0 = min3(m0, __uint_as_float(sr[e]), __uint_as_float(sr[e + 1]));
            m1 = min3(m1, __uint_as_float(sr[e + 2]), __uint_as_float(sr[e + 3]));
          }
          m0 = min3(m0, __uint_as_float(sr[126]), __uint_as_float(sr[127]));
          m_blk = fminf(m0, m1) * c;
        }
      }
      // online softmax (log2 units), lazy rescale as in the forward kernel
      const float m_new = fmaxf(m_run, m_blk);
      float alpha = 1.f;
      const bool rescale = m_new > m_run + RESCALE_THRESHOLD;
      if (rescale) {
        alpha = (m_run == -INFINITY) ? 0.f : fast_exp2(m_run - m_new);
        m_run = m_new;
      }
      const float mref = (m_run == -INFINITY) ? 0.f : m_run;
      const float2 cc2 = make_float2(c, c);
      const float2 nm2 = make_float2(-mref, -mref);
      float2 le = make_float2(0.f, 0.f), lr = make_float2(0.f, 0.f);
#pragma unroll
      for (int q4 = 0; q4 < 4; ++q4) {
        uint32_t pk[16];
        float2 le_q = make_float2(0.f, 0.f), lr_q = make_float2(0.f, 0.f);
#pragma unroll
        for (int e = 0; e < 16; ++e) {
          const float2 x = make_float2(__uint_as_float(sr[32 * q4 + 2 * e]),
                                       __uint_as_float(sr[32 * q4 + 2 * e + 1]));
          const float2 a = fma2(x, cc2, nm2);
          const float2 pe = make_float2(fast_exp2(a.x), fast_exp2(a.y));
          pk[e] = pack2<BF16>(pe.x, pe.y);
          le_q = add2(le_q, pe);
          lr_q = add2(lr_q, make_float2(unpack_lo<BF16>(pk[e]), unpack_hi<BF16>(pk[e])));
        }
        tmem_st_32x32b_x16(s_tmem + 16 * q4, pk);
        le = add2(le, le_q);
        lr = add2(lr, lr_q);
      }
      l_exact = l_exact * alpha + (le.x + le.y);
      l_round = l_round * alpha + (lr.x + lr.y);
      if (!first && __any_sync(0xffffffffu, rescale)) {
        // O_h holds the earlier tiles of this half (their P V completed before
        // the S MMA of this tile was issued)
        const uint32_t o_tmem = tmem + lane_base + T::O_COL0 + h * D;
#pragma unroll
        for (int cc = 0; cc < D / 32; ++cc) {
          uint32_t orr[32];
          tmem_ld_32x32b_x32(o_tmem + cc * 32, orr);
#pragma unroll
          for (int e = 0; e < 32; ++e) orr[e] = __float_as_uint(__uint_as_float(orr[e]) * alpha);
          tmem_st_32x32b_x32(o_tmem + cc * 32, orr);
        }
      }
      tmem_wait_st();
      tc_fence_before_sync();
      __syncwarp();
      if (lane == 0) mbar_arrive(bars + 8 * (T_P_FULL + h));
      first = false;
    }
    if (!ok) break;
    if (h == 1) {
      // the second half's row statistics for the first warpgroup's combine
      if (run.n >= 2) {
        stat[L] = m_run;
        stat[128 + L] = l_exact;
        stat[256 + L] = l_round;
        __syncwarp();
        if (lane == 0) mbar_arrive(bars + 8 * T_HALF);
      }
      continue;
    }
    // ---- run epilogue (first warpgroup): combine the halves, write the output
    ok = wait(bars + 8 * (T_O_FULL + 0), o_ph[0]);
    if (!ok) break;
    o_ph[0] ^= 1u;
    const bool two = run.n >= 2;
    float m1 = -INFINITY, le1 = 0.f, lr1 = 0.f;
    if (two) {
      ok = wait(bars + 8 * (T_O_FULL + 1), o_ph[1]);
      if (!ok) break;
      o_ph[1] ^= 1u;
      ok = wait(bars + 8 * T_HALF, half_ph);
      if (!ok) break;
      half_ph ^= 1u;
      m1 = stat[L];
      le1 = stat[128 + L];
      lr1 = stat[256 + L];
    }
    tc_fence_after_sync();
    const float M = fmaxf(m_run, m1);
    const float Mr = (M == -INFINITY) ? 0.f : M;
    const float a0 = (m_run == -INFINITY) ? 0.f : fast_exp2(m_run - Mr);
    const float a1 = (m1 == -INFINITY) ? 0.f : fast_exp2(m1 - Mr);
    const float lr_t = l_round * a0 + lr1 * a1;
    const float le_t = l_exact * a0 + le1 * a1;
    const bool has = le_t > 0.f;
    const float inv = has ? 1.f / lr_t : 0.f;
    const float lse_nat = has ? (M + __log2f(le_t)) * 0.69314718055994531f : -INFINITY;
    const bool direct = run.n_parts == 1;
    if (!direct && run.part >= p.max_parts) {
      // cannot happen for the host's partition; refuse to write out of bounds
      if (threadIdx.x == 0) atomicExch(p.status, -4);
      continue;
    }
    const size_t slot = (static_cast<size_t>(run.g) * p.max_parts + run.part) * p.R + (real ? r : 0);
#pragma unroll
    for (int cc = 0; cc < D / 16; ++cc) {
      uint32_t o0[16], o1[16];
      tmem_ld_32x32b_x16(tmem + lane_base + T::O_COL0 + cc * 16, o0);
      if (two) tmem_ld_32x32b_x16(tmem + lane_base + T::O_COL0 + D + cc * 16, o1);
#pragma unroll
      for (int e = 0; e < 16; ++e) {
        const float x = __uint_as_float(o0[e]) * a0 + (two ? __uint_as_float(o1[e]) * a1 : 0.f);
        o0[e] = __float_as_uint(x * inv);
      }
      if (real) {
        if (direct) {
          if constexpr (OUT_F32) {
            float4* dst = reinterpret_cast<float4*>(static_cast<float*>(p.o) + row_idx * D + cc * 16);
#pragma unroll
            for (int e = 0; e < 4; ++e)
              dst[e] = make_float4(__uint_as_float(o0[4 * e]), __uint_as_float(o0[4 * e + 1]),
                                   __uint_as_float(o0[4 * e + 2]), __uint_as_float(o0[4 * e + 3]));
          } else {
            uint4* dst = reinterpret_cast<uint4*>(static_cast<uint16_t*>(p.o) + row_idx * D + cc * 16);
#pragma unroll
            for (int e = 0; e < 2; ++e)
              dst[e] = make_uint4(
                  pack2<BF16>(__uint_as_float(o0[8 * e]), __uint_as_float(o0[8 * e + 1])),
                  pack2<BF16>(__uint_as_float(o0[8 * e + 2]), __uint_as_float(o0[8 * e + 3])),
                  pack2<BF16>(__uint_as_float(o0[8 * e + 4]), __uint_as_float(o0[8 * e + 5])),
                  pack2<BF16>(__uint_as_float(o0[8 * e + 6]), __uint_as_float(o0[8 * e + 7])));
          }
        } else {
          float4* dst = reinterpret_cast<float4*>(p.ws_o + slot * D + cc * 16);
#pragma unroll
          for (int e = 0; e < 4; ++e)
            dst[e] = make_float4(__uint_as_float(o0[4 * e]), __uint_as_float(o0[4 * e + 1]),
                                 __uint_as_float(o0[4 * e + 2]), __uint_as_float(o0[4 * e + 3]));
        }
      }
    }
    if (real) {
      if (direct) {
        if (p.lse != nullptr) p.lse[row_idx] = lse_nat;
      } else {
        p.ws_lse[slot] = lse_nat;
      }
    }
    tc_fence_before_sync();
  }
}

template <int D, bool BF16, bool OUT_F32>
__global__ void __launch_bounds__(NUM_THREADS, 1)
attn_decode_tc_kernel(const __grid_constant__ CUtensorMap tmK, const __grid_constant__ CUtensorMap tmV,
                      const DecTcParams p) {
  using T = DtGeo<D>;
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~static_cast<uintptr_t>(1023));
  const uint32_t sbase = smem_addr(smem);
  const uint32_t bars = sbase + T::BAR_OFF;
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + T::BAR_OFF + DT_ABORT_OFF);
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + T::BAR_OFF + DT_TMEM_SLOT_OFF);
  const int warp = threadIdx.x / 32;
  const int lane = threadIdx.x % 32;
  if (threadIdx.x == 0) {
    for (int s = 0; s < T::NST; ++s) {
      mbar_init(bars + 8 * (T_K_FULL + s), 1);
      mbar_init(bars + 8 * (T_K_EMPTY + s), 1);
      mbar_init(bars + 8 * (T_V_FULL + s), 1);
      mbar_init(bars + 8 * (T_V_EMPTY + s), 1);
    }
    for (int h = 0; h < 2; ++h) {
      mbar_init(bars + 8 * (T_S_FULL + h), 1);
      mbar_init(bars + 8 * (T_P_FULL + h), 4);   // one arrival per softmax warp
      mbar_init(bars + 8 * (T_O_FULL + h), 1);
    }
    mbar_init(bars + 8 * T_Q_FULL, 4);
    mbar_init(bars + 8 * T_HALF, 4);
    mbar_init(bars + 8 * T_DRAIN, 1);
    *abort_flag = 0;
    fence_barrier_init();
  }
  if (warp == MMA_WARP) {
    tmem_alloc(smem_addr(tmem_slot), TMEM_COLS);
    tmem_relinquish();
  }
  if (warp == TMA_WARP && lane == 0) {
    tma_prefetch_desc(&tmK);
    tma_prefetch_desc(&tmV);
  }
  // The set-up above touches no global memory, so it may overlap the end of
  // the previous grid of the stream; nothing below runs before that grid is done.
  grid_dependency_wait();
  grid_launch_dependents();
  tc_fence_before_sync();
  __syncthreads();
  tc_fence_after_sync();
  const uint32_t tmem = *tmem_slot;
  if (warp < 8) {
    regs_increase<SOFTMAX_REGS>();
    dt_softmax_role<D, BF16, OUT_F32>(p, tmem, smem, sbase, bars, warp / 4, warp % 4, lane, abort_flag);
    tc_fence_before_sync();
    __syncthreads();
  } else {
    regs_decrease<CONTROL_REGS>();
    if (warp == MMA_WARP) {
      dt_mma_role<D, BF16>(p, tmem, sbase, bars, abort_flag);
    } else if (warp == TMA_WARP) {
      dt_tma_role<D>(p, &tmK, &tmV, sbase, bars, abort_flag);
    }
    tc_fence_before_sync();
    __syncthreads();
    if (warp == MMA_WARP) {
      tc_fence_after_sync();
      tmem_dealloc(tmem, TMEM_COLS);
    }
  }
}

// Merges the parts of every group covered by more than one run: one CTA per
// group, one thread per (query row, 4 output columns); every load of a
// thread is independent of the others.
template <int D, bool BF16, bool OUT_F32>
__global__ void __launch_bounds__(256)
attn_decode_tc_merge(const DecTcParams p) {
  const int g = blockIdx.x;
  const long long FT = static_cast<long long>(p.n_groups) * p.tiles;
  const int c_first = dt_cta_of(static_cast<long long>(g) * p.tiles, FT, p.grid);
  const int c_last = dt_cta_of(static_cast<long long>(g + 1) * p.tiles - 1, FT, p.grid);
  const int n_parts = c_last - c_first + 1;
  if (n_parts <= 1) return;
  const int b = g / p.H_kv, gk = g % p.H_kv;
  const int G_heads = p.H / p.H_kv;
  // launched behind the split kernel, whose partials it reads (through L2)
  grid_dependency_wait();
  for (int idx = threadIdx.x; idx < p.R * (D / 4); idx += blockDim.x) {
    const int r = idx / (D / 4), c4 = idx % (D / 4);
    const size_t row_idx = ((static_cast<size_t>(b) * p.H + gk * G_heads + r / p.N_q) * p.N_q) + r % p.N_q;
    const float* ls = p.ws_lse + static_cast<size_t>(g) * p.max_parts * p.R + r;   // stride R
    float mx = -INFINITY;
    for (int s = 0; s < n_parts; ++s) mx = fmaxf(mx, __ldcg(ls + static_cast<size_t>(s) * p.R));
    float tot = 0.f;
    for (int s = 0; s < n_parts; ++s) {
      const float l = __ldcg(ls + static_cast<size_t>(s) * p.R);
      tot += (l == -INFINITY) ? 0.f : __expf(l - mx);
    }
    const float lse_nat = (mx == -INFINITY) ? -INFINITY : mx + __logf(tot);
    float4 o = make_float4(0.f, 0.f, 0.f, 0.f);
    for (int s = 0; s < n_parts; ++s) {
      const size_t sl = (static_cast<size_t>(g) * p.max_parts + s) * p.R + r;
      const float l = __ldcg(p.ws_lse + sl);
      if (l == -INFINITY) continue;
      const float wgt = __expf(l - lse_nat);
      const float4 x = __ldcg(reinterpret_cast<const float4*>(p.ws_o + sl * D) + c4);
      o.x = fmaf(wgt, x.x, o.x);
      o.y = fmaf(wgt, x.y, o.y);
      o.z = fmaf(wgt, x.z, o.z);
      o.w = fmaf(wgt, x.w, o.w);
    }
    if constexpr (OUT_F32) {
      reinterpret_cast<float4*>(static_cast<float*>(p.o) + row_idx * D)[c4] = o;
    } else {
      uint2 w;
      w.x = pack2<BF16>(o.x, o.y);
      w.y = pack2<BF16>(o.z, o.w);
      reinterpret_cast<uint2*>(static_cast<uint16_t*>(p.o) + row_idx * D)[c4] = w;
    }
    if (c4 == 0 && p.lse != nullptr) p.lse[row_idx] = lse_nat;
  }
}

}  // namespace attn

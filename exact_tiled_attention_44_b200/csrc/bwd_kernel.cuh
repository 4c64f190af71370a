// bwd_kernel.cuh -- gradients of exact tiled attention for sm_100a.
//
// "USAAIO Lesson 91", slide 9: the Flash Attention 2 backward pass recomputes
// the attention tiles instead of reading a stored N x N matrix.  Per head,
// with the forward's saved LSE (natural log) and D_i = dO_i . O_i:
//   P_ij  = exp(scale q_i.k_j + bias_ij - LSE_i)   (0 where masked)
//   dV_j  = sum_i P_ij dO_i
//   dP_ij = dO_i . v_j
//   dS_ij = scale P_ij (dP_ij - D_i)
//   dK_j  = sum_i dS_ij q_i ,   dQ_i = sum_j dS_ij k_j
// (scale is folded into dS, so dK and dQ need no final multiply).
//
// Work unit: one 128-key tile j of one K/V head (b, g).  The CTA keeps K_j and
// V_j in shared memory and dK_j, dV_j in tensor memory, and walks every query
// tile i (of every query head that reads this K/V head) that keeps a pair
// with tile j.  dK and dV are therefore owned by one CTA and written once;
// dQ_i gets one 128 x d contribution per key tile, added to an fp32 buffer by
// TMA bulk reductions (coalesced vector atomics for d < 64).
//
// Per step (query head h, query tile i), all products 128 x 128 (x d):
//   MMA warp  S^T  = K_j Q_i^T           TMEM X (keys on lanes, queries on columns)
//             dP^T = V_j dO_i^T          TMEM Y
//   compute   P^T  = exp2(S^T c - LSE2)  16-bit over X;  fp32 copy kept in registers
//   MMA warp  dV  += P^T dO_i            (A from TMEM)
//   compute   dS^T = P^T (dP^T - D) scale   16-bit over Y, and into shared memory
//   MMA warp  dK  += dS^T Q_i            (A from TMEM)
//             dQ   = dS K_j              (A = dS from shared memory, MN-major)
//   compute   dQ rows (queries on lanes) -> bulk reductions into the fp32 dQ buffer
//
// CTA (384 threads): warps 0-7 compute (two warpgroups; warpgroup w takes query columns
// [64 w, 64 w + 64) of each tile and output columns [w d/2, (w+1) d/2)),
// warp 8 issues MMAs (converged warp, one elected lane), warp 9 loads tiles
// with TMA and the per-row statistics with plain loads, warps 10-11 idle.
#pragma once

#include "attn_kernel.cuh"

namespace attn {

constexpr int BW_THREADS = 384;         // three warpgroups; warps 10-11 only donate registers
constexpr int BW_MMA_WARP = 8;
constexpr int BW_TMA_WARP = 9;
constexpr int BW_COMPUTE_WARPS = 8;
// Register split after launch (launch: 384 x 168 = 64512): the compute
// warpgroups hold an fp32 row of P (64 values) next to a 64-column TMEM load.
constexpr uint32_t BW_COMPUTE_REGS = 200;
constexpr uint32_t BW_CONTROL_REGS = 104;
constexpr int BW_LAUNCH_REGS = 168;
static_assert(256 * BW_COMPUTE_REGS + 128 * BW_CONTROL_REGS <= BW_THREADS * BW_LAUNCH_REGS,
              "register split exceeds the launch allocation");
constexpr int STATUS_LAYOUT = -4;   // matches ATTN_ERR_CUDA: shared memory base not usable

struct BwdParams {
  const float* lse;    // [B*H*N] forward log-sum-exp (natural log)
  const float* dsum;   // [B*H*N] D_i = dO_i . O_i
  float* dq_acc;       // [B*H*N*d] fp32, zeroed before the launch
  void* dk;            // [B*H_kv*N*d] output dtype
  void* dv;
  int* status;
  unsigned long long watchdog_ns;
  int B, H, H_kv, N;
  int causal, window, n_sink;
  float scale_log2;    // scale * log2(e)
  float scale;
  int n_tiles;         // ceil(N / 128)
  int num_units;       // B * H_kv * ceil(n_tiles / 2) pair units
  const float* alibi;  // ALiBi slope per query head, or nullptr
  int smem_alloc;      // dynamic shared memory bytes given at launch
  int withhold_loads;  // test hook: the copy warp issues nothing, so every wait runs out
  unsigned long long* block_count;  // test hook: (key tile, query tile) steps are added here
};

template <int D>
struct BwGeo {
  using G = Geo<D>;
  static constexpr int K_OFF = 0;
  static constexpr int V_OFF = K_OFF + G::TILE_BYTES;
  static constexpr int Q_OFF = V_OFF + G::TILE_BYTES;        // [2] stages
  static constexpr int DO_OFF = Q_OFF + 2 * G::TILE_BYTES;   // [2] stages
  static constexpr int DS_OFF = DO_OFF + 2 * G::TILE_BYTES;
  // dS tile for the dQ product: key rows of 128 bytes, two 64-query chunks,
  // 128-byte swizzle (the MN-major operand layout).
  static constexpr int DS_CHUNK = 128 * 128;
  static constexpr int DS_BYTES = 2 * DS_CHUNK;
  // per stage: 128 floats -LSE*log2(e), then 128 floats -scale*D
  static constexpr int ST_OFF = DS_OFF + DS_BYTES;
  static constexpr int ST_BYTES = 2 * 128 * 4;
  static constexpr int BAR_OFF = ST_OFF + 2 * ST_BYTES;
  static constexpr int SMEM_BYTES = BAR_OFF + 256;
  static constexpr uint32_t DV_COL = 0;
  static constexpr uint32_t DK_COL = 128;
  static constexpr uint32_t X_COL = 256;
  static constexpr uint32_t Y_COL = 384;
  // dQ takes the free half of the dV block when it fits, else Y: dS^T there
  // is dead once the dK product (issued before dQ) has read it, and X stays
  // free for the next tile's S^T, which can then be issued right behind dQ
  // instead of after the dQ read-out; only the next dP^T waits for that.
  static constexpr uint32_t DQ_COL = D <= 64 ? 64 : Y_COL;
  static_assert(SMEM_BYTES <= 232448, "shared memory budget");
  static_assert(G::TILE_BYTES % 1024 == 0, "tiles must stay on swizzle-atom boundaries");
};

enum BwBar : int {
  W_KV_FULL = 0,
  W_KV_EMPTY,
  W_QD_FULL,                    // [2]
  W_QD_EMPTY = W_QD_FULL + 2,   // [2]
  W_S_FULL = W_QD_EMPTY + 2,
  W_DP_FULL,
  W_P_FULL,
  W_DS_FULL,
  W_DQ_FULL,
  W_DQ_FREE,
  W_ACC_FULL,
  W_ACC_FREE,
  W_DRAIN,
  W_COUNT
};
constexpr int BW_TMEM_SLOT_OFF = 8 * W_COUNT;
constexpr int BW_ABORT_FLAG_OFF = BW_TMEM_SLOT_OFF + 4;

// ------------------------------------------------------------ schedule

struct BwUnit {
  int b, g, j, i_lo, n_i, n_steps;
};

// Work is handed out in pair units: unit u covers key tiles j = pi and
// j = n_tiles - 1 - pi of K/V head (b, g), with bg = u / ceil(n_tiles / 2)
// and pi = u % ceil(n_tiles / 2).  Under causality the two tiles together are
// kept by n_tiles + 1 query tiles whatever pi is, so every unit costs the
// same; units are numbered head-major, so the CTAs running at one time share
// a few heads and their Q, dO and dQ rows stay in L2.  One CTA processes the
// two key tiles of its unit one after the other (the "halves").
// For key tile j the query tiles visited are i_lo .. i_lo + n_i - 1, the
// tiles holding a kept pair with it.  Causal: i >= j.  Window: a query keeps
// a key less than `window` positions behind it, so the last query tile holds
// query k0 + 127 + window - 1, unless the key tile holds sink keys (those are
// kept by every later query).  Returns false for the absent second half of a
// unit whose two tiles coincide (odd n_tiles).
__device__ __forceinline__ bool bw_unit(int u, int half, const BwdParams& p, BwUnit* out) {
  const int np = (p.n_tiles + 1) / 2;
  const int bg = u / np;
  const int pi = u % np;
  const int j = half ? p.n_tiles - 1 - pi : pi;
  if (half && j == pi) return false;
  BwUnit U;
  U.j = j;
  U.b = bg / p.H_kv;
  U.g = bg % p.H_kv;
  U.i_lo = p.causal ? U.j : 0;
  int i_hi = p.n_tiles - 1;
  if (p.window > 0 && U.j * BN >= p.n_sink)
    i_hi = min(i_hi, (U.j * BN + BN - 1 + p.window - 1) / BM);
  U.n_i = i_hi - U.i_lo + 1;
  U.n_steps = U.n_i * (p.H / p.H_kv);
  *out = U;
  return true;
}

// The CTA's key-tile tasks: task k is half k % 2 of the unit the CTA takes in
// round k / 2.  bw_task returns false for a task the CTA does not have.
__device__ __forceinline__ int bw_num_tasks(const BwdParams& p) {
  return 2 * num_rounds(gridDim.x, p.num_units);
}

__device__ __forceinline__ bool bw_task(int k, const BwdParams& p, BwUnit* U) {
  const int u = unit_of_round(k >> 1, blockIdx.x, gridDim.x, p.num_units);
  if (u < 0) return false;
  return bw_unit(u, k & 1, p, U);
}

__device__ __forceinline__ void bw_step(const BwUnit& U, const BwdParams& p, int n, int* hq, int* i) {
  const int G = p.H / p.H_kv;
  *hq = U.g * G + n / U.n_i;
  *i = U.i_lo + n % U.n_i;
}

// True when some (query, key) pair of query tile rows [q0, q0+128) x key
// tile [k0, k0+128) is dropped (padding, causality, window).
__device__ __forceinline__ bool bw_needs_mask(const BwdParams& p, int q0, int k0) {
  if (k0 + BN > p.N || q0 + BM > p.N) return true;
  if (p.causal && k0 + BN - 1 > q0) return true;
  if (p.window > 0 && !(q0 + BM - 1 - k0 < p.window) && !(k0 + BN <= p.n_sink)) return true;
  return false;
}

__device__ __forceinline__ bool bw_kept(const BwdParams& p, int q, int kt) {
  if (q >= p.N || kt >= p.N) return false;
  if (p.causal && kt > q) return false;
  if (p.window > 0 && !(q - kt < p.window || kt < p.n_sink)) return false;
  return true;
}

// ------------------------------------------------------------ waits

__device__ __forceinline__ bool bw_wait(uint32_t bar, uint32_t parity, volatile int* abort_flag,
                                        const BwdParams& p) {
  if (mbar_try_wait(bar, parity)) return true;
  return wait_slow(bar, parity, abort_flag, p.status, p.watchdog_ns);
}

__device__ __forceinline__ bool bw_warp_wait(uint32_t bar, uint32_t parity,
                                             volatile int* abort_flag, const BwdParams& p) {
  const bool ok = bw_wait(bar, parity, abort_flag, p);
  return __all_sync(0xffffffffu, ok);
}

// ------------------------------------------------------------ TMEM helpers

__device__ __forceinline__ void bw_tmem_ld_x8(uint32_t taddr, uint32_t (&r)[8]) {
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x8.b32 {%0, %1, %2, %3, %4, %5, %6, %7}, [%8];\n\t"
      "tcgen05.wait::ld.sync.aligned;\n"
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]),
        "=r"(r[7])
      : "r"(taddr)
      : "memory");
}

// W (8, 16 or 32) consecutive 32-bit columns of this thread's lane.
template <int W>
__device__ __forceinline__ void bw_tmem_ld(uint32_t taddr, uint32_t (&r)[W]) {
  if constexpr (W == 32) tmem_ld_32x32b_x32(taddr, r);
  else if constexpr (W == 16) tmem_ld_32x32b_x16(taddr, r);
  else bw_tmem_ld_x8(taddr, r);
}

// ------------------------------------------------------------ shared memory

__device__ __forceinline__ float4 bw_lds4(uint32_t addr) {
  float4 v;
  asm volatile("ld.shared.v4.f32 {%0, %1, %2, %3}, [%4];"
               : "=f"(v.x), "=f"(v.y), "=f"(v.z), "=f"(v.w)
               : "r"(addr)
               : "memory");
  return v;
}

__device__ __forceinline__ void bw_sts(uint32_t addr, float v) {
  asm volatile("st.shared.f32 [%0], %1;" ::"r"(addr), "f"(v) : "memory");
}

// ------------------------------------------------------------ bulk reduction

// Adds a box of fp32 values from shared memory into global memory (the TMA
// unit performs the read-modify-write in L2); completion is tracked per
// issuing thread by bulk groups.
__device__ __forceinline__ void bw_tma_reduce_add_3d(const CUtensorMap* map, uint32_t src, int x,
                                                     int y, int z) {
  asm volatile(
      "cp.reduce.async.bulk.tensor.3d.global.shared::cta.add.tile.bulk_group [%0, {%2, %3, %4}], [%1];"
      ::"l"(reinterpret_cast<uint64_t>(map)), "r"(src), "r"(x), "r"(y), "r"(z)
      : "memory");
}

__device__ __forceinline__ void bw_bulk_commit() {
  asm volatile("cp.async.bulk.commit_group;" ::: "memory");
}

// Waits until this thread's bulk operations have finished reading shared memory.
__device__ __forceinline__ void bw_bulk_wait_read() {
  asm volatile("cp.async.bulk.wait_group.read 0;" ::: "memory");
}

// Waits until this thread's bulk operations have completed.
__device__ __forceinline__ void bw_bulk_wait_all() {
  asm volatile("cp.async.bulk.wait_group 0;" ::: "memory");
}

// ------------------------------------------------------------ MMA issue

// kind::f16 instruction descriptor with both operand major-ness bits (bit 15:
// A MN-major, bit 16: B MN-major).
__host__ __device__ constexpr uint32_t bw_idesc(bool bf16, int m, int n, bool a_mn, bool b_mn) {
  return instr_desc(bf16, m, n, b_mn) | ((a_mn ? 1u : 0u) << 15);
}

// C[keys x queries] = A[keys x d] B[queries x d]^T; A, B are K-major 128 x D
// tiles (K_j with Q_i, or V_j with dO_i).
template <int D, bool BF16>
__device__ __forceinline__ void bw_issue_rowdot(uint32_t c_tmem, uint32_t a_base, uint32_t b_base) {
  using G = Geo<D>;
  constexpr uint32_t idesc = bw_idesc(BF16, BM, BN, false, false);
#pragma unroll
  for (int kk = 0; kk < D / 16; ++kk) {
    const uint32_t off = (kk * 16 / G::CW) * G::CHUNK_BYTES + ((kk * 16) % G::CW) * 2;
    const uint64_t da = smem_desc(a_base + off, 16, 8 * G::CB, G::LAYOUT);
    const uint64_t db = smem_desc(b_base + off, 16, 8 * G::CB, G::LAYOUT);
    mma_ss(c_tmem, da, db, idesc, kk > 0 ? 1u : 0u);
  }
}

// C[keys x d] (+)= T[keys x queries] B[queries x d]: T is 16-bit in TMEM with
// queries 0-63 packed at columns +0..31 and queries 64-127 at +64..95; B
// (dO_i or Q_i) is read MN-major from its K-major-loaded tile.
template <int D, bool BF16>
__device__ __forceinline__ void bw_issue_tmem_a(uint32_t c_tmem, uint32_t t_tmem, uint32_t b_base,
                                                bool accumulate) {
  using G = Geo<D>;
  constexpr uint32_t idesc = bw_idesc(BF16, BM, D, false, true);
#pragma unroll
  for (int kk = 0; kk < BM / 16; ++kk) {
    const uint32_t a = t_tmem + (kk >> 2) * 64 + (kk & 3) * 8;
    const uint64_t db = smem_desc(b_base + kk * 16 * G::CB, G::CHUNK_BYTES, 8 * G::CB, G::LAYOUT);
    mma_ts(c_tmem, a, db, idesc, (accumulate || kk > 0) ? 1u : 0u);
  }
}

// dQ[queries x d] = dS[queries x keys] K[keys x d]: dS from its shared-memory
// tile (key rows, MN-major), K_j MN-major.
template <int D, bool BF16>
__device__ __forceinline__ void bw_issue_dq(uint32_t c_tmem, uint32_t ds_base, uint32_t k_base) {
  using G = Geo<D>;
  using W = BwGeo<D>;
  constexpr uint32_t idesc = bw_idesc(BF16, BM, D, true, true);
#pragma unroll
  for (int kk = 0; kk < BN / 16; ++kk) {
    const uint64_t da = smem_desc(ds_base + kk * 16 * 128, W::DS_CHUNK, 8 * 128, 2u);
    const uint64_t db = smem_desc(k_base + kk * 16 * G::CB, G::CHUNK_BYTES, 8 * G::CB, G::LAYOUT);
    mma_ss(c_tmem, da, db, idesc, kk > 0 ? 1u : 0u);
  }
}

// ------------------------------------------------------------ roles

template <int D>
__device__ void bw_tma_role(const BwdParams& p, const CUtensorMap* tmQ, const CUtensorMap* tmK,
                            const CUtensorMap* tmV, const CUtensorMap* tmDO, uint8_t* smem,
                            uint32_t sbase, uint32_t bars, int lane, volatile int* abort_flag) {
  using G = Geo<D>;
  using W = BwGeo<D>;
  // Failure-detection test: no copy is issued, so the other roles' bounded
  // waits expire and the CTA reports ATTN_ERR_DEVICE_TIMEOUT and exits.
  if (p.withhold_loads) return;
  uint32_t st_it = 0;
  int ul = 0;
  int kv_last = -1, qd_last[2] = {-1, -1};
  bool ok = true;
  const int tasks = bw_num_tasks(p);
  for (int tk = 0; tk < tasks && ok; ++tk) {
    BwUnit U;
    if (!bw_task(tk, p, &U)) continue;
    const int kvz = U.b * p.H_kv + U.g;
    ok = bw_warp_wait(bars + 8 * W_KV_EMPTY, (ul & 1) ^ 1, abort_flag, p);
    if (!ok) break;
    if (elect_one()) {
      mbar_arrive_expect_tx(bars + 8 * W_KV_FULL, 2 * G::TILE_BYTES);
      for (int c = 0; c < G::NCH; ++c) {
        tma_load_3d(sbase + W::K_OFF + c * G::CHUNK_BYTES, tmK, bars + 8 * W_KV_FULL, c * G::CW,
                    U.j * BN, kvz);
        tma_load_3d(sbase + W::V_OFF + c * G::CHUNK_BYTES, tmV, bars + 8 * W_KV_FULL, c * G::CW,
                    U.j * BN, kvz);
      }
    }
    __syncwarp();
    kv_last = ul & 1;
    for (int n = 0; n < U.n_steps; ++n, ++st_it) {
      const int s = st_it & 1;
      const uint32_t ph = (st_it >> 1) & 1u;
      int hq, i;
      bw_step(U, p, n, &hq, &i);
      const int bh = U.b * p.H + hq;
      const int q0 = i * BM;
      // statistics of the tile's 128 query rows, loaded before the wait for
      // the stage so that their latency overlaps it; rows past N get LSE = +inf
      // (P = 0)
      float nl[4], dd[4];
#pragma unroll
      for (int k = 0; k < 4; ++k) {
        const int q = q0 + lane + 32 * k;
        nl[k] = INFINITY;
        dd[k] = 0.f;
        if (q < p.N) {
          const size_t idx = static_cast<size_t>(bh) * p.N + q;
          nl[k] = __ldg(p.lse + idx);
          dd[k] = __ldg(p.dsum + idx);
        }
      }
      ok = bw_warp_wait(bars + 8 * (W_QD_EMPTY + s), ph ^ 1u, abort_flag, p);
      if (!ok) break;
      if (elect_one()) {
        mbar_arrive_expect_tx(bars + 8 * (W_QD_FULL + s), 2 * G::TILE_BYTES);
        for (int c = 0; c < G::NCH; ++c) {
          tma_load_3d(sbase + W::Q_OFF + s * G::TILE_BYTES + c * G::CHUNK_BYTES, tmQ,
                      bars + 8 * (W_QD_FULL + s), c * G::CW, q0, bh);
          tma_load_3d(sbase + W::DO_OFF + s * G::TILE_BYTES + c * G::CHUNK_BYTES, tmDO,
                      bars + 8 * (W_QD_FULL + s), c * G::CW, q0, bh);
        }
      }
      __syncwarp();
      const uint32_t st = sbase + W::ST_OFF + s * W::ST_BYTES;
#pragma unroll
      for (int k = 0; k < 4; ++k) {
        bw_sts(st + 4 * (lane + 32 * k), -nl[k] * 1.4426950408889634f);
        bw_sts(st + 4 * (128 + lane + 32 * k), -p.scale * dd[k]);
      }
      // every lane's statistics stores are released by its own arrival
      mbar_arrive(bars + 8 * (W_QD_FULL + s));
      qd_last[s] = static_cast<int>(ph);
    }
    ++ul;
  }
  if (!ok) {
    const unsigned long long lim = p.watchdog_ns;
    if (kv_last >= 0) drain_wait(bars + 8 * W_KV_FULL, kv_last, lim);
    for (int s = 0; s < 2; ++s)
      if (qd_last[s] >= 0) drain_wait(bars + 8 * (W_QD_FULL + s), qd_last[s], lim);
  }
}

template <int D, bool BF16>
__device__ void bw_mma_role(const BwdParams& p, uint32_t tmem, uint32_t sbase, uint32_t bars,
                            volatile int* abort_flag) {
  using G = Geo<D>;
  using W = BwGeo<D>;
  uint32_t st_it = 0, p_ph = 0, ds_ph = 0, dqf_ph = 0, accf_ph = 0;
  unsigned long long n_steps = 0;   // steps issued, for the test hook
  bool any_dq = false;
  bool ok = true;
  int ul = 0;
  const int tasks = bw_num_tasks(p);
  for (int tk = 0; tk < tasks && ok; ++tk) {
    BwUnit U;
    if (!bw_task(tk, p, &U)) continue;
    ok = bw_warp_wait(bars + 8 * W_KV_FULL, ul & 1, abort_flag, p);
    if (!ok) break;
    for (int n = 0; n < U.n_steps; ++n, ++st_it) {
      const int s = st_it & 1;
      const uint32_t ph = (st_it >> 1) & 1u;
      const uint32_t qa = sbase + W::Q_OFF + s * G::TILE_BYTES;
      const uint32_t da = sbase + W::DO_OFF + s * G::TILE_BYTES;
      ok = bw_warp_wait(bars + 8 * (W_QD_FULL + s), ph, abort_flag, p);
      if (!ok) break;
      tc_fence_after_sync();
      if (elect_one()) {
        bw_issue_rowdot<D, BF16>(tmem + W::X_COL, sbase + W::K_OFF, qa);
        mma_commit(bars + 8 * W_S_FULL);
      }
      __syncwarp();
      if (W::DQ_COL == W::Y_COL && any_dq) {
        // dP^T overwrites the previous dQ: wait until it has been read out
        ok = bw_warp_wait(bars + 8 * W_DQ_FREE, dqf_ph, abort_flag, p);
        if (!ok) break;
        dqf_ph ^= 1u;
        tc_fence_after_sync();
      }
      if (elect_one()) {
        bw_issue_rowdot<D, BF16>(tmem + W::Y_COL, sbase + W::V_OFF, da);
        mma_commit(bars + 8 * W_DP_FULL);
      }
      __syncwarp();
      ok = bw_warp_wait(bars + 8 * W_P_FULL, p_ph, abort_flag, p);
      if (!ok) break;
      p_ph ^= 1u;
      if (n == 0 && ul > 0) {
        // the previous unit's dK / dV have been read out
        ok = bw_warp_wait(bars + 8 * W_ACC_FREE, accf_ph, abort_flag, p);
        if (!ok) break;
        accf_ph ^= 1u;
      }
      tc_fence_after_sync();
      if (elect_one()) bw_issue_tmem_a<D, BF16>(tmem + W::DV_COL, tmem + W::X_COL, da, n > 0);
      __syncwarp();
      ok = bw_warp_wait(bars + 8 * W_DS_FULL, ds_ph, abort_flag, p);
      if (!ok) break;
      ds_ph ^= 1u;
      if (W::DQ_COL != W::Y_COL && any_dq) {
        ok = bw_warp_wait(bars + 8 * W_DQ_FREE, dqf_ph, abort_flag, p);
        if (!ok) break;
        dqf_ph ^= 1u;
      }
      tc_fence_after_sync();
      if (elect_one()) {
        bw_issue_tmem_a<D, BF16>(tmem + W::DK_COL, tmem + W::Y_COL, qa, n > 0);
        bw_issue_dq<D, BF16>(tmem + W::DQ_COL, sbase + W::DS_OFF, sbase + W::K_OFF);
        mma_commit(bars + 8 * W_DQ_FULL);
        mma_commit(bars + 8 * (W_QD_EMPTY + s));
      }
      __syncwarp();
      any_dq = true;
      ++n_steps;
    }
    if (!ok) break;
    if (elect_one()) {
      mma_commit(bars + 8 * W_ACC_FULL);
      mma_commit(bars + 8 * W_KV_EMPTY);
    }
    __syncwarp();
    ++ul;
  }
  if (p.block_count != nullptr) {
    if (elect_one()) atomicAdd(p.block_count, n_steps);
    __syncwarp();
  }
  if (elect_one()) mma_commit(bars + 8 * W_DRAIN);
  __syncwarp();
  drain_wait(bars + 8 * W_DRAIN, 0, p.watchdog_ns);
}

// Writes HD consecutive values of one row, fp32 or 16-bit.
template <int HD, bool BF16, bool OUT_F32>
__device__ __forceinline__ void bw_store_row(void* base, size_t off, const uint32_t (&v)[HD]) {
  if constexpr (OUT_F32) {
    float* dst = reinterpret_cast<float*>(base) + off;
#pragma unroll
    for (int e = 0; e < HD; e += 4)
      *reinterpret_cast<float4*>(dst + e) =
          make_float4(__uint_as_float(v[e]), __uint_as_float(v[e + 1]), __uint_as_float(v[e + 2]),
                      __uint_as_float(v[e + 3]));
  } else {
    uint16_t* dst = reinterpret_cast<uint16_t*>(base) + off;
#pragma unroll
    for (int e = 0; e < HD; e += 8)
      *reinterpret_cast<uint4*>(dst + e) = make_uint4(
          pack2<BF16>(__uint_as_float(v[e]), __uint_as_float(v[e + 1])),
          pack2<BF16>(__uint_as_float(v[e + 2]), __uint_as_float(v[e + 3])),
          pack2<BF16>(__uint_as_float(v[e + 4]), __uint_as_float(v[e + 5])),
          pack2<BF16>(__uint_as_float(v[e + 6]), __uint_as_float(v[e + 7])));
  }
}

template <int D, bool BF16, bool OUT_F32, bool ALIBI>
__device__ void bw_compute_role(const BwdParams& p, const CUtensorMap* tmDQ, uint32_t tmem,
                                uint32_t sbase, uint32_t bars, int wg, int w4, int lane,
                                volatile int* abort_flag) {
  using W = BwGeo<D>;
  constexpr int HD = D / 2;               // output columns of this warpgroup
  constexpr int OC = HD < 32 ? HD : 32;   // TMEM columns per load
  const int t = w4 * 32 + lane;           // TMEM lane
  const uint32_t lane_base = static_cast<uint32_t>(w4 * 32) << 16;
  const uint32_t x_t = tmem + lane_base + W::X_COL + 64 * wg;
  const uint32_t y_t = tmem + lane_base + W::Y_COL + 64 * wg;
  const uint32_t dq_t = tmem + lane_base + W::DQ_COL + wg * HD;
  const float c = p.scale_log2;
  const float2 c2 = make_float2(c, c);
  const float2 sc2 = make_float2(p.scale, p.scale);
  // dS tile row t (key), chunk wg (this warpgroup's 64 queries)
  const uint32_t ds_row = sbase + W::DS_OFF + wg * W::DS_CHUNK + t * 128;
  uint32_t st_it = 0, s_ph = 0, dp_ph = 0, dq_ph = 0, acc_ph = 0;
  bool stg_busy = false;   // a dQ bulk reduction may still read this warp's dS slice
  bool ok = true;
  const int tasks = bw_num_tasks(p);
  for (int tk = 0; tk < tasks && ok; ++tk) {
    BwUnit U;
    if (!bw_task(tk, p, &U)) continue;
    const int k0 = U.j * BN;
    const int kt = k0 + t;
    for (int n = 0; n < U.n_steps; ++n, ++st_it) {
      const int s = st_it & 1;
      const uint32_t ph = (st_it >> 1) & 1u;
      int hq, i;
      bw_step(U, p, n, &hq, &i);
      const int q0 = i * BM;
      const int qc = q0 + 64 * wg;           // first query of this warpgroup's columns
      const bool masked = bw_needs_mask(p, q0, k0);
      const uint32_t nl = sbase + W::ST_OFF + s * W::ST_BYTES + 4 * 64 * wg;   // -LSE log2(e)
      const uint32_t dd = nl + 4 * 128;                                        // -scale D
      ok = bw_warp_wait(bars + 8 * (W_QD_FULL + s), ph, abort_flag, p);
      if (!ok) break;
      ok = bw_warp_wait(bars + 8 * W_S_FULL, s_ph, abort_flag, p);
      if (!ok) break;
      s_ph ^= 1u;
      tc_fence_after_sync();
      uint32_t sr[64];
      tmem_ld_32x32b_x64(x_t, sr);
      float pv[64];
      if (!masked && !ALIBI) {
#pragma unroll
        for (int e = 0; e < 64; e += 4) {
          const float4 l4 = bw_lds4(nl + 4 * e);
          const float2 a = fma2(make_float2(__uint_as_float(sr[e]), __uint_as_float(sr[e + 1])), c2,
                                make_float2(l4.x, l4.y));
          const float2 b = fma2(make_float2(__uint_as_float(sr[e + 2]), __uint_as_float(sr[e + 3])),
                                c2, make_float2(l4.z, l4.w));
          pv[e] = fast_exp2(a.x);
          pv[e + 1] = fast_exp2(a.y);
          pv[e + 2] = fast_exp2(b.x);
          pv[e + 3] = fast_exp2(b.y);
        }
      } else {
        const float slope2 = ALIBI ? p.alibi[hq] * 1.4426950408889634f : 0.f;
        const float rel = static_cast<float>(qc - kt);   // (query - key) at column 0, exact
        float nle[4];
#pragma unroll
        for (int e = 0; e < 64; ++e) {
          if ((e & 3) == 0) {
            const float4 l4 = bw_lds4(nl + 4 * e);
            nle[0] = l4.x; nle[1] = l4.y; nle[2] = l4.z; nle[3] = l4.w;
          }
          float x = fmaf(__uint_as_float(sr[e]), c, nle[e & 3]);
          if constexpr (ALIBI) x = fmaf(-slope2, fabsf(rel + static_cast<float>(e)), x);
          if (masked && !bw_kept(p, qc + e, kt)) x = -INFINITY;
          pv[e] = fast_exp2(x);
        }
      }
      {
        uint32_t pk[32];
#pragma unroll
        for (int e = 0; e < 32; ++e) pk[e] = pack2<BF16>(pv[2 * e], pv[2 * e + 1]);
        tmem_st_32x32b_x32(x_t, pk);
      }
      tmem_wait_st();
      tc_fence_before_sync();
      __syncwarp();
      if (lane == 0) mbar_arrive(bars + 8 * W_P_FULL);

      ok = bw_warp_wait(bars + 8 * W_DP_FULL, dp_ph, abort_flag, p);
      if (!ok) break;
      dp_ph ^= 1u;
      tc_fence_after_sync();
      tmem_ld_32x32b_x64(y_t, sr);
      {
        uint32_t pk[32];
#pragma unroll
        for (int e = 0; e < 64; e += 4) {
          const float4 d4 = bw_lds4(dd + 4 * e);
          // dS = P (scale dP - scale D)
          const float2 ta = fma2(make_float2(__uint_as_float(sr[e]), __uint_as_float(sr[e + 1])),
                                 sc2, make_float2(d4.x, d4.y));
          const float2 tb = fma2(make_float2(__uint_as_float(sr[e + 2]), __uint_as_float(sr[e + 3])),
                                 sc2, make_float2(d4.z, d4.w));
          const float2 ga = mul2(make_float2(pv[e], pv[e + 1]), ta);
          const float2 gb = mul2(make_float2(pv[e + 2], pv[e + 3]), tb);
          pk[e / 2] = pack2<BF16>(ga.x, ga.y);
          pk[e / 2 + 1] = pack2<BF16>(gb.x, gb.y);
        }
        tmem_st_32x32b_x32(y_t, pk);
        // the warp's slice of the dS tile may still be read by its last dQ
        // bulk reduction
        if (stg_busy) {
          if (lane == 0) bw_bulk_wait_read();
          __syncwarp();
          stg_busy = false;
        }
        // the same 64 values into the dS tile: 8 16-byte units, 128-byte swizzle
#pragma unroll
        for (int un = 0; un < 8; ++un)
          st_shared_v4(ds_row + ((un ^ (t & 7)) << 4), pk[4 * un], pk[4 * un + 1], pk[4 * un + 2],
                       pk[4 * un + 3]);
      }
      tmem_wait_st();
      fence_proxy_async_smem();
      tc_fence_before_sync();
      __syncwarp();
      if (lane == 0) {
        mbar_arrive(bars + 8 * W_DS_FULL);
        mbar_arrive(bars + 8 * (W_QD_EMPTY + s));
      }

      // dQ rows: lane t now holds query q0 + t
      ok = bw_warp_wait(bars + 8 * W_DQ_FULL, dq_ph, abort_flag, p);
      if (!ok) break;
      dq_ph ^= 1u;
      tc_fence_after_sync();
      if constexpr (OC == 32) {
        // Each warp stages its 32 rows x 32 columns of dQ in its own 4 KB slice
        // of the dS tile (rows 32 w4 .. 32 w4 + 31 of chunk wg, free once the
        // dQ product has read it) in the 128-byte swizzle of the dQ tensor map,
        // and one lane adds the box to the fp32 dQ buffer with a TMA bulk
        // reduction.  The lane waits for the box to be read out of shared
        // memory only before the slice is written again.
        const uint32_t stg = ds_row - lane * 128;
        const int r0 = q0 + w4 * 32;
#pragma unroll
        for (int cc = 0; cc < HD / OC; ++cc) {
          uint32_t v[OC];
          bw_tmem_ld<OC>(dq_t + cc * OC, v);
          if (stg_busy) {
            if (lane == 0) bw_bulk_wait_read();
            __syncwarp();
            stg_busy = false;
          }
#pragma unroll
          for (int un = 0; un < 8; ++un)
            st_shared_v4(stg + lane * 128 + ((un ^ (lane & 7)) << 4), v[4 * un], v[4 * un + 1],
                         v[4 * un + 2], v[4 * un + 3]);
          fence_proxy_async_smem();
          __syncwarp();
          if (r0 < p.N) {
            if (lane == 0) {
              bw_tma_reduce_add_3d(tmDQ, stg, wg * HD + cc * OC, r0, U.b * p.H + hq);
              bw_bulk_commit();
            }
            stg_busy = true;
          }
        }
      } else {
        // Narrow heads: each warp turns its 32 rows x OC columns around
        // through its own slice of the dS tile, so that the atomic adds of one
        // instruction cover whole rows instead of 16 bytes of 32 rows.
        constexpr int UPR = OC / 4;          // 16-byte units per staged row
        constexpr int RPI = 32 / UPR;        // rows per read-back instruction
        const uint32_t stg = ds_row - lane * 128;   // this warp's slice
        const size_t row0 = static_cast<size_t>(U.b * p.H + hq) * p.N + q0 + w4 * 32;
#pragma unroll
        for (int cc = 0; cc < HD / OC; ++cc) {
          uint32_t v[OC];
          bw_tmem_ld<OC>(dq_t + cc * OC, v);
#pragma unroll
          for (int un = 0; un < UPR; ++un)
            st_shared_v4(stg + lane * (OC * 4) + ((un ^ (lane & (UPR - 1))) << 4), v[4 * un],
                         v[4 * un + 1], v[4 * un + 2], v[4 * un + 3]);
          __syncwarp();
#pragma unroll
          for (int k = 0; k < UPR; ++k) {
            const int r = k * RPI + lane / UPR;
            const int un = lane % UPR;
            const float4 x = bw_lds4(stg + r * (OC * 4) + ((un ^ (r & (UPR - 1))) << 4));
            if (q0 + w4 * 32 + r < p.N)
              atomicAdd(reinterpret_cast<float4*>(p.dq_acc + (row0 + r) * D + wg * HD + cc * OC +
                                                  4 * un), x);
          }
          __syncwarp();
        }
      }
      tc_fence_before_sync();
      __syncwarp();
      if (lane == 0) mbar_arrive(bars + 8 * W_DQ_FREE);
    }
    if (!ok) break;
    // epilogue: dV and dK rows of key kt
    ok = bw_warp_wait(bars + 8 * W_ACC_FULL, acc_ph, abort_flag, p);
    if (!ok) break;
    acc_ph ^= 1u;
    tc_fence_after_sync();
    {
      const size_t off = (static_cast<size_t>(U.b * p.H_kv + U.g) * p.N + kt) * D + wg * HD;
#pragma unroll
      for (int cc = 0; cc < HD / OC; ++cc) {
        uint32_t v[OC];
        bw_tmem_ld<OC>(tmem + lane_base + W::DV_COL + wg * HD + cc * OC, v);
        if (kt < p.N) bw_store_row<OC, BF16, OUT_F32>(p.dv, off + cc * OC, v);
        bw_tmem_ld<OC>(tmem + lane_base + W::DK_COL + wg * HD + cc * OC, v);
        if (kt < p.N) bw_store_row<OC, BF16, OUT_F32>(p.dk, off + cc * OC, v);
      }
    }
    tc_fence_before_sync();
    __syncwarp();
    if (lane == 0) mbar_arrive(bars + 8 * W_ACC_FREE);
  }
  // the dQ reductions this warp issued complete before the CTA exits
  if (lane == 0) bw_bulk_wait_all();
  __syncwarp();
}

template <int D, bool BF16, bool OUT_F32, bool ALIBI>
__global__ void __launch_bounds__(BW_THREADS, 1)
attn_bwd_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
                const __grid_constant__ CUtensorMap tmV, const __grid_constant__ CUtensorMap tmDO,
                const __grid_constant__ CUtensorMap tmDQ, const BwdParams p) {
  using W = BwGeo<D>;
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  const uintptr_t raw = reinterpret_cast<uintptr_t>(smem_raw);
  const uintptr_t aligned = (raw + 1023) & ~static_cast<uintptr_t>(1023);
  // The layout needs a 1024-byte aligned base; the launch gives SMEM_BYTES
  // plus whatever slack fits, so check that the aligned layout is inside.
  if (static_cast<int>(aligned - raw) + W::SMEM_BYTES > p.smem_alloc) {
    if (threadIdx.x == 0) atomicExch(p.status, STATUS_LAYOUT);
    return;
  }
  uint8_t* smem = reinterpret_cast<uint8_t*>(aligned);
  const uint32_t sbase = smem_addr(smem);
  const uint32_t bars = sbase + W::BAR_OFF;
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + W::BAR_OFF + BW_ABORT_FLAG_OFF);
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + W::BAR_OFF + BW_TMEM_SLOT_OFF);
  const int warp = threadIdx.x / 32;
  const int lane = threadIdx.x % 32;

  if (threadIdx.x == 0) {
    mbar_init(bars + 8 * W_KV_FULL, 1);
    mbar_init(bars + 8 * W_KV_EMPTY, 1);
    for (int s = 0; s < 2; ++s) {
      mbar_init(bars + 8 * (W_QD_FULL + s), 1 + 32);                 // TMA + statistics lanes
      mbar_init(bars + 8 * (W_QD_EMPTY + s), 1 + BW_COMPUTE_WARPS);  // MMA commit + compute warps
    }
    mbar_init(bars + 8 * W_S_FULL, 1);
    mbar_init(bars + 8 * W_DP_FULL, 1);
    mbar_init(bars + 8 * W_P_FULL, BW_COMPUTE_WARPS);
    mbar_init(bars + 8 * W_DS_FULL, BW_COMPUTE_WARPS);
    mbar_init(bars + 8 * W_DQ_FULL, 1);
    mbar_init(bars + 8 * W_DQ_FREE, BW_COMPUTE_WARPS);
    mbar_init(bars + 8 * W_ACC_FULL, 1);
    mbar_init(bars + 8 * W_ACC_FREE, BW_COMPUTE_WARPS);
    mbar_init(bars + 8 * W_DRAIN, 1);
    *abort_flag = 0;
    fence_barrier_init();
  }
  if (warp == BW_MMA_WARP) {
    tmem_alloc(smem_addr(tmem_slot), TMEM_COLS);
    tmem_relinquish();
  }
  if (warp == BW_TMA_WARP && lane == 0) {
    tma_prefetch_desc(&tmQ);
    tma_prefetch_desc(&tmK);
    tma_prefetch_desc(&tmV);
    tma_prefetch_desc(&tmDO);
  }
  tc_fence_before_sync();
  __syncthreads();
  tc_fence_after_sync();
  const uint32_t tmem = *tmem_slot;

  // Each branch ends on its own copy of the final barrier (code shared by
  // warps under different register budgets would have to fit the smaller).
  if (warp < BW_COMPUTE_WARPS) {
    regs_increase<BW_COMPUTE_REGS>();
    bw_compute_role<D, BF16, OUT_F32, ALIBI>(p, &tmDQ, tmem, sbase, bars, warp / 4, warp % 4,
                                            lane, abort_flag);
    tc_fence_before_sync();
    __syncthreads();
  } else {
    regs_decrease<BW_CONTROL_REGS>();
    if (warp == BW_MMA_WARP) {
      bw_mma_role<D, BF16>(p, tmem, sbase, bars, abort_flag);
    } else if (warp == BW_TMA_WARP) {
      bw_tma_role<D>(p, &tmQ, &tmK, &tmV, &tmDO, smem, sbase, bars, lane, abort_flag);
    }
    tc_fence_before_sync();
    __syncthreads();
    if (warp == BW_MMA_WARP) {
      tc_fence_after_sync();
      tmem_dealloc(tmem, TMEM_COLS);
    }
  }
}

// D_i = dO_i . O_i per query row (fp32 accumulation of 16-bit inputs), and
// zeroes the row's fp32 dQ accumulator.  One warp per row.
template <int D, bool BF16>
__global__ void __launch_bounds__(256)
attn_bwd_prep_kernel(const void* __restrict__ o, const void* __restrict__ dout,
                     float* __restrict__ dsum, float* __restrict__ dq_acc, long long rows) {
  const long long row = static_cast<long long>(blockIdx.x) * 8 + threadIdx.x / 32;
  const int lane = threadIdx.x % 32;
  if (row >= rows) return;
  constexpr int PER = D / 32 < 2 ? 2 : D / 32;   // elements per lane (an even count)
  float acc = 0.f;
  if (lane * PER < D) {
    const uint16_t* a = reinterpret_cast<const uint16_t*>(o) + row * D + lane * PER;
    const uint16_t* b = reinterpret_cast<const uint16_t*>(dout) + row * D + lane * PER;
#pragma unroll
    for (int e = 0; e < PER; e += 2) {
      const uint32_t wa = *reinterpret_cast<const uint32_t*>(a + e);
      const uint32_t wb = *reinterpret_cast<const uint32_t*>(b + e);
      acc = fmaf(unpack_lo<BF16>(wa), unpack_lo<BF16>(wb), acc);
      acc = fmaf(unpack_hi<BF16>(wa), unpack_hi<BF16>(wb), acc);
    }
  }
#pragma unroll
  for (int off = 16; off > 0; off >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, off);
  if (lane == 0) dsum[row] = acc;
  if (dq_acc != nullptr) {
    float* z = dq_acc + row * D;
    for (int e = lane * 4; e < D; e += 128) *reinterpret_cast<float4*>(z + e) = make_float4(0.f, 0.f, 0.f, 0.f);
  }
}

// dQ (16-bit) from the fp32 accumulator; n4 = elements / 4.
template <bool BF16>
__global__ void __launch_bounds__(256)
attn_bwd_dq_convert_kernel(const float* __restrict__ acc, void* __restrict__ dq, long long n4) {
  for (long long k = static_cast<long long>(blockIdx.x) * blockDim.x + threadIdx.x; k < n4;
       k += static_cast<long long>(gridDim.x) * blockDim.x) {
    const float4 v = reinterpret_cast<const float4*>(acc)[k];
    reinterpret_cast<uint2*>(dq)[k] = make_uint2(pack2<BF16>(v.x, v.y), pack2<BF16>(v.z, v.w));
  }
}

}  // namespace attn

// attn_kernel.cuh -- exact tiled attention forward for sm_100a.
//
// What it computes (per batch b, query head h, kv head g = h / (H / H_kv)):
//   O = softmax(scale * Q K^T + mask) V  and  LSE = ln sum_kept exp(scale q.k),
// tile by tile with the online softmax of "Tiled attention with online
// softmax" (Lab 3) and "USAAIO Lesson 91" slide 11: per query row a running
// max m, a running denominator l and an output accumulator rescaled by
// exp(m_old - m_new) when the max grows; O is divided by l and written to HBM
// once at the end ("Flash Attention", dileepadev: "Write output once").  The
// N x N score matrix never leaves the chip: each 128 x 128 score tile lives in
// tensor memory (TMEM) only.
//
// Layout of one CTA (persistent; one CTA per SM, 384 threads):
//   warps 0-3  softmax warpgroup for Q tile 0 (TMEM lanes 0-127 = its rows)
//   warps 4-7  softmax warpgroup for Q tile 1
//   warp 8     MMA issue (whole warp, one elected lane issues) + TMEM allocation
//   warp 9     TMA producer (whole warp, one elected lane issues)
//   warps 10-11 idle (they hand their registers to the softmax warpgroups)
// A work unit is, by default, (b, h, a pair of adjacent 128-row Q tiles); for
// few heads and short sequences one Q tile whose K/V blocks the two softmax
// warpgroups share out, and for grouped heads with short rows the same 128
// rows of two query heads of one K/V head (see decode_unit).  Both tiles of a
// unit consume one K/V block stream, so every K/V block loaded from HBM feeds
// two 128 x 128 x d MMAs per GEMM.
//
// Per K/V block j and Q tile t:
//   MMA warp   S_t = Q_t K_j^T         (tcgen05.mma, A and B from smem, fp32 in TMEM)
//   softmax t  reads S_t row-per-thread (tcgen05.ld 32x32b), adds the ALiBi
//              bias -slope_h |i - j| when asked ("USAAIO Lesson 91", slides
//              20-23) folded into the raw scores, masks boundary blocks,
//              updates m and l, writes
//              P_t = exp2(s*scale*log2e - m)
//              as 16-bit over the first half of S_t's columns, and rescales
//              O_t in TMEM when the max grew by more than 2^8 (lazy rescale:
//              otherwise the stale max is kept; exact, because O and l share it)
//   MMA warp   O_t += P_t V_j          (tcgen05.mma, A from TMEM, B from smem)
// The MMA warp interleaves the two Q tiles so that one tile's softmax overlaps
// the other tile's MMAs.
#pragma once

#include <cuda_bf16.h>
#include <cuda_fp16.h>

#include "ptx.cuh"

namespace attn {

constexpr int UK_PAIR = 0, UK_SPLIT = 1, UK_HEADS = 2;   // work-unit kinds (see decode_unit)
constexpr int BM = 128;           // query rows per Q tile
constexpr int BN = 128;           // keys per K/V block
constexpr int NUM_STAGES = 2;     // K ring depth (and V ring depth)
constexpr int Q_SLOTS = 3;        // Q tile slots
constexpr int NUM_THREADS = 384;           // three warpgroups
constexpr int MMA_WARP = 8;
constexpr int TMA_WARP = 9;
// Register split after launch: the two softmax warpgroups grow to 192 per
// thread, the MMA/TMA warpgroup shrinks to 120 (both regions then compile
// without spills; at 88 the MMA issue loop spilled).  The launch must give
// every thread at least LAUNCH_REGS so that 256 * 192 + 128 * 120 fits the
// block's allocation (384 * 168 = 64512); the host checks this before launching.
constexpr uint32_t SOFTMAX_REGS = 192;
constexpr uint32_t CONTROL_REGS = 120;
constexpr int LAUNCH_REGS = 168;
static_assert(256 * SOFTMAX_REGS + 128 * CONTROL_REGS <= NUM_THREADS * LAUNCH_REGS,
              "register split exceeds the launch allocation");
constexpr float RESCALE_THRESHOLD = 8.0f;  // log2 units: rescale when the max grows by > 256x
constexpr uint32_t TMEM_COLS = 512;
constexpr int STATUS_TIMEOUT = -5;         // matches ATTN_ERR_DEVICE_TIMEOUT

struct KernelParams {
  void* o;
  float* lse;
  int* status;
  unsigned long long watchdog_ns;
  int B, H, H_kv, N;
  int causal, window, n_sink;
  float scale_log2;   // scale * log2(e)
  int n_qpairs;       // ceil(N / 256)
  int n_qtiles;       // ceil(N / 128)
  int n_hpairs;       // ceil(G / 2): pairs of query heads of one K/V head (G = H / H_kv)
  int n_kblocks;      // ceil(N / 128)
  int num_units;      // B * H * n_qpairs (pair units), B * H * n_qtiles (split units)
                      // or B * H_kv * n_hpairs * n_qtiles (head-pair units)
  const float* alibi; // ALiBi slope per query head ([H], device), used by the ALIBI kernels
  int withhold_loads; // test hook: the TMA warp issues nothing, so every wait runs out
  unsigned long long* block_count;  // test hook: S tiles computed are added here (or nullptr)
};

// Shared-memory geometry for head dimension D (16-bit elements).  A 128 x D
// tile is stored as D / CW column chunks of 128 rows x CB bytes, each chunk in
// the TMA / tcgen05 swizzle of span CB (32, 64 or 128 bytes).
template <int D>
struct Geo {
  static constexpr int CW = D < 64 ? D : 64;
  static constexpr int CB = CW * 2;
  static constexpr int NCH = D / CW;
  static constexpr int TILE_BYTES = 128 * D * 2;
  static constexpr int CHUNK_BYTES = 128 * CB;
  // descriptor layout field: 6 = 32B swizzle, 4 = 64B, 2 = 128B
  static constexpr uint32_t LAYOUT = CB == 128 ? 2u : (CB == 64 ? 4u : 6u);
  // Three Q tile slots rotate over the CTA's units (tile t of the CTA's u-th
  // unit uses slot (2u + t) % 3), so the next unit's tile 0 lands in a slot
  // that is free long before the current unit ends.
  static constexpr int Q_OFF = 0;
  static constexpr int K_OFF = Q_OFF + Q_SLOTS * TILE_BYTES;
  static constexpr int V_OFF = K_OFF + NUM_STAGES * TILE_BYTES;
  static constexpr int BAR_OFF = V_OFF + NUM_STAGES * TILE_BYTES;
  // split units: softmax warpgroup 1 hands (m, l_exact, l_round) of each row
  // to warpgroup 0, which merges the two halves
  static constexpr int STATS_OFF = BAR_OFF + 256;
  static constexpr int SMEM_BYTES = STATS_OFF + 128 * 12;
  static constexpr uint32_t S_COL0 = 0;      // S_t at column 128 t
  static constexpr uint32_t O_COL0 = 256;    // O_t at column 256 + D t
  static_assert(D % 16 == 0 && D <= 128, "unsupported head dim");
  static_assert(O_COL0 + 2 * D <= TMEM_COLS, "TMEM budget");
  static_assert(SMEM_BYTES + 1024 <= 232448, "shared memory budget");
};

// Barrier slots (8 bytes each) after the tiles.
enum BarSlot : int {
  B_Q_FULL = 0, B_Q_EMPTY = B_Q_FULL + Q_SLOTS,   // [Q_SLOTS] each
  B_K_FULL = B_Q_EMPTY + Q_SLOTS, B_K_EMPTY = B_K_FULL + NUM_STAGES,
  B_V_FULL = B_K_EMPTY + NUM_STAGES, B_V_EMPTY = B_V_FULL + NUM_STAGES,
  B_S_FULL = B_V_EMPTY + NUM_STAGES,   // [2]
  B_P_FULL = B_S_FULL + 2,             // [2]
  B_O_FULL = B_P_FULL + 2,             // [2]
  B_DRAIN = B_O_FULL + 2,
  B_EPI = B_DRAIN + 1,                 // [2] a tile's output rows are staged in shared memory
  B_HALF = B_EPI + 2,                  // split units: warpgroup 1's row statistics are written
  B_HALF_FREE = B_HALF + 1,            // split units: warpgroup 0 has read them and O_1
  B_COUNT = B_HALF_FREE + 1
};
constexpr int TMEM_SLOT_OFF = 8 * B_COUNT;
constexpr int ABORT_FLAG_OFF = TMEM_SLOT_OFF + 4;

// ------------------------------------------------------------ descriptors

// tcgen05 shared-memory matrix descriptor: start address, leading and stride
// byte offsets (16-byte units), fixed version bits 46-47 = 1, swizzle mode in
// bits 61-63.
__device__ __forceinline__ uint64_t smem_desc(uint32_t saddr, uint32_t lbo, uint32_t sbo,
                                              uint32_t layout) {
  return static_cast<uint64_t>((saddr & 0x3FFFFu) >> 4) |
         (static_cast<uint64_t>((lbo >> 4) & 0x3FFFu) << 16) |
         (static_cast<uint64_t>((sbo >> 4) & 0x3FFFu) << 32) |
         (1ull << 46) |
         (static_cast<uint64_t>(layout) << 61);
}

// kind::f16 instruction descriptor: fp32 accumulator (bits 4-5 = 1), A and B
// format (bits 7-9, 10-12: 0 = f16, 1 = bf16), B major-ness (bit 16: 1 = MN
// major), N / 8 (bits 17-22), M / 16 (bits 24-28).
__host__ __device__ constexpr uint32_t instr_desc(bool bf16, int m, int n, bool b_mn_major) {
  return (1u << 4) | ((bf16 ? 1u : 0u) << 7) | ((bf16 ? 1u : 0u) << 10) |
         ((b_mn_major ? 1u : 0u) << 16) | (static_cast<uint32_t>(n >> 3) << 17) |
         (static_cast<uint32_t>(m >> 4) << 24);
}

// ------------------------------------------------------------ schedule

// One work unit of head (b, h): two 128-row Q tiles t = 0, 1 (rows from q0;
// see decode_unit for the three kinds of unit).  Key blocks are iterated as a
// sink prefix [0, sb) followed by [wlo, hi_max); in pair and head-pair units
// Q tile t uses block j iff j < sb_t or lo_t <= j < hi_t.  Blocks holding no
// kept pair for a tile are skipped ("Tiled attention with online softmax":
// key blocks past the query block are not visited; exercise 4: sinks and a
// window).
struct Unit {
  int bh, b, h, g, q0;
  int n_active;
  int sb, wlo, n_iter;
  int sb0, lo0, hi0, sb1, lo1, hi1;   // per Q tile: sink prefix, window range
  int last0, last1;                   // per Q tile: the last block it visits
};

// REV: blocks are visited in descending order.  The forward does so under a
// position bias: the bias grows towards the diagonal, so the nearest keys come
// first and the running row max seldom has to move (each move rescales O).
//
// UK, the unit kind:
//   UK_PAIR  two consecutive 128-row Q tiles of one head (t = 0, 1);
//   UK_SPLIT one Q tile, and the two softmax warpgroups ("tiles" t = 0, 1
//            below) share its rows: t takes the visited blocks at even (t = 0)
//            or odd (t = 1) positions, with its own S_t, O_t and running
//            (m, l); warpgroup 0 merges the halves in the epilogue.  Used when
//            pair units would leave SMs idle (few heads, short sequences);
//   UK_HEADS the same 128 rows of two query heads h, h + 1 that share one K/V
//            head (GQA / MQA): every K/V block loaded feeds both tiles.
template <bool REV, int UK>
__device__ __forceinline__ Unit decode_unit(int u, const KernelParams& p) {
  constexpr bool SPLIT = UK == UK_SPLIT, HEADS = UK == UK_HEADS;
  static_assert(!(REV && SPLIT), "split units visit blocks in ascending order");
  Unit U;
  if constexpr (HEADS) {
    // Longest first by row position; within one, the head pairs of a K/V
    // head are adjacent, so the CTAs in flight share K/V blocks in L2.
    const int per_pos = p.B * p.H_kv * p.n_hpairs;
    const int pos = p.n_qtiles - 1 - u / per_pos;
    const int rem = u % per_pos;
    const int G = p.H / p.H_kv;
    U.b = rem / (p.H_kv * p.n_hpairs);
    U.g = (rem / p.n_hpairs) % p.H_kv;
    const int hp = rem % p.n_hpairs;
    U.h = U.g * G + 2 * hp;
    U.bh = U.b * p.H + U.h;
    U.q0 = pos * BM;
    U.n_active = (2 * hp + 1 < G) ? 2 : 1;
  } else {
    const int BH = p.B * p.H;
    // Longest-processing-time first: causal cost grows with the pair (tile)
    // index, so units are handed out from the last pair of every head down.
    const int pair = (SPLIT ? p.n_qtiles : p.n_qpairs) - 1 - u / BH;
    U.bh = u % BH;
    U.b = U.bh / p.H;
    U.h = U.bh % p.H;
    U.g = U.h / (p.H / p.H_kv);
    U.q0 = pair * (SPLIT ? 1 : 2) * BM;
    U.n_active = (!SPLIT && U.q0 + BM < p.N) ? 2 : 1;
  }
  const int sink_blocks = (p.window > 0) ? (p.n_sink + BN - 1) / BN : 0;
  int sb = 0, lo_min = 1 << 30, hi_max = 0;
#pragma unroll
  for (int t = 0; t < 2; ++t) {
    const int r0 = U.q0 + (UK == UK_PAIR ? t * BM : 0);
    const int r_last = min(r0 + BM - 1, p.N - 1);
    int lo = 0, hi = p.n_kblocks;
    if (p.causal) hi = min(p.n_kblocks, r_last / BN + 1);
    if (p.window > 0) {
      const int k_min = r0 - p.window + 1;
      lo = k_min > 0 ? k_min / BN : 0;
    }
    const int tsb = min(sink_blocks, hi);
    if (t == 0) {
      U.sb0 = tsb; U.lo0 = lo; U.hi0 = hi;
    } else {
      U.sb1 = tsb; U.lo1 = lo; U.hi1 = hi;
    }
    if (t < U.n_active) {
      sb = max(sb, tsb);
      lo_min = min(lo_min, lo);
      hi_max = max(hi_max, hi);
    }
  }
  U.sb = sb;
  U.wlo = max(lo_min, sb);
  U.n_iter = sb + max(0, hi_max - U.wlo);
  // Visited blocks: [0, sb) then [wlo, hi_max).  In ascending order a tile's
  // last block is hi - 1; in descending order it is its lowest visited block:
  // 0 with sink blocks, else lo (visited as a sink-prefix block when lo < sb,
  // otherwise from wlo on).
  U.last0 = REV ? (U.sb0 > 0 ? 0 : (U.lo0 < sb ? U.lo0 : max(U.lo0, U.wlo))) : U.hi0 - 1;
  U.last1 = REV ? (U.sb1 > 0 ? 0 : (U.lo1 < sb ? U.lo1 : max(U.lo1, U.wlo))) : U.hi1 - 1;
  if constexpr (SPLIT) {
    // every visited block holds kept keys of the tile's rows; the last even
    // and the last odd position (none for t = 1 when only one block is visited)
    const int i0 = (U.n_iter - 1) & ~1;
    const int i1 = (U.n_iter - 1) & 1 ? U.n_iter - 1 : U.n_iter - 2;
    U.last0 = i0 < U.sb ? i0 : U.wlo + (i0 - U.sb);
    U.last1 = i1 < 0 ? -1 : (i1 < U.sb ? i1 : U.wlo + (i1 - U.sb));
  }
  return U;
}

// Work units handed to CTA `cta` of `grid`: round r takes unit r*grid + cta
// on even rounds and r*grid + (grid - 1 - cta) on odd rounds.  With units in
// descending cost order this "snake" assignment evens out the per-CTA totals
// (plain round robin gives the low-numbered CTAs the larger unit of every
// round).  Returns -1 when the CTA has no unit in round r.
__device__ __forceinline__ int unit_of_round(int r, int cta, int grid, int num_units) {
  const int u = r * grid + ((r & 1) ? (grid - 1 - cta) : cta);
  return u < num_units ? u : -1;
}

__device__ __forceinline__ int num_rounds(int grid, int num_units) {
  return (num_units + grid - 1) / grid;
}

// Q slot of tile t in the CTA's ul-th unit.
__device__ __forceinline__ int q_slot(int ul, int t) { return (2 * ul + t) % Q_SLOTS; }

template <bool REV>
__device__ __forceinline__ int block_at(const Unit& U, int idx) {
  const int k = REV ? U.n_iter - 1 - idx : idx;
  return k < U.sb ? k : U.wlo + (k - U.sb);
}

// First query row and (batch, head) index of tile t's rows.
template <int UK>
__device__ __forceinline__ int tile_row0_k(const Unit& U, int t) {
  return U.q0 + (UK == UK_PAIR ? t * BM : 0);
}

template <int UK>
__device__ __forceinline__ int tile_bh_k(const Unit& U, int t) {
  return U.bh + (UK == UK_HEADS ? t : 0);
}

template <int UK>
__device__ __forceinline__ bool tile_uses(const Unit& U, int t, int j) {
  if constexpr (UK == UK_SPLIT) {
    const int idx = j < U.sb ? j : U.sb + (j - U.wlo);   // position of visited block j
    return (idx & 1) == t;
  }
  const int sb = t == 0 ? U.sb0 : U.sb1;
  const int lo = t == 0 ? U.lo0 : U.lo1;
  const int hi = t == 0 ? U.hi0 : U.hi1;
  return t < U.n_active && (j < sb || (j >= lo && j < hi));
}

__device__ __forceinline__ int tile_last_block(const Unit& U, int t) {
  return t == 0 ? U.last0 : U.last1;
}

// True when some (row, key) of Q tile rows [r0, r0+128) x keys [c0, c0+128)
// is masked, so the element mask must be applied.
__device__ __forceinline__ bool block_needs_mask(const KernelParams& p, int r0, int c0) {
  if (c0 + BN > p.N) return true;
  if (p.causal && c0 + BN - 1 > r0) return true;
  if (p.window > 0 && !(r0 + BM - 1 - c0 < p.window) && !(c0 + BN <= p.n_sink)) return true;
  return false;
}

__device__ __forceinline__ bool kept(const KernelParams& p, int i, int j) {
  if (j >= p.N) return false;
  if (p.causal && j > i) return false;
  if (p.window > 0 && !(i - j < p.window || j < p.n_sink)) return false;
  return true;
}

// ------------------------------------------------------------ watchdog wait

// Waits for `parity` on `bar`.  Gives up when another role has aborted or when
// the wait exceeds the watchdog limit; the first to time out records the
// status and raises the CTA's abort flag.  Returns false on give-up.
__device__ __forceinline__ bool wait_slow(uint32_t bar, uint32_t parity, volatile int* abort_flag,
                                       int* status, unsigned long long limit_ns) {
  const uint64_t t0 = global_timer_ns();
  for (uint32_t it = 1;; ++it) {
    if (mbar_try_wait(bar, parity)) return true;
    if ((it & 31u) == 0) {
      if (*abort_flag) return false;
      if (global_timer_ns() - t0 > limit_ns) {
        *abort_flag = 1;
        atomicExch(status, STATUS_TIMEOUT);
        return false;
      }
    }
  }
}

__device__ __forceinline__ bool wait_or_abort(uint32_t bar, uint32_t parity,
                                              volatile int* abort_flag, const KernelParams& p) {
  if (mbar_try_wait(bar, parity)) return true;
  return wait_slow(bar, parity, abort_flag, p.status, p.watchdog_ns);
}

// wait_or_abort for a whole converged warp; every lane gets the same verdict.
__device__ __forceinline__ bool warp_wait(uint32_t bar, uint32_t parity, volatile int* abort_flag,
                                          const KernelParams& p) {
  const bool ok = wait_or_abort(bar, parity, abort_flag, p);
  return __all_sync(0xffffffffu, ok);
}

// Bounded wait used while draining after an abort (no status update).
__device__ __forceinline__ void drain_wait(uint32_t bar, uint32_t parity,
                                           unsigned long long limit_ns) {
  const uint64_t t0 = global_timer_ns();
  while (!mbar_try_wait(bar, parity)) {
    if (global_timer_ns() - t0 > limit_ns) return;
  }
}

// Two floats -> one 32-bit word of two 16-bit values (round to nearest
// even), the first in the low half.
template <bool BF16>
__device__ __forceinline__ uint32_t pack2(float lo, float hi) {
  if constexpr (BF16) {
    __nv_bfloat162 h2 = __floats2bfloat162_rn(lo, hi);
    return *reinterpret_cast<uint32_t*>(&h2);
  } else {
    __half2 h2 = __floats2half2_rn(lo, hi);
    return *reinterpret_cast<uint32_t*>(&h2);
  }
}

template <bool BF16>
__device__ __forceinline__ float unpack_lo(uint32_t w) {
  if constexpr (BF16) return __uint_as_float(w << 16);
  else return __half2float(__ushort_as_half(static_cast<unsigned short>(w & 0xFFFFu)));
}

template <bool BF16>
__device__ __forceinline__ float unpack_hi(uint32_t w) {
  if constexpr (BF16) return __uint_as_float(w & 0xFFFF0000u);
  else return __half2float(__ushort_as_half(static_cast<unsigned short>(w >> 16)));
}

template <int W>
__device__ __forceinline__ void tmem_ld_cols(uint32_t taddr, uint32_t (&r)[W]) {
  if constexpr (W == 32) tmem_ld_32x32b_x32(taddr, r);
  else tmem_ld_32x32b_x16(taddr, r);
}

// Split units: o0 <- o0 w0 + o1 w1 over W columns, o1 read from TMEM at
// taddr1 when the other half holds a sum (has1), else o0 <- o0 w0.
template <int W>
__device__ __forceinline__ void merge_half(uint32_t (&o0)[W], uint32_t taddr1, bool has1, float w0,
                                           float w1) {
  if (has1) {
    uint32_t o1[W];
    tmem_ld_cols<W>(taddr1, o1);
#pragma unroll
    for (int e = 0; e < W; ++e)
      o0[e] = __float_as_uint(fmaf(__uint_as_float(o0[e]), w0, __uint_as_float(o1[e]) * w1));
  } else {
#pragma unroll
    for (int e = 0; e < W; ++e) o0[e] = __float_as_uint(__uint_as_float(o0[e]) * w0);
  }
}

template <int W>
__device__ __forceinline__ void tmem_st_cols(uint32_t taddr, const uint32_t (&r)[W]) {
  if constexpr (W == 32) tmem_st_32x32b_x32(taddr, r);
  else tmem_st_32x32b_x16(taddr, r);
  tmem_wait_st();
}

// ------------------------------------------------------------ roles

template <int D, bool REV, int UK>
__device__ void tma_role(const KernelParams& p, const CUtensorMap* tmQ, const CUtensorMap* tmK,
                         const CUtensorMap* tmV, uint32_t sbase, uint32_t bars,
                         volatile int* abort_flag) {
  using G = Geo<D>;
  // Failure-detection test: no copy is issued, so the other roles' bounded
  // waits expire and the CTA reports ATTN_ERR_DEVICE_TIMEOUT and exits.
  if (p.withhold_loads) return;
  uint32_t kv_it = 0;
  uint32_t q_loads[Q_SLOTS] = {0, 0, 0};
  // parity of the last load issued into each barrier, for the drain
  int q_last[Q_SLOTS], k_last[NUM_STAGES], v_last[NUM_STAGES];
  for (int s = 0; s < Q_SLOTS; ++s) q_last[s] = -1;
  for (int s = 0; s < NUM_STAGES; ++s) k_last[s] = v_last[s] = -1;
  bool ok = true;
  // one Q tile into its slot, once the MMAs that read the slot before are done
  auto load_q = [&](const Unit& U, int ul, int t) {
    const int qs = q_slot(ul, t);
    const uint32_t ph = q_loads[qs] & 1u;
    if (!warp_wait(bars + 8 * (B_Q_EMPTY + qs), ph ^ 1u, abort_flag, p)) return false;
    if (elect_one()) {
      mbar_arrive_expect_tx(bars + 8 * (B_Q_FULL + qs), G::TILE_BYTES);
      for (int c = 0; c < G::NCH; ++c)
        tma_load_3d(sbase + G::Q_OFF + qs * G::TILE_BYTES + c * G::CHUNK_BYTES, tmQ,
                    bars + 8 * (B_Q_FULL + qs), c * G::CW, tile_row0_k<UK>(U, t), tile_bh_k<UK>(U, t));
    }
    __syncwarp();
    q_last[qs] = static_cast<int>(ph);
    ++q_loads[qs];
    return true;
  };
  const int rounds = num_rounds(gridDim.x, p.num_units);
  int ul = 0;
  for (int r = 0; r < rounds && ok; ++r) {
    const int u = unit_of_round(r, blockIdx.x, gridDim.x, p.num_units);
    if (u < 0) continue;
    const Unit U = decode_unit<REV, UK>(u, p);
    // Loads in the order their ring stages and Q slots are released, so
    // that no load waits behind one whose slot frees later: Q tile 0 (its
    // slot was released by the unit before last), the first K block (whose
    // stage the unit before released one block before its end: the early
    // S_0 of this unit needs it), the first V block, then Q tile 1 (its slot
    // frees only when the unit before has issued its last S MMAs).
    ok = load_q(U, ul, 0);
    if (!ok) break;
    const int kvz = U.b * p.H_kv + U.g;
    for (int idx = 0; idx < U.n_iter; ++idx, ++kv_it) {
      const int j = block_at<REV>(U, idx);
      const int s = kv_it % NUM_STAGES;
      const uint32_t ph = (kv_it / NUM_STAGES) & 1u;
      ok = warp_wait(bars + 8 * (B_K_EMPTY + s), ph ^ 1u, abort_flag, p);
      if (!ok) break;
      if (elect_one()) {
        mbar_arrive_expect_tx(bars + 8 * (B_K_FULL + s), G::TILE_BYTES);
        for (int c = 0; c < G::NCH; ++c)
          tma_load_3d(sbase + G::K_OFF + s * G::TILE_BYTES + c * G::CHUNK_BYTES, tmK,
                      bars + 8 * (B_K_FULL + s), c * G::CW, j * BN, kvz);
      }
      __syncwarp();
      k_last[s] = ph;
      ok = warp_wait(bars + 8 * (B_V_EMPTY + s), ph ^ 1u, abort_flag, p);
      if (!ok) break;
      if (elect_one()) {
        mbar_arrive_expect_tx(bars + 8 * (B_V_FULL + s), G::TILE_BYTES);
        for (int c = 0; c < G::NCH; ++c)
          tma_load_3d(sbase + G::V_OFF + s * G::TILE_BYTES + c * G::CHUNK_BYTES, tmV,
                      bars + 8 * (B_V_FULL + s), c * G::CW, j * BN, kvz);
      }
      __syncwarp();
      v_last[s] = ph;
      if (idx == 0 && U.n_active > 1) {
        ok = load_q(U, ul, 1);
        if (!ok) break;
      }
    }
    ++ul;
  }
  if (!ok) {
    // Let every copy this warp started land before the CTA can exit.
    const unsigned long long lim = p.watchdog_ns;
    for (int s = 0; s < Q_SLOTS; ++s)
      if (q_last[s] >= 0) drain_wait(bars + 8 * (B_Q_FULL + s), q_last[s], lim);
    for (int s = 0; s < NUM_STAGES; ++s) {
      if (k_last[s] >= 0) drain_wait(bars + 8 * (B_K_FULL + s), k_last[s], lim);
      if (v_last[s] >= 0) drain_wait(bars + 8 * (B_V_FULL + s), v_last[s], lim);
    }
  }
}

template <int D, bool BF16>
__device__ __forceinline__ void issue_qk(uint32_t tmem, uint32_t sbase, int t, int qs, int stage) {
  using G = Geo<D>;
  constexpr uint32_t idesc = instr_desc(BF16, BM, BN, false);
  const uint32_t qa = sbase + G::Q_OFF + qs * G::TILE_BYTES;
  const uint32_t ka = sbase + G::K_OFF + stage * G::TILE_BYTES;
#pragma unroll
  for (int kk = 0; kk < D / 16; ++kk) {
    // K-major operands: 16 elements (32 bytes) per step inside a swizzle row;
    // the next chunk starts CHUNK_BYTES later.  Stride between 8-row groups is
    // 8 * CB; the leading offset is unused for swizzled K-major layouts.
    const uint32_t off = (kk * 16 / G::CW) * G::CHUNK_BYTES + ((kk * 16) % G::CW) * 2;
    const uint64_t da = smem_desc(qa + off, 16, 8 * G::CB, G::LAYOUT);
    const uint64_t db = smem_desc(ka + off, 16, 8 * G::CB, G::LAYOUT);
    mma_ss(tmem + Geo<D>::S_COL0 + t * BN, da, db, idesc, kk > 0 ? 1u : 0u);
  }
}

template <int D, bool BF16>
__device__ __forceinline__ void issue_pv(uint32_t tmem, uint32_t sbase, int t, int stage,
                                         bool accumulate) {
  using G = Geo<D>;
  constexpr uint32_t idesc = instr_desc(BF16, BM, D, true);
  const uint32_t va = sbase + G::V_OFF + stage * G::TILE_BYTES;
#pragma unroll
  for (int kk = 0; kk < BN / 16; ++kk) {
    // A = P: 16 keys per step = 8 packed 32-bit TMEM columns.
    // B = V, MN-major: 16 key rows per step (16 * CB bytes); 8-row groups are
    // 8 * CB apart (stride offset); column chunks are CHUNK_BYTES apart
    // (leading offset).
    const uint64_t db = smem_desc(va + kk * 16 * G::CB, G::CHUNK_BYTES, 8 * G::CB, G::LAYOUT);
    mma_ts(tmem + G::O_COL0 + t * D, tmem + G::S_COL0 + t * BN + kk * 8, db, idesc,
           (accumulate || kk > 0) ? 1u : 0u);
  }
}

template <int D, bool BF16, bool REV, int UK>
__device__ void mma_role(const KernelParams& p, uint32_t tmem, uint32_t sbase, uint32_t bars,
                         volatile int* abort_flag) {
  constexpr bool SPLIT = UK == UK_SPLIT;
  uint32_t kv_it = 0, p_ph[2] = {0, 0};
  uint32_t q_uses[Q_SLOTS] = {0, 0, 0};
  unsigned long long n_s = 0;   // (Q tile, K/V block) score tiles issued, for the test hook
  bool ok = true;
  const int rounds = num_rounds(gridDim.x, p.num_units);
  int ul = 0;
  // S_0 of a unit's first block may already have been issued at the end of
  // the unit before (see below); its Q tile 0 has then been waited for too.
  bool s0_pre = false;
  for (int r = 0; r < rounds && ok; ++r) {
    const int u = unit_of_round(r, blockIdx.x, gridDim.x, p.num_units);
    if (u < 0) continue;
    const Unit U = decode_unit<REV, UK>(u, p);
    // split units: both tiles read the unit's one Q tile
    const int qs0 = q_slot(ul, 0), qs1 = SPLIT ? qs0 : q_slot(ul, 1);
    auto wait_q = [&](int qs) {
      if (!warp_wait(bars + 8 * (B_Q_FULL + qs), q_uses[qs] & 1u, abort_flag, p)) return false;
      ++q_uses[qs];
      tc_fence_after_sync();
      return true;
    };
    // Q tile t is waited for before its first S MMA of the unit
    bool q_ready[2] = {s0_pre, false};
    const bool this_s0_pre = s0_pre;
    s0_pre = false;
    auto need_q = [&](int t) {
      const int tq = SPLIT ? 0 : t;
      if (q_ready[tq]) return true;
      if (!wait_q(tq == 0 ? qs0 : qs1)) return false;
      q_ready[tq] = true;
      return true;
    };
    // the CTA's next unit, for issuing its first S_0 early
    int u_next = -1;
    for (int r2 = r + 1; r2 < rounds && u_next < 0; ++r2)
      u_next = unit_of_round(r2, blockIdx.x, gridDim.x, p.num_units);
    // prologue: S_t for the first block
    {
      const int j0 = block_at<REV>(U, 0);
      const int s = kv_it % NUM_STAGES;
      ok = warp_wait(bars + 8 * (B_K_FULL + s), (kv_it / NUM_STAGES) & 1u, abort_flag, p);
      if (!ok) break;
      tc_fence_after_sync();
      for (int t = 0; t < 2 && ok; ++t) {
        if (!tile_uses<UK>(U, t, j0)) continue;
        if (t == 0 && this_s0_pre) continue;        // issued at the end of the unit before
        ok = need_q(t);
        if (!ok) break;
        if (elect_one()) {
          issue_qk<D, BF16>(tmem, sbase, t, t == 0 ? qs0 : qs1, s);
          mma_commit(bars + 8 * (B_S_FULL + t));
        }
        __syncwarp();
        ++n_s;
      }
      if (!ok) break;
      if (elect_one()) {
        mma_commit(bars + 8 * (B_K_EMPTY + s));
        if (U.n_iter == 1) {
          mma_commit(bars + 8 * (B_Q_EMPTY + qs0));
          if (U.n_active > 1) mma_commit(bars + 8 * (B_Q_EMPTY + qs1));
        }
      }
      __syncwarp();
    }
    int pv_done[2] = {0, 0};
    if constexpr (SPLIT) {
      // Split unit: block idx belongs to tile t = idx & 1 and the next one to
      // the other tile, whose S does not wait for P_t: it is issued first, so
      // that the other warpgroup's softmax overlaps this one's.
      for (int idx = 0; idx < U.n_iter && ok; ++idx) {
        const int j = block_at<REV>(U, idx);
        const int t = idx & 1;
        const uint32_t it = kv_it + idx;
        const int s = it % NUM_STAGES;
        const bool has_next = idx + 1 < U.n_iter;
        if (has_next) {
          const uint32_t itn = it + 1;
          const int sn = itn % NUM_STAGES;
          ok = warp_wait(bars + 8 * (B_K_FULL + sn), (itn / NUM_STAGES) & 1u, abort_flag, p);
          if (!ok) break;
          tc_fence_after_sync();
          ok = need_q(1 - t);
          if (!ok) break;
          if (elect_one()) {
            // S_{1-t} overwrites P_{1-t} after the P_{1-t} V issued before it
            issue_qk<D, BF16>(tmem, sbase, 1 - t, qs0, sn);
            mma_commit(bars + 8 * (B_S_FULL + 1 - t));
            mma_commit(bars + 8 * (B_K_EMPTY + sn));
            if (idx + 2 == U.n_iter) mma_commit(bars + 8 * (B_Q_EMPTY + qs0));   // last S of the unit
          }
          __syncwarp();
          ++n_s;
        }
        ok = warp_wait(bars + 8 * (B_V_FULL + s), (it / NUM_STAGES) & 1u, abort_flag, p);
        if (!ok) break;
        ok = warp_wait(bars + 8 * (B_P_FULL + t), p_ph[t], abort_flag, p);
        if (!ok) break;
        p_ph[t] ^= 1u;
        tc_fence_after_sync();
        if (elect_one()) {
          issue_pv<D, BF16>(tmem, sbase, t, s, pv_done[t] > 0);
          if (j == tile_last_block(U, t)) mma_commit(bars + 8 * (B_O_FULL + t));
          mma_commit(bars + 8 * (B_V_EMPTY + s));
        }
        __syncwarp();
        ++pv_done[t];
        // Tile 0 done one block before the unit ends: issue the next unit's
        // first S_0 now (as for pair units below).
        if (t == 0 && !s0_pre && u_next >= 0 && idx + 2 == U.n_iter) {
          const uint32_t it2 = kv_it + U.n_iter;
          const int s2 = it2 % NUM_STAGES;
          ok = warp_wait(bars + 8 * (B_K_FULL + s2), (it2 / NUM_STAGES) & 1u, abort_flag, p);
          if (!ok) break;
          ok = wait_q(q_slot(ul + 1, 0));
          if (!ok) break;
          if (elect_one()) {
            issue_qk<D, BF16>(tmem, sbase, 0, q_slot(ul + 1, 0), s2);
            mma_commit(bars + 8 * (B_S_FULL + 0));
          }
          __syncwarp();
          ++n_s;
          s0_pre = true;
        }
      }
      kv_it += U.n_iter;
      ++ul;
      continue;
    }
    for (int idx = 0; idx < U.n_iter && ok; ++idx) {
      const int j = block_at<REV>(U, idx);
      const uint32_t it = kv_it + idx;
      const int s = it % NUM_STAGES;
      ok = warp_wait(bars + 8 * (B_V_FULL + s), (it / NUM_STAGES) & 1u, abort_flag, p);
      if (!ok) break;
      const bool has_next = idx + 1 < U.n_iter;
      const int jn = has_next ? block_at<REV>(U, idx + 1) : 0;
      const uint32_t itn = it + 1;
      const int sn = itn % NUM_STAGES;
      // Q tile 0: P0 V_j, then S0 for the next block
      if (tile_uses<UK>(U, 0, j)) {
        ok = warp_wait(bars + 8 * (B_P_FULL + 0), p_ph[0], abort_flag, p);
        if (!ok) break;
        p_ph[0] ^= 1u;
        tc_fence_after_sync();
        if (elect_one()) {
          issue_pv<D, BF16>(tmem, sbase, 0, s, pv_done[0] > 0);
          if (j == tile_last_block(U, 0)) mma_commit(bars + 8 * (B_O_FULL + 0));
        }
        __syncwarp();
        ++pv_done[0];
      }
      if (has_next) {
        ok = warp_wait(bars + 8 * (B_K_FULL + sn), (itn / NUM_STAGES) & 1u, abort_flag, p);
        if (!ok) break;
        tc_fence_after_sync();
        if (tile_uses<UK>(U, 0, jn)) {
          ok = need_q(0);
          if (!ok) break;
          if (elect_one()) {
            issue_qk<D, BF16>(tmem, sbase, 0, qs0, sn);
            mma_commit(bars + 8 * (B_S_FULL + 0));
          }
          __syncwarp();
          ++n_s;
        }
      }
      // Q tile 1: P1 V_j, then S1 for the next block
      if (tile_uses<UK>(U, 1, j)) {
        ok = warp_wait(bars + 8 * (B_P_FULL + 1), p_ph[1], abort_flag, p);
        if (!ok) break;
        p_ph[1] ^= 1u;
        tc_fence_after_sync();
        if (elect_one()) {
          issue_pv<D, BF16>(tmem, sbase, 1, s, pv_done[1] > 0);
          if (j == tile_last_block(U, 1)) mma_commit(bars + 8 * (B_O_FULL + 1));
        }
        __syncwarp();
        ++pv_done[1];
      }
      if (has_next && tile_uses<UK>(U, 1, jn)) {
        ok = need_q(1);
        if (!ok) break;
      }
      if (elect_one()) {
        mma_commit(bars + 8 * (B_V_EMPTY + s));
        if (has_next) {
          if (tile_uses<UK>(U, 1, jn)) {
            issue_qk<D, BF16>(tmem, sbase, 1, qs1, sn);
            mma_commit(bars + 8 * (B_S_FULL + 1));
          }
          mma_commit(bars + 8 * (B_K_EMPTY + sn));
          if (idx + 2 == U.n_iter) {
            // last S MMAs of the unit: both Q slots are free once they are done
            mma_commit(bars + 8 * (B_Q_EMPTY + qs0));
            if (U.n_active > 1) mma_commit(bars + 8 * (B_Q_EMPTY + qs1));
          }
        }
      }
      __syncwarp();
      if (has_next && tile_uses<UK>(U, 1, jn)) ++n_s;
      // Once Q tile 0 has no block left in this unit (its last P_0 V is
      // issued and no S_0 follows), its next S is the next unit's first one:
      // issue it now, so that softmax 0 finds it ready after its epilogue
      // instead of waiting for tile 1 to finish this unit.  S_0 overwrites
      // P_0 only after the P_0 V issued before it (the pipe runs in order).
      if (!s0_pre && u_next >= 0 && has_next && !tile_uses<UK>(U, 0, jn) && idx + 2 == U.n_iter) {
        const Unit UN = decode_unit<REV, UK>(u_next, p);
        const int jn0 = block_at<REV>(UN, 0);
        if (tile_uses<UK>(UN, 0, jn0)) {
          const uint32_t it2 = kv_it + U.n_iter;       // ring position of the next unit's first K
          const int s2 = it2 % NUM_STAGES;
          ok = warp_wait(bars + 8 * (B_K_FULL + s2), (it2 / NUM_STAGES) & 1u, abort_flag, p);
          if (!ok) break;
          ok = wait_q(q_slot(ul + 1, 0));
          if (!ok) break;
          if (elect_one()) {
            issue_qk<D, BF16>(tmem, sbase, 0, q_slot(ul + 1, 0), s2);
            mma_commit(bars + 8 * (B_S_FULL + 0));
          }
          __syncwarp();
          ++n_s;
          s0_pre = true;
        }
      }
    }
    kv_it += U.n_iter;
    ++ul;
  }
  if (p.block_count != nullptr) {
    if (elect_one()) atomicAdd(p.block_count, n_s);
    __syncwarp();
  }
  // Every MMA this warp issued has completed once the drain barrier flips.
  if (elect_one()) mma_commit(bars + 8 * B_DRAIN);
  __syncwarp();
  drain_wait(bars + 8 * B_DRAIN, 0, p.watchdog_ns);
}

template <int D, bool BF16, bool OUT_F32, bool ALIBI, int UK>
__device__ void softmax_role(const KernelParams& p, const CUtensorMap* tmO, uint32_t tmem,
                             uint32_t sbase, uint32_t bars, int t, int warp_in_wg, int lane,
                             volatile int* abort_flag) {
  constexpr bool SPLIT = UK == UK_SPLIT;
  using G = Geo<D>;
  constexpr int OC = D >= 32 ? 32 : 16;   // TMEM columns per O load/store
  const int row_in_tile = warp_in_wg * 32 + lane;
  const uint32_t lane_base = static_cast<uint32_t>(warp_in_wg * 32) << 16;
  const uint32_t s_tmem = tmem + lane_base + G::S_COL0 + t * BN;
  const uint32_t o_tmem = tmem + lane_base + G::O_COL0 + t * D;
  const uint32_t o1_tmem = tmem + lane_base + G::O_COL0 + D;   // split units: the other half's O
  // split units: warpgroup 1's (m, l_exact, l_round) for each row
  const uint32_t half_stats = sbase + G::STATS_OFF + 12 * row_in_tile;
  const float c = p.scale_log2;
  // 16-bit output rows of 128 bytes per 64-column chunk are staged in shared
  // memory and written by TMA; other outputs are stored from registers.
  constexpr bool STAGED = !OUT_F32 && G::CB == 128;
  uint32_t s_ph = 0, o_ph = 0, epi_ph = 0, half_ph = 0, o1_ph = 0;
  bool ok = true;
  int ul = -1;
  // Q_EMPTY barrier of the slot whose staged output a TMA store issued by
  // this thread (warp 0, lane 0) may still be reading, or 0.  The wait is
  // deferred to the next S wait, where the warp would idle anyway.
  uint32_t staged_slot = 0;
  auto release_stage = [&]() {
    if (STAGED && staged_slot != 0) {
      bulk_wait_group_read0();
      mbar_arrive(staged_slot);
      staged_slot = 0;
    }
  };
  const int rounds = num_rounds(gridDim.x, p.num_units);
  for (int r = 0; r < rounds && ok; ++r) {
    const int u = unit_of_round(r, blockIdx.x, gridDim.x, p.num_units);
    if (u < 0) continue;
    ++ul;
    const Unit U = decode_unit<ALIBI, UK>(u, p);
    if (!SPLIT && t >= U.n_active) continue;
    const int r0 = tile_row0_k<UK>(U, t);
    const int bh = tile_bh_k<UK>(U, t);
    if (SPLIT && t == 1 && ul > 0) {
      // O_1 and the row statistics of the CTA's previous unit must have been
      // read by warpgroup 0 before this unit's first P_1 V overwrites O_1
      ok = warp_wait(bars + 8 * B_HALF_FREE, (ul - 1) & 1u, abort_flag, p);
      if (!ok) break;
    }
    const int row = r0 + row_in_tile;
    // ALiBi slope of this query head in log2 units (the logits are kept in
    // units of log2 so that exp2 can be used)
    const float slope2 = ALIBI ? p.alibi[U.h + (UK == UK_HEADS ? t : 0)] * 1.4426950408889634f : 0.f;
    float m_run = -INFINITY, l_exact = 0.f, l_round = 0.f;
    bool first = true;
    for (int idx = 0; idx < U.n_iter; ++idx) {
      const int j = block_at<ALIBI>(U, idx);
      if (!tile_uses<UK>(U, t, j)) continue;
      release_stage();
      // one verdict for the whole warp: the TMEM load and the vote below are
      // warp-collective, so no lane may leave the loop alone
      ok = warp_wait(bars + 8 * (B_S_FULL + t), s_ph, abort_flag, p);
      if (!ok) break;
      s_ph ^= 1u;
      tc_fence_after_sync();
      uint32_t sr[128];
      const int c0 = j * BN;
      const bool masked = block_needs_mask(p, r0, c0);
      float m_blk;
      // ALiBi on a block whose kept keys all lie on one side of every row of
      // the tile: the bias -slope |i - j| is linear in the block-local
      // key index e, so it folds into the raw scores as y = s + sigma e'
      // (sigma = slope / scale, e' = e for keys at or before the rows,
      // BN - 1 - e for keys at or after them), and the logit is c y + kappa
      // with one constant kappa per row.
      bool linear = false, after = false;
      float kappa = 0.f;
      if constexpr (ALIBI) {
        // under the causal mask every kept key is at or before its row
        const bool before = p.causal || c0 + BN - 1 <= r0;
        after = !before && c0 >= r0 + BM - 1;
        linear = (before || after) && c != 0.f && fabsf(slope2 / c) < 1e30f;
        const float relf = static_cast<float>(row - c0);   // exact in fp32
        if (linear) kappa = after ? slope2 * (relf - static_cast<float>(BN - 1)) : -slope2 * relf;
      }
      // Logits already scaled (and biased) in sr, instead of raw scores.
      const bool prescaled = (ALIBI && !linear) || (masked && c == 0.f);
      if (!ALIBI && !masked && c >= 0.f) {
        // Interior block: the raw row maximum of each 32-column chunk is
        // taken while the next chunk is read from TMEM.
        uint32_t (&s0)[32] = *reinterpret_cast<uint32_t(*)[32]>(sr);
        uint32_t (&s1)[32] = *reinterpret_cast<uint32_t(*)[32]>(sr + 32);
        uint32_t (&s2)[32] = *reinterpret_cast<uint32_t(*)[32]>(sr + 64);
        uint32_t (&s3)[32] = *reinterpret_cast<uint32_t(*)[32]>(sr + 96);
        float m0 = -INFINITY, m1 = -INFINITY;
        auto chunk_max = [&](const uint32_t (&x)[32]) {
#pragma unroll
          for (int e = 0; e < 32; e += 4) {
            m0 = max3(m0, __uint_as_float(x[e]), __uint_as_float(x[e + 1]));
            m1 = max3(m1, __uint_as_float(x[e + 2]), __uint_as_float(x[e + 3]));
          }
        };
        tmem_ld_32x32b_x32_start(s_tmem, s0);
        tmem_wait_ld_x32(s0);
        tmem_ld_32x32b_x32_start(s_tmem + 32, s1);
        chunk_max(s0);
        tmem_wait_ld_x32(s1);
        tmem_ld_32x32b_x32_start(s_tmem + 64, s2);
        chunk_max(s1);
        tmem_wait_ld_x32(s2);
        tmem_ld_32x32b_x32_start(s_tmem + 96, s3);
        chunk_max(s2);
        tmem_wait_ld_x32(s3);
        chunk_max(s3);
        m_blk = fmaxf(m0, m1) * c;
      } else if (prescaled) {
        tmem_ld_32x32b_x128(s_tmem, sr);
        // Scale first (adding the position bias -slope |i - j|), then drop
        // masked keys with -inf (any sign of scale).  Kept keys of this row,
        // in block-local columns e = j - c0:
        //   e <= hi (causal limit and key padding) and (e >= lo (window) or e < sk (sinks))
        const int hi = (p.causal ? min(row, p.N - 1) : p.N - 1) - c0;
        const int lo = p.window > 0 ? row - p.window + 1 - c0 : -(1 << 30);
        const int sk = p.window > 0 ? p.n_sink - c0 : -(1 << 30);
        const float rel = static_cast<float>(row - c0);   // i - c0, exact in fp32
#pragma unroll
        for (int e = 0; e < 128; ++e) {
          float x = __uint_as_float(sr[e]) * c;
          if constexpr (ALIBI) x = fmaf(-slope2, fabsf(rel - static_cast<float>(e)), x);
          if (masked) {
            const bool keep = (e <= hi) && (e >= lo || e < sk);
            x = keep ? x : -INFINITY;
          }
          sr[e] = __float_as_uint(x);
        }
        float m0 = -INFINITY, m1 = -INFINITY;
#pragma unroll
        for (int e = 0; e < 128; e += 4) {
          m0 = max3(m0, __uint_as_float(sr[e]), __uint_as_float(sr[e + 1]));
          m1 = max3(m1, __uint_as_float(sr[e + 2]), __uint_as_float(sr[e + 3]));
        }
        m_blk = fmaxf(m0, m1);
      } else {
        tmem_ld_32x32b_x128(s_tmem, sr);
        if (masked) {
          // A masked key gets the raw score -inf (+inf for a negative scale),
          // which the scale turns into -inf; the raw extreme and the exps
          // below then run as for an interior block.  Kept keys of this row,
          // in block-local columns e = j - c0:
          //   e <= hi (causal limit and key padding) and (e >= lo (window) or e < sk (sinks)).
          // The block's geometry says which of the bounds can bite (the same
          // for every row), so most blocks test one or two of them.
          const uint32_t gone = c > 0.f ? 0xff800000u : 0x7f800000u;
          const int hi = (p.causal ? min(row, p.N - 1) : p.N - 1) - c0;
          const int lo = row - p.window + 1 - c0;
          const int sk = p.n_sink - c0;
          const bool win_in = p.window > 0 && r0 + BM - p.window > c0;          // a window starts inside
          const bool win_after = p.window > 0 && r0 - p.window + 1 - c0 >= BN;  // every window starts after
          const bool hi_in = c0 + BN > p.N || (p.causal && c0 + BN - 1 > r0);   // a causal / padding edge
          if (win_after && !hi_in) {
            // before every row's window: only the sinks are kept
#pragma unroll
            for (int e = 0; e < 128; ++e) sr[e] = (e < sk) ? sr[e] : gone;
          } else if (!win_in && !win_after) {
#pragma unroll
            for (int e = 0; e < 128; ++e) sr[e] = (e <= hi) ? sr[e] : gone;
          } else if (win_in && !hi_in && sk <= 0) {
#pragma unroll
            for (int e = 0; e < 128; ++e) sr[e] = (e >= lo) ? sr[e] : gone;
          } else {
#pragma unroll
            for (int e = 0; e < 128; ++e) sr[e] = ((e <= hi) && (e >= lo || e < sk)) ? sr[e] : gone;
          }
        }
        if (ALIBI && linear) {
          const float sigma = slope2 / c;
          if (after) {
#pragma unroll
            for (int e = 0; e < 128; ++e)
              sr[e] = __float_as_uint(fmaf(sigma, static_cast<float>(BN - 1 - e), __uint_as_float(sr[e])));
          } else {
#pragma unroll
            for (int e = 0; e < 128; ++e)
              sr[e] = __float_as_uint(fmaf(sigma, static_cast<float>(e), __uint_as_float(sr[e])));
          }
        }
        // raw-score extreme, then one multiply: max of s*c is c*max(s) for c >= 0
        // and c*min(s) for c < 0 (plus the row constant of a linear ALiBi block)
        float m0 = __uint_as_float(sr[0]), m1 = __uint_as_float(sr[1]);
        if (c >= 0.f) {
#pragma unroll
          for (int e = 2; e < 126; e += 4) {
            m0 = max3(m0, __uint_as_float(sr[e]), __uint_as_float(sr[e + 1]));
            m1 = max3(m1, __uint_as_float(sr[e + 2]), __uint_as_float(sr[e + 3]));
          }
          m0 = max3(m0, __uint_as_float(sr[126]), __uint_as_float(sr[127]));
          m_blk = fmaf(fmaxf(m0, m1), c, kappa);
        } else {
#pragma unroll
          for (int e = 2; e < 126; e += 4) {
            m0 = min3(m0, __uint_as_float(sr[e]), __uint_as_float(sr[e + 1]));
            m1 = min3(m1, __uint_as_float(sr[e + 2]), __uint_as_float(sr[e + 3]));
          }
          m0 = min3(m0, __uint_as_float(sr[126]), __uint_as_float(sr[127]));
          m_blk = fmaf(fminf(m0, m1), c, kappa);
        }
      }
      // online softmax update (log2 units); lazy rescale
      const float m_new = fmaxf(m_run, m_blk);
      float alpha = 1.f;
      const bool rescale = m_new > m_run + RESCALE_THRESHOLD;
      if (rescale) {
        alpha = (m_run == -INFINITY) ? 0.f : fast_exp2(m_run - m_new);
        m_run = m_new;
      }
      const float mref = (m_run == -INFINITY) ? 0.f : m_run;
      const float2 cc2 = prescaled ? make_float2(1.f, 1.f) : make_float2(c, c);
      const float2 nm2 = make_float2(kappa - mref, kappa - mref);
      // Two denominators: le sums the fp32 weights (for the LSE), lr sums the
      // same 16-bit-rounded weights the P V MMA consumes (for O, so that every
      // output row is a convex combination of V rows under those weights).
      float2 le = make_float2(0.f, 0.f), lr = make_float2(0.f, 0.f);
      // P in four 32-key chunks: 16 packed words each, stored as soon as they
      // are ready so that the score registers are released chunk by chunk.
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
      // O_t holds the previous blocks' sum (the MMA that produced S_t for this
      // block was issued after the previous P_t V, so that PV has completed).
      if (!first && __any_sync(0xffffffffu, rescale)) {
#pragma unroll
        for (int cc = 0; cc < D / OC; ++cc) {
          uint32_t orr[OC];
          tmem_ld_cols<OC>(o_tmem + cc * OC, orr);
#pragma unroll
          for (int e = 0; e < OC; e += 2) {
            const float2 r2 = mul2(make_float2(__uint_as_float(orr[e]), __uint_as_float(orr[e + 1])),
                                   make_float2(alpha, alpha));
            orr[e] = __float_as_uint(r2.x);
            orr[e + 1] = __float_as_uint(r2.y);
          }
          tmem_st_cols<OC>(o_tmem + cc * OC, orr);
        }
      }
      tmem_wait_st();
      tc_fence_before_sync();
      __syncwarp();
      if (lane == 0) mbar_arrive(bars + 8 * (B_P_FULL + t));
      first = false;
    }
    if (!ok) break;
    if (SPLIT && t == 1) {
      // hand this half's row statistics to warpgroup 0, which merges
      st_shared_f32(half_stats, m_run);
      st_shared_f32(half_stats + 4, l_exact);
      st_shared_f32(half_stats + 8, l_round);
      __syncwarp();
      if (lane == 0) mbar_arrive(bars + 8 * B_HALF);
      continue;
    }
    // epilogue: O = O_acc / l, written once; LSE = (m + log2 l) ln 2
    ok = warp_wait(bars + 8 * (B_O_FULL + t), o_ph, abort_flag, p);
    if (!ok) break;
    o_ph ^= 1u;
    tc_fence_after_sync();
    // Split units: merge warpgroup 1's half, (m1, l1, O_1), into this one:
    // m = max(m0, m1), each half weighted by exp2(m_half - m).
    float w0 = 1.f, w1 = 0.f;
    bool has1 = false;
    if constexpr (SPLIT) {
      ok = warp_wait(bars + 8 * B_HALF, half_ph, abort_flag, p);
      if (!ok) break;
      half_ph ^= 1u;
      has1 = U.last1 >= 0;   // O_1 holds a sum only when warpgroup 1 visited a block
      if (has1) {
        ok = warp_wait(bars + 8 * (B_O_FULL + 1), o1_ph, abort_flag, p);
        if (!ok) break;
        o1_ph ^= 1u;
        tc_fence_after_sync();
      }
      const float m1 = ld_shared_f32(half_stats), le1 = ld_shared_f32(half_stats + 4),
                  lr1 = ld_shared_f32(half_stats + 8);
      const float m = fmaxf(m_run, m1);
      w0 = (m_run == -INFINITY) ? 0.f : fast_exp2(m_run - m);
      w1 = (m1 == -INFINITY) ? 0.f : fast_exp2(m1 - m);
      l_exact = l_exact * w0 + le1 * w1;
      l_round = l_round * w0 + lr1 * w1;
      m_run = m;
    }
    const float inv_l = 1.f / l_round;
    w0 *= inv_l;
    w1 *= inv_l;
    // the per-element scale of O_0 (split units fold it into the merge below)
    const float sc = SPLIT ? 1.f : inv_l;
    const bool valid = row < p.N;
    const uint32_t q_empty = bars + 8 * (B_Q_EMPTY + q_slot(ul, t));
    if constexpr (STAGED) {
      // O / l as 16-bit rows in this tile's Q slot (no longer read: the O_FULL
      // commit follows the tile's last S MMA), in the layout of the output's
      // TMA box: 64-column chunks of 128 rows x 128 bytes, 128-byte swizzle.
      // Warp 0 then writes the tile with TMA stores (rows >= N are clipped)
      // and releases the slot once the stores have read it.
      const uint32_t stage = sbase + G::Q_OFF + q_slot(ul, t) * G::TILE_BYTES;
      const uint32_t row_addr = stage + row_in_tile * 128;
#pragma unroll
      for (int cc = 0; cc < D / 32; ++cc) {
        uint32_t orr[32];
        tmem_ld_32x32b_x32(o_tmem + cc * 32, orr);
        if constexpr (SPLIT) merge_half<32>(orr, o1_tmem + cc * 32, has1, w0, w1);
        uint32_t pk[16];
#pragma unroll
        for (int e = 0; e < 16; ++e)
          pk[e] = pack2<BF16>(__uint_as_float(orr[2 * e]) * sc, __uint_as_float(orr[2 * e + 1]) * sc);
#pragma unroll
        for (int k4 = 0; k4 < 4; ++k4) {
          const int unit = (cc & 1) * 4 + k4;   // 16-byte unit within the 128-byte row
          st_shared_v4(row_addr + (cc >> 1) * G::CHUNK_BYTES + ((unit ^ (row_in_tile & 7)) << 4),
                       pk[4 * k4], pk[4 * k4 + 1], pk[4 * k4 + 2], pk[4 * k4 + 3]);
        }
      }
      fence_proxy_async_smem();
      __syncwarp();
      if (lane == 0) mbar_arrive(bars + 8 * (B_EPI + t));
      if (warp_in_wg == 0) {
        ok = warp_wait(bars + 8 * (B_EPI + t), epi_ph, abort_flag, p);
        if (ok && lane == 0) {
#pragma unroll
          for (int cch = 0; cch < G::NCH; ++cch)
            tma_store_3d(tmO, stage + cch * G::CHUNK_BYTES, cch * G::CW, r0, bh);
          bulk_commit_group();
          // the slot is released once the store has read it (see release_stage)
          staged_slot = q_empty;
        }
        __syncwarp();
      }
      epi_ph ^= 1u;
    } else {
      const size_t row_off = (static_cast<size_t>(bh) * p.N + row) * D;
#pragma unroll
      for (int cc = 0; cc < D / OC; ++cc) {
        uint32_t orr[OC];
        tmem_ld_cols<OC>(o_tmem + cc * OC, orr);
        if constexpr (SPLIT) merge_half<OC>(orr, o1_tmem + cc * OC, has1, w0, w1);
        if (valid) {
          if constexpr (OUT_F32) {
            float* dst = reinterpret_cast<float*>(p.o) + row_off + cc * OC;
#pragma unroll
            for (int e = 0; e < OC; e += 4) {
              const float4 v4 = make_float4(
                  __uint_as_float(orr[e]) * sc, __uint_as_float(orr[e + 1]) * sc,
                  __uint_as_float(orr[e + 2]) * sc, __uint_as_float(orr[e + 3]) * sc);
              *reinterpret_cast<float4*>(dst + e) = v4;
            }
          } else {
            uint32_t packed[OC / 2];
#pragma unroll
            for (int e = 0; e < OC / 2; ++e)
              packed[e] = pack2<BF16>(__uint_as_float(orr[2 * e]) * sc,
                                      __uint_as_float(orr[2 * e + 1]) * sc);
            uint16_t* dst = reinterpret_cast<uint16_t*>(p.o) + row_off + cc * OC;
#pragma unroll
            for (int e = 0; e < OC / 2; e += 4)
              *reinterpret_cast<uint4*>(dst + 2 * e) =
                  make_uint4(packed[e], packed[e + 1], packed[e + 2], packed[e + 3]);
          }
        }
      }
      // the slot was not used for staging
      if (warp_in_wg == 0 && lane == 0) mbar_arrive(q_empty);
    }
    if constexpr (SPLIT) {
      // O_1 and the statistics are read: warpgroup 1 may start its next unit
      tc_fence_before_sync();
      __syncwarp();
      if (lane == 0) mbar_arrive(bars + 8 * B_HALF_FREE);
    }
    if (valid && p.lse != nullptr)
      p.lse[static_cast<size_t>(bh) * p.N + row] = (m_run + __log2f(l_exact)) * 0.69314718055994531f;
  }
  // the output stores this warp issued complete before the CTA can exit
  if (STAGED && warp_in_wg == 0) {
    if (lane == 0) {
      release_stage();
      bulk_wait_group0();
    }
    __syncwarp();
  }
}

template <int D, bool BF16, bool OUT_F32, bool ALIBI, int UK>
__global__ void __launch_bounds__(NUM_THREADS, 1)
attn_fwd_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
                const __grid_constant__ CUtensorMap tmV, const __grid_constant__ CUtensorMap tmO,
                const KernelParams p) {
  using G = Geo<D>;
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  // 1024-byte alignment keeps every tile on a swizzle-pattern boundary.
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~static_cast<uintptr_t>(1023));
  const uint32_t sbase = smem_addr(smem);
  const uint32_t bars = sbase + G::BAR_OFF;
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + G::BAR_OFF + ABORT_FLAG_OFF);
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + G::BAR_OFF + TMEM_SLOT_OFF);

  const int warp = threadIdx.x / 32;
  const int lane = threadIdx.x % 32;

  if (threadIdx.x == 0) {
    for (int s = 0; s < Q_SLOTS; ++s) {
      mbar_init(bars + 8 * (B_Q_FULL + s), 1);
      // the last S MMA that reads the slot, and the epilogue that stages the
      // tile's output in it afterwards
      mbar_init(bars + 8 * (B_Q_EMPTY + s), 2);
    }
    for (int s = 0; s < NUM_STAGES; ++s) {
      mbar_init(bars + 8 * (B_K_FULL + s), 1);
      mbar_init(bars + 8 * (B_K_EMPTY + s), 1);
      mbar_init(bars + 8 * (B_V_FULL + s), 1);
      mbar_init(bars + 8 * (B_V_EMPTY + s), 1);
    }
    for (int t = 0; t < 2; ++t) {
      mbar_init(bars + 8 * (B_S_FULL + t), 1);
      mbar_init(bars + 8 * (B_P_FULL + t), 4);   // one arrival per softmax warp
      mbar_init(bars + 8 * (B_O_FULL + t), 1);
    }
    mbar_init(bars + 8 * B_DRAIN, 1);
    mbar_init(bars + 8 * (B_EPI + 0), 4);   // one arrival per softmax warp
    mbar_init(bars + 8 * (B_EPI + 1), 4);
    mbar_init(bars + 8 * B_HALF, 4);        // one arrival per softmax warp of warpgroup 1
    mbar_init(bars + 8 * B_HALF_FREE, 4);   // one arrival per softmax warp of warpgroup 0
    *abort_flag = 0;
    fence_barrier_init();
  }
  if (warp == MMA_WARP) {
    tmem_alloc(smem_addr(tmem_slot), TMEM_COLS);
    tmem_relinquish();
  }
  if (warp == TMA_WARP && lane == 0) {
    tma_prefetch_desc(&tmQ);
    tma_prefetch_desc(&tmK);
    tma_prefetch_desc(&tmV);
    if (!OUT_F32) tma_prefetch_desc(&tmO);
  }
  // The set-up above touches no global memory, so it may overlap the end of
  // the previous grid of the stream; nothing below runs before that grid is done.
  grid_dependency_wait();
  grid_launch_dependents();
  tc_fence_before_sync();
  __syncthreads();
  tc_fence_after_sync();
  const uint32_t tmem = *tmem_slot;

  // Each branch ends on its own copy of the final barrier: code shared by
  // warps running under different register budgets would have to fit the
  // smaller one.
  if (warp < 8) {
    regs_increase<SOFTMAX_REGS>();
    softmax_role<D, BF16, OUT_F32, ALIBI, UK>(p, &tmO, tmem, sbase, bars, warp / 4, warp % 4, lane,
                                          abort_flag);
    tc_fence_before_sync();
    __syncthreads();
  } else {
    regs_decrease<CONTROL_REGS>();
    if (warp == MMA_WARP) {
      mma_role<D, BF16, ALIBI, UK>(p, tmem, sbase, bars, abort_flag);
    } else if (warp == TMA_WARP) {
      tma_role<D, ALIBI, UK>(p, &tmQ, &tmK, &tmV, sbase, bars, abort_flag);
    }
    tc_fence_before_sync();
    __syncthreads();
    if (warp == MMA_WARP) {
      tc_fence_after_sync();
      tmem_dealloc(tmem, TMEM_COLS);
    }
  }
}

}  // namespace attn

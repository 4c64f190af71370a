/*
 * attn.h -- C ABI of the exact tiled attention library (libattn.so): the
 * forward (attn_fwd, attn_fwd_alibi, attn_fwd_host), its backward (attn_bwd) and
 * the split-KV decoding step (attn_decode, attn_decode_noalloc).
 *
 * The library computes, for every batch b and query head h,
 *
 *     O[b,h]   = softmax(scale * Q[b,h] K[b,g]^T + mask) V[b,g]
 *     LSE[b,h] = log-sum-exp (natural log) of the same masked, scaled logits
 *
 * with g = h / (H / H_kv), tile by tile with the online softmax (a running row
 * max m, a running denominator l and a rescaled output accumulator), never
 * materialising the N x N score matrix.  Sources of the definition:
 *   - "Flash Attention" (dileepadev learn-ai), "The Problem with Standard
 *     Attention" (the formula) and "Mathematical Equivalence" (the tiled form
 *     gives the same result, it is not an approximation); "Write output once".
 *   - "Tiled attention with online softmax" (Lab 3): the causal tiled loop
 *     with running max, running denominator and running numerator, key blocks
 *     after the query block skipped; exercise 4 (sinks + sliding window).
 *   - "USAAIO Lesson 91", slide 11 (the tiled update equations) and slide 32
 *     (MQA / GQA: query heads share K/V heads).
 *   - "Hands-On Build Guide: Flash Attention ... in NumPy", Step 2 (causal
 *     mask: key j is kept for query i iff j <= i) and Step 5 (a log-sum-exp
 *     carried across tiles).
 *
 * Conventions shared by every entry point:
 *   - All tensors are contiguous, row-major.  q and o are [B, H, N, d];
 *     k and v are [B, H_kv, N, d]; lse is [B, H, N] float32.
 *   - The mask keeps key j for query i iff
 *       (!causal || j <= i) && (window == 0 || i - j < window || j < n_sink).
 *     window counts the query itself (window = 1 keeps only the diagonal);
 *     sink keys are positions 0 .. n_sink-1 and stay subject to causality.
 *   - LSE_i = ln( sum over kept j of exp(scale * q_i . k_j) ).
 *   - The library never allocates device or host memory in these calls; the
 *     caller owns every buffer.
 *   - Every call returns an attn_status_t.  Argument errors are detected
 *     before anything is enqueued.  Calls are asynchronous on `stream`
 *     (a cudaStream_t passed as void*; NULL = the legacy default stream);
 *     faults inside the kernel surface at the caller's next synchronisation,
 *     and watchdog expiries are reported by attn_get_status().
 *   - Results are deterministic: equal inputs give bitwise-equal outputs,
 *     except attn_bwd's dQ (see there).
 *   - Per device, the first call records device addresses of the library's
 *     own __device__ objects (its status word, the static scratch array of
 *     attn_decode_noalloc) and keeps them for the life of the process.  The
 *     library therefore does not support cudaDeviceReset (or any other loss
 *     of the primary context) between calls: after one, those addresses may
 *     be stale.
 */
#ifndef ATTN_H_
#define ATTN_H_

#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
  ATTN_OK = 0,
  ATTN_ERR_INVALID_ARG = -1,     /* a size, pointer or flag is out of range   */
  ATTN_ERR_UNSUPPORTED = -2,     /* valid request this library does not handle */
  ATTN_ERR_MISALIGNED = -3,      /* a tensor pointer is not 16-byte aligned    */
  ATTN_ERR_CUDA = -4,            /* a CUDA runtime/driver call failed          */
  ATTN_ERR_DEVICE_TIMEOUT = -5   /* a kernel wait exceeded its time limit      */
} attn_status_t;

/* dtype argument: element type of q, k, v (and o), optionally OR-ed with
 * ATTN_OUT_F32 to make o float32 (the fp32 accumulator divided by l, before
 * any 16-bit rounding). */
enum {
  ATTN_BF16 = 0,
  ATTN_FP16 = 1,
  ATTN_OUT_F32 = 0x10
};

/*
 * attn_fwd -- exact masked attention forward on device buffers.
 *
 *   q      device, [B, H, N, d] bf16/fp16 (dtype), 16-byte aligned, read only
 *   k, v   device, [B, H_kv, N, d], same element type, 16-byte aligned
 *   o      device, [B, H, N, d]: same element type, or float32 when
 *          dtype & ATTN_OUT_F32; 16-byte aligned; must not overlap q, k or v
 *   lse    device, [B, H, N] float32, or NULL to skip writing it
 *   B, H, H_kv, N   sizes; B, H, N >= 0 (any zero: nothing to do, ATTN_OK,
 *          pointers may then be NULL); H_kv >= 1 and H % H_kv == 0
 *   d      head dimension: 16, 32, 64 or 128 (else ATTN_ERR_UNSUPPORTED)
 *   causal 0 or 1
 *   window 0 (none) or >= 1 keys including the query itself; needs causal
 *          (window > 0 with causal == 0 is ATTN_ERR_UNSUPPORTED)
 *   n_sink >= 0 always-kept leading keys; only meaningful with window > 0
 *   scale  finite float multiplying q.k before masking (0 is allowed)
 *   dtype  ATTN_BF16 or ATTN_FP16, optionally | ATTN_OUT_F32
 *   stream cudaStream_t as void*
 *
 * Needs an sm_100 device (B200); other devices give ATTN_ERR_UNSUPPORTED.
 * Returns after the kernel is enqueued.  One launch, with programmatic stream
 * serialisation: its CTAs may set up (barriers, tensor memory) while the
 * previous kernel of `stream` drains, and read or write global memory only
 * after that kernel has completed, so stream order holds.  The kernel allows
 * the next kernel of `stream` to be scheduled early only if that kernel was
 * itself launched with programmatic stream serialisation; such a kernel must
 * wait for it (griddepcontrol.wait) before reading o or lse.
 */
int attn_fwd(const void* q, const void* k, const void* v, void* o, float* lse,
             int B, int H, int H_kv, int N, int d, int causal, int window, int n_sink,
             float scale, int dtype, void* stream);

/*
 * attn_fwd_host -- the same forward for HOST-resident inputs and outputs.
 *
 * Copies q, k, v to the caller's device staging buffers dq, dk, dv, runs
 * attn_fwd(dq, dk, dv, dout, dlse, ...) and copies dout back into o and
 * (when both are non-NULL) dlse into lse.  The work is cut into up to 16
 * chunks of consecutive (batch, K/V head) groups: the host->device copies of
 * one chunk, the forward of the previous one (on `stream`) and the
 * device->host copies of the one before overlap, the copies running on two
 * copy streams the library creates once per device.  Events order the
 * chunks, and `stream` waits for the last copy: work enqueued on `stream`
 * later sees o and lse complete, and the caller synchronises `stream` before
 * reading them.  Host buffers should be page-locked for the copies to be
 * asynchronous and overlap.  Results equal attn_fwd's bitwise.  Concurrent
 * calls from several host threads enqueue one after the other.  Sizes,
 * flags and errors are those of attn_fwd; every pointer must be 16-byte
 * aligned.
 */
int attn_fwd_host(const void* q, const void* k, const void* v, void* o, float* lse,
                  void* dq, void* dk, void* dv, void* dout, float* dlse,
                  int B, int H, int H_kv, int N, int d, int causal, int window, int n_sink,
                  float scale, int dtype, void* stream);

/*
 * attn_fwd_alibi -- attn_fwd with the ALiBi position bias ("USAAIO Lesson 91",
 * slides 20-23, "ALiBi position bias"): the logit of query i and key j is
 *
 *     scale * q_i . k_j  -  slopes[h] * |i - j|
 *
 * before masking and the softmax, for query head h.  LSE is the log-sum-exp of
 * these biased, masked logits.  The bias is added for every kept key, causal
 * or not (|i - j| on both sides of the diagonal).
 *
 *   slopes device, [H] float32, one slope per query head, 4-byte aligned, read
 *          only; any finite values (the pages' choice is attn_alibi_slopes).
 *          NULL is ATTN_ERR_INVALID_ARG; it must not overlap o or lse.
 * Every other argument, the layouts, the mask and the errors are those of
 * attn_fwd.
 */
int attn_fwd_alibi(const void* q, const void* k, const void* v, void* o, float* lse,
                   const float* slopes, int B, int H, int H_kv, int N, int d, int causal,
                   int window, int n_sink, float scale, int dtype, void* stream);

/*
 * attn_alibi_slopes -- host only: writes the pages' ALiBi slopes for H heads,
 * the geometric sequence slopes[h - 1] = 2^(-8 h / H), h = 1 .. H ("USAAIO
 * Lesson 91", slide 23), rounded to float32, into the caller's host array
 * `slopes` of H floats.  Returns ATTN_ERR_INVALID_ARG for H < 1 or NULL.
 */
int attn_alibi_slopes(int H, float* slopes);

/*
 * attn_decode -- attention of N_q new query rows against a K/V cache of N_kv
 * positions, split across the cache ("USAAIO Lesson 91", slide 31: every
 * decoding step re-reads the whole cache; slide 32: query heads share K/V
 * heads; "Building a FlashAttention-style tiled self-attention block in pure
 * NumPy", "Extending It", item 6: split the sequence, then reduce the partial
 * outputs).
 *
 *   q      device, [B, H, N_q, d] bf16/fp16; query row i sits at cache
 *          position N_kv - N_q + i (the last N_q tokens of the sequence)
 *   k, v   device, [B, H_kv, N_kv, d] (the cache), same element type
 *   o      device, [B, H, N_q, d] (16-bit or float32 with ATTN_OUT_F32)
 *   lse    device, [B, H, N_q] float32, or NULL
 *   workspace, workspace_bytes   device scratch of at least
 *          attn_decode_workspace_bytes(...) bytes, 256-byte aligned, owned by
 *          the caller and not read by it; it needs no initial contents and
 *          must not be shared by calls in flight at once.  It may be NULL
 *          when no (batch, K/V head) group is split (see below).
 *   1 <= N_q <= N_kv; d is 64 or 128; (H / H_kv) * N_q <= 64 query rows per
 *          K/V head (else ATTN_ERR_UNSUPPORTED)
 * The mask rule, scale, dtype, LSE and error conventions are those of
 * attn_fwd, with the query position N_kv - N_q + i in place of i.  The
 * query rows of one (batch, K/V head) group go through the tensor cores
 * together against each 128-key tile of the cache, which is read once.  The
 * tiles of all groups that hold a kept key are laid end to end and cut into
 * at most 148 equal ranges, one CTA each; a group that spans several ranges
 * gets one partial (O_s, LSE_s) per range in the workspace, and a second
 * kernel merges them in range order (LSE = ln sum exp(LSE_s),
 * O = sum exp(LSE_s - LSE) O_s), so results are deterministic.  One or two
 * kernel launches on `stream`, both with programmatic stream serialisation as
 * attn_fwd's (the merge waits for the split kernel before reading the
 * workspace).
 */
int attn_decode(const void* q, const void* k, const void* v, void* o, float* lse,
                void* workspace, long long workspace_bytes, int B, int H, int H_kv, int N_q,
                int N_kv, int d, int causal, int window, int n_sink, float scale, int dtype,
                void* stream);

/* Host only: bytes of workspace attn_decode may need for these sizes (an
 * upper bound that depends neither on the device, the cache length nor the
 * mask), 0 for an empty problem, or -1 for invalid sizes. */
long long attn_decode_workspace_bytes(int B, int H, int H_kv, int N_q, int N_kv, int d);

/*
 * attn_decode_noalloc -- attn_decode without a caller workspace (the paper has
 * no counterpart).  The partial results live in a static 4 MiB device array
 * that is part of the library image on every device, so the call allocates
 * nothing; nothing in the array needs to start at zero (every partial a call
 * reads was written earlier in the same call).  Sizes whose
 * attn_decode_workspace_bytes exceed 4 MiB return ATTN_ERR_UNSUPPORTED
 * before anything is enqueued.
 * Races: every call on a device shares that one array, so calls on one device
 * must not overlap in time (issue them on one stream, or synchronise the
 * streams in between); overlapping calls give unspecified results.  All other
 * arguments and conventions are those of attn_decode.
 */
int attn_decode_noalloc(const void* q, const void* k, const void* v, void* o, float* lse,
                        int B, int H, int H_kv, int N_q, int N_kv, int d, int causal,
                        int window, int n_sink, float scale, int dtype, void* stream);

/*
 * attn_bwd -- gradients dQ, dK, dV of attn_fwd's output O for an upstream
 * gradient dO ("USAAIO Lesson 91", slide 9: the Flash Attention 2 backward
 * recomputes the attention tiles from the saved statistics instead of storing
 * the N x N matrix).  With P_ij = exp(scale q_i.k_j + bias_ij - LSE_i) over
 * the kept pairs and D_i = dO_i . O_i:
 *     dV_j = sum_i P_ij dO_i,   dS_ij = scale P_ij (dO_i . v_j - D_i),
 *     dQ_i = sum_j dS_ij k_j,   dK_j = sum_i dS_ij q_i,
 * summed over the query heads of a group for dK and dV.  The pages state no
 * gradient formula; these are the chain rule through the definition of
 * attn_fwd, with LSE treated as a saved statistic that receives no gradient.
 *
 *   q, k, v   device, as for attn_fwd (16-bit)
 *   o, dout   device, [B, H, N, d], same 16-bit type: the forward's output and
 *             the upstream gradient
 *   lse       device, [B, H, N] float32: the forward's LSE for the same
 *             q, k, v, mask, scale and slopes
 *   slopes    device, [H] float32 ALiBi slopes as for attn_fwd_alibi, or NULL
 *             for no position bias
 *   dq        device, [B, H, N, d]; dk, dv device, [B, H_kv, N, d]: outputs,
 *             16-bit, or float32 with ATTN_OUT_F32 in dtype
 *   workspace, workspace_bytes   device scratch of at least
 *             attn_bwd_workspace_bytes(B, H, N, d, dtype) bytes, 256-byte
 *             aligned, owned by the caller; overwritten by the call and not to
 *             be shared by calls in flight at once
 * Outputs and workspace must not overlap each other or any input (else
 * ATTN_ERR_INVALID_ARG); inputs may alias each other.  Sizes, mask, scale,
 * dtype and the other error conventions are those of attn_fwd.  The call
 * enqueues three kernels on `stream`: D and the zeroing of the fp32 dQ
 * accumulator, the tiled backward, and (for 16-bit outputs) the conversion
 * of dQ.  dQ is summed over key tiles with floating-point atomic adds, so its
 * last bits may differ between calls with equal inputs; dK and dV are each
 * written by one CTA and are deterministic.
 */
int attn_bwd(const void* q, const void* k, const void* v, const void* o, const void* dout,
             const float* lse, const float* slopes, void* dq, void* dk, void* dv,
             void* workspace, long long workspace_bytes, int B, int H, int H_kv, int N, int d,
             int causal, int window, int n_sink, float scale, int dtype, void* stream);

/* Host only: bytes of workspace attn_bwd needs (one float per query row, plus
 * an fp32 dQ accumulator unless dtype has ATTN_OUT_F32), 0 for empty sizes,
 * -1 for invalid sizes or flags.  Independent of the device. */
long long attn_bwd_workspace_bytes(int B, int H, int N, int d, int dtype);

/* Human-readable name of a status code (static storage, never NULL). */
const char* attn_error_string(int status);

/*
 * attn_unmasked_pairs -- host only: the number of kept (query, key) pairs of
 * one head under the mask rule above (N*N non-causal, N(N+1)/2 causal).  This
 * is the work the FLOP count 4*d*pairs credits ("Tiled attention with online
 * softmax", exercise 3 compares visited work with the full n^2).  Returns -1
 * for invalid arguments.
 */
long long attn_unmasked_pairs(int N, int causal, int window, int n_sink);

/*
 * attn_visited_blocks -- host only: the number of (128-query-row block,
 * 128-key block) pairs the kernel's schedule computes for one head (the same
 * set for the forward and for attn_bwd).  A block
 * pair is visited iff it holds at least one kept pair (this generalises the
 * causal block skipping of "Tiled attention with online softmax", Lab 3, to
 * windows and sinks).
 * Returns -1 for invalid arguments.
 */
long long attn_visited_blocks(int N, int causal, int window, int n_sink);

/*
 * attn_fwd_unit_kind -- host only: the work-unit shape attn_fwd (alibi == 0)
 * or attn_fwd_alibi (alibi != 0) runs for these sizes on a device with
 * `sm_count` SMs (0: the current device's count, which needs an sm_100
 * device):
 *   0  pairs of consecutive 128-row query tiles of one head;
 *   1  single tiles whose key blocks the two softmax warpgroups share, when
 *      pairs would leave SMs idle (B * H * ceil(N / 256) < sm_count) and single
 *      tiles still fit two waves (B * H * ceil(N / 128) <= 2 * sm_count);
 *   2  the same rows of two query heads sharing a K/V head, for H / H_kv >= 2
 *      when a row sees at most 4096 keys (min(N, window) <= 4096).
 * Position-biased launches always use 0.  The result does not depend on
 * causal, n_sink, d or the data.  Returns ATTN_ERR_INVALID_ARG for B < 0,
 * H < 1, H_kv < 1, H % H_kv != 0, N < 0, window < 0 or sm_count < 0.
 */
int attn_fwd_unit_kind(int B, int H, int H_kv, int N, int window, int alibi, int sm_count);

/*
 * attn_get_status -- reads and clears the device status word of the current
 * device.  Every wait inside the kernel is bounded (about attn_watchdog_ns
 * nanoseconds); a CTA whose wait expires drains its own in-flight copies and
 * tensor-core work, releases its tensor memory, records
 * ATTN_ERR_DEVICE_TIMEOUT here and returns.  The backward kernel also records
 * ATTN_ERR_CUDA, and returns before doing any work, if the dynamic shared
 * memory it was given cannot hold its 1024-byte aligned layout (a launch
 * configuration fault; its outputs are then not written).  Synchronises the
 * device.
 */
int attn_get_status(void);

/* Sets the watchdog limit in nanoseconds for later launches on every device
 * (default 2e9, clamped to [1e6, 6e10]).  Returns the previous value. */
unsigned long long attn_set_watchdog_ns(unsigned long long ns);

/* Number of kernel launches enqueued by this process so far (all entry
 * points).  Lets a caller count the GPU launches of a region. */
unsigned long long attn_launch_count(void);

/*
 * attn_test_withhold_loads -- failure-detection test hook (the paper has no
 * counterpart).  The next `n_launches` launches of this process start their
 * copy warp without issuing a single copy, so every other wait in the kernel
 * runs into the watchdog: the CTAs record ATTN_ERR_DEVICE_TIMEOUT (read it with
 * attn_get_status), release their tensor memory and return; outputs are left
 * unspecified.  Nothing faults and the context stays usable.  0 turns the hook
 * off.  Returns ATTN_ERR_INVALID_ARG for n_launches < 0.
 */
int attn_test_withhold_loads(int n_launches);

/*
 * attn_test_count_blocks -- schedule test hook (the paper has no counterpart).
 * While `counter` is non-NULL, every later attn_fwd / attn_fwd_alibi launch
 * adds to the device uint64 at `counter` the number of (128-row query tile,
 * 128-key block) score tiles it computed, and every attn_bwd launch the
 * number of (key tile, query tile) steps of its tiled kernel, with one atomic
 * add per CTA.  A test compares the sum with attn_visited_blocks() times
 * B * H ("Tiled attention with online softmax", exercise 3: count the block
 * pairs the tiled loop visits).  `counter` is caller-owned device memory,
 * 8-byte aligned, zeroed by the caller; NULL turns the hook off (the default).
 * Process-wide and not synchronised with launches in flight: set it between
 * launches only.  Returns ATTN_OK.
 */
int attn_test_count_blocks(unsigned long long* counter);

/*
 * attn_test_force_units -- schedule test hook (the paper has no counterpart).
 * attn_fwd runs one of three work-unit shapes, chosen from the sizes alone:
 *   0  pairs of consecutive 128-row query tiles of one head (the two softmax
 *      warpgroups take one tile each);
 *   1  single tiles whose key blocks the two warpgroups share out and merge
 *      (LSE = log-sum of both halves, O the weighted sum), when pairs would
 *      leave SMs idle;
 *   2  the same 128 rows of two query heads that share a K/V head (GQA / MQA,
 *      "USAAIO Lesson 91", slide 32), so each K/V block loaded feeds both.
 * All compute the same function; 0 and 2 give bitwise-equal results, 1 may
 * differ in the last bits.  A mode forces that shape on every later attn_fwd
 * launch (ALiBi launches always use pairs); -1 restores the automatic choice
 * (the default).  Process-wide; set it between launches only.  Returns
 * ATTN_OK, or ATTN_ERR_INVALID_ARG for another mode.
 */
int attn_test_force_units(int mode);

#ifdef __cplusplus
}
#endif

#endif /* ATTN_H_ */

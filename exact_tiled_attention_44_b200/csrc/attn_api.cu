// attn_api.cu -- host side of libattn.so shared by every entry point: the
// per-device state, argument checks, TMA descriptors and the small host-only
// helpers of include/attn.h.  The launches are in fwd_api.cu, bwd_api.cu and
// decode_api.cu, one translation unit each.
#include <cmath>
#include <cstring>

#include "host.h"
#include "attn_kernel.cuh"

namespace {

// Device status word: written by a CTA whose wait timed out, read and cleared
// by attn_get_status().
__device__ int g_device_status = 0;

attn_host::DeviceState g_dev[attn_host::kMaxDevices];

}  // namespace

namespace attn_host {

std::mutex g_mu;
std::atomic<unsigned long long> g_watchdog_ns{2000000000ull};
std::atomic<unsigned long long> g_launches{0};
std::atomic<int> g_withhold{0};
std::atomic<int> g_force_units{-1};
std::atomic<unsigned long long*> g_block_count{nullptr};
std::mutex g_host_mu;
PFN_cuTensorMapEncodeTiled_v12000 g_encode = nullptr;

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


int take_withhold() {
  for (int n = g_withhold.load(); n > 0;) {
    if (g_withhold.compare_exchange_weak(n, n - 1)) return 1;
  }
  return 0;
}

}  // namespace attn_host

using namespace attn_host;

extern "C" {

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
  DeviceState* st = nullptr;
  rc = device_state(&st);
  if (rc != ATTN_OK) return rc;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  const bool with_lse = lse != nullptr && dlse != nullptr;
  // The problem is cut into chunks of consecutive (batch, K/V head) groups.
  // A group's q, o and lse rows (its H / H_kv query heads) and its k, v rows
  // are contiguous in every buffer, and a run of T groups is itself an
  // attention problem of T batches of G query heads over one K/V head.  The
  // host->device copies of chunk c+1 (copy stream 1), the forward of chunk c
  // (the caller's stream) and the device->host copies of chunk c-1 (copy
  // stream 2) overlap; events order them, and the caller's stream waits for
  // the last copy, so the contract of a single stream holds.
  const long long groups = static_cast<long long>(B) * H_kv;
  const int G = H / H_kv;
  // every chunk runs the work-unit shape attn_fwd would choose for the whole problem
  const int forced = g_force_units.load();
  const int uk = forced >= 0 ? forced : fwd_unit_kind(B, H, H_kv, N, window, false, st->sm_count);
  // chunked LSE rows must keep the 16-byte alignment attn_fwd requires
  const bool lse_ok = !with_lse || (static_cast<long long>(G) * N) % 4 == 0;
  const int n_chunks = lse_ok ? static_cast<int>(groups < kHostChunks ? groups : kHostChunks) : 1;
  const size_t q_grp = static_cast<size_t>(G) * N * d * sz.elem;
  const size_t kv_grp = static_cast<size_t>(N) * d * sz.elem;
  const size_t o_grp = sz.o_bytes / static_cast<size_t>(groups);
  const size_t l_grp = static_cast<size_t>(G) * N * sizeof(float);
  std::lock_guard<std::mutex> lock(g_host_mu);
  if (!st->host_ready) {
    if (cudaStreamCreateWithFlags(&st->copy_in, cudaStreamNonBlocking) != cudaSuccess ||
        cudaStreamCreateWithFlags(&st->copy_out, cudaStreamNonBlocking) != cudaSuccess)
      return ATTN_ERR_CUDA;
    for (int i = 0; i < 2 * kHostChunks + 2; ++i)
      if (cudaEventCreateWithFlags(&st->ev[i], cudaEventDisableTiming) != cudaSuccess)
        return ATTN_ERR_CUDA;
    st->host_ready = true;
  }
  cudaEvent_t start = st->ev[2 * kHostChunks], done = st->ev[2 * kHostChunks + 1];
  if (cudaEventRecord(start, s) != cudaSuccess ||
      cudaStreamWaitEvent(st->copy_in, start, 0) != cudaSuccess ||
      cudaStreamWaitEvent(st->copy_out, start, 0) != cudaSuccess)
    return ATTN_ERR_CUDA;
  const auto at = [](const void* base, size_t off) {
    return static_cast<const char*>(base) + off;
  };
  long long g0 = 0;
  for (int c = 0; c < n_chunks; ++c) {
    const long long g1 = groups * (c + 1) / n_chunks;
    const size_t T = static_cast<size_t>(g1 - g0);
    cudaEvent_t in = st->ev[2 * c], out = st->ev[2 * c + 1];
    char* dqc = const_cast<char*>(at(dq, g0 * q_grp));
    char* dkc = const_cast<char*>(at(dk, g0 * kv_grp));
    char* dvc = const_cast<char*>(at(dv, g0 * kv_grp));
    char* doc = const_cast<char*>(at(dout, g0 * o_grp));
    float* dlc = with_lse ? reinterpret_cast<float*>(const_cast<char*>(at(dlse, g0 * l_grp))) : nullptr;
    if (cudaMemcpyAsync(dqc, at(q, g0 * q_grp), T * q_grp, cudaMemcpyHostToDevice, st->copy_in) != cudaSuccess ||
        cudaMemcpyAsync(dkc, at(k, g0 * kv_grp), T * kv_grp, cudaMemcpyHostToDevice, st->copy_in) != cudaSuccess ||
        cudaMemcpyAsync(dvc, at(v, g0 * kv_grp), T * kv_grp, cudaMemcpyHostToDevice, st->copy_in) != cudaSuccess ||
        cudaEventRecord(in, st->copy_in) != cudaSuccess || cudaStreamWaitEvent(s, in, 0) != cudaSuccess)
      return ATTN_ERR_CUDA;
    rc = fwd_impl(dqc, dkc, dvc, doc, dlc, nullptr, static_cast<int>(T), G, 1, N, d, causal, window,
                  n_sink, scale, dtype, stream, uk);
    if (rc != ATTN_OK) return rc;
    if (cudaEventRecord(out, s) != cudaSuccess || cudaStreamWaitEvent(st->copy_out, out, 0) != cudaSuccess ||
        cudaMemcpyAsync(const_cast<char*>(at(o, g0 * o_grp)), doc, T * o_grp, cudaMemcpyDeviceToHost,
                        st->copy_out) != cudaSuccess)
      return ATTN_ERR_CUDA;
    if (with_lse && cudaMemcpyAsync(const_cast<char*>(at(lse, g0 * l_grp)), dlc, T * l_grp,
                                    cudaMemcpyDeviceToHost, st->copy_out) != cudaSuccess)
      return ATTN_ERR_CUDA;
    g0 = g1;
  }
  if (cudaEventRecord(done, st->copy_out) != cudaSuccess || cudaStreamWaitEvent(s, done, 0) != cudaSuccess)
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

int attn_test_count_blocks(unsigned long long* counter) {
  g_block_count.store(counter);
  return ATTN_OK;
}

int attn_test_force_units(int mode) {
  if (mode < -1 || mode > 2) return ATTN_ERR_INVALID_ARG;
  g_force_units.store(mode);
  return ATTN_OK;
}

unsigned long long attn_launch_count(void) { return g_launches.load(std::memory_order_relaxed); }

}  // extern "C"

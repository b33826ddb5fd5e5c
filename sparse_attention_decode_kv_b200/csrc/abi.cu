// abi.cu -- the extern "C" entry points of libcsa2.so declared in include/csa2.h.
//
// Every entry point validates its arguments on the host before touching CUDA, so an invalid
// call returns a status without launching anything (and works on a machine without a GPU).
#include <atomic>
#include <mutex>
#include <unordered_map>
#include <vector>

#include "common.cuh"
#include "internal.h"

namespace csa2 {

static std::atomic<uint64_t> g_launches{0};

void count_launches(int n) { g_launches.fetch_add(static_cast<uint64_t>(n)); }

static cudaEvent_t g_prof_start[CSA2_KERNEL_COUNT] = {};
static cudaEvent_t g_prof_stop[CSA2_KERNEL_COUNT] = {};

void profile_begin(int kernel, cudaStream_t s) {
  if (g_prof_start[kernel] != nullptr) cudaEventRecord(g_prof_start[kernel], s);
}

void profile_end(int kernel, cudaStream_t s) {
  if (g_prof_stop[kernel] != nullptr) cudaEventRecord(g_prof_stop[kernel], s);
}

TensorMapEncodeFn tensor_map_encoder() {
  static std::once_flag once;
  static TensorMapEncodeFn fn = nullptr;
  std::call_once(once, [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<TensorMapEncodeFn>(p);
  });
  return fn;
}

static std::mutex g_last_mu;
static std::unordered_map<const void*, bool> g_last_attend;

void note_call(cudaStream_t s, bool is_attend) {
  std::lock_guard<std::mutex> lock(g_last_mu);
  g_last_attend[static_cast<const void*>(s)] = is_attend;
}

bool last_call_was_attend(cudaStream_t s) {
  std::lock_guard<std::mutex> lock(g_last_mu);
  const auto it = g_last_attend.find(static_cast<const void*>(s));
  return it != g_last_attend.end() && it->second;
}

int device_sm_count() {
  static std::mutex mu;
  static std::vector<int> cache;
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return 148;
  std::lock_guard<std::mutex> lock(mu);
  if (dev >= static_cast<int>(cache.size())) cache.resize(dev + 1, 0);
  if (cache[dev] == 0) {
    int n = 0;
    if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || n <= 0)
      n = 148;
    cache[dev] = n;
  }
  return cache[dev];
}

}  // namespace csa2

namespace {

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

// null is rejected unless allowed; non-null must be 16-byte aligned
bool ptr_ok(const void* p, bool nullable = false) {
  if (p == nullptr) return nullable;
  return aligned16(p);
}

int cuda_status(cudaError_t e) { return e == cudaSuccess ? CSA2_OK : CSA2_ERR_CUDA; }

// Rows 0 .. N[b]-1 of every sequence between two [B, rows, row_bytes] layouts. A run of
// sequences that are full in both layouts is contiguous, so it goes as one copy.
cudaError_t copy_rows(void* dst, int64_t dst_rows, const void* src, int64_t src_rows,
                      int64_t row_bytes, int B, const int32_t* N, cudaMemcpyKind kind,
                      cudaStream_t s) {
  int b = 0;
  while (b < B) {
    int e = b + 1;
    int64_t rows = N[b];
    while (e < B && N[e - 1] == dst_rows && N[e - 1] == src_rows) rows += N[e++];
    if (rows > 0) {
      cudaError_t err = cudaMemcpyAsync(
          static_cast<uint8_t*>(dst) + static_cast<int64_t>(b) * dst_rows * row_bytes,
          static_cast<const uint8_t*>(src) + static_cast<int64_t>(b) * src_rows * row_bytes,
          static_cast<size_t>(rows * row_bytes), kind, s);
      if (err != cudaSuccess) return err;
    }
    b = e;
  }
  return cudaSuccess;
}

// The checks shared by csa2_cache_restore and csa2_cache_persist.
int cache_copy_args_ok(const void* codes, const void* scales, const void* ik, int B, int n_cap,
                       const int32_t* N, int n_host, const void* h_codes, const void* h_scales,
                       const void* h_ik) {
  if (B <= 0 || n_cap <= 0 || (n_cap % CSA2_S) != 0 || n_host < 0) return CSA2_ERR_INVALID;
  if (B > CSA2_MAX_B || n_cap > CSA2_MAX_NCAP || n_host > CSA2_MAX_NCAP) return CSA2_ERR_UNSUPPORTED;
  if (N == nullptr || !ptr_ok(codes) || !ptr_ok(scales) || !ptr_ok(h_codes) || !ptr_ok(h_scales))
    return CSA2_ERR_INVALID;
  if ((ik == nullptr) != (h_ik == nullptr) || !ptr_ok(ik, true) || !ptr_ok(h_ik, true))
    return CSA2_ERR_INVALID;
  for (int b = 0; b < B; ++b)
    if (N[b] < 0 || N[b] > n_cap || N[b] > n_host) return CSA2_ERR_INVALID;
  return CSA2_OK;
}

}  // namespace

extern "C" {

int csa2_abi_version(void) { return 3; }

uint64_t csa2_launch_count(void) { return csa2::g_launches.load(); }

int csa2_set_profile_events(int kernel, void* start_event, void* stop_event) {
  if (kernel < 0 || kernel >= CSA2_KERNEL_COUNT) return CSA2_ERR_INVALID;
  if ((start_event == nullptr) != (stop_event == nullptr)) return CSA2_ERR_INVALID;
  csa2::g_prof_start[kernel] = static_cast<cudaEvent_t>(start_event);
  csa2::g_prof_stop[kernel] = static_cast<cudaEvent_t>(stop_event);
  return CSA2_OK;
}

const char* csa2_status_string(int status) {
  switch (status) {
    case CSA2_OK: return "CSA2_OK";
    case CSA2_ERR_INVALID: return "CSA2_ERR_INVALID: null/misaligned pointer or inconsistent size";
    case CSA2_ERR_UNSUPPORTED: return "CSA2_ERR_UNSUPPORTED: size beyond this build's limits";
    case CSA2_ERR_WORKSPACE: return "CSA2_ERR_WORKSPACE: workspace too small";
    case CSA2_ERR_CUDA: return "CSA2_ERR_CUDA: CUDA runtime or launch error";
    case CSA2_ERR_DEVICE: return "CSA2_ERR_DEVICE: a kernel reported a device-side error";
    case CSA2_ERR_TIMEOUT: return "CSA2_ERR_TIMEOUT: a bounded wait inside a kernel gave up";
    default: return "unknown csa2 status";
  }
}

int csa2_append_quant(const void* x, const void* ik, int B, int n, const int32_t* pos, int n_cap,
                      uint8_t* codes, uint8_t* scales, void* ik_cache, uint8_t* swa,
                      float* swa_scale, int W, int32_t* dev_err, csa2_stream_t stream) {
  if (B <= 0 || n < 0 || n_cap <= 0 || (n_cap % CSA2_S) != 0 || W < 0) return CSA2_ERR_INVALID;
  if (B > CSA2_MAX_B || n_cap > CSA2_MAX_NCAP || W > CSA2_MAX_W) return CSA2_ERR_UNSUPPORTED;
  if (!ptr_ok(x) || !ptr_ok(pos) || !ptr_ok(codes) || !ptr_ok(scales)) return CSA2_ERR_INVALID;
  if ((ik == nullptr) != (ik_cache == nullptr) || !ptr_ok(ik, true) || !ptr_ok(ik_cache, true))
    return CSA2_ERR_INVALID;
  const bool ring = swa != nullptr || swa_scale != nullptr;
  if (ring && (W == 0 || !ptr_ok(swa) || swa_scale == nullptr)) return CSA2_ERR_INVALID;
  if (!ring && W != 0) return CSA2_ERR_INVALID;
  if (dev_err != nullptr && (reinterpret_cast<uintptr_t>(dev_err) & 3u)) return CSA2_ERR_INVALID;
  if (n == 0) return CSA2_OK;
  const cudaError_t launch_err = csa2::launch_append(x, ik, B, n, pos, n_cap, codes, scales, ik_cache, swa,
                                         swa_scale, W, dev_err,
                                         reinterpret_cast<cudaStream_t>(stream));
  csa2::note_call(reinterpret_cast<cudaStream_t>(stream), false);
  return cuda_status(launch_err);
}

int csa2_ced_project_quant(const void* h, const void* w, int B, int n, int d, const int32_t* pos,
                           int n_cap, uint8_t* codes, uint8_t* scales, int32_t* dev_err,
                           csa2_stream_t stream) {
  if (B <= 0 || n < 0 || n_cap <= 0 || (n_cap % CSA2_S) != 0) return CSA2_ERR_INVALID;
  if (d < CSA2_CED_D_ALIGN || (d % CSA2_CED_D_ALIGN) != 0) return CSA2_ERR_INVALID;
  if (B > CSA2_MAX_B || n_cap > CSA2_MAX_NCAP || d > CSA2_MAX_CED_D ||
      static_cast<int64_t>(B) * n > CSA2_MAX_CED_TOKENS)
    return CSA2_ERR_UNSUPPORTED;
  if (!ptr_ok(h) || !ptr_ok(w) || !ptr_ok(pos) || !ptr_ok(codes) || !ptr_ok(scales))
    return CSA2_ERR_INVALID;
  if (dev_err != nullptr && (reinterpret_cast<uintptr_t>(dev_err) & 3u)) return CSA2_ERR_INVALID;
  if (n == 0) return CSA2_OK;
  const cudaError_t launch_err = csa2::launch_ced_quant(h, w, B, n, d, pos, n_cap, codes, scales, dev_err,
                                            reinterpret_cast<cudaStream_t>(stream));
  csa2::note_call(reinterpret_cast<cudaStream_t>(stream), false);
  return cuda_status(launch_err);
}

size_t csa2_index_full_workspace_bytes(int B, int n_cap, int K, int P) {
  if (B <= 0 || n_cap <= 0 || K <= 0 || P <= 0) return 0;
  return csa2::index_full_workspace_bytes(B, n_cap, K, P);
}

int csa2_index_full(const void* iq, const float* w, const void* ik_cache, const int32_t* N, int B,
                    int n_cap, int K, int P, int32_t* topk, int32_t* pool, void* ws,
                    size_t ws_bytes, int32_t* dev_err, csa2_stream_t stream) {
  if (B <= 0 || n_cap <= 0 || (n_cap % CSA2_S) != 0 || K <= 0 || P <= 0) return CSA2_ERR_INVALID;
  if (B > CSA2_MAX_B || n_cap > CSA2_MAX_NCAP || K > CSA2_MAX_K || P > CSA2_MAX_P)
    return CSA2_ERR_UNSUPPORTED;
  if (!ptr_ok(iq) || !ptr_ok(w) || !ptr_ok(ik_cache) || !ptr_ok(N) || !ptr_ok(topk) ||
      !ptr_ok(pool) || !ptr_ok(ws))
    return CSA2_ERR_INVALID;
  if (dev_err != nullptr && (reinterpret_cast<uintptr_t>(dev_err) & 3u)) return CSA2_ERR_INVALID;
  if (ws_bytes < csa2::index_full_workspace_bytes(B, n_cap, K, P)) return CSA2_ERR_WORKSPACE;
  const cudaError_t launch_err = csa2::launch_index_full(iq, w, ik_cache, N, B, n_cap, K, P, topk, pool, ws,
                                             dev_err, reinterpret_cast<cudaStream_t>(stream));
  csa2::note_call(reinterpret_cast<cudaStream_t>(stream), false);
  return cuda_status(launch_err);
}

size_t csa2_index_reindex_workspace_bytes(int B, int L, int K) {
  if (B <= 0 || L <= 0 || K <= 0) return 0;
  return csa2::index_reindex_workspace_bytes(B, L, K);
}

int csa2_index_reindex(const void* iq, const float* w, const void* ik_cache, const int32_t* N,
                       int B, int n_cap, const int32_t* pool, int L, int K, int32_t* topk,
                       void* ws, size_t ws_bytes, int32_t* dev_err, csa2_stream_t stream) {
  if (B <= 0 || n_cap <= 0 || (n_cap % CSA2_S) != 0 || L <= 0 || K <= 0) return CSA2_ERR_INVALID;
  if (B > CSA2_MAX_B || n_cap > CSA2_MAX_NCAP || L > CSA2_MAX_POOL || K > CSA2_MAX_K)
    return CSA2_ERR_UNSUPPORTED;
  if (!ptr_ok(iq) || !ptr_ok(w) || !ptr_ok(ik_cache) || !ptr_ok(N) || !ptr_ok(pool) ||
      !ptr_ok(topk) || !ptr_ok(ws))
    return CSA2_ERR_INVALID;
  if (dev_err != nullptr && (reinterpret_cast<uintptr_t>(dev_err) & 3u)) return CSA2_ERR_INVALID;
  if (ws_bytes < csa2::index_reindex_workspace_bytes(B, L, K)) return CSA2_ERR_WORKSPACE;
  const cudaError_t launch_err = csa2::launch_index_reindex(iq, w, ik_cache, N, B, n_cap, pool, L, K, topk,
                                                ws, dev_err,
                                                reinterpret_cast<cudaStream_t>(stream));
  csa2::note_call(reinterpret_cast<cudaStream_t>(stream), false);
  return cuda_status(launch_err);
}

size_t csa2_attend_workspace_bytes(int B, int K, int W) {
  if (B <= 0 || K <= 0 || W < 0) return 0;
  return csa2::attend_workspace_bytes(B, K, W);
}

int csa2_attend(int mode, const void* q, float softmax_scale, const uint8_t* codes,
                const uint8_t* scales, int n_cap, const int32_t* N, const int32_t* idx, int K,
                const uint8_t* swa, const float* swa_scale, const int32_t* swa_len, int W, int B,
                float* out, float* lse, void* ws, size_t ws_bytes, int32_t* dev_err,
                csa2_stream_t stream) {
  if (mode != CSA2_MODE_FULL && mode != CSA2_MODE_REINDEX && mode != CSA2_MODE_REUSE)
    return CSA2_ERR_INVALID;
  if (B <= 0 || n_cap <= 0 || (n_cap % CSA2_S) != 0 || K <= 0 || W < 0) return CSA2_ERR_INVALID;
  if (B > CSA2_MAX_B || n_cap > CSA2_MAX_NCAP || K > CSA2_MAX_K || W > CSA2_MAX_W)
    return CSA2_ERR_UNSUPPORTED;
  if (!(softmax_scale == softmax_scale)) return CSA2_ERR_INVALID;  // NaN
  if (!ptr_ok(q) || !ptr_ok(codes) || !ptr_ok(scales) || !ptr_ok(N) || !ptr_ok(idx) ||
      !ptr_ok(out) || !ptr_ok(lse, true))
    return CSA2_ERR_INVALID;
  if (W > 0 && (!ptr_ok(swa) || !ptr_ok(swa_scale) || !ptr_ok(swa_len))) return CSA2_ERR_INVALID;
  if (dev_err != nullptr && (reinterpret_cast<uintptr_t>(dev_err) & 3u)) return CSA2_ERR_INVALID;
  const size_t need = csa2::attend_workspace_bytes(B, K, W);
  if (need > 0 && (ws == nullptr || !aligned16(ws) || ws_bytes < need)) return CSA2_ERR_WORKSPACE;
  const cudaError_t launch_err = csa2::launch_attend(q, softmax_scale, codes, scales, n_cap, N, idx, K,
                                         W > 0 ? swa : nullptr, W > 0 ? swa_scale : nullptr,
                                         W > 0 ? swa_len : nullptr, W, nullptr, nullptr, W, B, B,
                                         out, lse, ws, dev_err,
                                         mode == CSA2_MODE_REUSE && csa2::last_call_was_attend(
                                             reinterpret_cast<cudaStream_t>(stream)),
                                         reinterpret_cast<cudaStream_t>(stream));
  csa2::note_call(reinterpret_cast<cudaStream_t>(stream), true);
  return cuda_status(launch_err);
}

int csa2_attend_queries(const void* q, float softmax_scale, const uint8_t* codes,
                        const uint8_t* scales, int B, int n_cap, const int32_t* N,
                        const int32_t* qseq, const int32_t* idx, int K, const uint8_t* swa,
                        const float* swa_scale, int S, const int32_t* swa_lo,
                        const int32_t* swa_len, int W, int Q, float* out, float* lse, void* ws,
                        size_t ws_bytes, int32_t* dev_err, csa2_stream_t stream) {
  if (Q <= 0 || B <= 0 || n_cap <= 0 || (n_cap % CSA2_S) != 0 || K <= 0 || W < 0 || S < 0)
    return CSA2_ERR_INVALID;
  if (W > S) return CSA2_ERR_INVALID;  // a window never holds more rows than the buffer
  if (Q > CSA2_MAX_QUERIES || B > CSA2_MAX_B || n_cap > CSA2_MAX_NCAP || K > CSA2_MAX_K ||
      W > CSA2_MAX_W || S > CSA2_MAX_SWA_ROWS)
    return CSA2_ERR_UNSUPPORTED;
  if (!(softmax_scale == softmax_scale)) return CSA2_ERR_INVALID;  // NaN
  if (!ptr_ok(q) || !ptr_ok(codes) || !ptr_ok(scales) || !ptr_ok(N) || !ptr_ok(qseq) ||
      !ptr_ok(idx) || !ptr_ok(out) || !ptr_ok(lse, true))
    return CSA2_ERR_INVALID;
  if (W > 0 && (!ptr_ok(swa) || !ptr_ok(swa_scale) || !ptr_ok(swa_lo) || !ptr_ok(swa_len)))
    return CSA2_ERR_INVALID;
  if (dev_err != nullptr && (reinterpret_cast<uintptr_t>(dev_err) & 3u)) return CSA2_ERR_INVALID;
  const size_t need = csa2::attend_workspace_bytes(Q, K, W);
  if (need > 0 && (ws == nullptr || !aligned16(ws) || ws_bytes < need)) return CSA2_ERR_WORKSPACE;
  // the kernels check every qseq entry against B (a bad one gives an empty query and a flag)
  const cudaError_t launch_err = csa2::launch_attend(q, softmax_scale, codes, scales, n_cap, N, idx, K,
                                         W > 0 ? swa : nullptr, W > 0 ? swa_scale : nullptr,
                                         W > 0 ? swa_len : nullptr, W, qseq,
                                         W > 0 ? swa_lo : nullptr, S, B, Q, out, lse, ws, dev_err,
                                         false, reinterpret_cast<cudaStream_t>(stream));
  csa2::note_call(reinterpret_cast<cudaStream_t>(stream), true);
  return cuda_status(launch_err);
}

int csa2_cache_restore(const uint8_t* host_codes, const uint8_t* host_scales, const void* host_ik,
                       int B, int n_host, const int32_t* N, int n_cap, uint8_t* codes,
                       uint8_t* scales, void* ik_cache, csa2_stream_t stream) {
  const int st = cache_copy_args_ok(codes, scales, ik_cache, B, n_cap, N, n_host, host_codes,
                                    host_scales, host_ik);
  if (st != CSA2_OK) return st;
  const cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  cudaError_t e = copy_rows(codes, n_cap, host_codes, n_host, CSA2_D / 2, B, N,
                            cudaMemcpyHostToDevice, s);
  if (e == cudaSuccess)
    e = copy_rows(scales, n_cap, host_scales, n_host, CSA2_D / 16, B, N, cudaMemcpyHostToDevice, s);
  if (e == cudaSuccess && ik_cache != nullptr)
    e = copy_rows(ik_cache, n_cap, host_ik, n_host, CSA2_DI * 2, B, N, cudaMemcpyHostToDevice, s);
  csa2::note_call(reinterpret_cast<cudaStream_t>(stream), false);
  return cuda_status(e);
}

int csa2_cache_persist(const uint8_t* codes, const uint8_t* scales, const void* ik_cache, int B,
                       int n_cap, const int32_t* N, int n_host, uint8_t* host_codes,
                       uint8_t* host_scales, void* host_ik, csa2_stream_t stream) {
  const int st = cache_copy_args_ok(codes, scales, ik_cache, B, n_cap, N, n_host, host_codes,
                                    host_scales, host_ik);
  if (st != CSA2_OK) return st;
  const cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  cudaError_t e = copy_rows(host_codes, n_host, codes, n_cap, CSA2_D / 2, B, N,
                            cudaMemcpyDeviceToHost, s);
  if (e == cudaSuccess)
    e = copy_rows(host_scales, n_host, scales, n_cap, CSA2_D / 16, B, N, cudaMemcpyDeviceToHost, s);
  if (e == cudaSuccess && ik_cache != nullptr)
    e = copy_rows(host_ik, n_host, ik_cache, n_cap, CSA2_DI * 2, B, N, cudaMemcpyDeviceToHost, s);
  return cuda_status(e);
}

size_t csa2_swa_replay_workspace_bytes(int B, int Wr, int d) {
  if (B <= 0 || Wr <= 0 || d < CSA2_CED_D_ALIGN || (d % CSA2_CED_D_ALIGN) != 0) return 0;
  return csa2::swa_replay_workspace_bytes(B, Wr, d);
}

int csa2_swa_replay(const void* h, const void* w, int B, int Wr, int d, const int32_t* N,
                    uint8_t* swa, float* swa_scale, int W, void* ws, size_t ws_bytes,
                    int32_t* dev_err, csa2_stream_t stream) {
  if (B <= 0 || Wr < 0 || W <= 0 || Wr > W) return CSA2_ERR_INVALID;
  if (d < CSA2_CED_D_ALIGN || (d % CSA2_CED_D_ALIGN) != 0) return CSA2_ERR_INVALID;
  if (B > CSA2_MAX_B || W > CSA2_MAX_W || d > CSA2_MAX_CED_D) return CSA2_ERR_UNSUPPORTED;
  if (!ptr_ok(h) || !ptr_ok(w) || !ptr_ok(N) || !ptr_ok(swa) || !ptr_ok(swa_scale))
    return CSA2_ERR_INVALID;
  if (dev_err != nullptr && (reinterpret_cast<uintptr_t>(dev_err) & 3u)) return CSA2_ERR_INVALID;
  if (Wr == 0) return CSA2_OK;
  if (ws == nullptr || !aligned16(ws) || ws_bytes < csa2::swa_replay_workspace_bytes(B, Wr, d))
    return CSA2_ERR_WORKSPACE;
  const cudaError_t launch_err = csa2::launch_swa_replay(h, w, B, Wr, d, N, swa, swa_scale, W, ws, dev_err,
                                             reinterpret_cast<cudaStream_t>(stream));
  csa2::note_call(reinterpret_cast<cudaStream_t>(stream), false);
  return cuda_status(launch_err);
}

}  // extern "C"

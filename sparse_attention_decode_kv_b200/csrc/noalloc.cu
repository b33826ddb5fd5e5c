// noalloc.cu -- csa2_index_reindex_noalloc: the Reindex-mode indexer for callers that cannot hand
// the library a scratch buffer.
//
// Some callers are not allowed to allocate device memory at the point where they run the decode
// step: a serving runtime that owns every byte of device memory through its own pool and exposes
// no way to borrow scratch from it, a plugin that receives only its input and output tensors, or
// a latency-critical loop where cudaMalloc (which can synchronise the whole device) is not
// acceptable. For them this entry point keeps its scratch in a fixed-size array that lives in the
// library's own device image: every GPU that loads libcsa2.so holds it until the process exits.
//
// The scratch holds the per-slot rank keys the two Reindex kernels exchange; each call writes
// every slot it later reads, so nothing in it has to start at zero. All calls on a device share
// the one array, so calls whose kernels overlap on that GPU (another stream, another thread)
// race on it and must be serialised by the caller.
#include <mutex>
#include <vector>

#include "common.cuh"
#include "internal.h"

namespace csa2 {
namespace {

// 2 MiB: 262,144 slots of 8 bytes (for example 16 sequences x a 16,384-slot pool).
static __device__ __align__(256) uint64_t g_reindex_scratch[CSA2_NOALLOC_REINDEX_MAX_SLOTS];

std::mutex g_scratch_mu;
// Device address of g_reindex_scratch, per device, with the context it was looked up in. A
// device's primary context can be torn down and created again (cudaDeviceReset), which loads the
// module afresh; the address is then looked up again.
struct ScratchAddr {
  void* ctx = nullptr;
  void* ptr = nullptr;
};
std::vector<ScratchAddr> g_scratch;

// cuCtxGetCurrent from the driver, looked up once through the runtime (null if unavailable, in
// which case the address is looked up on every call).
using CtxGetCurrentFn = int (*)(void**);
CtxGetCurrentFn ctx_get_current() {
  static CtxGetCurrentFn fn = [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuCtxGetCurrent", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      return reinterpret_cast<CtxGetCurrentFn>(p);
    return static_cast<CtxGetCurrentFn>(nullptr);
  }();
  return fn;
}

// The array's name is a host-side stand-in in host code; its device address is looked up at
// set-up, once per device (and again if that device's context was re-created), with that device
// current.
cudaError_t scratch_for_current_device(void** out) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  // before the runtime has made a context current the answer is null, and the address is looked
  // up (which makes it current) without being remembered
  void* ctx = nullptr;
  const CtxGetCurrentFn get = ctx_get_current();
  const bool know_ctx = get != nullptr && get(&ctx) == 0 && ctx != nullptr;
  std::lock_guard<std::mutex> lock(g_scratch_mu);
  if (dev >= static_cast<int>(g_scratch.size())) g_scratch.resize(dev + 1);
  ScratchAddr& a = g_scratch[dev];
  if (!know_ctx || a.ptr == nullptr || a.ctx != ctx) {
    void* p = nullptr;
    e = cudaGetSymbolAddress(&p, g_reindex_scratch);
    if (e != cudaSuccess) return e;
    a.ptr = p;
    a.ctx = know_ctx ? ctx : nullptr;
  }
  *out = a.ptr;
  return cudaSuccess;
}

}  // namespace
}  // namespace csa2

extern "C" int csa2_index_reindex_noalloc(const void* iq, const float* w, const void* ik_cache,
                                          const int32_t* N, int B, int n_cap,
                                          const int32_t* pool, int L, int K, int32_t* topk,
                                          int32_t* dev_err, csa2_stream_t stream) {
  if (B <= 0 || n_cap <= 0 || (n_cap % CSA2_S) != 0 || L <= 0 || K <= 0) return CSA2_ERR_INVALID;
  if (B > CSA2_MAX_B || n_cap > CSA2_MAX_NCAP || L > CSA2_MAX_POOL || K > CSA2_MAX_K)
    return CSA2_ERR_UNSUPPORTED;
  // the scratch holds one 8-byte key per (sequence, pool slot)
  if (static_cast<int64_t>(B) * L > CSA2_NOALLOC_REINDEX_MAX_SLOTS) return CSA2_ERR_UNSUPPORTED;
  auto aligned = [](const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; };
  if (!iq || !w || !ik_cache || !N || !pool || !topk) return CSA2_ERR_INVALID;
  if (!aligned(iq) || !aligned(w) || !aligned(ik_cache) || !aligned(N) || !aligned(pool) ||
      !aligned(topk))
    return CSA2_ERR_INVALID;
  if (dev_err != nullptr && (reinterpret_cast<uintptr_t>(dev_err) & 3u)) return CSA2_ERR_INVALID;
  void* scratch = nullptr;
  if (csa2::scratch_for_current_device(&scratch) != cudaSuccess) return CSA2_ERR_CUDA;
  const cudaError_t e = csa2::launch_index_reindex(iq, w, ik_cache, N, B, n_cap, pool, L, K, topk,
                                                   scratch, dev_err,
                                                   reinterpret_cast<cudaStream_t>(stream));
  csa2::note_call(reinterpret_cast<cudaStream_t>(stream), false);
  return e == cudaSuccess ? CSA2_OK : CSA2_ERR_CUDA;
}

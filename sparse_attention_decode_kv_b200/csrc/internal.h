// internal.h -- host-side launchers behind the C ABI (not part of the public interface).
#pragma once

#include <cuda.h>
#include <cuda_runtime.h>
#include <stddef.h>
#include <stdint.h>

namespace csa2 {

void count_launches(int n);   // adds to the process-wide launch counter
void profile_begin(int kernel, cudaStream_t s);  // records the start event if one is set
void profile_end(int kernel, cudaStream_t s);    // records the stop event if one is set
int device_sm_count();        // SMs of the current device (cached per device)

// The library's last call on each stream: whether it was an attention (which writes only its
// outputs and workspace). A Reuse-mode attention starts gathering before its wait only then.
void note_call(cudaStream_t s, bool is_attend);
bool last_call_was_attend(cudaStream_t s);

// cuTensorMapEncodeTiled from the driver (looked up once through the runtime), or null.
typedef CUresult (*TensorMapEncodeFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*,
                                      const cuuint64_t*, const cuuint64_t*, const cuuint32_t*,
                                      const cuuint32_t*, CUtensorMapInterleave, CUtensorMapSwizzle,
                                      CUtensorMapL2promotion, CUtensorMapFloatOOBfill);
TensorMapEncodeFn tensor_map_encoder();

// Quantize-on-append; one warp per new entry.
cudaError_t launch_append(const void* x, const void* ik, int B, int n, const int32_t* pos,
                          int n_cap, uint8_t* codes, uint8_t* scales, void* ik_cache,
                          uint8_t* swa, float* swa_scale, int W, int32_t* dev_err,
                          cudaStream_t s);

// Sparse attention (split over item tiles, merged by log-sum-exp).
size_t attend_workspace_bytes(int B, int K, int W);
int attend_split_count(int B, int K, int W);
cudaError_t launch_attend(const void* q, float softmax_scale, const uint8_t* codes,
                          const uint8_t* scales, int n_cap, const int32_t* N, const int32_t* idx,
                          int K, const uint8_t* swa, const float* swa_scale,
                          const int32_t* swa_len, int W, const int32_t* qseq,
                          const int32_t* swa_lo, int S, int nseq, int B, float* out, float* lse,
                          void* ws, int32_t* dev_err, bool early_rows, cudaStream_t s);

// Log-sum-exp merge of per-split partials (m, l, unnormalised o) into out and lse; nsplit <= 128.
constexpr int kAttendMaxSplits = 128;
cudaError_t launch_attend_merge(const float* part_o, const float* part_ml, int nsplit, int B,
                                float* out, float* lse, cudaStream_t s);

// Sparse attention on the tcgen05 tensor cores (persistent, one CTA per SM), chosen by
// launch_attend from this batch size up.
constexpr int kTcMinBatch = 64;
bool attend_tc_selected(int B, int K, int W);
int attend_tc_split_count(int B, int K, int W);
size_t attend_tc_workspace_bytes(int B, int K, int W);
cudaError_t launch_attend_tc(const void* q, float softmax_scale, const uint8_t* codes,
                             const uint8_t* scales, int n_cap, const int32_t* N, const int32_t* idx,
                             int K, const uint8_t* swa, const float* swa_scale,
                             const int32_t* swa_len, int W, const int32_t* qseq,
                             const int32_t* swa_lo, int S, int nseq, int B, float* out, float* lse,
                             void* ws, int32_t* dev_err, bool early_rows, cudaStream_t s);

// Full-mode indexer.
size_t index_full_workspace_bytes(int B, int n_cap, int K, int P);
cudaError_t launch_index_full(const void* iq, const float* w, const void* ik_cache,
                              const int32_t* N, int B, int n_cap, int K, int P, int32_t* topk,
                              int32_t* pool, void* ws, int32_t* dev_err, cudaStream_t s);

// Reindex-mode indexer.
size_t index_reindex_workspace_bytes(int B, int L, int K);
cudaError_t launch_index_reindex(const void* iq, const float* w, const void* ik_cache,
                                 const int32_t* N, int B, int n_cap, const int32_t* pool, int L,
                                 int K, int32_t* topk, void* ws, int32_t* dev_err,
                                 cudaStream_t s);

// CED KV projection with the MXFP4 quantisation in the GEMM epilogue (tcgen05).
cudaError_t launch_ced_quant(const void* h, const void* w, int B, int n, int d, const int32_t* pos,
                             int n_cap, uint8_t* codes, uint8_t* scales, int32_t* dev_err,
                             cudaStream_t s);

// SWA bounded replay: split-K tcgen05 projection of the window rows, then bf16 rounding and the
// SWA codec into the ring.
size_t swa_replay_workspace_bytes(int B, int Wr, int d);
cudaError_t launch_swa_replay(const void* h, const void* w, int B, int Wr, int d, const int32_t* N,
                              uint8_t* swa, float* swa_scale, int W, void* ws, int32_t* dev_err,
                              cudaStream_t s);

}  // namespace csa2

/*
 * csa2.h -- C ABI of libcsa2.so: the CSA2 (Compressed Sparse Attention 2) decode path over an
 * MXFP4-compressed KV cache with an FP8 sliding-window (SWA) KV, on one sm_100a GPU.
 *
 * Source of the method: "DeepSeek V4.1 Flash 拆解：KV Cache 压掉 3/4 的工程胜利，与它没解决的三个问题"
 * (austincafe.tech/?p=406), section 一:
 *   - three layer modes: Full (own main KV, own indexer, new Top-K), Reindex (reuses the main KV
 *     and the indexer keys, rescoring with its own indexer query for its own Top-K), Reuse (also
 *     reuses the Top-K and runs sparse attention directly);
 *   - hierarchical sparse indexer: the first decoder layer (Full) selects a Top-512, then builds
 *     a candidate pool of 2048 blocks x 8 positions (16,384 positions) that later layers score;
 *   - FP4 KV cache: MXFP4 = E2M1 codes plus one E4M3 scale per 16 channels; the SWA KV stays FP8.
 * and "DeepSeek-V4.1-Flash: Pushing the Limits of KV Cache Compression", abstract (cross-layer KV
 * reuse in CSA2 plus an FP4 KV cache).
 *
 * The pages give no formulas; this library computes the following readings:
 *   score      I[b,t] = sum_h w[b,h] * ReLU(iq[b,h,:] . ik[b,t,:])      (4 heads, width 64, fp32)
 *   Top-K      the K largest I by (score descending, index ascending), output ascending, -1 pad
 *   block      M[b,j] = max of I over positions 8j..8j+7 below N[b]; Top-P blocks likewise
 *   pool       positions of the selected blocks, ascending block order, -1 for positions >= N[b]
 *   MXFP4      scale = E4M3 RNE-saturating(fp32 amax/6); code = E2M1 RNE-saturating(fp32 x/scale)
 *              with the sign of x; zero scale -> zero codes
 *   SWA FP8    scale = fp32 amax/448 per token; element = E4M3 RNE-saturating(fp32 x/scale)
 *   attention  z = softmax_scale * q . v over the selected entries (v = dequantised entry, K = V)
 *              and the valid SWA rows in ONE softmax; out = sum softmax(z) v; lse = log sum e^z
 *
 * Conventions shared by every entry point:
 *   - All array pointers are DEVICE pointers, owned by the caller; the library allocates nothing,
 *     frees nothing, never synchronises and launches only on `stream` (NULL = legacy default).
 *   - Every pointer must be 16-byte aligned. bf16 arrays are raw IEEE bfloat16.
 *   - Dimensions fixed at compile time: CSA2_D = 512, CSA2_HQ = 16, CSA2_HI = 4, CSA2_DI = 64,
 *     CSA2_S = 8. n_cap (rows per sequence in the caches) must be a positive multiple of 8.
 *   - Argument and workspace errors are returned synchronously, before any launch. Launch errors
 *     return CSA2_ERR_CUDA. Conditions only the GPU can see (an index outside [0, N[b]) that is not
 *     -1, an append row outside [0, n_cap), N[b] outside [0, n_cap], a bounded wait that gave up)
 *     skip the offending item and OR a CSA2_DEVERR_* flag into *dev_err (nullable, device int32,
 *     zeroed by the caller), which the caller reads after synchronising.
 *   - Workspaces: query the byte count with the matching *_workspace_bytes function; pass a device
 *     buffer of at least that many bytes. Contents need no initialisation.
 *   - Calls that share a workspace must not overlap on the GPU.
 *   - Kernels after the first of a call are launched with programmatic dependent launch: each may
 *     start while the kernel before it on the stream finishes, and waits for it before reading
 *     anything a kernel can have produced. Kernels outside this library never trigger that early
 *     start, so their results are complete before a call begins. The attention kernels read q, N,
 *     swa_len (and qseq, swa_lo) before the wait, since no kernel of this library writes them:
 *     they must not alias memory that the preceding calls of this library on the stream write.
 *     csa2_attend in CSA2_MODE_REUSE also reads idx and the first tile's codes and scales before
 *     the wait (see there).
 */
#ifndef CSA2_H
#define CSA2_H

#include <stddef.h>
#include <stdint.h>

#if defined(__GNUC__)
#define CSA2_API __attribute__((visibility("default")))
#else
#define CSA2_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

typedef struct CUstream_st *csa2_stream_t; /* a cudaStream_t */

enum { CSA2_D = 512, CSA2_HQ = 16, CSA2_HI = 4, CSA2_DI = 64, CSA2_S = 8 };

/* Limits of this build. */
enum {
  CSA2_MAX_B = 4096,       /* sequences per call */
  CSA2_MAX_K = 4096,       /* Top-K of the indexers; indices per sequence for attention */
  CSA2_MAX_P = 4096,       /* pool blocks */
  CSA2_MAX_POOL = 32768,   /* pool slots scored by a Reindex call */
  CSA2_MAX_W = 4096,       /* SWA ring length; SWA rows one query attends to */
  CSA2_MAX_QUERIES = 1 << 20,   /* queries of one csa2_attend_queries call */
  CSA2_MAX_SWA_ROWS = 1 << 24,  /* rows per sequence of the SWA buffer of csa2_attend_queries */
  CSA2_MAX_NCAP = 1 << 28  /* rows per sequence */
};

typedef enum {
  CSA2_OK = 0,
  CSA2_ERR_INVALID = -1,     /* null or misaligned pointer, non-positive or inconsistent size */
  CSA2_ERR_UNSUPPORTED = -2, /* a size beyond the limits above */
  CSA2_ERR_WORKSPACE = -3,   /* workspace smaller than the matching *_workspace_bytes */
  CSA2_ERR_CUDA = -4,        /* a CUDA runtime or launch error */
  CSA2_ERR_DEVICE = -5,      /* reserved for callers that fold *dev_err into a status */
  CSA2_ERR_TIMEOUT = -6      /* reserved for callers that fold CSA2_DEVERR_TIMEOUT into a status */
} csa2_status;

typedef enum { CSA2_MODE_FULL = 0, CSA2_MODE_REINDEX = 1, CSA2_MODE_REUSE = 2 } csa2_mode;

/* Flags OR-ed into *dev_err by the kernels. */
#define CSA2_DEVERR_INDEX_RANGE 1 /* an index outside [0, N[b]) (not -1) was skipped */
#define CSA2_DEVERR_POS_RANGE 2   /* an append row outside [0, n_cap) was skipped */
#define CSA2_DEVERR_TIMEOUT 4     /* a bounded wait inside a kernel gave up */
#define CSA2_DEVERR_NLEN 8        /* N[b] (or swa_len[b]) outside its valid range was clamped */

/*
 * Quantize-on-append (MXFP4 main KV, FP8 SWA ring, indexer-key copy).
 * Defines: the FP4 KV cache paragraph of section 一 (E2M1 + one E4M3 scale per 16 channels; SWA
 * KV stays FP8).
 *   x         bf16 [B, n, 512]: the new main-KV entries.
 *   ik        bf16 [B, n, 64]: their indexer keys, or NULL (then ik_cache is not written).
 *   pos       int32 [B] (device): row of the first new entry of each sequence; entry i of
 *             sequence b goes to row pos[b] + i.
 *   codes     uint8 [B, n_cap, 256]: E2M1 codes, channel 2j in the low nibble of byte j.
 *   scales    uint8 [B, n_cap, 32]: E4M3 scale of channels 16g..16g+15 in byte g.
 *   ik_cache  bf16 [B, n_cap, 64].
 *   swa       uint8 [B, W, 512] E4M3 ring (token at position p in slot p mod W; only the last W
 *             of the n new tokens are written) and swa_scale float [B, W]; both NULL or W = 0 to
 *             skip the ring.
 * Rows outside [0, n_cap) are skipped with CSA2_DEVERR_POS_RANGE.
 */
CSA2_API int csa2_append_quant(const void *x, const void *ik, int B, int n, const int32_t *pos, int n_cap,
                      uint8_t *codes, uint8_t *scales, void *ik_cache, uint8_t *swa,
                      float *swa_scale, int W, int32_t *dev_err, csa2_stream_t stream);

/*
 * CED KV projection with the MXFP4 quantisation in the GEMM epilogue: C = h w^T (bf16 inputs,
 * fp32 accumulation on the tcgen05 tensor cores), each 16-channel group of a row of C quantised
 * with csa2_append_quant's codec applied to the fp32 values (scale = E4M3 RNE of the fp32
 * quotient amax/6, codes = E2M1 RNE of the fp32 quotients x/scale), and the codes and scales
 * written to the cache rows; the projection output never reaches memory.
 * Defines: the CED paragraph of section 一 (the decoder layers' global KV is projected from the
 * middle layer's hidden state, C_l = H_{L/2} W^KV_l) with the FP4 KV cache paragraph.
 *   h         bf16 [B, n, d]: hidden states of the n new tokens of each sequence (row-major).
 *   w         bf16 [512, d]: the layer's KV projection, one row per latent channel (the layout of
 *             a linear layer's weight).
 *   d         a multiple of CSA2_CED_D_ALIGN (64), at most CSA2_MAX_CED_D.
 *   pos, n_cap, codes, scales: as csa2_append_quant (token i of sequence b goes to row pos[b]+i).
 * Rows outside [0, n_cap) are skipped with CSA2_DEVERR_POS_RANGE. B * n is at most
 * CSA2_MAX_CED_TOKENS. No workspace; launches one kernel (clusters of two CTAs sharing each
 * MMA when B * n >= 256, single CTAs below).
 */
enum { CSA2_CED_D_ALIGN = 64, CSA2_MAX_CED_D = 65536, CSA2_MAX_CED_TOKENS = 1 << 26 };
CSA2_API int csa2_ced_project_quant(const void *h, const void *w, int B, int n, int d,
                                    const int32_t *pos, int n_cap, uint8_t *codes,
                                    uint8_t *scales, int32_t *dev_err, csa2_stream_t stream);

/*
 * SWA bounded replay, part 1: restore a persisted sequence's cache rows from host memory.
 * Defines: "DeepSeek-V4.1-Flash: Pushing the Limits of KV Cache Compression", abstract (SWA
 * Bounded Replay brings the persistent KV cache on SSD or in host memory to about 1/8 of
 * DeepSeek-V4-Flash's), and the Juju Radar note on that report (the persistent cache rebuilds
 * the local sliding-window state instead of storing it). Reading: what persists is the global KV
 * (MXFP4 codes and scales) and the indexer keys; the FP8 SWA ring is rebuilt by
 * csa2_swa_replay.
 *   host_codes   uint8 [B, n_host, 256], host_scales uint8 [B, n_host, 32], host_ik bf16
 *                [B, n_host, 64] or NULL: the persisted rows (host memory; page-locked memory
 *                lets the copies run asynchronously on the stream, pageable memory makes the
 *                call return only after them).
 *   N            HOST int32 [B]: rows 0 .. N[b]-1 of sequence b are copied; 0 <= N[b] <=
 *                min(n_host, n_cap).
 *   codes, scales, ik_cache: the device cache (as csa2_append_quant); ik_cache NULL exactly when
 *                host_ik is NULL. Rows N[b] .. n_cap-1 are not touched.
 * Copies only (cudaMemcpyAsync on the stream; runs of full sequences are merged into one copy);
 * launches no kernel. Errors: CSA2_ERR_INVALID for bad sizes or pointers, CSA2_ERR_CUDA when a
 * copy cannot be queued.
 */
CSA2_API int csa2_cache_restore(const uint8_t *host_codes, const uint8_t *host_scales,
                                const void *host_ik, int B, int n_host, const int32_t *N,
                                int n_cap, uint8_t *codes, uint8_t *scales, void *ik_cache,
                                csa2_stream_t stream);

/*
 * The inverse copy: rows 0 .. N[b]-1 of the device cache to the host layout above (the state a
 * later csa2_cache_restore reads). Same arguments, same rules, directions swapped.
 */
CSA2_API int csa2_cache_persist(const uint8_t *codes, const uint8_t *scales, const void *ik_cache,
                                int B, int n_cap, const int32_t *N, int n_host,
                                uint8_t *host_codes, uint8_t *host_scales, void *host_ik,
                                csa2_stream_t stream);

/*
 * SWA bounded replay, part 2: rebuild the FP8 SWA ring of B restored sequences from the hidden
 * states of their last Wr tokens (same sources as csa2_cache_restore). Token r of sequence b is
 * position p = N[b] - Wr + r; its SWA row is x = bf16_RNE(h w^T) (bf16 inputs, fp32 accumulation
 * on the tcgen05 tensor cores), quantised with csa2_append_quant's SWA codec into ring slot
 * p mod W, so the slot holds exactly what an append of x at position p would have written.
 * Positions p < 0 (a sequence shorter than the window) are skipped; other slots are not touched.
 *   h         bf16 [B, Wr, d]: hidden states of the window tokens, oldest first.
 *   w         bf16 [512, d]: the layer's SWA KV projection, one row per channel.
 *   d         a multiple of CSA2_CED_D_ALIGN (64), at most CSA2_MAX_CED_D.
 *   N         device int32 [B]: tokens in each sequence (a negative N[b] skips the sequence and
 *             flags CSA2_DEVERR_NLEN).
 *   swa, swa_scale, W: the ring (as csa2_append_quant); 1 <= Wr <= W.
 *   ws        device workspace of csa2_swa_replay_workspace_bytes(B, Wr, d) bytes (fp32 partial
 *             sums of the split reduction), 16-byte aligned.
 * Launches two kernels (the split-K projection and the sum-round-quantise pass).
 */
CSA2_API size_t csa2_swa_replay_workspace_bytes(int B, int Wr, int d);
CSA2_API int csa2_swa_replay(const void *h, const void *w, int B, int Wr, int d, const int32_t *N,
                             uint8_t *swa, float *swa_scale, int W, void *ws, size_t ws_bytes,
                             int32_t *dev_err, csa2_stream_t stream);

/*
 * Full-mode indexer: scores every entry, selects the Top-K positions, takes block maxima over
 * 8-position blocks, selects the Top-P blocks and writes the pool.
 * Defines: the hierarchical sparse indexer paragraph of section 一 (Top-512, 2048 blocks x 8).
 *   iq        bf16 [B, 4, 64]: the layer's indexer query; w float [B, 4]: head weights.
 *   ik_cache  bf16 [B, n_cap, 64]; N int32 [B] (device): entries per sequence (0 <= N <= n_cap).
 *   topk      int32 [B, K] out: ascending positions, -1 padded when N[b] < K.
 *   pool      int32 [B, 8P] out: the selected blocks' positions (ascending block order), -1 for
 *             positions >= N[b] and for unused blocks.
 * Layout contract: the workspace starts with the fp32 scores I [B, n_cap] (valid for t < N[b]);
 * the fp32 block maxima [B, n_cap/8] follow at byte offset 4*B*n_cap rounded up to a multiple of
 * 256. Both stay readable until the workspace is reused.
 */
CSA2_API size_t csa2_index_full_workspace_bytes(int B, int n_cap, int K, int P);
CSA2_API int csa2_index_full(const void *iq, const float *w, const void *ik_cache, const int32_t *N, int B,
                    int n_cap, int K, int P, int32_t *topk, int32_t *pool, void *ws,
                    size_t ws_bytes, int32_t *dev_err, csa2_stream_t stream);

/*
 * Reindex-mode indexer: the layer's own iq/w score only the pool positions (-1 slots skipped);
 * Top-K by (score descending, position ascending); output ascending, -1 padded.
 * Defines: the Reindex mode of section 一 (reuse the main KV and indexer keys, rescore with the
 * layer's own indexer query, choose its own Top-K) and the pool of the hierarchical indexer.
 *   pool      int32 [B, L]: distinct positions or -1 (typically the Full layer's pool, L = 8P).
 *   Positions outside [0, N[b]) other than -1 are skipped with CSA2_DEVERR_INDEX_RANGE.
 */
CSA2_API size_t csa2_index_reindex_workspace_bytes(int B, int L, int K);
CSA2_API int csa2_index_reindex(const void *iq, const float *w, const void *ik_cache, const int32_t *N,
                       int B, int n_cap, const int32_t *pool, int L, int K, int32_t *topk,
                       void *ws, size_t ws_bytes, int32_t *dev_err, csa2_stream_t stream);

/*
 * Allocation-free Reindex-mode indexer (no counterpart on the pages; an interface addition).
 * Same arguments and results as csa2_index_reindex without the workspace: for callers that may
 * not allocate device memory where they run the decode step (a serving runtime that owns all
 * device memory through its own pool, a plugin handed only its tensors, a latency-critical loop
 * that cannot afford cudaMalloc's device-wide synchronisation). The scratch is a fixed array of
 * CSA2_NOALLOC_REINDEX_MAX_SLOTS 8-byte slots (2 MiB) inside the library's device image, held by
 * every GPU that loads the library until the process exits; B * L above that limit returns
 * CSA2_ERR_UNSUPPORTED. The first call on a device looks up the array's device address for that
 * device (make that first call before any stream capture); a call after the device's context was
 * re-created (cudaDeviceReset) looks it up again. All calls on a device share the
 * array: calls whose kernels overlap on the GPU race and must be serialised by the caller. The
 * array needs no clearing: each call writes every slot it reads. It allocates nothing.
 */
enum { CSA2_NOALLOC_REINDEX_MAX_SLOTS = 262144 };
CSA2_API int csa2_index_reindex_noalloc(const void *iq, const float *w, const void *ik_cache,
                                        const int32_t *N, int B, int n_cap, const int32_t *pool,
                                        int L, int K, int32_t *topk, int32_t *dev_err,
                                        csa2_stream_t stream);

/*
 * Sparse attention over the selected MXFP4 entries and the FP8 SWA rows, all 16 heads.
 * Defines: Reuse mode of section 一 ("sparse attention directly" over reused indices) and the
 * FP8 SWA KV. `mode` records which kind of layer produced idx; it does not change the result
 * (attend(REUSE, idx) == attend(FULL, idx) bit for bit). A Reuse layer's indices, and the cache
 * rows they name, were produced by an earlier layer, so with CSA2_MODE_REUSE the kernel starts
 * gathering them before it waits for the preceding kernel on the stream. It does so only when
 * the library's previous call on the same stream was csa2_attend or csa2_attend_queries (which
 * write only out, lse and their workspace), as in a decode step's run of Reuse layers; after any
 * other call of the library on the stream (an append, an index call, a CED projection, a cache
 * restore or a replay, which may write idx or the rows) it waits first. The library sees only
 * its own calls: the caller guarantees that no other code on the stream writes idx or the
 * entries' codes and scales between that attention and this one.
 *   q         bf16 [B, 16, 512]; every |q| must be below 65504 (fp16 range).
 *   codes/scales as written by csa2_append_quant; N int32 [B] (device).
 *   idx       int32 [B, K]: entry positions, -1 = none; duplicates count as separate entries.
 *   swa, swa_scale as written by csa2_append_quant, with W slots; swa_len int32 [B] (device):
 *             slots 0..swa_len[b]-1 are valid (min(tokens seen, W)); swa may be NULL iff W = 0.
 *   out       float [B, 16, 512]; lse float [B, 16] or NULL. An empty set gives out = 0,
 *             lse = -inf.
 */
CSA2_API size_t csa2_attend_workspace_bytes(int B, int K, int W);
CSA2_API int csa2_attend(int mode, const void *q, float softmax_scale, const uint8_t *codes,
                const uint8_t *scales, int n_cap, const int32_t *N, const int32_t *idx, int K,
                const uint8_t *swa, const float *swa_scale, const int32_t *swa_len, int W, int B,
                float *out, float *lse, void *ws, size_t ws_bytes, int32_t *dev_err,
                csa2_stream_t stream);

/*
 * Sparse attention of many queries per sequence (prefill, or verification of several drafted
 * tokens): query b reads the cache of sequence qseq[b], its own K indices idx[b] and the SWA
 * rows swa_lo[b] .. swa_lo[b] + swa_len[b] - 1 of that sequence's FP8 buffer; otherwise the same
 * computation as csa2_attend (which is the case of one query per sequence and the ring).
 * Defines: the Reuse mode of section 一 in prefill (each prompt token's layer attends to its own
 * selected entries plus its sliding window) and the 15-kernel prefill flow of section 二.
 *   q         bf16 [Q, 16, 512]; out float [Q, 16, 512]; lse float [Q, 16] or NULL.
 *   codes, scales, N: B cache sequences as for csa2_attend.
 *   qseq      int32 [Q] (device): sequence of each query; entries outside [0, B) give an empty
 *             query and CSA2_DEVERR_INDEX_RANGE.
 *   idx       int32 [Q, K]: entry positions of each query, -1 = none.
 *   swa       uint8 [B, S, 512] E4M3 rows and swa_scale float [B, S] (fp32 per-row scales);
 *             swa_lo, swa_len int32 [Q] (device): the query's rows, 0 <= swa_len <= W <= S
 *             (out-of-range windows are clamped and flagged with CSA2_DEVERR_NLEN). W = 0: no
 *             SWA rows, and swa, swa_scale, swa_lo, swa_len may be NULL.
 *   ws        csa2_attend_workspace_bytes(Q, K, W) bytes.
 */
CSA2_API int csa2_attend_queries(const void *q, float softmax_scale, const uint8_t *codes,
                                 const uint8_t *scales, int B, int n_cap, const int32_t *N,
                                 const int32_t *qseq, const int32_t *idx, int K,
                                 const uint8_t *swa, const float *swa_scale, int S,
                                 const int32_t *swa_lo, const int32_t *swa_len, int W, int Q,
                                 float *out, float *lse, void *ws, size_t ws_bytes,
                                 int32_t *dev_err, csa2_stream_t stream);

/*
 * Profiling hook (no counterpart on the pages): when events are set for a kernel id, every later
 * launch of that kernel is bracketed by cudaEventRecord(start) / cudaEventRecord(stop) on the
 * launching stream, so cudaEventElapsedTime gives the last launch's device time (this also works
 * inside stream capture, where the records become graph nodes). Pass NULL events to clear.
 * Process-wide and not synchronised: set it while no other thread is calling the library.
 */
enum {
  CSA2_KERNEL_APPEND = 0,      /* append_kernel */
  CSA2_KERNEL_INDEX_SCAN = 1,  /* Full-mode score scan (the O(N) kernel) */
  CSA2_KERNEL_INDEX_SELECT = 2,/* Full-mode candidate collect + final select (two kernels) */
  CSA2_KERNEL_REINDEX = 3,     /* Reindex score + select (two kernels) */
  CSA2_KERNEL_ATTEND = 4,      /* attention + merge (one or two kernels) */
  CSA2_KERNEL_CED = 5,         /* CED projection with the MXFP4 epilogue */
  CSA2_KERNEL_REPLAY = 6,      /* SWA replay: projection + sum/round/quantise (two kernels) */
  CSA2_KERNEL_COUNT = 7
};
CSA2_API int csa2_set_profile_events(int kernel, void *start_event, void *stop_event);

/* Human-readable name of a csa2_status value (static storage). */
CSA2_API const char *csa2_status_string(int status);

/* Number of kernels this library has launched in this process (all threads, all devices). */
CSA2_API uint64_t csa2_launch_count(void);

/* ABI version of this header (bumped on any signature change). */
CSA2_API int csa2_abi_version(void);

#ifdef __cplusplus
}
#endif
#endif /* CSA2_H */

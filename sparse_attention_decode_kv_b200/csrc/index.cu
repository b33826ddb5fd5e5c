// index.cu -- the CSA2 indexers: Full mode (score every entry, Top-K positions, block maxima,
// Top-P blocks, pool) and Reindex mode (score the pool with the layer's own query, Top-K).
//
// Method: "DeepSeek V4.1 Flash 拆解" (austincafe.tech), section 一: the first decoder layer (Full)
// selects a Top-512 and builds a pool of 2048 blocks x 8 positions; later layers (Reindex) score
// only that pool with their own indexer query and pick their own Top-K.
// Readings: I[b,t] = sum_h w_h ReLU(iq_h . ik_t) (4 heads, width 64, one key per entry); block
// score = max of I over the block's positions below N; ranking by (score desc, index asc).
//
// Full mode, three kernels on the caller's stream:
//   index_scan_kernel   persistent, one CTA per SM. One producer thread streams 128-entry key
//                       tiles (16 KiB, 128-byte swizzle) with cp.async.bulk.tensor into a
//                       6-stage mbarrier ring; 8 consumer warps run the 4-head q.K contraction
//                       on the tensor cores (m16n8k16 bf16, keys on M, heads padded to N = 8),
//                       then ReLU, weights, fp32 score store, block max over 8 positions and
//                       4096-bin histograms (top 12 key bits) of scores and block maxima.
//   topk_collect_kernel every CTA finds the histogram bin holding the K-th score (P-th block)
//                       and appends the rank keys of all items in or above that bin to a
//                       candidate buffer (warp-aggregated atomics).
//   topk_final_kernel   one CTA per (sequence, positions|blocks): exact radix select over the
//                       candidates (or, if they overflowed, over the full score array), bitonic
//                       sort of the winners by index, then topk / pool output.
// Every mbarrier wait is bounded; a timeout flags CSA2_DEVERR_TIMEOUT and the CTA drains its own
// bulk copies before exiting.
#include <mutex>
#include <vector>

#include "common.cuh"
#include "internal.h"
#include "select.cuh"

namespace csa2 {

namespace {

constexpr int kScanTile = 128;                    // entries per TMA tile
constexpr int kScanTileBytes = kScanTile * DI * 2;  // 16 KiB
constexpr int kScanStages = 6;
constexpr int kScanConsumerWarps = 8;             // 16 entries each per tile
constexpr int kScanThreads = (kScanConsumerWarps + 1) * 32;
constexpr int kCand = 16384;                      // candidate slots per (sequence, problem)
constexpr int kCollectChunk = 8192;
constexpr int kCollectThreads = 256;
constexpr int kFinalThreads = 1024;
constexpr int kMaxSel = 4096;                     // >= CSA2_MAX_K, CSA2_MAX_P

static_assert(kScanTileBytes == 16384, "tile size");

struct __align__(1024) ScanSmem {
  uint8_t tiles[kScanStages][kScanTileBytes];
  uint64_t full[kScanStages];
  uint64_t empty[kScanStages];
  uint32_t hist[2][kHistBins];
  int abort;
};

__device__ __forceinline__ void consumer_bar() {
  asm volatile("bar.sync 1, %0;" ::"n"(kScanConsumerWarps * 32) : "memory");
}

__device__ __forceinline__ bool wait_or_abort(uint64_t* bar, uint32_t parity, volatile int* abort) {
  if (mbar_try_wait(bar, parity)) return true;
  const uint64_t t0 = globaltimer_ns();
  while (!mbar_try_wait(bar, parity)) {
    if (*abort) return false;
    if (globaltimer_ns() - t0 > kWaitLimitNs) return false;
  }
  return true;
}

__device__ __forceinline__ int clamp_len(const int32_t* N, int b, int n_cap, int32_t* dev_err) {
  int nb = __ldg(N + b);
  if (nb < 0 || nb > n_cap) {
    flag_error(dev_err, CSA2_DEVERR_NLEN);
    nb = max(0, min(nb, n_cap));
  }
  return nb;
}

__global__ void __launch_bounds__(kScanThreads, 1)
    index_scan_kernel(const __grid_constant__ CUtensorMap keys, const uint16_t* __restrict__ iq,
                      const float* __restrict__ w, const int32_t* __restrict__ N, int B,
                      int n_cap, float* __restrict__ scores, float* __restrict__ bmax,
                      uint32_t* __restrict__ hist_g, int32_t* dev_err) {
  extern __shared__ __align__(1024) unsigned char smem_raw[];
  ScanSmem& sm = *reinterpret_cast<ScanSmem*>(smem_raw);
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int tiles_per_seq = (n_cap + kScanTile - 1) / kScanTile;
  const int64_t total = static_cast<int64_t>(B) * tiles_per_seq;
  const int64_t v_begin = total * blockIdx.x / gridDim.x;
  const int64_t v_end = total * (blockIdx.x + 1) / gridDim.x;

  for (int i = tid; i < 2 * kHistBins; i += kScanThreads) (&sm.hist[0][0])[i] = 0u;
  if (tid == 0) {
    for (int s = 0; s < kScanStages; ++s) {
      mbar_init(&sm.full[s], 1);
      mbar_init(&sm.empty[s], kScanConsumerWarps);
    }
    sm.abort = 0;
    fence_barrier_init();
  }
  __syncthreads();
  volatile int* abort = &sm.abort;

  if (warp == kScanConsumerWarps) {
    // ------------------------------------------------------------------ producer (one thread)
    if (lane == 0) {
      const uint64_t policy = l2_policy_evict_first();
      int64_t it = 0;
      for (int64_t v = v_begin; v < v_end && !*abort; ++v) {
        const int b = static_cast<int>(v / tiles_per_seq);
        const int t = static_cast<int>(v - static_cast<int64_t>(b) * tiles_per_seq);
        const int nb = max(0, min(__ldg(N + b), n_cap));
        if (t * kScanTile >= nb) continue;
        const int stage = static_cast<int>(it % kScanStages);
        const int64_t round = it / kScanStages;
        if (round > 0 && !wait_or_abort(&sm.empty[stage], static_cast<uint32_t>((round - 1) & 1), abort)) {
          flag_error(dev_err, CSA2_DEVERR_TIMEOUT);
          *abort = 1;
          break;
        }
        mbar_arrive_expect_tx(&sm.full[stage], kScanTileBytes);
        tma_load_3d(sm.tiles[stage], &keys, &sm.full[stage], 0, t * kScanTile, b, policy);
        ++it;
      }
      // drain: every issued copy must land before the CTA may exit
      const int64_t first = it > kScanStages ? it - kScanStages : 0;
      for (int64_t j = first; j < it; ++j) {
        const int stage = static_cast<int>(j % kScanStages);
        if (!mbar_wait(&sm.full[stage], static_cast<uint32_t>((j / kScanStages) & 1)))
          flag_error(dev_err, CSA2_DEVERR_TIMEOUT);
      }
    }
    return;
  }

  // -------------------------------------------------------------------- consumers (8 warps)
  const int g = lane >> 2, c = lane & 3;
  const int mi = lane >> 3;
  const int a_row = 16 * warp + (lane & 7) + ((mi & 1) << 3);
  int cur_b = -1, nb = 0;
  uint32_t bq0[4], bq1[4];
  float wa = 0.0f, wb = 0.0f;
  int64_t it = 0;

  auto flush = [&](int bseq) {
    consumer_bar();
    for (int i = tid; i < 2 * kHistBins; i += kScanConsumerWarps * 32) {
      const uint32_t v = (&sm.hist[0][0])[i];
      if (v) {
        atomicAdd(hist_g + static_cast<int64_t>(bseq) * 2 * kHistBins + i, v);
        (&sm.hist[0][0])[i] = 0u;
      }
    }
    consumer_bar();
  };

  for (int64_t v = v_begin; v < v_end; ++v) {
    const int b = static_cast<int>(v / tiles_per_seq);
    const int t = static_cast<int>(v - static_cast<int64_t>(b) * tiles_per_seq);
    if (b != cur_b) {
      if (cur_b >= 0) flush(cur_b);
      cur_b = b;
      nb = clamp_len(N, b, n_cap, lane == 0 && warp == 0 ? dev_err : nullptr);
      // B fragments: head g (< 4) of iq[b]; heads 4..7 are zero padding
#pragma unroll
      for (int s = 0; s < 4; ++s) {
        bq0[s] = bq1[s] = 0u;
        if (g < HI) {
          const uint32_t* qrow = reinterpret_cast<const uint32_t*>(iq + (static_cast<int64_t>(b) * HI + g) * DI);
          bq0[s] = __ldg(qrow + 8 * s + c);
          bq1[s] = __ldg(qrow + 8 * s + 4 + c);
        }
      }
      wa = c < 2 ? __ldg(w + b * HI + 2 * c) : 0.0f;
      wb = c < 2 ? __ldg(w + b * HI + 2 * c + 1) : 0.0f;
    }
    if (t * kScanTile >= nb) continue;
    const int stage = static_cast<int>(it % kScanStages);
    const uint32_t parity = static_cast<uint32_t>((it / kScanStages) & 1);
    ++it;
    // every lane waits (acquiring the tile), the warp then takes one decision
    const bool ok = __all_sync(0xFFFFFFFFu, !*abort && wait_or_abort(&sm.full[stage], parity, abort));
    if (!ok) {
      if (lane == 0 && !*abort) flag_error(dev_err, CSA2_DEVERR_TIMEOUT);
      *abort = 1;
      continue;
    }

    float acc[4] = {0.0f, 0.0f, 0.0f, 0.0f};
    const uint32_t tile = smem_u32(sm.tiles[stage]);
#pragma unroll
    for (int s = 0; s < 4; ++s) {
      const int chunk = 2 * s + (mi >> 1);
      uint32_t a0, a1, a2, a3;
      ldsm_x4(tile + a_row * 128 + ((chunk ^ (a_row & 7)) << 4), a0, a1, a2, a3);
      mma_bf16_16816(acc, a0, a1, a2, a3, bq0[s], bq1[s]);
    }
    __syncwarp();
    if (lane == 0) mbar_arrive(&sm.empty[stage]);

    // scores of rows g and g+8 (lanes c = 0 and 1 hold heads 0,1 and 2,3)
    float s0 = wa * fmaxf(acc[0], 0.0f) + wb * fmaxf(acc[1], 0.0f);
    float s1 = wa * fmaxf(acc[2], 0.0f) + wb * fmaxf(acc[3], 0.0f);
    s0 += __shfl_xor_sync(0xFFFFFFFFu, s0, 1);
    s1 += __shfl_xor_sync(0xFFFFFFFFu, s1, 1);
    s0 += 0.0f;  // fold -0 onto +0
    s1 += 0.0f;
    const int t0 = t * kScanTile + 16 * warp + g, t1 = t0 + 8;
    const bool v0 = t0 < nb, v1 = t1 < nb;
    if (c == 0) {
      float* srow = scores + static_cast<int64_t>(b) * n_cap;
      if (v0) {
        srow[t0] = s0;
        atomicAdd(&sm.hist[0][float_key(s0) >> kHistShift], 1u);
      }
      if (v1) {
        srow[t1] = s1;
        atomicAdd(&sm.hist[0][float_key(s1) >> kHistShift], 1u);
      }
    }
    float m0 = v0 ? s0 : -INFINITY, m1 = v1 ? s1 : -INFINITY;
#pragma unroll
    for (int off = 4; off < 32; off <<= 1) {
      m0 = fmaxf(m0, __shfl_xor_sync(0xFFFFFFFFu, m0, off));
      m1 = fmaxf(m1, __shfl_xor_sync(0xFFFFFFFFu, m1, off));
    }
    if (lane == 0) {
      const int j0 = (t * kScanTile + 16 * warp) / S;
      float* brow = bmax + static_cast<int64_t>(b) * (n_cap / S);
      if (j0 * S < nb) {
        brow[j0] = m0;
        atomicAdd(&sm.hist[1][float_key(m0) >> kHistShift], 1u);
      }
      if ((j0 + 1) * S < nb) {
        brow[j0 + 1] = m1;
        atomicAdd(&sm.hist[1][float_key(m1) >> kHistShift], 1u);
      }
    }
  }
  if (cur_b >= 0) flush(cur_b);
}

__global__ void __launch_bounds__(kCollectThreads)
    topk_collect_kernel(const float* __restrict__ scores, const float* __restrict__ bmax,
                        const int32_t* __restrict__ N, int n_cap, int K, int P,
                        const uint32_t* __restrict__ hist_g, uint32_t* __restrict__ cnt,
                        uint64_t* __restrict__ cand) {
  __shared__ uint32_t part[kCollectThreads];
  __shared__ int bin_sh;
  const int b = blockIdx.y, prob = blockIdx.z;
  const int nb = max(0, min(__ldg(N + b), n_cap));
  const int n_items = prob == 0 ? nb : (nb + S - 1) / S;
  const int k_take = min(prob == 0 ? K : P, n_items);
  const int start = blockIdx.x * kCollectChunk;
  if (k_take == 0 || start >= n_items) return;
  const int64_t pr = static_cast<int64_t>(b) * 2 + prob;
  const int T0 = block_find_bin4096(hist_g + pr * kHistBins, static_cast<uint32_t>(k_take), part,
                                    &bin_sh);
  const float* src = prob == 0 ? scores + static_cast<int64_t>(b) * n_cap
                               : bmax + static_cast<int64_t>(b) * (n_cap / S);
  uint32_t* counter = cnt + pr;
  uint64_t* out = cand + pr * kCand;
  const int end = min(start + kCollectChunk, n_items);
  const int lane = threadIdx.x & 31;
  for (int i0 = start; i0 < end; i0 += kCollectThreads) {
    const int i = i0 + threadIdx.x;
    float v = 0.0f;
    bool take = false;
    if (i < end) {
      v = src[i];
      take = static_cast<int>(float_key(v) >> kHistShift) >= T0;
    }
    const uint32_t ball = __ballot_sync(0xFFFFFFFFu, take);
    if (ball == 0) continue;
    uint32_t base = 0;
    if (lane == 0) base = atomicAdd(counter, __popc(ball));
    base = __shfl_sync(0xFFFFFFFFu, base, 0);
    if (take) {
      const uint32_t slot = base + __popc(ball & ((1u << lane) - 1u));
      if (slot < kCand) out[slot] = rank_key(v, static_cast<uint32_t>(i));
    }
  }
}

struct FinalSmem {
  uint64_t cand[kCand];
  int32_t sel[kMaxSel];
  uint32_t hist[256];
  RadixState st;
  int nsel;
};

__global__ void __launch_bounds__(kFinalThreads)
    topk_final_kernel(const float* __restrict__ scores, const float* __restrict__ bmax,
                      const int32_t* __restrict__ N, int n_cap, int K, int P,
                      const uint32_t* __restrict__ cnt, const uint64_t* __restrict__ cand,
                      int32_t* __restrict__ topk, int32_t* __restrict__ pool) {
  extern __shared__ __align__(1024) unsigned char smem_raw[];
  FinalSmem& sm = *reinterpret_cast<FinalSmem*>(smem_raw);
  const int b = blockIdx.x, prob = blockIdx.y, tid = threadIdx.x;
  const int nb = max(0, min(__ldg(N + b), n_cap));
  const int n_items = prob == 0 ? nb : (nb + S - 1) / S;
  const int kk = prob == 0 ? K : P;
  const int k_take = min(kk, n_items);
  const int64_t pr = static_cast<int64_t>(b) * 2 + prob;
  const uint32_t count = cnt[pr];
  if (tid == 0) sm.nsel = 0;

  if (k_take > 0 && count <= static_cast<uint32_t>(kCand)) {
    const uint64_t* src = cand + pr * kCand;
    for (int i = tid; i < static_cast<int>(count); i += kFinalThreads) sm.cand[i] = src[i];
    __syncthreads();
    const uint64_t* c = sm.cand;
    auto get = [c](int i) { return c[i]; };
    block_radix_select(get, static_cast<int>(count), static_cast<uint32_t>(k_take), sm.hist, &sm.st);
    const RadixState st = sm.st;
    for (int i = tid; i < static_cast<int>(count); i += kFinalThreads) {
      const uint64_t key = c[i];
      if (radix_selected(key, st)) {
        const int slot = atomicAdd(&sm.nsel, 1);
        if (slot < kMaxSel) sm.sel[slot] = static_cast<int32_t>(rank_key_index(key));
      }
    }
  } else if (k_take > 0) {
    // candidate overflow (many near-equal scores): exact select over the whole array
    const float* arr = prob == 0 ? scores + static_cast<int64_t>(b) * n_cap
                                 : bmax + static_cast<int64_t>(b) * (n_cap / S);
    auto get = [arr](int i) { return rank_key(arr[i], static_cast<uint32_t>(i)); };
    __syncthreads();
    block_radix_select(get, n_items, static_cast<uint32_t>(k_take), sm.hist, &sm.st);
    const RadixState st = sm.st;
    for (int i = tid; i < n_items; i += kFinalThreads) {
      if (radix_selected(get(i), st)) {
        const int slot = atomicAdd(&sm.nsel, 1);
        if (slot < kMaxSel) sm.sel[slot] = i;
      }
    }
  }
  __syncthreads();
  int n2 = 1;
  while (n2 < k_take) n2 <<= 1;
  for (int i = k_take + tid; i < n2; i += kFinalThreads) sm.sel[i] = 0x7FFFFFFF;
  __syncthreads();
  if (k_take > 1) block_bitonic_sort_i32(sm.sel, n2);
  if (prob == 0) {
    int32_t* dst = topk + static_cast<int64_t>(b) * K;
    for (int i = tid; i < K; i += kFinalThreads) dst[i] = i < k_take ? sm.sel[i] : -1;
  } else {
    int32_t* dst = pool + static_cast<int64_t>(b) * P * S;
    for (int i = tid; i < P * S; i += kFinalThreads) {
      const int j = i / S, r = i % S;
      int v = -1;
      if (j < k_take) {
        const int p = sm.sel[j] * S + r;
        v = p < nb ? p : -1;
      }
      dst[i] = v;
    }
  }
}

// ------------------------------------------------------------------------------------ Reindex

constexpr int kReSlotsPerCta = 256;
constexpr int kReThreads = 256;

// 8 lanes per pool slot, 8 dims (16 bytes of key) per lane; writes the slot's rank key (0 for an
// empty or out-of-range slot, which is below every real key).
__global__ void __launch_bounds__(kReThreads)
    reindex_score_kernel(const uint16_t* __restrict__ iq, const float* __restrict__ w,
                         const uint16_t* __restrict__ ik_cache, const int32_t* __restrict__ N,
                         int n_cap, const int32_t* __restrict__ pool, int L,
                         uint64_t* __restrict__ keys, int32_t* dev_err) {
  const int b = blockIdx.y;
  const int lane = threadIdx.x & 31, sub = lane & 7;
  const int nb = clamp_len(N, b, n_cap, threadIdx.x == 0 && blockIdx.x == 0 ? dev_err : nullptr);
  float qv[HI][8];
#pragma unroll
  for (int h = 0; h < HI; ++h) {
    const uint4 u = __ldg(reinterpret_cast<const uint4*>(iq + (static_cast<int64_t>(b) * HI + h) * DI) + sub);
    const uint32_t uw[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
    for (int k = 0; k < 4; ++k) {
      qv[h][2 * k] = bf16lo(uw[k]);
      qv[h][2 * k + 1] = bf16hi(uw[k]);
    }
  }
  float wh[HI];
#pragma unroll
  for (int h = 0; h < HI; ++h) wh[h] = __ldg(w + b * HI + h);
  const int slot0 = blockIdx.x * kReSlotsPerCta;
  const int slot_end = min(slot0 + kReSlotsPerCta, L);
  constexpr int per_iter = kReThreads / 8;
  // the trip count is the same for every thread of the CTA (shuffles below need whole warps)
  for (int s0 = slot0; s0 < slot_end; s0 += per_iter) {
    const int s = s0 + (threadIdx.x >> 3);
    const bool in_range = s < slot_end;
    const int pos = in_range ? __ldg(pool + static_cast<int64_t>(b) * L + s) : -1;
    const bool valid = pos >= 0 && pos < nb;
    if (!valid && pos != -1 && sub == 0) flag_error(dev_err, CSA2_DEVERR_INDEX_RANGE);
    float d[HI] = {0.0f, 0.0f, 0.0f, 0.0f};
    if (valid) {
      const uint4 u = ldg_nc_v4(reinterpret_cast<const uint4*>(ik_cache + (static_cast<int64_t>(b) * n_cap + pos) * DI) + sub);
      const uint32_t uw[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
      for (int k = 0; k < 4; ++k) {
        const float x0 = bf16lo(uw[k]), x1 = bf16hi(uw[k]);
#pragma unroll
        for (int h = 0; h < HI; ++h) d[h] = fmaf(qv[h][2 * k + 1], x1, fmaf(qv[h][2 * k], x0, d[h]));
      }
    }
#pragma unroll
    for (int h = 0; h < HI; ++h) {
      d[h] += __shfl_xor_sync(0xFFFFFFFFu, d[h], 1);
      d[h] += __shfl_xor_sync(0xFFFFFFFFu, d[h], 2);
      d[h] += __shfl_xor_sync(0xFFFFFFFFu, d[h], 4);
    }
    if (sub == 0 && in_range) {
      float score = 0.0f;
#pragma unroll
      for (int h = 0; h < HI; ++h) score = fmaf(wh[h], fmaxf(d[h], 0.0f), score);
      keys[static_cast<int64_t>(b) * L + s] = valid ? rank_key(score, static_cast<uint32_t>(pos)) : 0ull;
    }
  }
}

struct ReFinalSmem {
  uint64_t keys[kCand];
  int32_t sel[kMaxSel];
  uint32_t hist[256];
  RadixState st;
  int nsel;
  int nvalid;
};

__global__ void __launch_bounds__(kFinalThreads)
    reindex_final_kernel(const uint64_t* __restrict__ keys_g, int L, int K,
                         int32_t* __restrict__ topk) {
  extern __shared__ __align__(1024) unsigned char smem_raw[];
  ReFinalSmem& sm = *reinterpret_cast<ReFinalSmem*>(smem_raw);
  const int b = blockIdx.x, tid = threadIdx.x;
  const uint64_t* src = keys_g + static_cast<int64_t>(b) * L;
  const bool in_smem = L <= kCand;
  if (tid == 0) {
    sm.nsel = 0;
    sm.nvalid = 0;
  }
  __syncthreads();
  int nv = 0;
  for (int i = tid; i < L; i += kFinalThreads) {
    const uint64_t k = src[i];
    if (in_smem) sm.keys[i] = k;
    nv += k != 0ull;
  }
  nv = __reduce_add_sync(0xFFFFFFFFu, nv);
  if ((tid & 31) == 0) atomicAdd(&sm.nvalid, nv);
  __syncthreads();
  const int k_take = min(K, sm.nvalid);
  const uint64_t* c = in_smem ? sm.keys : src;
  auto get = [c](int i) { return c[i]; };
  block_radix_select(get, L, static_cast<uint32_t>(k_take), sm.hist, &sm.st);
  const RadixState st = sm.st;
  if (k_take > 0) {
    for (int i = tid; i < L; i += kFinalThreads) {
      const uint64_t key = c[i];
      if (key != 0ull && radix_selected(key, st)) {
        const int slot = atomicAdd(&sm.nsel, 1);
        if (slot < kMaxSel) sm.sel[slot] = static_cast<int32_t>(rank_key_index(key));
      }
    }
  }
  __syncthreads();
  int n2 = 1;
  while (n2 < k_take) n2 <<= 1;
  for (int i = k_take + tid; i < n2; i += kFinalThreads) sm.sel[i] = 0x7FFFFFFF;
  __syncthreads();
  if (k_take > 1) block_bitonic_sort_i32(sm.sel, n2);
  int32_t* dst = topk + static_cast<int64_t>(b) * K;
  for (int i = tid; i < K; i += kFinalThreads) dst[i] = i < k_take ? sm.sel[i] : -1;
}

// ------------------------------------------------------------------------------------ host

size_t align256(size_t x) { return (x + 255) & ~static_cast<size_t>(255); }

struct FullLayout {
  size_t scores, bmax, hist, cnt, cand, total, zero_begin, zero_bytes;
};

FullLayout full_layout(int B, int n_cap) {
  FullLayout l;
  size_t off = 0;
  l.scores = off;
  off = align256(off + static_cast<size_t>(B) * n_cap * sizeof(float));
  l.bmax = off;
  off = align256(off + static_cast<size_t>(B) * (n_cap / S) * sizeof(float));
  l.hist = off;
  off += static_cast<size_t>(B) * 2 * kHistBins * sizeof(uint32_t);
  l.cnt = off;
  off = align256(off + static_cast<size_t>(B) * 2 * sizeof(uint32_t));
  l.cand = off;
  off = align256(off + static_cast<size_t>(B) * 2 * kCand * sizeof(uint64_t));
  l.total = off;
  l.zero_begin = l.hist;
  l.zero_bytes = l.cand - l.hist;
  return l;
}

typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*,
                                  const cuuint64_t*, const cuuint64_t*, const cuuint32_t*,
                                  const cuuint32_t*, CUtensorMapInterleave, CUtensorMapSwizzle,
                                  CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn encode_fn() {
  static std::once_flag once;
  static EncodeTiledFn fn = nullptr;
  std::call_once(once, [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) ==
            cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<EncodeTiledFn>(p);
  });
  return fn;
}

template <class Kern>
cudaError_t set_smem(Kern k, size_t bytes, std::vector<int>& done) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  if (dev < static_cast<int>(done.size()) && done[dev]) return cudaSuccess;
  e = cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(bytes));
  if (e != cudaSuccess) return e;
  if (dev >= static_cast<int>(done.size())) done.resize(dev + 1, 0);
  done[dev] = 1;
  return cudaSuccess;
}

std::mutex g_attr_mu;

}  // namespace

size_t index_full_workspace_bytes(int B, int n_cap, int K, int P) {
  (void)K;
  (void)P;
  return full_layout(B, n_cap).total;
}

cudaError_t launch_index_full(const void* iq, const float* w, const void* ik_cache,
                              const int32_t* N, int B, int n_cap, int K, int P, int32_t* topk,
                              int32_t* pool, void* ws, int32_t* dev_err, cudaStream_t s) {
  const FullLayout l = full_layout(B, n_cap);
  unsigned char* base = static_cast<unsigned char*>(ws);
  float* scores = reinterpret_cast<float*>(base + l.scores);
  float* bmax = reinterpret_cast<float*>(base + l.bmax);
  uint32_t* hist = reinterpret_cast<uint32_t*>(base + l.hist);
  uint32_t* cnt = reinterpret_cast<uint32_t*>(base + l.cnt);
  uint64_t* cand = reinterpret_cast<uint64_t*>(base + l.cand);

  EncodeTiledFn enc = encode_fn();
  if (enc == nullptr) return cudaErrorNotSupported;
  CUtensorMap map;
  const cuuint64_t dims[3] = {static_cast<cuuint64_t>(DI), static_cast<cuuint64_t>(n_cap),
                              static_cast<cuuint64_t>(B)};
  const cuuint64_t strides[2] = {static_cast<cuuint64_t>(DI) * 2,
                                 static_cast<cuuint64_t>(n_cap) * DI * 2};
  const cuuint32_t box[3] = {static_cast<cuuint32_t>(DI), static_cast<cuuint32_t>(kScanTile), 1};
  const cuuint32_t estr[3] = {1, 1, 1};
  if (enc(&map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(ik_cache), dims, strides,
          box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
          CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
    return cudaErrorInvalidValue;

  {
    static std::vector<int> done_scan, done_final;
    std::lock_guard<std::mutex> lock(g_attr_mu);
    cudaError_t e = set_smem(index_scan_kernel, sizeof(ScanSmem), done_scan);
    if (e != cudaSuccess) return e;
    e = set_smem(topk_final_kernel, sizeof(FinalSmem), done_final);
    if (e != cudaSuccess) return e;
  }

  cudaError_t e = cudaMemsetAsync(base + l.zero_begin, 0, l.zero_bytes, s);
  if (e != cudaSuccess) return e;
  const int64_t tiles = static_cast<int64_t>(B) * ((n_cap + kScanTile - 1) / kScanTile);
  const int grid = static_cast<int>(std::min<int64_t>(device_sm_count(), tiles));
  profile_begin(CSA2_KERNEL_INDEX_SCAN, s);
  index_scan_kernel<<<grid, kScanThreads, sizeof(ScanSmem), s>>>(
      map, static_cast<const uint16_t*>(iq), w, N, B, n_cap, scores, bmax, hist, dev_err);
  profile_end(CSA2_KERNEL_INDEX_SCAN, s);
  count_launches(1);
  if ((e = cudaGetLastError()) != cudaSuccess) return e;
  profile_begin(CSA2_KERNEL_INDEX_SELECT, s);
  const dim3 cgrid((n_cap + kCollectChunk - 1) / kCollectChunk, B, 2);
  topk_collect_kernel<<<cgrid, kCollectThreads, 0, s>>>(scores, bmax, N, n_cap, K, P, hist, cnt,
                                                         cand);
  count_launches(1);
  if ((e = cudaGetLastError()) != cudaSuccess) return e;
  topk_final_kernel<<<dim3(B, 2), kFinalThreads, sizeof(FinalSmem), s>>>(scores, bmax, N, n_cap,
                                                                          K, P, cnt, cand, topk,
                                                                          pool);
  profile_end(CSA2_KERNEL_INDEX_SELECT, s);
  count_launches(1);
  return cudaGetLastError();
}

size_t index_reindex_workspace_bytes(int B, int L, int K) {
  (void)K;
  return align256(static_cast<size_t>(B) * L * sizeof(uint64_t));
}

cudaError_t launch_index_reindex(const void* iq, const float* w, const void* ik_cache,
                                 const int32_t* N, int B, int n_cap, const int32_t* pool, int L,
                                 int K, int32_t* topk, void* ws, int32_t* dev_err,
                                 cudaStream_t s) {
  uint64_t* keys = static_cast<uint64_t*>(ws);
  {
    static std::vector<int> done;
    std::lock_guard<std::mutex> lock(g_attr_mu);
    cudaError_t e = set_smem(reindex_final_kernel, sizeof(ReFinalSmem), done);
    if (e != cudaSuccess) return e;
  }
  const dim3 grid((L + kReSlotsPerCta - 1) / kReSlotsPerCta, B);
  profile_begin(CSA2_KERNEL_REINDEX, s);
  reindex_score_kernel<<<grid, kReThreads, 0, s>>>(static_cast<const uint16_t*>(iq), w,
                                                   static_cast<const uint16_t*>(ik_cache), N,
                                                   n_cap, pool, L, keys, dev_err);
  count_launches(1);
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  reindex_final_kernel<<<B, kFinalThreads, sizeof(ReFinalSmem), s>>>(keys, L, K, topk);
  profile_end(CSA2_KERNEL_REINDEX, s);
  count_launches(1);
  return cudaGetLastError();
}

}  // namespace csa2

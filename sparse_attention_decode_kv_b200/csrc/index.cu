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
//                       6-stage mbarrier ring; two groups of 8 consumer warps take alternate
//                       tiles and run the 4-head q.K contraction on the tensor cores (m16n8k16
//                       bf16, keys on M, heads padded to N = 8), then ReLU, weights, the fp32
//                       score store, the block max over 8 positions and a 4096-bin histogram
//                       (top 12 key bits) of the block maxima.
//   block_collect_kernel  finds the histogram bin holding the max(K, P)-th block and copies the
//                       rank keys of all blocks in or above it, in block order, into one region
//                       per 8192-block chunk.
//   index_final_kernel  two CTAs per sequence, running at once. The first selects the top P
//                       blocks among the candidates (held in registers; the scan's histogram
//                       fixes the top 12 key bits, the radix select refines them), compacts
//                       them in order (ascending block ids, no sort) and writes the pool. The
//                       second selects the top K blocks the same way, then the position Top-K
//                       over their positions, from the gathered scores and a histogram built
//                       while gathering them. Every Top-K position lies in one of the top K
//                       blocks: a block ranked above the block of a selected position holds its
//                       own maximum, which outranks that position, so fewer than K blocks
//                       outrank it.
// Every mbarrier wait is bounded; a timeout flags CSA2_DEVERR_TIMEOUT and the CTA drains its own
// bulk copies before exiting.
#include <mutex>
#include <type_traits>
#include <vector>

#include "common.cuh"
#include "internal.h"
#include "select.cuh"

namespace csa2 {

namespace {

constexpr int kScanTile = 128;                    // entries per TMA tile
constexpr int kScanTileBytes = kScanTile * DI * 2;  // 16 KiB
constexpr int kScanStages = 6;
// The two consumer groups take alternate tiles, so with an even stage count every stage is always
// read by the same group and no consumer can be two phases ahead on a stage. With an odd count the
// groups alternate on a stage, and a parity wait could take a phase two ahead for the one it wants.
static_assert(kScanStages % 2 == 0, "each ring stage must belong to one consumer group");
constexpr int kScanGroupWarps = 8;                // warps sharing one tile, 16 entries each
constexpr int kScanConsumerWarps = 2 * kScanGroupWarps;  // two groups take alternate tiles
constexpr int kScanThreads = (kScanConsumerWarps + 1) * 32;
constexpr int kCollectChunk = 8192;              // blocks per collect CTA (and per region)
constexpr int kCollectThreads = 256;
constexpr int kFinalThreads = 1024;
constexpr int kMaxSel = 4096;                     // >= CSA2_MAX_K, CSA2_MAX_P
constexpr int kSmemKeys = 16384;                  // 8-byte words of the index_final fallback buffer

static_assert(kScanTileBytes == 16384, "tile size");

struct __align__(1024) ScanSmem {  // checked against the 227 KiB limit below
  uint8_t tiles[kScanStages][kScanTileBytes];
  uint64_t full[kScanStages];
  uint64_t empty[kScanStages];
  uint32_t hist[kHistBins];  // block maxima
  int abort;
};

static_assert(sizeof(ScanSmem) <= 227 * 1024, "index_scan_kernel shared memory");

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
  const int n_tiles = static_cast<int>(v_end - v_begin);
  // (sequence, tile) of the first virtual tile; later ones are walked incrementally
  const int b_first = static_cast<int>(v_begin / tiles_per_seq);
  const int t_first = static_cast<int>(v_begin - static_cast<int64_t>(b_first) * tiles_per_seq);

  for (int i = tid; i < kHistBins; i += kScanThreads) sm.hist[i] = 0u;
  if (tid == 0) {
    for (int s = 0; s < kScanStages; ++s) {
      mbar_init(&sm.full[s], 1);
      mbar_init(&sm.empty[s], kScanGroupWarps);
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
      int b = b_first, t = t_first, nb = max(0, min(__ldg(N + b), n_cap));
      int stage = 0, issued = 0;
      uint32_t phase = 0;
      for (int k = 0; k < n_tiles && !*abort; ++k) {
        if (t * kScanTile < nb) {
          if (issued >= kScanStages && !wait_or_abort(&sm.empty[stage], phase ^ 1u, abort)) {
            flag_error(dev_err, CSA2_DEVERR_TIMEOUT);
            *abort = 1;
            break;
          }
          mbar_arrive_expect_tx(&sm.full[stage], kScanTileBytes);
          tma_load_3d(sm.tiles[stage], &keys, &sm.full[stage], 0, t * kScanTile, b, policy);
          ++issued;
          if (++stage == kScanStages) {
            stage = 0;
            phase ^= 1u;
          }
        }
        if (++t == tiles_per_seq && k + 1 < n_tiles) {
          t = 0;
          ++b;
          nb = max(0, min(__ldg(N + b), n_cap));
        }
      }
      // drain: every issued copy must land before the CTA may exit
      for (int j = max(0, issued - kScanStages); j < issued; ++j) {
        const int st = j % kScanStages;
        if (!mbar_wait(&sm.full[st], static_cast<uint32_t>((j / kScanStages) & 1)))
          flag_error(dev_err, CSA2_DEVERR_TIMEOUT);
      }
    }
    pdl_launch_dependents();
    return;
  }

  // ---------------------------------------------------------- consumers (2 groups of 8 warps)
  // Group gi takes the tiles whose issue index has parity gi; within a tile, warp wg of the
  // group takes rows 16 wg .. 16 wg + 15.
  const int gi = warp / kScanGroupWarps, wg = warp % kScanGroupWarps;
  const int g = lane >> 2, c = lane & 3;
  const int mi = lane >> 3;
  const int a_row = 16 * wg + (lane & 7) + ((mi & 1) << 3);
  int cur_b = -1, nb = 0;
  uint32_t bq0[4], bq1[4];
  float wa = 0.0f, wb = 0.0f;
  int stage = 0, issued = 0;
  uint32_t phase = 0;

  auto flush = [&](int bseq) {
    consumer_bar();
    for (int i = tid; i < kHistBins; i += kScanConsumerWarps * 32) {
      const uint32_t v = sm.hist[i];
      if (v) {
        atomicAdd(hist_g + static_cast<int64_t>(bseq) * kHistBins + i, v);
        sm.hist[i] = 0u;
      }
    }
    consumer_bar();
  };

  int b = b_first, t = t_first;
  for (int k = 0; k < n_tiles; ++k) {
    if (b != cur_b) {
      if (cur_b >= 0) flush(cur_b);
      cur_b = b;
      nb = clamp_len(N, b, n_cap, lane == 0 && warp == 0 ? dev_err : nullptr);
      // B fragments: head g (< 4) of iq[b]; heads 4..7 are zero padding
#pragma unroll
      for (int s = 0; s < 4; ++s) {
        bq0[s] = bq1[s] = 0u;
        if (g < HI) {
          const uint32_t* qrow =
              reinterpret_cast<const uint32_t*>(iq + (static_cast<int64_t>(b) * HI + g) * DI);
          bq0[s] = __ldg(qrow + 8 * s + c);
          bq1[s] = __ldg(qrow + 8 * s + 4 + c);
        }
      }
      wa = c < 2 ? __ldg(w + b * HI + 2 * c) : 0.0f;
      wb = c < 2 ? __ldg(w + b * HI + 2 * c + 1) : 0.0f;
    }
    const int tt = t;
    if (++t == tiles_per_seq) {
      t = 0;
      ++b;
    }
    if (tt * kScanTile >= nb) continue;
    const int my_stage = stage;
    const uint32_t my_phase = phase;
    const bool mine = (issued & 1) == gi;
    ++issued;
    if (++stage == kScanStages) {
      stage = 0;
      phase ^= 1u;
    }
    if (!mine) continue;
    // every lane waits (acquiring the tile), the warp then takes one decision
    const bool ok =
        __all_sync(0xFFFFFFFFu, !*abort && wait_or_abort(&sm.full[my_stage], my_phase, abort));
    if (!ok) {
      if (lane == 0 && !*abort) flag_error(dev_err, CSA2_DEVERR_TIMEOUT);
      *abort = 1;
      continue;
    }

    float acc[4] = {0.0f, 0.0f, 0.0f, 0.0f};
    const uint32_t tile = smem_u32(sm.tiles[my_stage]);
#pragma unroll
    for (int s = 0; s < 4; ++s) {
      const int chunk = 2 * s + (mi >> 1);
      uint32_t a0, a1, a2, a3;
      ldsm_x4(tile + a_row * 128 + ((chunk ^ (a_row & 7)) << 4), a0, a1, a2, a3);
      mma_bf16_16816(acc, a0, a1, a2, a3, bq0[s], bq1[s]);
    }
    __syncwarp();
    if (lane == 0) mbar_arrive(&sm.empty[my_stage]);

    // scores of rows g and g+8 (lanes c = 0 and 1 hold heads 0,1 and 2,3)
    float s0 = wa * fmaxf(acc[0], 0.0f) + wb * fmaxf(acc[1], 0.0f);
    float s1 = wa * fmaxf(acc[2], 0.0f) + wb * fmaxf(acc[3], 0.0f);
    s0 += __shfl_xor_sync(0xFFFFFFFFu, s0, 1);
    s1 += __shfl_xor_sync(0xFFFFFFFFu, s1, 1);
    s0 += 0.0f;  // fold -0 onto +0
    s1 += 0.0f;
    const int t0 = tt * kScanTile + 16 * wg + g, t1 = t0 + 8;
    const bool v0 = t0 < nb, v1 = t1 < nb;
    if (c == 0) {
      float* srow = scores + static_cast<int64_t>(cur_b) * n_cap;
      if (v0) srow[t0] = s0;
      if (v1) srow[t1] = s1;
    }
    float m0 = v0 ? s0 : -INFINITY, m1 = v1 ? s1 : -INFINITY;
#pragma unroll
    for (int off = 4; off < 32; off <<= 1) {
      m0 = fmaxf(m0, __shfl_xor_sync(0xFFFFFFFFu, m0, off));
      m1 = fmaxf(m1, __shfl_xor_sync(0xFFFFFFFFu, m1, off));
    }
    if (lane == 0) {
      const int j0 = (tt * kScanTile + 16 * wg) / S;
      float* brow = bmax + static_cast<int64_t>(cur_b) * (n_cap / S);
      if (j0 * S < nb) {
        brow[j0] = m0;
        atomicAdd(&sm.hist[float_key(m0) >> kHistShift], 1u);
      }
      if ((j0 + 1) * S < nb) {
        brow[j0 + 1] = m1;
        atomicAdd(&sm.hist[float_key(m1) >> kHistShift], 1u);
      }
    }
  }
  pdl_launch_dependents();
  if (cur_b >= 0) flush(cur_b);
}

// Block candidates: CTA (chunk, b) handles blocks [8192 chunk, 8192 chunk + 8192) of sequence
// b. Thread t loads its 32 consecutive block maxima at once, keeps those whose key bin is at or
// above the threshold bin of the max(K, P)-th block, and writes their rank keys in block order
// into the chunk's region (an exclusive scan over the threads orders them).
__global__ void __launch_bounds__(kCollectThreads)
    block_collect_kernel(const float* __restrict__ bmax, const int32_t* __restrict__ N, int n_cap,
                         int K, int P, const uint32_t* __restrict__ hist_g,
                         uint32_t* __restrict__ ccnt, uint64_t* __restrict__ cand) {
  constexpr int kPer = kCollectChunk / kCollectThreads;  // 32 blocks per thread
  __shared__ uint32_t part[kCollectThreads];
  __shared__ uint32_t scan[33];
  __shared__ int sh[6];
  pdl_wait();
  pdl_launch_dependents();
  const int b = blockIdx.y, chunk = blockIdx.x;
  const int nb = max(0, min(__ldg(N + b), n_cap));
  const int nbl = (nb + S - 1) / S;
  const int kw = min(max(K, P), nbl);
  const int start = chunk * kCollectChunk;
  if (kw == 0 || start >= nbl) return;
  const int nchunks = (n_cap / S + kCollectChunk - 1) / kCollectChunk;
  const float* src = bmax + static_cast<int64_t>(b) * (n_cap / S);
  const int i0 = start + kPer * threadIdx.x;
  float v[kPer];
  if (((reinterpret_cast<uintptr_t>(src + i0) & 15u) == 0) && i0 + kPer <= nbl) {
#pragma unroll
    for (int m = 0; m < kPer / 4; ++m) {
      const float4 f = __ldg(reinterpret_cast<const float4*>(src + i0) + m);
      v[4 * m] = f.x;
      v[4 * m + 1] = f.y;
      v[4 * m + 2] = f.z;
      v[4 * m + 3] = f.w;
    }
  } else {
#pragma unroll
    for (int j = 0; j < kPer; ++j) v[j] = i0 + j < nbl ? __ldg(src + i0 + j) : 0.0f;
  }
  const int T0 = block_find_bin4096(hist_g + static_cast<int64_t>(b) * kHistBins,
                                    static_cast<uint32_t>(kw), part, sh);
  uint32_t mask = 0, c = 0;
#pragma unroll
  for (int j = 0; j < kPer; ++j) {
    if (i0 + j < nbl && static_cast<int>(float_key(v[j]) >> kHistShift) >= T0) {
      mask |= 1u << j;
      ++c;
    }
  }
  uint32_t total;
  uint32_t slot = block_exclusive_scan(c, scan, &total);
  uint64_t* out = cand + (static_cast<int64_t>(b) * nchunks + chunk) * kCollectChunk;
#pragma unroll
  for (int j = 0; j < kPer; ++j)
    if ((mask >> j) & 1u) out[slot++] = rank_key(v[j], static_cast<uint32_t>(i0 + j));
  if (threadIdx.x == 0) ccnt[static_cast<int64_t>(b) * nchunks + chunk] = total;
}

constexpr int kRegKeys = 16;  // keys per thread of the register selections (16,384 per CTA)

struct FinalSmem {
  union {
    uint32_t skey[2 * kSmemKeys];    // position fallback: score keys of the wide blocks' positions
    struct {
      uint32_t fresh[kDigitBins];    // cleared histogram for the first refining pass
      uint32_t wc[544];              // per (register slot, warp) counts of the compaction
    } r;                             // the register selections (which use neither array above)
  } u;
  int32_t wide[kMaxSel];             // top max(K, P) blocks, ascending
  uint64_t wide_key[kMaxSel];        // their rank keys; later the position candidates
  union {
    int32_t chunk_pre[kMaxSel + 1];  // candidate prefix over chunks (while loading candidates)
  } v;
  SelectScratch sc;
};

static_assert(sizeof(FinalSmem) <= 227 * 1024, "index_final_kernel shared memory");

__global__ void __launch_bounds__(kFinalThreads)
    index_final_kernel(const float* __restrict__ scores, const int32_t* __restrict__ N, int n_cap,
                       int K, int P, const uint32_t* __restrict__ hist_g,
                       const uint32_t* __restrict__ ccnt,
                       const uint64_t* __restrict__ cand, int32_t* __restrict__ topk,
                       int32_t* __restrict__ pool) {
  extern __shared__ __align__(1024) unsigned char smem_raw[];
  FinalSmem& sm = *reinterpret_cast<FinalSmem*>(smem_raw);
  pdl_wait();
  pdl_launch_dependents();
  // role 0: the pool (top P blocks); role 1: the position Top-K, which needs nothing from role 0
  // (both take their blocks from the candidates, which hold the top max(K, P) blocks)
  const int b = blockIdx.x, role = blockIdx.y, tid = threadIdx.x;
  const int nb = max(0, min(__ldg(N + b), n_cap));
  const int nbl = (nb + S - 1) / S;
  const int kw = min(max(K, P), nbl);  // blocks that hold every Top-K position and the pool
  const int kp = min(P, nbl);
  const int kk = min(K, nb);
  const int nchunks = (n_cap / S + kCollectChunk - 1) / kCollectChunk;
  const int nch = (nbl + kCollectChunk - 1) / kCollectChunk;
  int32_t* pool_out = pool + static_cast<int64_t>(b) * P * S;
  int32_t* topk_out = topk + static_cast<int64_t>(b) * K;
  if (kw == 0) {
    if (role == 0)
      for (int i = tid; i < P * S; i += kFinalThreads) pool_out[i] = -1;
    else
      for (int i = tid; i < K; i += kFinalThreads) topk_out[i] = -1;
    return;
  }

  // ---- block candidates (every block whose maximum is in or above the bin of the kw-th one), in
  // block order
  const uint32_t* cnts = ccnt + static_cast<int64_t>(b) * nchunks;
  const uint64_t* cbase = cand + static_cast<int64_t>(b) * nchunks * kCollectChunk;
  // prefix over chunk counts (thread c owns chunks 4c..4c+3)
  {
    uint32_t cv[4];
    uint32_t sum = 0;
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      const int c = 4 * tid + j;
      cv[j] = c < nch ? __ldg(cnts + c) : 0u;
      sum += cv[j];
    }
    uint32_t total;
    uint32_t run = block_exclusive_scan(sum, sm.sc.scan, &total);
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      const int c = 4 * tid + j;
      if (c < nch) sm.v.chunk_pre[c] = static_cast<int32_t>(run);
      run += cv[j];
    }
    if (tid == 0) sm.v.chunk_pre[nch] = static_cast<int32_t>(total);
  }
  __syncthreads();
  const int C = sm.v.chunk_pre[nch];
  auto cand_at = [&](int i) -> uint64_t {  // candidate i in block order (chunk by binary search)
    int lo = 0, hi = nch - 1;
    while (lo < hi) {
      const int mid = (lo + hi + 1) >> 1;
      if (sm.v.chunk_pre[mid] <= i) lo = mid;
      else hi = mid - 1;
    }
    return __ldg(cbase + static_cast<int64_t>(lo) * kCollectChunk + (i - sm.v.chunk_pre[lo]));
  };

  // ---- the top kx blocks among the candidates, ascending, into sm.wide / sm.wide_key.
  // Candidate 1024 j + t in thread t's key j (NK keys per thread: 4 when they fit, else 16). The
  // scan's histogram of every block maximum fixes the top 12 bits of the kx-th key (the
  // candidates are all blocks at or above the bin of the kw-th one, kx <= kw); the radix select
  // goes on over the candidates in that bin.
  auto select_blocks_regs = [&](auto nk, int kx) {
    constexpr int NK = decltype(nk)::value;
    for (int i = tid; i < kDigitBins; i += kFinalThreads) sm.u.r.fresh[i] = 0u;
    uint64_t key[NK];
#pragma unroll
    for (int j = 0; j < NK; ++j) {
      const int i = j * kFinalThreads + tid;
      key[j] = i < C ? cand_at(i) : 0ull;
    }
    radix_state_from_top12(hist_g + static_cast<int64_t>(b) * kHistBins, static_cast<uint32_t>(kx),
                           sm.sc);
    block_radix_refine_visit(
        [&](auto f) {
#pragma unroll
          for (int j = 0; j < NK; ++j) f(key[j]);
        },
        sm.u.r.fresh, sm.sc);
    const RadixState st = sm.sc.st;
    block_ordered_compact_regs<NK, false>(
        [&](int j) { return key[j] != 0ull && radix_selected(key[j], st); },
        [&](int j, uint32_t slot) {
          if (slot < kMaxSel) {
            sm.wide[slot] = static_cast<int32_t>(rank_key_index(key[j]));
            sm.wide_key[slot] = key[j];
          }
        },
        sm.u.r.wc);
    __syncthreads();
  };
  auto select_blocks = [&](int kx) {
    if (C <= 4 * kFinalThreads) {
      select_blocks_regs(std::integral_constant<int, 4>{}, kx);
    } else if (C <= kRegKeys * kFinalThreads) {
      select_blocks_regs(std::integral_constant<int, kRegKeys>{}, kx);
    } else {
      block_radix_select(cand_at, C, static_cast<uint32_t>(kx), sm.sc);
      const RadixState st = sm.sc.st;
      block_ordered_compact(
          C, [&](int i) { return radix_selected(cand_at(i), st); },
          [&](int i, uint32_t slot) {
            if (slot < kMaxSel) {
              const uint64_t key = cand_at(i);
              sm.wide[slot] = static_cast<int32_t>(rank_key_index(key));
              sm.wide_key[slot] = key;
            }
          },
          sm.sc.scan);
    }
  };

  if (role == 0) {
    // ---- the pool: the top kp blocks, ascending, expanded to their positions
    select_blocks(kp);
    for (int i = tid; i < P * S; i += kFinalThreads) {
      const int j = i / S;
      const int p = j < kp ? sm.wide[j] * S + (i % S) : nb;
      pool_out[i] = p < nb ? p : -1;
    }
    return;
  }

  const float* srow = scores + static_cast<int64_t>(b) * n_cap;
  uint32_t n_sel = 0;
  {
    // ---- the position Top-K: the top kq blocks, then the Top-K over their positions. A block
    // ranked above the block of a Top-K position holds its own maximum, which outranks that
    // position, so fewer than K blocks outrank it: every Top-K position lies in the top K blocks.
    const int kq = min(K, nbl);
    select_blocks(kq);
    // position Top-K over every position of those blocks (item i = position i % 8 of block
    // wide[i / 8]: ascending positions). The score gather also histograms the top 12 bits of each
    // rank key, which fixes those bits of the K-th key; the radix select continues from there.
    const int L = kq * S;  // <= 32768
    // position item 1024 j + t in thread t's key j (NK keys per thread: 4 when they fit, else
    // 16; key 0: past N or past the blocks)
    auto positions_regs = [&](auto nk) -> uint32_t {
      constexpr int NK = decltype(nk)::value;
      for (int i = tid; i < kDigitBins; i += kFinalThreads) {
        sm.sc.hist[i] = 0u;
        sm.u.r.fresh[i] = 0u;
      }
      __syncthreads();
      // all score loads first: the high word holds the raw score bits until they land, the low
      // word the inverted position (never 0 for a real position)
      uint32_t hi[NK], lo[NK];
#pragma unroll
      for (int j = 0; j < NK; ++j) {
        const int i = j * kFinalThreads + tid;
        const int p = i < L ? sm.wide[i / S] * S + (i % S) : nb;
        lo[j] = p < nb ? ~static_cast<uint32_t>(p) : 0u;
        hi[j] = p < nb ? __float_as_uint(__ldg(srow + p)) : 0u;
      }
      uint64_t key[NK];
#pragma unroll
      for (int j = 0; j < NK; ++j) {
        key[j] = lo[j] != 0u ? rank_key(__uint_as_float(hi[j]), ~lo[j]) : 0ull;
        if (key[j] != 0ull) atomicAdd(&sm.sc.hist[static_cast<uint32_t>(key[j] >> 52)], 1u);
      }
      __syncthreads();
      radix_state_from_top12(sm.sc.hist, static_cast<uint32_t>(kk), sm.sc);
      block_radix_refine_visit(
          [&](auto f) {
#pragma unroll
            for (int j = 0; j < NK; ++j) f(key[j]);
          },
          sm.u.r.fresh, sm.sc);
      const RadixState st = sm.sc.st;
      return block_ordered_compact_regs<NK, false>(
          [&](int j) { return key[j] != 0ull && radix_selected(key[j], st); },
          [&](int j, uint32_t slot) {
            if (slot < static_cast<uint32_t>(K)) topk_out[slot] = static_cast<int32_t>(rank_key_index(key[j]));
          },
          sm.u.r.wc);
    };
    if (L <= 4 * kFinalThreads) {
      n_sel = positions_regs(std::integral_constant<int, 4>{});
    } else if (L <= kRegKeys * kFinalThreads) {
      n_sel = positions_regs(std::integral_constant<int, kRegKeys>{});
    } else {
      for (int i = tid; i < kDigitBins; i += kFinalThreads) sm.sc.hist[i] = 0u;
      __syncthreads();
      for (int base = 0; base < L; base += 8 * kFinalThreads) {
        float vals[8];
#pragma unroll
        for (int j = 0; j < 8; ++j) {
          const int i = base + j * kFinalThreads + tid;
          const int p = i < L ? sm.wide[i / S] * S + (i % S) : nb;
          vals[j] = p < nb ? __ldg(srow + p) : 0.0f;
        }
#pragma unroll
        for (int j = 0; j < 8; ++j) {
          const int i = base + j * kFinalThreads + tid;
          if (i < L) {
            const int p = sm.wide[i / S] * S + (i % S);
            const uint32_t key = p < nb ? float_key(vals[j]) : 0u;  // 0: below every real key
            sm.u.skey[i] = key;
            if (p < nb) atomicAdd(&sm.sc.hist[key >> kHistShift], 1u);
          }
        }
      }
      __syncthreads();
      auto pos_of = [&](int i) { return static_cast<uint32_t>(sm.wide[i / S] * S + (i % S)); };
      auto pos_key = [&](int i) -> uint64_t {
        const uint32_t hk = sm.u.skey[i];
        return hk == 0u ? 0ull : (static_cast<uint64_t>(hk) << 32) | static_cast<uint64_t>(~pos_of(i));
      };
      const int T0 = block_find_bin4096(sm.sc.hist, static_cast<uint32_t>(kk), sm.sc.part, sm.sc.ints);
      // candidates in slot order into the (now free) wide_key array
      uint64_t* cbuf = sm.wide_key;
      const uint32_t n_cand = block_ordered_compact(
          L, [&](int i) { const uint32_t k = sm.u.skey[i]; return k != 0u && static_cast<int>(k >> kHistShift) >= T0; },
          [&](int i, uint32_t slot) { if (slot < kMaxSel) cbuf[slot] = pos_key(i); }, sm.sc.scan);
      __syncthreads();
      if (n_cand <= static_cast<uint32_t>(kMaxSel)) {
        auto get = [cbuf](int i) { return cbuf[i]; };
        block_radix_select(get, static_cast<int>(n_cand), static_cast<uint32_t>(kk), sm.sc);
        const RadixState st = sm.sc.st;
        n_sel = block_ordered_compact(
            static_cast<int>(n_cand), [&](int i) { return radix_selected(cbuf[i], st); },
            [&](int i, uint32_t slot) {
              if (slot < static_cast<uint32_t>(K)) topk_out[slot] = static_cast<int32_t>(rank_key_index(cbuf[i]));
            },
            sm.sc.scan);
      } else {
        block_radix_select(pos_key, L, static_cast<uint32_t>(kk), sm.sc);
        const RadixState st = sm.sc.st;
        n_sel = block_ordered_compact(
            L, [&](int i) { const uint64_t k = pos_key(i); return k != 0ull && radix_selected(k, st); },
            [&](int i, uint32_t slot) {
              if (slot < static_cast<uint32_t>(K)) topk_out[slot] = static_cast<int32_t>(pos_of(i));
            },
            sm.sc.scan);
      }
    }
  }
  for (int i = static_cast<int>(n_sel) + tid; i < K; i += kFinalThreads) topk_out[i] = -1;
}

// ------------------------------------------------------------------------------------ Reindex

// Reindex scoring on the tensor cores. A warp takes tiles of 16 pool slots: lane (g, c) loads 32
// contiguous bytes (dims 16c .. 16c+15) of the keys of slots g and g+8 straight into registers,
// which is the m16n8k16 A fragment under a permutation of the 64 dims (k-step s, pair 2c ->
// dims 16c+4s, +1; pair 2c+8 -> dims 16c+4s+2, +3); the query fragments use the same permutation.
// All pool entries, then all key rows of a warp's tiles are loaded before any arithmetic.
constexpr int kReWarps = 8;
constexpr int kReThreads = kReWarps * 32;
constexpr int kReTilesPerWarp = 4;
constexpr int kReSlotsPerCta = kReWarps * kReTilesPerWarp * 16;  // 512

__global__ void __launch_bounds__(kReThreads)
    reindex_score_kernel(const uint16_t* __restrict__ iq, const float* __restrict__ w,
                         const uint16_t* __restrict__ ik_cache, const int32_t* __restrict__ N,
                         int n_cap, const int32_t* __restrict__ pool, int L,
                         uint64_t* __restrict__ keys, int32_t* dev_err) {
  pdl_wait();
  pdl_launch_dependents();
  const int b = blockIdx.y;
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int g = lane >> 2, c = lane & 3;
  const int nb = clamp_len(N, b, n_cap, threadIdx.x == 0 && blockIdx.x == 0 ? dev_err : nullptr);
  // query fragments: head g (< 4) of iq[b] under the dim permutation; heads 4..7 are zero
  uint32_t bq0[4], bq1[4];
  {
    const uint32_t* qrow = reinterpret_cast<const uint32_t*>(iq + (static_cast<int64_t>(b) * HI + min(g, HI - 1)) * DI);
#pragma unroll
    for (int s = 0; s < 4; ++s) {
      bq0[s] = g < HI ? __ldg(qrow + 8 * c + 2 * s) : 0u;
      bq1[s] = g < HI ? __ldg(qrow + 8 * c + 2 * s + 1) : 0u;
    }
  }
  const float wa = c < 2 ? __ldg(w + b * HI + 2 * c) : 0.0f;
  const float wb = c < 2 ? __ldg(w + b * HI + 2 * c + 1) : 0.0f;
  const int slot0 = blockIdx.x * kReSlotsPerCta + warp * kReTilesPerWarp * 16;
  const int32_t* prow = pool + static_cast<int64_t>(b) * L;
  int pos[kReTilesPerWarp][2];
#pragma unroll
  for (int t = 0; t < kReTilesPerWarp; ++t)
#pragma unroll
    for (int h = 0; h < 2; ++h) {
      const int s = slot0 + 16 * t + g + 8 * h;
      pos[t][h] = s < L ? __ldg(prow + s) : -1;
    }
  uint4 u[kReTilesPerWarp][2][2];
#pragma unroll
  for (int t = 0; t < kReTilesPerWarp; ++t)
#pragma unroll
    for (int h = 0; h < 2; ++h) {
      const int p = pos[t][h];
      const bool valid = p >= 0 && p < nb;
      if (!valid && p != -1 && c == 0) flag_error(dev_err, CSA2_DEVERR_INDEX_RANGE);
      const uint4* src = reinterpret_cast<const uint4*>(
                             ik_cache + (static_cast<int64_t>(b) * n_cap + (valid ? p : 0)) * DI) + 2 * c;
      u[t][h][0] = valid ? ldg_nc_v4(src) : make_uint4(0u, 0u, 0u, 0u);
      u[t][h][1] = valid ? ldg_nc_v4(src + 1) : make_uint4(0u, 0u, 0u, 0u);
    }
#pragma unroll
  for (int t = 0; t < kReTilesPerWarp; ++t) {
    const uint32_t r0[8] = {u[t][0][0].x, u[t][0][0].y, u[t][0][0].z, u[t][0][0].w,
                            u[t][0][1].x, u[t][0][1].y, u[t][0][1].z, u[t][0][1].w};
    const uint32_t r1[8] = {u[t][1][0].x, u[t][1][0].y, u[t][1][0].z, u[t][1][0].w,
                            u[t][1][1].x, u[t][1][1].y, u[t][1][1].z, u[t][1][1].w};
    float acc[4] = {0.0f, 0.0f, 0.0f, 0.0f};
#pragma unroll
    for (int s = 0; s < 4; ++s)
      mma_bf16_16816(acc, r0[2 * s], r1[2 * s], r0[2 * s + 1], r1[2 * s + 1], bq0[s], bq1[s]);
    float s0 = wa * fmaxf(acc[0], 0.0f) + wb * fmaxf(acc[1], 0.0f);
    float s1 = wa * fmaxf(acc[2], 0.0f) + wb * fmaxf(acc[3], 0.0f);
    s0 += __shfl_xor_sync(0xFFFFFFFFu, s0, 1);
    s1 += __shfl_xor_sync(0xFFFFFFFFu, s1, 1);
    if (c == 0) {
#pragma unroll
      for (int h = 0; h < 2; ++h) {
        const int s = slot0 + 16 * t + g + 8 * h;
        const int p = pos[t][h];
        if (s < L)
          keys[static_cast<int64_t>(b) * L + s] =
              (p >= 0 && p < nb) ? rank_key(h ? s1 : s0, static_cast<uint32_t>(p)) : 0ull;
      }
    }
  }
}

struct ReFinalSmem {
  int32_t sel[kMaxSel];
  uint32_t fresh[kDigitBins];  // cleared histogram for the first refining pass
  uint32_t wc[544];            // per (register slot, warp) counts of the compaction
  SelectScratch sc;
  int nvalid;
  int unsorted;
};

static_assert(sizeof(ReFinalSmem) <= 227 * 1024, "reindex_final_kernel shared memory");
static_assert(kFinalThreads == 1024, "the register compaction assumes 1,024 threads");

// One CTA per sequence: the Top-K of the pool's rank keys (0 = empty slot). Pools of up to
// 16,384 slots are held in registers, 16 keys per thread (slot 1024 j + t in thread t's key j);
// larger pools are read from global memory on every pass. The key load also histograms the top 12
// bits of every real key, which fixes those bits of the K-th key; the radix select continues from
// there over the keys that share them. Winners come out in pool order, which is ascending position
// for a pool built by the Full-mode indexer; any other pool order is sorted afterwards.
__global__ void __launch_bounds__(kFinalThreads)
    reindex_final_kernel(const uint64_t* __restrict__ keys_g, int L, int K,
                         int32_t* __restrict__ topk) {
  extern __shared__ __align__(1024) unsigned char smem_raw[];
  ReFinalSmem& sm = *reinterpret_cast<ReFinalSmem*>(smem_raw);
  pdl_wait();
  pdl_launch_dependents();
  const int b = blockIdx.x, tid = threadIdx.x;
  const uint64_t* src = keys_g + static_cast<int64_t>(b) * L;
  const bool in_regs = L <= kRegKeys * kFinalThreads;
  for (int i = tid; i < kDigitBins; i += kFinalThreads) {
    sm.sc.hist[i] = 0u;
    sm.fresh[i] = 0u;
  }
  if (tid == 0) {
    sm.nvalid = 0;
    sm.unsorted = 0;
  }
  __syncthreads();
  int nv = 0;
  uint64_t key[kRegKeys];
  if (in_regs) {
#pragma unroll
    for (int j = 0; j < kRegKeys; ++j) {
      const int i = j * kFinalThreads + tid;
      key[j] = i < L ? __ldg(src + i) : 0ull;
    }
#pragma unroll
    for (int j = 0; j < kRegKeys; ++j)
      if (key[j] != 0ull) {
        ++nv;
        atomicAdd(&sm.sc.hist[static_cast<uint32_t>(key[j] >> 52)], 1u);
      }
  } else {
#pragma unroll
    for (int j = 0; j < kRegKeys; ++j) key[j] = 0ull;
    for (int base = 0; base < L; base += 8 * kFinalThreads) {
      uint64_t v[8];
#pragma unroll
      for (int j = 0; j < 8; ++j) {
        const int i = base + j * kFinalThreads + tid;
        v[j] = i < L ? __ldg(src + i) : 0ull;
      }
#pragma unroll
      for (int j = 0; j < 8; ++j)
        if (v[j] != 0ull) {
          ++nv;
          atomicAdd(&sm.sc.hist[static_cast<uint32_t>(v[j] >> 52)], 1u);
        }
    }
  }
  nv = __reduce_add_sync(0xFFFFFFFFu, nv);
  if ((tid & 31) == 0) atomicAdd(&sm.nvalid, nv);
  __syncthreads();
  const int k_take = min(K, sm.nvalid);
  if (k_take > 0) {
    radix_state_from_top12(sm.sc.hist, static_cast<uint32_t>(k_take), sm.sc);
    if (in_regs) {
      block_radix_refine_visit(
          [&](auto f) {
#pragma unroll
            for (int j = 0; j < kRegKeys; ++j) f(key[j]);
          },
          sm.fresh, sm.sc);
      const RadixState st = sm.sc.st;
      block_ordered_compact_regs16<true>(
          [&](int j) { return key[j] != 0ull && radix_selected(key[j], st); },
          [&](int j, uint32_t slot) {
            if (slot < kMaxSel) sm.sel[slot] = static_cast<int32_t>(rank_key_index(key[j]));
          },
          sm.wc);
    } else {
      auto get = [src](int i) { return __ldg(src + i); };
      block_radix_refine(get, L, sm.fresh, sm.sc);
      const RadixState st = sm.sc.st;
      block_ordered_compact(
          L, [&](int i) { const uint64_t k = get(i); return k != 0ull && radix_selected(k, st); },
          [&](int i, uint32_t slot) {
            if (slot < kMaxSel) sm.sel[slot] = static_cast<int32_t>(rank_key_index(get(i)));
          },
          sm.sc.scan);
    }
    __syncthreads();
    for (int i = tid; i + 1 < k_take; i += kFinalThreads)
      if (sm.sel[i] >= sm.sel[i + 1]) sm.unsorted = 1;
    __syncthreads();
    if (sm.unsorted) {
      int n2 = 1;
      while (n2 < k_take) n2 <<= 1;
      for (int i = k_take + tid; i < n2; i += kFinalThreads) sm.sel[i] = 0x7FFFFFFF;
      __syncthreads();
      block_bitonic_sort_i32(sm.sel, n2);
    }
  }
  __syncthreads();
  int32_t* dst = topk + static_cast<int64_t>(b) * K;
  for (int i = tid; i < K; i += kFinalThreads) dst[i] = i < k_take ? sm.sel[i] : -1;
}

// ------------------------------------------------------------------------------------ host

size_t align256(size_t x) { return (x + 255) & ~static_cast<size_t>(255); }

struct FullLayout {
  size_t scores, bmax, hist, ccnt, cand, total;
  int nchunks;
};

FullLayout full_layout(int B, int n_cap) {
  FullLayout l;
  l.nchunks = (n_cap / S + kCollectChunk - 1) / kCollectChunk;
  size_t off = 0;
  l.scores = off;
  off = align256(off + static_cast<size_t>(B) * n_cap * sizeof(float));
  l.bmax = off;
  off = align256(off + static_cast<size_t>(B) * (n_cap / S) * sizeof(float));
  l.hist = off;
  off = align256(off + static_cast<size_t>(B) * kHistBins * sizeof(uint32_t));
  l.ccnt = off;
  off = align256(off + static_cast<size_t>(B) * l.nchunks * sizeof(uint32_t));
  l.cand = off;
  off = align256(off + static_cast<size_t>(B) * l.nchunks * kCollectChunk * sizeof(uint64_t));
  l.total = off;
  return l;
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
  uint32_t* ccnt = reinterpret_cast<uint32_t*>(base + l.ccnt);
  uint64_t* cand = reinterpret_cast<uint64_t*>(base + l.cand);

  const TensorMapEncodeFn enc = tensor_map_encoder();
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
    e = set_smem(index_final_kernel, sizeof(FinalSmem), done_final);
    if (e != cudaSuccess) return e;
  }

  // the block histogram accumulates across the scan's CTAs: zero it first
  cudaError_t e = cudaMemsetAsync(hist, 0, static_cast<size_t>(B) * kHistBins * sizeof(uint32_t), s);
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
  e = launch_pdl(block_collect_kernel, dim3(l.nchunks, B), dim3(kCollectThreads), 0, s,
                 static_cast<const float*>(bmax), N, n_cap, K, P,
                 static_cast<const uint32_t*>(hist), ccnt, cand);
  count_launches(1);
  if (e != cudaSuccess || (e = cudaGetLastError()) != cudaSuccess) return e;
  e = launch_pdl(index_final_kernel, dim3(B, 2), dim3(kFinalThreads), sizeof(FinalSmem), s,
                 static_cast<const float*>(scores), N, n_cap, K, P,
                 static_cast<const uint32_t*>(hist), static_cast<const uint32_t*>(ccnt),
                 static_cast<const uint64_t*>(cand), topk, pool);
  profile_end(CSA2_KERNEL_INDEX_SELECT, s);
  count_launches(1);
  return e != cudaSuccess ? e : cudaGetLastError();
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
  const dim3 grid((L + kReSlotsPerCta - 1) / kReSlotsPerCta, B);  // 32 CTAs per 16,384 slots
  profile_begin(CSA2_KERNEL_REINDEX, s);
  cudaError_t e = launch_pdl(reindex_score_kernel, grid, dim3(kReThreads), 0, s,
                             static_cast<const uint16_t*>(iq), w,
                             static_cast<const uint16_t*>(ik_cache), N, n_cap, pool, L, keys,
                             dev_err);
  count_launches(1);
  if (e != cudaSuccess || (e = cudaGetLastError()) != cudaSuccess) return e;
  e = launch_pdl(reindex_final_kernel, dim3(B), dim3(kFinalThreads), sizeof(ReFinalSmem), s,
                 static_cast<const uint64_t*>(keys), L, K, topk);
  profile_end(CSA2_KERNEL_REINDEX, s);
  count_launches(1);
  return e != cudaSuccess ? e : cudaGetLastError();
}

}  // namespace csa2

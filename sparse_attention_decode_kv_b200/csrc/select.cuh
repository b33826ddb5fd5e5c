// select.cuh -- exact Top-K selection helpers used by the indexer kernels.
//
// Ranking: "DeepSeek V4.1 Flash 拆解" (austincafe.tech), section 一, selects a Top-K of indexer
// scores (and a Top-2048 of blocks); ties go to the lower index. Every candidate carries a 64-bit
// rank key (monotone score key in the high word, inverted index in the low word), so the Top-K is
// the set of the k largest keys, which are all distinct. The selection is an MSB-first radix
// select over 8-bit digits of that key: each pass histograms the next digit of the keys that
// still match the known prefix, and stops as soon as the bin holding the k-th key is taken whole.
#pragma once

#include "common.cuh"

namespace csa2 {

constexpr int kHistBins = 4096;   // first-level histogram: top 12 bits of the 32-bit score key
constexpr int kHistShift = 20;

// One warp finds, in a 256-bin histogram, the largest digit d with sum_{d' >= d} h[d'] >= need.
// Returns d; *above = sum_{d' > d} h[d'].
__device__ __forceinline__ int warp_find_digit256(const uint32_t* h, uint32_t need,
                                                  uint32_t* above) {
  const int lane = threadIdx.x & 31;
  uint32_t q = 0;
#pragma unroll
  for (int i = 0; i < 8; ++i) q += h[8 * lane + i];
  uint32_t suf = q;  // inclusive suffix sum over lanes >= lane
#pragma unroll
  for (int off = 1; off < 32; off <<= 1) {
    const uint32_t v = __shfl_down_sync(0xFFFFFFFFu, suf, off);
    if (lane + off < 32) suf += v;
  }
  const uint32_t ball = __ballot_sync(0xFFFFFFFFu, suf >= need);
  const int L = ball ? 31 - __clz(ball) : 0;
  uint32_t run = __shfl_sync(0xFFFFFFFFu, suf, (L + 1) & 31);
  if (L == 31) run = 0;
  int d = 8 * L;
  if (lane == L) {
    for (int i = 7; i >= 0; --i) {
      const uint32_t c = h[8 * L + i];
      if (run + c >= need) {
        d = 8 * L + i;
        break;
      }
      run += c;
    }
  }
  d = __shfl_sync(0xFFFFFFFFu, d, L);
  run = __shfl_sync(0xFFFFFFFFu, run, L);
  *above = run;
  return d;
}

// The whole CTA finds the first-level threshold bin in a kHistBins histogram (global memory):
// the largest bin T with sum_{bins >= T} >= need. part must hold blockDim.x entries.
__device__ __forceinline__ int block_find_bin4096(const uint32_t* hist, uint32_t need,
                                                  uint32_t* part, int* result) {
  const int tid = threadIdx.x, nt = blockDim.x;
  const int per = kHistBins / nt;  // blockDim.x divides 4096
  uint32_t s = 0;
  for (int i = 0; i < per; ++i) s += hist[tid * per + i];
  part[tid] = s;
  __syncthreads();
  if (tid < 32) {
    // level 1: lanes own nt/32 parts each
    const int pl = nt / 32;
    uint32_t q = 0;
    for (int i = 0; i < pl; ++i) q += part[tid * pl + i];
    uint32_t suf = q;
#pragma unroll
    for (int off = 1; off < 32; off <<= 1) {
      const uint32_t v = __shfl_down_sync(0xFFFFFFFFu, suf, off);
      if (tid + off < 32) suf += v;
    }
    const uint32_t ball = __ballot_sync(0xFFFFFFFFu, suf >= need);
    const int L = ball ? 31 - __clz(ball) : 0;
    uint32_t run = __shfl_sync(0xFFFFFFFFu, suf, (L + 1) & 31);
    if (L == 31) run = 0;
    // level 2: walk lane L's parts from the top, then that part's bins
    int bin = 0;
    if (tid == 0) {
      int p = L * pl + pl - 1;
      for (; p > L * pl; --p) {
        if (run + part[p] >= need) break;
        run += part[p];
      }
      int i = p * per + per - 1;
      for (; i > p * per; --i) {
        const uint32_t c = hist[i];
        if (run + c >= need) break;
        run += c;
      }
      bin = i;
      *result = bin;
    }
  }
  __syncthreads();
  return *result;
}

struct RadixState {
  uint64_t prefix;
  int bits;  // number of known high bits of the threshold key
  uint32_t need;
  int done;
};

// Top-k of n distinct 64-bit keys by MSB-first radix select (whole CTA). get(i) returns key i.
// On return st->prefix / st->bits describe the threshold: key i is selected iff its top `bits`
// bits are >= those of prefix. k must be <= n. hist256: 256 shared words.
template <class Get>
__device__ void block_radix_select(const Get& get, int n, uint32_t k, uint32_t* hist256,
                                   RadixState* st) {
  const int tid = threadIdx.x, nt = blockDim.x;
  if (tid == 0) {
    st->prefix = 0;
    st->bits = 0;
    st->need = k;
    st->done = (k == 0);
  }
  __syncthreads();
  while (!st->done) {
    const int bits = st->bits;
    const uint64_t prefix = st->prefix;
    const int shift = 56 - bits;
    for (int i = tid; i < 256; i += nt) hist256[i] = 0;
    __syncthreads();
    for (int i = tid; i < n; i += nt) {
      const uint64_t key = get(i);
      if (bits == 0 || (key >> (64 - bits)) == (prefix >> (64 - bits)))
        atomicAdd(&hist256[(key >> shift) & 255u], 1u);
    }
    __syncthreads();
    if (tid < 32) {
      uint32_t above;
      const int d = warp_find_digit256(hist256, st->need, &above);
      if (tid == 0) {
        const uint32_t need = st->need - above;
        st->need = need;
        st->prefix = prefix | (static_cast<uint64_t>(d) << shift);
        st->bits = bits + 8;
        st->done = (hist256[d] == need) || (bits + 8 == 64);
      }
    }
    __syncthreads();
  }
}

__device__ __forceinline__ bool radix_selected(uint64_t key, const RadixState& st) {
  if (st.bits == 0) return true;
  return (key >> (64 - st.bits)) >= (st.prefix >> (64 - st.bits));
}

// Ascending bitonic sort of a[0..n2) in shared memory, n2 a power of two (whole CTA).
__device__ __forceinline__ void block_bitonic_sort_i32(int32_t* a, int n2) {
  const int tid = threadIdx.x, nt = blockDim.x;
  for (int k = 2; k <= n2; k <<= 1) {
    for (int j = k >> 1; j > 0; j >>= 1) {
      for (int i = tid; i < n2; i += nt) {
        const int l = i ^ j;
        if (l > i) {
          const int32_t x = a[i], y = a[l];
          const bool up = (i & k) == 0;
          if ((x > y) == up) {
            a[i] = y;
            a[l] = x;
          }
        }
      }
      __syncthreads();
    }
  }
}

}  // namespace csa2

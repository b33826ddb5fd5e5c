// select.cuh -- exact Top-K selection primitives used by the indexer kernels.
//
// Ranking: "DeepSeek V4.1 Flash 拆解" (austincafe.tech), section 一, selects a Top-K of indexer
// scores (and a Top-2048 of blocks); ties go to the lower index. Every item carries a 64-bit
// rank key (monotone score key in the high word, inverted index in the low word), so the Top-K is
// the set of the k largest keys, which are all distinct. The selection is an MSB-first radix
// select. Each pass histograms the next 12 bits of the keys that still match the known prefix
// (4,096 shared-memory bins) and stops as soon as the bin holding the k-th key is taken whole.
// The known prefix starts either from a min/max pass (the bits all keys share) or from a
// first-level histogram of the top 12 bits that the caller built while loading the keys.
// Winners are emitted in item order by an order-preserving compaction, over items in memory or
// over 16 items per thread held in registers, so item order (ascending index) needs no sort.
#pragma once

#include "common.cuh"

namespace csa2 {

constexpr int kHistBins = 4096;   // first-level histogram of the scan: top 12 bits of the key
constexpr int kHistShift = 20;
constexpr int kDigitBits = 12;    // radix digit of the in-CTA select
constexpr int kDigitBins = 1 << kDigitBits;

// ------------------------------------------------------------------------------- block scans

// Exclusive prefix sum of one value per thread over the CTA; *total receives the sum.
// scratch: 33 shared words. Must be called by every thread of the CTA.
__device__ __forceinline__ uint32_t block_exclusive_scan(uint32_t v, uint32_t* scratch,
                                                         uint32_t* total) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5, nw = (blockDim.x + 31) >> 5;
  uint32_t incl = v;
#pragma unroll
  for (int off = 1; off < 32; off <<= 1) {
    const uint32_t y = __shfl_up_sync(0xFFFFFFFFu, incl, off);
    if (lane >= off) incl += y;
  }
  if (lane == 31) scratch[warp] = incl;
  __syncthreads();
  if (warp == 0) {
    const uint32_t wv = lane < nw ? scratch[lane] : 0u;
    uint32_t wi = wv;
#pragma unroll
    for (int off = 1; off < 32; off <<= 1) {
      const uint32_t y = __shfl_up_sync(0xFFFFFFFFu, wi, off);
      if (lane >= off) wi += y;
    }
    if (lane < nw) scratch[lane] = wi - wv;  // exclusive warp offsets
    if (lane == 31) scratch[32] = wi;
  }
  __syncthreads();
  const uint32_t r = scratch[warp] + incl - v;
  *total = scratch[32];
  __syncthreads();  // scratch may be reused by the caller
  return r;
}

// ------------------------------------------------------------------------------ threshold bin

// The largest bin T of a 4096-bin histogram with sum_{bins >= T} >= need (whole CTA; blockDim.x
// is 256 or 1024, so each thread owns 16 or 4 consecutive bins). `hist` may live in global or
// shared memory. Each warp publishes its total; after one barrier every warp finds the crossing
// warp from the 32 totals on its own, and that warp finds the crossing thread and bin (kept in
// registers), so the search costs two barriers. part: >= 32 shared words; shared_int: 4 words;
// shared_int[3] receives the count in the bins above T.
__device__ __forceinline__ int block_find_bin4096(const uint32_t* hist, uint32_t need,
                                                  uint32_t* part, int* shared_int) {
  const int tid = threadIdx.x, nt = blockDim.x, lane = tid & 31, warp = tid >> 5;
  const int nw = nt >> 5;
  const int per = kHistBins / nt;
  uint32_t h[16];
#pragma unroll
  for (int i = 0; i < 16; ++i) h[i] = i < per ? hist[tid * per + i] : 0u;
  uint32_t s = 0;
#pragma unroll
  for (int i = 0; i < 16; ++i) s += h[i];
  uint32_t suf = s;  // this warp's bins owned by lanes >= lane
#pragma unroll
  for (int off = 1; off < 32; off <<= 1) {
    const uint32_t y = __shfl_down_sync(0xFFFFFFFFu, suf, off);
    if (lane + off < 32) suf += y;
  }
  if (lane == 0) part[warp] = suf;
  __syncthreads();
  // every warp: the crossing warp wl and the count in the warps above it
  const uint32_t v = lane < nw ? part[lane] : 0u;
  uint32_t sufw = v;
#pragma unroll
  for (int off = 1; off < 32; off <<= 1) {
    const uint32_t y = __shfl_down_sync(0xFFFFFFFFu, sufw, off);
    if (lane + off < 32) sufw += y;
  }
  const uint32_t ballw = __ballot_sync(0xFFFFFFFFu, lane < nw && sufw >= need);
  const int wl = ballw ? 31 - __clz(ballw) : 0;
  const uint32_t run = __shfl_sync(0xFFFFFFFFu, sufw - v, wl);
  if (warp == wl) {
    const uint32_t ball = __ballot_sync(0xFFFFFFFFu, run + suf >= need);
    const int jl = ball ? 31 - __clz(ball) : 0;
    if (lane == jl) {
      uint32_t r = run + suf - s;
      int bin = tid * per;
#pragma unroll
      for (int i = 15; i >= 0; --i) {
        if (i >= per) continue;
        if (r + h[i] >= need) {
          bin = tid * per + i;
          break;
        }
        r += h[i];
      }
      shared_int[2] = bin;
      shared_int[3] = static_cast<int>(r);
    }
  }
  __syncthreads();
  return shared_int[2];
}

// ------------------------------------------------------------------------------ radix select

struct RadixState {
  uint64_t prefix;
  int bits;  // number of known high bits of the threshold key
  uint32_t need;
  int done;
};

struct SelectScratch {
  uint32_t hist[kDigitBins];
  uint32_t part[1024];
  uint32_t scan[33];
  int ints[6];
  uint64_t red_min[32], red_max[32];
  RadixState st;
};

// Top-k of n distinct 64-bit keys (whole CTA). get(i) returns key i. On return sc.st describes
// the threshold: key i is selected iff its top `bits` bits are >= those of prefix. Requires
// 1 <= k <= n.
template <class Get>
__device__ void block_radix_select(const Get& get, int n, uint32_t k, SelectScratch& sc) {
  const int tid = threadIdx.x, nt = blockDim.x, lane = tid & 31, warp = tid >> 5;
  uint64_t kmin = ~0ull, kmax = 0ull;
  for (int i = tid; i < n; i += nt) {
    const uint64_t key = get(i);
    kmin = key < kmin ? key : kmin;
    kmax = key > kmax ? key : kmax;
  }
#pragma unroll
  for (int off = 16; off > 0; off >>= 1) {
    const uint64_t a = __shfl_xor_sync(0xFFFFFFFFu, kmin, off);
    const uint64_t b = __shfl_xor_sync(0xFFFFFFFFu, kmax, off);
    kmin = a < kmin ? a : kmin;
    kmax = b > kmax ? b : kmax;
  }
  if (lane == 0) {
    sc.red_min[warp] = kmin;
    sc.red_max[warp] = kmax;
  }
  __syncthreads();
  if (warp == 0) {
    const int nw = (nt + 31) / 32;
    kmin = lane < nw ? sc.red_min[lane] : ~0ull;
    kmax = lane < nw ? sc.red_max[lane] : 0ull;
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) {
      const uint64_t a = __shfl_xor_sync(0xFFFFFFFFu, kmin, off);
      const uint64_t b = __shfl_xor_sync(0xFFFFFFFFu, kmax, off);
      kmin = a < kmin ? a : kmin;
      kmax = b > kmax ? b : kmax;
    }
  }
  if (tid == 0) {
    const int common = (kmin == kmax) ? 64 : __clzll(static_cast<long long>(kmin ^ kmax));
    RadixState& st = sc.st;
    st.bits = common;
    st.prefix = common == 0 ? 0ull : (common == 64 ? kmax : (kmax & (~0ull << (64 - common))));
    st.need = k;
    st.done = (common == 64) || (static_cast<uint32_t>(n) == k);
    if (static_cast<uint32_t>(n) == k) {  // everything is selected
      st.bits = 0;
      st.prefix = 0ull;
    }
  }
  __syncthreads();
  while (!sc.st.done) {
    const int bits = sc.st.bits;
    const uint64_t prefix = sc.st.prefix;
    const int width = min(kDigitBits, 64 - bits);
    const int shift = 64 - bits - width;
    const uint64_t dmask = (1ull << width) - 1ull;
    for (int i = tid; i < kDigitBins; i += nt) sc.hist[i] = 0;
    __syncthreads();
    for (int i = tid; i < n; i += nt) {
      const uint64_t key = get(i);
      if (bits == 0 || (key >> (64 - bits)) == (prefix >> (64 - bits)))
        atomicAdd(&sc.hist[static_cast<uint32_t>((key >> shift) & dmask)], 1u);
    }
    __syncthreads();
    const uint32_t need = sc.st.need;
    const int d = block_find_bin4096(sc.hist, need, sc.part, sc.ints);
    if (tid == 0) {
      const uint32_t left = need - static_cast<uint32_t>(sc.ints[3]);
      sc.st.need = left;
      sc.st.prefix = prefix | (static_cast<uint64_t>(d) << shift);
      sc.st.bits = bits + width;
      sc.st.done = (sc.hist[d] == left) || (bits + width == 64);
    }
    __syncthreads();
  }
}

// Continues the radix select from sc.st when a first-level histogram of the top 12 key bits has
// already fixed them (bits = 12, need = what the bin of the k-th key still has to give), so no
// min/max pass runs. visit(f) calls f(key) for every key the calling thread holds; key 0 marks an
// empty item and is never counted. fresh: a 4096-word buffer that the caller cleared before its
// last barrier, used by the first pass so that it needs no clearing barrier (nullptr: clear
// sc.hist as every later pass does). Same stopping rule as block_radix_select.
template <class Visit>
__device__ void block_radix_refine_visit(const Visit& visit, uint32_t* fresh, SelectScratch& sc) {
  const int tid = threadIdx.x, nt = blockDim.x;
  bool first = true;
  while (!sc.st.done) {
    const int bits = sc.st.bits;  // 12 .. 63 here
    const uint64_t prefix = sc.st.prefix;
    const int width = min(kDigitBits, 64 - bits);
    const int shift = 64 - bits - width;
    const uint64_t dmask = (1ull << width) - 1ull;
    const uint64_t top = prefix >> (64 - bits);
    uint32_t* hist = sc.hist;
    if (first && fresh != nullptr) {
      hist = fresh;
    } else {
      for (int i = tid; i < kDigitBins; i += nt) sc.hist[i] = 0;
      __syncthreads();
    }
    first = false;
    visit([&](uint64_t key) {
      if (key != 0ull && (key >> (64 - bits)) == top)
        atomicAdd(&hist[static_cast<uint32_t>((key >> shift) & dmask)], 1u);
    });
    __syncthreads();
    const uint32_t need = sc.st.need;
    const int d = block_find_bin4096(hist, need, sc.part, sc.ints);
    if (tid == 0) {
      const uint32_t left = need - static_cast<uint32_t>(sc.ints[3]);
      sc.st.need = left;
      sc.st.prefix = prefix | (static_cast<uint64_t>(d) << shift);
      sc.st.bits = bits + width;
      sc.st.done = (hist[d] == left) || (bits + width == 64);
    }
    __syncthreads();
  }
}

// block_radix_refine_visit over n keys read with get(i).
template <class Get>
__device__ void block_radix_refine(const Get& get, int n, uint32_t* fresh, SelectScratch& sc) {
  const int tid = threadIdx.x, nt = blockDim.x;
  block_radix_refine_visit(
      [&](auto f) {
        for (int i = tid; i < n; i += nt) f(get(i));
      },
      fresh, sc);
}

// Sets sc.st after a first-level histogram `hist` of the top 12 bits of the nonzero keys (held
// in sc.hist or elsewhere): the bin T0 of the k-th key is fixed, and the select is done if that
// bin is taken whole. Whole CTA; 1 <= k <= the histogram's total.
__device__ __forceinline__ void radix_state_from_top12(const uint32_t* hist, uint32_t k,
                                                       SelectScratch& sc) {
  const int T0 = block_find_bin4096(hist, k, sc.part, sc.ints);
  if (threadIdx.x == 0) {
    const uint32_t left = k - static_cast<uint32_t>(sc.ints[3]);
    sc.st.prefix = static_cast<uint64_t>(T0) << (64 - kDigitBits);
    sc.st.bits = kDigitBits;
    sc.st.need = left;
    sc.st.done = hist[T0] == left;
  }
  __syncthreads();
}

// Is key among the selected ones, i.e. are its top st.bits bits >= those of the threshold? Every
// select leaves the bits of st.prefix below its top st.bits at zero (and st.prefix = 0 when
// st.bits = 0), so comparing the shifted words is the same as comparing the keys themselves.
__device__ __forceinline__ bool radix_selected(uint64_t key, const RadixState& st) {
  return key >= st.prefix;
}

// Order-preserving compaction over items 0..n-1 (whole CTA): emit(i, slot) is called for every
// item with pred(i), slot counting those items in item order. Warp w owns a contiguous segment of
// items and its lanes take consecutive items (conflict-free shared-memory reads); ballot prefix
// counts keep the order inside a warp and a scan over the warps' totals orders the segments.
// Returns the number of items emitted; everything emitted is visible to the whole CTA on return.
template <class Pred, class Emit>
__device__ uint32_t block_ordered_compact(int n, const Pred& pred, const Emit& emit,
                                          uint32_t* scan_scratch) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5, nw = (blockDim.x + 31) >> 5;
  const int seg = ((n + nw - 1) / nw + 31) & ~31;
  const int lo = min(n, warp * seg), hi = min(n, lo + seg);
  uint32_t c = 0;
  for (int i = lo + lane; i < hi; i += 32) c += pred(i) ? 1u : 0u;
  c = __reduce_add_sync(0xFFFFFFFFu, c);
  uint32_t total;
  // one value per thread: lane 0 carries the warp's count
  const uint32_t warp_off = block_exclusive_scan(lane == 0 ? c : 0u, scan_scratch, &total);
  uint32_t base = __shfl_sync(0xFFFFFFFFu, warp_off, 0);
  for (int i0 = lo; i0 < hi; i0 += 32) {
    const int i = i0 + lane;
    const bool p = i < hi && pred(i);
    const uint32_t ball = __ballot_sync(0xFFFFFFFFu, p);
    if (p) emit(i, base + __popc(ball & ((1u << lane) - 1u)));
    base += __popc(ball);
  }
  __syncthreads();
  return total;
}

// Order-preserving compaction over items held in registers by a CTA of 1,024 threads: thread t
// holds item 1024 j + t in its slot j (j < NK, NK = 4 or 16). emit(j, slot) runs for each item
// with sel(j), slot counting the selected items in item order. The (slot, warp) counts are
// published in item order and every warp takes its offsets from them after one barrier. wc: 544
// shared words (32 NK counts, one pad word after every 16 so that a lane's reads hit distinct
// banks). Returns the count; the caller synchronises before emitted data is read by other
// threads or wc is reused. kKeepMasks: keep the NK ballot masks in registers across the barrier,
// or form them again after it (for callers short of registers).
template <int NK, bool kKeepMasks, class Sel, class Emit>
__device__ uint32_t block_ordered_compact_regs(const Sel& sel, const Emit& emit, uint32_t* wc) {
  static_assert(NK == 4 || NK == 16, "4 or 16 items per thread");
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  uint32_t mk[NK];
#pragma unroll
  for (int j = 0; j < NK; ++j) {
    const uint32_t m = __ballot_sync(0xFFFFFFFFu, sel(j));
    if (kKeepMasks) mk[j] = m;
    const int e = 32 * j + warp;  // item order of (slot j, warp)
    if (lane == 0) wc[e + (e >> 4)] = static_cast<uint32_t>(__popc(m));
  }
  __syncthreads();
  // lane l holds entries NK l .. NK l + NK - 1; this warp's entries sit at offset warp % NK of
  // lanes (32 / NK) j + warp / NK
  uint32_t lsum = 0, lpre = 0;
#pragma unroll
  for (int q = 0; q < NK; ++q) {
    const int e = NK * lane + q;
    const uint32_t cq = wc[e + (e >> 4)];
    lpre += q < (warp % NK) ? cq : 0u;
    lsum += cq;
  }
  uint32_t incl = lsum;
#pragma unroll
  for (int off = 1; off < 32; off <<= 1) {
    const uint32_t y = __shfl_up_sync(0xFFFFFFFFu, incl, off);
    if (lane >= off) incl += y;
  }
  const uint32_t total = __shfl_sync(0xFFFFFFFFu, incl, 31);
  const uint32_t mine = incl - lsum + lpre;
  const uint32_t lt = (1u << lane) - 1u;
#pragma unroll
  for (int j = 0; j < NK; ++j) {
    const uint32_t base = __shfl_sync(0xFFFFFFFFu, mine, (32 / NK) * j + warp / NK);
    const uint32_t m = kKeepMasks ? mk[j] : __ballot_sync(0xFFFFFFFFu, sel(j));
    if ((m >> lane) & 1u) emit(j, base + static_cast<uint32_t>(__popc(m & lt)));
  }
  return total;
}

template <bool kKeepMasks, class Sel, class Emit>
__device__ uint32_t block_ordered_compact_regs16(const Sel& sel, const Emit& emit, uint32_t* wc) {
  return block_ordered_compact_regs<16, kKeepMasks>(sel, emit, wc);
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

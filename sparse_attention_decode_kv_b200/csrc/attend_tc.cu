// attend_tc.cu -- sparse attention of one query per row (16 heads x 512) over selected MXFP4 main-KV
// entries and FP8 SWA rows on the sm_100a tensor cores (tcgen05), for batches that fill the GPU.
// The mma.sync kernel in attend.cu computes the same result and serves small batches.
//
// Method: "DeepSeek V4.1 Flash 拆解" (austincafe.tech), section 一: a Reuse-mode layer reuses the
// indices and runs sparse attention directly; the main KV is MXFP4, the SWA KV stays FP8.
// Reading (as in attend.cu): K = V = the dequantised entry; z = softmax_scale * q . v over the
// selected entries and the valid SWA rows together; out = sum softmax(z) v; lse = log sum exp(z).
//
// Orientation: items on M = 128, the 16 heads on N. Per tile of 128 items
//   S^T [128 x 16]  = V [128 x 512] q^T       A = V in tensor memory (lane = item), B = q in smem
//   O^T [512 x 16] += V^T [512 x 128] P^T     A = the fp16 V tile in smem read MN-major, B = P
// with both accumulators in tensor memory. A tcgen05.mma of M = 128, N = 16, K = 16 holds the
// tensor core for 40-50 cycles whatever N up to 64 (measured on B200), so the two products cost
// 20-25 tensor cycles per item; the QK^T of a tile is issued by one thread and the P.V of the
// previous tile by another, so the two overlap on the tensor core.
//
// Warp roles (512 threads, one CTA per SM, persistent over (query, split) units):
//   warps 0, 3   gather, 64 items each: index loads, then TMA copies into a two-slot ring
//                completing on mbarriers: tile::gather4 of four items' 128-byte code halves and
//                32-byte scale rows per instruction, tiled 128 x 64-row loads of the contiguous SWA
//                window (the issue rate per warp bounds a gather, so two warps issue); the CTA's
//                first tile of indices is issued by the dequantisation warps, idle until it lands
//   warp 1       issues QK^T (and owns the tensor-memory allocation)
//   warp 2       issues P.V
//   warps 4-11   dequantise, one item per thread and half the dims per warp (dim half h = the P.V
//                blocks h and h + 2, dims 128 h .. + 127 and 256 + 128 h .. + 127): pass A writes the fp16
//                row into tensor memory for QK^T as soon as the previous tile's QK^T has read it
//                and frees the raw slot; pass B copies the row from tensor memory into the fp16 smem
//                tile block by block as the previous tile's P.V frees it (the smem holds one
//                128 KiB tile only)
//   warps 12-15  softmax: logits from tensor memory, per-head tile maxima, probabilities into the
//                fp16 P tile, lazy rescaling of O; then the unit's epilogue (O / l, lse or partials)
//
// Items that are not valid (index -1 or outside [0, N), SWA slots past the window) are gathered
// from an in-range row and zeroed by the dequantisation, with logit -inf.
//
// Numerics as in attend.cu: every dequantised MXFP4 value and every E4M3 element is exact in fp16;
// q is scaled per head by a power of two into fp16's range; the SWA token scale multiplies the
// logit and the probability, and P on SWA tiles carries a power of two that brings the largest
// token scale to [1, 2). Logits are kept in base-2 units. The reference maxima move only when a
// tile's maximum exceeds them by more than 2^8 (so P <= 2^9 stays in fp16 range); O and l are
// rescaled then, and both stay relative to the same maxima, so the result does not depend on when.
#include <math.h>

#include <stdint.h>

#include <algorithm>
#include <mutex>
#include <vector>

#include "common.cuh"
#include "internal.h"
#include "tcgen05.cuh"

namespace csa2 {

namespace {

constexpr int kT = 128;                  // items per tile
constexpr int kTcThreads = 512;          // 16 warps
constexpr int kCodeRow = D / 2;          // 256 code bytes per MXFP4 entry
constexpr int kScaleRow = D / 16;        // 32 scale bytes
constexpr uint32_t kVsBytes = kT * D * 2;                      // fp16 V: 8 dim-blocks of [128 x 128 B]
constexpr uint32_t kQBytes = HQ * D * 2;                       // fp16 q: 8 dim-blocks of [16 x 128 B]
constexpr uint32_t kPBytes = HQ * kT * 2;                      // fp16 P: 2 item-blocks of [16 x 128 B]
constexpr uint32_t kStage = kT * (kCodeRow + kScaleRow);       // one MXFP4 tile, or 64 SWA rows
// MXFP4 slot: code bytes 0..127 of the 128 items as [128 rows x 128 B] with 128-byte swizzle, bytes
// 128..255 likewise, then the scale rows [128 x 32 B]. SWA half slot: 4 column quarters of
// [64 rows x 128 B], 128-byte swizzle.
constexpr uint32_t kCodeHalf = kT * 128;
constexpr uint32_t kScalesAt = 2 * kCodeHalf;
constexpr uint32_t kSwaQuarter = 64 * 128;
constexpr uint32_t kOffQ = kVsBytes;
constexpr uint32_t kOffP = kOffQ + kQBytes;
constexpr uint32_t kOffRaw = kOffP + kPBytes;
constexpr uint32_t kOffSmall = kOffRaw + 2 * kStage;
// tensor-memory columns
constexpr uint32_t kColVa = 0;     // V for QK^T: lane = item, 256 columns of two fp16 dims
constexpr uint32_t kColS = 256;    // S^T: two slots of 16 columns
constexpr uint32_t kColO = 320;    // O^T: two slots (units) of 4 blocks x 16 columns
constexpr uint32_t kTmemCols = 512;
constexpr uint32_t kIdescQK = umma_idesc_f16_f32(128, 16, false);
constexpr uint32_t kIdescPV = umma_idesc_f16_f32(128, 16, true);
constexpr float kLog2e = 1.4426950408889634f;
constexpr float kLn2 = 0.6931471805599453f;
constexpr float kRescaleGap = 8.0f;  // base-2 units

struct TcSmall {
  uint64_t raw_full[2], raw_empty[2];
  uint64_t meta_full[3], meta_empty[3];
  uint64_t va_full[2], va_empty[2];
  uint64_t vs_full[4], vs_empty[4];
  uint64_t s_full[2], s_empty[2];
  uint64_t p_full, p_empty;
  uint64_t o_prog, o_full[2], o_empty[2];
  uint64_t q_full, drain;
  float meta[3][kT];           // per item: 1 (MXFP4) or the SWA token's scale; -1 when not valid
  float meta_smax[3][2];       // largest valid SWA token scale of each gather warp's items (0 if none)
  float red[2][4][HQ + 1];     // per-warp tile maxima and SWA scale maximum, by tile parity
  float lred[4][HQ];           // per-warp sums of l in the epilogue
  float scout[HQ];             // per head: the epilogue's scale of O
  float q_unscale[HQ];         // 2^(e_h - 14) * softmax_scale * log2(e)
  uint32_t tmem_base;
  int abort;
};
constexpr size_t kTcSmem = kOffSmall + sizeof(TcSmall) + 1024;  // + slack to align the base
static_assert(kTcSmem <= 232448, "shared memory of the tcgen05 attention");

// ------------------------------------------------------------------------------ small helpers

__device__ __forceinline__ bool tc_wait(uint64_t* bar, uint32_t parity, volatile int* abort) {
  if (mbar_try_wait(bar, parity)) return true;
  const uint64_t t0 = globaltimer_ns();
  while (!mbar_try_wait(bar, parity)) {
    if (*abort) return false;
    if (globaltimer_ns() - t0 > kWaitLimitNs) return false;
  }
  return true;
}

// Whole-warp wait: the warp goes on only if every lane saw the phase complete.
__device__ __forceinline__ bool tc_wait_warp(uint64_t* bar, uint32_t parity, volatile int* abort) {
  return __all_sync(0xFFFFFFFFu, tc_wait(bar, parity, abort));
}

__device__ __forceinline__ void tc_give_up(volatile int* abort, int32_t* dev_err) {
  if (!*abort) flag_error(dev_err, CSA2_DEVERR_TIMEOUT);
  *abort = 1;
}

// Named barrier of the four softmax warps, and the same barrier with an AND over a predicate.
__device__ __forceinline__ void softmax_sync() { asm volatile("bar.sync 1, 128;" ::: "memory"); }
__device__ __forceinline__ bool softmax_all(bool v) {
  uint32_t r;
  asm volatile(
      "{\n\t.reg .pred p, q;\n\tsetp.ne.u32 q, %1, 0;\n\tbar.red.and.pred p, 1, 128, q;\n\t"
      "selp.u32 %0, 1, 0, p;\n\t}"
      : "=r"(r)
      : "r"(static_cast<uint32_t>(v))
      : "memory");
  return r != 0;
}

__device__ __forceinline__ bool softmax_any(bool v) {
  uint32_t r;
  asm volatile(
      "{\n\t.reg .pred p, q;\n\tsetp.ne.u32 q, %1, 0;\n\tbar.red.or.pred p, 1, 128, q;\n\t"
      "selp.u32 %0, 1, 0, p;\n\t}"
      : "=r"(r)
      : "r"(static_cast<uint32_t>(v))
      : "memory");
  return r != 0;
}

__device__ __forceinline__ void fence_proxy_async_smem() {
  asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}

__device__ __forceinline__ uint4 lds16(uint32_t addr) {
  uint4 r;
  asm volatile("ld.shared.v4.u32 {%0, %1, %2, %3}, [%4];"
               : "=r"(r.x), "=r"(r.y), "=r"(r.z), "=r"(r.w)
               : "r"(addr));
  return r;
}

__device__ __forceinline__ uint2 lds8(uint32_t addr) {
  uint2 r;
  asm volatile("ld.shared.v2.u32 {%0, %1}, [%2];" : "=r"(r.x), "=r"(r.y) : "r"(addr));
  return r;
}

// The k-th of the eight 32-dim chunks of dim half h: the chunks of P.V blocks h and h + 2.
__device__ __forceinline__ int half_chunk(int h, int k) {
  return k < 4 ? 4 * h + k : 8 + 4 * h + (k - 4);
}

__device__ __forceinline__ void sts16(uint32_t addr, uint32_t a, uint32_t b, uint32_t c, uint32_t d) {
  asm volatile("st.shared.v4.u32 [%0], {%1, %2, %3, %4};" ::"r"(addr), "r"(a), "r"(b), "r"(c), "r"(d)
               : "memory");
}

__device__ __forceinline__ void sts_u16(uint32_t addr, uint16_t v) {
  asm volatile("st.shared.u16 [%0], %1;" ::"r"(addr), "h"(v) : "memory");
}

// 128-byte swizzle inside a region of 128-byte rows: 16-byte column c of row r.
__device__ __forceinline__ uint32_t swz(int r, int c) {
  return static_cast<uint32_t>(r * 128 + ((c ^ (r & 7)) << 4));
}

__device__ __forceinline__ float ex2f(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}

__device__ __forceinline__ float pow2f_tc(int k) {
  k = max(-126, min(127, k));
  return __uint_as_float(static_cast<uint32_t>(k + 127) << 23);
}

__device__ __forceinline__ int ilog2f_tc(float x) {
  const int e = static_cast<int>((__float_as_uint(x) >> 23) & 0xFF);
  return e == 0 ? -126 : e - 127;
}

// Four bytes of E2M1 pairs -> four half2 (byte j -> o[j], low nibble in .x).
__device__ __forceinline__ void e2m1x8_h2(uint32_t w, uint32_t& o0, uint32_t& o1, uint32_t& o2,
                                          uint32_t& o3) {
  asm("{\n\t.reg .b8 b0, b1, b2, b3;\n\tmov.b32 {b0, b1, b2, b3}, %4;\n\t"
      "cvt.rn.f16x2.e2m1x2 %0, b0;\n\tcvt.rn.f16x2.e2m1x2 %1, b1;\n\t"
      "cvt.rn.f16x2.e2m1x2 %2, b2;\n\tcvt.rn.f16x2.e2m1x2 %3, b3;\n\t}"
      : "=r"(o0), "=r"(o1), "=r"(o2), "=r"(o3)
      : "r"(w));
}

// Four E4M3 bytes -> two half2.
__device__ __forceinline__ void e4m3x4_h2(uint32_t w, uint32_t& o0, uint32_t& o1) {
  asm("{\n\t.reg .b16 h0, h1;\n\tmov.b32 {h0, h1}, %2;\n\t"
      "cvt.rn.f16x2.e4m3x2 %0, h0;\n\tcvt.rn.f16x2.e4m3x2 %1, h1;\n\t}"
      : "=r"(o0), "=r"(o1)
      : "r"(w));
}

// 32 dims (dims 32 c .. 32 c + 31) of item i as 16 half2 (r[j] = dims 32 c + 2 j, + 1), zero when
// the item is not valid. MXFP4: 16-byte column c & 7 of the code half c >> 3, swizzled by the row;
// `sc4` holds the 16 scale bytes of the warp's dims (groups 8 h .. 8 h + 7, then 16 + 8 h ..
// 16 + 8 h + 7) and k is the chunk's place among the warp's eight. SWA: row i & 63 of its half
// slot, 16-byte columns 2 c and 2 c + 1 of the 512-byte row.
__device__ __forceinline__ void convert_chunk(uint32_t st, bool is_swa, bool valid, int i, int c, int k,
                                              const uint4& sc4, uint32_t (&r)[16]) {
  if (!is_swa) {
    const uint4 cw = lds16(st + static_cast<uint32_t>((c >> 3) * kCodeHalf + i * 128 + (((c & 7) ^ (i & 7)) << 4)));
    const uint32_t sw = (k < 4 ? (k < 2 ? sc4.x : sc4.y) : (k < 6 ? sc4.z : sc4.w));
    const uint32_t s01 = e4m3x2_to_h2((sw >> (16 * (k & 1))) & 0xFFFFu);
    const uint32_t slo = __byte_perm(s01, 0, 0x1010), shi = __byte_perm(s01, 0, 0x3232);
    e2m1x8_h2(cw.x, r[0], r[1], r[2], r[3]);
    e2m1x8_h2(cw.y, r[4], r[5], r[6], r[7]);
    e2m1x8_h2(cw.z, r[8], r[9], r[10], r[11]);
    e2m1x8_h2(cw.w, r[12], r[13], r[14], r[15]);
#pragma unroll
    for (int j = 0; j < 8; ++j) r[j] = h2_mul(r[j], slo);
#pragma unroll
    for (int j = 8; j < 16; ++j) r[j] = h2_mul(r[j], shi);
  } else {
    const int rr = i & 63;
    const uint32_t q0 = st + static_cast<uint32_t>((c >> 2) * kSwaQuarter + rr * 128);
    const uint4 e0 = lds16(q0 + static_cast<uint32_t>(((2 * (c & 3)) ^ (rr & 7)) << 4));
    const uint4 e1 = lds16(q0 + static_cast<uint32_t>(((2 * (c & 3) + 1) ^ (rr & 7)) << 4));
    e4m3x4_h2(e0.x, r[0], r[1]);
    e4m3x4_h2(e0.y, r[2], r[3]);
    e4m3x4_h2(e0.z, r[4], r[5]);
    e4m3x4_h2(e0.w, r[6], r[7]);
    e4m3x4_h2(e1.x, r[8], r[9]);
    e4m3x4_h2(e1.y, r[10], r[11]);
    e4m3x4_h2(e1.z, r[12], r[13]);
    e4m3x4_h2(e1.w, r[14], r[15]);
  }
  if (!valid) {
#pragma unroll
    for (int j = 0; j < 16; ++j) r[j] = 0u;
  }
}

// Cache sequence, cached length and SWA window of query b (errors flagged when `report`).
struct QueryRows {
  int sb, nb, sl, slo;
  int64_t row0;  // first cache row of the sequence
};

__device__ QueryRows query_rows(int b, const int32_t* __restrict__ N, int n_cap, int W,
                                const int32_t* __restrict__ swa_len, const int32_t* __restrict__ qseq,
                                const int32_t* __restrict__ swa_lo, int S, int nseq, int32_t* dev_err,
                                bool report) {
  QueryRows q;
  int sb = qseq ? __ldg(qseq + b) : b;
  const bool sb_ok = sb >= 0 && sb < nseq;
  if (!sb_ok) {  // an unknown sequence: the query attends to nothing
    if (report) flag_error(dev_err, CSA2_DEVERR_INDEX_RANGE);
    sb = 0;
  }
  int nb = sb_ok ? __ldg(N + sb) : 0;
  if (nb < 0 || nb > n_cap) {
    if (report) flag_error(dev_err, CSA2_DEVERR_NLEN);
    nb = max(0, min(nb, n_cap));
  }
  int sl = 0;
  if (W > 0) {
    sl = (swa_len && sb_ok) ? __ldg(swa_len + b) : 0;
    if (sl < 0 || sl > W) {
      if (report) flag_error(dev_err, CSA2_DEVERR_NLEN);
      sl = max(0, min(sl, W));
    }
  }
  int slo = 0;
  if (swa_lo != nullptr && sl > 0) {
    slo = __ldg(swa_lo + b);
    if (slo < 0 || slo + sl > S) {
      if (report) flag_error(dev_err, CSA2_DEVERR_NLEN);
      slo = max(0, min(slo, S));
      sl = min(sl, S - slo);
    }
  }
  q.sb = sb;
  q.nb = nb;
  q.sl = sl;
  q.slo = slo;
  q.row0 = static_cast<int64_t>(sb) * n_cap;
  return q;
}

// Max (or sum) of 16 per-head values over the 32 lanes: after the exchange, lanes 2m and 2m + 1
// hold the result for head hd(lane) = 8 b4 + 4 b3 + 2 b2 + b1 (b = lane bits).
template <bool kMax>
__device__ __forceinline__ float warp_reduce16(float (&v)[HQ], int lane) {
  float a[8];
#pragma unroll
  for (int k = 0; k < 8; ++k) {
    const bool up = lane & 16;
    const float send = up ? v[k] : v[k + 8];
    const float keep = up ? v[k + 8] : v[k];
    const float got = __shfl_xor_sync(0xFFFFFFFFu, send, 16);
    a[k] = kMax ? fmaxf(keep, got) : keep + got;
  }
  float b[4];
#pragma unroll
  for (int k = 0; k < 4; ++k) {
    const bool up = lane & 8;
    const float send = up ? a[k] : a[k + 4];
    const float keep = up ? a[k + 4] : a[k];
    const float got = __shfl_xor_sync(0xFFFFFFFFu, send, 8);
    b[k] = kMax ? fmaxf(keep, got) : keep + got;
  }
  float c[2];
#pragma unroll
  for (int k = 0; k < 2; ++k) {
    const bool up = lane & 4;
    const float send = up ? b[k] : b[k + 2];
    const float keep = up ? b[k + 2] : b[k];
    const float got = __shfl_xor_sync(0xFFFFFFFFu, send, 4);
    c[k] = kMax ? fmaxf(keep, got) : keep + got;
  }
  const bool up = lane & 2;
  const float send = up ? c[0] : c[1];
  const float keep = up ? c[1] : c[0];
  const float got = __shfl_xor_sync(0xFFFFFFFFu, send, 2);
  float d = kMax ? fmaxf(keep, got) : keep + got;
  const float o = __shfl_xor_sync(0xFFFFFFFFu, d, 1);
  return kMax ? fmaxf(d, o) : d + o;
}

__device__ __forceinline__ int reduce16_head(int lane) {
  return ((lane >> 4) & 1) * 8 + ((lane >> 3) & 1) * 4 + ((lane >> 2) & 1) * 2 + ((lane >> 1) & 1);
}

struct TcArgs {
  const uint16_t* q;
  float softmax_scale;
  const uint8_t* codes;
  const uint8_t* scales;
  int n_cap;
  const int32_t* N;
  const int32_t* idx;
  int K;
  const uint8_t* swa;
  const float* swa_scale;
  const int32_t* swa_len;
  int W;
  const int32_t* qseq;
  const int32_t* swa_lo;
  int S;
  int nseq;
  int B;
  int nsplit;
  float* out;
  float* lse;
  float* part_o;
  float* part_ml;
  int32_t* dev_err;
  int early_rows;
};

// q of query b -> fp16 in the K-major smem tile with a per-head power of two; q_unscale[h].
// 128 softmax threads: head st / 8, dims 64 (st % 8) .. + 63.
__device__ void stage_q(const TcArgs& a, int b, int st, uint32_t q_smem, TcSmall& sm) {
  const int h = st >> 3, db = st & 7;
  const uint4* src = reinterpret_cast<const uint4*>(a.q + (static_cast<int64_t>(b) * HQ + h) * D + 64 * db);
  uint4 u[8];
#pragma unroll
  for (int k = 0; k < 8; ++k) u[k] = __ldg(src + k);
  float amax = 0.0f;
#pragma unroll
  for (int k = 0; k < 8; ++k) {
    const uint32_t w4[4] = {u[k].x, u[k].y, u[k].z, u[k].w};
#pragma unroll
    for (int e = 0; e < 4; ++e) amax = fmaxf(amax, fmaxf(fabsf(bf16lo(w4[e])), fabsf(bf16hi(w4[e]))));
  }
#pragma unroll
  for (int off = 4; off > 0; off >>= 1) amax = fmaxf(amax, __shfl_xor_sync(0xFFFFFFFFu, amax, off));
  const int eh = amax > 0.0f ? ilog2f_tc(amax) : 0;
  const float up = pow2f_tc(14 - eh);
  if (db == 0) sm.q_unscale[h] = pow2f_tc(eh - 14) * a.softmax_scale * kLog2e;
  const uint32_t base = q_smem + static_cast<uint32_t>(db * (HQ * 128));
#pragma unroll
  for (int k = 0; k < 8; ++k) {
    const uint32_t w4[4] = {u[k].x, u[k].y, u[k].z, u[k].w};
    uint32_t h2[4];
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      __half2 hv = __floats2half2_rn(bf16lo(w4[e]) * up, bf16hi(w4[e]) * up);
      h2[e] = *reinterpret_cast<uint32_t*>(&hv);
    }
    sts16(base + swz(h, k), h2[0], h2[1], h2[2], h2[3]);
  }
}

// The CTA's first tile is gathered by the dequantisation warps, which would otherwise wait for it,
// when it is a tile of indices (the gather warps then only post its expected bytes). Both sides
// decide from the same values.
__device__ __forceinline__ bool first_tile_by_dequant(int units, int nsplit, int tiles, int tiles_idx) {
  const int unit = static_cast<int>(blockIdx.x);
  if (unit >= units) return false;
  const int split = unit % nsplit;
  const int tb = static_cast<int>(static_cast<int64_t>(split) * tiles / nsplit);
  const int te = static_cast<int>(static_cast<int64_t>(split + 1) * tiles / nsplit);
  return tb < te && tb < tiles_idx;
}

__global__ void __launch_bounds__(kTcThreads, 1)
    attend_tc_kernel(const __grid_constant__ CUtensorMap tm_codes,
                     const __grid_constant__ CUtensorMap tm_scales,
                     const __grid_constant__ CUtensorMap tm_swa, const TcArgs a) {
  extern __shared__ __align__(1024) unsigned char smem_raw[];
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  // 1024-byte aligned base for the swizzled tiles
  const uint32_t raw_addr = smem_u32(smem_raw);
  const uint32_t base = (raw_addr + 1023u) & ~1023u;
  unsigned char* smem = smem_raw + (base - raw_addr);
  const uint32_t vs = base, q_smem = base + kOffQ, p_smem = base + kOffP, raw0 = base + kOffRaw;
  TcSmall& sm = *reinterpret_cast<TcSmall*>(smem + kOffSmall);
  volatile int* abort = &sm.abort;

  const int tiles_idx = (a.K + kT - 1) / kT;
  const int tiles = tiles_idx + (a.W + kT - 1) / kT;
  const int nsplit = a.nsplit;
  const int units = a.B * nsplit;

  if (tid == 0) {
    for (int s = 0; s < 2; ++s) {
      mbar_init(&sm.raw_full[s], 2);    // the gather warps' expect-tx arrivals, then the bytes
      mbar_init(&sm.raw_empty[s], 8);   // the eight dequantisation warps
      mbar_init(&sm.va_full[s], 4);     // the four warps of a dim half
      mbar_init(&sm.va_empty[s], 1);
      mbar_init(&sm.s_full[s], 1);
      mbar_init(&sm.s_empty[s], 4);
      mbar_init(&sm.o_full[s], 1);
      mbar_init(&sm.o_empty[s], 4);
    }
    for (int s = 0; s < 3; ++s) {
      mbar_init(&sm.meta_full[s], 64);
      mbar_init(&sm.meta_empty[s], 4);
    }
    for (int j = 0; j < 4; ++j) {
      mbar_init(&sm.vs_full[j], 4);
      mbar_init(&sm.vs_empty[j], 1);
    }
    mbar_init(&sm.p_full, 4);
    mbar_init(&sm.p_empty, 1);
    mbar_init(&sm.o_prog, 1);
    mbar_init(&sm.q_full, 4);
    mbar_init(&sm.drain, 2);
    sm.abort = 0;
    fence_barrier_init();
  }
  if (warp == 1) {
    tmem_alloc(&sm.tmem_base, kTmemCols);
    tmem_relinquish();
  }
  tcgen05_fence_before();
  __syncthreads();
  tcgen05_fence_after();
  const uint32_t tmem = sm.tmem_base;

  if (warp == 0 || warp == 3) {
    // -------------------------------------------------------------------------------- gather
    const int pw = warp == 0 ? 0 : 1;  // items 64 pw .. 64 pw + 63
    const int g = lane & 15;           // this lane's group of four items
    if (lane == 0) {  // the tensor maps are kernel parameters: fetch them while the CTA starts
      if (pw == 0) {
        asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(&tm_codes)) : "memory");
      } else {
        asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(&tm_scales)) : "memory");
        asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(&tm_swa)) : "memory");
      }
    }
    bool waited = a.early_rows == 0;
    if (waited) {
      pdl_wait();
      pdl_launch_dependents();
    }
    int gt = 0, sn = 0;
    int fills[2] = {0, 0};  // copies issued into each slot
    bool alive = true;
    const bool first_by_dequant = first_tile_by_dequant(units, nsplit, tiles, tiles_idx);
    for (int j = 0; alive; ++j) {
      const int unit = static_cast<int>(blockIdx.x) + j * static_cast<int>(gridDim.x);
      if (unit >= units) break;
      const int b = unit / nsplit, split = unit - b * nsplit;
      const int tb = static_cast<int>(static_cast<int64_t>(split) * tiles / nsplit);
      const int te = static_cast<int>(static_cast<int64_t>(split + 1) * tiles / nsplit);
      const QueryRows qr = query_rows(b, a.N, a.n_cap, a.W, a.swa_len, a.qseq, a.swa_lo, a.S, a.nseq,
                                      a.dev_err, pw == 0 && lane == 0);
      for (int tile = tb; tile < te; ++tile, ++gt) {
        const bool is_swa = tile >= tiles_idx;
        if (!waited && is_swa) {  // SWA rows: only after the preceding kernel
          pdl_wait();
          pdl_launch_dependents();
          waited = true;
        }
        const int tbase = is_swa ? (tile - tiles_idx) * kT : tile * kT;
        const int count = min(kT, (is_swa ? a.W : a.K) - tbase);
        const int ms = gt % 3;
        if (gt >= 3 && !tc_wait_warp(&sm.meta_empty[ms], static_cast<uint32_t>(((gt / 3) - 1) & 1), abort)) {
          alive = false;
          break;
        }
        if (!is_swa) {
          const int slot = sn & 1;
          if (sn >= 2 && !tc_wait_warp(&sm.raw_empty[slot], static_cast<uint32_t>(((sn >> 1) - 1) & 1), abort)) {
            alive = false;
            break;
          }
          // lanes l and l + 16 both hold the rows of items 64 pw + 4 g .. + 3
          int row[4];
#pragma unroll
          for (int k = 0; k < 4; ++k) {
            const int item = 64 * pw + 4 * g + k;
            const int p = item < count ? __ldg(a.idx + static_cast<int64_t>(b) * a.K + tbase + item) : -1;
            const bool v = p >= 0 && p < qr.nb;
            if (lane < 16) {
              if (!v && p != -1) flag_error(a.dev_err, CSA2_DEVERR_INDEX_RANGE);
              sm.meta[ms][item] = v ? 1.0f : -1.0f;
            }
            row[k] = static_cast<int>(qr.row0 + (v ? p : 0));  // row counts fit int32 (host check)
          }
          const uint32_t st = raw0 + static_cast<uint32_t>(slot) * kStage;
          if (lane == 0) mbar_arrive_expect_tx(&sm.raw_full[slot], kStage / 2);
          __syncwarp();
          const uint32_t grp = static_cast<uint32_t>(16 * pw + g);  // group of 4 items in the tile
          if (gt > 0 || !first_by_dequant) {
            // lanes 0..15: code bytes 0..127 and the scale rows; lanes 16..31: code bytes 128..255
            tma_gather4(st + (lane >> 4) * kCodeHalf + 512u * grp, &tm_codes, &sm.raw_full[slot],
                        128 * (lane >> 4), row[0], row[1], row[2], row[3]);
            if (lane < 16)
              tma_gather4(st + kScalesAt + 128u * grp, &tm_scales, &sm.raw_full[slot], 0, row[0], row[1],
                          row[2], row[3]);
          }
          ++fills[slot];
          sn += 1;
        } else {
          float smx = 0.0f;
#pragma unroll
          for (int k = 0; k < 2; ++k) {
            const int item = 64 * pw + 32 * k + lane, sidx = tbase + item;
            const bool v = item < count && sidx < qr.sl;
            const float sc = v ? __ldg(a.swa_scale + static_cast<int64_t>(qr.sb) * a.S + qr.slo + sidx) : -1.0f;
            sm.meta[ms][item] = sc;
            smx = fmaxf(smx, sc);
          }
#pragma unroll
          for (int off = 16; off > 0; off >>= 1) smx = fmaxf(smx, __shfl_xor_sync(0xFFFFFFFFu, smx, off));
          if (lane == 0) sm.meta_smax[ms][pw] = smx;
          // rows 0..63 in slot sn, rows 64..127 in slot sn + 1; this warp loads column quarters
          // 2 pw and 2 pw + 1 of both
          for (int hs = 0; hs < 2; ++hs) {
            const int s2 = sn + hs, slot = s2 & 1;
            if (s2 >= 2 && !tc_wait_warp(&sm.raw_empty[slot], static_cast<uint32_t>(((s2 >> 1) - 1) & 1), abort)) {
              alive = false;
              break;
            }
            if (lane == 0) {
              const uint32_t st = raw0 + static_cast<uint32_t>(slot) * kStage;
              const int y = static_cast<int>(static_cast<int64_t>(qr.sb) * a.S + qr.slo + tbase + 64 * hs);
              mbar_arrive_expect_tx(&sm.raw_full[slot], 2 * kSwaQuarter);
#pragma unroll
              for (int qq = 2 * pw; qq < 2 * pw + 2; ++qq)
                tma_load_2d(smem + (st - base) + qq * kSwaQuarter, &tm_swa, &sm.raw_full[slot], 128 * qq, y);
            }
            ++fills[slot];
            __syncwarp();
          }
          if (!alive) break;
          sn += 2;
        }
        mbar_arrive(&sm.meta_full[ms]);
        if (!waited) {
          pdl_wait();
          pdl_launch_dependents();
          waited = true;
        }
      }
    }
    if (!alive) tc_give_up(abort, a.dev_err);
    if (!waited) {
      pdl_wait();
      pdl_launch_dependents();
    }
    // every copy issued must have landed before the CTA may exit
    if (lane == 0) {
      for (int s = 0; s < 2; ++s)
        if (fills[s] > 0 && !mbar_wait(&sm.raw_full[s], static_cast<uint32_t>((fills[s] - 1) & 1)))
          flag_error(a.dev_err, CSA2_DEVERR_TIMEOUT);
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------------------- QK^T issuer
    if (lane == 0) {
      int gt = 0, u = 0;
      bool alive = true;
      for (int j = 0; alive; ++j, ++u) {
        const int unit = static_cast<int>(blockIdx.x) + j * static_cast<int>(gridDim.x);
        if (unit >= units) break;
        const int split = unit % nsplit;
        const int tb = static_cast<int>(static_cast<int64_t>(split) * tiles / nsplit);
        const int te = static_cast<int>(static_cast<int64_t>(split + 1) * tiles / nsplit);
        if (!tc_wait(&sm.q_full, static_cast<uint32_t>(u & 1), abort)) {
          alive = false;
          break;
        }
        for (int tile = tb; tile < te && alive; ++tile, ++gt) {
          const int ss = gt & 1;
          if (gt >= 2 && !tc_wait(&sm.s_empty[ss], static_cast<uint32_t>(((gt >> 1) - 1) & 1), abort)) {
            alive = false;
            break;
          }
          const uint32_t d = tmem + kColS + 16u * ss;
          for (int h = 0; h < 2; ++h) {
            if (!tc_wait(&sm.va_full[h], static_cast<uint32_t>(gt & 1), abort)) {
              alive = false;
              break;
            }
            tcgen05_fence_after();
#pragma unroll
            for (int s = 0; s < 16; ++s) {
              const int ks = 2 * half_chunk(h, s >> 1) + (s & 1);  // 16 dims per K-step
              umma_f16_ts(d, tmem + kColVa + 8u * ks,
                          umma_desc_k128(q_smem + static_cast<uint32_t>((ks >> 2) * (HQ * 128) + (ks & 3) * 32)),
                          kIdescQK, (h | s) != 0 ? 1u : 0u);
            }
            umma_commit(&sm.va_empty[h]);
          }
          if (!alive) break;
          umma_commit(&sm.s_full[ss]);
        }
      }
      if (!alive) tc_give_up(abort, a.dev_err);
      umma_commit(&sm.drain);
    }
  } else if (warp == 2) {
    // --------------------------------------------------------------------------- P.V issuer
    if (lane == 0) {
      int gt = 0, u = 0;
      bool alive = true;
      for (int j = 0; alive; ++j, ++u) {
        const int unit = static_cast<int>(blockIdx.x) + j * static_cast<int>(gridDim.x);
        if (unit >= units) break;
        const int split = unit % nsplit;
        const int tb = static_cast<int>(static_cast<int64_t>(split) * tiles / nsplit);
        const int te = static_cast<int>(static_cast<int64_t>(split + 1) * tiles / nsplit);
        const int os = u & 1;
        if (u >= 2 && !tc_wait(&sm.o_empty[os], static_cast<uint32_t>(((u >> 1) - 1) & 1), abort)) {
          alive = false;
          break;
        }
        for (int tile = tb; tile < te && alive; ++tile, ++gt) {
          if (!tc_wait(&sm.p_full, static_cast<uint32_t>(gt & 1), abort)) {
            alive = false;
            break;
          }
          tcgen05_fence_after();
          for (int jb = 0; jb < 4; ++jb) {
            if (!tc_wait(&sm.vs_full[jb], static_cast<uint32_t>(gt & 1), abort)) {
              alive = false;
              break;
            }
            tcgen05_fence_after();
            const uint32_t d = tmem + kColO + 64u * os + 16u * jb;
#pragma unroll
            for (int s = 0; s < 8; ++s)
              umma_f16_ss(d,
                          umma_desc_mn128(vs + static_cast<uint32_t>(2 * jb * (kT * 128) + s * 2048),
                                          kT * 128, 1024),
                          umma_desc_k128(p_smem + static_cast<uint32_t>((s >> 2) * (HQ * 128) + (s & 3) * 32)),
                          kIdescPV, (tile != tb || s != 0) ? 1u : 0u);
            umma_commit(&sm.vs_empty[jb]);
          }
          if (!alive) break;
          umma_commit(&sm.p_empty);
          umma_commit(&sm.o_prog);
        }
        if (!alive) break;
        if (tb < te) umma_commit(&sm.o_full[os]);
        else mbar_arrive(&sm.o_full[os]);
      }
      if (!alive) tc_give_up(abort, a.dev_err);
      umma_commit(&sm.drain);
    }
  } else if (warp >= 4 && warp < 12) {
    // ------------------------------------------------------------------------- dequantisation
    const int q4 = warp & 3, h = (warp - 4) >> 2;
    const int i = 32 * q4 + lane;  // item of this thread
    const uint32_t t_lane = static_cast<uint32_t>(32 * q4) << 16;
    if (first_tile_by_dequant(units, nsplit, tiles, tiles_idx)) {
      // the CTA's first tile into raw slot 0: this warp's 32 items, 8 groups of 4; lanes 0..7 the
      // code half h, lanes 8..15 (h = 0 only) the scale rows
      if (!a.early_rows) pdl_wait();
      const int unit = static_cast<int>(blockIdx.x);
      const int b0 = unit / nsplit, split0 = unit - b0 * nsplit;
      const int tile0 = static_cast<int>(static_cast<int64_t>(split0) * tiles / nsplit);
      if (lane < (h == 0 ? 16 : 8)) {
        const QueryRows qr = query_rows(b0, a.N, a.n_cap, a.W, a.swa_len, a.qseq, a.swa_lo, a.S, a.nseq,
                                        a.dev_err, false);
        const int g = lane & 7;
        const int count = min(kT, a.K - tile0 * kT);
        int row[4];
#pragma unroll
        for (int k = 0; k < 4; ++k) {
          const int item = 32 * q4 + 4 * g + k;
          const int p = item < count ? __ldg(a.idx + static_cast<int64_t>(b0) * a.K + tile0 * kT + item) : -1;
          row[k] = static_cast<int>(qr.row0 + ((p >= 0 && p < qr.nb) ? p : 0));
        }
        const uint32_t grp = static_cast<uint32_t>(8 * q4 + g);
        if (lane < 8)
          tma_gather4(raw0 + static_cast<uint32_t>(h) * kCodeHalf + 512u * grp, &tm_codes, &sm.raw_full[0],
                      128 * h, row[0], row[1], row[2], row[3]);
        else
          tma_gather4(raw0 + kScalesAt + 128u * grp, &tm_scales, &sm.raw_full[0], 0, row[0], row[1], row[2],
                      row[3]);
      }
      __syncwarp();
    }
    int gt = 0, sn = 0;
    bool alive = true;
    for (int j = 0; alive; ++j) {
      const int unit = static_cast<int>(blockIdx.x) + j * static_cast<int>(gridDim.x);
      if (unit >= units) break;
      const int split = unit % nsplit;
      const int tb = static_cast<int>(static_cast<int64_t>(split) * tiles / nsplit);
      const int te = static_cast<int>(static_cast<int64_t>(split + 1) * tiles / nsplit);
      for (int tile = tb; tile < te; ++tile, ++gt) {
        const bool is_swa = tile >= tiles_idx;
        const int s2 = is_swa ? sn + (q4 >> 1) : sn;  // SWA: items 64.. sit in the second slot
        const int slot = s2 & 1;
        if (!tc_wait_warp(&sm.meta_full[gt % 3], static_cast<uint32_t>((gt / 3) & 1), abort) ||
            !tc_wait_warp(&sm.raw_full[slot], static_cast<uint32_t>((s2 >> 1) & 1), abort)) {
          alive = false;
          break;
        }
        const bool valid = sm.meta[gt % 3][i] >= 0.0f;
        if (gt > 0 && !tc_wait_warp(&sm.va_empty[h], static_cast<uint32_t>((gt - 1) & 1), abort)) {
          alive = false;
          break;
        }
        const uint32_t st = raw0 + static_cast<uint32_t>(slot) * kStage;
        uint4 sc4 = make_uint4(0u, 0u, 0u, 0u);
        if (!is_swa) {
          const uint2 s0 = lds8(st + static_cast<uint32_t>(kScalesAt + i * kScaleRow + 8 * h));
          const uint2 s1 = lds8(st + static_cast<uint32_t>(kScalesAt + i * kScaleRow + 16 + 8 * h));
          sc4 = make_uint4(s0.x, s0.y, s1.x, s1.y);
        }
        // pass A: V rows into tensor memory for QK^T
#pragma unroll 2
        for (int k = 0; k < 8; ++k) {
          uint32_t r[16];
          const int c = half_chunk(h, k);
          convert_chunk(st, is_swa, valid, i, c, k, sc4, r);
          tmem_st16(tmem + t_lane + kColVa + 16u * c, r);
        }
        tmem_wait_st();
        tcgen05_fence_before();
        __syncwarp();
        if (lane == 0) {
          mbar_arrive(&sm.va_full[h]);
          // the raw rows are no longer read
          if (is_swa) {
            mbar_arrive(&sm.raw_empty[sn & 1]);
            mbar_arrive(&sm.raw_empty[(sn + 1) & 1]);
          } else {
            mbar_arrive(&sm.raw_empty[slot]);
          }
        }
        // pass B: the same fp16 rows from tensor memory into the smem tile for P.V, one 128-dim
        // block at a time: blocks h and h + 2, so that both halves wait for one early and one late
        // block of the previous tile's P.V
        for (int jb = h; jb < 4; jb += 2) {
          if (gt > 0 && !tc_wait_warp(&sm.vs_empty[jb], static_cast<uint32_t>((gt - 1) & 1), abort)) {
            alive = false;
            break;
          }
#pragma unroll
          for (int k2 = 0; k2 < 4; k2 += 2) {
            const int c0 = 4 * jb + k2;  // two 32-dim chunks
            uint32_t r0[16], r1[16];
            tmem_ld16(tmem + t_lane + kColVa + 16u * c0, r0);
            tmem_ld16(tmem + t_lane + kColVa + 16u * (c0 + 1), r1);
            tmem_wait_ld();
            const uint32_t vb = vs + static_cast<uint32_t>((c0 >> 1) * (kT * 128));
#pragma unroll
            for (int uu = 0; uu < 4; ++uu)
              sts16(vb + swz(i, uu), r0[4 * uu], r0[4 * uu + 1], r0[4 * uu + 2], r0[4 * uu + 3]);
#pragma unroll
            for (int uu = 0; uu < 4; ++uu)
              sts16(vb + swz(i, 4 + uu), r1[4 * uu], r1[4 * uu + 1], r1[4 * uu + 2], r1[4 * uu + 3]);
          }
          fence_proxy_async_smem();
          tcgen05_fence_before();
          __syncwarp();
          if (lane == 0) mbar_arrive(&sm.vs_full[jb]);
        }
        if (!alive) break;
        sn += is_swa ? 2 : 1;
      }
    }
    if (!alive) tc_give_up(abort, a.dev_err);
  } else if (warp >= 12) {
    // ------------------------------------------------------------------- softmax + epilogue
    const int sq = warp & 3, st = tid - 384;
    const int i = 32 * sq + lane;  // item (S) or dim within a 128-dim block (O)
    const uint32_t t_lane = static_cast<uint32_t>(32 * sq) << 16;
    int gt = 0, u = 0;
    bool alive = true;
    float qun[HQ];
    // the first unit's q (an input that no kernel of the library writes) before the wait
    if (static_cast<int>(blockIdx.x) < units) {
      stage_q(a, static_cast<int>(blockIdx.x) / nsplit, st, q_smem, sm);
      fence_proxy_async_smem();
      softmax_sync();
#pragma unroll
      for (int hh = 0; hh < HQ; ++hh) qun[hh] = sm.q_unscale[hh];
      __syncwarp();
      if (lane == 0) mbar_arrive(&sm.q_full);
    }
    pdl_wait();
    pdl_launch_dependents();
    for (int j = 0; alive; ++j, ++u) {
      const int unit = static_cast<int>(blockIdx.x) + j * static_cast<int>(gridDim.x);
      if (unit >= units) break;
      const int b = unit / nsplit, split = unit - b * nsplit;
      const int tb = static_cast<int>(static_cast<int64_t>(split) * tiles / nsplit);
      const int te = static_cast<int>(static_cast<int64_t>(split + 1) * tiles / nsplit);
      float m_ref[HQ], l_part[HQ];
#pragma unroll
      for (int hh = 0; hh < HQ; ++hh) {
        m_ref[hh] = -INFINITY;
        l_part[hh] = 0.0f;
      }
      float pf_cur = 1.0f;
      {  // the next unit's q into L2 now: it is staged from there when this unit ends
        const int nxt = unit + static_cast<int>(gridDim.x);
        if (nxt < units) {
          const char* qn = reinterpret_cast<const char*>(a.q + static_cast<int64_t>(nxt / nsplit) * HQ * D);
          asm volatile("prefetch.global.L2 [%0];" ::"l"(qn + 128 * st) : "memory");
        }
      }
      for (int tile = tb; tile < te; ++tile, ++gt) {
        const bool is_swa = tile >= tiles_idx, first = tile == tb;
        const int ms = gt % 3, ss = gt & 1;
        bool ok = tc_wait(&sm.meta_full[ms], static_cast<uint32_t>((gt / 3) & 1), abort);
        ok = ok && tc_wait(&sm.s_full[ss], static_cast<uint32_t>((gt >> 1) & 1), abort);
        // the P tile is free once the previous tile's P.V has read it
        ok = ok && (gt == 0 || tc_wait(&sm.p_empty, static_cast<uint32_t>((gt - 1) & 1), abort));
        if (!softmax_all(ok)) {
          alive = false;
          break;
        }
        const float sc = sm.meta[ms][i];
        const float smax = fmaxf(sm.meta_smax[ms][0], sm.meta_smax[ms][1]);
        uint32_t r[16];
        tcgen05_fence_after();
        tmem_ld16(tmem + t_lane + kColS + 16u * ss, r);
        tmem_wait_ld();
        const bool valid = sc >= 0.0f;
        const float f = is_swa ? sc : 1.0f;
        float z[HQ];
        bool need = first;
#pragma unroll
        for (int hh = 0; hh < HQ; ++hh) {
          z[hh] = valid ? __uint_as_float(r[hh]) * qun[hh] * f : -INFINITY;
          need = need || z[hh] > m_ref[hh] + kRescaleGap;
        }
        // does any item move a reference maximum (first tile: always)
        need = softmax_any(need);
        tcgen05_fence_before();
        __syncwarp();
        if (lane == 0) {
          mbar_arrive(&sm.s_empty[ss]);
          mbar_arrive(&sm.meta_empty[ms]);
        }
        float am[HQ];
#pragma unroll
        for (int hh = 0; hh < HQ; ++hh) am[hh] = 1.0f;
        bool any = false;
        if (need) {
          // tile maxima per head over the 128 items
          float zc[HQ];
#pragma unroll
          for (int hh = 0; hh < HQ; ++hh) zc[hh] = z[hh];
          const float mh = warp_reduce16<true>(zc, lane);
          if ((lane & 1) == 0) sm.red[gt & 1][sq][reduce16_head(lane)] = mh;
          softmax_sync();
#pragma unroll
          for (int hh = 0; hh < HQ; ++hh) {
            const float tmax = fmaxf(fmaxf(sm.red[gt & 1][0][hh], sm.red[gt & 1][1][hh]),
                                     fmaxf(sm.red[gt & 1][2][hh], sm.red[gt & 1][3][hh]));
            float mn = m_ref[hh];
            if (first || tmax > m_ref[hh] + kRescaleGap) mn = tmax;
            am[hh] = (first || mn == m_ref[hh]) ? 1.0f : ex2f(m_ref[hh] - mn);
            if (!first && mn != m_ref[hh]) any = true;
            m_ref[hh] = mn;
            l_part[hh] *= am[hh];
          }
        }
        float fsc = 1.0f;
        if (is_swa && smax > 0.0f) {
          const float pf = pow2f_tc(-ilog2f_tc(smax));
          fsc = pf / pf_cur;  // exact: both powers of two
          pf_cur = pf;
        }
        if (!first && fsc != 1.0f) any = true;
        // O is rescaled only after the previous tile's P.V has completed
        if (any) {
          const bool ok2 = tc_wait(&sm.o_prog, static_cast<uint32_t>((gt - 1) & 1), abort);
          if (!softmax_all(ok2)) {
            alive = false;
            break;
          }
        }
        const float pmul = is_swa ? sc * pf_cur : 1.0f;
        {
          const uint32_t pb = p_smem + static_cast<uint32_t>((i >> 6) * (HQ * 128) + 2 * (i & 7));
#pragma unroll
          for (int hh = 0; hh < HQ; ++hh) {
            const float p = (valid && m_ref[hh] != -INFINITY) ? ex2f(z[hh] - m_ref[hh]) : 0.0f;
            l_part[hh] += p;
            sts_u16(pb + swz(hh, (i & 63) >> 3), __half_as_ushort(__float2half_rn(p * pmul)));
          }
        }
        if (any) {
          tcgen05_fence_after();
#pragma unroll 1
          for (int jb = 0; jb < 4; ++jb) {
            uint32_t o[16];
            const uint32_t ta = tmem + t_lane + kColO + 64u * (u & 1) + 16u * jb;
            tmem_ld16(ta, o);
            tmem_wait_ld();
#pragma unroll
            for (int hh = 0; hh < HQ; ++hh) o[hh] = __float_as_uint(__uint_as_float(o[hh]) * (am[hh] * fsc));
            tmem_st16(ta, o);
          }
          tmem_wait_st();
        }
        fence_proxy_async_smem();
        tcgen05_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(&sm.p_full);
      }
      if (!alive) break;
      // the next unit's q: this unit's QK^T has all completed (its last S was read), so the next
      // unit's QK^T may start while this unit's last P.V and epilogue run
      const int next = unit + static_cast<int>(gridDim.x);
      if (next < units) {
        stage_q(a, next / nsplit, st, q_smem, sm);
        fence_proxy_async_smem();
      }
      // ---- epilogue: O / l (or the unnormalised partial), lse (or m, l)
      {
        float lc[HQ];
#pragma unroll
        for (int hh = 0; hh < HQ; ++hh) lc[hh] = l_part[hh];
        const float lh = warp_reduce16<false>(lc, lane);
        if ((lane & 1) == 0) sm.lred[sq][reduce16_head(lane)] = lh;
      }
      softmax_sync();  // the next q and the l partial sums are complete
      if (next < units) {
#pragma unroll
        for (int hh = 0; hh < HQ; ++hh) qun[hh] = sm.q_unscale[hh];
        __syncwarp();
        if (lane == 0) mbar_arrive(&sm.q_full);
      }
      const bool single = nsplit == 1;
      const int64_t pidx = static_cast<int64_t>(b) * nsplit + split;
      // one head per thread (st < 16): the scale of O and lse (or m, l), while the last P.V drains
      if (st < HQ) {
        const float l = (sm.lred[0][st] + sm.lred[1][st]) + (sm.lred[2][st] + sm.lred[3][st]);
        float m = -INFINITY;
#pragma unroll
        for (int hh = 0; hh < HQ; ++hh)
          if (hh == st) m = m_ref[hh];
        sm.scout[st] = single ? (l > 0.0f ? 1.0f / (l * pf_cur) : 0.0f) : 1.0f / pf_cur;
        if (single) {
          if (a.lse != nullptr) a.lse[static_cast<int64_t>(b) * HQ + st] = l > 0.0f ? m * kLn2 + logf(l) : -INFINITY;
        } else {
          a.part_ml[(pidx * HQ + st) * 2] = m == -INFINITY ? -INFINITY : m * kLn2;
          a.part_ml[(pidx * HQ + st) * 2 + 1] = l;
        }
      }
      softmax_sync();  // the scales are complete
      const bool ok = tc_wait(&sm.o_full[u & 1], static_cast<uint32_t>((u >> 1) & 1), abort);
      if (!softmax_all(ok)) {
        alive = false;
        break;
      }
      tcgen05_fence_after();
      float sc_out[HQ];
#pragma unroll
      for (int hh = 0; hh < HQ; ++hh) sc_out[hh] = sm.scout[hh];
#pragma unroll 1
      for (int jb = 0; jb < 4; ++jb) {
        uint32_t o[16];
        if (tb < te) {
          tmem_ld16(tmem + t_lane + kColO + 64u * (u & 1) + 16u * jb, o);
          tmem_wait_ld();
        } else {
#pragma unroll
          for (int hh = 0; hh < HQ; ++hh) o[hh] = 0u;
        }
        const int dim = 128 * jb + i;
        float* dst = single ? a.out + static_cast<int64_t>(b) * HQ * D : a.part_o + pidx * HQ * D;
#pragma unroll
        for (int hh = 0; hh < HQ; ++hh) dst[hh * D + dim] = __uint_as_float(o[hh]) * sc_out[hh];
      }
      tcgen05_fence_before();
      softmax_sync();  // every thread has read lred, the scales and O before they are reused
      if (lane == 0) mbar_arrive(&sm.o_empty[u & 1]);
    }
    if (!alive) tc_give_up(abort, a.dev_err);
  }

  // ---- teardown: every MMA has completed before the tensor memory is released
  tcgen05_fence_before();
  __syncthreads();
  if (warp == 1) {
    if (lane == 0 && !mbar_wait(&sm.drain, 0u)) flag_error(a.dev_err, CSA2_DEVERR_TIMEOUT);
    __syncwarp();
    tcgen05_fence_after();
    tmem_dealloc(tmem, kTmemCols);
  }
}

}  // namespace

bool attend_tc_selected(int B, int K, int W) {
  const int tiles = (K + kT - 1) / kT + (W + kT - 1) / kT;
  return tiles > 0 && B >= kTcMinBatch;
}

int attend_tc_split_count(int B, int K, int W) {
  const int tiles = (K + kT - 1) / kT + (W + kT - 1) / kT;
  const int sms = device_sm_count();
  int splits = sms / B;  // units fill at most one wave of one CTA per SM
  if (splits > tiles) splits = tiles;
  if (splits > kAttendMaxSplits) splits = kAttendMaxSplits;
  if (splits < 1) splits = 1;
  return splits;
}

// Tensor maps of the gathered operands: MXFP4 code rows (two 128-byte halves, 128-byte swizzle),
// scale rows (32 bytes, no swizzle), SWA rows (128-byte quarters x 64 rows, 128-byte swizzle).
// False when the rows do not fit int32 coordinates, a pointer is not 16-byte aligned or the
// driver refuses a map: the caller then runs the mma.sync kernel.
static bool encode_maps(const uint8_t* codes, const uint8_t* scales, const uint8_t* swa, int64_t rows,
                        int64_t swa_rows, CUtensorMap* mc, CUtensorMap* msc, CUtensorMap* msw) {
  const TensorMapEncodeFn enc = tensor_map_encoder();
  if (enc == nullptr) return false;
  if (rows <= 0 || rows > INT32_MAX || swa_rows > INT32_MAX) return false;
  if ((reinterpret_cast<uintptr_t>(codes) & 15u) || (reinterpret_cast<uintptr_t>(scales) & 15u) ||
      (reinterpret_cast<uintptr_t>(swa) & 15u))
    return false;
  const cuuint32_t estr[2] = {1, 1};
  {
    const cuuint64_t dims[2] = {static_cast<cuuint64_t>(kCodeRow), static_cast<cuuint64_t>(rows)};
    const cuuint64_t strides[1] = {static_cast<cuuint64_t>(kCodeRow)};
    const cuuint32_t box[2] = {128, 1};
    if (enc(mc, CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, const_cast<uint8_t*>(codes), dims, strides, box, estr,
            CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
            CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
      return false;
  }
  {
    const cuuint64_t dims[2] = {static_cast<cuuint64_t>(kScaleRow), static_cast<cuuint64_t>(rows)};
    const cuuint64_t strides[1] = {static_cast<cuuint64_t>(kScaleRow)};
    const cuuint32_t box[2] = {static_cast<cuuint32_t>(kScaleRow), 1};
    if (enc(msc, CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, const_cast<uint8_t*>(scales), dims, strides, box, estr,
            CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE, CU_TENSOR_MAP_L2_PROMOTION_L2_128B,
            CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
      return false;
  }
  if (swa != nullptr && swa_rows > 0) {
    const cuuint64_t dims[2] = {static_cast<cuuint64_t>(D), static_cast<cuuint64_t>(swa_rows)};
    const cuuint64_t strides[1] = {static_cast<cuuint64_t>(D)};
    const cuuint32_t box[2] = {128, 64};
    if (enc(msw, CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, const_cast<uint8_t*>(swa), dims, strides, box, estr,
            CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
            CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
      return false;
  } else {
    *msw = *mc;  // not read: no SWA tiles
  }
  return true;
}

cudaError_t launch_attend_tc(const void* q, float softmax_scale, const uint8_t* codes,
                             const uint8_t* scales, int n_cap, const int32_t* N, const int32_t* idx,
                             int K, const uint8_t* swa, const float* swa_scale,
                             const int32_t* swa_len, int W, const int32_t* qseq,
                             const int32_t* swa_lo, int S, int nseq, int B, float* out, float* lse,
                             void* ws, int32_t* dev_err, bool early_rows, cudaStream_t s) {
  CUtensorMap mc, msc, msw;
  if (!encode_maps(codes, scales, W > 0 ? swa : nullptr, static_cast<int64_t>(nseq) * n_cap,
                   W > 0 ? static_cast<int64_t>(nseq) * S : 0, &mc, &msc, &msw))
    return cudaErrorNotSupported;
  const int splits = attend_tc_split_count(B, K, W);
  TcArgs a;
  a.q = static_cast<const uint16_t*>(q);
  a.softmax_scale = softmax_scale;
  a.codes = codes;
  a.scales = scales;
  a.n_cap = n_cap;
  a.N = N;
  a.idx = idx;
  a.K = K;
  a.swa = swa;
  a.swa_scale = swa_scale;
  a.swa_len = swa_len;
  a.W = W;
  a.qseq = qseq;
  a.swa_lo = swa_lo;
  a.S = S;
  a.nseq = nseq;
  a.B = B;
  a.nsplit = splits;
  a.out = out;
  a.lse = lse;
  a.part_o = nullptr;
  a.part_ml = nullptr;
  if (splits > 1) {
    a.part_o = static_cast<float*>(ws);
    a.part_ml = a.part_o + static_cast<size_t>(B) * splits * HQ * D;
  }
  a.dev_err = dev_err;
  a.early_rows = early_rows ? 1 : 0;

  static std::mutex mu;
  static std::vector<char> configured;
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  {
    std::lock_guard<std::mutex> lock(mu);
    if (dev >= static_cast<int>(configured.size())) configured.resize(dev + 1, 0);
    if (!configured[dev]) {
      e = cudaFuncSetAttribute(attend_tc_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                               static_cast<int>(kTcSmem));
      if (e != cudaSuccess) return e;
      configured[dev] = 1;
    }
  }
  const int units = B * splits;
  const int grid = std::min(units, device_sm_count());
  profile_begin(CSA2_KERNEL_ATTEND, s);
  e = launch_pdl(attend_tc_kernel, dim3(grid), dim3(kTcThreads), kTcSmem, s, mc, msc, msw, a);
  count_launches(1);
  if (e == cudaSuccess) e = cudaGetLastError();
  if (e == cudaSuccess && splits > 1) e = launch_attend_merge(a.part_o, a.part_ml, splits, B, out, lse, s);
  profile_end(CSA2_KERNEL_ATTEND, s);
  return e;
}

size_t attend_tc_workspace_bytes(int B, int K, int W) {
  const int splits = attend_tc_split_count(B, K, W);
  if (splits == 1) return 0;
  return static_cast<size_t>(B) * splits * HQ * (D + 2) * sizeof(float);
}

}  // namespace csa2

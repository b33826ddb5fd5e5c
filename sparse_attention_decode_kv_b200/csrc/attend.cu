// attend.cu -- sparse attention of one decode query per sequence (16 heads x 512) over the
// selected MXFP4 main-KV entries and the FP8 SWA rows, merged into one softmax.
//
// Method: "DeepSeek V4.1 Flash 拆解" (austincafe.tech), section 一: a Reuse-mode layer reuses the
// indices and runs sparse attention directly; the main KV is MXFP4, the SWA KV stays FP8.
// Reading: K = V = the dequantised entry; z = softmax_scale * q . v over the selected entries and
// the valid SWA slots together; out = sum softmax(z) v; lse = log sum exp(z).
//
// Queries: in a decode step query b belongs to cache sequence b and its SWA rows are slots
// 0 .. swa_len[b]-1 of sequence b's ring. The multi-query form (prefill or verification of
// several tokens per sequence) maps query b to cache sequence qseq[b] and to rows swa_lo[b] ..
// swa_lo[b] + swa_len[b] - 1 of that sequence's FP8 SWA buffer of S rows; b below always names
// the query.
//
// Work split: the K index slots and the W SWA slots are cut into tiles of 64 items (index tiles
// and SWA tiles never mix); grid = (B, splits) and each CTA runs an online softmax over a
// contiguous run of tiles. With one split the CTA writes the result; otherwise it writes an
// unnormalised partial (m, l, o) and attend_merge_kernel combines the partials by log-sum-exp.
//
// Per tile: 16 threads per item gather 16-byte pieces (coalesced 256 B of codes + 32 B of scales
// per MXFP4 entry, 512 B per SWA row), dequantise in registers with the sm_100a e2m1x2/e4m3x2 ->
// f16x2 converts, and store an fp16 tile [64 x 512] in swizzled shared memory. Every dequantised
// MXFP4 value (<= 6 significant bits, magnitude in [2^-10, 2688]) and every E4M3 element is exact
// in fp16. QK^T and PV run on the tensor cores (m16n8k16, heads on M = 16, fp32 accumulate).
// q is scaled per head by a power of two into fp16's range (exact for bf16 inputs). The SWA
// per-token fp32 scale multiplies the logit and the probability instead of the value, so the
// value operand stays exact; P is rescaled per SWA tile by a power of two to stay in fp16's
// normal range.
#include <math.h>

#include "common.cuh"
#include "internal.h"

namespace csa2 {

namespace {

constexpr int kTile = 64;
constexpr int kWarps = 8;
constexpr int kThreads = kWarps * 32;
constexpr int kTargetCtas = 296;  // 148 SMs x 2 resident CTAs
constexpr int kRawRow = D / 2 + D / 16;  // 288 bytes: codes then scales of one MXFP4 entry
constexpr int kZs = kTile + 8;  // partial-logit row stride: the float2 stores of 16 lanes hit 16 bank pairs

struct __align__(16) AttendSmem {
  uint16_t q[HQ * D];        // fp16 [16][512], 16-byte chunks XOR-swizzled by (row & 7)
  uint16_t v[kTile * D];     // fp16 [64][512], same swizzle
  uint8_t raw[kTile * kRawRow];  // the next MXFP4 tile's rows, fetched during this tile;
                                 // 16-byte aligned (offset 81920) for the 16-byte copies
  uint16_t p[HQ * kTile];    // fp16 [16][64], same swizzle (8 chunks per row)
  float zp[2][HQ * kZs];     // partial logits of the current tile over dims 0..255 / 256..511
  float item_scale[kTile];   // 1 (MXFP4) or the SWA token's fp32 scale
  int item_valid[kTile];
  float q_unscale[HQ];       // 2^(e_h - 14) * softmax_scale
  float m_run[HQ], l_run[HQ], alpha[HQ];
  float tile_pf;             // power of two applied to P on SWA tiles
};

// 16-byte asynchronous copy global -> shared; src_bytes 0 fills the 16 bytes with zeros.
__device__ __forceinline__ void cp_async16(void* dst, const void* src, uint32_t src_bytes) {
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;" ::"r"(smem_u32(dst)), "l"(src),
               "r"(src_bytes)
               : "memory");
}
__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }
__device__ __forceinline__ void cp_async_wait_all() { asm volatile("cp.async.wait_group 0;" ::: "memory"); }

// Row of 64 16-byte chunks. The low three chunk bits are XORed with the row's low bits (the 8 rows
// of an ldmatrix read at one chunk fall in 8 distinct bank groups) and with the chunk's own bits
// 3..5 (the chunks 4r + k, r = 0..7, that 8 threads store at once also fall in 8 distinct groups).
// Four bytes of E2M1 pairs -> four half2 (byte j -> o[j], low nibble in .x). The byte unpack
// leaves the choice of byte operands to the compiler instead of a shift and mask per byte.
__device__ __forceinline__ void e2m1x8_to_h2x4(uint32_t w, uint32_t (&o)[4]) {
  asm("{\n\t.reg .b8 b0, b1, b2, b3;\n\tmov.b32 {b0, b1, b2, b3}, %4;\n\t"
      "cvt.rn.f16x2.e2m1x2 %0, b0;\n\tcvt.rn.f16x2.e2m1x2 %1, b1;\n\t"
      "cvt.rn.f16x2.e2m1x2 %2, b2;\n\tcvt.rn.f16x2.e2m1x2 %3, b3;\n\t}"
      : "=r"(o[0]), "=r"(o[1]), "=r"(o[2]), "=r"(o[3])
      : "r"(w));
}

// Four E4M3 bytes -> two half2 (bytes 0, 1 -> o[0]; bytes 2, 3 -> o[1]). Exact.
__device__ __forceinline__ void e4m3x4_to_h2x2(uint32_t w, uint32_t (&o)[2]) {
  asm("{\n\t.reg .b16 h0, h1;\n\tmov.b32 {h0, h1}, %2;\n\t"
      "cvt.rn.f16x2.e4m3x2 %0, h0;\n\tcvt.rn.f16x2.e4m3x2 %1, h1;\n\t}"
      : "=r"(o[0]), "=r"(o[1])
      : "r"(w));
}

__device__ __forceinline__ uint32_t swz1024(int row, int chunk) {
  return static_cast<uint32_t>(row * 1024 + ((chunk ^ (row & 7) ^ ((chunk >> 3) & 7)) << 4));
}
__device__ __forceinline__ uint32_t swz128(int row, int chunk) {  // 8 chunks per row
  return static_cast<uint32_t>(row * 128 + ((chunk ^ (row & 7)) << 4));
}

// 2^k as a float for k in [-126, 127].
__device__ __forceinline__ float pow2f(int k) {
  k = max(-126, min(127, k));
  return __uint_as_float(static_cast<uint32_t>(k + 127) << 23);
}

// floor(log2(x)) for finite x > 0 (subnormals clamp to -126).
__device__ __forceinline__ int ilog2f(float x) {
  const int e = static_cast<int>((__float_as_uint(x) >> 23) & 0xFF);
  return e == 0 ? -126 : e - 127;
}

__global__ void __launch_bounds__(kThreads, 2)
    attend_kernel(const uint16_t* __restrict__ q, float softmax_scale,
                  const uint8_t* __restrict__ codes, const uint8_t* __restrict__ scales,
                  int n_cap, const int32_t* __restrict__ N, const int32_t* __restrict__ idx, int K,
                  const uint8_t* __restrict__ swa, const float* __restrict__ swa_scale,
                  const int32_t* __restrict__ swa_len, int W, const int32_t* __restrict__ qseq,
                  const int32_t* __restrict__ swa_lo, int S, int nseq, float* __restrict__ out,
                  float* __restrict__ lse, float* __restrict__ part_o,
                  float* __restrict__ part_ml, int32_t* dev_err, int early_rows) {
  extern __shared__ __align__(1024) unsigned char smem_raw[];
  AttendSmem& sm = *reinterpret_cast<AttendSmem*>(smem_raw);
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int g = lane >> 2, c = lane & 3;
  const int b = blockIdx.x, split = blockIdx.y, nsplit = gridDim.y;  // b on x: up to 2^31 - 1
  // ---- q -> fp16 with a per-head power-of-two scale (16 threads per head, 32 dims each). No
  // kernel of this library writes q, so this runs before the wait on the preceding kernel and
  // overlaps its tail.
  {
    const int h = tid >> 4, r = tid & 15;
    const uint4* src = reinterpret_cast<const uint4*>(q + (static_cast<int64_t>(b) * HQ + h) * D) +
                       4 * r;
    uint4 u[4];
#pragma unroll
    for (int k = 0; k < 4; ++k) u[k] = __ldg(src + k);
    float amax = 0.0f;
#pragma unroll
    for (int k = 0; k < 4; ++k) {
      const uint32_t w4[4] = {u[k].x, u[k].y, u[k].z, u[k].w};
#pragma unroll
      for (int e = 0; e < 4; ++e)
        amax = fmaxf(amax, fmaxf(fabsf(bf16lo(w4[e])), fabsf(bf16hi(w4[e]))));
    }
#pragma unroll
    for (int off = 8; off > 0; off >>= 1) amax = fmaxf(amax, __shfl_xor_sync(0xFFFFFFFFu, amax, off));
    const int eh = amax > 0.0f ? ilog2f(amax) : 0;
    const float up = pow2f(14 - eh);
    if (r == 0) {
      sm.q_unscale[h] = pow2f(eh - 14) * softmax_scale;
      sm.m_run[h] = -INFINITY;
      sm.l_run[h] = 0.0f;
    }
#pragma unroll
    for (int k = 0; k < 4; ++k) {
      const uint32_t w4[4] = {u[k].x, u[k].y, u[k].z, u[k].w};
      uint32_t h2[4];
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        __half2 hv = __floats2half2_rn(bf16lo(w4[e]) * up, bf16hi(w4[e]) * up);
        h2[e] = *reinterpret_cast<uint32_t*>(&hv);
      }
      *reinterpret_cast<uint4*>(reinterpret_cast<unsigned char*>(sm.q) + swz1024(h, 4 * r + k)) =
          make_uint4(h2[0], h2[1], h2[2], h2[3]);
    }
  }

  const int tiles_idx = (K + kTile - 1) / kTile;
  const int tiles_swa = (W + kTile - 1) / kTile;
  const int tiles = tiles_idx + tiles_swa;
  const int t_begin = static_cast<int>(static_cast<int64_t>(split) * tiles / nsplit);
  const int t_end = static_cast<int>(static_cast<int64_t>(split + 1) * tiles / nsplit);

  // qseq, N, swa_len and swa_lo, like q, are inputs no kernel of this library writes: they are
  // read before the wait too
  int sb = qseq ? __ldg(qseq + b) : b;  // cache sequence of query b
  const bool sb_ok = sb >= 0 && sb < nseq;
  if (!sb_ok) {  // an unknown sequence: the query attends to nothing
    if (tid == 0) flag_error(dev_err, CSA2_DEVERR_INDEX_RANGE);
    sb = 0;
  }
  int nb = sb_ok ? __ldg(N + sb) : 0;
  if (nb < 0 || nb > n_cap) {
    if (tid == 0) flag_error(dev_err, CSA2_DEVERR_NLEN);
    nb = max(0, min(nb, n_cap));
  }
  int sl = 0;
  if (W > 0) {
    sl = (swa_len && sb_ok) ? __ldg(swa_len + b) : 0;
    if (sl < 0 || sl > W) {
      if (tid == 0) flag_error(dev_err, CSA2_DEVERR_NLEN);
      sl = max(0, min(sl, W));
    }
  }
  // first SWA row of this query in its sequence's buffer of S rows (the ring: 0, S = W)
  int slo = 0;
  if (swa_lo != nullptr && sl > 0) {
    slo = __ldg(swa_lo + b);
    if (slo < 0 || slo + sl > S) {
      if (tid == 0) flag_error(dev_err, CSA2_DEVERR_NLEN);
      slo = max(0, min(slo, S));
      sl = min(sl, S - slo);
    }
  }

  const int64_t seq_row0 = static_cast<int64_t>(sb) * n_cap;
  const bool first_mx = t_begin < t_end && t_begin < tiles_idx;

  // Software pipeline over MXFP4 tiles: while a tile is computed, the next one's rows stream
  // into sm.raw with cp.async (its indices were requested when the tile began), so only the
  // first tile of a CTA and the SWA tiles wait for their gather.
  int pos_staged[4] = {-1, -1, -1, -1};  // positions of the tile held in sm.raw
  bool staged = false;
  // Reuse mode: the indices and the rows they name come from an earlier layer, so the first
  // tile's gather starts before the wait on the preceding kernel (L2-only loads and copies).
  if (early_rows && first_mx) {
    const int r = tid & 15;
#pragma unroll
    for (int pass = 0; pass < 4; ++pass) {
      const int item = pass * 16 + (tid >> 4);
      pos_staged[pass] = item < min(kTile, K - t_begin * kTile)
                             ? __ldcg(idx + static_cast<int64_t>(b) * K + t_begin * kTile + item)
                             : -1;
    }
#pragma unroll
    for (int pass = 0; pass < 4; ++pass) {
      const int item = pass * 16 + (tid >> 4);
      const bool valid = pos_staged[pass] >= 0 && pos_staged[pass] < nb;
      const int64_t row = seq_row0 + (valid ? pos_staged[pass] : 0);
      uint8_t* rr = sm.raw + item * kRawRow;
      cp_async16(rr + 16 * r, codes + row * (D / 2) + 16 * r, valid ? 16u : 0u);
      if (r < 2) cp_async16(rr + D / 2 + 16 * r, scales + row * (D / 16) + 16 * r, valid ? 16u : 0u);
    }
    cp_async_commit();
    staged = true;
  }

  pdl_wait();
  pdl_launch_dependents();

  // the first tile's indices otherwise (possibly written by the preceding kernel)
  int pos_first[4] = {-1, -1, -1, -1};
  if (first_mx && !staged) {
#pragma unroll
    for (int pass = 0; pass < 4; ++pass) {
      const int item = pass * 16 + (tid >> 4);
      if (item < min(kTile, K - t_begin * kTile))
        pos_first[pass] = __ldg(idx + static_cast<int64_t>(b) * K + t_begin * kTile + item);
    }
  }

  float o[8][4];
#pragma unroll
  for (int j = 0; j < 8; ++j) o[j][0] = o[j][1] = o[j][2] = o[j][3] = 0.0f;

  const uint32_t q_base = smem_u32(sm.q), v_base = smem_u32(sm.v), p_base = smem_u32(sm.p);
  if (staged) {  // the early rows have landed (16 threads share an entry's scales)
    cp_async_wait_all();
    __syncthreads();
  }
  for (int tile = t_begin; tile < t_end; ++tile) {
    const bool is_swa = tile >= tiles_idx;
    const int base = is_swa ? (tile - tiles_idx) * kTile : tile * kTile;
    const int count = min(kTile, (is_swa ? W : K) - base);
    const bool next_mx = tile + 1 < t_end && tile + 1 < tiles_idx;
    int pos_next[4] = {-1, -1, -1, -1};
    if (next_mx) {
#pragma unroll
      for (int pass = 0; pass < 4; ++pass) {
        const int item = pass * 16 + (tid >> 4);
        if (item < min(kTile, K - (base + kTile)))
          pos_next[pass] = __ldg(idx + static_cast<int64_t>(b) * K + base + kTile + item);
      }
    }

    // ---- gather + dequantise: 16 threads per item, 32 channels per thread, 4 passes of 16 items.
    // All index loads, then all row loads, then the conversions: two memory round trips.
    {
      const int r = tid & 15;
      // item = 16 pass + tid / 16 has the row bits of tid / 16, so each pass's store address is
      // the pass's 16 KiB row block plus one of four per-thread offsets
      unsigned char* vrow = reinterpret_cast<unsigned char*>(sm.v);
      if (!is_swa) {
        uint32_t off[4];
#pragma unroll
        for (int k = 0; k < 4; ++k) off[k] = swz1024(tid >> 4, 4 * r + k);
        int pos[4];
#pragma unroll
        for (int pass = 0; pass < 4; ++pass) {
          const int item = pass * 16 + (tid >> 4);
          pos[pass] = staged ? pos_staged[pass]
                      : tile == t_begin ? pos_first[pass]
                      : (item < count ? __ldg(idx + static_cast<int64_t>(b) * K + base + item) : -1);
        }
        uint4 cw[4];
        uint32_t sw[4];
#pragma unroll
        for (int pass = 0; pass < 4; ++pass) {
          const int item = pass * 16 + (tid >> 4);
          const bool valid = pos[pass] >= 0 && pos[pass] < nb;
          if (!valid && pos[pass] != -1) flag_error(dev_err, CSA2_DEVERR_INDEX_RANGE);
          const int64_t row = seq_row0 + (valid ? pos[pass] : 0);
          if (staged) {  // fetched during the previous tile (zeros where the position is invalid)
            const uint8_t* rr = sm.raw + item * kRawRow;
            cw[pass] = *reinterpret_cast<const uint4*>(rr + 16 * r);
            sw[pass] = *reinterpret_cast<const uint16_t*>(rr + D / 2 + 2 * r);
          } else {
            cw[pass] = valid ? ldg_nc_v4(codes + row * (D / 2) + 16 * r) : make_uint4(0u, 0u, 0u, 0u);
            sw[pass] = valid ? __ldg(reinterpret_cast<const uint16_t*>(scales + row * (D / 16)) + r) : 0u;
          }
        }
#pragma unroll
        for (int pass = 0; pass < 4; ++pass) {
          const int item = pass * 16 + (tid >> 4);
          const bool valid = pos[pass] >= 0 && pos[pass] < nb;
          const uint32_t s01 = e4m3x2_to_h2(sw[pass]);  // .x: channels 32r..+15, .y: the next 16
          const uint32_t slo = __byte_perm(s01, 0, 0x1010), shi = __byte_perm(s01, 0, 0x3232);
          const uint32_t cws[4] = {cw[pass].x, cw[pass].y, cw[pass].z, cw[pass].w};
#pragma unroll
          for (int k = 0; k < 4; ++k) {  // word k: channels 32r + 8k .. + 7
            uint32_t hv[4];
            e2m1x8_to_h2x4(cws[k], hv);
            const uint32_t sk = k < 2 ? slo : shi;
            *reinterpret_cast<uint4*>(vrow + pass * (16 * 1024) + off[k]) =
                make_uint4(h2_mul(hv[0], sk), h2_mul(hv[1], sk), h2_mul(hv[2], sk), h2_mul(hv[3], sk));
          }
          if (r == 0) {
            sm.item_valid[item] = valid;
            sm.item_scale[item] = 1.0f;
          }
        }
      } else {
        uint32_t off[4];
#pragma unroll
        for (int k = 0; k < 4; ++k)  // chunks 2r, 2r + 1, 32 + 2r, 33 + 2r
          off[k] = swz1024(tid >> 4, 2 * r + (k & 1) + 32 * (k >> 1));
        uint4 e[4][2];
        float iscale[4];
#pragma unroll
        for (int pass = 0; pass < 4; ++pass) {
          const int item = pass * 16 + (tid >> 4);
          const int slot = base + item;
          const bool valid = item < count && slot < sl;
          const int64_t srow = static_cast<int64_t>(sb) * S + slo + (valid ? slot : 0);
          // thread r takes channels 16r .. 16r + 15 and 256 + 16r .. + 15: each load of the 16
          // threads of an item is 256 contiguous bytes
          const uint8_t* rowp = swa + srow * D + 16 * r;
          e[pass][0] = valid ? ldg_nc_v4(rowp) : make_uint4(0u, 0u, 0u, 0u);
          e[pass][1] = valid ? ldg_nc_v4(rowp + D / 2) : make_uint4(0u, 0u, 0u, 0u);
          iscale[pass] = valid ? __ldg(swa_scale + srow) : 1.0f;
        }
#pragma unroll
        for (int pass = 0; pass < 4; ++pass) {
          const int item = pass * 16 + (tid >> 4);
          const bool valid = item < count && base + item < sl;
          const uint32_t ew[8] = {e[pass][0].x, e[pass][0].y, e[pass][0].z, e[pass][0].w,
                                  e[pass][1].x, e[pass][1].y, e[pass][1].z, e[pass][1].w};
#pragma unroll
          for (int k = 0; k < 4; ++k) {
            uint32_t h0[2], h1[2];
            e4m3x4_to_h2x2(ew[2 * k], h0);
            e4m3x4_to_h2x2(ew[2 * k + 1], h1);
            *reinterpret_cast<uint4*>(vrow + pass * (16 * 1024) + off[k]) =
                make_uint4(h0[0], h0[1], h1[0], h1[1]);
          }
          if (r == 0) {
            sm.item_valid[item] = valid;
            sm.item_scale[item] = iscale[pass];
          }
        }
      }
    }
    __syncthreads();
    // every read of sm.raw for this tile is done: request the next MXFP4 tile's rows
    if (next_mx) {
      const int r = tid & 15;
#pragma unroll
      for (int pass = 0; pass < 4; ++pass) {
        const int item = pass * 16 + (tid >> 4);
        const bool valid = pos_next[pass] >= 0 && pos_next[pass] < nb;
        const int64_t row = seq_row0 + (valid ? pos_next[pass] : 0);
        uint8_t* rr = sm.raw + item * kRawRow;
        cp_async16(rr + 16 * r, codes + row * (D / 2) + 16 * r, valid ? 16u : 0u);
        if (r < 2) cp_async16(rr + D / 2 + 16 * r, scales + row * (D / 16) + 16 * r, valid ? 16u : 0u);
        pos_staged[pass] = pos_next[pass];
      }
      cp_async_commit();
    }
    staged = next_mx;
    if (warp == 0) {
      // P scale for SWA tiles: brings the largest token scale to [1, 2)
      float smax = 0.0f;
      if (is_swa) {
        smax = fmaxf(sm.item_valid[lane] ? sm.item_scale[lane] : 0.0f,
                     sm.item_valid[lane + 32] ? sm.item_scale[lane + 32] : 0.0f);
#pragma unroll
        for (int off = 16; off > 0; off >>= 1) smax = fmaxf(smax, __shfl_xor_sync(0xFFFFFFFFu, smax, off));
      }
      if (lane == 0) sm.tile_pf = smax > 0.0f ? pow2f(-ilog2f(smax)) : 1.0f;
    }

    // ---- logits: warp w takes items 16 (w % 4) .. +15 (two n-blocks, two independent
    // accumulator chains) over dims 256 (w / 4) .. +255, so each warp reads half of q; the two
    // halves are added in the softmax
    {
      float acc0[4] = {0.0f, 0.0f, 0.0f, 0.0f}, acc1[4] = {0.0f, 0.0f, 0.0f, 0.0f};
      const int ig = warp & 3, kh = warp >> 2;
      const int mi = lane >> 3;
      const int a_row = (lane & 7) + ((mi & 1) << 3);
      const int v_row = 16 * ig + (lane & 7) + ((lane >> 4) << 3);
      const int v_sub = mi & 1;
#pragma unroll 4
      for (int s = 16 * kh; s < 16 * kh + 16; ++s) {
        uint32_t a0, a1, a2, a3, b0, b1, b2, b3;
        ldsm_x4(q_base + swz1024(a_row, 2 * s + (mi >> 1)), a0, a1, a2, a3);
        ldsm_x4(v_base + swz1024(v_row, 2 * s + v_sub), b0, b1, b2, b3);
        mma_f16_16816(acc0, a0, a1, a2, a3, b0, b1);
        mma_f16_16816(acc1, a0, a1, a2, a3, b2, b3);
      }
      float* zp = sm.zp[kh];
      const int i0 = 16 * ig + 2 * c;
      *reinterpret_cast<float2*>(zp + g * kZs + i0) = make_float2(acc0[0], acc0[1]);
      *reinterpret_cast<float2*>(zp + (g + 8) * kZs + i0) = make_float2(acc0[2], acc0[3]);
      *reinterpret_cast<float2*>(zp + g * kZs + i0 + 8) = make_float2(acc1[0], acc1[1]);
      *reinterpret_cast<float2*>(zp + (g + 8) * kZs + i0 + 8) = make_float2(acc1[2], acc1[3]);
    }
    __syncthreads();

    // ---- online softmax: warp w updates heads 2w and 2w+1
    {
      const float pf = sm.tile_pf;
#pragma unroll
      for (int hh = 0; hh < 2; ++hh) {
        const int h = 2 * warp + hh;
        const float uh = sm.q_unscale[h];
        const float z0 = sm.item_valid[lane]
                             ? (sm.zp[0][h * kZs + lane] + sm.zp[1][h * kZs + lane]) * uh * sm.item_scale[lane]
                             : -INFINITY;
        const float z1 = sm.item_valid[lane + 32]
                             ? (sm.zp[0][h * kZs + lane + 32] + sm.zp[1][h * kZs + lane + 32]) * uh *
                                   sm.item_scale[lane + 32]
                             : -INFINITY;
        float mt = fmaxf(z0, z1);
#pragma unroll
        for (int off = 16; off > 0; off >>= 1) mt = fmaxf(mt, __shfl_xor_sync(0xFFFFFFFFu, mt, off));
        const float m_old = sm.m_run[h];
        const float m_new = fmaxf(m_old, mt);
        float p0 = 0.0f, p1 = 0.0f, alpha = 1.0f;
        if (m_new != -INFINITY) {
          p0 = __expf(z0 - m_new);
          p1 = __expf(z1 - m_new);
          alpha = __expf(m_old - m_new);
        }
        float ps = p0 + p1;
#pragma unroll
        for (int off = 16; off > 0; off >>= 1) ps += __shfl_xor_sync(0xFFFFFFFFu, ps, off);
        const float w0 = p0 * sm.item_scale[lane] * pf, w1 = p1 * sm.item_scale[lane + 32] * pf;
        unsigned char* prow = reinterpret_cast<unsigned char*>(sm.p);
        *reinterpret_cast<__half*>(prow + swz128(h, lane >> 3) + 2 * (lane & 7)) = __float2half_rn(w0);
        *reinterpret_cast<__half*>(prow + swz128(h, 4 + (lane >> 3)) + 2 * (lane & 7)) =
            __float2half_rn(w1);
        if (lane == 0) {
          sm.l_run[h] = sm.l_run[h] * alpha + ps;
          sm.m_run[h] = m_new;
          sm.alpha[h] = alpha;
        }
      }
    }
    __syncthreads();

    // ---- o[16 heads][64w .. 64w+64) = alpha * o + P V  (pf undone after the MMAs)
    {
      const float pf = sm.tile_pf;
      const float f0 = sm.alpha[g] * pf, f1 = sm.alpha[g + 8] * pf;
#pragma unroll
      for (int j = 0; j < 8; ++j) {
        o[j][0] *= f0;
        o[j][1] *= f0;
        o[j][2] *= f1;
        o[j][3] *= f1;
      }
      const int mi = lane >> 3;
      const int a_row = (lane & 7) + ((mi & 1) << 3);
#pragma unroll
      for (int s = 0; s < kTile / 16; ++s) {
        uint32_t a0, a1, a2, a3;
        ldsm_x4(p_base + swz128(a_row, 2 * s + (mi >> 1)), a0, a1, a2, a3);
        const int v_row = 16 * s + (lane & 7) + ((mi & 1) << 3);
#pragma unroll
        for (int j = 0; j < 8; j += 2) {
          uint32_t b0, b1, b2, b3;
          ldsm_x4_trans(v_base + swz1024(v_row, 8 * warp + j + (mi >> 1)), b0, b1, b2, b3);
          mma_f16_16816(o[j], a0, a1, a2, a3, b0, b1);
          mma_f16_16816(o[j + 1], a0, a1, a2, a3, b2, b3);
        }
      }
      if (pf != 1.0f) {
        const float inv = 1.0f / pf;  // exact: pf is a power of two
#pragma unroll
        for (int j = 0; j < 8; ++j) {
          o[j][0] *= inv;
          o[j][1] *= inv;
          o[j][2] *= inv;
          o[j][3] *= inv;
        }
      }
    }
    if (staged) cp_async_wait_all();  // the next tile's rows have landed (made visible below)
    __syncthreads();
  }

  // ---- epilogue: thread holds heads g and g+8, dims 64w + 8j + 2c (+1)
  const float l0 = sm.l_run[g], l1 = sm.l_run[g + 8];
  if (nsplit == 1) {
    const float r0 = l0 > 0.0f ? 1.0f / l0 : 0.0f, r1 = l1 > 0.0f ? 1.0f / l1 : 0.0f;
    float* o0 = out + (static_cast<int64_t>(b) * HQ + g) * D + 64 * warp + 2 * c;
    float* o1 = out + (static_cast<int64_t>(b) * HQ + g + 8) * D + 64 * warp + 2 * c;
#pragma unroll
    for (int j = 0; j < 8; ++j) {
      *reinterpret_cast<float2*>(o0 + 8 * j) = make_float2(o[j][0] * r0, o[j][1] * r0);
      *reinterpret_cast<float2*>(o1 + 8 * j) = make_float2(o[j][2] * r1, o[j][3] * r1);
    }
    if (lse != nullptr && tid < HQ) {
      const float l = sm.l_run[tid];
      lse[static_cast<int64_t>(b) * HQ + tid] = l > 0.0f ? sm.m_run[tid] + logf(l) : -INFINITY;
    }
  } else {
    const int64_t pidx = static_cast<int64_t>(b) * nsplit + split;
    float* o0 = part_o + (pidx * HQ + g) * D + 64 * warp + 2 * c;
    float* o1 = part_o + (pidx * HQ + g + 8) * D + 64 * warp + 2 * c;
#pragma unroll
    for (int j = 0; j < 8; ++j) {
      *reinterpret_cast<float2*>(o0 + 8 * j) = make_float2(o[j][0], o[j][1]);
      *reinterpret_cast<float2*>(o1 + 8 * j) = make_float2(o[j][2], o[j][3]);
    }
    if (tid < HQ) {
      part_ml[(pidx * HQ + tid) * 2] = sm.m_run[tid];
      part_ml[(pidx * HQ + tid) * 2 + 1] = sm.l_run[tid];
    }
  }
}

// Log-sum-exp merge of the split partials: grid = (16 heads, B), 128 threads x 4 dims. Every
// thread requests the partial (m, l) it owns and its float4 of every split's partial o at once
// (one memory round trip), then the weights exp(m_s - m) / l are formed in shared memory.
constexpr int kMaxSplits = kAttendMaxSplits;
constexpr int kMergeBatch = 16;  // partial-o requests in flight per thread
__global__ void __launch_bounds__(128)
    attend_merge_kernel(const float* __restrict__ part_o, const float* __restrict__ part_ml,
                        int nsplit, float* __restrict__ out, float* __restrict__ lse) {
  __shared__ float wgt[kMaxSplits];
  __shared__ float red[8];
  const int h = blockIdx.x, b = blockIdx.y, t = threadIdx.x, lane = t & 31, warp = t >> 5;
  pdl_wait();
  pdl_launch_dependents();
  const int64_t p0 = static_cast<int64_t>(b) * nsplit;
  float ms = -INFINITY, ls = 0.0f;
  if (t < nsplit) {
    const float2 ml = __ldg(reinterpret_cast<const float2*>(part_ml) + (p0 + t) * HQ + h);
    ms = ml.x;
    ls = ml.y;
  }
  const float4* src = reinterpret_cast<const float4*>(part_o + (p0 * HQ + h) * D) + t;
  const int64_t stride = static_cast<int64_t>(HQ) * D / 4;  // float4 between splits
  float4 v[kMergeBatch];
#pragma unroll
  for (int j = 0; j < kMergeBatch; ++j)
    v[j] = j < nsplit ? __ldg(src + j * stride) : make_float4(0.f, 0.f, 0.f, 0.f);
  // m = max over splits, l = sum exp(m_s - m) l_s (nsplit <= 128 = blockDim)
  float m = ms;
#pragma unroll
  for (int off = 16; off > 0; off >>= 1) m = fmaxf(m, __shfl_xor_sync(0xFFFFFFFFu, m, off));
  if (lane == 0) red[warp] = m;
  __syncthreads();
  m = fmaxf(fmaxf(red[0], red[1]), fmaxf(red[2], red[3]));
  const float f = (t < nsplit && ms != -INFINITY) ? __expf(ms - m) : 0.0f;
  float fl = f * ls;
#pragma unroll
  for (int off = 16; off > 0; off >>= 1) fl += __shfl_xor_sync(0xFFFFFFFFu, fl, off);
  if (lane == 0) red[4 + warp] = fl;
  if (t < nsplit) wgt[t] = f;
  __syncthreads();
  const float l = (red[4] + red[5]) + (red[6] + red[7]);
  float4 acc = make_float4(0.0f, 0.0f, 0.0f, 0.0f);
#pragma unroll
  for (int j = 0; j < kMergeBatch; ++j) {
    const float fj = j < nsplit ? wgt[j] : 0.0f;
    acc.x += fj * v[j].x;
    acc.y += fj * v[j].y;
    acc.z += fj * v[j].z;
    acc.w += fj * v[j].w;
  }
  for (int s0 = kMergeBatch; s0 < nsplit; s0 += kMergeBatch) {  // more splits than one batch
#pragma unroll
    for (int j = 0; j < kMergeBatch; ++j)
      v[j] = s0 + j < nsplit ? __ldg(src + (s0 + j) * stride) : make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll
    for (int j = 0; j < kMergeBatch; ++j) {
      const float fj = s0 + j < nsplit ? wgt[s0 + j] : 0.0f;
      acc.x += fj * v[j].x;
      acc.y += fj * v[j].y;
      acc.z += fj * v[j].z;
      acc.w += fj * v[j].w;
    }
  }
  const float rl = l > 0.0f ? 1.0f / l : 0.0f;
  reinterpret_cast<float4*>(out + (static_cast<int64_t>(b) * HQ + h) * D)[t] =
      make_float4(acc.x * rl, acc.y * rl, acc.z * rl, acc.w * rl);
  if (lse != nullptr && t == 0)
    lse[static_cast<int64_t>(b) * HQ + h] = l > 0.0f ? m + logf(l) : -INFINITY;
}

}  // namespace

int attend_split_count(int B, int K, int W) {
  const int tiles = (K + kTile - 1) / kTile + (W + kTile - 1) / kTile;
  // at most one wave of two CTAs per SM: from 148 queries up every CTA takes whole queries and
  // no partial outputs are written or merged
  int splits = kTargetCtas / B;
  if (splits > tiles) splits = tiles;
  if (splits > kMaxSplits) splits = kMaxSplits;
  if (splits < 1) splits = 1;
  return splits;
}

// Enough for either kernel: the tensor-core kernel falls back to this one when its operands cannot
// be described by TMA tensor maps.
size_t attend_workspace_bytes(int B, int K, int W) {
  const int splits = attend_split_count(B, K, W);
  const size_t own = splits == 1 ? 0 : static_cast<size_t>(B) * splits * HQ * (D + 2) * sizeof(float);
  if (!attend_tc_selected(B, K, W)) return own;
  const size_t tc = attend_tc_workspace_bytes(B, K, W);
  return tc > own ? tc : own;
}

cudaError_t launch_attend(const void* q, float softmax_scale, const uint8_t* codes,
                          const uint8_t* scales, int n_cap, const int32_t* N, const int32_t* idx,
                          int K, const uint8_t* swa, const float* swa_scale,
                          const int32_t* swa_len, int W, const int32_t* qseq,
                          const int32_t* swa_lo, int S, int nseq, int B, float* out, float* lse,
                          void* ws, int32_t* dev_err, bool early_rows, cudaStream_t s) {
  if (attend_tc_selected(B, K, W)) {
    const cudaError_t e = launch_attend_tc(q, softmax_scale, codes, scales, n_cap, N, idx, K, swa,
                                           swa_scale, swa_len, W, qseq, swa_lo, S, nseq, B, out, lse,
                                           ws, dev_err, early_rows, s);
    if (e != cudaErrorNotSupported) return e;  // else: operands TMA cannot describe
  }
  const int splits = attend_split_count(B, K, W);
  float* part_o = nullptr;
  float* part_ml = nullptr;
  if (splits > 1) {
    part_o = static_cast<float*>(ws);
    part_ml = part_o + static_cast<size_t>(B) * splits * HQ * D;
  }
  const size_t smem = sizeof(AttendSmem);
  static thread_local int configured_device = -1;
  int dev = 0;
  cudaGetDevice(&dev);
  if (configured_device != dev) {
    cudaError_t e = cudaFuncSetAttribute(attend_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         static_cast<int>(smem));
    if (e != cudaSuccess) return e;
    configured_device = dev;
  }
  profile_begin(CSA2_KERNEL_ATTEND, s);
  cudaError_t e = launch_pdl(attend_kernel, dim3(B, splits), dim3(kThreads), smem, s,
                             static_cast<const uint16_t*>(q), softmax_scale, codes, scales, n_cap,
                             N, idx, K, swa, swa_scale, swa_len, W, qseq, swa_lo, S, nseq, out,
                             lse, part_o, part_ml,
                             dev_err, early_rows ? 1 : 0);
  count_launches(1);
  if (e == cudaSuccess) e = cudaGetLastError();
  if (e == cudaSuccess && splits > 1) {
    e = launch_pdl(attend_merge_kernel, dim3(HQ, B), dim3(128), 0, s,
                   static_cast<const float*>(part_o), static_cast<const float*>(part_ml), splits,
                   out, lse);
    count_launches(1);
    if (e == cudaSuccess) e = cudaGetLastError();
  }
  profile_end(CSA2_KERNEL_ATTEND, s);
  return e;
}

cudaError_t launch_attend_merge(const float* part_o, const float* part_ml, int nsplit, int B,
                                float* out, float* lse, cudaStream_t s) {
  cudaError_t e = launch_pdl(attend_merge_kernel, dim3(HQ, B), dim3(128), 0, s, part_o, part_ml,
                             nsplit, out, lse);
  count_launches(1);
  if (e == cudaSuccess) e = cudaGetLastError();
  return e;
}

}  // namespace csa2

// append.cu -- quantize-on-append: MXFP4 main-KV entries, the FP8 SWA ring and the indexer-key
// copy, in one launch with one warp per new entry.
//
// Method: "DeepSeek V4.1 Flash 拆解" (austincafe.tech), section 一, FP4 KV Cache paragraph: the main
// KV is MXFP4 (E2M1 values, one E4M3 scale per 16 channels); the SWA KV is kept in FP8.
// Readings: scale = E4M3 RNE-saturating of the fp32 quotient amax/6; code = E2M1 RNE-saturating of
// the fp32 quotient x/scale with the sign of x; zero scale -> zero codes. SWA: per-token fp32
// scale amax/448, element = E4M3 RNE-saturating of the fp32 quotient x/scale.
//
// Lane l of the warp owns channels 16l..16l+15, i.e. exactly one MXFP4 group: it reads 32 bytes
// of bf16, writes 8 bytes of codes and 1 scale byte; the warp's traffic is one coalesced 1 KiB
// read, one 256-byte and one 32-byte write per entry (plus 512 + 4 bytes for SWA rows). The grid
// is one resident wave; each warp walks entries at the grid's stride and requests the next entry's
// row before it quantises the current one.
//
// Exactness of the element codes without a per-element division: x/scale is either exactly an
// E2M1 rounding midpoint or at least ~2^-11 away from every midpoint (x has 8 significant bits,
// the scale 4, a midpoint 3, so x - m*scale is a multiple of a power of two that bounds the
// gap). |x| * RN(1/scale) differs from x/scale by at most ~4e-7 in this range, and snapping that
// product to the 2^-14 grid (fma with 512, subtract 512: exact) restores every midpoint exactly
// while moving no other value across one. The hardware RNE conversion of the snapped magnitude
// is then the E2M1 RNE of x/scale.
#include <algorithm>
#include <mutex>
#include <vector>

#include "common.cuh"
#include "internal.h"
#include "swa_codec.cuh"

namespace csa2 {

namespace {

constexpr int kAppendWarps = 8;

// Codes of one 16-channel group; returns 8 bytes (channel 2j in the low nibble of byte j).
__device__ __forceinline__ uint2 mxfp4_group(const float* v, uint32_t& scale_byte) {
  float amax = 0.0f;
#pragma unroll
  for (int i = 0; i < 16; ++i) amax = fmaxf(amax, fabsf(v[i]));
  const float q = __fdiv_rn(amax, 6.0f);
  scale_byte = cvt_e4m3x2(q, 0.0f) & 0xFFu;
  const float s = e4m3_to_f32(scale_byte);
  uint32_t w[2] = {0u, 0u};
  if (s > 0.0f) {
    const float rs = __frcp_rn(s);
#pragma unroll
    for (int j = 0; j < 8; ++j) {
      // snapped magnitudes of channels 2j and 2j+1
      const float a0 = __fsub_rn(__fmaf_rn(fabsf(v[2 * j]), rs, 512.0f), 512.0f);
      const float a1 = __fsub_rn(__fmaf_rn(fabsf(v[2 * j + 1]), rs, 512.0f), 512.0f);
      uint32_t byte = cvt_e2m1x2(a0, a1);  // magnitudes: sign bits are 0
      byte |= (__float_as_uint(v[2 * j]) >> 31) << 3;
      byte |= (__float_as_uint(v[2 * j + 1]) >> 31) << 7;
      w[j >> 2] |= byte << (8 * (j & 3));
    }
  }
  return make_uint2(w[0], w[1]);
}

__global__ void __launch_bounds__(kAppendWarps * 32)
    append_kernel(const uint16_t* __restrict__ x, const uint16_t* __restrict__ ik, int B, int n,
                  const int32_t* __restrict__ pos, int n_cap, uint8_t* __restrict__ codes,
                  uint8_t* __restrict__ scales, uint16_t* __restrict__ ik_cache,
                  uint8_t* __restrict__ swa, float* __restrict__ swa_scale, int W,
                  int32_t* dev_err) {
  pdl_wait();
  pdl_launch_dependents();
  const int lane = threadIdx.x & 31;
  const int64_t total = static_cast<int64_t>(B) * n;
  const int64_t stride = static_cast<int64_t>(gridDim.x) * kAppendWarps;
  int64_t entry = static_cast<int64_t>(blockIdx.x) * kAppendWarps + (threadIdx.x >> 5);
  // the warp's entries entry, entry + stride, ...; the next entry's 16 bf16 channels of this
  // lane's group are requested before the current one is quantised
  uint4 u0 = make_uint4(0u, 0u, 0u, 0u), u1 = u0;
  if (entry < total) {
    const uint4* src = reinterpret_cast<const uint4*>(x + entry * D) + 2 * lane;
    u0 = ldg_nc_v4(src);
    u1 = ldg_nc_v4(src + 1);
  }
  for (; entry < total; entry += stride) {
    const uint32_t uw[8] = {u0.x, u0.y, u0.z, u0.w, u1.x, u1.y, u1.z, u1.w};
    const int64_t next = entry + stride;
    if (next < total) {
      const uint4* src = reinterpret_cast<const uint4*>(x + next * D) + 2 * lane;
      u0 = ldg_nc_v4(src);
      u1 = ldg_nc_v4(src + 1);
    }
    const int b = static_cast<int>(entry / n);
    const int i = static_cast<int>(entry - static_cast<int64_t>(b) * n);
    const int64_t p = static_cast<int64_t>(__ldg(pos + b)) + i;
    if (p < 0 || p >= n_cap) {
      if (lane == 0) flag_error(dev_err, CSA2_DEVERR_POS_RANGE);
      continue;
    }
    const int64_t row = static_cast<int64_t>(b) * n_cap + p;
    float v[16];
#pragma unroll
    for (int k = 0; k < 8; ++k) {
      v[2 * k] = bf16lo(uw[k]);
      v[2 * k + 1] = bf16hi(uw[k]);
    }

    uint32_t sb;
    const uint2 c = mxfp4_group(v, sb);
    reinterpret_cast<uint2*>(codes + row * (D / 2))[lane] = c;
    scales[row * (D / 16) + lane] = static_cast<uint8_t>(sb);

    if (ik != nullptr && lane < DI * 2 / 16) {
      const uint4 kv = ldg_nc_v4(reinterpret_cast<const uint4*>(ik + entry * DI) + lane);
      reinterpret_cast<uint4*>(ik_cache + row * DI)[lane] = kv;
    }

    // SWA ring: only the last W of the n new tokens survive, so only they are written (no two
    // writers of one slot within a call).
    if (swa != nullptr && W > 0 && i >= n - W) {
      uint32_t e[4];
      const float s = swa_quantize_row_lane(v, e);
      const int64_t slot = static_cast<int64_t>(b) * W + (p % W);
      reinterpret_cast<uint4*>(swa + slot * D)[lane] = make_uint4(e[0], e[1], e[2], e[3]);
      if (lane == 0) swa_scale[slot] = s;
    }
  }
}

}  // namespace

cudaError_t launch_append(const void* x, const void* ik, int B, int n, const int32_t* pos,
                          int n_cap, uint8_t* codes, uint8_t* scales, void* ik_cache,
                          uint8_t* swa, float* swa_scale, int W, int32_t* dev_err,
                          cudaStream_t s) {
  const int64_t entries = static_cast<int64_t>(B) * n;
  // one resident wave loops over the entries (a decode step's handful of entries takes that many
  // warps only)
  static std::mutex mu;
  static std::vector<int> per_sm;
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  int resident = 0;
  {
    std::lock_guard<std::mutex> lock(mu);
    if (dev >= static_cast<int>(per_sm.size())) per_sm.resize(dev + 1, 0);
    if (per_sm[dev] == 0) {
      e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm[dev], append_kernel,
                                                        kAppendWarps * 32, 0);
      if (e != cudaSuccess) return e;
      if (per_sm[dev] < 1) per_sm[dev] = 1;
    }
    resident = per_sm[dev];
  }
  const int64_t blocks = std::min<int64_t>((entries + kAppendWarps - 1) / kAppendWarps,
                                           static_cast<int64_t>(device_sm_count()) * resident);
  profile_begin(CSA2_KERNEL_APPEND, s);
  e = launch_pdl(append_kernel, dim3(static_cast<unsigned>(blocks)),
                             dim3(kAppendWarps * 32), 0, s, static_cast<const uint16_t*>(x),
                             static_cast<const uint16_t*>(ik), B, n, pos, n_cap, codes, scales,
                             static_cast<uint16_t*>(ik_cache), swa, swa_scale, W, dev_err);
  profile_end(CSA2_KERNEL_APPEND, s);
  count_launches(1);
  return e != cudaSuccess ? e : cudaGetLastError();
}

}  // namespace csa2

// ced.cu -- CED KV projection with the MXFP4 quantisation fused into the GEMM epilogue.
//
// Method: "DeepSeek V4.1 Flash 拆解" (austincafe.tech), section 一, CED paragraph: the decoder
// layers' global KV is projected from the hidden state of the middle layer, C_l = H_{L/2} W^KV_l,
// and (FP4 KV cache paragraph) stored as MXFP4: E2M1 codes with one E4M3 scale per 16 channels.
// Reading: C = H W^T with H bf16 [tokens, d] and W bf16 [512, d] (one row per latent channel),
// fp32 accumulation; each 16-channel group of a row of C is quantised like an appended entry:
// scale = E4M3 RNE-saturating of the fp32 quotient amax/6, code = E2M1 RNE-saturating of the fp32
// quotient x/scale with the sign of x, all codes 0 for a zero scale. Token i of sequence b goes to
// cache row pos[b] + i.
//
// ced_quant_kernel: persistent, one CTA per SM; CTA c takes tiles c, c + G, ... of 128 tokens x
// 256 channels, tile t covering tokens 128 (t / 2) .. and channels 256 (t % 2) .., so the two
// channel halves of a token tile run at the same time on neighbouring CTAs and the second reads
// its slice of H from L2.
//   warp 0, one thread  TMA producer: 64-wide d-slices of H (128 x 64) and W (256 x 64) with
//                       128-byte swizzle into a 4-stage ring of mbarrier-tracked buffers that runs
//                       on across tiles.
//   warp 1, one thread  MMA issuer: tcgen05.mma kind::f16 (bf16 x bf16 -> fp32, M 128, N 256,
//                       K 16 per instruction) into one of two 128-lane x 256-column TMEM
//                       accumulators (all 512 columns); tcgen05.commit frees each stage and
//                       hands a finished accumulator to the epilogue. The same warp allocates and
//                       frees the tensor memory.
//   warps 2..5          epilogue: each thread owns one token row (its TMEM lane), reads 16
//                       columns at a time with tcgen05.ld, quantises the group and writes 8 code
//                       bytes and 1 scale byte into the row's cache slot, then returns the
//                       accumulator; meanwhile the MMAs of the next tile fill the other one.
// Every mbarrier wait is bounded; a timeout flags CSA2_DEVERR_TIMEOUT, the producer drains its
// own bulk copies, the MMA issuer still commits, and the tensor memory is always freed.
#include <algorithm>
#include <mutex>
#include <vector>

#include "common.cuh"
#include "internal.h"
#include "tcgen05.cuh"

namespace csa2 {

namespace {

constexpr int kCedM = 128;         // tokens per tile = TMEM lanes
constexpr int kCedN = 256;         // channels per tile = fp32 TMEM columns per accumulator
constexpr int kCedK = 64;          // d per stage: one 128-byte swizzle row of bf16
constexpr int kCedStages = 4;
constexpr int kCedThreads = 192;   // warp 0 TMA, warp 1 MMA + TMEM, warps 2..5 epilogue
constexpr int kCedEpiWarps = 4;
constexpr int kCedATile = kCedM * kCedK * 2;  // 16 KiB
constexpr int kCedBTile = kCedN * kCedK * 2;  // 32 KiB
constexpr int kCedTmemCols = 2 * kCedN;       // two accumulators: the whole tensor memory
constexpr uint32_t kCedIdesc = umma_idesc_bf16_f32(kCedM, kCedN);

static_assert(kCedN * (D / kCedN) == D, "two channel tiles cover the 512 latent channels");

struct __align__(1024) CedSmem {
  uint8_t a[kCedStages][kCedATile];  // 1024-byte aligned (swizzle atoms)
  uint8_t b[kCedStages][kCedBTile];
  uint64_t full[kCedStages];
  uint64_t empty[kCedStages];
  uint64_t acc_full[2];   // MMA -> epilogue: accumulator ready
  uint64_t acc_empty[2];  // epilogue -> MMA: accumulator read out (one arrive per warp)
  uint64_t drain;         // used once, before the tensor memory is freed
  uint32_t tmem_base;
  int abort;
};

static_assert(sizeof(CedSmem) <= 227 * 1024, "ced_quant_kernel shared memory");

__device__ __forceinline__ bool bounded_wait(uint64_t* bar, uint32_t parity, volatile int* abort) {
  if (mbar_try_wait(bar, parity)) return true;
  const uint64_t t0 = globaltimer_ns();
  while (!mbar_try_wait(bar, parity)) {
    if (abort != nullptr && *abort) return false;
    if (globaltimer_ns() - t0 > kWaitLimitNs) return false;
  }
  return true;
}

// MXFP4 codes and scale of 16 fp32 channels (the quotients are correctly rounded fp32 divisions,
// then converted with the hardware's round-to-nearest-even, saturating E4M3 / E2M1 converts).
__device__ __forceinline__ uint2 quantize_group_f32(const float* v, uint32_t& scale_byte) {
  float amax = 0.0f;
#pragma unroll
  for (int i = 0; i < 16; ++i) amax = fmaxf(amax, fabsf(v[i]));
  scale_byte = cvt_e4m3x2(__fdiv_rn(amax, 6.0f), 0.0f) & 0xFFu;
  const float s = e4m3_to_f32(scale_byte);
  uint32_t w[2] = {0u, 0u};
  if (s > 0.0f) {
#pragma unroll
    for (int j = 0; j < 8; ++j) {
      uint32_t byte = cvt_e2m1x2(__fdiv_rn(fabsf(v[2 * j]), s), __fdiv_rn(fabsf(v[2 * j + 1]), s));
      byte |= (__float_as_uint(v[2 * j]) >> 31) << 3;
      byte |= (__float_as_uint(v[2 * j + 1]) >> 31) << 7;
      w[j >> 2] |= byte << (8 * (j & 3));
    }
  }
  return make_uint2(w[0], w[1]);
}

__global__ void __launch_bounds__(kCedThreads, 1)
    ced_quant_kernel(const __grid_constant__ CUtensorMap tm_h, const __grid_constant__ CUtensorMap tm_w,
                     int M, int n, int d, const int32_t* __restrict__ pos, int n_cap,
                     uint8_t* __restrict__ codes, uint8_t* __restrict__ scales, int32_t* dev_err) {
  extern __shared__ __align__(1024) unsigned char smem_raw[];
  CedSmem& sm = *reinterpret_cast<CedSmem*>(smem_raw);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int nk = d / kCedK;
  const int tiles = ((M + kCedM - 1) / kCedM) * (D / kCedN);
  const int my_tiles = tiles > static_cast<int>(blockIdx.x)
                           ? (tiles - 1 - static_cast<int>(blockIdx.x)) / static_cast<int>(gridDim.x) + 1
                           : 0;

  if (threadIdx.x == 0) {
    for (int s = 0; s < kCedStages; ++s) {
      mbar_init(&sm.full[s], 1);
      mbar_init(&sm.empty[s], 1);
    }
    for (int a = 0; a < 2; ++a) {
      mbar_init(&sm.acc_full[a], 1);
      mbar_init(&sm.acc_empty[a], kCedEpiWarps);
    }
    mbar_init(&sm.drain, 1);
    sm.abort = 0;
    fence_barrier_init();
  }
  if (warp == 1) {
    tmem_alloc(&sm.tmem_base, kCedTmemCols);
    tmem_relinquish();
  }
  tcgen05_fence_before();
  __syncthreads();
  tcgen05_fence_after();
  const uint32_t tmem = sm.tmem_base;
  volatile int* abort = &sm.abort;
  pdl_wait();  // H, W and pos may be written by the preceding kernel

  if (warp == 0) {
    // ------------------------------------------------------------------------ TMA producer
    if (lane == 0) {
      int it = 0;  // stage uses so far (the ring runs on across tiles)
      for (int j = 0; j < my_tiles && !*abort; ++j) {
        const int t = static_cast<int>(blockIdx.x) + j * static_cast<int>(gridDim.x);
        const int m0 = (t >> 1) * kCedM, n0 = (t & 1) * kCedN;
        for (int kc = 0; kc < nk; ++kc, ++it) {
          const int s = it % kCedStages;
          if (it >= kCedStages &&
              !bounded_wait(&sm.empty[s], static_cast<uint32_t>(((it / kCedStages) & 1) ^ 1), abort)) {
            if (!*abort) flag_error(dev_err, CSA2_DEVERR_TIMEOUT);
            *abort = 1;
            break;
          }
          mbar_arrive_expect_tx(&sm.full[s], kCedATile + kCedBTile);
          tma_load_2d(sm.a[s], &tm_h, &sm.full[s], kc * kCedK, m0);
          tma_load_2d(sm.b[s], &tm_w, &sm.full[s], kc * kCedK, n0);
        }
      }
      // drain: every issued copy must land before the CTA may exit
      for (int q = max(0, it - kCedStages); q < it; ++q)
        if (!mbar_wait(&sm.full[q % kCedStages], static_cast<uint32_t>((q / kCedStages) & 1)))
          flag_error(dev_err, CSA2_DEVERR_TIMEOUT);
    }
  } else if (warp == 1) {
    // -------------------------------------------------------------------------- MMA issuer
    if (lane == 0) {
      int it = 0;
      for (int j = 0; j < my_tiles && !*abort; ++j) {
        const int acc = j & 1;
        if (j >= 2 &&
            !bounded_wait(&sm.acc_empty[acc], static_cast<uint32_t>(((j >> 1) & 1) ^ 1), abort)) {
          if (!*abort) flag_error(dev_err, CSA2_DEVERR_TIMEOUT);
          *abort = 1;
          break;
        }
        tcgen05_fence_after();
        const uint32_t d_tmem = tmem + static_cast<uint32_t>(acc * kCedN);
        bool ok = true;
        for (int kc = 0; kc < nk; ++kc, ++it) {
          const int s = it % kCedStages;
          if (!bounded_wait(&sm.full[s], static_cast<uint32_t>((it / kCedStages) & 1), abort)) {
            if (!*abort) flag_error(dev_err, CSA2_DEVERR_TIMEOUT);
            *abort = 1;
            ok = false;
            break;
          }
          tcgen05_fence_after();
          const uint32_t a0 = smem_u32(sm.a[s]), b0 = smem_u32(sm.b[s]);
#pragma unroll
          for (int k4 = 0; k4 < kCedK / 16; ++k4)  // 16 bf16 = 32 bytes per instruction
            umma_bf16(d_tmem, umma_desc_k128(a0 + 32 * k4), umma_desc_k128(b0 + 32 * k4), kCedIdesc,
                      (kc | k4) != 0 ? 1u : 0u);
          umma_commit(&sm.empty[s]);  // the stage is free once these MMAs have read it
        }
        umma_commit(&sm.acc_full[acc]);  // every MMA issued so far has completed
        if (!ok) break;
      }
    }
  } else {
    // ---------------------------------------------------------------------------- epilogue
    const int quarter = warp & 3;  // this warp may read TMEM lanes 32 q .. 32 q + 31
    for (int j = 0; j < my_tiles; ++j) {
      const int acc = j & 1;
      const int t = static_cast<int>(blockIdx.x) + j * static_cast<int>(gridDim.x);
      const int m0 = (t >> 1) * kCedM, n0 = (t & 1) * kCedN;
      const bool ok = __all_sync(0xFFFFFFFFu,
                                 bounded_wait(&sm.acc_full[acc], static_cast<uint32_t>((j >> 1) & 1), abort));
      if (!ok) {  // the MMA issuer gave up (and has flagged it) or the wait ran out
        if (lane == 0 && !*abort) flag_error(dev_err, CSA2_DEVERR_TIMEOUT);
        break;
      }
      tcgen05_fence_after();
      const int row = m0 + 32 * quarter + lane;
      int64_t dst = -1;
      if (row < M) {
        const int b = row / n, i = row - (row / n) * n;
        const int64_t p = static_cast<int64_t>(__ldg(pos + b)) + i;
        if (p >= 0 && p < n_cap) dst = static_cast<int64_t>(b) * n_cap + p;
        else if (n0 == 0) flag_error(dev_err, CSA2_DEVERR_POS_RANGE);
      }
      const uint32_t tbase =
          tmem + static_cast<uint32_t>(acc * kCedN) + (static_cast<uint32_t>(32 * quarter) << 16);
      uint32_t sc[16];
#pragma unroll 1
      for (int g = 0; g < kCedN / 16; ++g) {
        uint32_t r[16];
        tmem_ld16(tbase + static_cast<uint32_t>(16 * g), r);
        tmem_wait_ld();
        float v[16];
#pragma unroll
        for (int i = 0; i < 16; ++i) v[i] = __uint_as_float(r[i]);
        uint32_t sb;
        const uint2 cw = quantize_group_f32(v, sb);
        sc[g] = sb;
        if (dst >= 0)
          *reinterpret_cast<uint2*>(codes + dst * (D / 2) + n0 / 2 + 8 * g) = cw;
      }
      // the accumulator is read out: hand it back to the MMA issuer
      tcgen05_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&sm.acc_empty[acc]);
      if (dst >= 0) {
        uint4 packed;
        packed.x = sc[0] | (sc[1] << 8) | (sc[2] << 16) | (sc[3] << 24);
        packed.y = sc[4] | (sc[5] << 8) | (sc[6] << 16) | (sc[7] << 24);
        packed.z = sc[8] | (sc[9] << 8) | (sc[10] << 16) | (sc[11] << 24);
        packed.w = sc[12] | (sc[13] << 8) | (sc[14] << 16) | (sc[15] << 24);
        *reinterpret_cast<uint4*>(scales + dst * (D / 16) + n0 / 16) = packed;
      }
    }
  }
  pdl_launch_dependents();
  __syncthreads();
  if (warp == 1) {
    // every MMA must have finished before the accumulators are freed (after an abort the
    // epilogue may not have waited for them): one more commit on a barrier used only here
    if (lane == 0) {
      umma_commit(&sm.drain);
      if (!bounded_wait(&sm.drain, 0u, nullptr)) flag_error(dev_err, CSA2_DEVERR_TIMEOUT);
    }
    __syncwarp();
    tcgen05_fence_after();
    tmem_dealloc(tmem, kCedTmemCols);
  }
}

std::mutex g_ced_mu;
std::vector<int> g_ced_ready;  // per device: shared-memory attribute set

}  // namespace

cudaError_t launch_ced_quant(const void* h, const void* w, int B, int n, int d, const int32_t* pos,
                             int n_cap, uint8_t* codes, uint8_t* scales, int32_t* dev_err,
                             cudaStream_t s) {
  const TensorMapEncodeFn enc = tensor_map_encoder();
  if (enc == nullptr) return cudaErrorNotSupported;
  const int64_t M = static_cast<int64_t>(B) * n;
  CUtensorMap map_h, map_w;
  {
    const cuuint64_t dims[2] = {static_cast<cuuint64_t>(d), static_cast<cuuint64_t>(M)};
    const cuuint64_t strides[1] = {static_cast<cuuint64_t>(d) * 2};
    const cuuint32_t box[2] = {static_cast<cuuint32_t>(kCedK), static_cast<cuuint32_t>(kCedM)};
    const cuuint32_t estr[2] = {1, 1};
    if (enc(&map_h, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(h), dims, strides, box,
            estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
            CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
      return cudaErrorInvalidValue;
  }
  {
    const cuuint64_t dims[2] = {static_cast<cuuint64_t>(d), static_cast<cuuint64_t>(D)};
    const cuuint64_t strides[1] = {static_cast<cuuint64_t>(d) * 2};
    const cuuint32_t box[2] = {static_cast<cuuint32_t>(kCedK), static_cast<cuuint32_t>(kCedN)};
    const cuuint32_t estr[2] = {1, 1};
    if (enc(&map_w, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(w), dims, strides, box,
            estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
            CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
      return cudaErrorInvalidValue;
  }
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  {
    std::lock_guard<std::mutex> lock(g_ced_mu);
    if (dev >= static_cast<int>(g_ced_ready.size())) g_ced_ready.resize(dev + 1, 0);
    if (!g_ced_ready[dev]) {
      e = cudaFuncSetAttribute(ced_quant_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                               static_cast<int>(sizeof(CedSmem)));
      if (e != cudaSuccess) return e;
      g_ced_ready[dev] = 1;
    }
  }
  const int64_t tiles = ((M + kCedM - 1) / kCedM) * (D / kCedN);
  const dim3 grid(static_cast<unsigned>(std::min<int64_t>(tiles, device_sm_count())));
  e = launch_pdl(ced_quant_kernel, grid, dim3(kCedThreads), sizeof(CedSmem), s, map_h, map_w,
                 static_cast<int>(M), n, d, pos, n_cap, codes, scales, dev_err);
  count_launches(1);
  return e != cudaSuccess ? e : cudaGetLastError();
}

}  // namespace csa2

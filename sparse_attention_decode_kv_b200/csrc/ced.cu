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
// Two kernels project: ced_pair_kernel (further down) for calls of 256 or more token rows, where
// the two CTAs of a cluster share each MMA, and ced_quant_kernel for smaller calls.
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
//
// SWA bounded replay. "DeepSeek-V4.1-Flash: Pushing the Limits of KV Cache Compression",
// abstract: SWA Bounded Replay keeps the persistent (host / SSD) KV cache at about 1/8 of
// DeepSeek-V4-Flash's; the Juju Radar note on the report: the persistent cache rebuilds the local
// sliding-window state instead of storing it. Reading: a restored sequence gets its FP8 SWA ring
// back from the hidden states of its last Wr tokens: token r of sequence b is position
// p = N[b] - Wr + r, its SWA row is x = bf16_RNE(h w^T) (fp32 accumulation), quantised with the
// append path's SWA codec into ring slot p mod W. Two kernels:
//   replay_proj_kernel  the same persistent tcgen05 GEMM with the d-slices split over ksplit tile
//                       groups (the window is a few hundred rows, so the K split is what fills the
//                       SMs); the epilogue stores each fp32 partial accumulator row to a workspace.
//   replay_swa_kernel   one warp per token row: adds the ksplit partials in a fixed order, rounds
//                       to bf16, and applies the SWA codec (swa_codec.cuh) into the ring slot.
#include <algorithm>
#include <mutex>
#include <vector>

#include "common.cuh"
#include "internal.h"
#include "swa_codec.cuh"
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
constexpr int kCedNHalf = kCedN / 2;           // channels of a tile one CTA of a pair loads
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

// What the epilogue does with a finished 128-row x 256-channel accumulator.
enum ProjEpilogue : int {
  kEpiMxfp4Cache = 0,  // quantise each 16-channel group into MXFP4 cache rows pos[b] + i
  kEpiF32Partial = 1,  // store the fp32 partial sums of this tile's d-range to the workspace
};

struct ProjArgs {
  int M;       // rows of h (tokens)
  int n;       // rows per sequence (kEpiMxfp4Cache: token i of sequence b is row b n + i)
  int d;       // reduction length, a multiple of kCedK
  int ksplit;  // tile groups the d-slices are split over (1 for kEpiMxfp4Cache), <= d / kCedK
  const int32_t* pos;
  int n_cap;
  uint8_t* codes;
  uint8_t* scales;
  float* part;  // kEpiF32Partial: [ksplit][M][512]
  int32_t* dev_err;
};

// Tile t: channel half t % 2; then (t / 2) = token tile * ksplit + d-split.
struct ProjTile {
  int m0, n0, kb, ke, ks;
};
__device__ __forceinline__ ProjTile proj_tile(int t, int ksplit, int nk) {
  ProjTile r;
  r.n0 = (t & 1) * kCedN;
  const int u = t >> 1;
  const int mt = u / ksplit;
  r.ks = u - mt * ksplit;
  r.m0 = mt * kCedM;
  r.kb = r.ks * nk / ksplit;
  r.ke = (r.ks + 1) * nk / ksplit;
  return r;
}

template <int kEpi>
__device__ __forceinline__ void proj_body(const CUtensorMap* tm_h, const CUtensorMap* tm_w,
                                          const ProjArgs& a) {
  extern __shared__ __align__(1024) unsigned char smem_raw[];
  CedSmem& sm = *reinterpret_cast<CedSmem*>(smem_raw);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int M = a.M, n = a.n, ksplit = a.ksplit;
  const int nk = a.d / kCedK;
  int32_t* dev_err = a.dev_err;
  const int tiles = ((M + kCedM - 1) / kCedM) * (D / kCedN) * ksplit;
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
        const ProjTile pt = proj_tile(t, ksplit, nk);
        for (int kc = pt.kb; kc < pt.ke; ++kc, ++it) {
          const int s = it % kCedStages;
          if (it >= kCedStages &&
              !bounded_wait(&sm.empty[s], static_cast<uint32_t>(((it / kCedStages) & 1) ^ 1), abort)) {
            if (!*abort) flag_error(dev_err, CSA2_DEVERR_TIMEOUT);
            *abort = 1;
            break;
          }
          mbar_arrive_expect_tx(&sm.full[s], kCedATile + kCedBTile);
          tma_load_2d(sm.a[s], tm_h, &sm.full[s], kc * kCedK, pt.m0);
          tma_load_2d(sm.b[s], tm_w, &sm.full[s], kc * kCedK, pt.n0);
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
        const ProjTile pt = proj_tile(static_cast<int>(blockIdx.x) + j * static_cast<int>(gridDim.x),
                                      ksplit, nk);
        bool ok = true;
        for (int kc = pt.kb; kc < pt.ke; ++kc, ++it) {
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
                      (kc != pt.kb || k4 != 0) ? 1u : 0u);
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
      const ProjTile pt = proj_tile(t, ksplit, nk);
      const int m0 = pt.m0, n0 = pt.n0;
      const bool ok = __all_sync(0xFFFFFFFFu,
                                 bounded_wait(&sm.acc_full[acc], static_cast<uint32_t>((j >> 1) & 1), abort));
      if (!ok) {  // the MMA issuer gave up (and has flagged it) or the wait ran out
        if (lane == 0 && !*abort) flag_error(dev_err, CSA2_DEVERR_TIMEOUT);
        break;
      }
      tcgen05_fence_after();
      const int row = m0 + 32 * quarter + lane;
      const uint32_t tbase =
          tmem + static_cast<uint32_t>(acc * kCedN) + (static_cast<uint32_t>(32 * quarter) << 16);
      if constexpr (kEpi == kEpiF32Partial) {
        float* prow = a.part + (static_cast<int64_t>(pt.ks) * M + row) * D + n0;
#pragma unroll 1
        for (int g = 0; g < kCedN / 16; ++g) {
          uint32_t r[16];
          tmem_ld16(tbase + static_cast<uint32_t>(16 * g), r);
          tmem_wait_ld();
          if (row < M) {
            float4* dst4 = reinterpret_cast<float4*>(prow + 16 * g);
#pragma unroll
            for (int q = 0; q < 4; ++q)
              dst4[q] = make_float4(__uint_as_float(r[4 * q]), __uint_as_float(r[4 * q + 1]),
                                    __uint_as_float(r[4 * q + 2]), __uint_as_float(r[4 * q + 3]));
          }
        }
        tcgen05_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(&sm.acc_empty[acc]);
        continue;
      }
      const int32_t* pos = a.pos;
      const int n_cap = a.n_cap;
      uint8_t* codes = a.codes;
      uint8_t* scales = a.scales;
      int64_t dst = -1;
      if (row < M) {
        const int b = row / n, i = row - (row / n) * n;
        const int64_t p = static_cast<int64_t>(__ldg(pos + b)) + i;
        if (p >= 0 && p < n_cap) dst = static_cast<int64_t>(b) * n_cap + p;
        else if (n0 == 0) flag_error(dev_err, CSA2_DEVERR_POS_RANGE);
      }
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

__global__ void __launch_bounds__(kCedThreads, 1)
    ced_quant_kernel(const __grid_constant__ CUtensorMap tm_h, const __grid_constant__ CUtensorMap tm_w,
                     const ProjArgs a) {
  proj_body<kEpiMxfp4Cache>(&tm_h, &tm_w, a);
}

__global__ void __launch_bounds__(kCedThreads, 1)
    replay_proj_kernel(const __grid_constant__ CUtensorMap tm_h,
                       const __grid_constant__ CUtensorMap tm_w, const ProjArgs a) {
  proj_body<kEpiF32Partial>(&tm_h, &tm_w, a);
}

// ---------------------------------------------------------------------------- CTA-pair kernel
//
// ced_pair_kernel: the same projection and MXFP4 epilogue with the MMA shared by the two CTAs of a
// cluster (tcgen05 cta_group::2). A pair tile is 256 tokens x 256 channels: CTA r of the pair
// loads its 128 token rows of h and channels 128 r .. 128 r + 127 of the tile's w rows (16 KiB
// each per 64-wide d-slice), the leader issues M 256 x N 256 x K 16 MMAs that read both CTAs'
// stages, and each CTA's tensor memory receives its own 128 rows x 256 channels. Per unit of MMA
// work each CTA streams a third less than a CTA of ced_quant_kernel (32 instead of 48 KiB per
// d-slice), and the freed shared memory holds six stages instead of four.
//   warp 0, one thread  TMA producer (both CTAs): loads this CTA's halves; the copies of both
//                       CTAs complete on the leader's stage barrier, whose producer alone posts the
//                       pair's byte count.
//   warp 1, one thread  MMA issuer (leader only): waits for a stage, issues four pair MMAs,
//                       commits to the stage's empty barrier in both CTAs; after a tile, commits
//                       to the accumulator-full barrier in both CTAs. Warp 1 of both CTAs
//                       allocates and frees the pair's tensor memory.
//   warps 2..5          epilogue (both CTAs): as in ced_quant_kernel on this CTA's rows, then one
//                       arrival per warp on the leader's accumulator-empty barrier (8 per tile).
constexpr int kPairStages = 6;
constexpr int kPairTile = 128 * kCedK * 2;  // 16 KiB: 128 rows of a 64-wide bf16 d-slice
constexpr uint32_t kPairIdesc = umma_idesc_bf16_f32(2 * kCedM, kCedN);

struct __align__(1024) CedPairSmem {
  uint8_t a[kPairStages][kPairTile];
  uint8_t b[kPairStages][kPairTile];
  uint64_t full[kPairStages];   // leader: both CTAs' copies of the stage have landed
  uint64_t empty[kPairStages];  // each CTA: the pair MMAs have read the stage
  uint64_t acc_full[2];         // each CTA: the accumulator is complete
  uint64_t acc_empty[2];        // leader: the 8 epilogue warps of the pair have read it out
  uint64_t drain;               // each CTA: every pair MMA has completed
  uint32_t tmem_base;
  int abort;
};

static_assert(sizeof(CedPairSmem) <= 227 * 1024, "ced_pair_kernel shared memory");

__global__ void __launch_bounds__(kCedThreads, 1)
    ced_pair_kernel(const __grid_constant__ CUtensorMap tm_h,
                    const __grid_constant__ CUtensorMap tm_w_half, const ProjArgs a) {
  extern __shared__ __align__(1024) unsigned char smem_raw[];
  CedPairSmem& sm = *reinterpret_cast<CedPairSmem*>(smem_raw);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const uint32_t rank = cluster_ctarank();
  const int pair = static_cast<int>(blockIdx.x >> 1), npairs = static_cast<int>(gridDim.x >> 1);
  const int M = a.M, n = a.n;
  const int nk = a.d / kCedK;
  int32_t* dev_err = a.dev_err;
  const int tiles = ((M + 2 * kCedM - 1) / (2 * kCedM)) * (D / kCedN);
  const int my_tiles = tiles > pair ? (tiles - 1 - pair) / npairs + 1 : 0;

  if (threadIdx.x == 0) {
    for (int s = 0; s < kPairStages; ++s) {
      mbar_init(&sm.full[s], 1);
      mbar_init(&sm.empty[s], 1);
    }
    for (int c = 0; c < 2; ++c) {
      mbar_init(&sm.acc_full[c], 1);
      mbar_init(&sm.acc_empty[c], 2 * kCedEpiWarps);
    }
    mbar_init(&sm.drain, 1);
    sm.abort = 0;
    fence_barrier_init();
  }
  if (warp == 1) {
    tmem_alloc_pair(&sm.tmem_base, kCedTmemCols);
    tmem_relinquish_pair();
  }
  tcgen05_fence_before();
  __syncthreads();
  cluster_sync();  // both CTAs' barriers are initialised before either signals the other's
  tcgen05_fence_after();
  const uint32_t tmem = sm.tmem_base;
  volatile int* abort = &sm.abort;
  pdl_wait();  // h, w and pos may be written by the preceding kernel

  if (warp == 0) {
    // ------------------------------------------------------------------------ TMA producer
    if (lane == 0) {
      int it = 0;
      for (int j = 0; j < my_tiles && !*abort; ++j) {
        const int t = pair + j * npairs;
        const int m0 = (t >> 1) * (2 * kCedM) + static_cast<int>(rank) * kCedM;
        const int n0 = (t & 1) * kCedN + static_cast<int>(rank) * kCedNHalf;
        for (int kc = 0; kc < nk; ++kc, ++it) {
          const int s = it % kPairStages;
          if (it >= kPairStages &&
              !bounded_wait(&sm.empty[s], static_cast<uint32_t>(((it / kPairStages) & 1) ^ 1), abort)) {
            if (!*abort) flag_error(dev_err, CSA2_DEVERR_TIMEOUT);
            *abort = 1;
            break;
          }
          const uint32_t full_leader = mapa_shared(smem_u32(&sm.full[s]), 0);
          if (rank == 0) mbar_arrive_expect_tx(&sm.full[s], 2 * 2 * kPairTile);
          tma_load_2d_pair(sm.a[s], &tm_h, full_leader, kc * kCedK, m0);
          tma_load_2d_pair(sm.b[s], &tm_w_half, full_leader, kc * kCedK, n0);
        }
      }
      // the leader's stage barriers count both CTAs' copies: its drain covers the pair's
      if (rank == 0)
        for (int q = max(0, it - kPairStages); q < it; ++q)
          if (!mbar_wait(&sm.full[q % kPairStages], static_cast<uint32_t>((q / kPairStages) & 1)))
            flag_error(dev_err, CSA2_DEVERR_TIMEOUT);
    }
  } else if (warp == 1) {
    // -------------------------------------------------------------------------- MMA issuer
    if (lane == 0 && rank == 0) {
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
          const int s = it % kPairStages;
          if (!bounded_wait(&sm.full[s], static_cast<uint32_t>((it / kPairStages) & 1), abort)) {
            if (!*abort) flag_error(dev_err, CSA2_DEVERR_TIMEOUT);
            *abort = 1;
            ok = false;
            break;
          }
          tcgen05_fence_after();
          const uint32_t a0 = smem_u32(sm.a[s]), b0 = smem_u32(sm.b[s]);
#pragma unroll
          for (int k4 = 0; k4 < kCedK / 16; ++k4)
            umma_bf16_pair(d_tmem, umma_desc_k128(a0 + 32 * k4), umma_desc_k128(b0 + 32 * k4),
                           kPairIdesc, (kc | k4) != 0 ? 1u : 0u);
          const uint32_t e = smem_u32(&sm.empty[s]);
          umma_commit_pair(mapa_shared(e, 0));  // both CTAs may refill the stage
          umma_commit_pair(mapa_shared(e, 1));
        }
        const uint32_t f = smem_u32(&sm.acc_full[acc]);
        umma_commit_pair(mapa_shared(f, 0));
        umma_commit_pair(mapa_shared(f, 1));
        if (!ok) break;
      }
    }
  } else {
    // ---------------------------------------------------------------------------- epilogue
    const int quarter = warp & 3;
    const uint32_t acc_empty_leader0 = mapa_shared(smem_u32(&sm.acc_empty[0]), 0);
    const uint32_t acc_empty_leader1 = mapa_shared(smem_u32(&sm.acc_empty[1]), 0);
    for (int j = 0; j < my_tiles; ++j) {
      const int acc = j & 1;
      const int t = pair + j * npairs;
      const int m0 = (t >> 1) * (2 * kCedM) + static_cast<int>(rank) * kCedM;
      const int n0 = (t & 1) * kCedN;
      const bool ok = __all_sync(0xFFFFFFFFu,
                                 bounded_wait(&sm.acc_full[acc], static_cast<uint32_t>((j >> 1) & 1), abort));
      if (!ok) {
        if (lane == 0 && !*abort) flag_error(dev_err, CSA2_DEVERR_TIMEOUT);
        break;
      }
      tcgen05_fence_after();
      const int row = m0 + 32 * quarter + lane;
      const uint32_t tbase =
          tmem + static_cast<uint32_t>(acc * kCedN) + (static_cast<uint32_t>(32 * quarter) << 16);
      int64_t dst = -1;
      if (row < M) {
        const int b = row / n, i = row - (row / n) * n;
        const int64_t p = static_cast<int64_t>(__ldg(a.pos + b)) + i;
        if (p >= 0 && p < a.n_cap) dst = static_cast<int64_t>(b) * a.n_cap + p;
        else if (n0 == 0) flag_error(dev_err, CSA2_DEVERR_POS_RANGE);
      }
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
        if (dst >= 0) *reinterpret_cast<uint2*>(a.codes + dst * (D / 2) + n0 / 2 + 8 * g) = cw;
      }
      tcgen05_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive_cluster(acc ? acc_empty_leader1 : acc_empty_leader0);
      if (dst >= 0) {
        uint4 packed;
        packed.x = sc[0] | (sc[1] << 8) | (sc[2] << 16) | (sc[3] << 24);
        packed.y = sc[4] | (sc[5] << 8) | (sc[6] << 16) | (sc[7] << 24);
        packed.z = sc[8] | (sc[9] << 8) | (sc[10] << 16) | (sc[11] << 24);
        packed.w = sc[12] | (sc[13] << 8) | (sc[14] << 16) | (sc[15] << 24);
        *reinterpret_cast<uint4*>(a.scales + dst * (D / 16) + n0 / 16) = packed;
      }
    }
  }
  pdl_launch_dependents();
  __syncthreads();
  if (warp == 1) {
    // every pair MMA must have completed before either CTA frees its tensor memory: the leader
    // commits once more to a barrier used only here, in both CTAs
    if (lane == 0) {
      if (rank == 0) {
        const uint32_t d = smem_u32(&sm.drain);
        umma_commit_pair(mapa_shared(d, 0));
        umma_commit_pair(mapa_shared(d, 1));
      }
      if (!bounded_wait(&sm.drain, 0u, nullptr)) flag_error(dev_err, CSA2_DEVERR_TIMEOUT);
    }
    __syncwarp();
  }
  tcgen05_fence_before();
  cluster_sync();  // neither CTA leaves while the pair's MMAs or copies may use its memory
  if (warp == 1) {
    tcgen05_fence_after();
    tmem_dealloc_pair(tmem, kCedTmemCols);
  }
}

// One warp per window row: sum of the partials (split 0 first), bf16 rounding, SWA codec.
constexpr int kReplayWarps = 8;
constexpr int kReplaySumBatch = 4;  // partial rows requested at once per lane
__global__ void __launch_bounds__(kReplayWarps * 32)
    replay_swa_kernel(const float* __restrict__ part, int ksplit, int M, int Wr,
                      const int32_t* __restrict__ N, uint8_t* __restrict__ swa,
                      float* __restrict__ swa_scale, int W, int32_t* dev_err) {
  pdl_wait();
  pdl_launch_dependents();
  const int lane = threadIdx.x & 31;
  const int row = static_cast<int>(blockIdx.x) * kReplayWarps + static_cast<int>(threadIdx.x >> 5);
  if (row >= M) return;
  const int b = row / Wr, r = row - (row / Wr) * Wr;
  const int nb = __ldg(N + b);
  if (nb < 0) {
    if (lane == 0 && r == 0) flag_error(dev_err, CSA2_DEVERR_NLEN);
    return;
  }
  const int64_t p = static_cast<int64_t>(nb) - Wr + r;
  if (p < 0) return;  // the sequence is shorter than the window: no such token
  float v[16];
#pragma unroll
  for (int k = 0; k < 16; ++k) v[k] = 0.0f;
  const float* base = part + static_cast<int64_t>(row) * D + 16 * lane;
  const int64_t split_stride = static_cast<int64_t>(M) * D;
  int ks = 0;
  for (; ks + kReplaySumBatch <= ksplit; ks += kReplaySumBatch) {  // loads of a batch in flight
    float4 f[kReplaySumBatch][4];
#pragma unroll
    for (int u = 0; u < kReplaySumBatch; ++u)
#pragma unroll
      for (int q = 0; q < 4; ++q)
        f[u][q] = __ldg(reinterpret_cast<const float4*>(base + (ks + u) * split_stride) + q);
#pragma unroll
    for (int u = 0; u < kReplaySumBatch; ++u)  // added in split order
#pragma unroll
      for (int q = 0; q < 4; ++q) {
        v[4 * q] += f[u][q].x;
        v[4 * q + 1] += f[u][q].y;
        v[4 * q + 2] += f[u][q].z;
        v[4 * q + 3] += f[u][q].w;
      }
  }
  for (; ks < ksplit; ++ks)
#pragma unroll
    for (int q = 0; q < 4; ++q) {
      const float4 f = __ldg(reinterpret_cast<const float4*>(base + ks * split_stride) + q);
      v[4 * q] += f.x;
      v[4 * q + 1] += f.y;
      v[4 * q + 2] += f.z;
      v[4 * q + 3] += f.w;
    }
#pragma unroll
  for (int k = 0; k < 16; ++k) v[k] = __bfloat162float(__float2bfloat16_rn(v[k]));
  uint32_t e[4];
  const float s = swa_quantize_row_lane(v, e);
  const int64_t slot = static_cast<int64_t>(b) * W + p % W;
  reinterpret_cast<uint4*>(swa + slot * D)[lane] = make_uint4(e[0], e[1], e[2], e[3]);
  if (lane == 0) swa_scale[slot] = s;
}

std::mutex g_ced_mu;
std::vector<int> g_ced_ready;  // per device: shared-memory attributes set

// Tensor maps of h [M, d] (boxes of 128 rows) and w [512, d] (boxes of 256 rows, and of 128
// rows, one CTA's share of a pair tile, when map_w_half is given), 64-wide d-slices with 128-byte
// swizzle.
cudaError_t proj_tensor_maps(const void* h, const void* w, int64_t M, int d, CUtensorMap* map_h,
                             CUtensorMap* map_w, CUtensorMap* map_w_half = nullptr) {
  const TensorMapEncodeFn enc = tensor_map_encoder();
  if (enc == nullptr) return cudaErrorNotSupported;
  const cuuint64_t strides[1] = {static_cast<cuuint64_t>(d) * 2};
  const cuuint32_t estr[2] = {1, 1};
  {
    const cuuint64_t dims[2] = {static_cast<cuuint64_t>(d), static_cast<cuuint64_t>(M)};
    const cuuint32_t box[2] = {static_cast<cuuint32_t>(kCedK), static_cast<cuuint32_t>(kCedM)};
    if (enc(map_h, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(h), dims, strides, box,
            estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
            CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
      return cudaErrorInvalidValue;
  }
  for (int half = 0; half < (map_w_half != nullptr ? 2 : 1); ++half) {
    const cuuint64_t dims[2] = {static_cast<cuuint64_t>(d), static_cast<cuuint64_t>(D)};
    const cuuint32_t box[2] = {static_cast<cuuint32_t>(kCedK),
                               static_cast<cuuint32_t>(half ? kCedNHalf : kCedN)};
    if (enc(half ? map_w_half : map_w, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(w),
            dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
            CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
      return cudaErrorInvalidValue;
  }
  return cudaSuccess;
}

cudaError_t proj_configure() {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  std::lock_guard<std::mutex> lock(g_ced_mu);
  if (dev >= static_cast<int>(g_ced_ready.size())) g_ced_ready.resize(dev + 1, 0);
  if (!g_ced_ready[dev]) {
    e = cudaFuncSetAttribute(ced_quant_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             static_cast<int>(sizeof(CedSmem)));
    if (e == cudaSuccess)
      e = cudaFuncSetAttribute(replay_proj_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                               static_cast<int>(sizeof(CedSmem)));
    if (e == cudaSuccess)
      e = cudaFuncSetAttribute(ced_pair_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                               static_cast<int>(sizeof(CedPairSmem)));
    if (e != cudaSuccess) return e;
    g_ced_ready[dev] = 1;
  }
  return cudaSuccess;
}

constexpr int kReplayTargetCtas = 148;  // one B200's SMs: the K split aims to fill them once

int replay_ksplit(int64_t M, int d) {
  const int64_t mn_tiles = ((M + kCedM - 1) / kCedM) * (D / kCedN);
  int64_t k = kReplayTargetCtas / std::max<int64_t>(mn_tiles, 1);
  k = std::min<int64_t>(k, d / kCedK);
  return static_cast<int>(std::max<int64_t>(k, 1));
}

}  // namespace

cudaError_t launch_ced_quant(const void* h, const void* w, int B, int n, int d, const int32_t* pos,
                             int n_cap, uint8_t* codes, uint8_t* scales, int32_t* dev_err,
                             cudaStream_t s) {
  const int64_t M = static_cast<int64_t>(B) * n;
  CUtensorMap map_h, map_w, map_w_half;
  cudaError_t e = proj_tensor_maps(h, w, M, d, &map_h, &map_w, &map_w_half);
  if (e == cudaSuccess) e = proj_configure();
  if (e != cudaSuccess) return e;
  if (M >= 2 * kCedM) {  // CTA pairs: 256-token tiles, one cluster of 2 per tile slot
    ProjArgs a{};
    a.M = static_cast<int>(M);
    a.n = n;
    a.d = d;
    a.ksplit = 1;
    a.pos = pos;
    a.n_cap = n_cap;
    a.codes = codes;
    a.scales = scales;
    a.dev_err = dev_err;
    const int64_t pair_tiles = ((M + 2 * kCedM - 1) / (2 * kCedM)) * (D / kCedN);
    const int64_t pairs = std::min<int64_t>(pair_tiles, device_sm_count() / 2);
    profile_begin(CSA2_KERNEL_CED, s);
    e = launch_pdl_cluster(ced_pair_kernel, dim3(static_cast<unsigned>(2 * pairs)),
                           dim3(kCedThreads), sizeof(CedPairSmem), s, 2, map_h, map_w_half, a);
    profile_end(CSA2_KERNEL_CED, s);
    count_launches(1);
    return e != cudaSuccess ? e : cudaGetLastError();
  }
  // fewer than 256 tokens: single CTAs on 128-token tiles
  const int64_t tiles = ((M + kCedM - 1) / kCedM) * (D / kCedN);
  ProjArgs a{};
  a.M = static_cast<int>(M);
  a.n = n;
  a.d = d;
  a.ksplit = 1;
  a.pos = pos;
  a.n_cap = n_cap;
  a.codes = codes;
  a.scales = scales;
  a.dev_err = dev_err;
  const dim3 grid(static_cast<unsigned>(std::min<int64_t>(tiles, device_sm_count())));
  profile_begin(CSA2_KERNEL_CED, s);
  e = launch_pdl(ced_quant_kernel, grid, dim3(kCedThreads), sizeof(CedSmem), s, map_h, map_w, a);
  profile_end(CSA2_KERNEL_CED, s);
  count_launches(1);
  return e != cudaSuccess ? e : cudaGetLastError();
}

size_t swa_replay_workspace_bytes(int B, int Wr, int d) {
  const int64_t M = static_cast<int64_t>(B) * Wr;
  return static_cast<size_t>(replay_ksplit(M, d)) * static_cast<size_t>(M) * D * sizeof(float);
}

cudaError_t launch_swa_replay(const void* h, const void* w, int B, int Wr, int d, const int32_t* N,
                              uint8_t* swa, float* swa_scale, int W, void* ws, int32_t* dev_err,
                              cudaStream_t s) {
  const int64_t M = static_cast<int64_t>(B) * Wr;
  CUtensorMap map_h, map_w;
  cudaError_t e = proj_tensor_maps(h, w, M, d, &map_h, &map_w);
  if (e == cudaSuccess) e = proj_configure();
  if (e != cudaSuccess) return e;
  const int ksplit = replay_ksplit(M, d);
  ProjArgs a{};
  a.M = static_cast<int>(M);
  a.n = Wr;
  a.d = d;
  a.ksplit = ksplit;
  a.part = static_cast<float*>(ws);
  a.dev_err = dev_err;
  const int64_t tiles = ((M + kCedM - 1) / kCedM) * (D / kCedN) * ksplit;
  const dim3 grid(static_cast<unsigned>(std::min<int64_t>(tiles, device_sm_count())));
  profile_begin(CSA2_KERNEL_REPLAY, s);
  e = launch_pdl(replay_proj_kernel, grid, dim3(kCedThreads), sizeof(CedSmem), s, map_h, map_w, a);
  count_launches(1);
  if (e == cudaSuccess) e = cudaGetLastError();
  if (e == cudaSuccess) {
    const dim3 grid2(static_cast<unsigned>((M + kReplayWarps - 1) / kReplayWarps));
    e = launch_pdl(replay_swa_kernel, grid2, dim3(kReplayWarps * 32), 0, s,
                   static_cast<const float*>(ws), ksplit, static_cast<int>(M), Wr, N, swa,
                   swa_scale, W, dev_err);
    count_launches(1);
    if (e == cudaSuccess) e = cudaGetLastError();
  }
  profile_end(CSA2_KERNEL_REPLAY, s);
  return e;
}

}  // namespace csa2

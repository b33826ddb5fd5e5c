// row_gather.cu -- measurement probe (not part of the library) behind the gather in
// csrc/attend_tc.cu: bandwidth of random-row gathers of 256-byte code rows and 32-byte scale rows
// (an MXFP4 cache) into shared memory, by method and by the number of issuing warps: cp.async
// 16 B (16 lanes per row), TMA tile::gather4 (two 128-byte code halves with 128-byte swizzle plus the
// scale rows), one cp.async.bulk per row, plain 16-byte loads into registers (16 lanes per row), and
// one thread per row loading its own row (uncoalesced). One CTA per SM,
// persistent over tiles of 128 rows, a two-slot ring and a consumer warp that touches each row.
// All waits are bounded; every index stays inside its buffer.
//
// Build and run on a B200:
//   nvcc -gencode arch=compute_100a,code=sm_100a -O3 -std=c++17 -o /tmp/row_gather \
//        sparse_attention_decode_kv_b200/probes/row_gather.cu && /tmp/row_gather
#include <cstdio>
#include <cstdint>
#include <cstdlib>
#include <vector>
#include <cuda.h>
#include <cuda_runtime.h>

constexpr int kT = 128;
constexpr int kStage = kT * 288;

__device__ __forceinline__ uint32_t smem_u32(const void* p) { return (uint32_t)__cvta_generic_to_shared(p); }
__device__ __forceinline__ uint64_t gtime() { uint64_t t; asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t)); return t; }
__device__ __forceinline__ void mbar_init(uint64_t* b, uint32_t c) { asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(smem_u32(b)), "r"(c) : "memory"); }
__device__ __forceinline__ bool mbar_try(uint64_t* b, uint32_t ph) {
  uint32_t ok;
  asm volatile("{\n\t.reg .pred p;\n\tmbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\tselp.u32 %0, 1, 0, p;\n\t}" : "=r"(ok) : "r"(smem_u32(b)), "r"(ph) : "memory");
  return ok;
}
__device__ bool mbar_wait(uint64_t* b, uint32_t ph) {
  const uint64_t t0 = gtime();
  while (!mbar_try(b, ph)) if (gtime() - t0 > 500000000ull) return false;
  return true;
}
__device__ __forceinline__ void mbar_arrive(uint64_t* b) { asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(smem_u32(b)) : "memory"); }
__device__ __forceinline__ void mbar_expect(uint64_t* b, uint32_t bytes) { asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(smem_u32(b)), "r"(bytes) : "memory"); }
__device__ __forceinline__ void cp16(uint32_t dst, const void* src) { asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(dst), "l"(src) : "memory"); }
__device__ __forceinline__ void cp_arrive(uint64_t* b) { asm volatile("cp.async.mbarrier.arrive.noinc.shared::cta.b64 [%0];" ::"r"(smem_u32(b)) : "memory"); }
__device__ __forceinline__ void gather4(uint32_t dst, const CUtensorMap* m, uint64_t* b, int x, int y0, int y1, int y2, int y3) {
  asm volatile("cp.async.bulk.tensor.2d.shared::cluster.global.tile::gather4.mbarrier::complete_tx::bytes [%0], [%1, {%3, %4, %5, %6, %7}], [%2];"
               ::"r"(dst), "l"((uint64_t)m), "r"(smem_u32(b)), "r"(x), "r"(y0), "r"(y1), "r"(y2), "r"(y3) : "memory");
}
__device__ __forceinline__ void bulk(uint32_t dst, const void* src, uint32_t bytes, uint64_t* b) {
  asm volatile("cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(dst), "l"(src), "r"(bytes), "r"(smem_u32(b)) : "memory");
}

struct Smem {
  alignas(1024) unsigned char raw[2][kStage];
  uint64_t full[2], empty[2];
};

// method: 0 cp.async (16 lanes per row), 1 TMA gather4 (code halves 128 B swizzled + scales),
//         2 cp.async.bulk per row (256 B + 32 B), 3 ld.global.nc.v4 into registers (no smem),
//         4 one thread per row, 16-byte loads of its own row into registers (no smem)
template <int METHOD, int PW>
__global__ void __launch_bounds__(32 * (PW + 1), 1)
    gather_kernel(const __grid_constant__ CUtensorMap mc, const __grid_constant__ CUtensorMap ms,
                  const uint8_t* codes, const uint8_t* scales, const int* idx, int tiles_per_cta,
                  unsigned* sink, int* err) {
  extern __shared__ __align__(1024) unsigned char sraw[];
  Smem& sm = *reinterpret_cast<Smem*>(sraw);
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  if (tid == 0) {
    for (int s = 0; s < 2; ++s) {
      mbar_init(&sm.full[s], METHOD == 0 ? 32 * PW : 1);
      mbar_init(&sm.empty[s], 1);
    }
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
  }
  __syncthreads();
  const int* my_idx = idx + (size_t)blockIdx.x * tiles_per_cta * kT;
  unsigned acc = 0;
  if (METHOD == 4) {
    // one thread per row: each thread loads its own row's 16 code pieces and 2 scale pieces, one
    // tile of 128 rows per 4 warps, the next tile's pieces requested before the current are used
    {
      for (int e = threadIdx.x; e < tiles_per_cta * kT; e += blockDim.x) {
        const int row = my_idx[e];
        const uint4* src = reinterpret_cast<const uint4*>(codes + (size_t)row * 256);
        uint4 v[16];
#pragma unroll
        for (int c = 0; c < 16; ++c) v[c] = __ldg(src + c);
        const uint4 s0 = __ldg(reinterpret_cast<const uint4*>(scales + (size_t)row * 32));
        const uint4 s1 = __ldg(reinterpret_cast<const uint4*>(scales + (size_t)row * 32) + 1);
#pragma unroll
        for (int c = 0; c < 16; ++c) acc ^= v[c].x ^ v[c].w;
        acc ^= s0.y ^ s1.z;
      }
    }
    sink[blockIdx.x * blockDim.x + tid] = acc;
    return;
  }
  if (METHOD == 3) {
    // every warp loads its share of rows straight into registers, 16 lanes per row
    const int nw = PW + 1;
    for (int t = 0; t < tiles_per_cta; ++t) {
      for (int r = warp * 2 + (lane >> 4); r < kT; r += 2 * nw) {
        const int row = my_idx[t * kT + r];
        const uint4 v = *reinterpret_cast<const uint4*>(codes + (size_t)row * 256 + 16 * (lane & 15));
        acc ^= v.x ^ v.w;
        if ((lane & 15) < 2) {
          const uint4 s = *reinterpret_cast<const uint4*>(scales + (size_t)row * 32 + 16 * (lane & 15));
          acc ^= s.y;
        }
      }
    }
    sink[blockIdx.x * blockDim.x + tid] = acc;
    return;
  }
  if (warp < PW) {
    for (int t = 0; t < tiles_per_cta; ++t) {
      const int slot = t & 1;
      if (t >= 2 && !mbar_wait(&sm.empty[slot], ((t >> 1) - 1) & 1)) { atomicExch(err, 1); break; }
      const uint32_t st = smem_u32(sm.raw[slot]);
      const int* ti = my_idx + t * kT;
      if (METHOD == 0) {
        // warp w: rows w, w + PW, ... two rows per instruction
        for (int r2 = warp * 2; r2 < kT; r2 += 2 * PW) {
          const int r = r2 + (lane >> 4), c = lane & 15;
          const int row = ti[r];
          cp16(st + r * 256 + ((c ^ (r & 15)) << 4), codes + (size_t)row * 256 + 16 * c);
        }
        for (int r = warp * 16 + (lane >> 1); r < kT; r += 16 * PW) {
          const int row = ti[r];
          cp16(st + kT * 256 + r * 32 + 16 * (lane & 1), scales + (size_t)row * 32 + 16 * (lane & 1));
        }
        cp_arrive(&sm.full[slot]);
      } else if (METHOD == 1) {
        if (warp == 0 && lane == 0) mbar_expect(&sm.full[slot], kStage);
        // all PW warps: lane groups of 4 rows
        for (int g = warp + PW * lane; g < kT / 4; g += 32 * PW) {
          const int r0 = ti[4 * g], r1 = ti[4 * g + 1], r2 = ti[4 * g + 2], r3 = ti[4 * g + 3];
          gather4(st + 512 * g, &mc, &sm.full[slot], 0, r0, r1, r2, r3);
          gather4(st + kT * 128 + 512 * g, &mc, &sm.full[slot], 128, r0, r1, r2, r3);
          gather4(st + kT * 256 + 128 * g, &ms, &sm.full[slot], 0, r0, r1, r2, r3);
        }
      } else {
        if (warp == 0 && lane == 0) mbar_expect(&sm.full[slot], kStage);
        for (int r = warp * 32 + lane; r < kT; r += 32 * PW) {
          const int row = ti[r];
          bulk(st + r * 256, codes + (size_t)row * 256, 256, &sm.full[slot]);
          bulk(st + kT * 256 + r * 32, scales + (size_t)row * 32, 32, &sm.full[slot]);
        }
      }
    }
  } else {
    // consumer: wait each slot, read one word per row, release
    for (int t = 0; t < tiles_per_cta; ++t) {
      const int slot = t & 1;
      if (!mbar_wait(&sm.full[slot], (t >> 1) & 1)) { atomicExch(err, 2); break; }
      for (int r = lane; r < kT; r += 32) acc ^= *reinterpret_cast<const unsigned*>(sm.raw[slot] + r * 256 + 16 * (r & 7));
      __syncwarp();
      if (lane == 0) mbar_arrive(&sm.empty[slot]);
    }
    sink[blockIdx.x * 32 + lane] = acc;
  }
  __syncthreads();
  // drain: every slot fill landed
  if (tid == 0 && METHOD != 3) {
    for (int s = 0; s < 2; ++s) {
      const int fills = (tiles_per_cta + 1 - s) / 2;
      if (fills > 0 && !mbar_wait(&sm.full[s], (fills - 1) & 1)) atomicExch(err, 3);
    }
  }
}

typedef CUresult (*EncFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*, const cuuint64_t*,
                          const cuuint32_t*, const cuuint32_t*, CUtensorMapInterleave, CUtensorMapSwizzle,
                          CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

template <int METHOD, int PW>
void run(const char* name, CUtensorMap mc, CUtensorMap ms, const uint8_t* codes, const uint8_t* scales, const int* idx,
         int tiles_per_cta, unsigned* sink, int* err, int sms) {
  auto k = gather_kernel<METHOD, PW>;
  const int smem = sizeof(Smem) + 1024;
  cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
  cudaEvent_t a, b;
  cudaEventCreate(&a);
  cudaEventCreate(&b);
  k<<<sms, 32 * (PW + 1), smem>>>(mc, ms, codes, scales, idx, tiles_per_cta, sink, err);
  cudaEventRecord(a);
  k<<<sms, 32 * (PW + 1), smem>>>(mc, ms, codes, scales, idx, tiles_per_cta, sink, err);
  cudaEventRecord(b);
  cudaError_t e = cudaEventSynchronize(b);
  float ms_ = 0;
  cudaEventElapsedTime(&ms_, a, b);
  int h = 0;
  cudaMemcpy(&h, err, 4, cudaMemcpyDeviceToHost);
  const double bytes = (double)sms * tiles_per_cta * kT * 288;
  printf("%-34s warps %2d: %8.1f GB/s  (%.3f ms) err=%d %s\n", name, PW, bytes / ms_ / 1e6, ms_, h, cudaGetErrorString(e));
}

int main() {
  int sms = 0;
  cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, 0);
  const size_t R = 8u << 20;  // rows: 2 GiB of codes + 256 MiB of scales
  uint8_t *codes, *scales;
  cudaMalloc(&codes, R * 256);
  cudaMalloc(&scales, R * 32);
  cudaMemset(codes, 1, R * 256);
  cudaMemset(scales, 2, R * 32);
  const int tiles_per_cta = 64;
  const size_t nidx = (size_t)sms * tiles_per_cta * kT;
  std::vector<int> h(nidx);
  uint64_t s = 88172645463325252ull;
  for (size_t i = 0; i < nidx; ++i) { s ^= s << 13; s ^= s >> 7; s ^= s << 17; h[i] = (int)(s % R); }
  int* idx;
  cudaMalloc(&idx, nidx * 4);
  cudaMemcpy(idx, h.data(), nidx * 4, cudaMemcpyHostToDevice);
  unsigned* sink;
  cudaMalloc(&sink, (size_t)sms * 1024 * 4);
  int* err;
  cudaMalloc(&err, 4);
  cudaMemset(err, 0, 4);
  void* p = nullptr;
  cudaDriverEntryPointQueryResult q;
  cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q);
  EncFn enc = (EncFn)p;
  CUtensorMap mc, ms;
  {
    cuuint64_t dims[2] = {256, R}, str[1] = {256};
    cuuint32_t box[2] = {128, 1}, es[2] = {1, 1};
    CUresult r = enc(&mc, CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, codes, dims, str, box, es, CU_TENSOR_MAP_INTERLEAVE_NONE,
                     CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    cuuint64_t dims2[2] = {32, R}, str2[1] = {32};
    cuuint32_t box2[2] = {32, 1};
    CUresult r2 = enc(&ms, CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, scales, dims2, str2, box2, es, CU_TENSOR_MAP_INTERLEAVE_NONE,
                      CU_TENSOR_MAP_SWIZZLE_NONE, CU_TENSOR_MAP_L2_PROMOTION_L2_128B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    printf("encode %d %d\n", (int)r, (int)r2);
    if (r || r2) return 1;
  }
  run<0, 2>("cp.async 16B", mc, ms, codes, scales, idx, tiles_per_cta, sink, err, sms);
  run<0, 4>("cp.async 16B", mc, ms, codes, scales, idx, tiles_per_cta, sink, err, sms);
  run<0, 8>("cp.async 16B", mc, ms, codes, scales, idx, tiles_per_cta, sink, err, sms);
  run<0, 16>("cp.async 16B", mc, ms, codes, scales, idx, tiles_per_cta, sink, err, sms);
  run<1, 1>("TMA gather4 (2x128B + 32B)", mc, ms, codes, scales, idx, tiles_per_cta, sink, err, sms);
  run<1, 2>("TMA gather4 (2x128B + 32B)", mc, ms, codes, scales, idx, tiles_per_cta, sink, err, sms);
  run<1, 4>("TMA gather4 (2x128B + 32B)", mc, ms, codes, scales, idx, tiles_per_cta, sink, err, sms);
  run<2, 1>("bulk per row (256B + 32B)", mc, ms, codes, scales, idx, tiles_per_cta, sink, err, sms);
  run<2, 4>("bulk per row (256B + 32B)", mc, ms, codes, scales, idx, tiles_per_cta, sink, err, sms);
  run<4, 3>("thread per row, 16-B loads", mc, ms, codes, scales, idx, tiles_per_cta, sink, err, sms);
  run<4, 7>("thread per row, 16-B loads", mc, ms, codes, scales, idx, tiles_per_cta, sink, err, sms);
  run<4, 15>("thread per row, 16-B loads", mc, ms, codes, scales, idx, tiles_per_cta, sink, err, sms);
  run<3, 7>("ld.global.v4 to registers", mc, ms, codes, scales, idx, tiles_per_cta, sink, err, sms);
  run<3, 15>("ld.global.v4 to registers", mc, ms, codes, scales, idx, tiles_per_cta, sink, err, sms);
  run<3, 31>("ld.global.v4 to registers", mc, ms, codes, scales, idx, tiles_per_cta, sink, err, sms);
  return 0;
}

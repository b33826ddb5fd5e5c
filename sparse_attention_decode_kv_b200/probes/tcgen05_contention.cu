// tcgen05_contention.cu -- measurement probe (not part of the library): what an M = 128, N = 16,
// K = 16 tcgen05.mma with A in tensor memory (the QK^T form of csrc/attend_tc.cu) costs while the
// CTA's other warps keep the SM busy the way the attention's other roles do.
//
// One CTA of 512 threads per SM. Warp 1's lane 0 issues batches of 64 MMAs (one commit and a
// bounded wait per batch) and times them with clock64; meanwhile, by mode:
//   0 idle           the other warps wait at the end
//   1 alu, same SMSP warps 5, 9 and 13 (warp 1's sub-partition) run a dequantisation-like ALU loop:
//                    E2M1 -> f16x2 converts, f16x2 multiplies and fp32 FMAs
//   2 alu, all       every warp but warp 1 runs that loop
//   3 tmem ld/st     warps 4-15 load and store tensor-memory columns 384-511 (not the MMA's)
//   4 tmem ld of A   warps 4-15 load the columns the MMAs read as A (0-255), as a copy out of
//                    tensor memory would
//   5 smem stores    warps 4-15 store 16 bytes per lane into shared memory, conflict-free
//   6 mixed          warps 4-11 load A columns and store them to shared memory, the rest run the
//                    ALU loop: the attention's steady state in outline
// The busy loops stop when the issuer raises a flag, and after at most kMaxIt iterations; every
// wait is bounded, every index stays inside its buffer. Operand contents are not initialised:
// only the time matters.
//
// Build and run on a B200:
//   nvcc -gencode arch=compute_100a,code=sm_100a -O3 -std=c++17 -o /tmp/tcgen05_contention \
//        sparse_attention_decode_kv_b200/probes/tcgen05_contention.cu && /tmp/tcgen05_contention
#include <cstdio>
#include <cstdint>
#include <vector>
#include <cuda_runtime.h>

constexpr int kThreads = 512;
constexpr int kBusyWarps = 12;   // warps 4..15
constexpr int kMaxIt = 1 << 20;  // cap of every busy loop
constexpr int kReps = 64;        // timed batches of 64 MMAs

__device__ __forceinline__ uint32_t smem_u32(const void* p) {
  return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}
__device__ __forceinline__ uint64_t gtime() {
  uint64_t t;
  asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
  return t;
}
__device__ __forceinline__ void mbar_init(uint64_t* b, uint32_t c) {
  asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(smem_u32(b)), "r"(c) : "memory");
}
__device__ __forceinline__ bool mbar_try(uint64_t* b, uint32_t ph) {
  uint32_t ok;
  asm volatile(
      "{\n\t.reg .pred p;\n\tmbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\tselp.u32 %0, 1, 0, p;\n\t}"
      : "=r"(ok)
      : "r"(smem_u32(b)), "r"(ph)
      : "memory");
  return ok;
}
__device__ bool mbar_wait(uint64_t* b, uint32_t ph) {
  const uint64_t t0 = gtime();
  while (!mbar_try(b, ph))
    if (gtime() - t0 > 200000000ull) return false;  // 0.2 s
  return true;
}
__device__ __forceinline__ uint64_t desc_k128(uint32_t addr) {
  uint64_t d = (addr >> 4) & 0x3FFFu;
  d |= 1ull << 16;
  d |= 64ull << 32;  // 1024-byte stride between 8-row groups
  d |= 1ull << 46;
  d |= 2ull << 61;   // 128-byte swizzle
  return d;
}
__host__ __device__ constexpr uint32_t idesc_f16(int M, int N) {
  return (1u << 4) | (static_cast<uint32_t>(N >> 3) << 17) | (static_cast<uint32_t>(M >> 4) << 24);
}
__device__ __forceinline__ void mma_ts(uint32_t d, uint32_t a, uint64_t b, uint32_t id, uint32_t acc) {
  asm volatile(
      "{\n\t.reg .pred p;\n\tsetp.ne.b32 p, %4, 0;\n\ttcgen05.mma.cta_group::1.kind::f16 [%0], [%1], %2, %3, p;\n\t}" ::"r"(d),
      "r"(a), "l"(b), "r"(id), "r"(acc)
      : "memory");
}
__device__ __forceinline__ void commit(uint64_t* b) {
  asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(smem_u32(b))
               : "memory");
}
__device__ __forceinline__ void fence_before() { asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory"); }
__device__ __forceinline__ void fence_after() { asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory"); }
__device__ __forceinline__ void ld16(uint32_t ta, uint32_t (&r)[16]) {
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x16.b32 {%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15}, [%16];"
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]), "=r"(r[8]),
        "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]), "=r"(r[15])
      : "r"(ta)
      : "memory");
}
__device__ __forceinline__ void st16(uint32_t ta, const uint32_t (&r)[16]) {
  asm volatile(
      "tcgen05.st.sync.aligned.32x32b.x16.b32 [%0], {%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,%16};" ::"r"(ta),
      "r"(r[0]), "r"(r[1]), "r"(r[2]), "r"(r[3]), "r"(r[4]), "r"(r[5]), "r"(r[6]), "r"(r[7]), "r"(r[8]), "r"(r[9]),
      "r"(r[10]), "r"(r[11]), "r"(r[12]), "r"(r[13]), "r"(r[14]), "r"(r[15])
      : "memory");
}
__device__ __forceinline__ void wait_ld() { asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory"); }
__device__ __forceinline__ void wait_st() { asm volatile("tcgen05.wait::st.sync.aligned;" ::: "memory"); }
__device__ __forceinline__ uint32_t e2m1x2_h2(uint32_t byte) {
  uint32_t r;
  asm volatile("{\n\t.reg .b8 t;\n\tcvt.u8.u32 t, %1;\n\tcvt.rn.f16x2.e2m1x2 %0, t;\n\t}" : "=r"(r) : "r"(byte));
  return r;
}
__device__ __forceinline__ uint32_t hmul2(uint32_t a, uint32_t b) {
  uint32_t r;
  asm volatile("mul.rn.f16x2 %0, %1, %2;" : "=r"(r) : "r"(a), "r"(b));
  return r;
}

struct Smem {
  uint16_t q[8 * 16 * 64];                  // B operand: 8 blocks of [16 rows x 128 B], 16 KiB
  uint4 scratch[kBusyWarps][8][32];         // 4 KiB per busy warp for mode 5 and 6 stores
  uint64_t bar;
  uint32_t tmem;
  int done;
};
constexpr size_t kSmem = sizeof(Smem) + 1024;
constexpr size_t kSmemLaunch = 160 * 1024;  // one CTA per SM
static_assert(kSmem <= kSmemLaunch, "shared memory");

__device__ Smem& get_smem(unsigned char* raw) {
  const uint32_t a = smem_u32(raw);
  return *reinterpret_cast<Smem*>(raw + (((a + 1023) & ~1023u) - a));
}

// A dequantisation-like ALU loop body: 8 converts, 8 f16x2 multiplies, 8 fp32 FMAs.
__device__ __forceinline__ void alu_body(uint32_t (&h)[8], float (&f)[8], uint32_t seed) {
#pragma unroll
  for (int k = 0; k < 8; ++k) {
    h[k] = hmul2(e2m1x2_h2((seed >> (4 * k)) & 0xFFu), h[k] | 0x3C003C00u);
    f[k] = fmaf(f[k], 1.0001f, 0.5f);
  }
}

__global__ void __launch_bounds__(kThreads, 1) contention_kernel(int mode, long long* cyc, int* err,
                                                                 float* sink) {
  extern __shared__ unsigned char raw[];
  Smem& sm = get_smem(raw);
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  if (tid == 0) {
    mbar_init(&sm.bar, 1);
    sm.done = 0;
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
  }
  if (warp == 0) {
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(smem_u32(&sm.tmem)),
                 "r"(512)
                 : "memory");
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
  }
  fence_before();
  __syncthreads();
  fence_after();
  const uint32_t tm = sm.tmem;
  const uint32_t t_lane = static_cast<uint32_t>(32 * (warp & 3)) << 16;
  volatile int* done = &sm.done;
  uint32_t h[8] = {0, 0, 0, 0, 0, 0, 0, 0};
  float f[8] = {0, 1, 2, 3, 4, 5, 6, 7};
  uint32_t acc = 0;

  if (warp == 1) {
    if (lane == 0) {
      const uint64_t db = desc_k128(smem_u32(sm.q));
      constexpr uint32_t id = idesc_f16(128, 16);
      uint32_t ph = 0;
      long long t0 = 0;
      for (int r = -2; r < kReps; ++r) {  // two untimed batches while the other warps start
        if (r == 0) t0 = clock64();
#pragma unroll
        for (int s = 0; s < 64; ++s) mma_ts(tm + 256, tm + 8 * (s % 32), db + 2 * (s % 4), id, s > 0);
        commit(&sm.bar);
        if (!mbar_wait(&sm.bar, ph)) {
          atomicExch(err, 1);
          break;
        }
        ph ^= 1;
      }
      cyc[blockIdx.x] = clock64() - t0;
      *done = 1;
    }
    __syncwarp();
  } else {
    const int bw = warp - 4;  // busy-warp index for modes 3-6
    const bool alu = (mode == 1 && (warp & 3) == 1) || (mode == 2) || (mode == 6 && (warp < 4 || warp >= 12));
    const bool tmem_ldst = mode == 3 && warp >= 4;
    const bool tmem_lda = (mode == 4 || mode == 6) && warp >= 4 && (mode == 4 || warp < 12);
    const bool smem_st = (mode == 5 || mode == 6) && warp >= 4 && (mode == 5 || warp < 12);
    if (alu || tmem_ldst || tmem_lda || smem_st) {
      for (int it = 0; it < kMaxIt; ++it) {
        if (__shfl_sync(0xFFFFFFFFu, *done, 0)) break;  // warp-uniform: the loop holds .sync.aligned ops
        if (alu) alu_body(h, f, static_cast<uint32_t>(it) * 2654435761u + static_cast<uint32_t>(tid));
        uint32_t r[16];
        if (tmem_ldst) {
          ld16(tm + t_lane + 384 + 16 * (it & 7), r);
          wait_ld();
          st16(tm + t_lane + 384 + 16 * ((it + 1) & 7), r);
          wait_st();
          acc += r[it & 15];
        }
        if (tmem_lda) {
          ld16(tm + t_lane + 16 * (it & 15), r);
          wait_ld();
          acc += r[it & 15];
          if (!smem_st) continue;
        }
        if (smem_st) {
          const uint4 v = make_uint4(acc + it, acc ^ it, acc, it);
#pragma unroll
          for (int k = 0; k < 8; ++k) sm.scratch[bw][k][lane] = v;
        }
      }
    }
  }
  float sum = static_cast<float>(acc);
#pragma unroll
  for (int k = 0; k < 8; ++k) sum += f[k] + static_cast<float>(h[k] & 0xFF);
  if (sum == 12345.678f) sink[tid] = sum;  // keeps the busy work alive
  fence_before();
  __syncthreads();
  if (warp == 0) {
    fence_after();
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tm), "r"(512) : "memory");
  }
}

int main() {
  int sms = 0;
  cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, 0);
  long long* dCyc;
  int* dErr;
  float* dSink;
  cudaMalloc(&dCyc, sms * sizeof(long long));
  cudaMalloc(&dErr, sizeof(int));
  cudaMalloc(&dSink, kThreads * sizeof(float));
  cudaMemset(dErr, 0, sizeof(int));
  cudaFuncSetAttribute(contention_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(kSmemLaunch));
  const char* names[7] = {"idle", "alu on the issuer's SMSP (warps 5, 9, 13)", "alu on every other warp",
                          "tmem ld/st of other columns (warps 4-15)", "tmem ld of the A columns (warps 4-15)",
                          "smem 16-byte stores (warps 4-15)", "mixed: A ld + smem st (4-11), alu (0, 2, 3, 12-15)"};
  for (int mode = 0; mode < 7; ++mode) {
    contention_kernel<<<sms, kThreads, kSmemLaunch>>>(mode, dCyc, dErr, dSink);
    contention_kernel<<<sms, kThreads, kSmemLaunch>>>(mode, dCyc, dErr, dSink);
    const cudaError_t e = cudaDeviceSynchronize();
    std::vector<long long> c(sms);
    cudaMemcpy(c.data(), dCyc, sms * sizeof(long long), cudaMemcpyDeviceToHost);
    double mean = 0;
    for (long long x : c) mean += static_cast<double>(x);
    mean /= sms;
    printf("mode %d %-52s %7.2f cycles per MMA  %s\n", mode, names[mode], mean / kReps / 64, cudaGetErrorString(e));
    if (e != cudaSuccess) return 1;
  }
  int herr = 0;
  cudaMemcpy(&herr, dErr, sizeof(int), cudaMemcpyDeviceToHost);
  printf("wait_err %d\n", herr);
  return herr ? 2 : 0;
}

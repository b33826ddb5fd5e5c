// tcgen05_shapes.cu -- measurement probe (not part of the library) behind the choice of tensor-core
// forms in csrc/attend_tc.cu.
//
// Checks, exactly against the host, the three tcgen05 forms an attention with items on M needs:
//   (1) S = V q^T, A = V [128 items x 512] K-major (128-byte swizzle) in shared memory,
//       B = q [16 x 512] K-major;
//   (2) the same with A = V in tensor memory (lane = item, two fp16 per column);
//   (3) O^T = V^T P^T, A = V^T read MN-major from the same shared tile, B = P [16 x 128] K-major.
// Then times, with one CTA per SM: the three forms; M = 64 / 128 x N = 16 .. 256 chains into 1 to 8
// accumulators; 1, 2 and 4 issuing warps; and tcgen05 next to mma.sync m16n8k16 warps on one SM.
// All waits are bounded; every index stays inside its buffer.
//
// Build and run on a B200:
//   nvcc -gencode arch=compute_100a,code=sm_100a -O3 -std=c++17 -o /tmp/tcgen05_shapes \
//        sparse_attention_decode_kv_b200/probes/tcgen05_shapes.cu && /tmp/tcgen05_shapes
#include <cstdio>
#include <cstdint>
#include <cstdlib>
#include <cstring>
#include <vector>
#include <cuda_runtime.h>
#include <cuda_fp16.h>

constexpr int T = 128, D = 512, H = 16;

__device__ __forceinline__ uint32_t smem_u32(const void* p) {
  return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}
__device__ __forceinline__ uint64_t gtime() { uint64_t t; asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t)); return t; }
__device__ __forceinline__ void mbar_init(uint64_t* b, uint32_t c) { asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(smem_u32(b)), "r"(c) : "memory"); }
__device__ __forceinline__ bool mbar_try(uint64_t* b, uint32_t ph) {
  uint32_t ok;
  asm volatile("{\n\t.reg .pred p;\n\tmbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\tselp.u32 %0, 1, 0, p;\n\t}" : "=r"(ok) : "r"(smem_u32(b)), "r"(ph) : "memory");
  return ok;
}
__device__ bool mbar_wait(uint64_t* b, uint32_t ph) {
  const uint64_t t0 = gtime();
  while (!mbar_try(b, ph)) if (gtime() - t0 > 200000000ull) return false;  // 0.2 s
  return true;
}
__device__ __forceinline__ uint64_t desc(uint32_t addr, uint32_t lbo, uint32_t sbo) {
  uint64_t d = (addr >> 4) & 0x3FFFu;
  d |= (uint64_t)((lbo >> 4) & 0x3FFFu) << 16;
  d |= (uint64_t)((sbo >> 4) & 0x3FFFu) << 32;
  d |= 1ull << 46;
  d |= 2ull << 61;
  return d;
}
__host__ __device__ constexpr uint32_t idesc_f16(int M, int N, int a_mn) {
  return (1u << 4) | (0u << 7) | (0u << 10) | ((uint32_t)a_mn << 15) | ((uint32_t)(N >> 3) << 17) | ((uint32_t)(M >> 4) << 24);
}
__device__ __forceinline__ void mma_ss(uint32_t d, uint64_t a, uint64_t b, uint32_t id, uint32_t acc) {
  asm volatile("{\n\t.reg .pred p;\n\tsetp.ne.b32 p, %4, 0;\n\ttcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n\t}" ::"r"(d), "l"(a), "l"(b), "r"(id), "r"(acc) : "memory");
}
__device__ __forceinline__ void mma_ts(uint32_t d, uint32_t a, uint64_t b, uint32_t id, uint32_t acc) {
  asm volatile("{\n\t.reg .pred p;\n\tsetp.ne.b32 p, %4, 0;\n\ttcgen05.mma.cta_group::1.kind::f16 [%0], [%1], %2, %3, p;\n\t}" ::"r"(d), "r"(a), "l"(b), "r"(id), "r"(acc) : "memory");
}
__device__ __forceinline__ void commit(uint64_t* b) {
  asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(smem_u32(b)) : "memory");
}
__device__ __forceinline__ void fence_before() { asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory"); }
__device__ __forceinline__ void fence_after() { asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory"); }
__device__ __forceinline__ void fence_async_smem() { asm volatile("fence.proxy.async.shared::cta;" ::: "memory"); }
__device__ __forceinline__ void ld16(uint32_t ta, uint32_t (&r)[16]) {
  asm volatile("tcgen05.ld.sync.aligned.32x32b.x16.b32 {%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15}, [%16];"
               : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]),
                 "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]), "=r"(r[15])
               : "r"(ta) : "memory");
}
__device__ __forceinline__ void st16(uint32_t ta, const uint32_t (&r)[16]) {
  asm volatile("tcgen05.st.sync.aligned.32x32b.x16.b32 [%0], {%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,%16};"
               ::"r"(ta), "r"(r[0]), "r"(r[1]), "r"(r[2]), "r"(r[3]), "r"(r[4]), "r"(r[5]), "r"(r[6]), "r"(r[7]),
                 "r"(r[8]), "r"(r[9]), "r"(r[10]), "r"(r[11]), "r"(r[12]), "r"(r[13]), "r"(r[14]), "r"(r[15]) : "memory");
}
__device__ __forceinline__ void wait_ld() { asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory"); }
__device__ __forceinline__ void wait_st() { asm volatile("tcgen05.wait::st.sync.aligned;" ::: "memory"); }

// SW128 byte offset of (row r, 16-byte chunk c) inside a region of 128-byte rows (1024-aligned).
__device__ __forceinline__ uint32_t sw(int r, int c) { return r * 128 + ((c ^ (r & 7)) << 4); }

struct Smem {
  uint16_t v[8 * T * 64];  // 8 dim-blocks x 128 rows x 128 B
  uint16_t q[8 * H * 64];  // 8 dim-blocks x 16 rows x 128 B
  uint16_t p[2 * H * 64];  // 2 item-blocks x 16 rows x 128 B
  uint64_t bar;
  uint32_t tmem;
};
constexpr size_t kSmem = sizeof(Smem) + 1024;

__device__ Smem& get_smem(unsigned char* raw) {
  const uint32_t a = smem_u32(raw);
  return *reinterpret_cast<Smem*>(raw + (((a + 1023) & ~1023u) - a));
}

// Fill smem (and TMEM A) from the global arrays. 128 threads.
__device__ void fill(Smem& sm, const uint16_t* V, const uint16_t* Q, const uint16_t* P, uint32_t tmem) {
  const int tid = threadIdx.x;
  unsigned char* vb = reinterpret_cast<unsigned char*>(sm.v);
  unsigned char* qb = reinterpret_cast<unsigned char*>(sm.q);
  unsigned char* pb = reinterpret_cast<unsigned char*>(sm.p);
  for (int e = tid; e < T * 64; e += 128) {  // 16-byte chunks of V: item i, chunk c (8 dims)
    const int i = e / 64, c = e % 64;
    const uint4 w = *reinterpret_cast<const uint4*>(V + i * D + 8 * c);
    *reinterpret_cast<uint4*>(vb + (c / 8) * (T * 128) + sw(i, c % 8)) = w;
  }
  for (int e = tid; e < H * 64; e += 128) {
    const int h = e / 64, c = e % 64;
    const uint4 w = *reinterpret_cast<const uint4*>(Q + h * D + 8 * c);
    *reinterpret_cast<uint4*>(qb + (c / 8) * (H * 128) + sw(h, c % 8)) = w;
  }
  for (int e = tid; e < H * 16; e += 128) {  // P[h][item], 16 chunks of 8 items per row
    const int h = e / 16, c = e % 16;
    const uint4 w = *reinterpret_cast<const uint4*>(P + h * T + 8 * c);
    *reinterpret_cast<uint4*>(pb + (c / 8) * (H * 128) + sw(h, c % 8)) = w;
  }
  // TMEM A: warp w writes lanes 32w..32w+31 = items; column j holds dims 2j, 2j+1
  const int warp = tid >> 5, lane = tid & 31, i = 32 * warp + lane;
  for (int cc = 0; cc < 16; ++cc) {
    uint32_t r[16];
    for (int j = 0; j < 16; ++j) r[j] = *reinterpret_cast<const uint32_t*>(V + i * D + 32 * cc + 2 * j);
    st16(tmem + ((uint32_t)(32 * warp) << 16) + 16 * cc, r);
  }
  wait_st();
}

__device__ void issue_qk_ss(Smem& sm, uint32_t d) {
  const uint32_t v0 = smem_u32(sm.v), q0 = smem_u32(sm.q);
  for (int s = 0; s < 32; ++s)
    mma_ss(d, desc(v0 + (s / 4) * (T * 128) + (s % 4) * 32, 16, 1024),
           desc(q0 + (s / 4) * (H * 128) + (s % 4) * 32, 16, 1024), idesc_f16(128, 16, 0), s > 0);
}
__device__ void issue_qk_ts(Smem& sm, uint32_t d, uint32_t a_tmem) {
  const uint32_t q0 = smem_u32(sm.q);
  for (int s = 0; s < 32; ++s)
    mma_ts(d, a_tmem + 8 * s, desc(q0 + (s / 4) * (H * 128) + (s % 4) * 32, 16, 1024), idesc_f16(128, 16, 0), s > 0);
}
__device__ void issue_pv_ss(Smem& sm, uint32_t d) {
  const uint32_t v0 = smem_u32(sm.v), p0 = smem_u32(sm.p);
  for (int j = 0; j < 4; ++j)
    for (int s = 0; s < 8; ++s)
      mma_ss(d + 16 * j, desc(v0 + 2 * j * (T * 128) + s * 2048, T * 128, 1024),
             desc(p0 + (s / 4) * (H * 128) + (s % 4) * 32, 16, 1024), idesc_f16(128, 16, 1), s > 0);
}

// TMEM columns: [0,256) A; [256,272) S ss; [272,288) S ts; [320,384) O^T
__global__ void __launch_bounds__(128, 1) check_kernel(const uint16_t* V, const uint16_t* Q, const uint16_t* P,
                                                       float* S_ss, float* S_ts, float* O, int* err) {
  extern __shared__ unsigned char raw[];
  Smem& sm = get_smem(raw);
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  if (tid == 0) { mbar_init(&sm.bar, 1); asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory"); }
  if (warp == 0) {
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(smem_u32(&sm.tmem)), "r"(512) : "memory");
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
  }
  fence_before();
  __syncthreads();
  fence_after();
  const uint32_t tm = sm.tmem;
  fill(sm, V, Q, P, tm);
  fence_async_smem();
  fence_before();
  __syncthreads();
  fence_after();
  if (tid == 0) {
    issue_qk_ss(sm, tm + 256);
    issue_qk_ts(sm, tm + 272, tm);
    issue_pv_ss(sm, tm + 320);
    commit(&sm.bar);
  }
  __syncwarp();
  const bool ok = mbar_wait(&sm.bar, 0);
  if (!ok && lane == 0) atomicExch(err, 1);
  fence_after();
  const int row = 32 * warp + lane;
  const uint32_t tl = tm + ((uint32_t)(32 * warp) << 16);
  uint32_t r[16];
  ld16(tl + 256, r); wait_ld();
  for (int h = 0; h < 16; ++h) S_ss[row * H + h] = __uint_as_float(r[h]);
  ld16(tl + 272, r); wait_ld();
  for (int h = 0; h < 16; ++h) S_ts[row * H + h] = __uint_as_float(r[h]);
  for (int j = 0; j < 4; ++j) {
    ld16(tl + 320 + 16 * j, r); wait_ld();
    for (int h = 0; h < 16; ++h) O[(128 * j + row) * H + h] = __uint_as_float(r[h]);  // O^T[dim][h]
  }
  fence_before();
  __syncthreads();
  if (warp == 0) {
    fence_after();
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tm), "r"(512) : "memory");
  }
}

// Timing: form 0 = QK ss, 1 = QK ts, 2 = PV ss; `reps` batches of 32 MMAs, one commit per batch.
__global__ void __launch_bounds__(128, 1) time_kernel(const uint16_t* V, const uint16_t* Q, const uint16_t* P,
                                                      int form, int reps, long long* cyc, int* err) {
  extern __shared__ unsigned char raw[];
  Smem& sm = get_smem(raw);
  const int tid = threadIdx.x, warp = tid >> 5;
  if (tid == 0) { mbar_init(&sm.bar, 1); asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory"); }
  if (warp == 0) {
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(smem_u32(&sm.tmem)), "r"(512) : "memory");
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
  }
  fence_before();
  __syncthreads();
  fence_after();
  const uint32_t tm = sm.tmem;
  fill(sm, V, Q, P, tm);
  fence_async_smem();
  fence_before();
  __syncthreads();
  fence_after();
  if (tid == 0) {
    long long t0 = clock64();
    uint32_t ph = 0;
    for (int r = 0; r < reps; ++r) {
      if (form == 0) issue_qk_ss(sm, tm + 256);
      else if (form == 1) issue_qk_ts(sm, tm + 272, tm);
      else issue_pv_ss(sm, tm + 320);
      commit(&sm.bar);
      if (!mbar_wait(&sm.bar, ph)) { atomicExch(err, 1); break; }
      ph ^= 1;
      fence_after();
    }
    cyc[blockIdx.x] = clock64() - t0;
  }
  fence_before();
  __syncthreads();
  if (warp == 0) {
    fence_after();
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tm), "r"(512) : "memory");
  }
}


// Sweep: 64 MMAs of M x N x 16 per batch (A = V dim-block 0 K-slices, B = 128 B-wide rows in the
// second half of sm.v), cycling over NACC accumulators of N columns each. Compile-time shapes and
// descriptors advanced by constants, so the issuing thread does little besides the MMAs.
template <int M, int N, int NACC, bool TS>
__global__ void __launch_bounds__(128, 1) sweep_kernel(const uint16_t* V, const uint16_t* Q, const uint16_t* P,
                                                       int reps, long long* cyc, int* err) {
  extern __shared__ unsigned char raw[];
  Smem& sm = get_smem(raw);
  const int tid = threadIdx.x, warp = tid >> 5;
  if (tid == 0) { mbar_init(&sm.bar, 1); asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory"); }
  if (warp == 0) {
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(smem_u32(&sm.tmem)), "r"(512) : "memory");
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
  }
  fence_before();
  __syncthreads();
  fence_after();
  const uint32_t tm = sm.tmem;
  fill(sm, V, Q, P, tm);
  fence_async_smem();
  fence_before();
  __syncthreads();
  fence_after();
  if (warp == 0) {
    const uint32_t v0 = smem_u32(sm.v), q0 = smem_u32(sm.v) + 65536;
    const uint64_t da = desc(v0, 16, 1024), db = desc(q0, 16, 1024);
    constexpr uint32_t id = idesc_f16(M, N, 0);
    const uint32_t d0 = tm + 256;  // accumulators in columns 256.. (A for TS in 0..255)
    long long t0 = clock64();
    uint32_t ph = 0;
    for (int r = 0; r < reps; ++r) {
      if (threadIdx.x == 0) {
#pragma unroll
        for (int s = 0; s < 64; ++s) {
          const uint32_t d = d0 + (uint32_t)((s % NACC) * N);
          if (TS) mma_ts(d, tm + 8 * (s % 32), db + 2 * (s % 4), id, s >= NACC);
          else mma_ss(d, da + 2 * (s % 4), db + 2 * (s % 4), id, s >= NACC);
        }
        commit(&sm.bar);
      }
      __syncwarp();
      if (!mbar_wait(&sm.bar, ph)) { if (threadIdx.x == 0) atomicExch(err, 1); break; }
      ph ^= 1;
      fence_after();
    }
    if (threadIdx.x == 0) cyc[blockIdx.x] = clock64() - t0;
  }
  fence_before();
  __syncthreads();
  if (warp == 0) {
    fence_after();
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tm), "r"(512) : "memory");
  }
}

template <int M, int N, int NACC, bool TS>
void run_sweep(const uint16_t* dV, const uint16_t* dQ, const uint16_t* dP, long long* dCyc, int* dErr, int sms) {
  cudaFuncSetAttribute(sweep_kernel<M, N, NACC, TS>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)kSmem);
  const int reps = 32;
  sweep_kernel<M, N, NACC, TS><<<sms, 128, kSmem>>>(dV, dQ, dP, reps, dCyc, dErr);
  sweep_kernel<M, N, NACC, TS><<<sms, 128, kSmem>>>(dV, dQ, dP, reps, dCyc, dErr);
  cudaError_t e = cudaDeviceSynchronize();
  std::vector<long long> cv(sms);
  cudaMemcpy(cv.data(), dCyc, sms * 8, cudaMemcpyDeviceToHost);
  double mean = 0;
  for (long long x : cv) mean += x;
  mean /= sms;
  const double per = mean / reps / 64;
  printf("%s M=%3d N=%3d acc=%2d: %7.2f cycles per MMA, %7.1f MAC/clk  %s\n", TS ? "ts" : "ss", M, N, NACC, per,
         (double)M * N * 16 / per, cudaGetErrorString(e));
}

// ISSUERS warps each issue 64 MMAs (M=128, N=16) per batch into their own accumulator and commit
// to their own barrier.
template <int ISSUERS>
__global__ void __launch_bounds__(128, 1) multi_kernel(const uint16_t* V, const uint16_t* Q, const uint16_t* P,
                                                       int reps, long long* cyc, int* err) {
  extern __shared__ unsigned char raw[];
  Smem& sm = get_smem(raw);
  __shared__ uint64_t bars[4];
  const int tid = threadIdx.x, warp = tid >> 5;
  if (tid == 0) {
    for (int i = 0; i < 4; ++i) mbar_init(&bars[i], 1);
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
  }
  if (warp == 0) {
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(smem_u32(&sm.tmem)), "r"(512) : "memory");
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
  }
  fence_before();
  __syncthreads();
  fence_after();
  const uint32_t tm = sm.tmem;
  fill(sm, V, Q, P, tm);
  fence_async_smem();
  fence_before();
  __syncthreads();
  fence_after();
  if (warp < ISSUERS) {
    const uint32_t v0 = smem_u32(sm.v), q0 = smem_u32(sm.v) + 65536;
    const uint64_t da = desc(v0, 16, 1024), db = desc(q0, 16, 1024);
    constexpr uint32_t id = idesc_f16(128, 16, 0);
    const uint32_t d0 = tm + 256 + 16 * warp;
    long long t0 = clock64();
    uint32_t ph = 0;
    for (int r = 0; r < reps; ++r) {
      if ((threadIdx.x & 31) == 0) {
#pragma unroll
        for (int s = 0; s < 64; ++s) mma_ss(d0, da + 2 * (s % 4), db + 2 * (s % 4), id, s > 0);
        commit(&bars[warp]);
      }
      __syncwarp();
      if (!mbar_wait(&bars[warp], ph)) { if ((threadIdx.x & 31) == 0) atomicExch(err, 1); break; }
      ph ^= 1;
      fence_after();
    }
    if ((threadIdx.x & 31) == 0) cyc[blockIdx.x * 4 + warp] = clock64() - t0;
  }
  fence_before();
  __syncthreads();
  if (warp == 0) {
    fence_after();
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tm), "r"(512) : "memory");
  }
}

template <int ISSUERS>
void run_multi(const uint16_t* dV, const uint16_t* dQ, const uint16_t* dP, long long* dCyc, int* dErr, int sms) {
  cudaFuncSetAttribute(multi_kernel<ISSUERS>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)kSmem);
  const int reps = 32;
  multi_kernel<ISSUERS><<<sms, 128, kSmem>>>(dV, dQ, dP, reps, dCyc, dErr);
  multi_kernel<ISSUERS><<<sms, 128, kSmem>>>(dV, dQ, dP, reps, dCyc, dErr);
  cudaError_t e = cudaDeviceSynchronize();
  std::vector<long long> cv(sms * 4);
  cudaMemcpy(cv.data(), dCyc, sms * 4 * 8, cudaMemcpyDeviceToHost);
  double mx = 0;
  for (int b = 0; b < sms; ++b) for (int w = 0; w < ISSUERS; ++w) mx += cv[b * 4 + w];
  mx /= sms * ISSUERS;
  const double per_sm = mx / reps / (64.0 * ISSUERS);  // cycles per MMA per SM (all issuers)
  printf("issuers %d: %7.2f cycles per MMA per issuer, %7.2f per SM -> %7.1f MAC/clk/SM  %s\n", ISSUERS,
         mx / reps / 64, per_sm, 128.0 * 16 * 16 / per_sm, cudaGetErrorString(e));
}

// Concurrency: warp 0 (lane 0) issues tcgen05 M=128 N=16 chains when `tc` is set; warps 1..7 run
// independent mma.sync m16n8k16 chains when `hm` is set. Cycles per side reported.
__global__ void __launch_bounds__(256, 1) conc_kernel(const uint16_t* V, const uint16_t* Q, const uint16_t* P,
                                                      int tc, int hm, int reps, long long* cyc, float* sink, int* err) {
  extern __shared__ unsigned char raw[];
  Smem& sm = get_smem(raw);
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  if (tid == 0) { mbar_init(&sm.bar, 1); asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory"); }
  if (warp == 0) {
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(smem_u32(&sm.tmem)), "r"(512) : "memory");
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
  }
  fence_before();
  __syncthreads();
  fence_after();
  const uint32_t tm = sm.tmem;
  if (warp < 4) fill(sm, V, Q, P, tm);
  fence_async_smem();
  fence_before();
  __syncthreads();
  fence_after();
  if (warp == 0) {
    if (tc) {
      const uint32_t v0 = smem_u32(sm.v), q0 = smem_u32(sm.v) + 65536;
      const uint64_t da = desc(v0, 16, 1024), db = desc(q0, 16, 1024);
      constexpr uint32_t id = idesc_f16(128, 16, 0);
      long long t0 = clock64();
      uint32_t ph = 0;
      for (int r = 0; r < reps; ++r) {
        if (lane == 0) {
#pragma unroll
          for (int s = 0; s < 64; ++s) mma_ss(tm + 256, da + 2 * (s % 4), db + 2 * (s % 4), id, s > 0);
          commit(&sm.bar);
        }
        __syncwarp();
        if (!mbar_wait(&sm.bar, ph)) { if (lane == 0) atomicExch(err, 1); break; }
        ph ^= 1;
        fence_after();
      }
      if (lane == 0) cyc[blockIdx.x * 2] = clock64() - t0;
    }
  } else if (hm) {
    float acc[8][4] = {};
    uint32_t a0 = 0x3C003C00u + lane, a1 = a0 ^ 1, a2 = a0 ^ 2, a3 = a0 ^ 3, b0 = 0x38003800u + warp, b1 = b0 ^ 5;
    long long t0 = clock64();
    for (int r = 0; r < reps * 8; ++r) {
#pragma unroll
      for (int i = 0; i < 8; ++i)
        asm volatile("mma.sync.aligned.m16n8k16.row.col.f32.f16.f16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, {%0,%1,%2,%3};"
                     : "+f"(acc[i][0]), "+f"(acc[i][1]), "+f"(acc[i][2]), "+f"(acc[i][3])
                     : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
    }
    long long t1 = clock64();
    float s = 0;
    for (int i = 0; i < 8; ++i) s += acc[i][0] + acc[i][3];
    sink[blockIdx.x * 256 + tid] = s;
    if (warp == 1 && lane == 0) cyc[blockIdx.x * 2 + 1] = t1 - t0;
  }
  fence_before();
  __syncthreads();
  if (warp == 0) {
    fence_after();
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tm), "r"(512) : "memory");
  }
}

void run_conc(const uint16_t* dV, const uint16_t* dQ, const uint16_t* dP, long long* dCyc, float* dSink, int* dErr, int sms) {
  cudaFuncSetAttribute(conc_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)kSmem);
  const int reps = 32;
  for (int mode = 1; mode <= 3; ++mode) {
    const int tc = mode & 1, hm = (mode >> 1) & 1;
    cudaMemset(dCyc, 0, 1024 * 8);
    conc_kernel<<<sms, 256, kSmem>>>(dV, dQ, dP, tc, hm, reps, dCyc, dSink, dErr);
    conc_kernel<<<sms, 256, kSmem>>>(dV, dQ, dP, tc, hm, reps, dCyc, dSink, dErr);
    cudaError_t e = cudaDeviceSynchronize();
    std::vector<long long> cv(sms * 2);
    cudaMemcpy(cv.data(), dCyc, sms * 2 * 8, cudaMemcpyDeviceToHost);
    double t_tc = 0, t_hm = 0;
    for (int b = 0; b < sms; ++b) { t_tc += cv[2 * b]; t_hm += cv[2 * b + 1]; }
    t_tc /= sms; t_hm /= sms;
    const double tc_rate = tc ? (reps * 64.0 * 128 * 16 * 16) / t_tc : 0;      // MAC/clk/SM
    const double hm_rate = hm ? (reps * 8.0 * 8 * 7 * 2048) / t_hm : 0;         // 7 warps x mma
    printf("conc tc=%d hm=%d: tcgen05 %7.1f MAC/clk/SM, mma.sync %7.1f MAC/clk/SM (%.3f mma/clk/SM)  %s\n", tc, hm,
           tc_rate, hm_rate, hm_rate / 2048, cudaGetErrorString(e));
  }
}

static uint16_t h16(float f) { __half h = __float2half(f); uint16_t u; memcpy(&u, &h, 2); return u; }

int main() {
  std::vector<uint16_t> V(T * D), Q(H * D), P(H * T);
  std::vector<float> Vf(T * D), Qf(H * D), Pf(H * T);
  uint32_t s = 12345;
  auto rnd = [&]() { s = s * 1664525u + 1013904223u; return (int)((s >> 16) & 15) - 8; };
  for (int i = 0; i < T * D; ++i) { Vf[i] = rnd() / 8.0f; V[i] = h16(Vf[i]); }
  for (int i = 0; i < H * D; ++i) { Qf[i] = rnd() / 8.0f; Q[i] = h16(Qf[i]); }
  for (int i = 0; i < H * T; ++i) { Pf[i] = rnd() / 8.0f; P[i] = h16(Pf[i]); }
  uint16_t *dV, *dQ, *dP; float *dS1, *dS2, *dO; int* dErr; long long* dCyc;
  cudaMalloc(&dV, V.size() * 2); cudaMalloc(&dQ, Q.size() * 2); cudaMalloc(&dP, P.size() * 2);
  cudaMalloc(&dS1, T * H * 4); cudaMalloc(&dS2, T * H * 4); cudaMalloc(&dO, D * H * 4);
  cudaMalloc(&dErr, 4); cudaMalloc(&dCyc, 1024 * 8);
  cudaMemset(dErr, 0, 4);
  cudaMemcpy(dV, V.data(), V.size() * 2, cudaMemcpyHostToDevice);
  cudaMemcpy(dQ, Q.data(), Q.size() * 2, cudaMemcpyHostToDevice);
  cudaMemcpy(dP, P.data(), P.size() * 2, cudaMemcpyHostToDevice);
  cudaFuncSetAttribute(check_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)kSmem);
  cudaFuncSetAttribute(time_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)kSmem);
  check_kernel<<<1, 128, kSmem>>>(dV, dQ, dP, dS1, dS2, dO, dErr);
  cudaError_t e = cudaDeviceSynchronize();
  printf("check: %s\n", cudaGetErrorString(e));
  if (e != cudaSuccess) return 1;
  std::vector<float> S1(T * H), S2(T * H), O(D * H);
  int herr = 0;
  cudaMemcpy(S1.data(), dS1, T * H * 4, cudaMemcpyDeviceToHost);
  cudaMemcpy(S2.data(), dS2, T * H * 4, cudaMemcpyDeviceToHost);
  cudaMemcpy(O.data(), dO, D * H * 4, cudaMemcpyDeviceToHost);
  cudaMemcpy(&herr, dErr, 4, cudaMemcpyDeviceToHost);
  int bad1 = 0, bad2 = 0, bad3 = 0;
  for (int i = 0; i < T; ++i)
    for (int h = 0; h < H; ++h) {
      double acc = 0;
      for (int d = 0; d < D; ++d) acc += (double)Vf[i * D + d] * Qf[h * D + d];
      if (S1[i * H + h] != (float)acc) { if (bad1 < 4) printf("ss S[%d][%d] = %g want %g\n", i, h, S1[i * H + h], acc); ++bad1; }
      if (S2[i * H + h] != (float)acc) { if (bad2 < 4) printf("ts S[%d][%d] = %g want %g\n", i, h, S2[i * H + h], acc); ++bad2; }
    }
  for (int d = 0; d < D; ++d)
    for (int h = 0; h < H; ++h) {
      double acc = 0;
      for (int i = 0; i < T; ++i) acc += (double)Vf[i * D + d] * Pf[h * T + i];
      if (O[d * H + h] != (float)acc) { if (bad3 < 4) printf("pv O[%d][%d] = %g want %g\n", d, h, O[d * H + h], acc); ++bad3; }
    }
  printf("mismatches: qk_ss %d  qk_ts %d  pv_ss %d  (of %d, %d, %d)  wait_err %d\n", bad1, bad2, bad3, T * H, T * H, D * H, herr);
  if (bad1 || bad2 || bad3 || herr) return 2;
  int sms = 0;
  cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, 0);
  const char* names[3] = {"QK ss (A=V smem)", "QK ts (A=V tmem)", "PV ss (A=V^T smem MN)"};
  for (int form = 0; form < 3; ++form)
    for (int grid : {1, sms}) {
      const int reps = 64;
      time_kernel<<<grid, 128, kSmem>>>(dV, dQ, dP, form, reps, dCyc, dErr);
      time_kernel<<<grid, 128, kSmem>>>(dV, dQ, dP, form, reps, dCyc, dErr);
      e = cudaDeviceSynchronize();
      std::vector<long long> c(grid);
      cudaMemcpy(c.data(), dCyc, grid * 8, cudaMemcpyDeviceToHost);
      double mean = 0;
      for (long long x : c) mean += x;
      mean /= grid;
      printf("%-24s grid %3d: %8.1f cycles per 32 MMAs (%.2f per MMA, M=128 N=16 K=16) -> %.2f cycles per item  %s\n",
             names[form], grid, mean / reps, mean / reps / 32, mean / reps / 128, cudaGetErrorString(e));
    }

  float* dSink; cudaMalloc(&dSink, 1024 * 256 * 4);
  run_conc(dV, dQ, dP, dCyc, dSink, dErr, sms);
  run_multi<1>(dV, dQ, dP, dCyc, dErr, sms);
  run_multi<2>(dV, dQ, dP, dCyc, dErr, sms);
  run_multi<4>(dV, dQ, dP, dCyc, dErr, sms);
  run_sweep<128, 16, 1, false>(dV, dQ, dP, dCyc, dErr, sms);
  run_sweep<128, 16, 2, false>(dV, dQ, dP, dCyc, dErr, sms);
  run_sweep<128, 16, 4, false>(dV, dQ, dP, dCyc, dErr, sms);
  run_sweep<128, 16, 8, false>(dV, dQ, dP, dCyc, dErr, sms);
  run_sweep<128, 16, 1, true>(dV, dQ, dP, dCyc, dErr, sms);
  run_sweep<128, 16, 4, true>(dV, dQ, dP, dCyc, dErr, sms);
  run_sweep<128, 32, 1, false>(dV, dQ, dP, dCyc, dErr, sms);
  run_sweep<128, 32, 4, false>(dV, dQ, dP, dCyc, dErr, sms);
  run_sweep<128, 64, 1, false>(dV, dQ, dP, dCyc, dErr, sms);
  run_sweep<128, 64, 4, false>(dV, dQ, dP, dCyc, dErr, sms);
  run_sweep<128, 128, 1, false>(dV, dQ, dP, dCyc, dErr, sms);
  run_sweep<128, 256, 1, false>(dV, dQ, dP, dCyc, dErr, sms);
  run_sweep<64, 16, 1, false>(dV, dQ, dP, dCyc, dErr, sms);
  run_sweep<64, 16, 4, false>(dV, dQ, dP, dCyc, dErr, sms);
  run_sweep<64, 64, 4, false>(dV, dQ, dP, dCyc, dErr, sms);
  cudaMemcpy(&herr, dErr, 4, cudaMemcpyDeviceToHost);
  printf("wait_err %d\n", herr);
  return herr ? 3 : 0;
}

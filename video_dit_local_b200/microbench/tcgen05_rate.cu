// tcgen05.mma issue-rate micro-benchmark (sm_100a): cycles per instruction
// of kind::f16 MMAs with M = 128 (one CTA per SM, one issuing thread), as a
// function of N, operand source (A from shared memory or TMEM), B major-ness,
// concurrent TMEM traffic from other warps, and the barrier operations placed
// between groups of 16 MMAs; the CTA-pair form (cta_group::2, M = 256); and
// whether a second CTA per SM, with its own issuing thread, covers the pauses
// one issuing thread leaves between MMA groups.
//
// Build and run on one B200:
//   nvcc -gencode arch=compute_100a,code=sm_100a -O3 -std=c++17 \
//        -I video_dit_local_b200/csrc -o /tmp/tcgen05_rate \
//        video_dit_local_b200/microbench/tcgen05_rate.cu && /tmp/tcgen05_rate
//
// Operands are random bf16 in +-[0.5, 1); results are not read.  Every wait is
// bounded by %globaltimer (2 s) and reported through an error word.
#include <cuda.h>

#include <algorithm>
#include <cstdint>
#include <cstdio>
#include <cstdlib>
#include <vector>

#include "common.cuh"

using namespace vattn;

namespace {

struct Res {
  long long cyc, ns;
};

__device__ __forceinline__ uint32_t hash32(uint32_t x) {
  x ^= x >> 16;
  x *= 0x7feb352dU;
  x ^= x >> 15;
  x *= 0x846ca68bU;
  x ^= x >> 16;
  return x;
}
// two bf16 in +-[0.5, 1): random sign and 7-bit mantissa, exponent 126
__device__ __forceinline__ uint32_t rand_bf16x2(uint32_t i) {
  const uint32_t h = hash32(i * 2654435761u + 12345u);
  const uint32_t lo = ((h & 1u) << 15) | (126u << 7) | ((h >> 1) & 0x7Fu);
  const uint32_t hi = (((h >> 8) & 1u) << 15) | (126u << 7) | ((h >> 9) & 0x7Fu);
  return lo | (hi << 16);
}

__device__ __forceinline__ bool bounded_wait(uint64_t* bar, uint32_t parity) {
  const uint64_t lim = globaltimer_ns() + 2000000000ull;
  bool ok;
  while (!(ok = mbar_try_wait(bar, parity)) && globaltimer_ns() < lim) {
  }
  return ok;
}

// Shared memory (1024-aligned): A 32 KB at 0 (128 rows x K=128, two 64-column
// swizzle boxes), B 32 KB at 32 KB.  TMEM: D in columns [0, 256), A for the
// TMEM-operand form in [256, 320), other warps' traffic in [384, 512).
//   TS:   A from TMEM (else shared memory)
//   BMN:  B MN-major (else K-major)
//   LOAD: warps 1..4 load and store TMEM columns [384, 512) until the MMAs end
//   SYNC: per 16 MMAs, 3 commits + 2 fence::after_thread_sync + 2 try_waits on
//         a completed barrier (the attention kernel's per-block pattern)
template <int N, int TS, int BMN, int LOAD, int SYNC>
__global__ void __launch_bounds__(160, 1) rate_kernel(Res* out, int iters, int* err) {
  extern __shared__ uint8_t raw[];
  __shared__ uint64_t bar, cb[3], done_bar;
  __shared__ uint32_t tbase;
  __shared__ volatile int done;
  const uint32_t base = (smem_u32(raw) + 1023u) & ~1023u;
  uint8_t* p = raw + (base - smem_u32(raw));
  for (int i = threadIdx.x; i < (64 * 1024) / 4; i += blockDim.x)
    reinterpret_cast<uint32_t*>(p)[i] = rand_bf16x2(i + blockIdx.x * 77777u);
  const int warp = threadIdx.x / 32, lane = threadIdx.x & 31;
  if (threadIdx.x == 0) {
    mbar_init(&bar, 1);
    for (int i = 0; i < 3; ++i) mbar_init(&cb[i], 1);
    mbar_init(&done_bar, 1);
    fence_mbar_init();
    done = 0;
  }
  if (warp == 0) {
    tmem_alloc(&tbase, 512);
    tmem_relinquish();
  }
  asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tm = tbase;
  if (warp < 4) {  // A operand in TMEM: 128 lanes x 64 columns (K = 128 bf16)
    uint32_t r[32];
    for (int c = 0; c < 2; ++c) {
      for (int i = 0; i < 32; ++i) r[i] = rand_bf16x2(threadIdx.x * 64 + c * 32 + i);
      tmem_st32(tm + ((uint32_t)(32 * warp) << 16) + 256 + 32 * c, r);
    }
    tmem_wait_st();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == 0 && lane == 0) {
    mbar_arrive(&done_bar);  // one completed phase to poll
    constexpr uint32_t idesc = idesc_bf16_f32(128, N, 0, BMN);
    const uint32_t a_s = base, b_s = base + 32768;
    uint32_t spins = 0;
    const long long t0 = clock64();
    const uint64_t g0 = globaltimer_ns();
    for (int it = 0; it < iters; ++it) {
      for (int half = 0; half < 2; ++half) {
        if (SYNC) {
          spins += !mbar_try_wait(&done_bar, 0);
          tc_fence_after();
        }
#pragma unroll
        for (int kk = 0; kk < 8; ++kk) {
          const uint32_t koff = (kk & 3) * 32 + (kk >> 2) * 16384;
          // MN-major B: 64-column boxes 8 KB apart (K = 64 rows), K step = 16 rows
          const uint64_t bd = BMN ? smem_desc_sw128(b_s + (kk & 3) * 2048, 8192, 1024)
                                  : smem_desc_sw128(b_s + koff, 16, 1024);
          if (TS)
            mma_ts(tm + (uint32_t)(half * 0), tm + 256 + kk * 8, bd, idesc, (it | half | kk) != 0);
          else
            mma_ss(tm, smem_desc_sw128(a_s + koff, 16, 1024), bd, idesc, (it | half | kk) != 0);
        }
        if (SYNC) {
          tc_commit(&cb[half]);
          if (half) tc_commit(&cb[2]);
        }
      }
    }
    tc_commit(&bar);
    const bool ok = bounded_wait(&bar, 0);
    const long long t1 = clock64();
    const uint64_t g1 = globaltimer_ns();
    if (!ok || spins) atomicExch(err, 1);
    out[blockIdx.x].cyc = t1 - t0;
    out[blockIdx.x].ns = (long long)(g1 - g0);
    done = 1;
  }
  if (LOAD && warp >= 1) {  // warp w may access TMEM lanes 32 * (w % 4)
    const uint32_t lane_base = (uint32_t)(32 * (warp & 3)) << 16;
    uint32_t acc = 0;
    for (int n = 0; n < 2000000 && !done; ++n) {
      uint32_t r[32];
      tmem_ld32(tm + lane_base + 384 + 32 * (n & 3), r);
      tmem_wait_ld();
      for (int i = 0; i < 32; ++i) acc += r[i];
      tmem_st32(tm + lane_base + 384 + 32 * ((n + 2) & 3), r);
      tmem_wait_st();
    }
    if (acc == 0x12345678u) atomicExch(err, 2);
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == 0) tmem_dealloc(tm, 512);
}

__device__ __forceinline__ uint32_t cluster_rank() {
  uint32_t r;
  asm volatile("mov.u32 %0, %%cluster_ctarank;" : "=r"(r));
  return r;
}
__device__ __forceinline__ void cluster_sync_all() {
  asm volatile("barrier.cluster.arrive.release.aligned;\n\tbarrier.cluster.wait.acquire.aligned;" ::: "memory");
}

// CTA pair (cta_group::2): M = 256, each CTA holds 128 rows of A and N/2 rows
// of B (K-major); the leader issues, a multicast commit reaches both CTAs.
template <int N>
__global__ void __cluster_dims__(2, 1, 1) __launch_bounds__(128) pair_kernel(Res* out, int iters, int* err) {
  extern __shared__ uint8_t raw[];
  __shared__ uint64_t bar;
  __shared__ uint32_t tbase;
  const uint32_t base = (smem_u32(raw) + 1023u) & ~1023u;
  uint8_t* p = raw + (base - smem_u32(raw));
  for (int i = threadIdx.x; i < (48 * 1024) / 4; i += blockDim.x)
    reinterpret_cast<uint32_t*>(p)[i] = rand_bf16x2(i + blockIdx.x * 77777u);
  const int warp = threadIdx.x / 32;
  const uint32_t rank = cluster_rank();
  if (threadIdx.x == 0) {
    mbar_init(&bar, 1);
    fence_mbar_init();
  }
  if (warp == 0) {
    asm volatile("tcgen05.alloc.cta_group::2.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(smem_u32(&tbase)),
                 "r"(512)
                 : "memory");
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::2.sync.aligned;" ::: "memory");
  }
  asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
  tc_fence_before();
  __syncthreads();
  cluster_sync_all();
  tc_fence_after();
  const uint32_t tm = tbase;
  const uint32_t a_s = base, b_s = base + 16384;
  if (threadIdx.x == 0) {
    const long long t0 = clock64();
    const uint64_t g0 = globaltimer_ns();
    if (rank == 0) {
      constexpr uint32_t idesc = idesc_bf16_f32(256, N, 0, 0);
      for (int it = 0; it < iters; ++it) {
#pragma unroll
        for (int kk = 0; kk < 4; ++kk) {
          const uint32_t acc = (it | kk) != 0;
          asm volatile(
              "{\n\t.reg .pred p;\n\tsetp.ne.b32 p, %4, 0;\n\t"
              "tcgen05.mma.cta_group::2.kind::f16 [%0], %1, %2, %3, p;\n\t}" ::"r"(tm),
              "l"(smem_desc_sw128(a_s + kk * 32, 16, 1024)), "l"(smem_desc_sw128(b_s + kk * 32, 16, 1024)),
              "r"(idesc), "r"(acc)
              : "memory");
        }
      }
      asm volatile(
          "tcgen05.commit.cta_group::2.mbarrier::arrive::one.shared::cluster.multicast::cluster.b64 [%0], %1;" ::"r"(
              smem_u32(&bar)),
          "h"((uint16_t)3)
          : "memory");
    }
    const bool ok = bounded_wait(&bar, 0);
    const long long t1 = clock64();
    const uint64_t g1 = globaltimer_ns();
    if (!ok) atomicExch(err, 3);
    if (rank == 0) {
      out[blockIdx.x / 2].cyc = t1 - t0;
      out[blockIdx.x / 2].ns = (long long)(g1 - g0);
    }
  }
  tc_fence_before();
  __syncthreads();
  cluster_sync_all();
  tc_fence_after();
  if (warp == 0) asm volatile("tcgen05.dealloc.cta_group::2.sync.aligned.b32 %0, %1;" ::"r"(tm), "r"(512) : "memory");
}

// Per CTA: 256 TMEM columns (S/P at 0, O at 128) and 96 KB of shared memory,
// so two CTAs fit on one SM.  Groups of 8 TMEM x SMEM + 8 SMEM x SMEM MMAs
// (the attention forward's per-block pattern), then `pause` idle cycles.
__global__ void __launch_bounds__(128, 2) two_cta_kernel(Res* out, int iters, int pause, int* err) {
  extern __shared__ uint8_t raw[];
  __shared__ uint64_t bar;
  __shared__ uint32_t tbase;
  const uint32_t base = (smem_u32(raw) + 1023u) & ~1023u;
  uint8_t* p = raw + (base - smem_u32(raw));
  for (int i = threadIdx.x; i < (96 * 1024) / 4; i += blockDim.x)
    reinterpret_cast<uint32_t*>(p)[i] = rand_bf16x2(i + blockIdx.x * 77777u);
  const int warp = threadIdx.x / 32, lane = threadIdx.x & 31;
  if (threadIdx.x == 0) {
    mbar_init(&bar, 1);
    fence_mbar_init();
  }
  if (warp == 0) {
    tmem_alloc(&tbase, 256);
    tmem_relinquish();
  }
  asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tm = tbase;
  {
    uint32_t r[32];
    for (int c = 0; c < 4; ++c) {
      for (int i = 0; i < 32; ++i) r[i] = rand_bf16x2(threadIdx.x * 128 + c * 32 + i);
      tmem_st32(tm + ((uint32_t)(32 * warp) << 16) + 32 * c, r);
    }
    tmem_wait_st();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == 0 && lane == 0) {
    constexpr uint32_t IQK = idesc_bf16_f32(128, 128, 0, 0);
    constexpr uint32_t IPV = idesc_bf16_f32(128, 128, 0, 1);
    const uint32_t q_s = base, k_s = base + 32768, v_s = base + 65536;
    const long long t0 = clock64();
    const uint64_t g0 = globaltimer_ns();
    for (int it = 0; it < iters; ++it) {
#pragma unroll
      for (int kk = 0; kk < 8; ++kk)
        mma_ts(tm + 128, tm + kk * 8, smem_desc_sw128(v_s + kk * 2048, 16384, 1024), IPV, 1);
#pragma unroll
      for (int kk = 0; kk < 8; ++kk) {
        const uint32_t off = (kk >> 2) * 16384 + (kk & 3) * 32;
        mma_ss(tm, smem_desc_sw128(q_s + off, 16, 1024), smem_desc_sw128(k_s + off, 16, 1024), IQK, kk > 0);
      }
      const long long s0 = clock64();
      while (clock64() - s0 < pause) {
      }
    }
    tc_commit(&bar);
    const bool ok = bounded_wait(&bar, 0);
    const long long t1 = clock64();
    const uint64_t g1 = globaltimer_ns();
    if (!ok) atomicExch(err, 4);
    out[blockIdx.x].cyc = t1 - t0;
    out[blockIdx.x].ns = (long long)(g1 - g0);
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == 0) tmem_dealloc(tm, 256);
}

void report(const char* name, const std::vector<Res>& h, double instrs, double flop_per_sm_instr, int herr) {
  std::vector<double> c;
  double ghz = 0;
  for (const Res& r : h) {
    c.push_back((double)r.cyc / instrs);
    ghz += (double)r.cyc / (double)r.ns / (double)h.size();
  }
  std::sort(c.begin(), c.end());
  const double med = c[c.size() / 2];
  printf("%-40s cycles/MMA median %6.1f (min %6.1f max %6.1f)  FLOP/cycle/SM %5.0f  clock %.2f GHz  err %d\n", name,
         med, c.front(), c.back(), flop_per_sm_instr / med, ghz, herr);
}

template <int N, int TS, int BMN, int LOAD, int SYNC>
void run(const char* name, Res* d_out, int* d_err) {
  auto k = rate_kernel<N, TS, BMN, LOAD, SYNC>;
  const int smem = 120 * 1024;  // one CTA per SM
  cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
  const int iters = 128;
  for (int rep = 0; rep < 3; ++rep) {
    k<<<148, 160, smem>>>(d_out, iters, d_err);
    const cudaError_t e = cudaDeviceSynchronize();
    if (e != cudaSuccess) {
      printf("%s: %s\n", name, cudaGetErrorString(e));
      exit(1);
    }
  }
  std::vector<Res> h(148);
  int herr = 0;
  cudaMemcpy(&herr, d_err, 4, cudaMemcpyDeviceToHost);
  cudaMemcpy(h.data(), d_out, h.size() * sizeof(Res), cudaMemcpyDeviceToHost);
  report(name, h, iters * 16.0, 2.0 * 128 * N * 16, herr);
}

template <int N>
void run_pair(const char* name, Res* d_out, int* d_err) {
  auto k = pair_kernel<N>;
  const int smem = 120 * 1024;
  cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
  const int iters = 256;
  for (int rep = 0; rep < 3; ++rep) {
    k<<<148, 128, smem>>>(d_out, iters, d_err);
    const cudaError_t e = cudaDeviceSynchronize();
    if (e != cudaSuccess) {
      printf("%s: %s\n", name, cudaGetErrorString(e));
      exit(1);
    }
  }
  std::vector<Res> h(74);
  int herr = 0;
  cudaMemcpy(&herr, d_err, 4, cudaMemcpyDeviceToHost);
  cudaMemcpy(h.data(), d_out, h.size() * sizeof(Res), cudaMemcpyDeviceToHost);
  report(name, h, iters * 4.0, 2.0 * 256 * N * 16 / 2, herr);  // per-SM share of one pair MMA
}

}  // namespace

int main() {
  Res* d_out;
  int* d_err;
  cudaMalloc(&d_out, 148 * sizeof(Res));
  cudaMalloc(&d_err, 4);
  cudaMemset(d_err, 0, 4);
  run<64, 0, 0, 0, 0>("SMEMxSMEM N=64", d_out, d_err);
  run<128, 0, 0, 0, 0>("SMEMxSMEM N=128", d_out, d_err);
  run<256, 0, 0, 0, 0>("SMEMxSMEM N=256", d_out, d_err);
  run<128, 0, 1, 0, 0>("SMEMxSMEM N=128, B MN-major", d_out, d_err);
  run<64, 1, 0, 0, 0>("TMEMxSMEM N=64", d_out, d_err);
  run<128, 1, 1, 0, 0>("TMEMxSMEM N=128, B MN-major", d_out, d_err);
  run<256, 1, 1, 0, 0>("TMEMxSMEM N=256, B MN-major", d_out, d_err);
  run<128, 0, 0, 1, 0>("SMEMxSMEM N=128 + TMEM ld/st warps", d_out, d_err);
  run<128, 1, 1, 1, 0>("TMEMxSMEM N=128 + TMEM ld/st warps", d_out, d_err);
  run<128, 0, 0, 0, 1>("SMEMxSMEM N=128 + per-16 sync ops", d_out, d_err);
  run<128, 1, 1, 0, 1>("TMEMxSMEM N=128 + per-16 sync ops", d_out, d_err);
  run_pair<128>("CTA pair M=256 N=128 (per SM)", d_out, d_err);
  run_pair<256>("CTA pair M=256 N=256 (per SM)", d_out, d_err);
  // one or two CTAs per SM, each pausing between 16-MMA groups
  Res* d_out2;
  cudaMalloc(&d_out2, 296 * sizeof(Res));
  const int smem2 = 100 * 1024;
  cudaFuncSetAttribute(two_cta_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, smem2);
  for (int pause : {0, 400, 800}) {
    for (int per_sm = 1; per_sm <= 2; ++per_sm) {
      const int ctas = 148 * per_sm, iters = 256;
      for (int rep = 0; rep < 3; ++rep) {
        two_cta_kernel<<<ctas, 128, smem2>>>(d_out2, iters, pause, d_err);
        const cudaError_t e = cudaDeviceSynchronize();
        if (e != cudaSuccess) {
          printf("two_cta: %s\n", cudaGetErrorString(e));
          return 1;
        }
      }
      std::vector<Res> h(ctas);
      int herr = 0;
      cudaMemcpy(&herr, d_err, 4, cudaMemcpyDeviceToHost);
      cudaMemcpy(h.data(), d_out2, h.size() * sizeof(Res), cudaMemcpyDeviceToHost);
      std::vector<double> c;
      for (const Res& r : h) c.push_back((double)r.cyc / iters);
      std::sort(c.begin(), c.end());
      const double med = c[c.size() / 2];
      printf("pause %3d cycles, %d CTA(s) per SM: %6.1f cycles per 16-MMA group and CTA, tensor pipe busy %5.1f%%  err %d\n",
             pause, per_sm, med, 100.0 * per_sm * 16 * 64.2 / med, herr);
    }
  }
  return 0;
}

// Sustained tcgen05.mma.cta_group::2 rate (M = 256 split over the two SMs of
// a cluster pair; the leader issues, one commit to each CTA's barrier) for
// SS 256x128x16, SS 256x256x16 and TS 256x128x16, to compare the per-SM rate
// of paired MMAs with the single-SM shapes of umma_rate.cu.
#include <cstdio>
#include <cuda_runtime.h>
#include "../csrc/apb_internal.h"
#include "../csrc/sm100_ptx.cuh"
using namespace apb;

__device__ __forceinline__ uint32_t cluster_rank() { uint32_t r; asm volatile("mov.u32 %0, %%cluster_ctarank;" : "=r"(r)); return r; }
__device__ __forceinline__ void cluster_sync() {
  asm volatile("barrier.cluster.arrive.release.aligned;\n\tbarrier.cluster.wait.acquire.aligned;" ::: "memory");
}
__device__ __forceinline__ void umma2_ss(uint32_t d, uint64_t a, uint64_t b, uint32_t idesc, uint32_t acc) {
  asm volatile("{\n\t.reg .pred p;\n\tsetp.ne.b32 p, %4, 0;\n\t"
               "tcgen05.mma.cta_group::2.kind::f16 [%0], %1, %2, %3, p;\n\t}"
               :: "r"(d), "l"(a), "l"(b), "r"(idesc), "r"(acc) : "memory");
}
__device__ __forceinline__ void umma2_ts(uint32_t d, uint32_t a, uint64_t b, uint32_t idesc, uint32_t acc) {
  asm volatile("{\n\t.reg .pred p;\n\tsetp.ne.b32 p, %4, 0;\n\t"
               "tcgen05.mma.cta_group::2.kind::f16 [%0], [%1], %2, %3, p;\n\t}"
               :: "r"(d), "r"(a), "l"(b), "r"(idesc), "r"(acc) : "memory");
}

// mode 0: SS M256 N128 ; 1: SS M256 N256 ; 2: TS M256 N128
__global__ void __cluster_dims__(2, 1, 1) __launch_bounds__(128, 1)
umma2_rate(int mode, int iters, long long* out, unsigned* err) {
  extern __shared__ uint8_t raw[];
  uint8_t* sm = (uint8_t*)(((uintptr_t)raw + 1023) & ~uintptr_t(1023));
  __shared__ uint64_t bar;
  __shared__ uint32_t tm;
  __shared__ uint32_t zero;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const uint32_t rank = cluster_rank();
  for (int i = threadIdx.x; i < 48 * 1024 / 16; i += blockDim.x) ((uint4*)sm)[i] = make_uint4(0, 0, 0, 0);
  if (threadIdx.x == 0) { ptx::mbar_init(&bar, 1); ptx::fence_mbar_init(); zero = 0; }
  if (warp == 0) {
    asm volatile("tcgen05.alloc.cta_group::2.sync.aligned.shared::cta.b32 [%0], %1;" :: "r"(ptx::smem_u32(&tm)), "r"(512) : "memory");
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::2.sync.aligned;" ::: "memory");
  }
  ptx::fence_proxy_async_smem();
  ptx::tc_fence_before();
  cluster_sync();
  ptx::tc_fence_after();
  const uint32_t tmem = tm;
  if (rank == 0 && warp == 1 && lane == 0) {
    const int N = mode == 1 ? 256 : 128;
    const uint32_t idesc = ptx::idesc_bf16_f32(256, N, 0);
    const uint64_t dA = ptx::sdesc_sw128(ptx::smem_u32(sm), 16, 1024);
    const uint64_t dB = ptx::sdesc_sw128(ptx::smem_u32(sm + 16384), 16, 1024);
    long long t0 = clock64();
    // straight-line UMMA runs (no branch between consecutive UMMAs)
    if (mode == 2) {
      for (int it = 0; it < iters; ++it) {
#pragma unroll
        for (int kk = 0; kk < 8; ++kk) {
          const uint32_t off = ((kk & 3) * 32) >> 4;
          umma2_ts(tmem, tmem + 256 + kk * 8, dB + off, idesc, 1u);
        }
      }
    } else {
      for (int it = 0; it < iters; ++it) {
#pragma unroll
        for (int kk = 0; kk < 8; ++kk) {
          const uint32_t off = ((kk & 3) * 32) >> 4;
          umma2_ss(tmem, dA + off, dB + off, idesc, 1u);
        }
      }
    }
    // one arrival on each CTA's barrier once every UMMA above has completed
    uint32_t peer_bar;
    asm volatile("mapa.shared::cluster.u32 %0, %1, 1;" : "=r"(peer_bar) : "r"(ptx::smem_u32(&bar)));
    asm volatile("tcgen05.commit.cta_group::2.mbarrier::arrive::one.shared::cluster.b64 [%0];"
                 :: "r"(ptx::smem_u32(&bar)) : "memory");
    asm volatile("tcgen05.commit.cta_group::2.mbarrier::arrive::one.shared::cluster.b64 [%0];"
                 :: "r"(peer_bar) : "memory");
    out[blockIdx.x] = clock64() - t0;   // issue time only; completion below
  }
  if (threadIdx.x == 0) {
    bool ok = ptx::mbar_wait_bounded(&bar, 0, &zero, 2000000000ull);
    if (!ok) atomicOr(err, 1u);
    if (rank == 0) out[gridDim.x + blockIdx.x] = clock64();
  }
  ptx::tc_fence_before();
  cluster_sync();
  if (warp == 0) {
    ptx::tc_fence_after();
    asm volatile("tcgen05.dealloc.cta_group::2.sync.aligned.b32 %0, %1;" :: "r"(tmem), "r"(512) : "memory");
  }
}

int main() {
  int sms; cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, 0);
  const int ctas = (sms / 2) * 2;
  long long* d; unsigned* err; cudaMalloc(&d, 2 * ctas * sizeof(long long)); cudaMalloc(&err, 4); cudaMemset(err, 0, 4);
  int smem = 48 * 1024 + 1024;
  cudaFuncSetAttribute(umma2_rate, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
  const char* names[] = {"2SM SS 256x128x16", "2SM SS 256x256x16", "2SM TS 256x128x16"};
  for (int mode = 0; mode < 3; ++mode) {
    const int iters = 2000;
    for (int rep = 0; rep < 2; ++rep) {
      cudaEvent_t e0, e1; cudaEventCreate(&e0); cudaEventCreate(&e1);
      cudaEventRecord(e0);
      umma2_rate<<<ctas, 128, smem>>>(mode, iters, d, err);
      cudaError_t le = cudaGetLastError();
      cudaEventRecord(e1); cudaError_t e = cudaEventSynchronize(e1);
      float ms; cudaEventElapsedTime(&ms, e0, e1);
      unsigned herr = 0; cudaMemcpy(&herr, err, 4, cudaMemcpyDeviceToHost);
      const int N = mode == 1 ? 256 : 128;
      double n_umma = (double)iters * 8;
      double flop = 2.0 * 256 * N * 16 * n_umma * (ctas / 2);
      double per_sm_cycles = (ms * 1e-3) * 1.9e9 / n_umma;   // rough, at ~1.9 GHz
      printf("%s: %.0f TFLOP/s by events (%.3f ms, ~%.1f cycles/UMMA per pair at 1.9GHz; 1-SM ideal %d) err=%u launch=%s sync=%s\n",
             names[mode], flop / (ms * 1e-3) / 1e12, ms, per_sm_cycles, N / 2, herr, cudaGetErrorString(le), cudaGetErrorString(e));
      if (e != cudaSuccess || le != cudaSuccess) return 1;
    }
  }
  return 0;
}

// Sustained tcgen05.mma issue rate on every SM for the operand shapes the
// attention kernel uses (SS 128x128x16 for S = QK^T, TS 128x128x16 for
// O += PV with P in TMEM) and for SS 128x256x16.  One CTA per SM issues a long
// run of UMMAs on fixed shared-memory / TMEM operands; cycles per UMMA against
// the ideal (N/2 cycles at 8192 FLOP per clock per SM) give the ceiling the
// attention kernel is measured against.
#include <cstdio>
#include <cuda_runtime.h>
#include "../csrc/apb_internal.h"
#include "../csrc/sm100_ptx.cuh"
using namespace apb;

// mode 0: SS M128 N128; mode 1: SS M128 N256; mode 2: TS M128 N128 (A from TMEM)
__global__ void __launch_bounds__(128, 1) umma_rate(int mode, int iters, long long* out, unsigned* err) {
  extern __shared__ uint8_t raw[];
  uint8_t* sm = (uint8_t*)(((uintptr_t)raw + 1023) & ~uintptr_t(1023));
  __shared__ uint64_t bar;
  __shared__ uint32_t tm;
  __shared__ uint32_t zero;
  int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  // zero the operand smem (A 16 KB at 0, B 32 KB at 16 KB)
  for (int i = threadIdx.x; i < 48 * 1024 / 16; i += blockDim.x) ((uint4*)sm)[i] = make_uint4(0,0,0,0);
  if (threadIdx.x == 0) { ptx::mbar_init(&bar, 1); ptx::fence_mbar_init(); zero = 0; }
  if (warp == 0) { ptx::tmem_alloc(&tm, 512); ptx::tmem_relinquish(); }
  ptx::fence_proxy_async_smem();
  ptx::tc_fence_before(); __syncthreads(); ptx::tc_fence_after();
  uint32_t tmem = tm;
  if (warp == 1 && lane == 0) {
    const int N = mode == 1 ? 256 : 128;
    const uint32_t idesc = ptx::idesc_bf16_f32(128, N, 0);
    const uint64_t dA = ptx::sdesc_sw128(ptx::smem_u32(sm), 16, 1024);
    const uint64_t dB = ptx::sdesc_sw128(ptx::smem_u32(sm + 16384), 16, 1024);
    long long t0 = clock64();
    // one straight-line run of UMMAs per mode: a branch between consecutive
    // UMMAs (e.g. choosing the form inside the unrolled loop) slows the
    // stream to ~104 (SS) / ~93 (TS) cycles per 128x128x16 UMMA
    if (mode == 2) {
      for (int it = 0; it < iters; ++it) {
#pragma unroll
        for (int kk = 0; kk < 8; ++kk) {
          const uint32_t off = ((kk & 3) * 32) >> 4;   // stay inside the first 64-column block
          ptx::umma_bf16_ts(tmem, tmem + 256 + kk * 8, dB + off, idesc, 1u);
        }
      }
    } else {
      for (int it = 0; it < iters; ++it) {
#pragma unroll
        for (int kk = 0; kk < 8; ++kk) {
          const uint32_t off = ((kk & 3) * 32) >> 4;
          ptx::umma_bf16_ss(tmem, dA + off, dB + off, idesc, 1u);
        }
      }
    }
    ptx::umma_commit(&bar);
    bool ok = ptx::mbar_wait_bounded(&bar, 0, &zero, 2000000000ull);
    long long t1 = clock64();
    out[blockIdx.x] = t1 - t0;
    if (!ok) atomicOr(err, 1u);
  }
  ptx::tc_fence_before(); __syncthreads();
  if (warp == 0) { ptx::tc_fence_after(); ptx::tmem_dealloc(tmem, 512); }
}

int main() {
  int sms; cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, 0);
  long long* d; unsigned* err; cudaMalloc(&d, sms * sizeof(long long)); cudaMalloc(&err, 4); cudaMemset(err, 0, 4);
  int smem = 48 * 1024 + 1024;
  cudaFuncSetAttribute(umma_rate, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
  const char* names[] = {"SS 128x128x16", "SS 128x256x16", "TS 128x128x16"};
  for (int mode = 0; mode < 3; ++mode) {
    const int iters = 2000;
    for (int rep = 0; rep < 2; ++rep) {
      cudaEvent_t e0, e1; cudaEventCreate(&e0); cudaEventCreate(&e1);
      cudaEventRecord(e0);
      umma_rate<<<sms, 128, smem>>>(mode, iters, d, err);
      cudaEventRecord(e1); cudaError_t e = cudaEventSynchronize(e1);
      float ms; cudaEventElapsedTime(&ms, e0, e1);
      long long h[256]; cudaMemcpy(h, d, sms * sizeof(long long), cudaMemcpyDeviceToHost);
      unsigned herr; cudaMemcpy(&herr, err, 4, cudaMemcpyDeviceToHost);
      double cyc = 0; for (int i = 0; i < sms; ++i) cyc += h[i]; cyc /= sms;
      const int N = mode == 1 ? 256 : 128;
      double n_umma = (double)iters * 8;
      double flop = 2.0 * 128 * N * 16 * n_umma * sms;
      printf("%s: %.1f cycles/UMMA (ideal %d), %.0f TFLOP/s by events, err=%u %s\n", names[mode],
             cyc / n_umma, N / 2, flop / (ms * 1e-3) / 1e12, herr, cudaGetErrorString(e));
    }
  }
  return 0;
}

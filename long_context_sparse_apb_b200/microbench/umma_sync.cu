// What a UMMA-issuing thread pays for touching shared memory between UMMA
// runs.  One CTA per SM; the issuing thread streams 128x128x16 SS UMMAs
// (8 per iteration, 512 cycles of tensor work) and does one of the accesses
// below between iterations; cycles per iteration by clock64 on the issuing
// SM.  The attention kernel's issue loop is laid out from these numbers.
#include <cstdio>
#include <cuda_runtime.h>
#include "../csrc/apb_internal.h"
#include "../csrc/sm100_ptx.cuh"
using namespace apb;

enum Mode {
  kPlain = 0,        // 8 UMMAs + commit
  kTestWait,         // + mbarrier.test_wait on a barrier that completed long ago
  kTryWait,          // + mbarrier.try_wait on the same
  kLoadVolatile,     // + ld.volatile.shared of a flag word
  kLoadAcquire,      // + ld.acquire.cta.shared of a flag word
  kSplitWaits,       // 4 UMMAs, test_wait, 4 UMMAs, test_wait, commit
  kIdleThenWait,     // + 1500 cycles idle on the clock, then test_wait
  kIdleOnly,         // + 1500 cycles idle on the clock
  kBranch,           // + a data-dependent branch (no memory access)
  kTwoIssuers,       // two issuing warps, each as kTestWait (16 UMMAs per iteration in all)
  kNumModes
};

__device__ __forceinline__ void umma8(uint32_t d, uint64_t dA, uint64_t dB, uint32_t idesc) {
#pragma unroll
  for (int kk = 0; kk < 8; ++kk) {
    const uint32_t off = ((kk & 3) * 32) >> 4;
    ptx::umma_bf16_ss(d, dA + off, dB + off, idesc, 1u);
  }
}
__device__ __forceinline__ void umma4(uint32_t d, uint64_t dA, uint64_t dB, uint32_t idesc) {
#pragma unroll
  for (int kk = 0; kk < 4; ++kk) {
    const uint32_t off = ((kk & 3) * 32) >> 4;
    ptx::umma_bf16_ss(d, dA + off, dB + off, idesc, 1u);
  }
}

// One instantiation per mode, so that the issue loop holds no branch on the
// mode (a branch inside the stream has a cost of its own, see kBranch).
template <int MODE>
__global__ void __launch_bounds__(128, 1) umma_sync(int iters, long long* out, unsigned* err) {
  extern __shared__ uint8_t raw[];
  uint8_t* sm = (uint8_t*)(((uintptr_t)raw + 1023) & ~uintptr_t(1023));
  __shared__ uint64_t bar[5];   // 0, 1: commits of issuer 0 / 1; 2: a completed barrier; 3, 4: drains
  __shared__ uint32_t tm;
  __shared__ uint32_t zero;
  __shared__ volatile uint32_t flag;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  for (int i = threadIdx.x; i < 48 * 1024 / 16; i += blockDim.x)
    reinterpret_cast<uint4*>(sm)[i] = make_uint4(0, 0, 0, 0);
  if (threadIdx.x == 0) {
    for (int i = 0; i < 5; ++i) ptx::mbar_init(&bar[i], 1);
    ptx::fence_mbar_init();
    zero = 0;
    flag = 0;
  }
  if (warp == 0) {
    ptx::tmem_alloc(&tm, 512);
    ptx::tmem_relinquish();
  }
  ptx::fence_proxy_async_smem();
  ptx::tc_fence_before();
  __syncthreads();
  ptx::tc_fence_after();
  if (threadIdx.x == 0) ptx::mbar_arrive(&bar[2]);   // phase 0 of bar[2] completes
  __syncthreads();
  const uint32_t tmem = tm;
  constexpr bool two = MODE == kTwoIssuers;
  if ((warp == 1 || (two && warp == 2)) && lane == 0) {
    const int me = warp - 1;
    const uint32_t idesc = ptx::idesc_bf16_f32(128, 128, 0);
    const uint64_t dA = ptx::sdesc_sw128(ptx::smem_u32(sm), 16, 1024);
    const uint64_t dB = ptx::sdesc_sw128(ptx::smem_u32(sm + 16384), 16, 1024);
    const uint32_t d = tmem + 256 * me;
    uint64_t* cb = &bar[me];
    bool ok = true;
    uint32_t acc = 0;
    const long long t0 = clock64();
    for (int it = 0; it < iters; ++it) {
      if (MODE == kSplitWaits) {
        umma4(d, dA, dB, idesc);
        ok &= ptx::mbar_spin_bounded(&bar[2], 0, &zero, 1000000000ull);
        umma4(d, dA, dB, idesc);
        ok &= ptx::mbar_spin_bounded(&bar[2], 0, &zero, 1000000000ull);
        ptx::umma_commit(cb);
        continue;
      }
      umma8(d, dA, dB, idesc);
      ptx::umma_commit(cb);
      if (MODE == kTestWait || MODE == kTwoIssuers) {
        ok &= ptx::mbar_spin_bounded(&bar[2], 0, &zero, 1000000000ull);
      } else if (MODE == kTryWait) {
        ok &= ptx::mbar_wait_bounded(&bar[2], 0, &zero, 1000000000ull);
      } else if (MODE == kLoadVolatile) {
        ok &= flag == 0u;
      } else if (MODE == kLoadAcquire) {
        uint32_t v;
        asm volatile("ld.acquire.cta.shared::cta.u32 %0, [%1];"
                     : "=r"(v)
                     : "r"(ptx::smem_u32((const void*)&flag))
                     : "memory");
        ok &= v == 0u;
      } else if (MODE == kIdleThenWait || MODE == kIdleOnly) {
        const long long t = clock64();
        while (clock64() - t < 1500) {
        }
        if (MODE == kIdleThenWait) ok &= ptx::mbar_spin_bounded(&bar[2], 0, &zero, 1000000000ull);
      } else if (MODE == kBranch) {
        if ((clock64() & 7) == 3) acc += 1;   // data-dependent, no memory access
      }
    }
    const long long t1 = clock64();
    // every MMA of this thread completes before TMEM is freed
    ptx::umma_commit(&bar[3 + me]);
    ok &= ptx::mbar_spin_bounded(&bar[3 + me], 0, &zero, 2000000000ull);
    if (blockIdx.x == 0) out[me] = t1 - t0 + (acc == 0xffffffffu);
    if (!ok) atomicOr(err, 1u);
  }
  ptx::tc_fence_before();
  __syncthreads();
  if (warp == 0) {
    ptx::tc_fence_after();
    ptx::tmem_dealloc(tmem, 512);
  }
}

template <int MODE>
int run_mode(const char* name, int sms, long long* d, unsigned* err) {
  const int smem = 48 * 1024 + 1024;
  cudaFuncSetAttribute(umma_sync<MODE>, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
  const int iters = 2000;
  cudaMemset(d, 0, 2 * sizeof(long long));
  umma_sync<MODE><<<sms, 128, smem>>>(iters, d, err);
  const cudaError_t e = cudaDeviceSynchronize();
  long long h[2];
  cudaMemcpy(h, d, sizeof(h), cudaMemcpyDeviceToHost);
  unsigned herr;
  cudaMemcpy(&herr, err, 4, cudaMemcpyDeviceToHost);
  printf("%-40s: %7.1f cycles per iteration (8 UMMAs of one issuer = 512)", name, (double)h[0] / iters);
  if (MODE == kTwoIssuers) printf(", second issuer %.1f (16 UMMAs in all = 1024)", (double)h[1] / iters);
  printf("%s%s\n", herr ? " WAIT FAILED" : "", e != cudaSuccess ? cudaGetErrorString(e) : "");
  return (herr != 0u) || (e != cudaSuccess);
}

int main() {
  int sms;
  cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, 0);
  long long* d;
  unsigned* err;
  cudaMalloc(&d, 2 * sizeof(long long));
  cudaMalloc(&err, 4);
  cudaMemset(err, 0, 4);
  int rc = 0;
  rc |= run_mode<kPlain>("8 UMMA + commit", sms, d, err);
  rc |= run_mode<kTestWait>("+ test_wait (completed barrier)", sms, d, err);
  rc |= run_mode<kTryWait>("+ try_wait (completed barrier)", sms, d, err);
  rc |= run_mode<kLoadVolatile>("+ ld.volatile.shared", sms, d, err);
  rc |= run_mode<kLoadAcquire>("+ ld.acquire.shared", sms, d, err);
  rc |= run_mode<kSplitWaits>("4 UMMA, test_wait, 4 UMMA, test_wait", sms, d, err);
  rc |= run_mode<kIdleThenWait>("+ 1500 cycles idle, then test_wait", sms, d, err);
  rc |= run_mode<kIdleOnly>("+ 1500 cycles idle", sms, d, err);
  rc |= run_mode<kBranch>("+ data-dependent branch", sms, d, err);
  rc |= run_mode<kTwoIssuers>("two issuers, each + test_wait", sms, d, err);
  return rc;
}

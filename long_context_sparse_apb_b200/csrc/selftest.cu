// Self-test of the bounded-wait machinery shared by the kernels: a launch of
// two CTAs in which CTA 0 waits on an mbarrier that nothing ever completes,
// with a short wall-clock limit, and CTA 1 waits on another such barrier with
// a long limit.  CTA 0's wait runs out and records the failure; CTA 1 must
// then leave its wait through the launch-wide abort flag well before its own
// limit.  Nothing faults, traps or hangs.
#include "device_status.cuh"
#include "sm100_ptx.cuh"

namespace apb {
namespace {

__global__ void selftest_wait_kernel(DeviceStatus* status, uint64_t short_ns, uint64_t long_ns,
                                     unsigned long long* elapsed_ns) {
  __shared__ uint64_t bar;
  __shared__ uint32_t zero;
  if (threadIdx.x == 0) {
    ptx::mbar_init(&bar, 1);
    ptx::fence_mbar_init();
    zero = 0u;
  }
  __syncthreads();
  if (threadIdx.x == 0) {
    const uint64_t t0 = ptx::globaltimer();
    const volatile uint32_t* abort = &status->abort;
    const bool ok = ptx::mbar_wait_bounded(&bar, 0, blockIdx.x == 0 ? &zero : abort,
                                           blockIdx.x == 0 ? short_ns : long_ns);
    if (!ok) record_failure(status, 90 + blockIdx.x, 0);
    elapsed_ns[blockIdx.x] = ptx::globaltimer() - t0;
  }
}

}  // namespace
}  // namespace apb

namespace apb {

cudaError_t launch_wait_selftest(DeviceStatus* status, uint32_t limit_us,
                                 unsigned long long* elapsed_ns, cudaStream_t st) {
  cudaError_t e = cudaMemsetAsync(&status->abort, 0, sizeof(uint32_t), st);
  if (e != cudaSuccess) return e;
  const uint64_t short_ns = (uint64_t)limit_us * 1000ull;
  selftest_wait_kernel<<<2, 32, 0, st>>>(status, short_ns, 20ull * short_ns + 1000000000ull,
                                         elapsed_ns);
  return cudaGetLastError();
}

}  // namespace apb

extern "C" apb_status apb_selftest_wait_timeout(void* workspace, size_t ws_bytes,
                                                uint32_t limit_us, void* stream) {
  if (!workspace || ws_bytes < apb::kStatusBytes || (reinterpret_cast<uintptr_t>(workspace) & 15))
    return apb::fail(APB_ERR_INVALID_ARG,
                     "apb_selftest_wait_timeout: workspace NULL, unaligned or < %zu bytes",
                     apb::kStatusBytes);
  if (limit_us == 0 || limit_us > 1000000)
    return apb::fail(APB_ERR_INVALID_ARG, "apb_selftest_wait_timeout: limit_us=%u not in [1, 1e6]",
                     limit_us);
  auto* status = static_cast<apb::DeviceStatus*>(workspace);
  // elapsed times of the two waits go to the spare bytes of the status block
  auto* elapsed = reinterpret_cast<unsigned long long*>(static_cast<char*>(workspace) + 64);
  const cudaError_t e = apb::launch_wait_selftest(status, limit_us, elapsed,
                                                  reinterpret_cast<cudaStream_t>(stream));
  return e == cudaSuccess ? APB_OK : apb::cuda_fail(e, "self-test kernel");
}

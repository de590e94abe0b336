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

extern "C" apb_status apb_selftest_wait_timeout(void* workspace, size_t ws_bytes,
                                                uint32_t limit_us, void* stream) {
  if (!workspace || ws_bytes < apb::kStatusBytes || (reinterpret_cast<uintptr_t>(workspace) & 15))
    return APB_ERR_INVALID_ARG;
  if (limit_us == 0 || limit_us > 1000000) return APB_ERR_INVALID_ARG;
  cudaStream_t cs = reinterpret_cast<cudaStream_t>(stream);
  auto* status = static_cast<apb::DeviceStatus*>(workspace);
  // elapsed times of the two waits go to the spare bytes of the status block
  auto* elapsed = reinterpret_cast<unsigned long long*>(static_cast<char*>(workspace) + 64);
  if (cudaMemsetAsync(&status->abort, 0, sizeof(uint32_t), cs) != cudaSuccess) return APB_ERR_CUDA;
  const uint64_t short_ns = (uint64_t)limit_us * 1000ull;
  apb::selftest_wait_kernel<<<2, 32, 0, cs>>>(status, short_ns, 20ull * short_ns + 1000000000ull,
                                             elapsed);
  return cudaGetLastError() == cudaSuccess ? APB_OK : APB_ERR_CUDA;
}

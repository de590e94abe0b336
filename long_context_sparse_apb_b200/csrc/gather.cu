// Passing-block construction: the on-GPU stand-in for the all-gather of
// compressed blocks ("APB 的主要功能", communication).  With H virtual hosts
// on one GPU the all-gather is a gather in HBM:
//     pass[h*keep + r, g, :] = src[idx[h, g, r], g, :]      (K and V)
// The passing layout is token-major like K and V, so host h's passing block
// is the prefix of h*keep rows and the blocks of a range of hosts are one
// contiguous chunk (what a multi-GPU all-gather exchanges).
// Each output row is d bf16 = 128 or 256 bytes; consecutive threads copy
// consecutive 16-byte chunks of a row, so reads of a source row and writes of
// the destination rows are both fully coalesced.
#include "apb_internal.h"

namespace apb {
namespace {

__global__ void __launch_bounds__(256) gather_passing_kernel(
    const uint4* __restrict__ k, const uint4* __restrict__ v, const int32_t* __restrict__ idx,
    uint4* __restrict__ pk, uint4* __restrict__ pv, int H, int Hkv, int keep, int chunks_per_row,
    long long N) {
  const long long rows = (long long)H * Hkv * keep;
  const long long total = rows * chunks_per_row;
  const long long stride = (long long)gridDim.x * blockDim.x;
  for (long long i = (long long)blockIdx.x * blockDim.x + threadIdx.x; i < total; i += stride) {
    const long long row = i / chunks_per_row;       // = (h*Hkv + g)*keep + r
    const int c = (int)(i - row * chunks_per_row);
    const int r = (int)(row % keep);
    const long long hg = row / keep;
    const int g = (int)(hg % Hkv);
    const int h = (int)(hg / Hkv);
    const long long t = __ldg(idx + row);
    const long long dst = (((long long)h * keep + r) * Hkv + g) * chunks_per_row + c;
    uint4 a = make_uint4(0, 0, 0, 0), b = make_uint4(0, 0, 0, 0);
    if (t >= 0 && t < N) {
      const long long src = (t * Hkv + g) * chunks_per_row + c;
      a = __ldg(k + src);
      b = __ldg(v + src);
    }
    pk[dst] = a;
    pv[dst] = b;
  }
}

}  // namespace

cudaError_t launch_gather(const Shape& s, const void* k, const void* v, const int32_t* idx,
                          void* pass_k, void* pass_v, cudaStream_t st) {
  const int cpr = s.d * 2 / 16;
  const long long total = (long long)s.H * s.Hkv * s.keep * cpr;
  int dev = 0, sms = 148;
  cudaGetDevice(&dev);
  cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  long long want = (total + 255) / 256;
  int grid = (int)(want < (long long)sms * 8 ? want : (long long)sms * 8);
  if (grid < 1) grid = 1;
  gather_passing_kernel<<<grid, 256, 0, st>>>(
      static_cast<const uint4*>(k), static_cast<const uint4*>(v), idx, static_cast<uint4*>(pass_k),
      static_cast<uint4*>(pass_v), s.H, s.Hkv, s.keep, cpr, s.N);
  return cudaGetLastError();
}

}  // namespace apb

// Top-k compression of every (host, kv head): keep the `keep` positions of
// the host's block with the largest retaining-head score ("APB 的技术原理":
// the compressed block holds the important KV pairs).
//
// One CTA per (host, kv head).  Scores map to order-preserving uint32 keys
// (-0 folded onto +0); four 8-bit MSB-first radix passes find the key T of
// the keep-th largest element and how many elements equal to T are still to
// be taken.  A final pass walks the block in position order and writes every
// element with key > T, plus the first `need` elements with key == T, so the
// output is ascending and ties go to the lower position -- deterministic.
// The block's keys are staged in shared memory when they fit, else re-read
// from global memory (L2-resident) in every pass.
//
// The fused form (launch_topk_gather) then builds the (host, kv head)'s
// compressed block straight from the selection: the same CTA copies the
// selected K and V rows into the passing buffers (one launch and no second
// read of the indices from another kernel).
#include "apb_internal.h"

namespace apb {
namespace {

constexpr int kThreads = 1024;
constexpr int kMaxSmemKeys = 48 * 1024;   // 192 KB of keys

__device__ __forceinline__ uint32_t order_key(float f) {
  uint32_t u = __float_as_uint(f);
  if (u == 0x80000000u) u = 0u;
  return (u & 0x80000000u) ? ~u : (u | 0x80000000u);
}

// Exclusive block-wide prefix count of `flag` in thread order; returns the
// prefix for this thread and writes the block total to *total.
__device__ __forceinline__ int block_exclusive_count(bool flag, int* warp_sums, int* total) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const unsigned bal = __ballot_sync(0xffffffffu, flag);
  const int in_warp = __popc(bal & ((1u << lane) - 1u));
  if (lane == 0) warp_sums[warp] = __popc(bal);
  __syncthreads();
  if (warp == 0) {
    int x = warp_sums[lane];
    int incl = x;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      int y = __shfl_up_sync(0xffffffffu, incl, o);
      if (lane >= o) incl += y;
    }
    warp_sums[lane] = incl - x;          // exclusive
    if (lane == 31) warp_sums[32] = incl;
  }
  __syncthreads();
  const int res = warp_sums[warp] + in_warp;
  *total = warp_sums[32];
  __syncthreads();
  return res;
}

struct GatherArgs {
  const uint4* k;   // [N, Hkv, d] bf16 as 16-byte chunks
  const uint4* v;
  uint4* pass_k;    // [H * keep, Hkv, d]
  uint4* pass_v;
  int chunks_per_row;
};

template <bool GATHER>
__global__ void __launch_bounds__(kThreads) topk_kernel(const float* __restrict__ scores,
                                                        int32_t* __restrict__ idx, int n, int keep,
                                                        long long N, int Hkv, bool stage,
                                                        GatherArgs ga) {
  extern __shared__ uint32_t skeys[];
  __shared__ int hist[256];
  __shared__ int warp_sums[kThreads / 32 + 1];
  __shared__ uint32_t s_digit;
  __shared__ int s_above;

  const int g = blockIdx.x, h = blockIdx.y;
  const float* src = scores + (long long)g * N + (long long)h * n;
  int32_t* out = idx + ((long long)h * Hkv + g) * keep;

  if (stage) {
    for (int i = threadIdx.x; i < n; i += kThreads) skeys[i] = order_key(src[i]);
    __syncthreads();
  }
  auto key_at = [&](int i) -> uint32_t { return stage ? skeys[i] : order_key(__ldg(src + i)); };

  uint32_t prefix = 0, mask = 0;
  int remaining = keep;   // elements still to take among those matching prefix
  for (int pass = 0; pass < 4; ++pass) {
    const int shift = 24 - 8 * pass;
    for (int i = threadIdx.x; i < 256; i += kThreads) hist[i] = 0;
    __syncthreads();
    for (int i = threadIdx.x; i < n; i += kThreads) {
      const uint32_t u = key_at(i);
      if ((u & mask) == prefix) atomicAdd(&hist[(u >> shift) & 255u], 1);
    }
    __syncthreads();
    if (threadIdx.x < 32) {
      // lane l owns digits [248 - 8l, 255 - 8l] (descending); suffix counts
      const int lane = threadIdx.x;
      int cnt[8], tot = 0;
#pragma unroll
      for (int j = 0; j < 8; ++j) { cnt[j] = hist[255 - 8 * lane - j]; tot += cnt[j]; }
      int incl = tot;
#pragma unroll
      for (int o = 1; o < 32; o <<= 1) {
        int y = __shfl_up_sync(0xffffffffu, incl, o);
        if (lane >= o) incl += y;
      }
      int above = incl - tot;   // elements with a larger digit than this lane's first
      const bool mine = above < remaining && remaining <= incl;
      if (mine) {
        int j = 0;
        while (above + cnt[j] < remaining) { above += cnt[j]; ++j; }
        s_digit = (uint32_t)(255 - 8 * lane - j);
        s_above = above;
      }
    }
    __syncthreads();
    prefix |= s_digit << shift;
    mask |= 255u << shift;
    remaining -= s_above;
    __syncthreads();
  }
  const uint32_t T = prefix;
  const int need_eq = remaining;   // elements equal to T to take, lowest positions first

  int written = 0, eq_seen = 0;
  for (int base = 0; base < n; base += kThreads) {
    const int i = base + threadIdx.x;
    const bool valid = i < n;
    const uint32_t u = valid ? key_at(i) : 0u;
    const bool gt = valid && u > T;
    const bool eq = valid && u == T;
    int eq_tot;
    const int eq_rank = block_exclusive_count(eq, warp_sums, &eq_tot);
    const bool sel = gt || (eq && eq_seen + eq_rank < need_eq);
    int sel_tot;
    const int pos = block_exclusive_count(sel, warp_sums, &sel_tot);
    if (sel) out[written + pos] = (int32_t)((long long)h * n + i);
    written += sel_tot;
    eq_seen += eq_tot;
  }
  if (GATHER) {
    // pass[h*keep + r, g, :] = src[idx[h, g, r], g, :] for K and V; the
    // indices were written above by this CTA (visible after the barrier;
    // read with plain loads, not the read-only path).  Consecutive threads
    // copy consecutive 16-byte chunks of a row.
    __syncthreads();
    const int cpr = ga.chunks_per_row;
    const long long row0 = (long long)h * keep;
    for (int e = threadIdx.x; e < keep * cpr; e += kThreads) {
      const int r = e / cpr, c = e - r * cpr;
      const long long t = out[r];
      uint4 a = make_uint4(0, 0, 0, 0), b = make_uint4(0, 0, 0, 0);
      if (t >= 0 && t < N) {
        const long long src = (t * Hkv + g) * cpr + c;
        a = __ldg(ga.k + src);
        b = __ldg(ga.v + src);
      }
      const long long dst = ((row0 + r) * Hkv + g) * cpr + c;
      ga.pass_k[dst] = a;
      ga.pass_v[dst] = b;
    }
  }
}

template <bool GATHER>
cudaError_t launch(const Shape& s, const float* scores, int32_t* idx, GatherArgs ga,
                   cudaStream_t st) {
  const bool stage = s.n <= kMaxSmemKeys;
  const size_t smem = stage ? (size_t)s.n * sizeof(uint32_t) : 0;
  if (stage) {
    cudaError_t e = cudaFuncSetAttribute(topk_kernel<GATHER>,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
  }
  dim3 grid(s.Hkv, s.H);
  topk_kernel<GATHER><<<grid, kThreads, smem, st>>>(scores, idx, s.n, s.keep, s.N, s.Hkv, stage,
                                                    ga);
  return cudaGetLastError();
}

}  // namespace

cudaError_t launch_topk(const Shape& s, const float* scores, int32_t* idx, cudaStream_t st) {
  return launch<false>(s, scores, idx, GatherArgs{}, st);
}

cudaError_t launch_topk_gather(const Shape& s, const float* scores, int32_t* idx, const void* k,
                               const void* v, void* pass_k, void* pass_v, cudaStream_t st) {
  GatherArgs ga{static_cast<const uint4*>(k), static_cast<const uint4*>(v),
                static_cast<uint4*>(pass_k), static_cast<uint4*>(pass_v), s.d * 2 / 16};
  return launch<true>(s, scores, idx, ga, st);
}

}  // namespace apb

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
// from global memory (L2-resident) in every pass.  Each thread takes four
// consecutive keys per step, so the ordered pass needs one block-wide scan
// per 4096 keys.
//
// The fused form (launch_topk_gather) then builds the (host, kv head)'s
// compressed block straight from the selection: the CTAs that made it copy
// the selected K and V rows into the passing buffers (one launch and no
// second read of the indices from another kernel).
#include <algorithm>

#include "apb_internal.h"

namespace apb {
namespace {

constexpr int kThreads = 1024;
constexpr int kPer = 4;                      // consecutive keys per thread and step
constexpr int kStep = kThreads * kPer;
constexpr int kMaxSmemKeys = 48 * 1024;      // 192 KB of keys

__device__ __forceinline__ uint32_t order_key(float f) {
  uint32_t u = __float_as_uint(f);
  if (u == 0x80000000u) u = 0u;
  return (u & 0x80000000u) ? ~u : (u | 0x80000000u);
}

// Keys i .. i+3 of the block (i < n, a multiple of 4): from the staged copy
// (padded to a multiple of 4 entries) or from global memory; keys at or past
// n are returned as 0 and must be masked by the caller.
__device__ __forceinline__ void load_keys(const uint32_t* skeys, const float* src, bool stage,
                                          int i, int n, uint32_t (&u)[kPer]) {
  if (stage) {
    const uint4 w = *reinterpret_cast<const uint4*>(skeys + i);
    u[0] = w.x;
    u[1] = w.y;
    u[2] = w.z;
    u[3] = w.w;
  } else {
#pragma unroll
    for (int k = 0; k < kPer; ++k) u[k] = i + k < n ? order_key(__ldg(src + i + k)) : 0u;
  }
}

// Exclusive block-wide prefix sum of v in thread order; returns the prefix
// for this thread and writes the block total to *total.
__device__ __forceinline__ int block_exclusive_sum(int v, int* warp_sums, int* total) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  int incl = v;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const int y = __shfl_up_sync(0xffffffffu, incl, o);
    if (lane >= o) incl += y;
  }
  if (lane == 31) warp_sums[warp] = incl;
  __syncthreads();
  if (warp == 0) {
    const int x = warp_sums[lane];
    int w = x;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int y = __shfl_up_sync(0xffffffffu, w, o);
      if (lane >= o) w += y;
    }
    warp_sums[lane] = w - x;   // exclusive
    if (lane == 31) warp_sums[32] = w;
  }
  __syncthreads();
  const int res = warp_sums[warp] + incl - v;
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

// The fused form runs `parts` CTAs per (host, kv head) (gridDim.z): each
// repeats the (cheap, shared-memory) selection, writes its own run of the
// selected positions and copies those rows, so the copy is spread over parts
// times as many SMs.  The launch picks parts so that the grid stays within one
// CTA per SM (the fused kernel's registers allow one 1024-thread CTA per SM)
// and every part copies at least kMinRowsPerPart rows.
constexpr int kMinRowsPerPart = 128;

// One 16-byte chunk of the gather: chunk e of the selected rows (row e / cpr)
// read from K and V, and its place in the passing buffers (-1 past the end).
struct Chunk {
  uint4 k, v;
  long long dst;
};

__device__ __forceinline__ Chunk load_chunk(const GatherArgs& ga, const int32_t* sel, int e,
                                            int e1, int cpr, long long row0, int g, int Hkv,
                                            long long N) {
  Chunk x{make_uint4(0, 0, 0, 0), make_uint4(0, 0, 0, 0), -1};
  if (e >= e1) return x;
  const int r = e / cpr, c = e - r * cpr;
  const long long t = sel[r];
  if (t >= 0 && t < N) {
    const long long src = (t * Hkv + g) * cpr + c;
    x.k = __ldg(ga.k + src);
    x.v = __ldg(ga.v + src);
  }
  x.dst = ((row0 + r) * Hkv + g) * cpr + c;
  return x;
}

template <bool GATHER>
__global__ void __launch_bounds__(kThreads) topk_kernel(const float* __restrict__ scores,
                                                        int32_t* __restrict__ idx, int n, int keep,
                                                        long long N, int Hkv, bool stage,
                                                        GatherArgs ga) {
  extern __shared__ __align__(16) uint32_t skeys[];   // read 16 bytes at a time
  __shared__ int hist[256];
  __shared__ int warp_sums[kThreads / 32 + 1];
  __shared__ uint32_t s_digit;
  __shared__ int s_above;

  const int g = blockIdx.x, h = blockIdx.y, part = blockIdx.z;
  // this CTA's rows [r0, r1) of the selection (all of it without the gather)
  const int rows_per_part = (keep + (int)gridDim.z - 1) / (int)gridDim.z;
  const int r0 = min(keep, part * rows_per_part);
  const int r1 = min(keep, r0 + rows_per_part);
  const float* src = scores + (long long)g * N + (long long)h * n;
  int32_t* out = idx + ((long long)h * Hkv + g) * keep;

  if (stage) {
    // eight loads in flight per thread before the first store
    constexpr int kLoads = 8;
    for (int base = 0; base < n; base += kLoads * kThreads) {
      float f[kLoads];
#pragma unroll
      for (int u = 0; u < kLoads; ++u) {
        const int i = base + u * kThreads + threadIdx.x;
        f[u] = i < n ? __ldg(src + i) : 0.f;
      }
#pragma unroll
      for (int u = 0; u < kLoads; ++u) {
        const int i = base + u * kThreads + threadIdx.x;
        if (i < n) skeys[i] = order_key(f[u]);
      }
    }
    __syncthreads();
  }
  const int lane = threadIdx.x & 31;

  uint32_t prefix = 0, mask = 0;
  int remaining = keep;   // elements still to take among those matching prefix
  for (int pass = 0; pass < 4; ++pass) {
    const int shift = 24 - 8 * pass;
    for (int i = threadIdx.x; i < 256; i += kThreads) hist[i] = 0;
    __syncthreads();
    // Scores of one block share their leading bits (sign and exponent), so in
    // the first passes most lanes of a warp fall in the same bin: the lanes
    // with the first counted lane's digit add their count with one atomic.
    for (int base = 0; base < n; base += kStep) {
      const int i = base + kPer * threadIdx.x;
      uint32_t u[kPer] = {0u, 0u, 0u, 0u};
      if (i < n) load_keys(skeys, src, stage, i, n, u);
#pragma unroll
      for (int k = 0; k < kPer; ++k) {
        const bool in = i + k < n && (u[k] & mask) == prefix;
        const uint32_t digit = in ? (u[k] >> shift) & 255u : 256u;
        const unsigned counted = __ballot_sync(0xffffffffu, in);
        if (counted) {
          const int leader = __ffs(counted) - 1;
          const uint32_t lead = __shfl_sync(0xffffffffu, digit, leader);
          const unsigned same = __ballot_sync(0xffffffffu, digit == lead);
          if (lane == leader) atomicAdd(&hist[lead], __popc(same));
          if (in && digit != lead) atomicAdd(&hist[digit], 1);
        }
      }
    }
    __syncthreads();
    if (threadIdx.x < 32) {
      // lane l owns digits [248 - 8l, 255 - 8l] (descending); suffix counts
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

  // Ordered pass.  The selected elements are every key > T and the first
  // need_eq keys == T, so the output slot of a selected element at position i
  // is (keys > T before i) + min(keys == T before i, need_eq); one scan per
  // step counts both (packed 16 + 16 bits; at most kStep per step).
  int gt_done = 0, eq_done = 0;
  for (int base = 0; base < n; base += kStep) {
    const int i = base + kPer * threadIdx.x;
    uint32_t u[kPer] = {0u, 0u, 0u, 0u};
    if (i < n) load_keys(skeys, src, stage, i, n, u);
    int ngt = 0, neq = 0;
#pragma unroll
    for (int k = 0; k < kPer; ++k) {
      ngt += (i + k < n && u[k] > T) ? 1 : 0;
      neq += (i + k < n && u[k] == T) ? 1 : 0;
    }
    int tot;
    const int pre = block_exclusive_sum(ngt | (neq << 16), warp_sums, &tot);
    int gt_before = gt_done + (pre & 0xffff);
    int eq_before = eq_done + (pre >> 16);
#pragma unroll
    for (int k = 0; k < kPer; ++k) {
      if (i + k >= n) break;
      int slot = -1;
      if (u[k] > T) {
        slot = gt_before + min(eq_before, need_eq);
        ++gt_before;
      } else if (u[k] == T) {
        if (eq_before < need_eq) slot = gt_before + eq_before;
        ++eq_before;
      }
      if (slot >= r0 && slot < r1) out[slot] = (int32_t)((long long)h * n + i + k);
    }
    gt_done += tot & 0xffff;
    eq_done += tot >> 16;
  }
  if (GATHER) {
    // pass[h*keep + r, g, :] = src[idx[h, g, r], g, :] for K and V and the
    // rows r in [r0, r1), whose positions this CTA wrote above (visible to it
    // after the barrier; plain loads, not the read-only path).  Consecutive
    // threads copy consecutive 16-byte chunks of a row; each thread has the
    // loads of two chunks in flight before it stores them.
    __syncthreads();
    const int cpr = ga.chunks_per_row;
    const long long row0 = (long long)h * keep;
    const int e1 = r1 * cpr;
    for (int e = r0 * cpr + threadIdx.x; e < e1; e += 2 * kThreads) {
      const Chunk x0 = load_chunk(ga, out, e, e1, cpr, row0, g, Hkv, N);
      const Chunk x1 = load_chunk(ga, out, e + kThreads, e1, cpr, row0, g, Hkv, N);
      ga.pass_k[x0.dst] = x0.k;
      ga.pass_v[x0.dst] = x0.v;
      if (x1.dst >= 0) {
        ga.pass_k[x1.dst] = x1.k;
        ga.pass_v[x1.dst] = x1.v;
      }
    }
  }
}

template <bool GATHER>
cudaError_t launch(const Shape& s, const float* scores, int32_t* idx, GatherArgs ga,
                   cudaStream_t st) {
  const bool stage = s.n <= kMaxSmemKeys;
  const size_t smem = stage ? (size_t)((s.n + kPer - 1) / kPer * kPer) * sizeof(uint32_t) : 0;
  if (stage) {
    cudaError_t e = cudaFuncSetAttribute(topk_kernel<GATHER>,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
  }
  int parts = 1;
  if (GATHER) {
    int dev = 0, sms = 148;
    cudaGetDevice(&dev);
    cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    const long long units = (long long)s.Hkv * s.H;
    const long long by_sms = sms / units;
    const long long by_rows = s.keep / kMinRowsPerPart;
    parts = (int)std::max(1ll, std::min(by_sms, by_rows));
  }
  dim3 grid(s.Hkv, s.H, parts);
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

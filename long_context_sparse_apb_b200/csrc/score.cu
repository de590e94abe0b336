// Retaining-head stand-in scores on the tensor cores ("APB 的主要功能": each
// host compresses its KV with retaining heads).  For token t and kv head g:
//     x = [k[t,g] ; v[t,g] ; mean_{j in group g} q[t,j]]          (3d)
//     s[g,t] = w2[g] . SiLU(W1[g] x + b1[g]) + b2[g]
//
// The product W1 x must be fp32-accurate (the top-k that follows orders the
// scores), while the tensor cores multiply bf16.  Two exact rewrites make that
// possible:
//   * the group mean is folded into the weights: W1_q (1/G) sum_j q_j =
//     sum_j (W1_q / G) q_j, so every input row is an exact bf16 row of K, V or
//     one q head, and no averaged (inexact) q ever exists;
//   * each fp32 weight w is split into bf16 hi + lo (hi = rn(w), lo = rn(w -
//     hi)), leaving |w - hi - lo| <= 2^-17 |w|; both halves are multiplied
//     with fp32 accumulation.
// So Z = X W1^T is computed as sum over the 2 + G input blocks of
// X_b (Wh_b + Wl_b)^T with UMMA (M = 128 tokens, N = 256 hidden, K = 16),
// accumulated in TMEM, and the epilogue applies b1, SiLU, w2 and b2 in fp32.
//
// split_weights_kernel writes Wh, Wl ([Hkv, 2, hidden, 3d] bf16) into the
// workspace once per call.  score_kernel: one CTA = 256 tokens (two M = 128
// accumulators, TMEM columns [0,256) and [256,512)) of one kv head; warp 8
// streams B tiles (Wh, Wl of one 64-feature chunk, 2 x 32 KB, 2 stages) and
// A tiles (128 tokens x 64 features of K, V or a q head, 16 KB, 4 stages)
// with TMA; warp 9 issues the UMMAs; warps 0-7 run the epilogue, one token
// row per thread.  Waits are bounded like the attention kernel's.
#include <cuda_bf16.h>

#include "apb_internal.h"
#include "device_status.cuh"
#include "sm100_ptx.cuh"

namespace apb {
namespace {

constexpr int kHid = 256;
constexpr int kTile = 128;                 // tokens per accumulator
constexpr int kChunk = 64;                 // features per chunk (128-byte rows)
constexpr int kAStages = 4;
constexpr int kBStages = 2;
constexpr int kATile = kTile * kChunk * 2;          // 16 KB
constexpr int kBHalf = kHid * kChunk * 2;           // 32 KB (hi or lo)
constexpr int kSmemA = 0;
constexpr int kSmemB = kAStages * kATile;           // 64 KB
constexpr int kSmemBars = kSmemB + kBStages * 2 * kBHalf;   // 192 KB
constexpr int kSmemBytes = kSmemBars + 256 + 2 * kHid * 4 + 1024;
constexpr int kThreads = 320;
constexpr uint64_t kWaitLimitNs = 1000000000ull;

enum Bar { A_FULL = 0, A_EMPTY = 4, B_FULL = 8, B_EMPTY = 10, ACC_FULL = 12, DRAIN = 13, NUM = 14 };

__global__ void __launch_bounds__(256) split_weights_kernel(const float* __restrict__ w1,
                                                            __nv_bfloat16* __restrict__ ws,
                                                            int Hkv, int F, int d, int G) {
  const long long per_head = (long long)kHid * F;
  const long long total = (long long)Hkv * per_head;
  for (long long i = (long long)blockIdx.x * blockDim.x + threadIdx.x; i < total;
       i += (long long)gridDim.x * blockDim.x) {
    const long long g = i / per_head;
    const long long rem = i - g * per_head;
    const int f = (int)(rem % F);
    float w = w1[i];
    if (f >= 2 * d) w = __fdiv_rn(w, (float)G);   // group mean folded in (exact for G = 2^k)
    const __nv_bfloat16 hi = __float2bfloat16_rn(w);
    const __nv_bfloat16 lo = __float2bfloat16_rn(w - __bfloat162float(hi));
    ws[(2 * g) * per_head + rem] = hi;
    ws[(2 * g + 1) * per_head + rem] = lo;
  }
}

// Query-aware variant: the q input of the MLP is the same for every token,
// qseg[g] = mean of q over the query segment rows [0, q_len) and the group's
// G heads, so its product folds into the first-layer bias:
//     qbias[g, u] = b1[g, u] + sum_f W1[g, u, 2d + f] * qseg[g, f]
// One CTA per kv head; fp32 sums (q_len * G bf16 terms, then d products).
__global__ void __launch_bounds__(256) query_bias_kernel(const __nv_bfloat16* __restrict__ q,
                                                         const float* __restrict__ w1,
                                                         const float* __restrict__ b1,
                                                         float* __restrict__ qbias, int ql, int Hq,
                                                         int G, int d) {
  __shared__ float qm[128];
  const int g = blockIdx.x;
  const int F = 3 * d;
  for (int f = threadIdx.x; f < d; f += blockDim.x) {
    float acc = 0.f;
    for (int r = 0; r < ql; ++r)
      for (int j = 0; j < G; ++j)
        acc += __bfloat162float(q[((long long)r * Hq + (long long)g * G + j) * d + f]);
    qm[f] = ql > 0 ? __fdiv_rn(acc, (float)(ql * G)) : 0.f;
  }
  __syncthreads();
  for (int u = threadIdx.x; u < kHid; u += blockDim.x) {
    const float* wrow = w1 + ((long long)g * kHid + u) * F + 2 * d;
    float z = b1[g * kHid + u];
    for (int f = 0; f < d; ++f) z = fmaf(wrow[f], qm[f], z);
    qbias[g * kHid + u] = z;
  }
}

struct ScoreParams {
  long long N;
  int Hq, Hkv, G, d, F, n_chunks;
  const float* b1;
  const float* w2;
  const float* b2;
  float* scores;
  DeviceStatus* status;
};

// A tiles of one chunk: 1 input block for k and v chunks, G for q chunks,
// each for both 128-token halves.
__device__ __forceinline__ int chunk_blocks(int c, int d, int G) {
  return (c * kChunk) / d < 2 ? 1 : G;
}

__global__ void __launch_bounds__(kThreads, 1)
    score_kernel(const __grid_constant__ CUtensorMap mQ, const __grid_constant__ CUtensorMap mK,
                 const __grid_constant__ CUtensorMap mV, const __grid_constant__ CUtensorMap mW,
                 const ScoreParams p) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + kSmemBars);
  uint32_t* s_tmem = reinterpret_cast<uint32_t*>(bars + NUM);
  uint32_t* s_flags = s_tmem + 1;
  float* s_b1 = reinterpret_cast<float*>(smem + kSmemBars + 256);
  float* s_w2 = s_b1 + kHid;

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int g = blockIdx.y;
  const long long t0 = (long long)blockIdx.x * (2 * kTile);
  const volatile uint32_t* gabort = &p.status->abort;

  if (threadIdx.x == 0) {
    for (int i = 0; i < NUM; ++i) ptx::mbar_init(&bars[i], 1);
    ptx::fence_mbar_init();
    s_flags[0] = *gabort;
    s_flags[1] = 0u;
  }
  if (threadIdx.x < kHid) {
    s_b1[threadIdx.x] = p.b1[g * kHid + threadIdx.x];
    s_w2[threadIdx.x] = p.w2[g * kHid + threadIdx.x];
  }
  if (warp == 9) {
    ptx::tmem_alloc(s_tmem, 512);
    ptx::tmem_relinquish();
  }
  if (warp == 8 && lane == 0) {
    ptx::tma_prefetch_desc(&mQ);
    ptx::tma_prefetch_desc(&mK);
    ptx::tma_prefetch_desc(&mV);
    ptx::tma_prefetch_desc(&mW);
  }
  ptx::tc_fence_before();
  __syncthreads();
  ptx::tc_fence_after();
  const uint32_t tmem = *s_tmem;
  const volatile uint32_t* never = s_flags + 1;
  const bool skip = s_flags[0] != 0u;

  if (warp == 8) {
    // ------------------------------------------------------------ producer
    if (lane == 0 && !skip) {
      int lastA[kAStages] = {-1, -1, -1, -1}, lastB[kBStages] = {-1, -1};
      int ai = 0;
      bool ok = true;
      for (int c = 0; c < p.n_chunks && ok; ++c) {
        const int bs = c & 1;
        const uint32_t bpar = (c >> 1) & 1;
        if (!ptx::mbar_wait_bounded(&bars[B_EMPTY + bs], bpar ^ 1, gabort, kWaitLimitNs)) {
          record_failure(p.status, 70 + bs, c);
          break;
        }
        uint8_t* bdst = smem + kSmemB + bs * 2 * kBHalf;
        ptx::mbar_arrive_expect_tx(&bars[B_FULL + bs], 2 * kBHalf);
        ptx::tma_load_3d(bdst, &mW, &bars[B_FULL + bs], c * kChunk, 0, 2 * g);
        ptx::tma_load_3d(bdst + kBHalf, &mW, &bars[B_FULL + bs], c * kChunk, 0, 2 * g + 1);
        lastB[bs] = (int)bpar;
        const int sec = (c * kChunk) / p.d;
        const int off = c * kChunk - sec * p.d;
        const int nb = chunk_blocks(c, p.d, p.G);
        for (int b = 0; b < nb && ok; ++b) {
          for (int m = 0; m < 2; ++m, ++ai) {
            const int as = ai % kAStages;
            const uint32_t apar = (ai / kAStages) & 1;
            if (!ptx::mbar_wait_bounded(&bars[A_EMPTY + as], apar ^ 1, gabort, kWaitLimitNs)) {
              record_failure(p.status, 72, ai);
              ok = false;
              break;
            }
            uint8_t* adst = smem + kSmemA + as * kATile;
            const int row = (int)(t0 + m * kTile);
            ptx::mbar_arrive_expect_tx(&bars[A_FULL + as], kATile);
            if (sec == 0)
              ptx::tma_load_3d(adst, &mK, &bars[A_FULL + as], off, g, row);
            else if (sec == 1)
              ptx::tma_load_3d(adst, &mV, &bars[A_FULL + as], off, g, row);
            else
              ptx::tma_load_3d(adst, &mQ, &bars[A_FULL + as], off, g * p.G + b, row);
            lastA[as] = (int)apar;
          }
        }
      }
      for (int s = 0; s < kAStages; ++s)
        if (lastA[s] >= 0) ptx::mbar_wait_bounded(&bars[A_FULL + s], lastA[s], never, kWaitLimitNs);
      for (int s = 0; s < kBStages; ++s)
        if (lastB[s] >= 0) ptx::mbar_wait_bounded(&bars[B_FULL + s], lastB[s], never, kWaitLimitNs);
    }
  } else if (warp == 9) {
    // ------------------------------------------------------------ MMA issuer
    if (lane == 0 && !skip) {
      const uint32_t idesc = ptx::idesc_bf16_f32(kTile, kHid, 0);
      const uint32_t aA = ptx::smem_u32(smem + kSmemA);
      const uint32_t aB = ptx::smem_u32(smem + kSmemB);
      bool started[2] = {false, false};
      int ai = 0;
      bool ok = true;
      for (int c = 0; c < p.n_chunks && ok; ++c) {
        const int bs = c & 1;
        if (!ptx::mbar_wait_bounded(&bars[B_FULL + bs], (c >> 1) & 1, gabort, kWaitLimitNs)) {
          record_failure(p.status, 74, c);
          break;
        }
        ptx::tc_fence_after();
        const int nb = chunk_blocks(c, p.d, p.G);
        for (int b = 0; b < nb && ok; ++b) {
          for (int m = 0; m < 2; ++m, ++ai) {
            const int as = ai % kAStages;
            if (!ptx::mbar_wait_bounded(&bars[A_FULL + as], (ai / kAStages) & 1, gabort,
                                        kWaitLimitNs)) {
              record_failure(p.status, 75, ai);
              ok = false;
              break;
            }
            ptx::tc_fence_after();
#pragma unroll
            for (int ks = 0; ks < kChunk / 16; ++ks) {
#pragma unroll
              for (int part = 0; part < 2; ++part) {
                ptx::umma_bf16_ss(tmem + 256 * m,
                                  ptx::sdesc_sw128(aA + as * kATile + ks * 32, 16, 1024),
                                  ptx::sdesc_sw128(aB + bs * 2 * kBHalf + part * kBHalf + ks * 32,
                                                   16, 1024),
                                  idesc, started[m] ? 1u : 0u);
                started[m] = true;
              }
            }
            ptx::umma_commit(&bars[A_EMPTY + as]);
          }
        }
        if (ok) ptx::umma_commit(&bars[B_EMPTY + bs]);
      }
      if (ok) ptx::umma_commit(&bars[ACC_FULL]);
      ptx::umma_commit(&bars[DRAIN]);
      ptx::mbar_wait_bounded(&bars[DRAIN], 0, never, kWaitLimitNs);
    }
  } else if (!skip) {
    // ------------------------------------------------------------ epilogue
    const int m = warp >> 2;                        // token half
    const int row = threadIdx.x & 127;
    const uint32_t taddr = tmem + 256 * m + ((uint32_t)((warp & 3) * 32) << 16);
    bool ok = ptx::mbar_wait_bounded(&bars[ACC_FULL], 0, gabort, kWaitLimitNs);
    if (!__all_sync(0xffffffffu, ok)) {
      if (lane == 0) record_failure(p.status, 76, m);
    } else {
      ptx::tc_fence_after();
      float part = 0.f;
#pragma unroll 1
      for (int cc = 0; cc < kHid / 32; ++cc) {
        uint32_t z[32];
        APB_TMEM_LD32(taddr + 32 * cc, z);
#pragma unroll
        for (int x = 0; x < 32; ++x) {
          const float zz = __uint_as_float(z[x]) + s_b1[32 * cc + x];
          const float silu = __fdividef(zz, 1.0f + __expf(-zz));
          part = fmaf(s_w2[32 * cc + x], silu, part);
        }
      }
      const long long t = t0 + m * kTile + row;
      if (t < p.N) p.scores[(long long)g * p.N + t] = part + p.b2[g];
    }
  }

  ptx::tc_fence_before();
  __syncthreads();
  if (warp == 9) {
    ptx::tc_fence_after();
    ptx::tmem_dealloc(tmem, 512);
  }
}

}  // namespace

cudaError_t launch_score(const Shape& s, const void* q, const void* k, const void* v,
                         const float* w1, const float* b1, const float* w2, const float* b2,
                         float* scores, void* wsplit, float* qbias, DeviceStatus* status,
                         cudaStream_t st, const char** why) {
  const int F = 3 * s.d;
  const int G = s.Hq / s.Hkv;
  int dev = 0, sms = 148;
  cudaGetDevice(&dev);
  cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  split_weights_kernel<<<sms * 4, 256, 0, st>>>(w1, static_cast<__nv_bfloat16*>(wsplit), s.Hkv,
                                                F, s.d, G);
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return e;

  if (qbias) {
    query_bias_kernel<<<s.Hkv, 256, 0, st>>>(static_cast<const __nv_bfloat16*>(q), w1, b1, qbias,
                                             s.ql, s.Hq, G, s.d);
    e = cudaGetLastError();
    if (e != cudaSuccess) return e;
  }

  CUtensorMap mQ, mK, mV, mW;
  const uint64_t N = (uint64_t)s.N;
  bool ok = encode_bf16_3d(&mQ, q, s.d, s.Hq, N, (uint64_t)s.d * 2, (uint64_t)s.Hq * s.d * 2, 64,
                           1, kTile) &&
            encode_bf16_3d(&mK, k, s.d, s.Hkv, N, (uint64_t)s.d * 2, (uint64_t)s.Hkv * s.d * 2, 64,
                           1, kTile) &&
            encode_bf16_3d(&mV, v, s.d, s.Hkv, N, (uint64_t)s.d * 2, (uint64_t)s.Hkv * s.d * 2, 64,
                           1, kTile) &&
            encode_bf16_3d(&mW, wsplit, F, kHid, (uint64_t)s.Hkv * 2, (uint64_t)F * 2,
                           (uint64_t)kHid * F * 2, 64, kHid, 1);
  if (!ok) {
    *why = "cuTensorMapEncodeTiled failed (driver entry point or argument)";
    return cudaErrorInvalidValue;
  }
  ScoreParams p;
  p.N = s.N;
  p.Hq = s.Hq;
  p.Hkv = s.Hkv;
  p.G = G;
  p.d = s.d;
  p.F = F;
  // the query-aware variant stops after the k and v sections: its q section
  // is a per-head constant already folded into qbias
  p.n_chunks = (qbias ? 2 * s.d : F) / kChunk;
  p.b1 = qbias ? qbias : b1;
  p.w2 = w2;
  p.b2 = b2;
  p.scores = scores;
  p.status = status;
  e = cudaFuncSetAttribute(score_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, kSmemBytes);
  if (e != cudaSuccess) return e;
  dim3 grid((unsigned)((s.N + 2 * kTile - 1) / (2 * kTile)), s.Hkv);
  score_kernel<<<grid, kThreads, kSmemBytes, st>>>(mQ, mK, mV, mW, p);
  return cudaGetLastError();
}

}  // namespace apb

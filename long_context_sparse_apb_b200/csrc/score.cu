// Retaining-head stand-in scores on the tensor cores ("APB 的主要功能": each
// host compresses its KV with retaining heads).  For token t and kv head g:
//     x = [k[t,g] ; v[t,g] ; mean_{j in group g} q[t,j]]          (3d)
//     s[g,t] = w2[g] . SiLU(W1[g] x + b1[g]) + b2[g]
//
// The product W1 x must be fp32-accurate (the top-k that follows orders the
// scores), while the tensor cores multiply bf16.  Every operand is therefore
// split into bf16 parts whose products are accumulated in fp32:
//   * each fp32 weight w into hi + lo (hi = rn(w), lo = rn(w - hi)), leaving
//     |w - hi - lo| <= 2^-17 |w|;
//   * k and v are exact bf16 and multiply both weight parts;
//   * the group mean qbar (fp32 sum of G bf16 values, divided by G) into
//     qh + ql the same way, multiplied as qh.Wh + qh.Wl + ql.Wh (the dropped
//     ql.Wl term is below 2^-16 of the product).
// So Z = X W1^T takes 2 + 2 + 3 UMMA groups per 16 input features instead of
// one, with UMMA M = 128 tokens, N = 256 hidden, K = 16 accumulating in TMEM;
// the epilogue applies b1, SiLU, w2 and b2 in fp32.
//
// split_weights_kernel writes Wh, Wl ([Hkv, 2, hidden, 3d] bf16) into the
// workspace once per call.  score_kernel: one CTA = 256 tokens (two M = 128
// accumulators, TMEM columns [0,256) and [256,512)) of one kv head.  A
// 4-slot ring of A tiles (128 tokens x 64 features, 16 KB) is filled by TMA
// (warp 8) for the k and v features and, for the q features, by warps 0-7,
// which read the group's q heads from global memory, form qbar in fp32 and
// write qh and ql in the 128-byte-swizzled layout UMMA reads; warp 8 also
// streams the B tiles (Wh, Wl of one 64-feature chunk, 2 x 32 KB, 2 stages);
// warp 9 issues the UMMAs; warps 0-7 then run the epilogue, one token row per
// thread.  Waits are bounded like the attention kernel's.
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

// HANDOFF: the producer has issued its last A load.  A converter waiting on
// A_EMPTY before that could see the parity of a phase two completions old
// (its first use of a slot is the slot's third) and overwrite a k or v tile.
enum Bar {
  A_FULL = 0, A_EMPTY = 4, B_FULL = 8, B_EMPTY = 10, ACC_FULL = 12, DRAIN = 13, HANDOFF = 14,
  NUM = 15
};

__global__ void __launch_bounds__(256) split_weights_kernel(const float* __restrict__ w1,
                                                            __nv_bfloat16* __restrict__ ws,
                                                            int Hkv, int F) {
  const long long per_head = (long long)kHid * F;
  const long long total = (long long)Hkv * per_head;
  for (long long i = (long long)blockIdx.x * blockDim.x + threadIdx.x; i < total;
       i += (long long)gridDim.x * blockDim.x) {
    const long long g = i / per_head;
    const long long rem = i - g * per_head;
    const float w = w1[i];
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
  const __nv_bfloat16* q;
  const float* b1;
  const float* w2;
  const float* b2;
  float* scores;
  DeviceStatus* status;
};

// Section of feature chunk c: 0 k, 1 v, 2 q.  A k or v chunk takes one A
// tile per 128-token half (by TMA); a q chunk two (qh, ql) per half.
__device__ __forceinline__ int chunk_section(int c, int d) { return (c * kChunk) / d; }

// q features [off, off + 64) of one 128-token tile, in warps 0-7: thread tid
// forms the group mean of 8 features (16 bytes of a row) for the 4 tokens
// tid / 8 + 32 i, in fp32, and splits it into bf16 hi + lo.
struct QTile {
  uint32_t hi[4][4], lo[4][4];
};

__device__ __forceinline__ void q_tile_mean(const ScoreParams& p, long long row0, int g, int off,
                                            float invG, QTile& o) {
  const int tid = threadIdx.x;
  const int piece = tid & 7;
  const int rbase = tid >> 3;
  float acc[4][8];
#pragma unroll
  for (int i = 0; i < 4; ++i)
#pragma unroll
    for (int e = 0; e < 8; ++e) acc[i][e] = 0.f;
  const long long head_stride = (long long)p.d;               // elements
  const long long row_stride = (long long)p.Hq * p.d;
  const __nv_bfloat16* base = p.q + (long long)g * p.G * head_stride + off + piece * 8;
#pragma unroll 1
  for (int j0 = 0; j0 < p.G; j0 += 4) {
    uint4 raw[4][4];
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      const long long t = row0 + rbase + 32 * i;
#pragma unroll
      for (int u = 0; u < 4; ++u) {
        raw[i][u] = make_uint4(0u, 0u, 0u, 0u);
        if (t < p.N && j0 + u < p.G)
          raw[i][u] = __ldg(reinterpret_cast<const uint4*>(base + t * row_stride +
                                                           (long long)(j0 + u) * head_stride));
      }
    }
#pragma unroll
    for (int i = 0; i < 4; ++i)
#pragma unroll
      for (int u = 0; u < 4; ++u) {
        const uint32_t w[4] = {raw[i][u].x, raw[i][u].y, raw[i][u].z, raw[i][u].w};
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          acc[i][2 * e] += __uint_as_float(w[e] << 16);
          acc[i][2 * e + 1] += __uint_as_float(w[e] & 0xffff0000u);
        }
      }
  }
#pragma unroll
  for (int i = 0; i < 4; ++i)
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      const float x0 = acc[i][2 * e] * invG, x1 = acc[i][2 * e + 1] * invG;
      const __nv_bfloat162 h = __floats2bfloat162_rn(x0, x1);
      const __nv_bfloat162 l = __floats2bfloat162_rn(x0 - __low2float(h), x1 - __high2float(h));
      o.hi[i][e] = *reinterpret_cast<const uint32_t*>(&h);
      o.lo[i][e] = *reinterpret_cast<const uint32_t*>(&l);
    }
}

// Writes a QTile into two A slots in the 128-byte-swizzled K-major layout
// UMMA reads (16-byte chunk index XOR row % 8 inside each 1024-byte group of
// 8 rows: what a TMA load with 128-byte swizzle would have written).
__device__ __forceinline__ void q_tile_store(const QTile& o, uint8_t* slot_h, uint8_t* slot_l) {
  const int piece = threadIdx.x & 7;
  const int rbase = threadIdx.x >> 3;
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const int r = rbase + 32 * i;
    const int at = r * 128 + ((piece ^ (r & 7)) << 4);
    *reinterpret_cast<uint4*>(slot_h + at) = make_uint4(o.hi[i][0], o.hi[i][1], o.hi[i][2], o.hi[i][3]);
    *reinterpret_cast<uint4*>(slot_l + at) = make_uint4(o.lo[i][0], o.lo[i][1], o.lo[i][2], o.lo[i][3]);
  }
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
  const int q_chunk0 = 2 * p.d / kChunk;      // first chunk of the q section
  const int q_slot0 = 2 * q_chunk0;           // its first A slot (k and v: 2 per chunk)

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
      // the q rows the converters read, into L2 ahead of them
      for (int c = q_chunk0; c < p.n_chunks; ++c)
        for (int j = 0; j < p.G; ++j)
          for (int m = 0; m < 2; ++m)
            ptx::tma_prefetch_l2_3d(&mQ, c * kChunk - 2 * p.d, g * p.G + j,
                                    (int)(t0 + m * kTile));
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
        const int sec = chunk_section(c, p.d);
        if (sec == 2) {       // q slots are filled by the converter warps
          ai += 4;
          continue;
        }
        const int off = c * kChunk - sec * p.d;
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
          ptx::tma_load_3d(adst, sec == 0 ? &mK : &mV, &bars[A_FULL + as], off, g, row);
          lastA[as] = (int)apar;
        }
        if (ok && c == q_chunk0 - 1) ptx::mbar_arrive(&bars[HANDOFF]);
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
        const uint32_t bh = aB + bs * 2 * kBHalf, bl = bh + kBHalf;
        const bool qsec = chunk_section(c, p.d) == 2;
        for (int m = 0; m < 2 && ok; ++m) {
          // k, v: one A slot (x, exact bf16); q: two (qh, ql)
          const int nslots = qsec ? 2 : 1;
          for (int u = 0; u < nslots; ++u) {
            const int as = (ai + u) % kAStages;
            if (!ptx::mbar_wait_bounded(&bars[A_FULL + as], ((ai + u) / kAStages) & 1, gabort,
                                        kWaitLimitNs)) {
              record_failure(p.status, 75, ai + u);
              ok = false;
            }
            if (!ok) break;
          }
          if (!ok) break;
          ptx::tc_fence_after();
          const uint32_t ah = aA + (ai % kAStages) * kATile;
          const uint32_t al = aA + ((ai + 1) % kAStages) * kATile;
          const uint32_t acc = tmem + 256 * m;
#pragma unroll
          for (int ks = 0; ks < kChunk / 16; ++ks) {
            const uint64_t dAh = ptx::sdesc_sw128(ah + ks * 32, 16, 1024);
            const uint64_t dBh = ptx::sdesc_sw128(bh + ks * 32, 16, 1024);
            const uint64_t dBl = ptx::sdesc_sw128(bl + ks * 32, 16, 1024);
            ptx::umma_bf16_ss(acc, dAh, dBh, idesc, started[m] ? 1u : 0u);
            started[m] = true;
            ptx::umma_bf16_ss(acc, dAh, dBl, idesc, 1u);
            if (qsec)
              ptx::umma_bf16_ss(acc, ptx::sdesc_sw128(al + ks * 32, 16, 1024), dBh, idesc, 1u);
          }
          for (int u = 0; u < nslots; ++u) ptx::umma_commit(&bars[A_EMPTY + (ai + u) % kAStages]);
          ai += nslots;
        }
        if (ok) ptx::umma_commit(&bars[B_EMPTY + bs]);
      }
      if (ok) ptx::umma_commit(&bars[ACC_FULL]);
      ptx::umma_commit(&bars[DRAIN]);
      ptx::mbar_wait_bounded(&bars[DRAIN], 0, never, kWaitLimitNs);
    }
  } else if (!skip) {
    // ---------------------------------------------- q converters, then epilogue
    {
      const float invG = 1.0f / (float)p.G;     // exact for G = 2^k
      int ai = q_slot0;
      for (int c = q_chunk0; c < p.n_chunks; ++c) {
        bool ok = true;
        for (int m = 0; m < 2; ++m, ai += 2) {
          const int sh = ai % kAStages, sl = (ai + 1) % kAStages;
          const uint32_t par = ((ai / kAStages) & 1) ^ 1;
          // loads first: their latency overlaps the wait for the slots
          QTile qt;
          q_tile_mean(p, t0 + m * kTile, g, c * kChunk - 2 * p.d, invG, qt);
          if (threadIdx.x == 0) {
            ok = (ai != q_slot0 ||
                  ptx::mbar_wait_bounded(&bars[HANDOFF], 0, gabort, kWaitLimitNs)) &&
                 ptx::mbar_wait_bounded(&bars[A_EMPTY + sh], par, gabort, kWaitLimitNs) &&
                 ptx::mbar_wait_bounded(&bars[A_EMPTY + sl], par, gabort, kWaitLimitNs);
            if (!ok) record_failure(p.status, 77, ai);
          }
          ok = ptx::barrier_and(1, 256, ok);
          if (!ok) break;
          q_tile_store(qt, smem + kSmemA + sh * kATile, smem + kSmemA + sl * kATile);
          ptx::fence_proxy_async_smem();
          ptx::named_barrier_sync(1, 256);
          if (threadIdx.x == 0) {
            ptx::mbar_arrive(&bars[A_FULL + sh]);
            ptx::mbar_arrive(&bars[A_FULL + sl]);
          }
        }
        if (!ok) break;
      }
    }
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
                                                F);
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
  p.q = static_cast<const __nv_bfloat16*>(q);
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

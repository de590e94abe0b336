// Retaining-head stand-in scores ("APB 的主要功能": each host compresses its
// KV with retaining heads).  For token t and kv head g:
//     x = [k[t,g] ; v[t,g] ; mean_{j in group g} q[t,j]]         (3d, fp32)
//     s[g,t] = w2[g] . SiLU(W1[g] x + b1[g]) + b2[g]
// computed in fp32 on the CUDA cores (the top-k that follows needs fp32-level
// ordering of the scores).
//
// Tiling: a CTA owns 64 tokens of one kv head and all 256 hidden units, i.e.
// a [64 x 3d] x [3d x 256] product.  The 3d input features stream through
// shared memory in chunks of 32: the token chunk is gathered from bf16 K, V
// and the G q heads of the group (averaged in fp32), the W1 chunk is read
// along its contiguous feature axis and stored transposed.  Each of the 256
// threads accumulates a 4-token x 16-hidden register tile; the epilogue
// applies b1, SiLU and w2 and reduces the 16 hidden groups with shuffles.
#include <cuda_bf16.h>

#include "apb_internal.h"

namespace apb {
namespace {

constexpr int kTok = 64;        // tokens per CTA
constexpr int kHid = 256;       // hidden units (all of them)
constexpr int kChunk = 32;      // input features per shared-memory chunk
constexpr int kXLd = kTok + 4;  // padded row of the transposed token chunk
constexpr int kThreads = 256;

__device__ __forceinline__ void bf16x8_to_f32(const uint4& u, float* f) {
  const __nv_bfloat162* p = reinterpret_cast<const __nv_bfloat162*>(&u);
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    float2 t = __bfloat1622float2(p[i]);
    f[2 * i] = t.x;
    f[2 * i + 1] = t.y;
  }
}

__global__ void __launch_bounds__(kThreads, 2) score_kernel(
    const __nv_bfloat16* __restrict__ q, const __nv_bfloat16* __restrict__ k,
    const __nv_bfloat16* __restrict__ v, const float* __restrict__ w1,
    const float* __restrict__ b1, const float* __restrict__ w2, const float* __restrict__ b2,
    float* __restrict__ scores, long long N, int Hq, int Hkv, int d) {
  __shared__ __align__(16) float xs[kChunk][kXLd];
  __shared__ __align__(16) float ws[kChunk][kHid];

  const int g = blockIdx.y;
  const long long t0 = (long long)blockIdx.x * kTok;
  const int G = Hq / Hkv;
  const int F = 3 * d;
  const int tid = threadIdx.x;
  const int tg = tid >> 4;    // token group: tokens 4*tg .. 4*tg+3
  const int hg = tid & 15;    // hidden group: units 4*hg + 64*i + j
  const float* w1g = w1 + (long long)g * kHid * F;

  float acc[4][16];
#pragma unroll
  for (int a = 0; a < 4; ++a)
#pragma unroll
    for (int b = 0; b < 16; ++b) acc[a][b] = 0.f;

  // loader roles
  const int ld_tok = tid >> 2;          // 0..63
  const int ld_part = tid & 3;          // 8 features each
  const long long ld_t = t0 + ld_tok;
  const bool ld_ok = ld_t < N;
  const float invG = 1.0f / (float)G;

  for (int f0 = 0; f0 < F; f0 += kChunk) {
    // ---- token chunk: features [f0, f0+32) of 64 tokens
    {
      const int sec = f0 / d;            // 0: k, 1: v, 2: mean q
      const int off = f0 - sec * d + ld_part * 8;
      float f[8];
      if (!ld_ok) {
#pragma unroll
        for (int i = 0; i < 8; ++i) f[i] = 0.f;
      } else if (sec < 2) {
        const __nv_bfloat16* base = (sec == 0 ? k : v) + (ld_t * Hkv + g) * d + off;
        bf16x8_to_f32(__ldg(reinterpret_cast<const uint4*>(base)), f);
      } else {
        float s8[8];
#pragma unroll
        for (int i = 0; i < 8; ++i) f[i] = 0.f;
        for (int j = 0; j < G; ++j) {
          const __nv_bfloat16* base = q + (ld_t * Hq + (long long)g * G + j) * d + off;
          bf16x8_to_f32(__ldg(reinterpret_cast<const uint4*>(base)), s8);
#pragma unroll
          for (int i = 0; i < 8; ++i) f[i] += s8[i];
        }
        if ((G & (G - 1)) == 0) {
#pragma unroll
          for (int i = 0; i < 8; ++i) f[i] *= invG;
        } else {
#pragma unroll
          for (int i = 0; i < 8; ++i) f[i] = __fdiv_rn(f[i], (float)G);
        }
      }
#pragma unroll
      for (int i = 0; i < 8; ++i) xs[ld_part * 8 + i][ld_tok] = f[i];
    }
    // ---- W1 chunk: thread = hidden unit, 32 contiguous features, transposed
    {
      const float4* wrow = reinterpret_cast<const float4*>(w1g + (long long)tid * F + f0);
#pragma unroll
      for (int c = 0; c < kChunk / 4; ++c) {
        float4 w = __ldg(wrow + c);
        ws[4 * c + 0][tid] = w.x;
        ws[4 * c + 1][tid] = w.y;
        ws[4 * c + 2][tid] = w.z;
        ws[4 * c + 3][tid] = w.w;
      }
    }
    __syncthreads();
#pragma unroll 4
    for (int kk = 0; kk < kChunk; ++kk) {
      const float4 xa = *reinterpret_cast<const float4*>(&xs[kk][tg * 4]);
      const float xr[4] = {xa.x, xa.y, xa.z, xa.w};
      float wr[16];
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        const float4 w = *reinterpret_cast<const float4*>(&ws[kk][hg * 4 + 64 * i]);
        wr[4 * i + 0] = w.x;
        wr[4 * i + 1] = w.y;
        wr[4 * i + 2] = w.z;
        wr[4 * i + 3] = w.w;
      }
#pragma unroll
      for (int a = 0; a < 4; ++a)
#pragma unroll
        for (int b = 0; b < 16; ++b) acc[a][b] = fmaf(xr[a], wr[b], acc[a][b]);
    }
    __syncthreads();
  }

  // ---- epilogue: b1, SiLU, w2, reduce over the 16 hidden groups
  const float* b1g = b1 + (long long)g * kHid;
  const float* w2g = w2 + (long long)g * kHid;
  float bb[16], ww[16];
#pragma unroll
  for (int i = 0; i < 4; ++i)
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      const int u = hg * 4 + 64 * i + j;
      bb[4 * i + j] = __ldg(b1g + u);
      ww[4 * i + j] = __ldg(w2g + u);
    }
  const float bias2 = __ldg(b2 + g);
#pragma unroll
  for (int a = 0; a < 4; ++a) {
    float part = 0.f;
#pragma unroll
    for (int b = 0; b < 16; ++b) {
      const float z = acc[a][b] + bb[b];
      const float silu = z / (1.0f + expf(-z));
      part = fmaf(ww[b], silu, part);
    }
#pragma unroll
    for (int o = 8; o >= 1; o >>= 1) part += __shfl_xor_sync(0xffffffffu, part, o);
    const long long t = t0 + tg * 4 + a;
    if (hg == 0 && t < N) scores[(long long)g * N + t] = part + bias2;
  }
}

}  // namespace

cudaError_t launch_score(const Shape& s, const void* q, const void* k, const void* v,
                         const float* w1, const float* b1, const float* w2, const float* b2,
                         float* scores, cudaStream_t st) {
  dim3 grid((unsigned)((s.N + kTok - 1) / kTok), s.Hkv);
  score_kernel<<<grid, kThreads, 0, st>>>(
      static_cast<const __nv_bfloat16*>(q), static_cast<const __nv_bfloat16*>(k),
      static_cast<const __nv_bfloat16*>(v), w1, b1, w2, b2, scores, s.N, s.Hq, s.Hkv, s.d);
  return cudaGetLastError();
}

}  // namespace apb

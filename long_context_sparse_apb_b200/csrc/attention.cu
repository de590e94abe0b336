// Block-masked prefill attention of APB on sm_100a ("APB 的主要功能":
// computation over the anchor block, the passing block and the local block;
// the passing block is not kept afterwards).
//
// One CTA computes one 128-row query tile of one q head of one host.  Its KV
// sequence is three ranges, walked as 128-row tiles:
//   anchor  : k[0:A, g]             (hosts h >= 1)      full visibility
//   passing : pass_k[g, 0:h*keep]                       full visibility
//   local   : k[h*n : h*n + q0 + 128, g]                causal, diagonal kept
// so masked tiles beyond the diagonal are never visited and only the last
// tile of each range needs a mask.
//
// Warp roles (192 threads):
//   warps 0-3  softmax + epilogue; thread r owns query row r, which is also
//              TMEM lane r of every accumulator;
//   warp 4     TMA producer (Q once, then K and V tiles into 2-stage rings);
//   warp 5     TMEM allocator and the single UMMA-issuing thread.
// TMEM columns: S0 [0,128), S1 [128,256), O [256, 256+d).
// Per KV tile j:   S(j) = Q K(j)^T            (tcgen05.mma, into S[j&1])
//                  softmax reads S(j), writes P(j) (bf16, SW128 K-major) to
//                  shared memory, rescales O in TMEM when the running max
//                  grew by more than 2^8 (lazy rescaling), signals P_FULL;
//                  O += P(j) V(j)          (A = P from smem, B = V MN-major)
// The MMA thread issues S(j+2) right after PV(j), so the tensor core works
// on the next score tile while the softmax warps process the current one.
//
// Every mbarrier wait is bounded (wall-clock limit plus a launch-wide abort
// flag); a wait that runs out records an error in the status block, the CTA
// drains its outstanding TMA loads and MMAs, frees TMEM and returns.
#include <cuda_bf16.h>
#include <cudaTypedefs.h>

#include <mutex>

#include "apb_internal.h"
#include "sm100_ptx.cuh"

namespace apb {
namespace {

constexpr int kRows = 128;                    // query rows per tile = KV rows per tile
constexpr int kThreads = 192;
constexpr uint64_t kWaitLimitNs = 1000000000ull;   // 1 s per wait
constexpr float kLog2e = 1.4426950408889634f;
constexpr float kRescaleThreshold = 8.0f;     // log2 units

enum Bar {
  Q_FULL = 0,
  K_FULL = 1,    // 2 stages
  K_EMPTY = 3,   // 2
  V_FULL = 5,    // 2
  V_EMPTY = 7,   // 2
  S_FULL = 9,    // 2
  P_FULL = 11,
  O_DONE = 12,
  DRAIN = 13,
  NUM_BARS = 14
};

template <int D>
struct Layout {
  static constexpr int kTile = kRows * D * 2;   // bytes of one Q/K/V tile
  static constexpr int kP = kRows * kRows * 2;  // bytes of the P tile
  static constexpr int kQ = 0;
  static constexpr int kK0 = kTile;
  static constexpr int kV0 = 3 * kTile;
  static constexpr int kPoff = 5 * kTile;
  static constexpr int kBars = kPoff + kP;
  static constexpr int kBytes = kBars + 256;
};
// Both head sizes request the d = 128 footprint so that one CTA runs per SM
// (each CTA allocates all 512 TMEM columns).
constexpr int kSmemBytes = Layout<128>::kBytes + 1024;

struct Params {
  int H, n, A, keep, Hq, Hkv, G, n_qtiles;
  long long N;
  float scale_log2;
  __nv_bfloat16* out;
  float* lse;
  DeviceStatus* status;
};

__device__ void record_failure(DeviceStatus* st, uint32_t where, uint32_t tile) {
  if (atomicOr(&st->sticky, kErrWaitTimeout) == 0u) {
    st->where = where;
    st->tile = tile;
  }
  atomicExch(&st->abort, 1u);
  __threadfence();
}

template <int D>
__device__ __forceinline__ void load_kv_tile(const CUtensorMap* m_kv, const CUtensorMap* m_pass,
                                             uint8_t* dst, uint64_t* bar, int j, int na, int np,
                                             int g, int local_row0) {
  if (j < na) {
#pragma unroll
    for (int kb = 0; kb < D / 64; ++kb)
      ptx::tma_load_3d(dst + kb * (kRows * 128), m_kv, bar, kb * 64, g, j * kRows);
  } else if (j < na + np) {
#pragma unroll
    for (int kb = 0; kb < D / 64; ++kb)
      ptx::tma_load_3d(dst + kb * (kRows * 128), m_pass, bar, kb * 64, (j - na) * kRows, g);
  } else {
#pragma unroll
    for (int kb = 0; kb < D / 64; ++kb)
      ptx::tma_load_3d(dst + kb * (kRows * 128), m_kv, bar, kb * 64, g,
                       local_row0 + (j - na - np) * kRows);
  }
}

template <int D>
__global__ void __launch_bounds__(kThreads, 1)
    apb_attention_kernel(const __grid_constant__ CUtensorMap mQ,
                         const __grid_constant__ CUtensorMap mK,
                         const __grid_constant__ CUtensorMap mV,
                         const __grid_constant__ CUtensorMap mPK,
                         const __grid_constant__ CUtensorMap mPV, const Params p) {
  using L = Layout<D>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + L::kBars);
  uint32_t* s_tmem = reinterpret_cast<uint32_t*>(bars + 16);
  uint32_t* s_flags = s_tmem + 1;   // [0]: launch already aborted, [1]: constant 0

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;

  // heavy units first: the last query tiles of the last hosts
  const int t = p.n_qtiles - 1 - (int)blockIdx.x;
  const int head = (int)blockIdx.y;
  const int h = p.H - 1 - (int)blockIdx.z;
  const int g = head / p.G;
  const int q0 = t * kRows;
  const int na = (h >= 1 && p.A > 0) ? (p.A + kRows - 1) / kRows : 0;
  const int P = h * p.keep;
  const int np = (P + kRows - 1) / kRows;
  const int T = na + np + t + 1;
  const int local_row0 = h * p.n;        // first K row of this host's block

  const volatile uint32_t* gabort = &p.status->abort;

  if (threadIdx.x == 0) {
    for (int i = 0; i < NUM_BARS; ++i) ptx::mbar_init(&bars[i], 1);
    ptx::mbar_init(&bars[P_FULL], 128);
    ptx::fence_mbar_init();
    s_flags[0] = *gabort;
    s_flags[1] = 0u;
  }
  if (warp == 5) {
    ptx::tmem_alloc(s_tmem, 512);
    ptx::tmem_relinquish();
  }
  if (warp == 4 && lane == 0) {
    ptx::tma_prefetch_desc(&mQ);
    ptx::tma_prefetch_desc(&mK);
    ptx::tma_prefetch_desc(&mV);
    ptx::tma_prefetch_desc(&mPK);
    ptx::tma_prefetch_desc(&mPV);
  }
  ptx::tc_fence_before();
  __syncthreads();
  ptx::tc_fence_after();
  const uint32_t tmem = *s_tmem;
  const volatile uint32_t* never = s_flags + 1;
  const bool skip = s_flags[0] != 0u;

  uint8_t* sQ = smem + L::kQ;
  uint8_t* sK0 = smem + L::kK0;   // stage s at sK0 + s * kTile
  uint8_t* sV0 = smem + L::kV0;
  uint8_t* sP = smem + L::kPoff;

  if (warp == 4) {
    // ------------------------------------------------------------ producer
    if (lane == 0 && !skip) {
      int lastK[2] = {-1, -1}, lastV[2] = {-1, -1};   // parity of the last load per slot
      ptx::mbar_arrive_expect_tx(&bars[Q_FULL], L::kTile);
#pragma unroll
      for (int kb = 0; kb < D / 64; ++kb)
        ptx::tma_load_3d(sQ + kb * (kRows * 128), &mQ, &bars[Q_FULL], kb * 64, head,
                         local_row0 + q0);
      for (int j = 0; j < T; ++j) {
        const int s = j & 1;
        const uint32_t par = (j >> 1) & 1;
        if (!ptx::mbar_wait_bounded(&bars[K_EMPTY + s], par ^ 1, gabort, kWaitLimitNs)) {
          record_failure(p.status, 40 + s, j);
          break;
        }
        ptx::mbar_arrive_expect_tx(&bars[K_FULL + s], L::kTile);
        load_kv_tile<D>(&mK, &mPK, sK0 + s * L::kTile, &bars[K_FULL + s], j, na, np, g, local_row0);
        lastK[s] = (int)par;
        if (!ptx::mbar_wait_bounded(&bars[V_EMPTY + s], par ^ 1, gabort, kWaitLimitNs)) {
          record_failure(p.status, 42 + s, j);
          break;
        }
        ptx::mbar_arrive_expect_tx(&bars[V_FULL + s], L::kTile);
        load_kv_tile<D>(&mV, &mPV, sV0 + s * L::kTile, &bars[V_FULL + s], j, na, np, g, local_row0);
        lastV[s] = (int)par;
      }
      // drain: every load issued must have landed before the CTA exits
      ptx::mbar_wait_bounded(&bars[Q_FULL], 0, never, kWaitLimitNs);
      for (int s = 0; s < 2; ++s) {
        if (lastK[s] >= 0) ptx::mbar_wait_bounded(&bars[K_FULL + s], lastK[s], never, kWaitLimitNs);
        if (lastV[s] >= 0) ptx::mbar_wait_bounded(&bars[V_FULL + s], lastV[s], never, kWaitLimitNs);
      }
    }
  } else if (warp == 5) {
    // ------------------------------------------------------------ MMA issuer
    if (lane == 0 && !skip) {
      const uint32_t idesc_s = ptx::idesc_bf16_f32(kRows, kRows, 0);
      const uint32_t idesc_pv = ptx::idesc_bf16_f32(kRows, D, 1);
      const uint32_t aQ = ptx::smem_u32(sQ), aP = ptx::smem_u32(sP);
      const uint32_t aK0 = ptx::smem_u32(sK0), aV0 = ptx::smem_u32(sV0);
      const uint32_t tO = tmem + 256;
      bool ok = ptx::mbar_wait_bounded(&bars[Q_FULL], 0, gabort, kWaitLimitNs);
      if (!ok) record_failure(p.status, 50, 0);

      auto issue_s = [&](int jj) -> bool {
        const int s = jj & 1;
        if (!ptx::mbar_wait_bounded(&bars[K_FULL + s], (jj >> 1) & 1, gabort, kWaitLimitNs)) {
          record_failure(p.status, 51 + s, jj);
          return false;
        }
        ptx::tc_fence_after();
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk) {
          const uint32_t off = (kk >> 2) * (kRows * 128) + (kk & 3) * 32;
          ptx::umma_bf16_ss(tmem + 128 * s, ptx::sdesc_sw128(aQ + off, 16, 1024),
                            ptx::sdesc_sw128(aK0 + s * L::kTile + off, 16, 1024), idesc_s,
                            kk > 0);
        }
        ptx::umma_commit(&bars[K_EMPTY + s]);
        ptx::umma_commit(&bars[S_FULL + s]);
        return true;
      };

      if (ok) ok = issue_s(0);
      if (ok && T > 1) ok = issue_s(1);
      for (int j = 0; ok && j < T; ++j) {
        const int s = j & 1;
        if (!ptx::mbar_wait_bounded(&bars[P_FULL], j & 1, gabort, kWaitLimitNs)) {
          record_failure(p.status, 53, j);
          break;
        }
        if (!ptx::mbar_wait_bounded(&bars[V_FULL + s], (j >> 1) & 1, gabort, kWaitLimitNs)) {
          record_failure(p.status, 54 + s, j);
          break;
        }
        ptx::tc_fence_after();
#pragma unroll
        for (int kk = 0; kk < kRows / 16; ++kk) {
          const uint32_t offp = (kk >> 2) * (kRows * 128) + (kk & 3) * 32;
          ptx::umma_bf16_ss(tO, ptx::sdesc_sw128(aP + offp, 16, 1024),
                            ptx::sdesc_sw128(aV0 + s * L::kTile + kk * 2048, kRows * 128, 1024), idesc_pv,
                            (j > 0 || kk > 0) ? 1u : 0u);
        }
        ptx::umma_commit(&bars[V_EMPTY + s]);
        ptx::umma_commit(&bars[O_DONE]);
        if (j + 2 < T) ok = issue_s(j + 2);
      }
      // drain every MMA issued so far
      ptx::umma_commit(&bars[DRAIN]);
      ptx::mbar_wait_bounded(&bars[DRAIN], 0, never, kWaitLimitNs);
    }
  } else if (!skip) {
    // ------------------------------------------------------------ softmax
    const int row = threadIdx.x;                       // 0..127
    const uint32_t lane_off = (uint32_t)(warp * 32) << 16;
    const uint32_t tS0 = tmem + lane_off;   // S buffer s at tS0 + 128 * s
    const uint32_t tO = tmem + 256 + lane_off;
    uint8_t* prow = sP + row * 128;
    const int swz = row & 7;
    float m = -INFINITY, l = 0.f;
    bool ok = true;
    for (int j = 0; j < T; ++j) {
      const int s = j & 1;
      ok = ptx::mbar_wait_bounded(&bars[S_FULL + s], (j >> 1) & 1, gabort, kWaitLimitNs);
      if (!__all_sync(0xffffffffu, ok)) {
        if (lane == 0) record_failure(p.status, 60 + s, j);
        ok = false;
        break;
      }
      ptx::tc_fence_after();
      uint32_t sr[128];
#pragma unroll
      for (int c = 0; c < 4; ++c) {
        uint32_t* r = sr + 32 * c;
        APB_TMEM_LD32(tS0 + 128 * s + 32 * c, r);
      }
      // visible columns of this row in this tile
      int lim;
      if (j < na) {
        lim = min(kRows, p.A - j * kRows);
      } else if (j < na + np) {
        lim = min(kRows, P - (j - na) * kRows);
      } else {
        lim = (j == T - 1) ? row + 1 : kRows;
      }
      if (lim < kRows) {
#pragma unroll
        for (int c = 0; c < kRows; ++c)
          if (c >= lim) sr[c] = 0xff800000u;   // -inf
      }
      float mx[8];
#pragma unroll
      for (int i = 0; i < 8; ++i) mx[i] = __uint_as_float(sr[i]);
#pragma unroll
      for (int c = 8; c < kRows; ++c) mx[c & 7] = fmaxf(mx[c & 7], __uint_as_float(sr[c]));
      float tmax = fmaxf(fmaxf(fmaxf(mx[0], mx[1]), fmaxf(mx[2], mx[3])),
                         fmaxf(fmaxf(mx[4], mx[5]), fmaxf(mx[6], mx[7])));
      const float m_tile = tmax * p.scale_log2;
      float alpha = 1.f;
      bool rescale = false;
      if (j == 0) {
        m = m_tile;
      } else if (m_tile > m + kRescaleThreshold) {
        alpha = ptx::ex2(m - m_tile);
        m = m_tile;
        l *= alpha;
        rescale = true;
      }
      const float mneg = -m;
      uint32_t pk[64];
      float sum[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
      for (int c = 0; c < 64; ++c) {
        const float p0 = ptx::ex2(fmaf(__uint_as_float(sr[2 * c]), p.scale_log2, mneg));
        const float p1 = ptx::ex2(fmaf(__uint_as_float(sr[2 * c + 1]), p.scale_log2, mneg));
        sum[c & 3] += p0 + p1;
        pk[c] = ptx::pack_bf16x2(p0, p1);
      }
      l += (sum[0] + sum[1]) + (sum[2] + sum[3]);
      // P buffer and O are free once PV(j-1) has completed
      if (j > 0) {
        ok = ptx::mbar_wait_bounded(&bars[O_DONE], (j - 1) & 1, gabort, kWaitLimitNs);
        if (!__all_sync(0xffffffffu, ok)) {
          if (lane == 0) record_failure(p.status, 62, j);
          ok = false;
          break;
        }
      }
      if (__any_sync(0xffffffffu, rescale)) {
        ptx::tc_fence_after();
#pragma unroll
        for (int c = 0; c < D / 32; ++c) {
          uint32_t o[32];
          APB_TMEM_LD32(tO + 32 * c, o);
#pragma unroll
          for (int i = 0; i < 32; ++i) o[i] = __float_as_uint(__uint_as_float(o[i]) * alpha);
          APB_TMEM_ST32(tO + 32 * c, o);
        }
        ptx::tmem_st_wait();
      }
#pragma unroll
      for (int c8 = 0; c8 < 16; ++c8) {
        const int kb = c8 >> 3, ch = c8 & 7;
        uint4 val = make_uint4(pk[4 * c8], pk[4 * c8 + 1], pk[4 * c8 + 2], pk[4 * c8 + 3]);
        *reinterpret_cast<uint4*>(prow + kb * (kRows * 128) + ((ch ^ swz) << 4)) = val;
      }
      ptx::fence_proxy_async_smem();
      ptx::tc_fence_before();
      ptx::mbar_arrive(&bars[P_FULL]);
    }
    if (ok) {
      ok = ptx::mbar_wait_bounded(&bars[O_DONE], (T - 1) & 1, gabort, kWaitLimitNs);
      if (!__all_sync(0xffffffffu, ok)) {
        if (lane == 0) record_failure(p.status, 63, T);
        ok = false;
      }
    }
    if (ok) {
      ptx::tc_fence_after();
      const float inv = 1.0f / l;
      const bool valid = q0 + row < p.n;
      const long long tok = (long long)local_row0 + q0 + row;
      __nv_bfloat16* orow = p.out + (tok * p.Hq + head) * D;
#pragma unroll
      for (int c = 0; c < D / 32; ++c) {
        uint32_t o[32];
        APB_TMEM_LD32(tO + 32 * c, o);
        uint32_t w[16];
#pragma unroll
        for (int i = 0; i < 16; ++i)
          w[i] = ptx::pack_bf16x2(__uint_as_float(o[2 * i]) * inv,
                                  __uint_as_float(o[2 * i + 1]) * inv);
        if (valid) {
          uint4* dst = reinterpret_cast<uint4*>(orow + 32 * c);
#pragma unroll
          for (int i = 0; i < 4; ++i)
            dst[i] = make_uint4(w[4 * i], w[4 * i + 1], w[4 * i + 2], w[4 * i + 3]);
        }
      }
      if (p.lse && valid) p.lse[(long long)head * p.N + tok] = (m + __log2f(l)) * 0.6931471805599453f;
    }
  }

  ptx::tc_fence_before();
  __syncthreads();
  if (warp == 5) {
    ptx::tc_fence_after();
    ptx::tmem_dealloc(tmem, 512);
  }
}

// ---------------------------------------------------------------- host side

PFN_cuTensorMapEncodeTiled_v12000 encode_fn() {
  static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* ptr = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPointByVersion("cuTensorMapEncodeTiled", &ptr, 12000, cudaEnableDefault,
                                         &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(ptr);
  });
  return fn;
}

bool encode_bf16_3d(CUtensorMap* m, const void* base, uint64_t d0, uint64_t d1, uint64_t d2,
                    uint64_t stride1_bytes, uint64_t stride2_bytes, uint32_t b0, uint32_t b1,
                    uint32_t b2) {
  auto fn = encode_fn();
  if (!fn) return false;
  cuuint64_t dims[3] = {d0, d1, d2};
  cuuint64_t strides[2] = {stride1_bytes, stride2_bytes};
  cuuint32_t box[3] = {b0, b1, b2};
  cuuint32_t estr[3] = {1, 1, 1};
  CUresult r = fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(base), dims, strides,
                  box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                  CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

template <int D>
cudaError_t launch_d(const Shape& s, const void* q, const void* k, const void* v,
                     const void* pass_k, const void* pass_v, void* out, float* lse,
                     DeviceStatus* status, cudaStream_t st, const char** why) {
  CUtensorMap mQ, mK, mV, mPK, mPV;
  const uint64_t N = (uint64_t)s.N;
  bool ok = encode_bf16_3d(&mQ, q, D, s.Hq, N, (uint64_t)D * 2, (uint64_t)s.Hq * D * 2, 64, 1,
                           kRows) &&
            encode_bf16_3d(&mK, k, D, s.Hkv, N, (uint64_t)D * 2, (uint64_t)s.Hkv * D * 2, 64, 1,
                           kRows) &&
            encode_bf16_3d(&mV, v, D, s.Hkv, N, (uint64_t)D * 2, (uint64_t)s.Hkv * D * 2, 64, 1,
                           kRows);
  if (ok && pass_k) {
    const uint64_t rows = (uint64_t)s.H * s.keep;
    ok = encode_bf16_3d(&mPK, pass_k, D, rows, s.Hkv, (uint64_t)D * 2, rows * D * 2, 64, kRows,
                        1) &&
         encode_bf16_3d(&mPV, pass_v, D, rows, s.Hkv, (uint64_t)D * 2, rows * D * 2, 64, kRows,
                        1);
  } else {
    mPK = mK;   // no passing block: never loaded
    mPV = mV;
  }
  if (!ok) {
    *why = "cuTensorMapEncodeTiled failed (driver entry point or argument)";
    return cudaErrorInvalidValue;
  }
  Params p;
  p.H = s.H;
  p.n = s.n;
  p.A = s.A;
  p.keep = pass_k ? s.keep : 0;
  p.Hq = s.Hq;
  p.Hkv = s.Hkv;
  p.G = s.Hq / s.Hkv;
  p.n_qtiles = (s.n + kRows - 1) / kRows;
  p.N = s.N;
  p.scale_log2 = s.scale * kLog2e;
  p.out = static_cast<__nv_bfloat16*>(out);
  p.lse = lse;
  p.status = status;
  cudaError_t e = cudaFuncSetAttribute(apb_attention_kernel<D>,
                                       cudaFuncAttributeMaxDynamicSharedMemorySize, kSmemBytes);
  if (e != cudaSuccess) return e;
  dim3 grid(p.n_qtiles, s.Hq, s.H);
  apb_attention_kernel<D><<<grid, kThreads, kSmemBytes, st>>>(mQ, mK, mV, mPK, mPV, p);
  return cudaGetLastError();
}

}  // namespace

cudaError_t launch_attention(const Shape& s, const void* q, const void* k, const void* v,
                             const void* pass_k, const void* pass_v, void* out, float* lse,
                             DeviceStatus* status, cudaStream_t st, const char** why) {
  if (s.d == 128) return launch_d<128>(s, q, k, v, pass_k, pass_v, out, lse, status, st, why);
  return launch_d<64>(s, q, k, v, pass_k, pass_v, out, lse, status, st, why);
}

}  // namespace apb

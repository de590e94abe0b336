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
// one; the epilogue applies b1, SiLU, w2 and b2 in fp32.
//
// split_weights_kernel writes Wh, Wl ([Hkv, 2, hidden, 3d] bf16) into the
// workspace once per call.  score_kernel is persistent and runs on CTA pairs
// (clusters of 2, one per TPC): a tile is 256 tokens of one kv head, 128 per
// CTA, and one tcgen05.mma.cta_group::2 of M = 256 tokens, N = 256 hidden,
// K = 16 covers the pair, so each CTA stages only its 128 tokens and its 128
// hidden rows of Wh / Wl.  The pair's even CTA issues every UMMA; the
// accumulators are double-buffered in TMEM (2 x 256 columns), so the
// epilogue of tile i runs under the UMMAs of tile i + 1.  Per CTA:
//   warp 14    TMA producer of the k and v tiles (128 tokens x 64 features,
//              16 KB, 4-slot ring);
//   warp 12    TMA producer of the Wh / Wl halves of a 64-feature chunk
//              (2 x 16 KB, 3 stages);
//   warps 4-11 q converters: read the group's G q heads from global memory
//              (the loads in flight sit in their registers), form qbar in
//              fp32 and write qh, ql (2-pair ring) in the 128-byte-swizzled
//              K-major layout UMMA reads;
//   warp 13    UMMA issuer (even CTA) / TMEM allocation (both);
//   warps 0-3  epilogue, one token row per thread.
// Full barriers live in the even CTA and count both CTAs' arrivals; empty
// barriers live in both and get one commit each.  Waits are bounded like the
// attention kernel's.
#include <cuda_bf16.h>

#include "apb_internal.h"
#include "device_status.cuh"
#include "sm100_pair.cuh"
#include "sm100_ptx.cuh"

namespace apb {
namespace {

constexpr int kHid = 256;
constexpr int kTile = 128;                 // tokens per CTA and tile (the pair: 256)
constexpr int kHalf = kHid / 2;            // hidden rows of B per CTA
constexpr int kChunk = 64;                 // features per chunk (128-byte rows)
constexpr int kKVStages = 4;
constexpr int kQStages = 2;                // (qh, ql) pairs
constexpr int kBStages = 3;
constexpr int kATile = kTile * kChunk * 2;          // 16 KB
constexpr int kBPart = kHalf * kChunk * 2;          // 16 KB (hi or lo half)
constexpr int kSmemKV = 0;
constexpr int kSmemQ = kSmemKV + kKVStages * kATile;          // 64 KB
constexpr int kSmemB = kSmemQ + kQStages * 2 * kATile;        // 128 KB
constexpr int kSmemBars = kSmemB + kBStages * 2 * kBPart;     // 224 KB
constexpr int kSmemB1 = kSmemBars + 256;                     // b1, w2 of the current head
// The tiles need 1024-byte alignment; the dynamic shared memory of this
// kernel (which has no static shared memory) starts at such an address, and
// the kernel checks that instead of reserving slack for it.
constexpr int kSmemBytes = kSmemB1 + 2 * kHid * 4;
constexpr int kEpiThreads = 128;           // warps 0-3
constexpr int kConvThreads = 256;          // warps 4-11
constexpr int kBWarp = 12;
constexpr int kMmaWarp = 13;
constexpr int kKVWarp = 14;
constexpr int kThreads = 480;
constexpr uint64_t kWaitLimitNs = 1000000000ull;   // drains at the end of a launch
constexpr uint64_t kDrainLimitNs = 100000000ull;

// Full barriers (KV_FULL, Q_FULL, B_FULL) and ACC_EMPTY are used in the even
// CTA only, with 2 arrivals per phase (one per CTA); the others get one
// arrival (a UMMA commit) in each CTA.
enum Bar {
  KV_FULL = 0,
  KV_EMPTY = KV_FULL + kKVStages,
  Q_FULL = KV_EMPTY + kKVStages,
  Q_EMPTY = Q_FULL + kQStages,
  B_FULL = Q_EMPTY + kQStages,
  B_EMPTY = B_FULL + kBStages,
  ACC_FULL = B_EMPTY + kBStages,
  ACC_EMPTY = ACC_FULL + 2,
  DRAIN = ACC_EMPTY + 2,
  NUM = DRAIN + 1
};
static_assert(NUM * 8 + 8 <= 256, "barriers and the TMEM address fit their 256 bytes");

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
  int tiles_per_head, n_tiles;       // tiles of 256 tokens
  const __nv_bfloat16* q;
  const float* b1;
  const float* w2;
  const float* b2;
  float* scores;
  DeviceStatus* status;
  uint64_t wait_ns;   // limit of the bounded waits (1 s; shorter in self-tests)
};

// Section of feature chunk c: 0 k, 1 v, 2 q.
__device__ __forceinline__ int chunk_section(int c, int d) { return (c * kChunk) / d; }

// The q section of the CTA's 128 tokens, every q chunk at once, in two
// passes of 64 tokens (warps 4-11).  In pass sp, thread ct takes the 16-byte
// piece ct % 8 (8 features) of every q chunk for the tokens
// sp * 64 + ct / 8 + 32 i, i < 2, and reads it from the group's G heads, 4
// heads at a time: the 8 lanes of a token cover a whole 128-byte line per
// load (streaming loads that skip L1), and a pass reads each token's
// G * d * 2 contiguous bytes.  The sums
// run in fp32; the mean (x 1/G) is split into bf16 hi + lo.
constexpr int kMaxQChunks = 2;             // d <= 128

struct QLoad {
  uint4 v[kMaxQChunks][2][4];              // [chunk][token][head of the group]
};
struct QAcc {
  float a[kMaxQChunks][2][8];              // [chunk][token][feature]
};

__device__ __forceinline__ void q_issue(const ScoreParams& p, long long row0, int g, int sp,
                                        int j0, int n_q, int ct, QLoad& L) {
  const int piece = ct & 7;
#pragma unroll
  for (int i = 0; i < 2; ++i) {
    const long long t = row0 + sp * 64 + (ct >> 3) + 32 * i;
    const __nv_bfloat16* base =
        p.q + t * ((long long)p.Hq * p.d) + (long long)(g * p.G + j0) * p.d + piece * 8;
#pragma unroll
    for (int c = 0; c < kMaxQChunks; ++c)
#pragma unroll
      for (int u = 0; u < 4; ++u) {
        L.v[c][i][u] = make_uint4(0u, 0u, 0u, 0u);
        if (c < n_q && t < p.N && j0 + u < p.G)
          L.v[c][i][u] =
              ptx::ld_stream_16(base + (long long)u * p.d + c * kChunk);
      }
  }
}

__device__ __forceinline__ void q_accumulate(const QLoad& L, QAcc& A) {
#pragma unroll
  for (int c = 0; c < kMaxQChunks; ++c)
#pragma unroll
    for (int i = 0; i < 2; ++i)
#pragma unroll
      for (int u = 0; u < 4; ++u) {
        const uint32_t w[4] = {L.v[c][i][u].x, L.v[c][i][u].y, L.v[c][i][u].z, L.v[c][i][u].w};
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          A.a[c][i][2 * e] += __uint_as_float(w[e] << 16);
          A.a[c][i][2 * e + 1] += __uint_as_float(w[e] & 0xffff0000u);
        }
      }
}

// Splits a pass's sums (x 1/G) into bf16 hi + lo and writes them into the
// (qh, ql) slot pair of each q chunk, in the 128-byte-swizzled K-major
// layout UMMA reads (16-byte chunk index XOR row % 8 inside each 1024-byte
// group of 8 rows: what a TMA load with 128-byte swizzle would have written).
// Piece by piece, so no second copy of the pass is held in registers.
__device__ __forceinline__ void q_split_store(const QAcc& A, float invG, int sp, int n_q, int ct,
                                              uint8_t* qbase, int qu) {
  const int piece = ct & 7;
#pragma unroll
  for (int c = 0; c < kMaxQChunks; ++c) {
    if (c >= n_q) break;
    uint8_t* slot = qbase + ((qu + c) % kQStages) * 2 * kATile;
#pragma unroll
    for (int i = 0; i < 2; ++i) {
      const int r = sp * 64 + (ct >> 3) + 32 * i;
      uint32_t hi[4], lo[4];
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        const float x0 = A.a[c][i][2 * e] * invG, x1 = A.a[c][i][2 * e + 1] * invG;
        const __nv_bfloat162 h = __floats2bfloat162_rn(x0, x1);
        const __nv_bfloat162 l = __floats2bfloat162_rn(x0 - __low2float(h), x1 - __high2float(h));
        hi[e] = *reinterpret_cast<const uint32_t*>(&h);
        lo[e] = *reinterpret_cast<const uint32_t*>(&l);
      }
      const int at = r * 128 + ((piece ^ (r & 7)) << 4);
      *reinterpret_cast<uint4*>(slot + at) = make_uint4(hi[0], hi[1], hi[2], hi[3]);
      *reinterpret_cast<uint4*>(slot + kATile + at) = make_uint4(lo[0], lo[1], lo[2], lo[3]);
    }
  }
}

__global__ void __launch_bounds__(512, 1)   // 512: caps registers at 128 (launched with 480)
    score_kernel(const __grid_constant__ CUtensorMap mQ, const __grid_constant__ CUtensorMap mK,
                 const __grid_constant__ CUtensorMap mV, const __grid_constant__ CUtensorMap mW,
                 const ScoreParams p) {
  extern __shared__ __align__(1024) uint8_t smem[];
  if ((ptx::smem_u32(smem) & 1023u) != 0u) {      // same in both CTAs of the pair
    if (threadIdx.x == 0) record_failure(p.status, 90, 0);
    return;
  }
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + kSmemBars);
  float* s_b1 = reinterpret_cast<float*>(smem + kSmemB1);
  float* s_w2 = s_b1 + kHid;
  uint32_t* s_tmem = reinterpret_cast<uint32_t*>(bars + NUM);
  uint32_t* s_flags = s_tmem + 1;

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const uint32_t rank = pair::cta_rank();
  const int cl = (int)pair::cluster_id_x(), ncl = (int)pair::n_clusters_x();
  const volatile uint32_t* gabort = &p.status->abort;
  const int q_chunk0 = 2 * p.d / kChunk;      // first chunk of the q section
  const int n_q = p.n_chunks - q_chunk0;      // q chunks per tile (0: query-aware)
  // A tile's chunks run q first, then k, v: the converters then have the whole
  // k and v part of a tile to prepare the next tile's q.
  auto chunk_at = [&](int i) { return i < n_q ? q_chunk0 + i : i - n_q; };
  // the token rows of this CTA in tile t, and its kv head
  auto tile_g = [&](int t) { return t / p.tiles_per_head; };
  auto tile_row = [&](int t) {
    return (long long)(t % p.tiles_per_head) * (2 * kTile) + (long long)rank * kTile;
  };

  if (threadIdx.x == 0) {
    for (int i = 0; i < NUM; ++i) {
      const bool two = (i < KV_EMPTY) || (i >= Q_FULL && i < Q_EMPTY) ||
                       (i >= B_FULL && i < B_EMPTY) || (i >= ACC_EMPTY && i < DRAIN);
      ptx::mbar_init(&bars[i], two ? 2 : 1);
    }
    ptx::fence_mbar_init();
    s_flags[0] = *gabort;
    s_flags[1] = 0u;
  }
  if (warp == kMmaWarp) {
    pair::tmem_alloc(s_tmem, 512);
    pair::tmem_relinquish();
  }
  if (warp == kBWarp && lane == 0) {
    ptx::tma_prefetch_desc(&mQ);
    ptx::tma_prefetch_desc(&mK);
    ptx::tma_prefetch_desc(&mV);
    ptx::tma_prefetch_desc(&mW);
  }
  ptx::tc_fence_before();
  __syncthreads();
  pair::cluster_sync();       // barriers of both CTAs initialised before any arrival
  ptx::tc_fence_after();
  const uint32_t tmem = *s_tmem;
  const volatile uint32_t* never = s_flags + 1;
  const bool skip = s_flags[0] != 0u;

  if (warp == kBWarp || warp == kKVWarp) {
    // ------------------------------------------------------------ producers
    // Two threads, so that neither ring waits on the other: warp 12 streams
    // the B halves (every chunk), warp 14 the k and v tiles (k, v chunks).
    if (lane == 0 && !skip) {
      const bool isB = warp == kBWarp;
      const int stages = isB ? kBStages : kKVStages;
      uint64_t* full = &bars[isB ? B_FULL : KV_FULL];
      uint64_t* empty = &bars[isB ? B_EMPTY : KV_EMPTY];
      int u = 0;
      bool ok = true;
      for (int t = cl; t < p.n_tiles && ok; t += ncl) {
        const int g = tile_g(t);
        const int row = (int)tile_row(t);
        for (int i = 0; i < p.n_chunks; ++i) {
          const int c = chunk_at(i);
          const int sec = chunk_section(c, p.d);
          if (!isB && sec == 2) continue;       // q tiles come from the converters
          const int s = u % stages;
          if (!ptx::mbar_wait_bounded(&empty[s], ((u / stages) & 1) ^ 1, gabort, p.wait_ns)) {
            record_failure(p.status, (isB ? 80 : 82) + rank, u);
            ok = false;
            break;
          }
          const uint32_t fc = pair::map_to(&full[s], 0);
          if (isB) {
            uint8_t* dst = smem + kSmemB + s * 2 * kBPart;
            pair::arrive_expect_tx_relaxed(fc, 2 * kBPart);
            pair::tma_load_3d(dst, &mW, fc, c * kChunk, (int)rank * kHalf, 2 * g);
            pair::tma_load_3d(dst + kBPart, &mW, fc, c * kChunk, (int)rank * kHalf, 2 * g + 1);
          } else {
            pair::arrive_expect_tx_relaxed(fc, kATile);
            pair::tma_load_3d(smem + kSmemKV + s * kATile, sec == 0 ? &mK : &mV, fc,
                              c * kChunk - sec * p.d, g, row);
          }
          ++u;
        }
      }
      // copies in flight land before the CTA may exit: wait until the UMMAs
      // have released the last use of every slot (bounded; on a failure the
      // copies have long completed when the limit passes)
      for (int v = u - stages; v < u; ++v)
        if (v >= 0)
          ptx::mbar_wait_bounded(&empty[v % stages], (v / stages) & 1, never,
                                 ok ? kWaitLimitNs : kDrainLimitNs);
    }
  } else if (warp == kMmaWarp) {
    // ------------------------------------------------------------ UMMA issuer
    if (lane == 0 && rank == 0 && !skip) {
      const uint32_t idesc = ptx::idesc_bf16_f32(2 * kTile, kHid, 0);
      const uint32_t aKV = ptx::smem_u32(smem + kSmemKV);
      const uint32_t aQ = ptx::smem_u32(smem + kSmemQ);
      const uint32_t aB = ptx::smem_u32(smem + kSmemB);
      // a commit tracks every UMMA issued before it; one to each CTA's barrier
      auto commit_both = [&](int bar) {
        pair::umma_commit(pair::map_to(&bars[bar], 0));
        pair::umma_commit(pair::map_to(&bars[bar], 1));
      };
      int kvu = 0, qu = 0, bu = 0, it = 0;
      bool ok = true;
      for (int t = cl; t < p.n_tiles && ok; t += ncl, ++it) {
        const int b = it & 1;
        if (!pair::spin_cluster_bounded(&bars[ACC_EMPTY + b], ((it >> 1) & 1) ^ 1, gabort,
                                        p.wait_ns)) {
          record_failure(p.status, 84, it);
          break;
        }
        ptx::tc_fence_after();
        const uint32_t acc = tmem + 256 * b;
        bool first = true;
        for (int i = 0; i < p.n_chunks && ok; ++i) {
          const int c = chunk_at(i);
          const int bs = bu % kBStages;
          const bool qsec = chunk_section(c, p.d) == 2;
          const int s = qsec ? qu % kQStages : kvu % kKVStages;
          ok = pair::spin_cluster_bounded(&bars[B_FULL + bs], (bu / kBStages) & 1, gabort,
                                          p.wait_ns) &&
               (qsec ? pair::spin_cluster_bounded(&bars[Q_FULL + s], (qu / kQStages) & 1, gabort,
                                                  p.wait_ns)
                     : pair::spin_cluster_bounded(&bars[KV_FULL + s], (kvu / kKVStages) & 1,
                                                  gabort, p.wait_ns));
          if (!ok) {
            record_failure(p.status, 85, c);
            break;
          }
          ptx::tc_fence_after();
          const uint32_t bh = aB + bs * 2 * kBPart, bl = bh + kBPart;
          const uint32_t xh = qsec ? aQ + s * 2 * kATile : aKV + s * kATile;
          const uint32_t xl = xh + kATile;     // ql (q chunks only)
          const uint32_t acc0 = first ? 0u : 1u;
          first = false;
          // the two forms as separate straight-line runs: a branch between
          // consecutive UMMAs slows the tensor core's stream (~1.6x here)
          if (qsec) {
#pragma unroll
            for (int ks = 0; ks < kChunk / 16; ++ks) {
              const uint64_t dXh = ptx::sdesc_sw128(xh + ks * 32, 16, 1024);
              const uint64_t dXl = ptx::sdesc_sw128(xl + ks * 32, 16, 1024);
              const uint64_t dBh = ptx::sdesc_sw128(bh + ks * 32, 16, 1024);
              const uint64_t dBl = ptx::sdesc_sw128(bl + ks * 32, 16, 1024);
              pair::umma_bf16_ss(acc, dXh, dBh, idesc, ks == 0 ? acc0 : 1u);
              pair::umma_bf16_ss(acc, dXh, dBl, idesc, 1u);
              pair::umma_bf16_ss(acc, dXl, dBh, idesc, 1u);
            }
          } else {
#pragma unroll
            for (int ks = 0; ks < kChunk / 16; ++ks) {
              const uint64_t dXh = ptx::sdesc_sw128(xh + ks * 32, 16, 1024);
              const uint64_t dBh = ptx::sdesc_sw128(bh + ks * 32, 16, 1024);
              const uint64_t dBl = ptx::sdesc_sw128(bl + ks * 32, 16, 1024);
              pair::umma_bf16_ss(acc, dXh, dBh, idesc, ks == 0 ? acc0 : 1u);
              pair::umma_bf16_ss(acc, dXh, dBl, idesc, 1u);
            }
          }
          commit_both(qsec ? Q_EMPTY + s : KV_EMPTY + s);
          commit_both(B_EMPTY + bs);
          ++bu;
          if (qsec) ++qu; else ++kvu;
        }
        if (ok) commit_both(ACC_FULL + b);
      }
      commit_both(DRAIN);
      ptx::mbar_wait_bounded(&bars[DRAIN], 0, never, kWaitLimitNs);
    }
  } else if (warp >= 4) {
    // ------------------------------------------------------------ q converters
    // Units of work: (tile, pass, group of 4 heads).  The loads of unit k + 1
    // are issued before unit k is split and stored, so they are in flight
    // while this thread waits for free slots and writes shared memory.
    if (!skip && n_q > 0) {
      const int ct = threadIdx.x - 128;
      const float invG = 1.0f / (float)p.G;     // exact for G = 2^k
      const int ng = (p.G + 3) / 4;
      const int my_tiles = cl < p.n_tiles ? (p.n_tiles - 1 - cl) / ncl + 1 : 0;
      const int n_units = my_tiles * 2 * ng;
      auto issue = [&](int k, QLoad& L) {
        const int ti = k / (2 * ng), rem = k - ti * 2 * ng;
        const int t = cl + ti * ncl;
        q_issue(p, tile_row(t), tile_g(t), rem / ng, (rem % ng) * 4, n_q, ct, L);
      };
      QLoad L;
      QAcc A;
      if (n_units > 0) issue(0, L);
      int qu = 0;                                // q pair uses so far (n_q per tile)
      bool ok = true;
      for (int k = 0; k < n_units && ok; ++k) {
        const int rem = k % (2 * ng), sp = rem / ng, jg = rem % ng;
        if (jg == 0) {
#pragma unroll
          for (int c = 0; c < kMaxQChunks; ++c)
#pragma unroll
            for (int pp = 0; pp < 2; ++pp)
#pragma unroll
              for (int e = 0; e < 8; ++e) A.a[c][pp][e] = 0.f;   // [chunk][token][feature]
        }
        q_accumulate(L, A);
        if (k + 1 < n_units) issue(k + 1, L);   // in flight during the wait and the stores
        if (jg != ng - 1) continue;
        if (sp == 0) {          // the tile's slots, released by the UMMAs of the last use
          if (ct == 0)
            for (int c = 0; c < n_q && ok; ++c) {
              const int u = qu + c;
              ok = ptx::mbar_wait_bounded(&bars[Q_EMPTY + u % kQStages],
                                          ((u / kQStages) & 1) ^ 1, gabort, p.wait_ns);
              if (!ok) record_failure(p.status, 86 + rank, u);
            }
          ok = ptx::barrier_and(1, kConvThreads, ok);
          if (!ok) break;
        }
        q_split_store(A, invG, sp, n_q, ct, smem + kSmemQ, qu);
        if (sp == 1) {          // tile complete: publish its pairs to the issuer
          ptx::fence_proxy_async_smem();
          ptx::named_barrier_sync(1, kConvThreads);
          if (ct == 0)
            for (int c = 0; c < n_q; ++c)
              pair::arrive_remote(pair::map_to(&bars[Q_FULL + (qu + c) % kQStages], 0));
          qu += n_q;
        }
      }
    }
  } else {
    // ------------------------------------------------------------ epilogue
    if (!skip) {
      const int row = threadIdx.x;                      // 0..127 = TMEM lane
      const uint32_t lane_off = (uint32_t)((warp & 3) * 32) << 16;
      int it = 0, cur_g = -1;
      for (int t = cl; t < p.n_tiles; t += ncl, ++it) {
        const int b = it & 1;
        const int g = tile_g(t);
        if (g != cur_g) {       // this head's b1, w2 into shared memory
          ptx::named_barrier_sync(2, kEpiThreads);
          for (int u = row; u < kHid; u += kEpiThreads) {
            s_b1[u] = p.b1[g * kHid + u];
            s_w2[u] = p.w2[g * kHid + u];
          }
          ptx::named_barrier_sync(2, kEpiThreads);
          cur_g = g;
        }
        const float4* b1 = reinterpret_cast<const float4*>(s_b1);
        const float4* w2 = reinterpret_cast<const float4*>(s_w2);
        const bool ok = ptx::mbar_wait_bounded(&bars[ACC_FULL + b], (it >> 1) & 1, gabort,
                                               p.wait_ns);
        if (!ptx::barrier_and(2, kEpiThreads, ok)) {
          if (row == 0) record_failure(p.status, 88 + rank, it);
          break;
        }
        ptx::tc_fence_after();
        const uint32_t taddr = tmem + 256 * b + lane_off;
        // column chunks of 32, the load of chunk cc + 1 in flight while
        // chunk cc is evaluated (two register sets)
        uint32_t z0[32], z1[32];
        float part[4] = {0.f, 0.f, 0.f, 0.f};     // 4 chains: no serial FFMA latency
        auto eval = [&](const uint32_t* z, int cc) {
#pragma unroll
          for (int x4 = 0; x4 < 8; ++x4) {
            const float4 bb = b1[8 * cc + x4];
            const float4 ww = w2[8 * cc + x4];
            const float bv[4] = {bb.x, bb.y, bb.z, bb.w}, wv[4] = {ww.x, ww.y, ww.z, ww.w};
#pragma unroll
            for (int e = 0; e < 4; ++e) {
              const float zz = __uint_as_float(z[4 * x4 + e]) + bv[e];
              const float silu = __fdividef(zz, 1.0f + __expf(-zz));
              part[e] = fmaf(wv[e], silu, part[e]);
            }
          }
        };
        APB_TMEM_LD32_ASYNC(taddr, z0);
        APB_TMEM_WAIT32(z0);
#pragma unroll 1
        for (int cc = 0; cc < kHid / 32; cc += 2) {
          APB_TMEM_LD32_ASYNC(taddr + 32 * (cc + 1), z1);
          eval(z0, cc);
          APB_TMEM_WAIT32(z1);
          if (cc + 2 < kHid / 32) APB_TMEM_LD32_ASYNC(taddr + 32 * (cc + 2), z0);
          eval(z1, cc + 1);
          if (cc + 2 < kHid / 32) APB_TMEM_WAIT32(z0);
        }
        // accumulator b read out by all 128 rows: hand it back to the issuer
        ptx::tc_fence_before();
        ptx::named_barrier_sync(2, kEpiThreads);
        if (row == 0) pair::arrive_remote(pair::map_to(&bars[ACC_EMPTY + b], 0));
        const long long tok = tile_row(t) + row;
        if (tok < p.N)
          p.scores[(long long)g * p.N + tok] = ((part[0] + part[1]) + (part[2] + part[3])) + __ldg(p.b2 + g);
      }
    }
  }

  // Both CTAs stay resident until the pair is done: the even CTA's UMMAs read
  // the odd CTA's shared memory, and the odd CTA arrives on the even one's
  // barriers.
  ptx::tc_fence_before();
  __syncthreads();
  pair::cluster_sync();
  if (warp == kMmaWarp) {
    ptx::tc_fence_after();
    pair::tmem_dealloc(tmem, 512);
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
                           (uint64_t)kHid * F * 2, 64, kHalf, 1);
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
  p.wait_ns = wait_limit_ns();
  p.tiles_per_head = (int)((s.N + 2 * kTile - 1) / (2 * kTile));
  p.n_tiles = p.tiles_per_head * s.Hkv;
  if (p.n_tiles == 0) return cudaSuccess;
  e = cudaFuncSetAttribute(score_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, kSmemBytes);
  if (e != cudaSuccess) return e;

  // persistent: as many CTA pairs as can be resident at once (once per device)
  cudaLaunchConfig_t lc = {};
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = 2;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  lc.blockDim = dim3(kThreads);
  lc.dynamicSmemBytes = kSmemBytes;
  lc.stream = st;
  lc.attrs = attr;
  lc.numAttrs = 1;
  static int resident_pairs[64] = {0};
  int pairs = dev >= 0 && dev < 64 ? resident_pairs[dev] : 0;
  if (pairs == 0) {
    lc.gridDim = dim3(2 * (sms / 2));
    e = cudaOccupancyMaxActiveClusters(&pairs, score_kernel, &lc);
    if (e != cudaSuccess) return e;
    if (pairs < 1) {
      *why = "score kernel: no CTA pair fits on the device";
      return cudaErrorInvalidConfiguration;
    }
    if (dev >= 0 && dev < 64) resident_pairs[dev] = pairs;
  }
  if (pairs > p.n_tiles) pairs = p.n_tiles;
  lc.gridDim = dim3(2 * pairs);
  return cudaLaunchKernelEx(&lc, score_kernel, mQ, mK, mV, mW, p);
}

}  // namespace apb

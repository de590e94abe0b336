// Block-masked prefill attention of APB on sm_100a ("APB 的主要功能":
// computation over the anchor block, the passing block and the local block;
// the passing block is not kept afterwards).
//
// One CTA computes two consecutive 128-row query tiles (A, B) of one q head
// of one host.  Their KV sequence is three ranges walked as 128-row tiles:
//   anchor  : k[0:A, g]             (hosts h >= 1)      full visibility
//   passing : pass_k[g, 0:h*keep]                       full visibility
//   local   : k[h*n : h*n + qB0 + 128, g]               causal, diagonal kept
// Tile A stops one KV tile earlier than tile B (its own diagonal); tiles
// beyond a diagonal are never visited and only the last tile of each range
// needs a mask.  Every K and V tile in shared memory feeds both query tiles.
//
// Warp roles (352 threads):
//   warps 0-3  softmax + epilogue of query tile A (thread r owns row r, which
//              is TMEM lane r of S_A, P_A and O_A);
//   warps 4-7  the same for query tile B;
//   warp 8     TMA producer (Q_A, Q_B once, K in a 2-stage and V in a 3-stage
//              ring);
//   warp 9     TMEM allocator and the single UMMA-issuing thread, which never
//              reads shared memory inside its loop;
//   warp 10    watcher: waits on the TMA barriers the issuer depends on (Q, K,
//              V landed) and hands each one over to the issuer at a named
//              barrier; the softmax warps hand each P half over themselves,
//              at named barriers of their own.
// TMEM columns: S_A [0,128), S_B [128,256), O_A [256,384), O_B [384,512).
// P_A (bf16, two per 32-bit column) overwrites S_A columns [0,64) once the
// softmax has read S_A; likewise P_B in S_B.
// Per KV tile j and query tile i:
//   S_i(j) = Q_i K(j)^T         tcgen05.mma, A and B from shared memory
//   softmax_i reads S_i(j), exponentiates against a lazily moved row maximum
//   (O_i is rescaled in TMEM only when that base moves), writes P_i(j) to
//   TMEM in two 64-column halves and hands each half to the issuer at a
//   named barrier
//   O_i += P_i(j) V(j)          tcgen05.mma, A = P_i from TMEM, B = V
// The MMA thread issues PV_A(j), S_A(j+1), PV_B(j), S_B(j+1): while one
// softmax warpgroup works on its tile the tensor core serves the other.
// tcgen05 MMAs of one thread execute in issue order, so S_i(j+1) overwrites
// P_i(j) only after PV_i(j) has read it, and the commit that signals
// S_i(j+1) also covers PV_i(j): when the softmax sees S_i(j+1), O_i is
// stable and may be rescaled.
//
// Every mbarrier wait is bounded (wall-clock limit plus a launch-wide abort
// flag); a wait that runs out records an error in the status block, the CTA
// drains its outstanding TMA loads and MMAs, frees TMEM and returns.
#include <cuda_bf16.h>
#include "apb_internal.h"
#include "device_status.cuh"
#include "sm100_ptx.cuh"

namespace apb {
namespace {

constexpr int kRows = 128;                    // query rows per tile = KV rows per tile
constexpr int kThreads = 352;
constexpr int kProducerWarp = 8;
constexpr int kIssuerWarp = 9;
constexpr int kWatcherWarp = 10;
constexpr int kHandoffBar = 1;                // named barrier: watcher -> issuer (64 threads)
// Named barriers 2..5: P_i(j) half h written -> issuer, id kPBar + 2 * i + h;
// the 128 softmax threads of tile i arrive, the issuer warp waits.
constexpr int kPBar = 2;
constexpr int kPBarThreads = 128 + 32;
constexpr uint64_t kWaitLimitNs = 1000000000ull;   // 1 s: drains of copies and MMAs
constexpr float kLog2e = 1.4426950408889634f;
constexpr int kKStages = 2;
constexpr int kVStages = 3;   // V is released later than K: one more stage of prefetch
static_assert(kKStages + kVStages == 5, "shared memory holds Q_A, Q_B and five K/V stages");

// Failure codes ("where" in the status block) of this kernel's waits.
constexpr uint32_t kWhereKEmpty = 40;   // producer, + K slot
constexpr uint32_t kWhereVEmpty = 45;   // producer, + V slot
constexpr uint32_t kWhereQ = 50;        // issuer: Q_A, Q_B landed
constexpr uint32_t kWhereKFull = 51;    // issuer, + K slot
constexpr uint32_t kWhereVFull = 54;    // issuer, + V slot
constexpr uint32_t kWhereS = 60;        // softmax, + query tile
constexpr uint32_t kWhereO = 63;        // epilogue, + query tile
constexpr uint32_t kWherePV0 = 74;      // softmax, + query tile (rare rescale path)

enum Bar {
  Q_FULL = 0,
  K_FULL = 1,                       // kKStages
  K_EMPTY = K_FULL + kKStages,      // kKStages
  V_FULL = K_EMPTY + kKStages,      // kVStages
  V_EMPTY = V_FULL + kVStages,      // kVStages
  S_FULL = V_EMPTY + kVStages,      // per query tile (A, B)
  O_FINAL = S_FULL + 2,             // per query tile
  DRAIN = O_FINAL + 2,
  PV0_DONE = DRAIN + 1,             // per query tile: PV_i(j) on the first P half has run
  NUM_BARS = PV0_DONE + 2
};

template <int D>
struct Layout {
  static constexpr int kTile = kRows * D * 2;   // bytes of one Q/K/V tile
  static constexpr int kQ = 0;                  // Q_A, Q_B
  static constexpr int kK0 = 2 * kTile;         // K stages
  static constexpr int kV0 = kK0 + kKStages * kTile;   // V stages
  static constexpr int kBars = kV0 + kVStages * kTile;
};
// Both head sizes request the d = 128 footprint (+256 bytes of barriers,
// +1024 of alignment slack) so that one CTA runs per SM (each CTA allocates
// all 512 TMEM columns).
constexpr int kSmemBytes = Layout<128>::kBars + 256 + 1024;

struct Params {
  int H, n, A, keep, Hq, Hkv, G, n_ctas_per_host;
  // hosts h0 + i * hstride, i < hcount, of this launch, one after another in
  // the Q/out and K/V buffers from rows q_row0 / k_row0; the anchor's first
  // token at K/V row anchor_row0
  int h0, hcount, hstride, q_row0, k_row0, anchor_row0;
  long long N;   // rows of the Q/out buffer (the lse row stride)
  float scale_log2;
  uint64_t wait_ns;   // limit of the bounded waits (1 s; shorter in self-tests)
  __nv_bfloat16* out;
  float* lse;
  DeviceStatus* status;
};

template <int D>
__device__ __forceinline__ void load_kv_tile(const CUtensorMap* m_kv, const CUtensorMap* m_pass,
                                             uint8_t* dst, uint64_t* bar, int j, int na, int np,
                                             int g, int local_row0, int anchor_row0) {
  if (j < na) {
#pragma unroll
    for (int kb = 0; kb < D / 64; ++kb)
      ptx::tma_load_3d(dst + kb * (kRows * 128), m_kv, bar, kb * 64, g, anchor_row0 + j * kRows);
  } else if (j < na + np) {
#pragma unroll
    for (int kb = 0; kb < D / 64; ++kb)
      ptx::tma_load_3d(dst + kb * (kRows * 128), m_pass, bar, kb * 64, g, (j - na) * kRows);
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
  uint32_t* s_tmem = reinterpret_cast<uint32_t*>(bars + NUM_BARS);
  uint32_t* s_flags = s_tmem + 1;   // [0]: launch already aborted, [1]: constant 0

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;

  // heavy units first: the last query tiles of the last hosts
  const int u = p.n_ctas_per_host - 1 - (int)blockIdx.x;
  const int head = (int)blockIdx.y;
  const int li = p.hcount - 1 - (int)blockIdx.z;   // launch-local host index
  const int h = p.h0 + li * p.hstride;
  const int g = head / p.G;
  const int qA0 = 2 * u * kRows;                 // first local row of tile A
  const int na = (h >= 1 && p.A > 0) ? (p.A + kRows - 1) / kRows : 0;
  const int P = h * p.keep;
  const int np = (P + kRows - 1) / kRows;
  const int TA = na + np + 2 * u + 1;            // KV tiles of query tile A
  const int TB = (qA0 + kRows < p.n) ? TA + 1 : 0;   // of tile B (0: beyond the block)
  const int Tmax = TB > 0 ? TB : TA;
  const int local_row0 = p.k_row0 + li * p.n;   // K/V row of this host's token 0
  const int q_row0 = p.q_row0 + li * p.n;       // Q/out row of this host's token 0

  const volatile uint32_t* gabort = &p.status->abort;

  if (threadIdx.x == 0) {
    for (int i = 0; i < NUM_BARS; ++i) ptx::mbar_init(&bars[i], 1);
    ptx::fence_mbar_init();
    s_flags[0] = *gabort;
    s_flags[1] = 0u;
  }
  if (warp == kIssuerWarp) {
    ptx::tmem_alloc(s_tmem, 512);
    ptx::tmem_relinquish();
  }
  if (warp == kProducerWarp && lane == 0) {
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

  uint8_t* sQ = smem + L::kQ;     // tile i at sQ + i * kTile
  uint8_t* sK0 = smem + L::kK0;   // stage s at sK0 + s * kTile
  uint8_t* sV0 = smem + L::kV0;

  if (warp == kProducerWarp) {
    // ------------------------------------------------------------ producer
    if (lane == 0 && !skip) {
      int lastK[kKStages], lastV[kVStages];   // last load parity per slot (-1: never loaded)
      for (int i = 0; i < kKStages; ++i) lastK[i] = -1;
      for (int i = 0; i < kVStages; ++i) lastV[i] = -1;
      ptx::mbar_arrive_expect_tx(&bars[Q_FULL], (TB > 0 ? 2 : 1) * L::kTile);
      for (int i = 0; i < (TB > 0 ? 2 : 1); ++i) {
#pragma unroll
        for (int kb = 0; kb < D / 64; ++kb)
          ptx::tma_load_3d(sQ + i * L::kTile + kb * (kRows * 128), &mQ, &bars[Q_FULL], kb * 64,
                           head, q_row0 + qA0 + i * kRows);
      }
      for (int j = 0; j < Tmax; ++j) {
        const int ks = j % kKStages, vs = j % kVStages;
        const uint32_t kpar = (j / kKStages) & 1, vpar = (j / kVStages) & 1;
        if (!ptx::mbar_wait_bounded(&bars[K_EMPTY + ks], kpar ^ 1, gabort, p.wait_ns)) {
          record_failure(p.status, kWhereKEmpty + ks, j);
          break;
        }
        ptx::mbar_arrive_expect_tx(&bars[K_FULL + ks], L::kTile);
        load_kv_tile<D>(&mK, &mPK, sK0 + ks * L::kTile, &bars[K_FULL + ks], j, na, np, g,
                        local_row0, p.anchor_row0);
        lastK[ks] = (int)kpar;
        if (!ptx::mbar_wait_bounded(&bars[V_EMPTY + vs], vpar ^ 1, gabort, p.wait_ns)) {
          record_failure(p.status, kWhereVEmpty + vs, j);
          break;
        }
        ptx::mbar_arrive_expect_tx(&bars[V_FULL + vs], L::kTile);
        load_kv_tile<D>(&mV, &mPV, sV0 + vs * L::kTile, &bars[V_FULL + vs], j, na, np, g,
                        local_row0, p.anchor_row0);
        lastV[vs] = (int)vpar;
      }
      // drain: every load issued must have landed before the CTA exits
      ptx::mbar_wait_bounded(&bars[Q_FULL], 0, never, kWaitLimitNs);
      for (int s = 0; s < kKStages; ++s)
        if (lastK[s] >= 0) ptx::mbar_wait_bounded(&bars[K_FULL + s], lastK[s], never, kWaitLimitNs);
      for (int s = 0; s < kVStages; ++s)
        if (lastV[s] >= 0) ptx::mbar_wait_bounded(&bars[V_FULL + s], lastV[s], never, kWaitLimitNs);
    }
  } else if (warp == kIssuerWarp) {
    // ------------------------------------------------------------ MMA issuer
    // Lane 0 issues every UMMA and commit.  The warp never touches shared
    // memory in the loop: a shared-memory access (an mbarrier check above
    // all) right after UMMAs holds the issuing thread until they have read
    // their operands, which lets the tensor core drain at every check.  The
    // TMA checks are made by the watcher warp and handed over at named
    // barrier kHandoffBar; each half of P_i is handed over by tile i's
    // softmax threads at named barrier kPBar + 2i + h (they arrive, the
    // issuer waits).  A named barrier costs the tensor core nothing.  Every
    // party walks the same sequence of handoffs, so they stay in step
    // whatever happens: after a failed wait the watcher goes on handing over
    // at once (the abort flag is set), a softmax warp that gave up meets the
    // issuer at each remaining P barrier, and the issuer finishes its loop on
    // stale operands, whose results are never stored.
    if (!skip) {
      const uint32_t idesc_s = ptx::idesc_bf16_f32(kRows, kRows, 0);
      const uint32_t idesc_pv = ptx::idesc_bf16_f32(kRows, D, 1);
      // Descriptors of the first K step of every operand buffer; a K step
      // (or a stage) moves only the start-address field (bits 0-13, in
      // 16-byte units), so each UMMA needs one add.
      const uint64_t dQ = ptx::sdesc_sw128(ptx::smem_u32(sQ), 16, 1024);
      const uint64_t dK = ptx::sdesc_sw128(ptx::smem_u32(sK0), 16, 1024);
      const uint64_t dV = ptx::sdesc_sw128(ptx::smem_u32(sV0), kRows * 128, 1024);
      constexpr uint32_t kTile16 = L::kTile >> 4;
      const int T[2] = {TA, TB};
      const bool issuer = lane == 0;

      // S_i(jj) = Q_i K(jj)^T into S_i; K(jj) must have landed
      auto issue_s = [&](int i, int jj) {
        const uint64_t q = dQ + i * kTile16;
        const uint64_t k = dK + (jj % kKStages) * kTile16;
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk) {
          const uint32_t off = ((kk >> 2) * (kRows * 128) + (kk & 3) * 32) >> 4;
          ptx::umma_bf16_ss(tmem + 128 * i, q + off, k + off, idesc_s, kk > 0);
        }
        ptx::umma_commit(&bars[S_FULL + i]);
      };
      // the watcher's next check has passed
      auto handoff = [&]() {
        __syncwarp();
        ptx::named_barrier_sync(kHandoffBar, 64);
        ptx::tc_fence_after();
      };
      // the softmax threads of tile i have written half h of P_i
      auto p_ready = [&](int i, int h) {
        __syncwarp();
        ptx::named_barrier_sync(kPBar + 2 * i + h, kPBarThreads);
        ptx::tc_fence_after();
      };

      handoff();                                   // Q_A, Q_B, K(0)
      if (issuer) {
        issue_s(0, 0);
        if (TB > 0) issue_s(1, 0);
        ptx::umma_commit(&bars[K_EMPTY + 0]);
      }
      for (int j = 0; j < Tmax; ++j) {
        const int s = j % kVStages;
        const bool k_next = j + 1 < Tmax;
        handoff();                                 // V(j) and K(j+1)
#pragma unroll
        for (int i = 0; i < 2; ++i) {
          if (j >= T[i]) continue;
          const uint32_t tP = tmem + 128 * i;
          const uint32_t tOi = tmem + 256 + 128 * i;
          const uint64_t v = dV + s * kTile16;
          const uint32_t acc0 = j > 0 ? 1u : 0u;
          // P_i(j) arrives in two 64-column halves; PV on the first half
          // overlaps the softmax's exponentials of the second
          p_ready(i, 0);
          if (issuer) {
#pragma unroll
            for (int kk = 0; kk < 4; ++kk)
              ptx::umma_bf16_ts(tOi, tP + kk * 8, v + ((kk * 2048) >> 4), idesc_pv,
                                kk > 0 ? 1u : acc0);
            ptx::umma_commit(&bars[PV0_DONE + i]);
          }
          p_ready(i, 1);
          if (issuer) {
#pragma unroll
            for (int kk = 4; kk < 8; ++kk)
              ptx::umma_bf16_ts(tOi, tP + kk * 8, v + ((kk * 2048) >> 4), idesc_pv, 1u);
            // V(j)'s last reader is PV_B(j) (or PV_A(j) when tile B has no tile
            // j): release its slot now, before the next S MMA
            if (i == 1 || j >= T[1]) ptx::umma_commit(&bars[V_EMPTY + s]);
            if (j + 1 < T[i]) {
              issue_s(i, j + 1);
            } else {
              ptx::umma_commit(&bars[O_FINAL + i]);
            }
          }
        }
        if (issuer && k_next) ptx::umma_commit(&bars[K_EMPTY + (j + 1) % kKStages]);
      }
      // drain every MMA issued so far
      if (issuer) {
        ptx::umma_commit(&bars[DRAIN]);
        ptx::mbar_wait_bounded(&bars[DRAIN], 0, never, kWaitLimitNs);
      }
    }
  } else if (warp == kWatcherWarp) {
    // ------------------------------------------------------------ watcher
    // Makes the issuer's checks of the TMA loads (Q, K(j+1) with V(j)), in
    // the issuer's order, and hands each one over at kHandoffBar.  After a
    // failed wait (recorded, abort flag set) the remaining waits return at
    // once, so the hand-overs continue and the issuer is never left waiting.
    if (!skip) {
      bool ok = true;
      auto check = [&](uint64_t* bar, uint32_t parity, uint32_t where, int tile) {
        bool got = true;
        if (lane == 0) {
          // polled: this warp's reaction time is on the issuer's path
          got = ptx::mbar_spin_bounded(bar, parity, gabort, p.wait_ns);
          if (!got && ok) record_failure(p.status, where, tile);
        }
        ok = __shfl_sync(0xffffffffu, (int)(got && ok), 0) != 0;
      };
      auto handoff = [&]() {
        __syncwarp();
        ptx::named_barrier_sync(kHandoffBar, 64);
      };
      check(&bars[Q_FULL], 0, kWhereQ, 0);
      check(&bars[K_FULL], 0, kWhereKFull, 0);
      handoff();
      for (int j = 0; j < Tmax; ++j) {
        const int s = j % kVStages;
        check(&bars[V_FULL + s], (j / kVStages) & 1, kWhereVFull + s, j);
        if (j + 1 < Tmax)
          check(&bars[K_FULL + (j + 1) % kKStages], ((j + 1) / kKStages) & 1,
                kWhereKFull + (j + 1) % kKStages, j + 1);
        handoff();
      }
    }
  } else if (!skip) {
    // ------------------------------------------------------------ softmax
    const int i = warp >> 2;                           // query tile A (0) or B (1)
    const int row = threadIdx.x & 127;
    const int T = i == 0 ? TA : TB;
    const uint32_t lane_off = (uint32_t)((warp & 3) * 32) << 16;
    const uint32_t tS = tmem + 128 * i + lane_off;     // S_i, and P_i in its first 64 columns
    const uint32_t tO = tmem + 256 + 128 * i + lane_off;
    const int q0 = qA0 + i * kRows;
    float m = -INFINITY, l = 0.f;
    bool ok = true;
    int arrived = 0;   // P halves handed to the issuer so far (2 per KV tile)
    for (int j = 0; j < T; ++j) {
      ok = ptx::mbar_wait_bounded(&bars[S_FULL + i], j & 1, gabort, p.wait_ns);
      if (!__all_sync(0xffffffffu, ok)) {
        if (lane == 0) record_failure(p.status, kWhereS + i, j);
        ok = false;
        break;
      }
      ptx::tc_fence_after();
      // visible columns of this row in this tile
      int lim;
      if (j < na) {
        lim = min(kRows, p.A - j * kRows);
      } else if (j < na + np) {
        lim = min(kRows, P - (j - na) * kRows);
      } else {
        lim = (j == T - 1) ? row + 1 : kRows;
      }
      // Lazy maximum.  m is the tile-0 row maximum and moves only when a
      // 64-column half would otherwise produce probabilities beyond 2^64
      // (detected from the half's row sum, which the pass computes anyway):
      // P = 2^(s*scale - m) <= 2^64 stays finite in bf16, and summed over up to
      // 2^20 keys it keeps O and l inside the fp32 range for |V| up to ~2^40;
      // the tiles after the first need no pass over the scores for their
      // maximum.  The result is that of the
      // running-maximum softmax up to rounding (O and l share the base m).
      uint32_t sr[64];
      APB_TMEM_LD64(tS, sr);
      if (lim < 64) {
#pragma unroll
        for (int c = 0; c < 64; ++c)
          if (c >= lim) sr[c] = 0xff800000u;   // -inf
      }
      if (j == 0) {
        // the first tile's maximum, the second half read 32 columns at a time
        float mx[8];
#pragma unroll
        for (int x = 0; x < 8; ++x)
          mx[x] = fmaxf(__uint_as_float(sr[2 * x]), __uint_as_float(sr[2 * x + 1]));
#pragma unroll
        for (int c = 16; c < 64; c += 2)
          mx[(c >> 1) & 7] = ptx::fmax3(mx[(c >> 1) & 7], __uint_as_float(sr[c]),
                                        __uint_as_float(sr[c + 1]));
#pragma unroll
        for (int part = 0; part < 2; ++part) {
          uint32_t t[32];
          APB_TMEM_LD32(tS + 64 + 32 * part, t);
#pragma unroll
          for (int x = 0; x < 32; x += 2) {
            const int c = 64 + 32 * part + x;
            const float a0 = c < lim ? __uint_as_float(t[x]) : -INFINITY;
            const float a1 = c + 1 < lim ? __uint_as_float(t[x + 1]) : -INFINITY;
            mx[(x >> 1) & 7] = ptx::fmax3(mx[(x >> 1) & 7], a0, a1);
          }
        }
        m = fmaxf(ptx::fmax3(mx[0], mx[1], mx[2]),
                  fmaxf(ptx::fmax3(mx[3], mx[4], mx[5]), fmaxf(mx[6], mx[7]))) *
            p.scale_log2;
      }
      auto half_max = [&]() -> float {   // this half's maximum (log2 units)
        float mx[4] = {-INFINITY, -INFINITY, -INFINITY, -INFINITY};
#pragma unroll
        for (int c = 0; c < 64; c += 2)
          mx[(c >> 1) & 3] = ptx::fmax3(mx[(c >> 1) & 3], __uint_as_float(sr[c]),
                                        __uint_as_float(sr[c + 1]));
        return fmaxf(fmaxf(mx[0], mx[1]), fmaxf(mx[2], mx[3])) * p.scale_log2;
      };
      // exponentials and row sum of the 64 scores in sr (columns 64*half..)
      auto exps = [&](float mneg, uint32_t (&pk)[32], float (&acc)[4]) {
#pragma unroll
        for (int x = 0; x < 4; ++x) acc[x] = 0.f;
#pragma unroll
        for (int cc = 0; cc < 32; ++cc) {
          float x0, x1, p0, p1;
          ptx::ffma2_scalar(x0, x1, __uint_as_float(sr[2 * cc]), __uint_as_float(sr[2 * cc + 1]),
                            p.scale_log2, mneg);
          p0 = ptx::ex2(x0);
          p1 = ptx::ex2(x1);
          ptx::fadd2_acc(acc[(cc & 1) * 2], acc[(cc & 1) * 2 + 1], p0, p1);
          pk[cc] = ptx::pack_bf16x2(p0, p1);
        }
      };
      constexpr float kSumLimit = 18446744073709551616.0f;   // 2^64
      float sum[4];
      uint32_t pk[32];
      // ---- first half
      exps(-m, pk, sum);
      bool rescale = false;
      float alpha = 1.f;
      if (!((sum[0] + sum[1]) + (sum[2] + sum[3]) < kSumLimit)) {   // rare (and NaN-safe)
        const float m_new = fmaxf(m, half_max());
        alpha = ptx::ex2(m - m_new);
        m = m_new;
        l *= alpha;
        rescale = true;
        exps(-m, pk, sum);
      }
      // O_i is stable here (the commit that signalled S_i(j) covers
      // PV_i(j-1)); it must be rescaled before PV_i(j) starts on half 0
      if (__any_sync(0xffffffffu, rescale)) {
#pragma unroll 1
        for (int c = 0; c < D / 32; ++c) {
          uint32_t o[32];
          APB_TMEM_LD32(tO + 32 * c, o);
#pragma unroll
          for (int x = 0; x < 32; ++x) o[x] = __float_as_uint(__uint_as_float(o[x]) * alpha);
          APB_TMEM_ST32(tO + 32 * c, o);
        }
      }
      APB_TMEM_ST32(tS, pk);
      ptx::tmem_st_wait();
      ptx::tc_fence_before();
      ptx::named_barrier_arrive(kPBar + 2 * i, kPBarThreads);
      ++arrived;
      // ---- second half
      APB_TMEM_LD64(tS + 64, sr);
      if (lim < kRows) {
#pragma unroll
        for (int c = 0; c < 64; ++c)
          if (64 + c >= lim) sr[c] = 0xff800000u;   // -inf
      }
      float sum1[4];
      exps(-m, pk, sum1);
      const bool big = !((sum1[0] + sum1[1]) + (sum1[2] + sum1[3]) < kSumLimit);
      if (__any_sync(0xffffffffu, big)) {
        // rare: m moves after the first half's probabilities went out, so O
        // (which PV_i(j) on the first half is adding to) is rescaled once that
        // PV has run, before the second half's
        const bool w = ptx::mbar_wait_bounded(&bars[PV0_DONE + i], j & 1, gabort, p.wait_ns);
        if (!__all_sync(0xffffffffu, w)) {
          if (lane == 0) record_failure(p.status, kWherePV0 + i, j);
          ok = false;
          break;
        }
        ptx::tc_fence_after();
        float a1 = 1.f;
        if (big) {
          const float m_new = fmaxf(m, half_max());
          a1 = ptx::ex2(m - m_new);
          m = m_new;
          l *= a1;
#pragma unroll
          for (int x = 0; x < 4; ++x) sum[x] *= a1;
          exps(-m, pk, sum1);
        }
        __syncwarp();   // the rows that moved m rejoin before the warp-collective TMEM access
#pragma unroll 1
        for (int c = 0; c < D / 32; ++c) {
          uint32_t o[32];
          APB_TMEM_LD32(tO + 32 * c, o);
#pragma unroll
          for (int x = 0; x < 32; ++x) o[x] = __float_as_uint(__uint_as_float(o[x]) * a1);
          APB_TMEM_ST32(tO + 32 * c, o);
        }
      }
      APB_TMEM_ST32(tS + 32, pk);
      ptx::tmem_st_wait();
      ptx::tc_fence_before();
      ptx::named_barrier_arrive(kPBar + 2 * i + 1, kPBarThreads);
      ++arrived;
#pragma unroll
      for (int x = 0; x < 4; ++x) sum[x] += sum1[x];
      l += (sum[0] + sum[1]) + (sum[2] + sum[3]);
    }
    if (!ok) {
      // The issuer waits for every P half of this tile at named barriers,
      // which have no time limit: meet it at each remaining one (blocking,
      // so that this warp never runs a phase ahead of it).
      for (int a = arrived; a < 2 * T; ++a) {
        __syncwarp();
        ptx::named_barrier_sync(kPBar + 2 * i + (a & 1), kPBarThreads);
      }
    }
    if (ok && T > 0) {
      ok = ptx::mbar_wait_bounded(&bars[O_FINAL + i], 0, gabort, p.wait_ns);
      if (!__all_sync(0xffffffffu, ok)) {
        if (lane == 0) record_failure(p.status, kWhereO + i, T);
        ok = false;
      }
      if (ok) {
        ptx::tc_fence_after();
        const float inv = 1.0f / l;
        const bool valid = q0 + row < p.n;
        const long long tok = (long long)q_row0 + q0 + row;
        __nv_bfloat16* orow = p.out + (tok * p.Hq + head) * D;
#pragma unroll
        for (int c = 0; c < D / 32; ++c) {
          uint32_t o[32];
          APB_TMEM_LD32(tO + 32 * c, o);
          uint32_t w[16];
#pragma unroll
          for (int x = 0; x < 16; ++x)
            w[x] = ptx::pack_bf16x2(__uint_as_float(o[2 * x]) * inv,
                                    __uint_as_float(o[2 * x + 1]) * inv);
          if (valid) {
            uint4* dst = reinterpret_cast<uint4*>(orow + 32 * c);
#pragma unroll
            for (int x = 0; x < 4; ++x)
              dst[x] = make_uint4(w[4 * x], w[4 * x + 1], w[4 * x + 2], w[4 * x + 3]);
          }
        }
        if (p.lse && valid)
          p.lse[(long long)head * p.N + tok] = (m + __log2f(l)) * 0.6931471805599453f;
      }
    }
  }

  ptx::tc_fence_before();
  __syncthreads();
  if (warp == kIssuerWarp) {
    ptx::tc_fence_after();
    ptx::tmem_dealloc(tmem, 512);
  }
}

// ---------------------------------------------------------------- host side

template <int D>
cudaError_t launch_d(const Shape& s, const HostRange& r, const void* q, const void* k,
                     const void* v, const void* pass_k, const void* pass_v, void* out, float* lse,
                     DeviceStatus* status, cudaStream_t st, const char** why) {
  CUtensorMap mQ, mK, mV, mPK, mPV;
  const uint64_t NQ = (uint64_t)r.q_rows, NK = (uint64_t)r.k_rows;
  bool ok = encode_bf16_3d(&mQ, q, D, s.Hq, NQ, (uint64_t)D * 2, (uint64_t)s.Hq * D * 2, 64, 1,
                           kRows) &&
            encode_bf16_3d(&mK, k, D, s.Hkv, NK, (uint64_t)D * 2, (uint64_t)s.Hkv * D * 2, 64, 1,
                           kRows) &&
            encode_bf16_3d(&mV, v, D, s.Hkv, NK, (uint64_t)D * 2, (uint64_t)s.Hkv * D * 2, 64, 1,
                           kRows);
  if (ok && pass_k) {
    // token-major [H*keep, Hkv, d], read like K
    const uint64_t rows = (uint64_t)s.H * s.keep;
    ok = encode_bf16_3d(&mPK, pass_k, D, s.Hkv, rows, (uint64_t)D * 2, (uint64_t)s.Hkv * D * 2,
                        64, 1, kRows) &&
         encode_bf16_3d(&mPV, pass_v, D, s.Hkv, rows, (uint64_t)D * 2, (uint64_t)s.Hkv * D * 2,
                        64, 1, kRows);
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
  p.n_ctas_per_host = ((s.n + kRows - 1) / kRows + 1) / 2;
  p.h0 = r.h0;
  p.hcount = r.count;
  p.hstride = r.stride;
  p.q_row0 = r.q_row0;
  p.k_row0 = r.k_row0;
  p.anchor_row0 = r.anchor_row0;
  p.N = r.q_rows;
  p.scale_log2 = s.scale * kLog2e;
  p.wait_ns = wait_limit_ns();
  p.out = static_cast<__nv_bfloat16*>(out);
  p.lse = lse;
  p.status = status;
  cudaError_t e = cudaFuncSetAttribute(apb_attention_kernel<D>,
                                       cudaFuncAttributeMaxDynamicSharedMemorySize, kSmemBytes);
  if (e != cudaSuccess) return e;
  dim3 grid(p.n_ctas_per_host, s.Hq, r.count);
  apb_attention_kernel<D><<<grid, kThreads, kSmemBytes, st>>>(mQ, mK, mV, mPK, mPV, p);
  return cudaGetLastError();
}

}  // namespace

cudaError_t launch_attention(const Shape& s, const HostRange& r, const void* q, const void* k,
                             const void* v, const void* pass_k, const void* pass_v, void* out,
                             float* lse, DeviceStatus* status, cudaStream_t st, const char** why) {
  if (s.d == 128) return launch_d<128>(s, r, q, k, v, pass_k, pass_v, out, lse, status, st, why);
  return launch_d<64>(s, r, q, k, v, pass_k, pass_v, out, lse, status, st, why);
}

}  // namespace apb

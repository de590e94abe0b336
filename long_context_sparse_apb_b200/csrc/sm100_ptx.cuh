// Thin inline-PTX wrappers for the sm_100a features the attention kernel
// uses: mbarriers with bounded waits, TMA tile loads, tcgen05 (TMEM
// allocation, UMMA issue/commit, TMEM loads/stores) and the shared-memory
// matrix descriptors UMMA reads its operands through.
#pragma once

#include <cuda.h>
#include <stdint.h>

namespace apb {
namespace ptx {

__device__ __forceinline__ uint32_t smem_u32(const void* p) {
  return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

// 16 bytes of read-only global data that is read once: not allocated in L1,
// so the stream does not take L1 fills from the shared-memory traffic of the
// same SM.  Volatile so that it is never hoisted above the caller's bounds
// check.
__device__ __forceinline__ uint4 ld_stream_16(const void* p) {
  uint4 r;
  asm volatile("ld.global.nc.L1::no_allocate.v4.u32 {%0, %1, %2, %3}, [%4];"
               : "=r"(r.x), "=r"(r.y), "=r"(r.z), "=r"(r.w)
               : "l"(p));
  return r;
}

__device__ __forceinline__ uint64_t globaltimer() {
  uint64_t t;
  asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
  return t;
}

// ------------------------------------------------------------------ mbarrier
__device__ __forceinline__ void mbar_init(uint64_t* bar, uint32_t count) {
  asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(smem_u32(bar)), "r"(count)
               : "memory");
}

__device__ __forceinline__ void fence_mbar_init() {
  asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
}

__device__ __forceinline__ void mbar_arrive(uint64_t* bar) {
  asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(smem_u32(bar)) : "memory");
}

__device__ __forceinline__ void mbar_arrive_expect_tx(uint64_t* bar, uint32_t bytes) {
  asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(smem_u32(bar)),
               "r"(bytes)
               : "memory");
}

__device__ __forceinline__ bool mbar_try_wait(uint32_t bar, uint32_t parity) {
  uint32_t ok;
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
      "selp.u32 %0, 1, 0, p;\n\t}"
      : "=r"(ok)
      : "r"(bar), "r"(parity)
      : "memory");
  return ok != 0;
}

__device__ __forceinline__ bool mbar_test_wait(uint32_t bar, uint32_t parity) {
  uint32_t ok;
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "mbarrier.test_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
      "selp.u32 %0, 1, 0, p;\n\t}"
      : "=r"(ok)
      : "r"(bar), "r"(parity)
      : "memory");
  return ok != 0;
}

// Like mbar_wait_bounded below, but polls without suspending the thread, for
// the single thread whose reaction time is on the critical path (the UMMA
// issuer): it sees the phase flip within a few cycles instead of after a
// suspend/wake round trip.
__device__ __forceinline__ bool mbar_spin_bounded(uint64_t* bar, uint32_t parity,
                                                  const volatile uint32_t* abort,
                                                  uint64_t limit_ns) {
  const uint32_t a = smem_u32(bar);
  if (mbar_test_wait(a, parity)) return true;
  const uint64_t t0 = globaltimer();
  while (true) {
#pragma unroll 1
    for (int i = 0; i < 256; ++i)
      if (mbar_test_wait(a, parity)) return true;
    if (*abort != 0u) return false;
    if (globaltimer() - t0 > limit_ns) return false;
  }
}

// Waits for the phase of parity `parity` of `bar` to complete.  Gives up and
// returns false when `limit_ns` of wall time pass, or when *abort (a flag in
// global memory that another CTA of the launch may set) becomes non-zero.
__device__ __forceinline__ bool mbar_wait_bounded(uint64_t* bar, uint32_t parity,
                                                  const volatile uint32_t* abort,
                                                  uint64_t limit_ns) {
  const uint32_t a = smem_u32(bar);
  if (mbar_try_wait(a, parity)) return true;
  const uint64_t t0 = globaltimer();
  while (true) {
#pragma unroll 1
    for (int i = 0; i < 32; ++i)
      if (mbar_try_wait(a, parity)) return true;
    if (*abort != 0u) return false;
    if (globaltimer() - t0 > limit_ns) return false;
  }
}

// ------------------------------------------------------------------ TMA
__device__ __forceinline__ void tma_prefetch_desc(const CUtensorMap* m) {
  asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(m)) : "memory");
}

__device__ __forceinline__ void tma_load_3d(void* dst, const CUtensorMap* m, uint64_t* bar, int c0,
                                            int c1, int c2) {
  asm volatile(
      "cp.async.bulk.tensor.3d.shared::cluster.global.mbarrier::complete_tx::bytes"
      " [%0], [%1, {%3, %4, %5}], [%2];" ::"r"(smem_u32(dst)),
      "l"(reinterpret_cast<uint64_t>(m)), "r"(smem_u32(bar)), "r"(c0), "r"(c1), "r"(c2)
      : "memory");
}

// Warms L2 with one box of a tensor map (no shared memory, no barrier).
__device__ __forceinline__ void tma_prefetch_l2_3d(const CUtensorMap* m, int c0, int c1, int c2) {
  asm volatile("cp.async.bulk.prefetch.tensor.3d.L2.global.tile [%0, {%1, %2, %3}];" ::"l"(
                   reinterpret_cast<uint64_t>(m)),
               "r"(c0), "r"(c1), "r"(c2)
               : "memory");
}

// AND of `pred` over the `nthreads` threads meeting at named barrier `id`.
__device__ __forceinline__ bool barrier_and(int id, int nthreads, bool pred) {
  uint32_t out;
  asm volatile(
      "{\n .reg .pred pi, po;\n setp.ne.u32 pi, %1, 0;\n"
      " bar.red.and.pred po, %2, %3, pi;\n selp.u32 %0, 1, 0, po;\n}"
      : "=r"(out)
      : "r"((uint32_t)pred), "r"(id), "r"(nthreads)
      : "memory");
  return out != 0u;
}

__device__ __forceinline__ void named_barrier_sync(int id, int nthreads) {
  asm volatile("bar.sync %0, %1;" ::"r"(id), "r"(nthreads) : "memory");
}

// Arrives at named barrier `id` (counting `nthreads` in all) without waiting.
__device__ __forceinline__ void named_barrier_arrive(int id, int nthreads) {
  asm volatile("bar.arrive %0, %1;" ::"r"(id), "r"(nthreads) : "memory");
}

__device__ __forceinline__ void fence_proxy_async_smem() {
  asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}

// ------------------------------------------------------------------ tcgen05
__device__ __forceinline__ void tmem_alloc(uint32_t* dst_smem, uint32_t ncols) {
  asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(
                   smem_u32(dst_smem)),
               "r"(ncols)
               : "memory");
}
__device__ __forceinline__ void tmem_relinquish() {
  asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
}
__device__ __forceinline__ void tmem_dealloc(uint32_t taddr, uint32_t ncols) {
  asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(taddr), "r"(ncols)
               : "memory");
}
__device__ __forceinline__ void tc_fence_before() {
  asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
}
__device__ __forceinline__ void tc_fence_after() {
  asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
}

// D[tmem] (+)= A[smem] * B[smem], kind::f16 (bf16 inputs, fp32 accumulate).
__device__ __forceinline__ void umma_bf16_ss(uint32_t d_tmem, uint64_t a_desc, uint64_t b_desc,
                                             uint32_t idesc, uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n\t}" ::"r"(d_tmem),
      "l"(a_desc), "l"(b_desc), "r"(idesc), "r"(accumulate)
      : "memory");
}

// Arrives once on `bar` when every tcgen05 operation this thread issued
// before it has completed.
__device__ __forceinline__ void umma_commit(uint64_t* bar) {
  asm volatile(
      "tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(
          smem_u32(bar))
      : "memory");
}

// Instruction descriptor of kind::f16: bf16 A and B, fp32 D, M x N tile;
// b_mn_major selects an MN-major B operand (else K-major).
__host__ __device__ constexpr uint32_t idesc_bf16_f32(int M, int N, int b_mn_major) {
  return (1u << 4)                              // D format: f32
         | (1u << 7)                            // A format: bf16
         | (1u << 10)                           // B format: bf16
         | ((uint32_t)b_mn_major << 16)         // B major
         | ((uint32_t)(N >> 3) << 17)           // N / 8
         | ((uint32_t)(M >> 4) << 24);          // M / 16
}

// Shared-memory matrix descriptor, 128-byte swizzle (sm_100 version bit set).
// lbo/sbo in bytes.
__device__ __forceinline__ uint64_t sdesc_sw128(uint32_t smem_addr, uint32_t lbo, uint32_t sbo) {
  uint64_t d = 0;
  d |= (uint64_t)((smem_addr >> 4) & 0x3FFFu);
  d |= (uint64_t)((lbo >> 4) & 0x3FFFu) << 16;
  d |= (uint64_t)((sbo >> 4) & 0x3FFFu) << 32;
  d |= (uint64_t)1u << 46;   // descriptor version for sm_100
  d |= (uint64_t)2u << 61;   // SWIZZLE_128B
  return d;
}

// 32 lanes x 32 consecutive 32-bit columns per warp; this thread receives
// its lane's columns.  The wait is inside the same statement so no register
// can be consumed before the data has landed.
#define APB_TMEM_LD32(taddr, r)                                                                  \
  asm volatile(                                                                                  \
      "tcgen05.ld.sync.aligned.32x32b.x32.b32 {%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14," \
      "%15,%16,%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31}, [%32];\n\t"         \
      "tcgen05.wait::ld.sync.aligned;"                                                           \
      : "=r"((r)[0]), "=r"((r)[1]), "=r"((r)[2]), "=r"((r)[3]), "=r"((r)[4]), "=r"((r)[5]), "=r"((r)[6]),      \
        "=r"((r)[7]), "=r"((r)[8]), "=r"((r)[9]), "=r"((r)[10]), "=r"((r)[11]), "=r"((r)[12]), "=r"((r)[13]),  \
        "=r"((r)[14]), "=r"((r)[15]), "=r"((r)[16]), "=r"((r)[17]), "=r"((r)[18]), "=r"((r)[19]),            \
        "=r"((r)[20]), "=r"((r)[21]), "=r"((r)[22]), "=r"((r)[23]), "=r"((r)[24]), "=r"((r)[25]),            \
        "=r"((r)[26]), "=r"((r)[27]), "=r"((r)[28]), "=r"((r)[29]), "=r"((r)[30]), "=r"((r)[31])             \
      : "r"(taddr)                                                                               \
      : "memory")

// The same load without its wait, so that it overlaps other work; the
// registers may be read only after APB_TMEM_WAIT32 on the same array, which
// lists them as read-written so the compiler cannot move a use above it.
#define APB_TMEM_LD32_ASYNC(taddr, r)                                                            \
  asm volatile(                                                                                  \
      "tcgen05.ld.sync.aligned.32x32b.x32.b32 {%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14," \
      "%15,%16,%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31}, [%32];"            \
      : "=r"((r)[0]), "=r"((r)[1]), "=r"((r)[2]), "=r"((r)[3]), "=r"((r)[4]), "=r"((r)[5]), "=r"((r)[6]),      \
        "=r"((r)[7]), "=r"((r)[8]), "=r"((r)[9]), "=r"((r)[10]), "=r"((r)[11]), "=r"((r)[12]), "=r"((r)[13]),  \
        "=r"((r)[14]), "=r"((r)[15]), "=r"((r)[16]), "=r"((r)[17]), "=r"((r)[18]), "=r"((r)[19]),            \
        "=r"((r)[20]), "=r"((r)[21]), "=r"((r)[22]), "=r"((r)[23]), "=r"((r)[24]), "=r"((r)[25]),            \
        "=r"((r)[26]), "=r"((r)[27]), "=r"((r)[28]), "=r"((r)[29]), "=r"((r)[30]), "=r"((r)[31])             \
      : "r"(taddr)                                                                               \
      : "memory")

#define APB_TMEM_WAIT32(r)                                                                       \
  asm volatile("tcgen05.wait::ld.sync.aligned;"                                                  \
               : "+r"((r)[0]), "+r"((r)[1]), "+r"((r)[2]), "+r"((r)[3]), "+r"((r)[4]), "+r"((r)[5]),          \
                 "+r"((r)[6]), "+r"((r)[7]), "+r"((r)[8]), "+r"((r)[9]), "+r"((r)[10]), "+r"((r)[11]),        \
                 "+r"((r)[12]), "+r"((r)[13]), "+r"((r)[14]), "+r"((r)[15]), "+r"((r)[16]), "+r"((r)[17]),    \
                 "+r"((r)[18]), "+r"((r)[19]), "+r"((r)[20]), "+r"((r)[21]), "+r"((r)[22]), "+r"((r)[23]),    \
                 "+r"((r)[24]), "+r"((r)[25]), "+r"((r)[26]), "+r"((r)[27]), "+r"((r)[28]), "+r"((r)[29]),    \
                 "+r"((r)[30]), "+r"((r)[31])                                                    \
               :                                                                                 \
               : "memory")

#define APB_TMEM_ST32(taddr, r)                                                                  \
  asm volatile(                                                                                  \
      "tcgen05.st.sync.aligned.32x32b.x32.b32 [%0], {%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13," \
      "%14,%15,%16,%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31,%32};" ::"r"(taddr), \
      "r"((r)[0]), "r"((r)[1]), "r"((r)[2]), "r"((r)[3]), "r"((r)[4]), "r"((r)[5]), "r"((r)[6]), "r"((r)[7]),    \
      "r"((r)[8]), "r"((r)[9]), "r"((r)[10]), "r"((r)[11]), "r"((r)[12]), "r"((r)[13]), "r"((r)[14]),          \
      "r"((r)[15]), "r"((r)[16]), "r"((r)[17]), "r"((r)[18]), "r"((r)[19]), "r"((r)[20]), "r"((r)[21]),        \
      "r"((r)[22]), "r"((r)[23]), "r"((r)[24]), "r"((r)[25]), "r"((r)[26]), "r"((r)[27]), "r"((r)[28]),        \
      "r"((r)[29]), "r"((r)[30]), "r"((r)[31])                                                         \
      : "memory")

// 32 lanes x 128 consecutive 32-bit columns (one full 128-column S tile per
// thread row), waited on inside the same statement.
#define APB_TMEM_LD128(taddr, r)                                              \
  asm volatile(                                                              \
      "tcgen05.ld.sync.aligned.32x32b.x128.b32 {%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,%16,%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31,%32,%33,%34,%35,%36,%37,%38,%39,%40,%41,%42,%43,%44,%45,%46,%47,%48,%49,%50,%51,%52,%53,%54,%55,%56,%57,%58,%59,%60,%61,%62,%63,%64,%65,%66,%67,%68,%69,%70,%71,%72,%73,%74,%75,%76,%77,%78,%79,%80,%81,%82,%83,%84,%85,%86,%87,%88,%89,%90,%91,%92,%93,%94,%95,%96,%97,%98,%99,%100,%101,%102,%103,%104,%105,%106,%107,%108,%109,%110,%111,%112,%113,%114,%115,%116,%117,%118,%119,%120,%121,%122,%123,%124,%125,%126,%127}, [%128];\n\t" \
      "tcgen05.wait::ld.sync.aligned;"                                       \
      : "=r"((r)[0]), "=r"((r)[1]), "=r"((r)[2]), "=r"((r)[3]), "=r"((r)[4]), "=r"((r)[5]), "=r"((r)[6]), "=r"((r)[7]), "=r"((r)[8]), "=r"((r)[9]), "=r"((r)[10]), "=r"((r)[11]), "=r"((r)[12]), "=r"((r)[13]), "=r"((r)[14]), "=r"((r)[15]), "=r"((r)[16]), "=r"((r)[17]), "=r"((r)[18]), "=r"((r)[19]), "=r"((r)[20]), "=r"((r)[21]), "=r"((r)[22]), "=r"((r)[23]), "=r"((r)[24]), "=r"((r)[25]), "=r"((r)[26]), "=r"((r)[27]), "=r"((r)[28]), "=r"((r)[29]), "=r"((r)[30]), "=r"((r)[31]), "=r"((r)[32]), "=r"((r)[33]), "=r"((r)[34]), "=r"((r)[35]), "=r"((r)[36]), "=r"((r)[37]), "=r"((r)[38]), "=r"((r)[39]), "=r"((r)[40]), "=r"((r)[41]), "=r"((r)[42]), "=r"((r)[43]), "=r"((r)[44]), "=r"((r)[45]), "=r"((r)[46]), "=r"((r)[47]), "=r"((r)[48]), "=r"((r)[49]), "=r"((r)[50]), "=r"((r)[51]), "=r"((r)[52]), "=r"((r)[53]), "=r"((r)[54]), "=r"((r)[55]), "=r"((r)[56]), "=r"((r)[57]), "=r"((r)[58]), "=r"((r)[59]), "=r"((r)[60]), "=r"((r)[61]), "=r"((r)[62]), "=r"((r)[63]), "=r"((r)[64]), "=r"((r)[65]), "=r"((r)[66]), "=r"((r)[67]), "=r"((r)[68]), "=r"((r)[69]), "=r"((r)[70]), "=r"((r)[71]), "=r"((r)[72]), "=r"((r)[73]), "=r"((r)[74]), "=r"((r)[75]), "=r"((r)[76]), "=r"((r)[77]), "=r"((r)[78]), "=r"((r)[79]), "=r"((r)[80]), "=r"((r)[81]), "=r"((r)[82]), "=r"((r)[83]), "=r"((r)[84]), "=r"((r)[85]), "=r"((r)[86]), "=r"((r)[87]), "=r"((r)[88]), "=r"((r)[89]), "=r"((r)[90]), "=r"((r)[91]), "=r"((r)[92]), "=r"((r)[93]), "=r"((r)[94]), "=r"((r)[95]), "=r"((r)[96]), "=r"((r)[97]), "=r"((r)[98]), "=r"((r)[99]), "=r"((r)[100]), "=r"((r)[101]), "=r"((r)[102]), "=r"((r)[103]), "=r"((r)[104]), "=r"((r)[105]), "=r"((r)[106]), "=r"((r)[107]), "=r"((r)[108]), "=r"((r)[109]), "=r"((r)[110]), "=r"((r)[111]), "=r"((r)[112]), "=r"((r)[113]), "=r"((r)[114]), "=r"((r)[115]), "=r"((r)[116]), "=r"((r)[117]), "=r"((r)[118]), "=r"((r)[119]), "=r"((r)[120]), "=r"((r)[121]), "=r"((r)[122]), "=r"((r)[123]), "=r"((r)[124]), "=r"((r)[125]), "=r"((r)[126]), "=r"((r)[127])                                                             \
      : "r"(taddr)                                                           \
      : "memory")

// 32 lanes x 64 consecutive 32-bit columns (half of a 128-column S tile),
// waited on inside the same statement.
#define APB_TMEM_LD64(taddr, r)                                               \
  asm volatile(                                                              \
      "tcgen05.ld.sync.aligned.32x32b.x64.b32 {%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,%16,%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31,%32,%33,%34,%35,%36,%37,%38,%39,%40,%41,%42,%43,%44,%45,%46,%47,%48,%49,%50,%51,%52,%53,%54,%55,%56,%57,%58,%59,%60,%61,%62,%63}, [%64];\n\t" \
      "tcgen05.wait::ld.sync.aligned;"                                       \
      : "=r"((r)[0]), "=r"((r)[1]), "=r"((r)[2]), "=r"((r)[3]), "=r"((r)[4]), "=r"((r)[5]), "=r"((r)[6]), "=r"((r)[7]), "=r"((r)[8]), "=r"((r)[9]), "=r"((r)[10]), "=r"((r)[11]), "=r"((r)[12]), "=r"((r)[13]), "=r"((r)[14]), "=r"((r)[15]), "=r"((r)[16]), "=r"((r)[17]), "=r"((r)[18]), "=r"((r)[19]), "=r"((r)[20]), "=r"((r)[21]), "=r"((r)[22]), "=r"((r)[23]), "=r"((r)[24]), "=r"((r)[25]), "=r"((r)[26]), "=r"((r)[27]), "=r"((r)[28]), "=r"((r)[29]), "=r"((r)[30]), "=r"((r)[31]), "=r"((r)[32]), "=r"((r)[33]), "=r"((r)[34]), "=r"((r)[35]), "=r"((r)[36]), "=r"((r)[37]), "=r"((r)[38]), "=r"((r)[39]), "=r"((r)[40]), "=r"((r)[41]), "=r"((r)[42]), "=r"((r)[43]), "=r"((r)[44]), "=r"((r)[45]), "=r"((r)[46]), "=r"((r)[47]), "=r"((r)[48]), "=r"((r)[49]), "=r"((r)[50]), "=r"((r)[51]), "=r"((r)[52]), "=r"((r)[53]), "=r"((r)[54]), "=r"((r)[55]), "=r"((r)[56]), "=r"((r)[57]), "=r"((r)[58]), "=r"((r)[59]), "=r"((r)[60]), "=r"((r)[61]), "=r"((r)[62]), "=r"((r)[63])                                                 \
      : "r"(taddr)                                                           \
      : "memory")

// Stores 64 consecutive 32-bit columns of this thread's lane.
#define APB_TMEM_ST64(taddr, r)                                               \
  asm volatile(                                                              \
      "tcgen05.st.sync.aligned.32x32b.x64.b32 [%0], {%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,%16,%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31,%32,%33,%34,%35,%36,%37,%38,%39,%40,%41,%42,%43,%44,%45,%46,%47,%48,%49,%50,%51,%52,%53,%54,%55,%56,%57,%58,%59,%60,%61,%62,%63,%64};"        \
      :: "r"(taddr), "r"((r)[0]), "r"((r)[1]), "r"((r)[2]), "r"((r)[3]), "r"((r)[4]), "r"((r)[5]), "r"((r)[6]), "r"((r)[7]), "r"((r)[8]), "r"((r)[9]), "r"((r)[10]), "r"((r)[11]), "r"((r)[12]), "r"((r)[13]), "r"((r)[14]), "r"((r)[15]), "r"((r)[16]), "r"((r)[17]), "r"((r)[18]), "r"((r)[19]), "r"((r)[20]), "r"((r)[21]), "r"((r)[22]), "r"((r)[23]), "r"((r)[24]), "r"((r)[25]), "r"((r)[26]), "r"((r)[27]), "r"((r)[28]), "r"((r)[29]), "r"((r)[30]), "r"((r)[31]), "r"((r)[32]), "r"((r)[33]), "r"((r)[34]), "r"((r)[35]), "r"((r)[36]), "r"((r)[37]), "r"((r)[38]), "r"((r)[39]), "r"((r)[40]), "r"((r)[41]), "r"((r)[42]), "r"((r)[43]), "r"((r)[44]), "r"((r)[45]), "r"((r)[46]), "r"((r)[47]), "r"((r)[48]), "r"((r)[49]), "r"((r)[50]), "r"((r)[51]), "r"((r)[52]), "r"((r)[53]), "r"((r)[54]), "r"((r)[55]), "r"((r)[56]), "r"((r)[57]), "r"((r)[58]), "r"((r)[59]), "r"((r)[60]), "r"((r)[61]), "r"((r)[62]), "r"((r)[63])                                                 \
      : "memory")

// D[tmem] (+)= A[tmem] * B[smem], kind::f16: A (M x 16 per instruction) is
// read from tensor memory, lane = row, each 32-bit column holding two
// consecutive K elements; B from a shared-memory descriptor.
__device__ __forceinline__ void umma_bf16_ts(uint32_t d_tmem, uint32_t a_tmem, uint64_t b_desc,
                                             uint32_t idesc, uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], [%1], %2, %3, p;\n\t}" ::"r"(d_tmem),
      "r"(a_tmem), "l"(b_desc), "r"(idesc), "r"(accumulate)
      : "memory");
}

__device__ __forceinline__ void tmem_st_wait() {
  asm volatile("tcgen05.wait::st.sync.aligned;" ::: "memory");
}

__device__ __forceinline__ float ex2(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}

__device__ __forceinline__ uint32_t pack_bf16x2(float lo, float hi) {
  uint32_t r;
  asm("cvt.rn.bf16x2.f32 %0, %1, %2;" : "=r"(r) : "f"(hi), "f"(lo));
  return r;
}

// ---------------------------------------------------------------- packed fp32
// (x0, x1) * (a, a) + (b, b) as one packed f32x2 FMA.
__device__ __forceinline__ void ffma2_scalar(float& y0, float& y1, float x0, float x1, float a,
                                             float b) {
  asm("{\n\t.reg .b64 u, v, w, r;\n\t"
      "mov.b64 u, {%2, %3};\n\t"
      "mov.b64 v, {%4, %4};\n\t"
      "mov.b64 w, {%5, %5};\n\t"
      "fma.rn.f32x2 r, u, v, w;\n\t"
      "mov.b64 {%0, %1}, r;\n\t}"
      : "=f"(y0), "=f"(y1)
      : "f"(x0), "f"(x1), "f"(a), "f"(b));
}

// (acc0, acc1) += (x0, x1) as one packed f32x2 add.
__device__ __forceinline__ void fadd2_acc(float& acc0, float& acc1, float x0, float x1) {
  asm("{\n\t.reg .b64 u, v;\n\t"
      "mov.b64 u, {%0, %1};\n\t"
      "mov.b64 v, {%2, %3};\n\t"
      "add.rn.f32x2 u, u, v;\n\t"
      "mov.b64 {%0, %1}, u;\n\t}"
      : "+f"(acc0), "+f"(acc1)
      : "f"(x0), "f"(x1));
}

__device__ __forceinline__ float fmax3(float a, float b, float c) {
  float d;
  asm("max.f32 %0, %1, %2, %3;" : "=f"(d) : "f"(a), "f"(b), "f"(c));
  return d;
}

}  // namespace ptx
}  // namespace apb

// Internal launchers shared by the C-ABI layer (apb_abi.cu) and the kernels.
#pragma once

#include <cuda.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "../../include/apb.h"

namespace apb {

// Sets the thread-local message that apb_last_error() returns (printf-style)
// and returns `st`; cuda_fail does the same for a CUDA runtime error, as
// APB_ERR_CUDA with "<what>: <CUDA error string>".
apb_status fail(apb_status st, const char* fmt, ...);
apb_status cuda_fail(cudaError_t e, const char* what);

// Time limit of the kernels' bounded waits for launches made now (1 s
// unless a test shortened it with apb_selftest_set_wait_limit).
uint64_t wait_limit_ns();

// Status block at the start of every workspace.
// "where" codes: 40-75 the attention kernel (named kWhere* in
// attention.cu), 80-90 the score kernel (80/82 + CTA rank: weight / k,v
// producer; 84 accumulator free; 85 chunk operands; 86 + rank q converter
// slots; 88 + rank epilogue; 90 shared-memory alignment check).
struct DeviceStatus {
  uint32_t sticky;     // OR of error bits since last clear
  uint32_t abort;      // set inside a launch once one CTA gave up
  uint32_t where;      // role/barrier id of the first failed wait
  uint32_t tile;       // tile index of the first failed wait
};
// Bytes [64, 80) of the status block: elapsed times written by the wait
// self-test; the rest of the 256 bytes is reserved.
constexpr uint32_t kErrWaitTimeout = 1u;
constexpr size_t kStatusBytes = 256;

struct Shape {
  int H, n, A, ql, keep, Hq, Hkv, d, hidden;
  long long N;
  float scale;
};

// 3-D bf16 tensor map with 128-byte swizzle, zero fill out of bounds.
bool encode_bf16_3d(CUtensorMap* m, const void* base, uint64_t d0, uint64_t d1, uint64_t d2,
                    uint64_t stride1_bytes, uint64_t stride2_bytes, uint32_t b0, uint32_t b1,
                    uint32_t b2);

// Bytes of the bf16 hi/lo split of W1 kept in the workspace.
inline size_t weight_split_bytes(const Shape& s) {
  return (size_t)s.Hkv * 2 * s.hidden * 3 * s.d * 2;
}
// Bytes of the folded first-layer bias of the query-aware score variant.
inline size_t query_bias_bytes(const Shape& s) { return (size_t)s.Hkv * s.hidden * 4; }

// qbias == nullptr: the retaining-score stand-in on each token's own q.
// qbias != nullptr: the query-aware variant; the query segment's mean q is
// folded into a first-layer bias written to qbias ([Hkv, hidden] fp32) and
// the q section of the product is skipped.
cudaError_t launch_score(const Shape& s, const void* q, const void* k, const void* v,
                         const float* w1, const float* b1, const float* w2,
                         const float* b2, float* scores, void* wsplit, float* qbias,
                         DeviceStatus* status, cudaStream_t st, const char** why);
cudaError_t launch_topk(const Shape& s, const float* scores, int32_t* idx, cudaStream_t st);
// Top-k and the passing-block gather in one launch (pass_k / pass_v as in
// launch_gather).
cudaError_t launch_topk_gather(const Shape& s, const float* scores, int32_t* idx, const void* k,
                               const void* v, void* pass_k, void* pass_v, cudaStream_t st);
cudaError_t launch_gather(const Shape& s, const void* k, const void* v, const int32_t* idx,
                          void* pass_k, void* pass_v, cudaStream_t st);
// Hosts [hb, he) of one attention launch and where their rows sit: row of
// host hb's first token in the Q/out buffer (q_row0) and in the K/V buffer
// (k_row0), row of the anchor's first token in K/V, and the buffers' rows.
// The hosts h0, h0 + stride, ..., h0 + (count - 1) * stride of one attention
// launch, whose rows sit one after another (in that order) in the Q/out and
// K/V buffers from q_row0 and k_row0; the anchor's rows start at anchor_row0.
struct HostRange {
  int h0, count, stride, q_row0, k_row0, anchor_row0;
  long long q_rows, k_rows;
};

// The bounded-wait self-test on `status` (two CTAs waiting on barriers that
// nothing completes; CTA 0 gives up after limit_us, CTA 1 through the abort
// flag); the two waits' durations go to elapsed_ns[0..1].
cudaError_t launch_wait_selftest(DeviceStatus* status, uint32_t limit_us,
                                 unsigned long long* elapsed_ns, cudaStream_t st);

// Returns cudaSuccess or an error; sets *why when a TMA descriptor could not
// be built (reported as APB_ERR_CUDA with a message).
cudaError_t launch_attention(const Shape& s, const HostRange& r, const void* q, const void* k,
                             const void* v, const void* pass_k, const void* pass_v, void* out,
                             float* lse, DeviceStatus* status, cudaStream_t st, const char** why);

}  // namespace apb

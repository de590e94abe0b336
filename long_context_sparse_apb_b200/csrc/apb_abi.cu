// C-ABI layer: argument checks, workspace layout, status reporting.
// Every entry point validates on the host before launching anything and
// returns an apb_status; no exception or abort crosses the boundary.
#include <atomic>
#include <cmath>
#include <cstdarg>
#include <cstdio>
#include <cstring>

#include "apb_internal.h"

namespace {
thread_local char g_last_error[512] = "";
constexpr uint64_t kDefaultWaitNs = 1000000000ull;   // 1 s
std::atomic<uint64_t> g_wait_ns{kDefaultWaitNs};
}  // namespace

namespace apb {

apb_status fail(apb_status st, const char* fmt, ...) {
  va_list ap;
  va_start(ap, fmt);
  vsnprintf(g_last_error, sizeof(g_last_error), fmt, ap);
  va_end(ap);
  return st;
}

apb_status cuda_fail(cudaError_t e, const char* what) {
  return fail(APB_ERR_CUDA, "%s: %s", what, cudaGetErrorString(e));
}

uint64_t wait_limit_ns() { return g_wait_ns.load(std::memory_order_relaxed); }

}  // namespace apb

namespace {

using apb::cuda_fail;
using apb::fail;

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

// Checks the shape rules of apb_config; fills `s` on success.
apb_status check_config(const apb_config* c, apb::Shape* s) {
  if (!c) return fail(APB_ERR_INVALID_ARG, "config is NULL");
  if (c->n_hosts < 1) return fail(APB_ERR_INVALID_ARG, "n_hosts=%d < 1", c->n_hosts);
  if (c->block_len < 1) return fail(APB_ERR_INVALID_ARG, "block_len=%d < 1", c->block_len);
  if (c->query_len < 0 || c->query_len > c->anchor_len || c->anchor_len > c->block_len)
    return fail(APB_ERR_INVALID_ARG, "need 0 <= query_len(%d) <= anchor_len(%d) <= block_len(%d)",
                c->query_len, c->anchor_len, c->block_len);
  if (c->keep < 0 || c->keep > c->block_len)
    return fail(APB_ERR_INVALID_ARG, "need 0 <= keep(%d) <= block_len(%d)", c->keep, c->block_len);
  if (c->n_q_heads < 1 || c->n_kv_heads < 1 || c->n_q_heads % c->n_kv_heads != 0)
    return fail(APB_ERR_INVALID_ARG, "n_q_heads(%d) must be a positive multiple of n_kv_heads(%d)",
                c->n_q_heads, c->n_kv_heads);
  if (!(c->softmax_scale == c->softmax_scale))
    return fail(APB_ERR_INVALID_ARG, "softmax_scale is NaN");
  if (c->head_dim != 64 && c->head_dim != 128)
    return fail(APB_ERR_UNSUPPORTED, "head_dim=%d (supported: 64, 128)", c->head_dim);
  if (c->mlp_hidden != 256)
    return fail(APB_ERR_UNSUPPORTED, "mlp_hidden=%d (supported: 256)", c->mlp_hidden);
  long long N = (long long)c->n_hosts * c->block_len;
  if (N > (1ll << 31) - 1) return fail(APB_ERR_UNSUPPORTED, "sequence length %lld >= 2^31", N);
  if ((long long)c->n_hosts * c->keep > (1ll << 31) - 1)
    return fail(APB_ERR_UNSUPPORTED, "n_hosts*keep >= 2^31");
  s->H = c->n_hosts;
  s->n = c->block_len;
  s->A = c->anchor_len;
  s->ql = c->query_len;
  s->keep = c->keep;
  s->Hq = c->n_q_heads;
  s->Hkv = c->n_kv_heads;
  s->d = c->head_dim;
  s->hidden = c->mlp_hidden;
  s->N = N;
  s->scale = c->softmax_scale > 0.f ? c->softmax_scale : 1.0f / std::sqrt((float)c->head_dim);
  return APB_OK;
}

size_t round256(size_t x) { return (x + 255) & ~size_t(255); }

}  // namespace

extern "C" {

size_t apb_workspace_bytes(const apb_config* cfg) {
  apb::Shape s;
  if (check_config(cfg, &s) != APB_OK) return 0;
  return apb::kStatusBytes + round256(apb::weight_split_bytes(s)) +
         round256(apb::query_bias_bytes(s)) + round256((size_t)s.Hkv * (size_t)s.N * sizeof(float));
}

}  // extern "C"

namespace {

// pass_k / pass_v non-NULL: the passing block is built in the top-k launch.
apb_status score_compress_impl(const char* who, bool query_aware, const apb_config* cfg,
                               const void* q, const void* k, const void* v, const float* w1,
                               const float* b1, const float* w2, const float* b2, float* scores,
                               int32_t* idx, void* pass_k, void* pass_v, void* workspace,
                               size_t ws_bytes, void* stream) {
  apb::Shape s;
  apb_status st = check_config(cfg, &s);
  if (st != APB_OK) return st;
  if (!q || !k || !v || !w1 || !b1 || !w2 || !b2 || !workspace)
    return fail(APB_ERR_INVALID_ARG, "%s: NULL input or workspace", who);
  if (s.keep > 0 && !idx) return fail(APB_ERR_INVALID_ARG, "%s: idx is NULL", who);
  const bool fused = pass_k || pass_v;
  if (fused && s.keep > 0 && (!pass_k || !pass_v || !aligned16(pass_k) || !aligned16(pass_v)))
    return fail(APB_ERR_INVALID_ARG, "%s: pass_k / pass_v NULL or not 16-byte aligned", who);
  if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(w1) || !aligned16(workspace) ||
      (scores && !aligned16(scores)) || (idx && !aligned16(idx)))
    return fail(APB_ERR_INVALID_ARG, "%s: pointers must be 16-byte aligned", who);
  const size_t wsplit = round256(apb::weight_split_bytes(s));
  const size_t qbias = round256(apb::query_bias_bytes(s));
  const size_t need = scores ? apb::kStatusBytes + wsplit + (query_aware ? qbias : 0)
                             : apb_workspace_bytes(cfg);
  if (ws_bytes < need)
    return fail(APB_ERR_INVALID_ARG, "%s: workspace %zu < %zu bytes", who, ws_bytes, need);
  cudaStream_t cs = reinterpret_cast<cudaStream_t>(stream);
  char* ws = static_cast<char*>(workspace);
  auto* status = reinterpret_cast<apb::DeviceStatus*>(ws);
  float* sc = scores ? scores : reinterpret_cast<float*>(ws + apb::kStatusBytes + wsplit + qbias);
  float* qb = query_aware ? reinterpret_cast<float*>(ws + apb::kStatusBytes + wsplit) : nullptr;
  cudaError_t e = cudaMemsetAsync(&status->abort, 0, sizeof(uint32_t), cs);
  if (e != cudaSuccess) return cuda_fail(e, "clearing abort flag");
  const char* why = nullptr;
  e = apb::launch_score(s, q, k, v, w1, b1, w2, b2, sc, ws + apb::kStatusBytes, qb, status, cs,
                        &why);
  if (why) return fail(APB_ERR_CUDA, "score: %s", why);
  if (e != cudaSuccess) return cuda_fail(e, "score kernel");
  if (s.keep > 0) {
    e = fused ? apb::launch_topk_gather(s, sc, idx, k, v, pass_k, pass_v, cs)
              : apb::launch_topk(s, sc, idx, cs);
    if (e != cudaSuccess) return cuda_fail(e, "top-k kernel");
  }
  return APB_OK;
}


}  // namespace

extern "C" {

apb_status apb_score_compress(const apb_config* cfg, const void* q, const void* k,
                              const void* v, const float* w1, const float* b1,
                              const float* w2, const float* b2, float* scores,
                              int32_t* idx, void* workspace, size_t ws_bytes,
                              void* stream) {
  return score_compress_impl("apb_score_compress", false, cfg, q, k, v, w1, b1, w2, b2, scores,
                             idx, nullptr, nullptr, workspace, ws_bytes, stream);
}

apb_status apb_score_compress_pass(const apb_config* cfg, const void* q, const void* k,
                                   const void* v, const float* w1, const float* b1,
                                   const float* w2, const float* b2, float* scores, int32_t* idx,
                                   void* pass_k, void* pass_v, void* workspace, size_t ws_bytes,
                                   void* stream) {
  return score_compress_impl("apb_score_compress_pass", false, cfg, q, k, v, w1, b1, w2, b2,
                             scores, idx, pass_k, pass_v, workspace, ws_bytes, stream);
}

apb_status apb_score_compress_query_aware(const apb_config* cfg, const void* q, const void* k,
                                          const void* v, const float* w1, const float* b1,
                                          const float* w2, const float* b2, float* scores,
                                          int32_t* idx, void* workspace, size_t ws_bytes,
                                          void* stream) {
  return score_compress_impl("apb_score_compress_query_aware", true, cfg, q, k, v, w1, b1, w2, b2,
                             scores, idx, nullptr, nullptr, workspace, ws_bytes, stream);
}

apb_status apb_build_passing(const apb_config* cfg, const void* k, const void* v,
                             const int32_t* idx, void* pass_k, void* pass_v, void* stream) {
  apb::Shape s;
  apb_status st = check_config(cfg, &s);
  if (st != APB_OK) return st;
  if (s.keep == 0) return APB_OK;
  if (!k || !v || !idx || !pass_k || !pass_v)
    return fail(APB_ERR_INVALID_ARG, "apb_build_passing: NULL pointer");
  if (!aligned16(k) || !aligned16(v) || !aligned16(pass_k) || !aligned16(pass_v) || !aligned16(idx))
    return fail(APB_ERR_INVALID_ARG, "apb_build_passing: pointers must be 16-byte aligned");
  cudaError_t e = apb::launch_gather(s, k, v, idx, pass_k, pass_v,
                                     reinterpret_cast<cudaStream_t>(stream));
  if (e != cudaSuccess) return cuda_fail(e, "gather kernel");
  return APB_OK;
}

// Attention of the hosts h0, h0 + stride, ..., h0 + (count - 1) * stride.
// local: rank-local buffers (Q/out hold those hosts' rows in that order; K/V
// the anchor rows, then the hosts' rows); else whole-sequence buffers (then
// stride must be 1).
static apb_status attention_impl(const char* who, const apb_config* cfg, int h0, int count,
                                 int stride, bool local, const void* q, const void* k, const void* v,
                                 const void* pass_k, const void* pass_v, void* out, float* lse,
                                 void* workspace, size_t ws_bytes, void* stream) {
  apb::Shape s;
  apb_status st = check_config(cfg, &s);
  if (st != APB_OK) return st;
  if (h0 < 0 || count < 1 || stride < 1 || (!local && stride != 1) ||
      (long long)h0 + (long long)(count - 1) * stride >= s.H)
    return fail(APB_ERR_INVALID_ARG, "%s: hosts %d + i*%d, i < %d, not inside [0, %d)", who, h0,
                stride, count, s.H);
  const int h_last = h0 + (count - 1) * stride;
  if (!q || !k || !v || !out || !workspace)
    return fail(APB_ERR_INVALID_ARG, "%s: NULL q/k/v/out/workspace", who);
  // hosts h >= 1 read pass rows [0, h*keep)
  const bool need_pass = s.keep > 0 && h_last >= 1;
  if (need_pass && (!pass_k || !pass_v))
    return fail(APB_ERR_INVALID_ARG, "%s: NULL pass_k/pass_v with keep > 0", who);
  if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(out) || !aligned16(workspace) ||
      (need_pass && (!aligned16(pass_k) || !aligned16(pass_v))) || (lse && !aligned16(lse)))
    return fail(APB_ERR_INVALID_ARG, "%s: pointers must be 16-byte aligned", who);
  if (ws_bytes < apb::kStatusBytes)
    return fail(APB_ERR_INVALID_ARG, "%s: workspace %zu < %zu bytes", who, ws_bytes,
                apb::kStatusBytes);
  apb::HostRange r;
  r.h0 = h0;
  r.count = count;
  r.stride = stride;
  if (local) {
    // rank-local buffers: Q/out hold the hosts' rows; K/V hold the anchor rows
    // [0, A) followed by those hosts' rows
    r.q_row0 = 0;
    r.k_row0 = s.A;
    r.anchor_row0 = 0;
    r.q_rows = (long long)count * s.n;
    r.k_rows = s.A + r.q_rows;
  } else {
    r.q_row0 = h0 * s.n;
    r.k_row0 = h0 * s.n;
    r.anchor_row0 = 0;
    r.q_rows = s.N;
    r.k_rows = s.N;
  }
  cudaStream_t cs = reinterpret_cast<cudaStream_t>(stream);
  auto* status = static_cast<apb::DeviceStatus*>(workspace);
  // clear the in-launch abort flag (the sticky bits stay until cleared)
  cudaError_t e = cudaMemsetAsync(&status->abort, 0, sizeof(uint32_t), cs);
  if (e != cudaSuccess) return cuda_fail(e, "clearing abort flag");
  const char* why = nullptr;
  e = apb::launch_attention(s, r, q, k, v, need_pass ? pass_k : nullptr,
                            need_pass ? pass_v : nullptr, out, lse, status, cs, &why);
  if (why) return fail(APB_ERR_CUDA, "attention: %s", why);
  if (e != cudaSuccess) return cuda_fail(e, "attention kernel");
  return APB_OK;
}

apb_status apb_block_attention(const apb_config* cfg, const void* q, const void* k,
                               const void* v, const void* pass_k, const void* pass_v,
                               void* out, float* lse, void* workspace, size_t ws_bytes,
                               void* stream) {
  const int H = cfg ? cfg->n_hosts : 1;
  return attention_impl("apb_block_attention", cfg, 0, H, 1, false, q, k, v, pass_k, pass_v, out,
                        lse, workspace, ws_bytes, stream);
}

apb_status apb_block_attention_hosts(const apb_config* cfg, int32_t host_begin, int32_t host_end,
                                     const void* q, const void* kv_k, const void* kv_v,
                                     const void* pass_k, const void* pass_v, void* out,
                                     float* lse, void* workspace, size_t ws_bytes, void* stream) {
  return attention_impl("apb_block_attention_hosts", cfg, host_begin, host_end - host_begin, 1,
                        true, q, kv_k, kv_v, pass_k, pass_v, out, lse, workspace, ws_bytes,
                        stream);
}

apb_status apb_block_attention_range(const apb_config* cfg, int32_t host_begin, int32_t host_end,
                                     const void* q, const void* k, const void* v,
                                     const void* pass_k, const void* pass_v, void* out,
                                     float* lse, void* workspace, size_t ws_bytes, void* stream) {
  return attention_impl("apb_block_attention_range", cfg, host_begin, host_end - host_begin, 1,
                        false, q, k, v, pass_k, pass_v, out, lse, workspace, ws_bytes, stream);
}

apb_status apb_block_attention_host_set(const apb_config* cfg, int32_t host_first,
                                        int32_t host_count, int32_t host_stride, const void* q,
                                        const void* kv_k, const void* kv_v, const void* pass_k,
                                        const void* pass_v, void* out, float* lse,
                                        void* workspace, size_t ws_bytes, void* stream) {
  return attention_impl("apb_block_attention_host_set", cfg, host_first, host_count, host_stride,
                        true, q, kv_k, kv_v, pass_k, pass_v, out, lse, workspace, ws_bytes,
                        stream);
}

// ---------------------------------------------------------------- one call

// Workspace of apb_prefill: status block, W1 split, query-aware bias slot,
// then scores of hosts 0..H-2, their indices, and the passing K and V blocks
// (H*keep rows each; the last host's rows are never written or read).
struct PrefillLayout {
  size_t wsplit, scores, idx, pass_k, pass_v, total;
};

static PrefillLayout prefill_layout(const apb::Shape& s) {
  PrefillLayout L;
  const size_t h1 = s.H > 1 ? (size_t)(s.H - 1) : 0;
  const size_t pass = round256((size_t)s.H * s.keep * s.Hkv * s.d * 2);
  L.wsplit = apb::kStatusBytes;
  L.scores = L.wsplit + round256(apb::weight_split_bytes(s)) + round256(apb::query_bias_bytes(s));
  L.idx = L.scores + round256(h1 * s.n * s.Hkv * sizeof(float));
  L.pass_k = L.idx + round256(h1 * s.Hkv * s.keep * sizeof(int32_t));
  L.pass_v = L.pass_k + pass;
  L.total = L.pass_v + pass;
  return L;
}

size_t apb_prefill_workspace_bytes(const apb_config* cfg) {
  apb::Shape s;
  if (check_config(cfg, &s) != APB_OK) return 0;
  return prefill_layout(s).total;
}

apb_status apb_prefill(const apb_config* cfg, const void* q, const void* k, const void* v,
                       const float* w1, const float* b1, const float* w2, const float* b2,
                       void* out, float* lse, void* workspace, size_t ws_bytes, void* stream) {
  apb::Shape s;
  apb_status st = check_config(cfg, &s);
  if (st != APB_OK) return st;
  if (!q || !k || !v || !w1 || !b1 || !w2 || !b2 || !out || !workspace)
    return fail(APB_ERR_INVALID_ARG, "apb_prefill: NULL pointer");
  if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(w1) || !aligned16(out) ||
      !aligned16(workspace) || (lse && !aligned16(lse)))
    return fail(APB_ERR_INVALID_ARG, "apb_prefill: pointers must be 16-byte aligned");
  const PrefillLayout L = prefill_layout(s);
  if (ws_bytes < L.total)
    return fail(APB_ERR_INVALID_ARG, "apb_prefill: workspace %zu < %zu bytes", ws_bytes, L.total);
  cudaStream_t cs = reinterpret_cast<cudaStream_t>(stream);
  char* ws = static_cast<char*>(workspace);
  auto* status = reinterpret_cast<apb::DeviceStatus*>(ws);
  cudaError_t e = cudaMemsetAsync(&status->abort, 0, sizeof(uint32_t), cs);
  if (e != cudaSuccess) return cuda_fail(e, "clearing abort flag");
  const bool compress = s.H > 1 && s.keep > 0;
  if (compress) {
    // hosts 0..H-2 only: the last host's compressed block has no successor
    apb::Shape s1 = s;
    s1.H = s.H - 1;
    s1.N = (long long)s1.H * s.n;
    float* scores = reinterpret_cast<float*>(ws + L.scores);
    int32_t* idx = reinterpret_cast<int32_t*>(ws + L.idx);
    const char* why = nullptr;
    e = apb::launch_score(s1, q, k, v, w1, b1, w2, b2, scores, ws + L.wsplit, nullptr, status, cs,
                          &why);
    if (why) return fail(APB_ERR_CUDA, "score: %s", why);
    if (e != cudaSuccess) return cuda_fail(e, "score kernel");
    // selection and the passing-block gather in one launch
    e = apb::launch_topk_gather(s1, scores, idx, k, v, ws + L.pass_k, ws + L.pass_v, cs);
    if (e != cudaSuccess) return cuda_fail(e, "top-k + gather kernel");
  }
  apb::HostRange r{0, s.H, 1, 0, 0, 0, s.N, s.N};
  const char* why = nullptr;
  e = apb::launch_attention(s, r, q, k, v, compress ? ws + L.pass_k : nullptr,
                            compress ? ws + L.pass_v : nullptr, out, lse, status, cs, &why);
  if (why) return fail(APB_ERR_CUDA, "attention: %s", why);
  if (e != cudaSuccess) return cuda_fail(e, "attention kernel");
  return APB_OK;
}

apb_status apb_device_status(void* workspace, void* stream, int clear) {
  if (!workspace) return fail(APB_ERR_INVALID_ARG, "apb_device_status: NULL workspace");
  cudaStream_t cs = reinterpret_cast<cudaStream_t>(stream);
  cudaError_t e = cudaStreamSynchronize(cs);
  if (e != cudaSuccess) return cuda_fail(e, "stream synchronize");
  apb::DeviceStatus h{};
  e = cudaMemcpy(&h, workspace, sizeof(h), cudaMemcpyDeviceToHost);
  if (e != cudaSuccess) return cuda_fail(e, "reading status block");
  if (clear) {
    e = cudaMemset(workspace, 0, sizeof(h));
    if (e != cudaSuccess) return cuda_fail(e, "clearing status block");
  }
  if (h.sticky & apb::kErrWaitTimeout)
    return fail(APB_ERR_TIMEOUT, "a bounded on-chip wait ran out (barrier %u, tile %u)", h.where,
                h.tile);
  return APB_OK;
}

const char* apb_status_string(apb_status status) {
  switch (status) {
    case APB_OK: return "APB_OK";
    case APB_ERR_INVALID_ARG: return "APB_ERR_INVALID_ARG";
    case APB_ERR_UNSUPPORTED: return "APB_ERR_UNSUPPORTED";
    case APB_ERR_CUDA: return "APB_ERR_CUDA";
    case APB_ERR_TIMEOUT: return "APB_ERR_TIMEOUT";
  }
  return "APB_ERR_UNKNOWN";
}

const char* apb_last_error(void) { return g_last_error; }

apb_status apb_selftest_set_wait_limit(uint64_t limit_ns) {
  if (limit_ns != 0 && limit_ns < 100)
    return fail(APB_ERR_INVALID_ARG, "apb_selftest_set_wait_limit: limit_ns=%llu < 100",
                (unsigned long long)limit_ns);
  g_wait_ns.store(limit_ns == 0 ? kDefaultWaitNs : limit_ns, std::memory_order_relaxed);
  return APB_OK;
}

}  // extern "C"

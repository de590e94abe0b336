/*
 * apb.h -- C ABI of the APB per-host prefill path on one B200 (sm_100a).
 *
 * Method: "APB: Accelerating Distributed Long-Context Inference by Passing
 * Compressed Context Blocks across GPUs" (arXiv 2502.12085).  The juejin.cn
 * post on APB, sections "APB 的主要功能" (main features) and "APB 的技术原理"
 * (technical principles), states the steps implemented here:
 *   - the sequence is split evenly into H context blocks (hosts); each host's
 *     block is preceded by an anchor block, the start of the sequence, with
 *     the query embedded at its start;
 *   - each host compresses its KV with retaining heads and keeps the
 *     important KV pairs (apb_score_compress);
 *   - the compressed blocks are all-gathered and each host builds a passing
 *     block from the blocks of the hosts before it (apb_build_passing); on one
 *     GPU the H hosts are virtual and the all-gather is a local gather;
 *   - each host attends over anchor + passing + its local block, and the
 *     passing block is discarded afterwards (apb_block_attention).
 *
 * Conventions for every call:
 *   - All tensor arguments are DEVICE pointers owned by the caller; the
 *     library allocates no device memory and keeps no state between calls
 *     other than a per-process cache of driver entry points.
 *   - Layouts are contiguous and token-major (row-major, last index fastest):
 *       q      [N, Hq,  d]   bf16      (N = n_hosts * block_len)
 *       k, v   [N, Hkv, d]   bf16
 *       out    [N, Hq,  d]   bf16
 *     Every tensor pointer must be 16-byte aligned.
 *   - q head j uses kv head j / (Hq / Hkv) (consecutive grouping).
 *   - Calls are asynchronous on `stream` (a cudaStream_t; NULL = the legacy
 *     default stream) and never synchronise, except apb_device_status.
 *   - Arguments are checked on the host before anything is launched; a bad
 *     argument returns APB_ERR_INVALID_ARG (or APB_ERR_UNSUPPORTED for a
 *     valid but unimplemented shape) and launches nothing.  A failed launch
 *     returns APB_ERR_CUDA.  Nothing aborts or throws across this boundary.
 *   - Kernels that wait on on-chip barriers bound every wait; a wait that
 *     runs out records APB_ERR_TIMEOUT in the workspace status word, the
 *     kernel releases what it holds and returns, and apb_device_status
 *     reports it.
 */
#ifndef APB_H_
#define APB_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
  APB_OK = 0,
  APB_ERR_INVALID_ARG = 1,
  APB_ERR_UNSUPPORTED = 2,
  APB_ERR_CUDA = 3,
  APB_ERR_TIMEOUT = 4
} apb_status;

/* Sizes of one prefill.  Constraints (else APB_ERR_INVALID_ARG):
 *   n_hosts >= 1, block_len >= 1, 0 <= query_len <= anchor_len <= block_len,
 *   0 <= keep <= block_len, n_q_heads % n_kv_heads == 0.
 * head_dim must be 64 or 128 and mlp_hidden 256 (else APB_ERR_UNSUPPORTED).
 * softmax_scale <= 0 selects 1/sqrt(head_dim).  query_len only documents
 * where the query segment sits (rows [0, query_len) of the anchor); no
 * kernel treats those rows differently. */
typedef struct apb_config {
  int32_t n_hosts;      /* H */
  int32_t block_len;    /* n: tokens per host */
  int32_t anchor_len;   /* A: anchor rows [0, A), seen by hosts 1..H-1 */
  int32_t query_len;    /* q_len */
  int32_t keep;         /* top-k per (host, kv head) */
  int32_t n_q_heads;    /* Hq */
  int32_t n_kv_heads;   /* Hkv */
  int32_t head_dim;     /* d */
  int32_t mlp_hidden;   /* retaining-head hidden width */
  float softmax_scale;
} apb_config;

/* Bytes of device workspace that apb_score_compress and apb_block_attention
 * need: a 256-byte status block, then the bf16 hi/lo split of W1
 * (Hkv*hidden*3d*4 bytes, rounded up to 256), then the query-aware bias
 * (Hkv*hidden*4 bytes, rounded up to 256), then Hkv*N*4 bytes (rounded up to
 * 256) for the scores when a score call is given scores == NULL.
 * Returns 0 for a NULL or invalid config.  The caller zero-fills a workspace
 * once before its first use (the status block must start at zero). */
size_t apb_workspace_bytes(const apb_config* cfg);

/* Step 1 (main features: KV compression with retaining heads; technical
 * principles: the compressed block holds the important KV pairs).
 * For every token t and kv head g the retaining-head stand-in computes
 *     x = [k[t,g] ; v[t,g] ; mean_{j: j/G == g} q[t,j]]            (3d)
 *     s[g,t] = w2[g] . SiLU(W1[g] x + b1[g]) + b2[g]
 * in fp32, then keeps, for every host h and kv head g, the `keep` positions
 * of [h*n, h*n+n) with the largest s (ties: the lower position wins).
 *   w1 [Hkv, hidden, 3d], b1 [Hkv, hidden], w2 [Hkv, hidden], b2 [Hkv]: fp32
 *   scores [Hkv, N] fp32 (out, may be NULL: then held in the workspace)
 *   idx [H, Hkv, keep] int32 (out): global positions, ascending per (h, g)
 *   workspace/ws_bytes: apb_workspace_bytes(cfg) bytes, or, when scores is
 *   given, the status block and the weight split only.
 * The products run on the tensor cores in bf16 with fp32 accumulation on
 * split operands: each fp32 weight is split into bf16 hi + lo, and the group
 * mean of q (summed in fp32, then scaled by 1/G) likewise; k and v are exact
 * bf16 and multiply both weight parts, the q mean as hi.hi + hi.lo + lo.hi.
 * The rounding beyond fp32 is about 2^-17 relative per product. */
apb_status apb_score_compress(const apb_config* cfg, const void* q, const void* k,
                              const void* v, const float* w1, const float* b1,
                              const float* w2, const float* b2, float* scores,
                              int32_t* idx, void* workspace, size_t ws_bytes,
                              void* stream);

/* Step 1, query-aware variant (technical principles: the query is embedded
 * at the start of the anchor so the compressor sees it and keeps the KV pairs
 * that matter for it).  Same arguments, outputs and selection rule as
 * apb_score_compress, but the q part of the MLP input is, for every token,
 * the mean of q over the query segment (rows [0, query_len)) and the group's
 * q heads (zero when query_len == 0):
 *     x = [k[t,g] ; v[t,g] ; mean_{r < q_len, j: j/G == g} q[r,j]]
 * That part is constant per kv head, so it is folded exactly into the first
 * layer's bias (fp32) and the product runs over the k and v sections only;
 * Q rows beyond the query segment are not read.  The workspace additionally
 * holds that bias (Hkv*hidden*4 bytes): apb_workspace_bytes(cfg) bytes, or,
 * when scores is given, the status block, the weight split and the bias. */
apb_status apb_score_compress_query_aware(const apb_config* cfg, const void* q, const void* k,
                                          const void* v, const float* w1, const float* b1,
                                          const float* w2, const float* b2, float* scores,
                                          int32_t* idx, void* workspace, size_t ws_bytes,
                                          void* stream);

/* Step 2 (main features: communication; the all-gather of compressed blocks
 * and the passing block built from the preceding hosts' blocks).
 *   pass_k[h*keep + r, g, :] = k[idx[h, g, r], g, :]   (and likewise v)
 *   pass_k, pass_v [H*keep, Hkv, d] bf16 (out, token-major like k and v),
 *   copied bit-exactly.
 * Host h's passing block is rows [0, h*keep) of this layout, and the blocks
 * of hosts [a, b) are the contiguous rows [a*keep, b*keep): what one
 * all-gather exchanges when hosts live on different GPUs.  idx may hold
 * positions relative to the k/v pointers given (e.g. one host's block).  An
 * index outside [0, N) yields a zero row instead of a read. */
apb_status apb_build_passing(const apb_config* cfg, const void* k, const void* v,
                             const int32_t* idx, void* pass_k, void* pass_v,
                             void* stream);

/* Steps 1 and 2 with the passing block emitted straight from the selection
 * (the fusion of selection and gather): the same scores, idx and selection
 * rule as apb_score_compress, and pass_k / pass_v exactly as
 * apb_build_passing writes them, in two launches (score; top-k + gather).
 *   pass_k, pass_v [H*keep, Hkv, d] bf16 (out), 16-byte aligned; both NULL
 *   only when keep == 0.
 * Other arguments and the workspace as for apb_score_compress. */
apb_status apb_score_compress_pass(const apb_config* cfg, const void* q, const void* k,
                                   const void* v, const float* w1, const float* b1,
                                   const float* w2, const float* b2, float* scores, int32_t* idx,
                                   void* pass_k, void* pass_v, void* workspace, size_t ws_bytes,
                                   void* stream);

/* Step 3 (main features: computation over anchor, passing and local block;
 * the passing block is not kept afterwards).  For host h, local row i
 * (t = h*n + i) and q head j (g = j / G):
 *     keys = k[0:A, g] (only if h >= 1) ++ pass_k[g, 0:h*keep]
 *            ++ k[h*n : t+1, g]
 *     out[t, j] = softmax(q[t, j] . keys^T * scale) @ values
 * bf16 tensor-core products, fp32 accumulation and online softmax.
 *   out [N, Hq, d] bf16 (out); lse [Hq, N] fp32 natural log-sum-exp of the
 *   scaled logits (out, may be NULL).
 *   workspace/ws_bytes: at least 256 bytes (status block). */
apb_status apb_block_attention(const apb_config* cfg, const void* q, const void* k,
                               const void* v, const void* pass_k, const void* pass_v,
                               void* out, float* lse, void* workspace, size_t ws_bytes,
                               void* stream);

/* Step 3 for the hosts [host_begin, host_end) only, on the whole-sequence
 * buffers of apb_block_attention (q, k, v, out [N, ...]; lse [Hq, N]): the
 * rows of those hosts in out (and lse) are written, nothing else.  Lets a
 * caller attend host h as soon as its own rows and the compressed blocks of
 * hosts 0..h-1 are in place (main features: each host attends over the
 * anchor, the passing block of the hosts before it and its own block), e.g.
 * while later hosts' inputs are still being copied in.
 * 0 <= host_begin < host_end <= n_hosts, else APB_ERR_INVALID_ARG. */
apb_status apb_block_attention_range(const apb_config* cfg, int32_t host_begin, int32_t host_end,
                                     const void* q, const void* k, const void* v,
                                     const void* pass_k, const void* pass_v, void* out,
                                     float* lse, void* workspace, size_t ws_bytes, void* stream);

/* Step 3 for a range of hosts on rank-local buffers (main features: the
 * sequence is split over hosts, each host's context block is preceded by the
 * anchor block, and the passing block is built from the all-gathered
 * compressed blocks).  Computes exactly what apb_block_attention computes
 * for hosts [host_begin, host_end), with buffers that hold only what those
 * hosts need:
 *   q, out  [(host_end-host_begin)*n, Hq, d]: the hosts' rows, in host order;
 *   kv_k, kv_v [A + (host_end-host_begin)*n, Hkv, d]: the anchor's A rows
 *           (the start of the sequence, which every host prepends to its
 *           block), then the hosts' rows;
 *   pass_k, pass_v [H*keep, Hkv, d]: all hosts' compressed blocks in host
 *           order (rows [0, (host_end-1)*keep) are read);
 *   lse [Hq, (host_end-host_begin)*n] (may be NULL).
 * 0 <= host_begin < host_end <= n_hosts, else APB_ERR_INVALID_ARG. */
apb_status apb_block_attention_hosts(const apb_config* cfg, int32_t host_begin, int32_t host_end,
                                     const void* q, const void* kv_k, const void* kv_v,
                                     const void* pass_k, const void* pass_v, void* out,
                                     float* lse, void* workspace, size_t ws_bytes, void* stream);

/* Step 3 for an evenly spaced set of hosts on rank-local buffers: the hosts
 * host_first + i*host_stride, i < host_count (main features: hosts are spread
 * over devices; a round-robin assignment, rank r of W owning hosts r, r+W,
 * ..., balances the work, which grows with the host index because each host
 * attends to the compressed blocks of all hosts before it).  Same
 * computation and buffer conventions as apb_block_attention_hosts, with the
 * set's hosts in increasing order in place of a contiguous range:
 *   q, out  [host_count*n, Hq, d]; kv_k, kv_v [A + host_count*n, Hkv, d]
 *   (anchor rows, then the hosts' rows); pass_k, pass_v [H*keep, Hkv, d] in
 *   host order (rows [0, h_last*keep) are read); lse [Hq, host_count*n].
 * host_first >= 0, host_count >= 1, host_stride >= 1 and
 * host_first + (host_count-1)*host_stride < n_hosts, else
 * APB_ERR_INVALID_ARG.  apb_block_attention_hosts(b, e) is this call with
 * (b, e - b, 1). */
apb_status apb_block_attention_host_set(const apb_config* cfg, int32_t host_first,
                                        int32_t host_count, int32_t host_stride, const void* q,
                                        const void* kv_k, const void* kv_v, const void* pass_k,
                                        const void* pass_v, void* out, float* lse,
                                        void* workspace, size_t ws_bytes, void* stream);

/* The whole path in one call: steps 1-3 on one GPU for all hosts, writing
 * out [N, Hq, d] (and lse [Hq, N] when not NULL).  The last host's
 * compressed block is not computed: no host follows it, so no passing block
 * contains it (main features: each passing block holds the preceding hosts'
 * blocks); out and lse equal those of apb_score_compress + apb_build_passing
 * + apb_block_attention.  workspace: apb_prefill_workspace_bytes(cfg) bytes,
 * zero-filled before first use; it holds the scores, indices and passing
 * blocks between the steps. */
size_t apb_prefill_workspace_bytes(const apb_config* cfg);
apb_status apb_prefill(const apb_config* cfg, const void* q, const void* k, const void* v,
                       const float* w1, const float* b1, const float* w2, const float* b2,
                       void* out, float* lse, void* workspace, size_t ws_bytes, void* stream);

/* No counterpart in the paper: an allocation-free variant of
 * apb_score_compress, for callers that cannot hand this library any device
 * memory besides the tensors themselves (a host framework whose allocator
 * owns all device memory and only exposes inputs and outputs to plug-ins, or
 * a service that must not allocate after start-up).  Same computation,
 * arguments and outputs as apb_score_compress with scores == NULL, but the
 * fp32 scores and the weight split live in fixed device arrays inside the
 * library instead of a workspace; nothing is allocated by the call.
 *   - The arrays hold apb_score_compress_static_max_floats() floats (16 MiB)
 *     of scores and 8 MiB of split weights; every GPU that loads the library
 *     keeps them until the process exits.  n_kv_heads * N above the first,
 *     or n_kv_heads * mlp_hidden * 3 * head_dim * 4 bytes above the second,
 *     returns APB_ERR_UNSUPPORTED with the exceeded limit in
 *     apb_last_error().  A bounded wait that runs out inside this variant is
 *     recorded in the library's own status block, which
 *     apb_score_compress_static_status reads.
 *   - Every call looks up the arrays' device addresses on the current device
 *     (cudaGetSymbolAddress, a host-side lookup), so the call works on
 *     whichever device is current and after cudaDeviceReset; the first call
 *     on a device should still come before any stream capture (it may load
 *     the module on that device).
 *   - All calls share the arrays and they keep the last call's contents.
 *     Each call writes every score it reads, so nothing needs clearing, but
 *     two calls whose kernels overlap on the GPU (other streams or threads)
 *     race on it: serialise them. */
size_t apb_score_compress_static_max_floats(void);
apb_status apb_score_compress_static(const apb_config* cfg, const void* q, const void* k,
                                     const void* v, const float* w1, const float* b1,
                                     const float* w2, const float* b2, int32_t* idx,
                                     void* stream);

/* No counterpart in the paper.  apb_device_status for the fixed status block
 * of apb_score_compress_static on the current device: synchronises `stream`,
 * returns APB_ERR_TIMEOUT if one of its kernels recorded a bounded wait that
 * ran out since the block was last cleared (the top-k that followed then
 * read incomplete scores: discard idx), else APB_OK.  clear != 0 resets the
 * block afterwards. */
apb_status apb_score_compress_static_status(void* stream, int clear);

/* No counterpart in the paper: apb_selftest_wait_timeout run on the fixed
 * status block of apb_score_compress_static (current device), so that a
 * caller can check that apb_score_compress_static_status reports a wait that
 * ran out.  limit_us in [1, 1000000]. */
apb_status apb_score_compress_static_selftest(uint32_t limit_us, void* stream);

/* No counterpart in the paper: a self-test of the bounded waits every kernel
 * uses.  Launches two CTAs that each wait on an on-chip barrier that nothing
 * completes: CTA 0 with a limit of limit_us microseconds (1..1000000), CTA 1
 * with a limit 20 times longer plus 1 s.  CTA 0's wait runs out and records
 * APB_ERR_TIMEOUT in the status block of `workspace` (>= 256 bytes, zeroed
 * before first use); CTA 1 leaves its wait through the launch-wide abort
 * flag.  Bytes 64..79 of the block receive the two waits' elapsed
 * nanoseconds.  apb_device_status then reports APB_ERR_TIMEOUT.  Nothing
 * faults, traps or hangs. */
apb_status apb_selftest_wait_timeout(void* workspace, size_t ws_bytes, uint32_t limit_us,
                                     void* stream);

/* No counterpart in the paper: failure-path self-test.  Sets the time limit
 * of the bounded on-chip waits of every kernel launched afterwards by this
 * process (default 1 s; limit_ns = 0 restores it; otherwise limit_ns must be
 * >= 100).  A wait gives up only after its barrier has failed 32 or more
 * polls and the limit has passed, so a short limit makes the waits that
 * really block (on the tensor core, the copies, the other warps) run out
 * mid-run: every kernel must still finish (each CTA drains its copies and
 * MMAs and meets its partner warps at every remaining named barrier) and
 * apb_device_status then reports APB_ERR_TIMEOUT; the outputs of such a call
 * are undefined.  Process-wide, not thread-safe against concurrent launches;
 * meant for tests.  Nothing faults, traps or hangs. */
apb_status apb_selftest_set_wait_limit(uint64_t limit_ns);

/* Synchronises `stream`, then reads the status block of `workspace`:
 * APB_ERR_TIMEOUT if a kernel recorded a bounded wait that ran out since the
 * block was last cleared, else APB_OK (APB_ERR_CUDA if the reads fail).
 * clear != 0 resets the block to zero afterwards. */
apb_status apb_device_status(void* workspace, void* stream, int clear);

/* Static, NUL-terminated name of a status code. */
const char* apb_status_string(apb_status status);

/* Human-readable detail of the last failure returned on the calling thread
 * (static storage, valid until the next call on that thread). */
const char* apb_last_error(void);

#ifdef __cplusplus
}
#endif

#endif /* APB_H_ */

// apb_score_compress_static: the score + top-k step for callers that cannot
// give this library any device memory besides the tensors themselves -- for
// example a host framework whose allocator owns all device memory and only
// exposes input and output buffers to plug-ins, or a service that must not
// allocate once it has started.  The fp32 scores that apb_score_compress
// keeps in the caller's workspace live here in a fixed, file-scope device
// array instead, so the call needs no workspace and allocates nothing.
//
// The arrays hold kStaticScoreFloats floats (16 MiB) for the scores and
// kStaticWsBytes bytes (8 MiB + 256) for the status block and the bf16 split of
// W1.  Every GPU that loads this library reserves them until the process exits.
#include "apb_internal.h"

namespace {

constexpr size_t kStaticScoreFloats = size_t(4) << 20;   // Hkv * N <= 4,194,304
constexpr size_t kStaticWsBytes = 256 + (size_t(8) << 20);   // status + W1 split

static __device__ __align__(256) float g_score_scratch[kStaticScoreFloats];
static __device__ __align__(256) unsigned char g_ws_scratch[kStaticWsBytes];

// Device addresses of the two arrays on the current device.  In host code a
// __device__ symbol is only a host-side handle, so the addresses come from
// cudaGetSymbolAddress with the device current.  The lookup is a cheap host
// call and is made on every call, so that an address never outlives the
// context it belongs to (cudaDeviceReset, or a primary context torn down and
// created again, loads the module anew and may move the arrays).
apb_status scratch_address(const char* who, float** out, void** ws) {
  void* p = nullptr;
  void* w = nullptr;
  cudaError_t e = cudaGetSymbolAddress(&p, g_score_scratch);
  if (e != cudaSuccess) return apb::cuda_fail(e, who);
  e = cudaGetSymbolAddress(&w, g_ws_scratch);
  if (e != cudaSuccess) return apb::cuda_fail(e, who);
  *out = static_cast<float*>(p);
  *ws = w;
  return APB_OK;
}

}  // namespace

extern "C" {
size_t apb_score_compress_static_max_floats(void) { return kStaticScoreFloats; }

apb_status apb_score_compress_static(const apb_config* cfg, const void* q, const void* k,
                                     const void* v, const float* w1, const float* b1,
                                     const float* w2, const float* b2, int32_t* idx,
                                     void* stream) {
  // An invalid config: let apb_score_compress report it (it fails on the
  // config before looking at any pointer).
  if (apb_workspace_bytes(cfg) == 0)
    return apb_score_compress(cfg, q, k, v, w1, b1, w2, b2, nullptr, idx, nullptr, 0, stream);
  const size_t need = (size_t)cfg->n_kv_heads * (size_t)cfg->n_hosts * (size_t)cfg->block_len;
  const size_t split = (size_t)cfg->n_kv_heads * 2 * cfg->mlp_hidden * 3 * cfg->head_dim * 2;
  const size_t split_room = kStaticWsBytes - 256;
  if (need > kStaticScoreFloats)
    return apb::fail(APB_ERR_UNSUPPORTED,
                     "apb_score_compress_static: n_kv_heads*N = %zu scores > %zu (fixed array)",
                     need, kStaticScoreFloats);
  if (((split + 255) & ~size_t(255)) > split_room)
    return apb::fail(APB_ERR_UNSUPPORTED,
                     "apb_score_compress_static: W1 split %zu B > %zu B (fixed array)", split,
                     split_room);
  if (!q || !k || !v || !w1 || !b1 || !w2 || !b2 || (cfg->keep > 0 && !idx))
    return apb::fail(APB_ERR_INVALID_ARG, "apb_score_compress_static: NULL input or idx");
  float* scratch = nullptr;
  void* ws = nullptr;
  const apb_status st = scratch_address("apb_score_compress_static: cudaGetSymbolAddress",
                                        &scratch, &ws);
  if (st != APB_OK) return st;
  // The arrays take the place of the caller's scores buffer and workspace.
  // Every score and weight the kernels read is written by this same call
  // first; the status block starts at zero (static storage) and its abort
  // flag is cleared by every call, so nothing else needs clearing.  A bounded
  // wait that runs out is recorded in this private status block and reported
  // by apb_score_compress_static_status.
  return apb_score_compress(cfg, q, k, v, w1, b1, w2, b2, scratch, idx, ws, kStaticWsBytes,
                            stream);
}

apb_status apb_score_compress_static_status(void* stream, int clear) {
  float* scratch = nullptr;
  void* ws = nullptr;
  const apb_status st = scratch_address("apb_score_compress_static_status: cudaGetSymbolAddress",
                                        &scratch, &ws);
  if (st != APB_OK) return st;
  // the same synchronise / read / clear as for a caller's workspace
  return apb_device_status(ws, stream, clear);
}

apb_status apb_score_compress_static_selftest(uint32_t limit_us, void* stream) {
  if (limit_us == 0 || limit_us > 1000000)
    return apb::fail(APB_ERR_INVALID_ARG,
                     "apb_score_compress_static_selftest: limit_us=%u not in [1, 1e6]", limit_us);
  float* scratch = nullptr;
  void* ws = nullptr;
  const apb_status st = scratch_address(
      "apb_score_compress_static_selftest: cudaGetSymbolAddress", &scratch, &ws);
  if (st != APB_OK) return st;
  auto* status = static_cast<apb::DeviceStatus*>(ws);
  auto* elapsed = reinterpret_cast<unsigned long long*>(static_cast<char*>(ws) + 64);
  const cudaError_t e =
      apb::launch_wait_selftest(status, limit_us, elapsed, reinterpret_cast<cudaStream_t>(stream));
  return e == cudaSuccess ? APB_OK : apb::cuda_fail(e, "self-test kernel");
}

}  // extern "C"

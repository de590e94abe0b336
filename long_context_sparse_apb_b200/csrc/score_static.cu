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
#include <mutex>

#include "apb_internal.h"

namespace {

constexpr size_t kStaticScoreFloats = size_t(4) << 20;   // Hkv * N <= 4,194,304
constexpr size_t kStaticWsBytes = 256 + (size_t(8) << 20);   // status + W1 split
constexpr int kMaxDevices = 64;

static __device__ __align__(256) float g_score_scratch[kStaticScoreFloats];
static __device__ __align__(256) unsigned char g_ws_scratch[kStaticWsBytes];

std::mutex g_mutex;
float* g_scratch_ptr[kMaxDevices] = {};
void* g_ws_ptr[kMaxDevices] = {};

// Device addresses of the two arrays on the current device.  In host code a
// __device__ symbol is only a host-side handle, so the addresses must come
// from cudaGetSymbolAddress, once per device, with that device current.
cudaError_t scratch_address(float** out, void** ws) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  if (dev < 0 || dev >= kMaxDevices) return cudaErrorInvalidDevice;
  std::lock_guard<std::mutex> lock(g_mutex);
  if (!g_scratch_ptr[dev]) {
    void* p = nullptr;
    void* w = nullptr;
    e = cudaGetSymbolAddress(&p, g_score_scratch);
    if (e != cudaSuccess) return e;
    e = cudaGetSymbolAddress(&w, g_ws_scratch);
    if (e != cudaSuccess) return e;
    g_scratch_ptr[dev] = static_cast<float*>(p);
    g_ws_ptr[dev] = w;
  }
  *out = g_scratch_ptr[dev];
  *ws = g_ws_ptr[dev];
  return cudaSuccess;
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
  if (need > kStaticScoreFloats || 256 + ((split + 255) & ~size_t(255)) > kStaticWsBytes)
    return APB_ERR_UNSUPPORTED;
  if (!q || !k || !v || !w1 || !b1 || !w2 || !b2 || (cfg->keep > 0 && !idx))
    return APB_ERR_INVALID_ARG;
  float* scratch = nullptr;
  void* ws = nullptr;
  if (scratch_address(&scratch, &ws) != cudaSuccess) return APB_ERR_CUDA;
  // The arrays take the place of the caller's scores buffer and workspace.
  // Every score and weight the kernels read is written by this same call
  // first; the status block starts at zero (static storage) and its abort
  // flag is cleared by every call, so nothing else needs clearing.  A bounded
  // wait that runs out is recorded in this private status block, which no
  // call reports.
  return apb_score_compress(cfg, q, k, v, w1, b1, w2, b2, scratch, idx, ws, kStaticWsBytes,
                            stream);
}

}  // extern "C"

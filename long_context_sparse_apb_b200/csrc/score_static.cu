// apb_score_compress_static: the score + top-k step for callers that cannot
// give this library any device memory besides the tensors themselves -- for
// example a host framework whose allocator owns all device memory and only
// exposes input and output buffers to plug-ins, or a service that must not
// allocate once it has started.  The fp32 scores that apb_score_compress
// keeps in the caller's workspace live here in a fixed, file-scope device
// array instead, so the call needs no workspace and allocates nothing.
//
// The array holds kStaticScoreFloats floats (16 MiB).  Every GPU that loads
// this library reserves it until the process exits.
#include <mutex>

#include "apb_internal.h"

namespace {

constexpr size_t kStaticScoreFloats = size_t(4) << 20;   // Hkv * N <= 4,194,304
constexpr int kMaxDevices = 64;

static __device__ __align__(256) float g_score_scratch[kStaticScoreFloats];

std::mutex g_mutex;
float* g_scratch_ptr[kMaxDevices] = {};

// Device address of g_score_scratch on the current device.  In host code the
// symbol is only a host-side handle, so the address must come from
// cudaGetSymbolAddress, once per device, with that device current.
cudaError_t scratch_address(float** out) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  if (dev < 0 || dev >= kMaxDevices) return cudaErrorInvalidDevice;
  std::lock_guard<std::mutex> lock(g_mutex);
  if (!g_scratch_ptr[dev]) {
    void* p = nullptr;
    e = cudaGetSymbolAddress(&p, g_score_scratch);
    if (e != cudaSuccess) return e;
    g_scratch_ptr[dev] = static_cast<float*>(p);
  }
  *out = g_scratch_ptr[dev];
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
  if (need > kStaticScoreFloats) return APB_ERR_UNSUPPORTED;
  if (!q || !k || !v || !w1 || !b1 || !w2 || !b2 || (cfg->keep > 0 && !idx))
    return APB_ERR_INVALID_ARG;
  float* scratch = nullptr;
  if (scratch_address(&scratch) != cudaSuccess) return APB_ERR_CUDA;
  // The scratch takes the place of the caller-owned scores buffer: every
  // score the top-k reads is written by this same call first, so nothing in
  // it needs clearing.  With a scores buffer given, apb_score_compress never
  // touches its workspace argument; the scratch address fills that slot.
  return apb_score_compress(cfg, q, k, v, w1, b1, w2, b2, scratch, idx, scratch,
                            apb::kStatusBytes, stream);
}

}  // extern "C"

// Allocation-free forward entry point (relpos_attn_fwd_noalloc).
//
// Some callers cannot call cudaMalloc: a plugin running inside a host framework
// that owns the whole device-memory budget (its own pool would be bypassed, and
// an allocation can fail or fragment the pool), or a latency-critical loop where
// cudaMalloc / cudaFree would synchronise the device.  For them the forward
// pass takes its scratch (T5 per-offset bias vectors, Transformer-XL u.k and v.r,
// DeBERTa end-row products) from one statically sized device array compiled into
// this library instead of a caller-provided workspace.
//
// Properties of that array:
//   * RELPOS_NOALLOC_SCRATCH_BYTES (16 MiB) per GPU, held by every GPU that loads
//     the library until the process exits;
//   * shared by every call: calls that overlap on the GPU (different streams, no
//     ordering between them) race on it and must not be issued;
//   * it keeps the previous call's contents; the forward pass writes every scratch
//     value it reads before reading it, so nothing needs clearing;
//   * its device address is looked up once per device (cudaGetSymbolAddress, with
//     that device current) on the first call made on the device; make that first
//     call before any stream capture.
#include <cuda_runtime.h>

#include <mutex>

#include "relpos_attn.h"

namespace {

constexpr size_t kScratchBytes = RELPOS_NOALLOC_SCRATCH_BYTES;
constexpr int kMaxDevices = 64;

static __device__ __align__(256) unsigned char g_scratch[kScratchBytes];

std::mutex g_mutex;
void *g_scratch_ptr[kMaxDevices];  // device address of g_scratch, per device ordinal

// Device address of the scratch array on the current device (looked up once).
int scratch_address(void **out) {
  int dev = -1;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) {
    cudaGetLastError();
    return RELPOS_ERR_CUDA;
  }
  std::lock_guard<std::mutex> lock(g_mutex);
  if (!g_scratch_ptr[dev]) {
    void *p = nullptr;
    if (cudaGetSymbolAddress(&p, g_scratch) != cudaSuccess || !p) {
      cudaGetLastError();
      return RELPOS_ERR_CUDA;
    }
    g_scratch_ptr[dev] = p;
  }
  *out = g_scratch_ptr[dev];
  return RELPOS_OK;
}

}  // namespace

extern "C" int relpos_attn_fwd_noalloc(const relpos_params_t *params, const void *q, const void *k, const void *v,
                                       const void *const rel[3], void *o, float *lse, int32_t *dev_status,
                                       void *stream) {
  size_t need = 0;
  int e = relpos_attn_workspace_size(params, 0, &need);
  if (e) return e;
  if (need > kScratchBytes) return RELPOS_ERR_WORKSPACE;  // larger than the built-in scratch
  void *scratch = nullptr;
  if (need > 0 && (e = scratch_address(&scratch)) != RELPOS_OK) return e;
  return relpos_attn_fwd(params, q, k, v, rel, o, lse, need ? scratch : nullptr, need ? kScratchBytes : 0, dev_status,
                         stream);
}

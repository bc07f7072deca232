// noalloc.cu -- kdv_verify_attn with a scratch buffer built into the library.
//
// Some callers cannot hand the library a workspace: a serving engine that
// reserved all free device memory for its KV-cache pool when it started, a
// plug-in whose host framework owns every device allocation, or a latency-
// critical loop where an allocation on the call path is not acceptable. For
// them kdv_verify_attn_noalloc keeps the split partials in a fixed array of
// this file instead of caller memory, and allocates nothing itself.
#include <cuda_runtime.h>

#include "kdv.h"

namespace {

// Device-resident scratch for the split partials; every GPU that loads the
// library holds one copy until the process exits. Host code must not pass
// the name of this array to a kernel: on the host it is only a stand-in
// symbol, so its device address is looked up once per device below.
static __device__ __align__(256) unsigned char kdv_noalloc_scratch[KDV_NOALLOC_SCRATCH_BYTES];

constexpr int kMaxDevices = 64;
void* g_scratch_ptr[kMaxDevices] = {};

// Device address of the scratch array on the current device, looked up on
// the first call per device and cached for the life of the process (a
// cudaDeviceReset of the device would leave the cached address stale; the
// header says so). Concurrent first calls from several host threads all
// store the same value.
kdv_status scratch_for_current_device(void** out) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) {
    cudaGetLastError();
    return KDV_ERR_CUDA;
  }
  if (dev < 0 || dev >= kMaxDevices) return KDV_ERR_UNSUPPORTED;
  if (g_scratch_ptr[dev] == nullptr) {
    void* ptr = nullptr;
    if (cudaGetSymbolAddress(&ptr, kdv_noalloc_scratch) != cudaSuccess || ptr == nullptr) {
      cudaGetLastError();
      return KDV_ERR_CUDA;
    }
    g_scratch_ptr[dev] = ptr;
  }
  *out = g_scratch_ptr[dev];
  return KDV_OK;
}

}  // namespace

extern "C" {

kdv_status kdv_verify_attn_noalloc(const kdv_verify_params* p, void* stream) {
  if (p == nullptr) return KDV_ERR_INVALID_ARG;
  size_t need = 0;
  kdv_status st = kdv_verify_attn_workspace(p, &need);
  if (st != KDV_OK) return st;
  if (need > (size_t)KDV_NOALLOC_SCRATCH_BYTES) return KDV_ERR_WORKSPACE;
  void* scratch = nullptr;
  st = scratch_for_current_device(&scratch);
  if (st != KDV_OK) return st;
  kdv_verify_params q = *p;
  q.workspace = scratch;
  q.workspace_bytes = (size_t)KDV_NOALLOC_SCRATCH_BYTES;
  return kdv_verify_attn(&q, stream);
}

}  // extern "C"

// mask_build.cu -- parent[] to ancestor bitmask.
//
// The tree visibility mask of page "The Architecture of Diagnosis", section
// "Phase 1: Custom CUDA Kernels", item 2: node i sees itself and each of its
// ancestors, so bit u of mask[i] is set iff u is on the path from i to its
// root. One thread per node walks parent[] upwards (at most T steps, T <= 64);
// the work is a few hundred integer operations per tree, far below a
// microsecond, so one CTA of 64 threads per request is plenty.
#include "kdv_internal.cuh"

namespace kdv {
namespace {

__global__ void __launch_bounds__(KDV_MAX_TREE)
mask_build_kernel(const int32_t* __restrict__ parent, const int32_t* __restrict__ tree_off,
                  int32_t max_T, uint64_t* __restrict__ mask, int32_t* __restrict__ depth,
                  int32_t* d_err) {
  const int b = blockIdx.x;
  const int i = threadIdx.x;
  int32_t base = 0, T = max_T;
  if (tree_off != nullptr) {
    base = tree_off[b];
    T = tree_off[b + 1] - base;
    if (T < 0 || T > max_T) {
      if (i == 0) record_error(d_err, KDV_DERR_BAD_PARENT);
      return;
    }
  }
  if (i >= T) return;
  uint64_t m = 0;
  int32_t d = 0;
  bool ok = true;
  int32_t u = i;
  // walk to the root; every step must go to a strictly smaller index
  for (int step = 0; step <= KDV_MAX_TREE; ++step) {
    m |= (uint64_t)1 << u;
    const int32_t p = parent[base + u];
    if (p == -1) break;
    if (p < 0 || p >= u) { ok = false; break; }
    u = p;
    ++d;
  }
  if (!ok) {
    record_error(d_err, KDV_DERR_BAD_PARENT);
    m = 0;
    d = -1;
  }
  mask[base + i] = m;
  if (depth != nullptr) depth[base + i] = d;
}

}  // namespace

cudaError_t launch_mask_build(const int32_t* parent, const int32_t* tree_off, int32_t batch,
                              int32_t max_T, uint64_t* mask, int32_t* depth, int32_t* d_err,
                              cudaStream_t stream) {
  mask_build_kernel<<<batch, KDV_MAX_TREE, 0, stream>>>(parent, tree_off, max_T, mask, depth,
                                                        d_err);
  return cudaGetLastError();
}

}  // namespace kdv

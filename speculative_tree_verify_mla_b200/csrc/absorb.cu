// absorb.cu -- the projections on either side of absorbed-form attention.
//
// Absorbing the latent projection into the attention (page "The Architecture
// of Diagnosis", section "Phase 1: Custom CUDA Kernels", item 2) moves two
// small per-head products out of the attention kernel:
//   q_lat[t,h] = W_UK[h] q_nope[t,h]        (W_UK[h]: D_c x D_n, row-major)
//   out[t,h]   = W_UV[h]^T o_lat[t,h]       (W_UV[h]: D_c x D_v, row-major)
// Rows are node-major (row = t*H + h), so head h owns rows h, H+h, 2H+h, ...
// Both read every weight once per call (2 x 8.4 MB in bf16 for the Kimi shape)
// and do ~2*T flops per weight, so they are HBM-bound; the arithmetic is
// fp32 on CUDA cores. One CTA handles one head and a block of 128 output
// columns; each thread owns one output column for up to 32 rows at a time,
// with the head's input rows staged in shared memory.
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include "kdv.h"

namespace kdv {
namespace {

constexpr int THREADS = 128;
constexpr int RCH = 32;              // rows per pass (accumulators per thread)

__device__ __forceinline__ float ld_elem(const void* p, int64_t i, int dtype) {
  return dtype == KDV_BF16 ? __bfloat162float(static_cast<const __nv_bfloat16*>(p)[i])
                           : static_cast<const float*>(p)[i];
}
__device__ __forceinline__ void st_elem(void* p, int64_t i, int dtype, float v) {
  if (dtype == KDV_BF16) static_cast<__nv_bfloat16*>(p)[i] = __float2bfloat16_rn(v);
  else static_cast<float*>(p)[i] = v;
}

// q_lat[row][d] = sum_k W_UK[h][d][k] q_nope[row][k], one column d per thread.
__global__ void __launch_bounds__(THREADS)
absorb_q_kernel(int32_t rows_per_head, int32_t H, int32_t D_c, int32_t D_n, const void* __restrict__ q_nope,
                int64_t q_stride, int q_dtype, const void* __restrict__ w_uk, int w_dtype, void* __restrict__ q_lat,
                int64_t o_stride, int o_dtype) {
  extern __shared__ float s_q[];     // [RCH][D_n]
  const int h = blockIdx.x;
  const int d = blockIdx.y * THREADS + threadIdx.x;
  const int64_t wrow = ((int64_t)h * D_c + (d < D_c ? d : 0)) * D_n;
  for (int r0 = 0; r0 < rows_per_head; r0 += RCH) {
    const int nr = min(RCH, rows_per_head - r0);
    __syncthreads();
    for (int i = threadIdx.x; i < nr * D_n; i += THREADS) {
      const int r = i / D_n, k = i - r * D_n;
      s_q[i] = ld_elem(q_nope, (int64_t)((r0 + r) * H + h) * q_stride + k, q_dtype);
    }
    __syncthreads();
    if (d < D_c) {
      float acc[RCH];
#pragma unroll
      for (int r = 0; r < RCH; ++r) acc[r] = 0.f;
      for (int k = 0; k < D_n; ++k) {
        const float w = ld_elem(w_uk, wrow + k, w_dtype);
#pragma unroll
        for (int r = 0; r < RCH; ++r)
          if (r < nr) acc[r] = fmaf(w, s_q[r * D_n + k], acc[r]);
      }
#pragma unroll
      for (int r = 0; r < RCH; ++r)
        if (r < nr) st_elem(q_lat, (int64_t)((r0 + r) * H + h) * o_stride + d, o_dtype, acc[r]);
    }
  }
}

// out[row][v] = sum_d W_UV[h][d][v] o_lat[row][d], one column v per thread
// (a warp reads 32 consecutive v of each weight row: coalesced).
__global__ void __launch_bounds__(THREADS)
unabsorb_o_kernel(int32_t rows_per_head, int32_t H, int32_t D_c, int32_t D_v, const float* __restrict__ o_lat,
                  int64_t i_stride, const void* __restrict__ w_uv, int w_dtype, void* __restrict__ out,
                  int64_t o_stride, int o_dtype) {
  extern __shared__ float s_o[];     // [RCH][D_c]
  const int h = blockIdx.x;
  const int v = blockIdx.y * THREADS + threadIdx.x;
  const int64_t wbase = (int64_t)h * D_c * D_v + (v < D_v ? v : 0);
  for (int r0 = 0; r0 < rows_per_head; r0 += RCH) {
    const int nr = min(RCH, rows_per_head - r0);
    __syncthreads();
    for (int i = threadIdx.x; i < nr * D_c; i += THREADS) {
      const int r = i / D_c, k = i - r * D_c;
      s_o[i] = o_lat[(int64_t)((r0 + r) * H + h) * i_stride + k];
    }
    __syncthreads();
    if (v < D_v) {
      float acc[RCH];
#pragma unroll
      for (int r = 0; r < RCH; ++r) acc[r] = 0.f;
      for (int dd = 0; dd < D_c; ++dd) {
        const float w = ld_elem(w_uv, wbase + (int64_t)dd * D_v, w_dtype);
#pragma unroll
        for (int r = 0; r < RCH; ++r)
          if (r < nr) acc[r] = fmaf(w, s_o[r * D_c + dd], acc[r]);
      }
#pragma unroll
      for (int r = 0; r < RCH; ++r)
        if (r < nr) st_elem(out, (int64_t)((r0 + r) * H + h) * o_stride + v, o_dtype, acc[r]);
    }
  }
}

bool dtype_ok(int d) { return d == KDV_BF16 || d == KDV_F32; }

kdv_status check_common(int32_t rows, int32_t H, int32_t D_in, int32_t D_out, const void* in, int64_t in_stride,
                        const void* w, int w_dtype, void* out, int64_t out_stride, int out_dtype) {
  if (rows < 0 || H < 1 || D_in < 1 || D_out < 1) return KDV_ERR_INVALID_ARG;
  if (rows % H != 0) return KDV_ERR_INVALID_ARG;
  if (!dtype_ok(w_dtype) || !dtype_ok(out_dtype)) return KDV_ERR_INVALID_ARG;
  if (rows > 0 && (in == nullptr || w == nullptr || out == nullptr)) return KDV_ERR_INVALID_ARG;
  if (in_stride < D_in || out_stride < D_out) return KDV_ERR_INVALID_ARG;
  return KDV_OK;
}

}  // namespace
}  // namespace kdv

using namespace kdv;

extern "C" {

kdv_status kdv_absorb_q(int32_t rows, int32_t num_heads, int32_t d_latent, int32_t d_nope, const void* q_nope,
                        int64_t q_nope_stride, int32_t q_dtype, const void* w_uk, int32_t w_dtype, void* q_lat,
                        int64_t q_lat_stride, int32_t out_dtype, void* stream) {
  kdv_status st = check_common(rows, num_heads, d_nope, d_latent, q_nope, q_nope_stride, w_uk, w_dtype, q_lat,
                               q_lat_stride, out_dtype);
  if (st != KDV_OK) return st;
  if (!dtype_ok(q_dtype)) return KDV_ERR_INVALID_ARG;
  if (d_nope > 512 || d_latent > 4096) return KDV_ERR_UNSUPPORTED;
  if (rows == 0) return KDV_OK;
  const size_t smem = (size_t)RCH * d_nope * sizeof(float);
  static bool attr_set[64] = {};
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return KDV_ERR_CUDA;
  if (dev >= 0 && dev < 64 && !attr_set[dev]) {
    if (cudaFuncSetAttribute(absorb_q_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, RCH * 512 * 4) !=
        cudaSuccess)
      return KDV_ERR_CUDA;
    attr_set[dev] = true;
  }
  const dim3 grid((unsigned)num_heads, (unsigned)((d_latent + THREADS - 1) / THREADS));
  absorb_q_kernel<<<grid, THREADS, smem, static_cast<cudaStream_t>(stream)>>>(
      rows / num_heads, num_heads, d_latent, d_nope, q_nope, q_nope_stride, q_dtype, w_uk, w_dtype, q_lat,
      q_lat_stride, out_dtype);
  return cudaGetLastError() == cudaSuccess ? KDV_OK : KDV_ERR_CUDA;
}

kdv_status kdv_unabsorb_o(int32_t rows, int32_t num_heads, int32_t d_latent, int32_t d_v, const float* o_lat,
                          int64_t o_lat_stride, const void* w_uv, int32_t w_dtype, void* out, int64_t out_stride,
                          int32_t out_dtype, void* stream) {
  kdv_status st = check_common(rows, num_heads, d_latent, d_v, o_lat, o_lat_stride, w_uv, w_dtype, out,
                               out_stride, out_dtype);
  if (st != KDV_OK) return st;
  if (d_latent > 512 || d_v > 4096) return KDV_ERR_UNSUPPORTED;
  if (rows == 0) return KDV_OK;
  const size_t smem = (size_t)RCH * d_latent * sizeof(float);
  static bool attr_set[64] = {};
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return KDV_ERR_CUDA;
  if (dev >= 0 && dev < 64 && !attr_set[dev]) {
    if (cudaFuncSetAttribute(unabsorb_o_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, RCH * 512 * 4) !=
        cudaSuccess)
      return KDV_ERR_CUDA;
    attr_set[dev] = true;
  }
  const dim3 grid((unsigned)num_heads, (unsigned)((d_v + THREADS - 1) / THREADS));
  unabsorb_o_kernel<<<grid, THREADS, smem, static_cast<cudaStream_t>(stream)>>>(
      rows / num_heads, num_heads, d_latent, d_v, o_lat, o_lat_stride, w_uv, w_dtype, out, out_stride, out_dtype);
  return cudaGetLastError() == cudaSuccess ? KDV_OK : KDV_ERR_CUDA;
}

}  // extern "C"

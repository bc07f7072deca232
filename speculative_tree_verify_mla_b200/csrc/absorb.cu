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
// fp32 on CUDA cores. Both kernels stage a head's input rows in shared
// memory and issue each thread's weight loads before any arithmetic, so the
// weights stream in one memory round trip.
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include "kdv.h"

namespace kdv {
namespace {

constexpr int THREADS = 128;
constexpr int RCH = 16;              // absorb: rows per pass (accumulators per thread)
constexpr int U_THREADS = 512;       // unabsorb: 16 d-groups x 32 column pairs
constexpr int U_GROUPS = 16;
constexpr int U_VB = 64;             // unabsorb: output columns per CTA
constexpr int U_RCH = 16;            // unabsorb: rows per pass
constexpr int U_MAX_DG = 32;         // d per group (D_c <= 512)
constexpr int STAGE_UNROLL = 8;      // staging: loads in flight per thread

// Stage rows [r0, r0+nr) of head h (row stride `stride` elements) into a
// dense [nr][n] fp32 array in shared memory; every thread issues up to
// STAGE_UNROLL loads before its first store.
__device__ __forceinline__ void stage_rows(float* dst, const void* src, int dtype, int64_t stride, int r0, int nr,
                                           int H, int h, int n, int nthreads) {
  const int total = nr * n;
  for (int base = threadIdx.x; base < total; base += nthreads * STAGE_UNROLL) {
    float v[STAGE_UNROLL];
#pragma unroll
    for (int u = 0; u < STAGE_UNROLL; ++u) {
      const int i = base + u * nthreads;
      v[u] = 0.f;
      if (i < total) {
        const int r = i / n, k = i - r * n;
        v[u] = dtype == KDV_BF16
                   ? __bfloat162float(static_cast<const __nv_bfloat16*>(src)[(int64_t)((r0 + r) * H + h) * stride + k])
                   : static_cast<const float*>(src)[(int64_t)((r0 + r) * H + h) * stride + k];
      }
    }
#pragma unroll
    for (int u = 0; u < STAGE_UNROLL; ++u) {
      const int i = base + u * nthreads;
      if (i < total) dst[i] = v[u];
    }
  }
}

__device__ __forceinline__ float ld_elem(const void* p, int64_t i, int dtype) {
  return dtype == KDV_BF16 ? __bfloat162float(static_cast<const __nv_bfloat16*>(p)[i])
                           : static_cast<const float*>(p)[i];
}
__device__ __forceinline__ void st_elem(void* p, int64_t i, int dtype, float v) {
  if (dtype == KDV_BF16) static_cast<__nv_bfloat16*>(p)[i] = __float2bfloat16_rn(v);
  else static_cast<float*>(p)[i] = v;
}
__device__ __forceinline__ float bf16_lo(uint32_t w) { return __uint_as_float(w << 16); }
__device__ __forceinline__ float bf16_hi(uint32_t w) { return __uint_as_float(w & 0xffff0000u); }

// q_lat[row][d] = sum_k W_UK[h][d][k] q_nope[row][k], one column d per thread.
// VEC: bf16 weights, D_n a multiple of 8 and rows 16-byte aligned -- the
// thread issues the 16-byte loads of a 128-weight chunk of its row before
// using any of them, so the whole weight matrix is in flight at once.
template <bool VEC>
__global__ void __launch_bounds__(THREADS)
absorb_q_kernel(int32_t rows_per_head, int32_t H, int32_t D_c, int32_t D_n, const void* __restrict__ q_nope,
                int64_t q_stride, int q_dtype, const void* __restrict__ w_uk, int w_dtype, void* __restrict__ q_lat,
                int64_t o_stride, int o_dtype) {
  extern __shared__ float s_q[];     // [RCH][D_n]
  const int h = blockIdx.x;
  const int d = blockIdx.y * THREADS + threadIdx.x;
  const bool active = d < D_c;
  const int64_t wrow = ((int64_t)h * D_c + (active ? d : 0)) * D_n;
  for (int r0 = 0; r0 < rows_per_head; r0 += RCH) {
    const int nr = min(RCH, rows_per_head - r0);
    __syncthreads();
    stage_rows(s_q, q_nope, q_dtype, q_stride, r0, nr, H, h, D_n, THREADS);
    __syncthreads();
    float acc[RCH];
#pragma unroll
    for (int r = 0; r < RCH; ++r) acc[r] = 0.f;
    if (VEC) {
      const uint4* wp = reinterpret_cast<const uint4*>(static_cast<const __nv_bfloat16*>(w_uk) + wrow);
      for (int kc = 0; kc < D_n; kc += 128) {
        const int n8 = min(16, (D_n - kc) / 8);
        uint4 w[16];
#pragma unroll
        for (int j = 0; j < 16; ++j) w[j] = (j < n8) ? __ldg(wp + kc / 8 + j) : make_uint4(0, 0, 0, 0);
        // weights outer (each converted once), rows inner
#pragma unroll
        for (int j = 0; j < 16; ++j) {
          if (j < n8) {
            const float wf[8] = {bf16_lo(w[j].x), bf16_hi(w[j].x), bf16_lo(w[j].y), bf16_hi(w[j].y),
                                 bf16_lo(w[j].z), bf16_hi(w[j].z), bf16_lo(w[j].w), bf16_hi(w[j].w)};
#pragma unroll
            for (int r = 0; r < RCH; ++r) {
              if (r < nr) {
                const float* q = s_q + r * D_n + kc + 8 * j;
                const float4 qa = *reinterpret_cast<const float4*>(q);
                const float4 qb = *reinterpret_cast<const float4*>(q + 4);
                float a = acc[r];
                a = fmaf(wf[0], qa.x, a);
                a = fmaf(wf[1], qa.y, a);
                a = fmaf(wf[2], qa.z, a);
                a = fmaf(wf[3], qa.w, a);
                a = fmaf(wf[4], qb.x, a);
                a = fmaf(wf[5], qb.y, a);
                a = fmaf(wf[6], qb.z, a);
                a = fmaf(wf[7], qb.w, a);
                acc[r] = a;
              }
            }
          }
        }
      }
    } else {
      for (int k = 0; k < D_n; ++k) {
        const float w = ld_elem(w_uk, wrow + k, w_dtype);
#pragma unroll
        for (int r = 0; r < RCH; ++r)
          if (r < nr) acc[r] = fmaf(w, s_q[r * D_n + k], acc[r]);
      }
    }
    if (active) {
#pragma unroll
      for (int r = 0; r < RCH; ++r)
        if (r < nr) st_elem(q_lat, (int64_t)((r0 + r) * H + h) * o_stride + d, o_dtype, acc[r]);
    }
  }
}

// out[row][v] = sum_d W_UV[h][d][v] o_lat[row][d]. One CTA per (head, block
// of 64 columns): thread (g, c) holds columns 2c, 2c+1 of the 32-d group g
// (D_c <= 512 split in 16 groups) -- it loads those 2 x 32 weights (two
// 2-byte loads per d, a warp covering 128 contiguous bytes) before any
// arithmetic -- and the 16 groups' partial sums are added through shared
// memory.
template <bool WBF16>
__global__ void __launch_bounds__(U_THREADS)
unabsorb_o_kernel(int32_t rows_per_head, int32_t H, int32_t D_c, int32_t D_v, const float* __restrict__ o_lat,
                  int64_t i_stride, const void* __restrict__ w_uv, int w_dtype, void* __restrict__ out,
                  int64_t o_stride, int o_dtype) {
  extern __shared__ float smem_u[];
  float* s_o = smem_u;                                   // [U_RCH][D_c]
  float* s_part = smem_u + U_RCH * D_c;                  // [U_GROUPS][U_RCH][U_VB]
  const int h = blockIdx.x;
  const int g = threadIdx.x / (U_VB / 2), c = threadIdx.x % (U_VB / 2);
  const int v0 = blockIdx.y * U_VB + 2 * c;
  const int dg = (D_c + U_GROUPS - 1) / U_GROUPS;
  const bool vec_o = dg % 4 == 0 && D_c % 4 == 0;          // 16-byte aligned group starts
  const int d0 = g * dg;
  const int nd = max(0, min(dg, D_c - d0));
  // this thread's weights W_UV[h][d0 + j][v0 .. v0+1]; bf16 pairs stay
  // packed in one register (bf16 -> fp32 is a shift)
  uint32_t wp[U_MAX_DG];
  float w0[WBF16 ? 1 : U_MAX_DG], w1[WBF16 ? 1 : U_MAX_DG];
#pragma unroll
  for (int j = 0; j < U_MAX_DG; ++j) {
    if (WBF16) {
      wp[j] = 0u;
      if (j < nd) {
        const int64_t e = ((int64_t)h * D_c + d0 + j) * D_v + v0;
        const uint16_t* wb = static_cast<const uint16_t*>(w_uv);
        const uint32_t lo = v0 < D_v ? wb[e] : 0u, hi = v0 + 1 < D_v ? wb[e + 1] : 0u;
        wp[j] = lo | (hi << 16);
      }
    } else {
      w0[j] = 0.f;
      w1[j] = 0.f;
      if (j < nd) {
        const int64_t e = ((int64_t)h * D_c + d0 + j) * D_v + v0;
        if (v0 < D_v) w0[j] = ld_elem(w_uv, e, w_dtype);
        if (v0 + 1 < D_v) w1[j] = ld_elem(w_uv, e + 1, w_dtype);
      }
    }
  }
  float wl[U_MAX_DG], wh[U_MAX_DG];               // converted once
#pragma unroll
  for (int j = 0; j < U_MAX_DG; ++j) {
    wl[j] = WBF16 ? bf16_lo(wp[j]) : w0[j];
    wh[j] = WBF16 ? bf16_hi(wp[j]) : w1[j];
  }
  auto wlo = [&](int j) { return wl[j]; };
  auto whi = [&](int j) { return wh[j]; };
  for (int r0 = 0; r0 < rows_per_head; r0 += U_RCH) {
    const int nr = min(U_RCH, rows_per_head - r0);
    __syncthreads();
    stage_rows(s_o, o_lat, KDV_F32, i_stride, r0, nr, H, h, D_c, U_THREADS);
    __syncthreads();
    for (int r = 0; r < nr; ++r) {
      const float* o = s_o + r * D_c + d0;
      float a0 = 0.f, a1 = 0.f, b0 = 0.f, b1 = 0.f;
      if (vec_o && nd == U_MAX_DG) {
#pragma unroll
        for (int j = 0; j < U_MAX_DG; j += 4) {          // float4 broadcast reads
          const float4 o4 = *reinterpret_cast<const float4*>(o + j);
          a0 = fmaf(wlo(j), o4.x, a0);
          b0 = fmaf(whi(j), o4.x, b0);
          a1 = fmaf(wlo(j + 1), o4.y, a1);
          b1 = fmaf(whi(j + 1), o4.y, b1);
          a0 = fmaf(wlo(j + 2), o4.z, a0);
          b0 = fmaf(whi(j + 2), o4.z, b0);
          a1 = fmaf(wlo(j + 3), o4.w, a1);
          b1 = fmaf(whi(j + 3), o4.w, b1);
        }
      } else {
#pragma unroll
        for (int j = 0; j < U_MAX_DG; ++j) {
          if (j < nd) {
            a0 = fmaf(wlo(j), o[j], a0);
            b0 = fmaf(whi(j), o[j], b0);
          }
        }
      }
      s_part[(g * U_RCH + r) * U_VB + 2 * c] = a0 + a1;
      s_part[(g * U_RCH + r) * U_VB + 2 * c + 1] = b0 + b1;
    }
    __syncthreads();
    for (int i = threadIdx.x; i < nr * U_VB; i += U_THREADS) {
      const int r = i / U_VB, col = i % U_VB, v = blockIdx.y * U_VB + col;
      float sum = 0.f;
#pragma unroll
      for (int gg = 0; gg < U_GROUPS; ++gg) sum += s_part[(gg * U_RCH + r) * U_VB + col];
      if (v < D_v) st_elem(out, (int64_t)((r0 + r) * H + h) * o_stride + v, o_dtype, sum);
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
  const bool vec = w_dtype == KDV_BF16 && d_nope % 8 == 0 && (reinterpret_cast<uintptr_t>(w_uk) & 15) == 0;
  static bool attr_set[64] = {};
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return KDV_ERR_CUDA;
  if (dev >= 0 && dev < 64 && !attr_set[dev]) {
    if (cudaFuncSetAttribute(absorb_q_kernel<true>, cudaFuncAttributeMaxDynamicSharedMemorySize, RCH * 512 * 4) !=
            cudaSuccess ||
        cudaFuncSetAttribute(absorb_q_kernel<false>, cudaFuncAttributeMaxDynamicSharedMemorySize, RCH * 512 * 4) !=
            cudaSuccess)
      return KDV_ERR_CUDA;
    attr_set[dev] = true;
  }
  const dim3 grid((unsigned)num_heads, (unsigned)((d_latent + THREADS - 1) / THREADS));
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  if (vec)
    absorb_q_kernel<true><<<grid, THREADS, smem, s>>>(rows / num_heads, num_heads, d_latent, d_nope, q_nope,
                                                      q_nope_stride, q_dtype, w_uk, w_dtype, q_lat, q_lat_stride,
                                                      out_dtype);
  else
    absorb_q_kernel<false><<<grid, THREADS, smem, s>>>(rows / num_heads, num_heads, d_latent, d_nope, q_nope,
                                                       q_nope_stride, q_dtype, w_uk, w_dtype, q_lat, q_lat_stride,
                                                       out_dtype);
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
  const size_t smem = ((size_t)U_RCH * d_latent + (size_t)U_GROUPS * U_RCH * U_VB) * sizeof(float);
  static bool attr_set[64] = {};
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return KDV_ERR_CUDA;
  if (dev >= 0 && dev < 64 && !attr_set[dev]) {
    const int bytes = (U_RCH * 512 + U_GROUPS * U_RCH * U_VB) * 4;
    if (cudaFuncSetAttribute(unabsorb_o_kernel<true>, cudaFuncAttributeMaxDynamicSharedMemorySize, bytes) !=
            cudaSuccess ||
        cudaFuncSetAttribute(unabsorb_o_kernel<false>, cudaFuncAttributeMaxDynamicSharedMemorySize, bytes) !=
            cudaSuccess)
      return KDV_ERR_CUDA;
    attr_set[dev] = true;
  }
  const dim3 grid((unsigned)num_heads, (unsigned)((d_v + U_VB - 1) / U_VB));
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  if (w_dtype == KDV_BF16)
    unabsorb_o_kernel<true><<<grid, U_THREADS, smem, s>>>(rows / num_heads, num_heads, d_latent, d_v, o_lat,
                                                          o_lat_stride, w_uv, w_dtype, out, out_stride, out_dtype);
  else
    unabsorb_o_kernel<false><<<grid, U_THREADS, smem, s>>>(rows / num_heads, num_heads, d_latent, d_v, o_lat,
                                                           o_lat_stride, w_uv, w_dtype, out, out_stride, out_dtype);
  return cudaGetLastError() == cudaSuccess ? KDV_OK : KDV_ERR_CUDA;
}

}  // extern "C"

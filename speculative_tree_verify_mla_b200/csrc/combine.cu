// combine.cu -- log-sum-exp merge of split partials.
//
// The prefix / tree-tail merge of page "The Three Acts of Engineering",
// reference [1] (one kernel for the long prefix, another for the small tree
// tail), generalised to any number of key splits: with per-split results
// (o_k, lse_k), LSE = ln sum_k exp(lse_k) and o = sum_k exp(lse_k - LSE) o_k.
// HBM-bound: it reads S*(d+1) floats and writes d+1 floats per row. One CTA
// of 128 threads per row, each thread owning 4 consecutive dims (float4).
#include "kdv_internal.cuh"

namespace kdv {
namespace {

constexpr int THREADS = 128;

// o_row[c] = sum_k w_k part(k)[c], part(k) = base + k * split_stride (floats).
__device__ inline void combine_row(const float* __restrict__ base_o, int64_t split_stride_o,
                                   const float* __restrict__ base_l, int64_t split_stride_l,
                                   int32_t S, int32_t d, float* __restrict__ out,
                                   float* __restrict__ lse_out) {
  __shared__ float w[64];
  float m = -INFINITY;
  for (int k = 0; k < S; ++k) m = fmaxf(m, base_l[k * split_stride_l]);
  if (m == -INFINITY) {
    for (int c = threadIdx.x; c < d; c += THREADS) out[c] = 0.f;
    if (threadIdx.x == 0 && lse_out) *lse_out = -INFINITY;
    return;
  }
  float z = 0.f;
  for (int k = 0; k < S; ++k) z += expf(base_l[k * split_stride_l] - m);
  const float LSE = m + logf(z);
  if (threadIdx.x == 0 && lse_out) *lse_out = LSE;
  const bool vec = (d % 4 == 0) && ((reinterpret_cast<uintptr_t>(base_o) & 15) == 0) &&
                   ((split_stride_o & 3) == 0) && ((reinterpret_cast<uintptr_t>(out) & 15) == 0);
  for (int k0 = 0; k0 < S; k0 += 64) {
    const int kn = min(64, S - k0);
    __syncthreads();
    if (threadIdx.x < kn) {
      const float lk = base_l[(k0 + threadIdx.x) * split_stride_l];
      w[threadIdx.x] = (lk == -INFINITY) ? 0.f : expf(lk - LSE);
    }
    __syncthreads();
    if (vec) {
      for (int c = threadIdx.x * 4; c < d; c += THREADS * 4) {
        float4 acc = k0 == 0 ? make_float4(0.f, 0.f, 0.f, 0.f)
                             : *reinterpret_cast<const float4*>(out + c);
        for (int k = 0; k < kn; ++k) {
          const float wk = w[k];
          if (wk == 0.f) continue;
          const float4 v = __ldg(reinterpret_cast<const float4*>(base_o + (k0 + k) * split_stride_o + c));
          acc.x = fmaf(wk, v.x, acc.x);
          acc.y = fmaf(wk, v.y, acc.y);
          acc.z = fmaf(wk, v.z, acc.z);
          acc.w = fmaf(wk, v.w, acc.w);
        }
        *reinterpret_cast<float4*>(out + c) = acc;
      }
    } else {
      for (int c = threadIdx.x; c < d; c += THREADS) {
        float acc = k0 == 0 ? 0.f : out[c];
        for (int k = 0; k < kn; ++k) {
          const float wk = w[k];
          if (wk == 0.f) continue;
          acc = fmaf(wk, base_o[(k0 + k) * split_stride_o + c], acc);
        }
        out[c] = acc;
      }
    }
  }
}

__global__ void __launch_bounds__(THREADS)
combine_uniform_kernel(const float* __restrict__ o_part, const float* __restrict__ lse_part,
                       int32_t S, int64_t rows, int32_t d, float* __restrict__ o,
                       float* __restrict__ lse) {
  for (int64_t r = blockIdx.x; r < rows; r += gridDim.x) {
    combine_row(o_part + r * d, rows * d, lse_part + r, rows, S, d, o + r * d,
                lse ? lse + r : nullptr);
    __syncthreads();
  }
}

__global__ void __launch_bounds__(THREADS)
combine_plan_kernel(const float* __restrict__ ws_o, const float* __restrict__ ws_lse,
                    const VerifyPlan p, int32_t d, float* __restrict__ o,
                    float* __restrict__ lse) {
  for (int64_t row = blockIdx.x; row < p.total_rows; row += gridDim.x) {
    // request of this global row: tree_base[b]*H <= row < tree_base[b+1]*H
    int b = 0;
    while (b + 1 < p.B && (int64_t)p.tree_base[b + 1] * p.H <= row) ++b;
    const int64_t r = row - (int64_t)p.tree_base[b] * p.H;
    const int64_t rows_b = (int64_t)p.T[b] * p.H;
    const int64_t first = p.part_base[b] + r;
    combine_row(ws_o + first * d, rows_b * d, ws_lse + first, rows_b, p.S[b], d, o + row * d,
                lse ? lse + row : nullptr);
    __syncthreads();
  }
}

}  // namespace

cudaError_t launch_combine_uniform(const float* o_part, const float* lse_part, int32_t S,
                                   int64_t rows, int32_t d, float* o, float* lse,
                                   cudaStream_t stream) {
  if (rows == 0) return cudaSuccess;
  const int64_t grid = rows < 65535 * 4 ? rows : 65535 * 4;
  combine_uniform_kernel<<<(unsigned)grid, THREADS, 0, stream>>>(o_part, lse_part, S, rows, d, o, lse);
  return cudaGetLastError();
}

cudaError_t launch_combine_plan(const float* ws_o, const float* ws_lse, const VerifyPlan& p,
                                int32_t d, float* o, float* lse, cudaStream_t stream) {
  if (p.total_rows == 0) return cudaSuccess;
  combine_plan_kernel<<<p.total_rows, THREADS, 0, stream>>>(ws_o, ws_lse, p, d, o, lse);
  return cudaGetLastError();
}

}  // namespace kdv

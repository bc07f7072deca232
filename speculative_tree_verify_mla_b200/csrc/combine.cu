// combine.cu -- log-sum-exp merge of split partials.
//
// The prefix / tree-tail merge of page "The Three Acts of Engineering",
// reference [1] (one kernel for the long prefix, another for the small tree
// tail), generalised to any number of key splits: with per-split results
// (o_k, lse_k), LSE = ln sum_k exp(lse_k) and o = sum_k exp(lse_k - LSE) o_k.
// HBM-bound: it reads S*(d+1) floats and writes d+1 floats per row. One CTA
// per row.
#include "kdv_internal.cuh"

namespace kdv {
namespace {

constexpr int THREADS = 128;
constexpr int KB = 8;              // splits whose loads are in flight together

// One CTA merges one row: o_row[c] = sum_k w_k part(k)[c] with
// part(k) = base_o + k * sso (floats), lse_k = base_l[k * ssl] and
// w_k = exp(lse_k - LSE). Each thread owns 4 consecutive columns (float4)
// and issues the loads of KB splits before it reads the split LSEs, so a
// row costs about one memory round trip; every thread reduces the (cached)
// LSEs itself instead of waiting on a block-wide reduction.
__device__ inline void combine_row(const float* __restrict__ base_o, int64_t sso,
                                   const float* __restrict__ base_l, int64_t ssl, int32_t S,
                                   int32_t d, float* __restrict__ out,
                                   float* __restrict__ lse_out) {
  const bool vec = (d % 4 == 0) && ((reinterpret_cast<uintptr_t>(base_o) & 15) == 0) &&
                   ((sso & 3) == 0) && ((reinterpret_cast<uintptr_t>(out) & 15) == 0);
  const int step = vec ? 4 : 1;
  const int c0 = threadIdx.x * step;
  float4 v[KB];
  if (vec && c0 < d) {
#pragma unroll
    for (int u = 0; u < KB; ++u)
      if (u < S) v[u] = __ldg(reinterpret_cast<const float4*>(base_o + u * sso + c0));
  }
  float m = -INFINITY;
  for (int k = 0; k < S; ++k) m = fmaxf(m, __ldg(base_l + k * ssl));
  if (m == -INFINITY) {
    for (int c = threadIdx.x; c < d; c += THREADS) out[c] = 0.f;
    if (threadIdx.x == 0 && lse_out) *lse_out = -INFINITY;
    return;
  }
  float z = 0.f;
  for (int k = 0; k < S; ++k) z += expf(__ldg(base_l + k * ssl) - m);
  const float LSE = m + logf(z);
  if (threadIdx.x == 0 && lse_out) *lse_out = LSE;
  if (vec) {
    for (int c = c0; c < d; c += THREADS * 4) {
      float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
      for (int k0 = 0; k0 < S; k0 += KB) {
        if (c != c0 || k0 != 0) {      // the first batch was loaded above
#pragma unroll
          for (int u = 0; u < KB; ++u)
            if (k0 + u < S) v[u] = __ldg(reinterpret_cast<const float4*>(base_o + (k0 + u) * sso + c));
        }
#pragma unroll
        for (int u = 0; u < KB; ++u) {
          if (k0 + u < S) {
            const float lk = __ldg(base_l + (k0 + u) * ssl);
            const float wk = (lk == -INFINITY) ? 0.f : expf(lk - LSE);
            acc.x = fmaf(wk, v[u].x, acc.x);
            acc.y = fmaf(wk, v[u].y, acc.y);
            acc.z = fmaf(wk, v[u].z, acc.z);
            acc.w = fmaf(wk, v[u].w, acc.w);
          }
        }
      }
      *reinterpret_cast<float4*>(out + c) = acc;
    }
  } else {
    for (int c = c0; c < d; c += THREADS) {
      float acc = 0.f;
      for (int k = 0; k < S; ++k) {
        const float lk = __ldg(base_l + k * ssl);
        const float wk = (lk == -INFINITY) ? 0.f : expf(lk - LSE);
        acc = fmaf(wk, base_o[k * sso + c], acc);
      }
      out[c] = acc;
    }
  }
}

__global__ void __launch_bounds__(THREADS)
combine_uniform_kernel(const float* __restrict__ o_part, const float* __restrict__ lse_part,
                       int32_t S, int64_t rows, int32_t d, float* __restrict__ o,
                       float* __restrict__ lse) {
  for (int64_t r = blockIdx.x; r < rows; r += gridDim.x)
    combine_row(o_part + r * d, rows * d, lse_part + r, rows, S, d, o + r * d,
                lse ? lse + r : nullptr);
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
  }
}

}  // namespace

cudaError_t launch_combine_uniform(const float* o_part, const float* lse_part, int32_t S,
                                   int64_t rows, int32_t d, float* o, float* lse,
                                   cudaStream_t stream) {
  if (rows == 0) return cudaSuccess;
  const int64_t grid = rows < (int64_t)1 << 30 ? rows : (int64_t)1 << 30;
  combine_uniform_kernel<<<(unsigned)grid, THREADS, 0, stream>>>(o_part, lse_part, S, rows, d, o, lse);
  return cudaGetLastError();
}

cudaError_t launch_combine_plan(const float* ws_o, const float* ws_lse, const VerifyPlan& p,
                                int32_t d, float* o, float* lse, cudaStream_t stream) {
  if (p.total_rows == 0) return cudaSuccess;
  const int64_t grid = p.total_rows < (int64_t)1 << 30 ? p.total_rows : (int64_t)1 << 30;
  combine_plan_kernel<<<(unsigned)grid, THREADS, 0, stream>>>(ws_o, ws_lse, p, d, o, lse);
  return cudaGetLastError();
}

}  // namespace kdv

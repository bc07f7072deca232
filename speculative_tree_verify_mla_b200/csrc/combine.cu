// combine.cu -- log-sum-exp merge of split partials.
//
// The prefix / tree-tail merge of page "The Three Acts of Engineering",
// reference [1] (one kernel for the long prefix, another for the small tree
// tail), generalised to any number of key splits: with per-split results
// (o_k, lse_k), LSE = ln sum_k exp(lse_k) and o = sum_k exp(lse_k - LSE) o_k.
// HBM-bound: it reads S*(d+1) floats and writes d+1 floats per row. One warp
// per row, four rows per CTA.
#include "kdv_internal.cuh"

namespace kdv {
namespace {

constexpr int THREADS = 128;
constexpr int ROWS_PER_CTA = THREADS / 32;     // one warp per row

__device__ __forceinline__ float warp_max(float v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, o));
  return v;
}
__device__ __forceinline__ float warp_sum(float v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  return v;
}

// One warp merges one row: o_row[c] = sum_k w_k part(k)[c] with
// part(k) = base_o + k * sso (floats) and lse_k = base_l[k * ssl]. The lanes
// read the split LSEs 32 at a time and reduce them with shuffles; then each
// lane owns 4 columns of every 128 (float4) and issues the loads of four
// splits back to back.
__device__ inline void combine_row_warp(const float* __restrict__ base_o, int64_t sso,
                                        const float* __restrict__ base_l, int64_t ssl, int32_t S,
                                        int32_t d, float* __restrict__ out,
                                        float* __restrict__ lse_out) {
  const int lane = threadIdx.x & 31;
  float m = -INFINITY;
  for (int k = lane; k < S; k += 32) m = fmaxf(m, base_l[k * ssl]);
  m = warp_max(m);
  if (m == -INFINITY) {
    for (int c = lane; c < d; c += 32) out[c] = 0.f;
    if (lane == 0 && lse_out) *lse_out = -INFINITY;
    return;
  }
  float z = 0.f;
  for (int k = lane; k < S; k += 32) z += expf(base_l[k * ssl] - m);
  z = warp_sum(z);
  const float LSE = m + logf(z);
  if (lane == 0 && lse_out) *lse_out = LSE;
  const bool vec = (d % 4 == 0) && ((reinterpret_cast<uintptr_t>(base_o) & 15) == 0) &&
                   ((sso & 3) == 0) && ((reinterpret_cast<uintptr_t>(out) & 15) == 0);
  for (int k0 = 0; k0 < S; k0 += 32) {
    const int kn = min(32, S - k0);
    float wl = 0.f;
    if (lane < kn) {
      const float lk = base_l[(k0 + lane) * ssl];
      wl = (lk == -INFINITY) ? 0.f : expf(lk - LSE);
    }
    if (vec) {
      for (int c = lane * 4; c < d; c += 128) {
        float4 acc = k0 == 0 ? make_float4(0.f, 0.f, 0.f, 0.f) : *reinterpret_cast<const float4*>(out + c);
        int k = 0;
        for (; k + 4 <= kn; k += 4) {
          float4 v[4];
#pragma unroll
          for (int u = 0; u < 4; ++u)
            v[u] = __ldg(reinterpret_cast<const float4*>(base_o + (k0 + k + u) * sso + c));
#pragma unroll
          for (int u = 0; u < 4; ++u) {
            const float wk = __shfl_sync(0xffffffffu, wl, k + u);
            if (wk != 0.f) {
              acc.x = fmaf(wk, v[u].x, acc.x);
              acc.y = fmaf(wk, v[u].y, acc.y);
              acc.z = fmaf(wk, v[u].z, acc.z);
              acc.w = fmaf(wk, v[u].w, acc.w);
            }
          }
        }
        for (; k < kn; ++k) {
          const float wk = __shfl_sync(0xffffffffu, wl, k);
          if (wk != 0.f) {
            const float4 v = __ldg(reinterpret_cast<const float4*>(base_o + (k0 + k) * sso + c));
            acc.x = fmaf(wk, v.x, acc.x);
            acc.y = fmaf(wk, v.y, acc.y);
            acc.z = fmaf(wk, v.z, acc.z);
            acc.w = fmaf(wk, v.w, acc.w);
          }
        }
        *reinterpret_cast<float4*>(out + c) = acc;
      }
    } else {
      for (int c = lane; c < d; c += 32) {
        float acc = k0 == 0 ? 0.f : out[c];
        for (int k = 0; k < kn; ++k) {
          const float wk = __shfl_sync(0xffffffffu, wl, k);
          if (wk != 0.f) acc = fmaf(wk, base_o[(k0 + k) * sso + c], acc);
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
  const int64_t stride = (int64_t)gridDim.x * ROWS_PER_CTA;
  for (int64_t r = (int64_t)blockIdx.x * ROWS_PER_CTA + (threadIdx.x >> 5); r < rows; r += stride)
    combine_row_warp(o_part + r * d, rows * d, lse_part + r, rows, S, d, o + r * d,
                     lse ? lse + r : nullptr);
}

__global__ void __launch_bounds__(THREADS)
combine_plan_kernel(const float* __restrict__ ws_o, const float* __restrict__ ws_lse,
                    const VerifyPlan p, int32_t d, float* __restrict__ o,
                    float* __restrict__ lse) {
  const int64_t stride = (int64_t)gridDim.x * ROWS_PER_CTA;
  for (int64_t row = (int64_t)blockIdx.x * ROWS_PER_CTA + (threadIdx.x >> 5); row < p.total_rows;
       row += stride) {
    // request of this global row: tree_base[b]*H <= row < tree_base[b+1]*H
    int b = 0;
    while (b + 1 < p.B && (int64_t)p.tree_base[b + 1] * p.H <= row) ++b;
    const int64_t r = row - (int64_t)p.tree_base[b] * p.H;
    const int64_t rows_b = (int64_t)p.T[b] * p.H;
    const int64_t first = p.part_base[b] + r;
    combine_row_warp(ws_o + first * d, rows_b * d, ws_lse + first, rows_b, p.S[b], d, o + row * d,
                     lse ? lse + row : nullptr);
  }
}

}  // namespace

cudaError_t launch_combine_uniform(const float* o_part, const float* lse_part, int32_t S,
                                   int64_t rows, int32_t d, float* o, float* lse,
                                   cudaStream_t stream) {
  if (rows == 0) return cudaSuccess;
  const int64_t ctas = (rows + ROWS_PER_CTA - 1) / ROWS_PER_CTA;
  const int64_t grid = ctas < 65535 * 4 ? ctas : 65535 * 4;
  combine_uniform_kernel<<<(unsigned)grid, THREADS, 0, stream>>>(o_part, lse_part, S, rows, d, o, lse);
  return cudaGetLastError();
}

cudaError_t launch_combine_plan(const float* ws_o, const float* ws_lse, const VerifyPlan& p,
                                int32_t d, float* o, float* lse, cudaStream_t stream) {
  if (p.total_rows == 0) return cudaSuccess;
  const int64_t ctas = (p.total_rows + ROWS_PER_CTA - 1) / ROWS_PER_CTA;
  const int64_t grid = ctas < 65535 * 4 ? ctas : 65535 * 4;
  combine_plan_kernel<<<(unsigned)grid, THREADS, 0, stream>>>(ws_o, ws_lse, p, d, o, lse);
  return cudaGetLastError();
}

}  // namespace kdv

// combine.cu -- log-sum-exp merge of split partials.
//
// The prefix / tree-tail merge of page "The Three Acts of Engineering",
// reference [1] (one kernel for the long prefix, another for the small tree
// tail), generalised to any number of key splits: with per-split results
// (o_k, lse_k), LSE = ln sum_k exp(lse_k) and o = sum_k exp(lse_k - LSE) o_k.
// HBM-bound: it reads S*(d+1) partial values and writes d+1 floats per row.
#include <cuda_fp16.h>

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

// The internal merge of the tensor-core kernel's fp16 partials (d = 512):
// one warp per row, lane l owning columns [16l, 16l+16). The loads of the
// first eight splits are issued together with those of the split LSEs,
// which are read once (lane k keeps lse_k), so a row with S <= 8 costs
// about one memory round trip.
constexpr int W16_WARPS = 4;
constexpr int W16_KB = 8;
constexpr int W16_SMEM = 100 * 1024;   // reserved, unused: two CTAs per SM at most

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
__device__ __forceinline__ void fma_half8(float (&acc)[16], int base, float w, uint4 x) {
  const uint32_t u[4] = {x.x, x.y, x.z, x.w};
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const float2 f = __half22float2(*reinterpret_cast<const __half2*>(&u[i]));
    acc[base + 2 * i] = fmaf(w, f.x, acc[base + 2 * i]);
    acc[base + 2 * i + 1] = fmaf(w, f.y, acc[base + 2 * i + 1]);
  }
}

__global__ void __launch_bounds__(32 * W16_WARPS)
combine_plan_f16_kernel(const __half* __restrict__ ws_o, const float* __restrict__ ws_lse,
                        const VerifyPlan p, float* __restrict__ o, float* __restrict__ lse) {
  constexpr int D = 512;
  const int lane = threadIdx.x & 31;
  // launched as a programmatic dependent of the attention kernel: wait for
  // it to complete (and its partials to be visible)
  asm volatile("griddepcontrol.wait;" ::: "memory");
  for (int64_t row = (int64_t)blockIdx.x * W16_WARPS + (threadIdx.x >> 5); row < p.total_rows;
       row += (int64_t)gridDim.x * W16_WARPS) {
    int b = 0;
    while (b + 1 < p.B && (int64_t)p.tree_base[b + 1] * p.H <= row) ++b;
    const int64_t rows_b = (int64_t)p.T[b] * p.H;
    const int64_t first = p.part_base[b] + (row - (int64_t)p.tree_base[b] * p.H);
    const int S = p.S[b];
    const __half* col0 = ws_o + first * D + lane * 16;
    uint4 x[W16_KB][2];
#pragma unroll
    for (int u = 0; u < W16_KB; ++u)
      if (u < S) {
        const uint4* src = reinterpret_cast<const uint4*>(col0 + (int64_t)u * rows_b * D);
        x[u][0] = __ldg(src);
        x[u][1] = __ldg(src + 1);
      }
    const float lk0 = lane < S ? __ldg(ws_lse + first + (int64_t)lane * rows_b) : -INFINITY;
    float m = fmaxf(-INFINITY, lk0);
    for (int k = lane + 32; k < S; k += 32) m = fmaxf(m, __ldg(ws_lse + first + (int64_t)k * rows_b));
    m = warp_max(m);
    float acc[16];
#pragma unroll
    for (int i = 0; i < 16; ++i) acc[i] = 0.f;
    float LSE = -INFINITY;
    if (m != -INFINITY) {
      float z = 0.f;
      if (lane < S) z += lk0 == -INFINITY ? 0.f : expf(lk0 - m);
      for (int k = lane + 32; k < S; k += 32) {
        const float lk = __ldg(ws_lse + first + (int64_t)k * rows_b);
        z += lk == -INFINITY ? 0.f : expf(lk - m);
      }
      LSE = m + logf(warp_sum(z));
      for (int k0 = 0; k0 < S; k0 += 32) {
        const int kk = k0 + lane;
        const float lk = k0 == 0 ? lk0 : kk < S ? __ldg(ws_lse + first + (int64_t)kk * rows_b) : -INFINITY;
        const float wk = lk == -INFINITY ? 0.f : expf(lk - LSE);
        const int n = min(32, S - k0);
        for (int j = 0; j < n; j += W16_KB) {
          if (k0 + j > 0) {      // the first batch was loaded above
#pragma unroll
            for (int u = 0; u < W16_KB; ++u)
              if (j + u < n) {
                const uint4* src = reinterpret_cast<const uint4*>(col0 + (int64_t)(k0 + j + u) * rows_b * D);
                x[u][0] = __ldg(src);
                x[u][1] = __ldg(src + 1);
              }
          }
#pragma unroll
          for (int u = 0; u < W16_KB; ++u) {
            const float w = __shfl_sync(0xffffffffu, wk, (j + u) & 31);
            if (j + u < n) {
              fma_half8(acc, 0, w, x[u][0]);
              fma_half8(acc, 8, w, x[u][1]);
            }
          }
        }
      }
    }
    float* orow = o + row * D + lane * 16;
    if ((reinterpret_cast<uintptr_t>(o) & 15) == 0) {
      float4* dst = reinterpret_cast<float4*>(orow);
#pragma unroll
      for (int i = 0; i < 4; ++i) dst[i] = make_float4(acc[4 * i], acc[4 * i + 1], acc[4 * i + 2], acc[4 * i + 3]);
    } else {
#pragma unroll
      for (int i = 0; i < 16; ++i) orow[i] = acc[i];
    }
    if (lane == 0 && lse != nullptr) lse[row] = LSE;
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

cudaError_t launch_combine_plan(const void* ws_o, const float* ws_lse, const VerifyPlan& p,
                                int32_t d, float* o, float* lse, cudaStream_t stream) {
  if (p.total_rows == 0) return cudaSuccess;
  if (p.part_f16) {
    if (d != 512) return cudaErrorInvalidValue;
    const int64_t blocks = (p.total_rows + W16_WARPS - 1) / W16_WARPS;
    const int64_t grid = blocks < (int64_t)1 << 30 ? blocks : (int64_t)1 << 30;
    // Launched as a programmatic dependent of the attention kernel, whose
    // CTAs signal it from their epilogue: its CTAs take the SMs the
    // attention kernel leaves free and wait there, so it starts without a
    // launch gap. The shared memory it reserves (and does not use) keeps
    // at most two of its CTAs on an SM, so the early ones do not gather the
    // whole merge on the few free SMs.
    static bool smem_set[64] = {};
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    if (dev < 0 || dev >= 64 || !smem_set[dev]) {
      e = cudaFuncSetAttribute(combine_plan_f16_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, W16_SMEM);
      if (e != cudaSuccess) return e;
      if (dev >= 0 && dev < 64) smem_set[dev] = true;
    }
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3((unsigned)grid);
    cfg.blockDim = dim3(32 * W16_WARPS);
    cfg.dynamicSmemBytes = W16_SMEM;
    cfg.stream = stream;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    return cudaLaunchKernelEx(&cfg, combine_plan_f16_kernel, static_cast<const __half*>(ws_o), ws_lse, p, o, lse);
  }
  const int64_t grid = p.total_rows < (int64_t)1 << 30 ? p.total_rows : (int64_t)1 << 30;
  combine_plan_kernel<<<(unsigned)grid, THREADS, 0, stream>>>(static_cast<const float*>(ws_o), ws_lse, p, d, o,
                                                              lse);
  return cudaGetLastError();
}

}  // namespace kdv

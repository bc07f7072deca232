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
// fp32 on CUDA cores. The main kernels (bf16 weights whose rows are a
// multiple of 16 bytes) bring a CTA's whole weight tile into shared memory
// with one round of TMA copies and keep many warps busy on it: each thread
// holds a small block of outputs (two weight rows x four nodes, or four
// columns x four nodes) so that every shared-memory read feeds several packed
// fp32 FMAs (two correctly rounded fp32 FMAs per instruction). The general
// kernels below them (fp32 weights, other alignments) stage a head's input
// rows and issue each thread's weight loads before any arithmetic.
#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include "kdv.h"
#include "sm100_ptx.cuh"

namespace kdv {

// absorb_tc.cu: the tensor-core forms (bf16 weights; see the conditions below)
size_t absorb_tc_smem(int D_n);
size_t unabsorb_tc_smem(int D_c);
// early_weights: launch as a programmatic dependent of the preceding kernel
// (the weight copy may start before that kernel finishes)
cudaError_t launch_absorb_q_tc(const CUtensorMap& tmap, int32_t rows, int32_t H, int32_t D_c, int32_t D_n,
                               const void* q_nope, int64_t q_stride, void* q_lat, int64_t o_stride, int32_t o_dtype,
                               bool early_weights, cudaStream_t s);
cudaError_t launch_unabsorb_o_tc(const CUtensorMap& tmap, int32_t rows, int32_t H, int32_t D_c, int32_t D_v,
                                 const float* o_lat, int64_t i_stride, void* out, int64_t o_stride, int32_t o_dtype,
                                 bool early_weights, cudaStream_t s);

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


// ---------------------------------------------------------------------------
// TMA-staged kernels (bf16 weights)
// ---------------------------------------------------------------------------
constexpr int P_THREADS = 256;
constexpr int PA_ROWS = 128;         // absorb: weight rows (d) per CTA
constexpr int PA_TB = 16;            // absorb: nodes per pass (4 groups x 4)
constexpr int PU_V = 32;             // unabsorb: output columns per CTA
constexpr int PU_TB = 16;            // unabsorb: nodes per pass (4 groups x 4)
constexpr int PU_DG = 8;             // unabsorb: d interleave (d = g + 8 j)
constexpr int PU_MAX_DC = 512;
constexpr unsigned long long WAIT_NS = 2000000000ull;   // a TMA that has not landed in 2 s never will

__device__ __forceinline__ unsigned char* align1024(unsigned char* p) {
  return reinterpret_cast<unsigned char*>((reinterpret_cast<uintptr_t>(p) + 1023) & ~static_cast<uintptr_t>(1023));
}
__device__ __forceinline__ unsigned long long gtimer() {
  unsigned long long t;
  asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
  return t;
}
// Wait for phase 0 of `bar`, for at most WAIT_NS; false if it never completed.
__device__ __forceinline__ bool wait_landed(uint32_t bar) {
  if (ptx::mbar_try_wait(bar, 0)) return true;
  const unsigned long long t0 = gtimer();
  while (!ptx::mbar_try_wait(bar, 0))
    if (gtimer() - t0 > WAIT_NS) return false;
  return true;
}
__device__ __forceinline__ float2 bf16x2_to_float2(uint32_t w) { return make_float2(bf16_lo(w), bf16_hi(w)); }

// Stage rows [r0, r0+nr) of head h into shared memory as fp32 (DUP: as
// (x, x) pairs), 8 elements per 16- or 32-byte unit, every load of a thread
// issued before its first store. Needs n % 8 == 0, a 16-byte aligned base
// and a row stride that is a multiple of 8 elements.
template <bool DUP>
__device__ __forceinline__ void stage_rows_vec(void* dst, const void* src, int dtype, int64_t stride, int r0, int nr,
                                               int H, int h, int n) {
  constexpr int U = 4;
  const int units = n / 8, total = nr * units;
  for (int base = threadIdx.x; base < total; base += P_THREADS * U) {
    float v[U][8];
#pragma unroll
    for (int u = 0; u < U; ++u) {
      const int i = base + u * P_THREADS;
      if (i < total) {
        const int r = i / units, k8 = (i - r * units) * 8;
        const int64_t e = (int64_t)((r0 + r) * H + h) * stride + k8;
        if (dtype == KDV_BF16) {
          const uint4 w = *reinterpret_cast<const uint4*>(static_cast<const __nv_bfloat16*>(src) + e);
          v[u][0] = bf16_lo(w.x); v[u][1] = bf16_hi(w.x); v[u][2] = bf16_lo(w.y); v[u][3] = bf16_hi(w.y);
          v[u][4] = bf16_lo(w.z); v[u][5] = bf16_hi(w.z); v[u][6] = bf16_lo(w.w); v[u][7] = bf16_hi(w.w);
        } else {
          const float4 a = *reinterpret_cast<const float4*>(static_cast<const float*>(src) + e);
          const float4 b = *reinterpret_cast<const float4*>(static_cast<const float*>(src) + e + 4);
          v[u][0] = a.x; v[u][1] = a.y; v[u][2] = a.z; v[u][3] = a.w;
          v[u][4] = b.x; v[u][5] = b.y; v[u][6] = b.z; v[u][7] = b.w;
        }
      }
    }
#pragma unroll
    for (int u = 0; u < U; ++u) {
      const int i = base + u * P_THREADS;
      if (i < total) {
        const int r = i / units, k8 = (i - r * units) * 8;
        if (DUP) {
          float4* d4 = reinterpret_cast<float4*>(static_cast<float2*>(dst) + r * n + k8);
#pragma unroll
          for (int j = 0; j < 4; ++j) d4[j] = make_float4(v[u][2 * j], v[u][2 * j], v[u][2 * j + 1], v[u][2 * j + 1]);
        } else {
          float4* d4 = reinterpret_cast<float4*>(static_cast<float*>(dst) + r * n + k8);
          d4[0] = make_float4(v[u][0], v[u][1], v[u][2], v[u][3]);
          d4[1] = make_float4(v[u][4], v[u][5], v[u][6], v[u][7]);
        }
      }
    }
  }
}

// q_lat[row][d] = sum_k W_UK[h][d][k] q_nope[row][k]. CTA = (128 rows d of
// head h); its W_UK tile arrives as ceil(D_n/64) TMA boxes of [128 rows][64 k]
// with the 128-byte swizzle (16-byte chunk c of row r sits at chunk c ^ (r%8)),
// so the 32 rows a warp reads at one k land in distinct banks. Thread
// (rp = tid % 64, tg = tid / 64) owns rows rp and rp + 64 and nodes tg,
// tg+4, tg+8, tg+12 of each 16-node pass; a warp shares its nodes, so the
// node reads are broadcasts. k runs in pairs: the even and odd k of a row
// accumulate in the two halves of a float2 and are added at the end.
__global__ void __launch_bounds__(P_THREADS)
absorb_q_tma_kernel(const __grid_constant__ CUtensorMap tmap_w, int32_t rows_per_head, int32_t H, int32_t D_c,
                    int32_t D_n, const void* __restrict__ q_nope, int64_t q_stride, int q_dtype,
                    void* __restrict__ q_lat, int64_t o_stride, int o_dtype) {
  extern __shared__ unsigned char smem_raw[];
  __shared__ __align__(8) unsigned long long bar;
  unsigned char* s_w = align1024(smem_raw);
  const int nbox = (D_n + 63) / 64;
  float* s_q = reinterpret_cast<float*>(s_w + nbox * 16384);      // [PA_TB][D_n]
  const int h = blockIdx.y, d0 = blockIdx.x * PA_ROWS;
  const uint32_t b = ptx::smem_u32(&bar);
  if (threadIdx.x == 0) {
    ptx::mbar_init(b, 1);
    ptx::fence_mbar_init();
    ptx::mbar_arrive_expect_tx(b, (uint32_t)nbox * 16384u);
    for (int i = 0; i < nbox; ++i) ptx::tma_load_2d(ptx::smem_u32(s_w + i * 16384), &tmap_w, b, i * 64, h * D_c + d0);
  }
  const int rp = threadIdx.x & 63, tg = threadIdx.x >> 6;
  const int ra = rp, rb = rp + 64;
  const int da = d0 + ra, db = d0 + rb;
  bool landed = false, ok = true;
  for (int tb0 = 0; tb0 < rows_per_head; tb0 += PA_TB) {
    const int nr = min(PA_TB, rows_per_head - tb0);
    __syncthreads();                                 // barrier init seen; s_q free
    // element-wise: a few loads per thread already fit one round trip, and
    // the 16-byte form costs registers that this kernel's FMAs need
    stage_rows(s_q, q_nope, q_dtype, q_stride, tb0, nr, H, h, D_n, P_THREADS);
    __syncthreads();
    if (!landed) {
      ok = wait_landed(b);
      landed = true;
    }
    float2 acc[4][2];
#pragma unroll
    for (int i = 0; i < 4; ++i) acc[i][0] = acc[i][1] = make_float2(0.f, 0.f);
    const int nchunk = D_n / 8;
    for (int c = 0; c < nchunk; ++c) {
      const unsigned char* box = s_w + (c >> 3) * 16384;
      const int cc = c & 7;
      const uint4 wa = *reinterpret_cast<const uint4*>(box + ra * 128 + ((cc ^ (ra & 7)) << 4));
      const uint4 wb = *reinterpret_cast<const uint4*>(box + rb * 128 + ((cc ^ (rb & 7)) << 4));
      const float2 fa[4] = {bf16x2_to_float2(wa.x), bf16x2_to_float2(wa.y), bf16x2_to_float2(wa.z),
                            bf16x2_to_float2(wa.w)};
      const float2 fb[4] = {bf16x2_to_float2(wb.x), bf16x2_to_float2(wb.y), bf16x2_to_float2(wb.z),
                            bf16x2_to_float2(wb.w)};
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        const int t = tg + 4 * i;
        if (t < nr) {                                // uniform over the warp
          const float4 q0 = *reinterpret_cast<const float4*>(s_q + t * D_n + 8 * c);
          const float4 q1 = *reinterpret_cast<const float4*>(s_q + t * D_n + 8 * c + 4);
          const float2 p[4] = {make_float2(q0.x, q0.y), make_float2(q0.z, q0.w), make_float2(q1.x, q1.y),
                               make_float2(q1.z, q1.w)};
#pragma unroll
          for (int j = 0; j < 4; ++j) {
            acc[i][0] = __ffma2_rn(fa[j], p[j], acc[i][0]);
            acc[i][1] = __ffma2_rn(fb[j], p[j], acc[i][1]);
          }
        }
      }
    }
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      const int t = tg + 4 * i;
      if (t < nr) {
        const int64_t row = (int64_t)(tb0 + t) * H + h;
        if (da < D_c) st_elem(q_lat, row * o_stride + da, o_dtype, ok ? acc[i][0].x + acc[i][0].y : __int_as_float(0x7fc00000));
        if (db < D_c) st_elem(q_lat, row * o_stride + db, o_dtype, ok ? acc[i][1].x + acc[i][1].y : __int_as_float(0x7fc00000));
      }
    }
  }
}

// out[row][v] = sum_d W_UV[h][d][v] o_lat[row][d]. CTA = (32 columns of head
// h); its W_UV slice [D_c rows][32 v] arrives as TMA boxes of [256 rows][32 v]
// (64-byte rows, no swizzle). Thread (q = v quad, g = d phase, tg = node
// group) accumulates columns 4q..4q+3 for nodes tg, tg+4, tg+8, tg+12 over
// d = g, g+8, g+16, ...; a warp is 8 quads x 4 consecutive phases, so its
// weight reads cover 256 contiguous bytes and its node reads 4 words. Node
// rows are staged duplicated ((o, o) pairs) so one 8-byte read gives the
// packed-FMA operand. The 8 phases' partial sums are added in shared memory.
__global__ void __launch_bounds__(P_THREADS)
unabsorb_o_tma_kernel(const __grid_constant__ CUtensorMap tmap_w, int32_t rows_per_head, int32_t H, int32_t D_c,
                      int32_t D_v, const float* __restrict__ o_lat, int64_t i_stride, int o_vec,
                      void* __restrict__ out, int64_t o_stride, int o_dtype) {
  extern __shared__ unsigned char smem_raw[];
  __shared__ __align__(8) unsigned long long bar;
  unsigned char* s_w = align1024(smem_raw);                   // [D_c padded to 256][32] bf16
  const int nbox = (D_c + 255) / 256;
  float2* s_o = reinterpret_cast<float2*>(s_w + nbox * 256 * PU_V * 2);   // [PU_TB][D_c] (o, o)
  float* s_part = reinterpret_cast<float*>(s_o);                          // reused: [PU_DG][PU_TB][PU_V]
  const int h = blockIdx.y, v0 = blockIdx.x * PU_V;
  const uint32_t b = ptx::smem_u32(&bar);
  if (threadIdx.x == 0) {
    ptx::mbar_init(b, 1);
    ptx::fence_mbar_init();
    ptx::mbar_arrive_expect_tx(b, (uint32_t)nbox * 256u * PU_V * 2u);
    for (int i = 0; i < nbox; ++i)
      ptx::tma_load_2d(ptx::smem_u32(s_w + i * 256 * PU_V * 2), &tmap_w, b, v0, h * D_c + i * 256);
  }
  const int lane = threadIdx.x & 31, w = threadIdx.x >> 5;
  const int q = lane & 7;                                     // columns 4q .. 4q+3
  const int g = (lane >> 3) + 4 * (w & 1);                    // d phase 0..7
  const int tg = w >> 1;                                      // node group 0..3
  bool landed = false, ok = true;
  for (int tb0 = 0; tb0 < rows_per_head; tb0 += PU_TB) {
    const int nr = min(PU_TB, rows_per_head - tb0);
    __syncthreads();                                          // barrier init seen; s_o / s_part free
    if (o_vec) {
      stage_rows_vec<true>(s_o, o_lat, KDV_F32, i_stride, tb0, nr, H, h, D_c);
    } else {
      for (int i = threadIdx.x; i < nr * D_c; i += P_THREADS) {
        const int r = i / D_c, d = i - r * D_c;
        const float x = o_lat[((int64_t)(tb0 + r) * H + h) * i_stride + d];
        s_o[r * D_c + d] = make_float2(x, x);
      }
    }
    __syncthreads();
    if (!landed) {
      ok = wait_landed(b);
      landed = true;
    }
    float2 acc[4][2];
#pragma unroll
    for (int i = 0; i < 4; ++i) acc[i][0] = acc[i][1] = make_float2(0.f, 0.f);
    for (int d = g; d < D_c; d += PU_DG) {
      const uint2 wv = *reinterpret_cast<const uint2*>(s_w + d * (PU_V * 2) + q * 8);
      const float2 f0 = bf16x2_to_float2(wv.x), f1 = bf16x2_to_float2(wv.y);
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        const int t = tg + 4 * i;
        if (t < nr) {                                         // uniform over the warp
          const float2 o2 = s_o[t * D_c + d];
          acc[i][0] = __ffma2_rn(f0, o2, acc[i][0]);
          acc[i][1] = __ffma2_rn(f1, o2, acc[i][1]);
        }
      }
    }
    __syncthreads();                                          // every read of s_o done
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      const int t = tg + 4 * i;
      if (t < nr) {
        float* dst = s_part + (g * PU_TB + t) * PU_V + 4 * q;
        *reinterpret_cast<float4*>(dst) = make_float4(acc[i][0].x, acc[i][0].y, acc[i][1].x, acc[i][1].y);
      }
    }
    __syncthreads();
    for (int i = threadIdx.x; i < nr * PU_V; i += P_THREADS) {
      const int t = i / PU_V, col = i - t * PU_V, v = v0 + col;
      float sum = 0.f;
#pragma unroll
      for (int gg = 0; gg < PU_DG; ++gg) sum += s_part[(gg * PU_TB + t) * PU_V + col];
      if (v < D_v)
        st_elem(out, ((int64_t)(tb0 + t) * H + h) * o_stride + v, o_dtype, ok ? sum : __int_as_float(0x7fc00000));
    }
  }
}

typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                                  const cuuint64_t*, const cuuint32_t*, const cuuint32_t*,
                                  CUtensorMapInterleave, CUtensorMapSwizzle, CUtensorMapL2promotion,
                                  CUtensorMapFloatOOBfill);

EncodeTiledFn encode_fn() {
  static EncodeTiledFn fn = nullptr;
  if (fn == nullptr) {
    void* ptr = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &ptr, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<EncodeTiledFn>(ptr);
  }
  return fn;
}

// bf16 weights [rows][cols] (row pitch = cols) as a 2D tensor map with boxes
// of [box_rows][box_cols]; false if the driver refuses it.
bool weight_map(CUtensorMap* m, const void* w, uint64_t rows, uint64_t cols, uint32_t box_cols, uint32_t box_rows,
                CUtensorMapSwizzle swz) {
  EncodeTiledFn enc = encode_fn();
  if (enc == nullptr) return false;
  const cuuint64_t dims[2] = {(cuuint64_t)cols, (cuuint64_t)rows};
  const cuuint64_t strides[1] = {(cuuint64_t)cols * 2};
  const cuuint32_t box[2] = {box_cols, box_rows};
  const cuuint32_t estr[2] = {1, 1};
  return enc(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(w), dims, strides, box, estr,
             CU_TENSOR_MAP_INTERLEAVE_NONE, swz, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
             CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

size_t absorb_tma_smem(int D_n) { return 1024 + (size_t)((D_n + 63) / 64) * 16384 + (size_t)PA_TB * D_n * 4; }
size_t unabsorb_tma_smem(int D_c) {
  const size_t part = (size_t)PU_DG * PU_TB * PU_V * 4, o = (size_t)PU_TB * D_c * 8;
  return 1024 + (size_t)((D_c + 255) / 256) * 256 * PU_V * 2 + (o > part ? o : part);
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

kdv_status kdv_absorb_q_ex(int32_t rows, int32_t num_heads, int32_t d_latent, int32_t d_nope, const void* q_nope,
                           int64_t q_nope_stride, int32_t q_dtype, const void* w_uk, int32_t w_dtype, void* q_lat,
                           int64_t q_lat_stride, int32_t out_dtype, uint32_t flags, void* stream) {
  if ((flags & ~KDV_PROJ_STATIC_WEIGHTS) != 0) return KDV_ERR_INVALID_ARG;
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
            cudaSuccess ||
        cudaFuncSetAttribute(absorb_q_tma_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             (int)absorb_tma_smem(512)) != cudaSuccess)
      return KDV_ERR_CUDA;
    attr_set[dev] = true;
  }
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  CUtensorMap tmap;
  // tensor cores: bf16 weights and q_nope, whole 128-row weight tiles,
  // 64-dim K-blocks, 16-byte aligned rows
  if (vec && q_dtype == KDV_BF16 && d_latent % 128 == 0 && d_nope % 64 == 0 && d_nope <= 256 &&
      q_nope_stride % 8 == 0 && (reinterpret_cast<uintptr_t>(q_nope) & 15) == 0 &&
      (int64_t)num_heads * d_latent <= 0x7fffffff &&
      weight_map(&tmap, w_uk, (uint64_t)num_heads * d_latent, (uint64_t)d_nope, 64, 128,
                 CU_TENSOR_MAP_SWIZZLE_128B))
    return launch_absorb_q_tc(tmap, rows, num_heads, d_latent, d_nope, q_nope, q_nope_stride, q_lat, q_lat_stride,
                              out_dtype, (flags & KDV_PROJ_STATIC_WEIGHTS) != 0, s) == cudaSuccess ? KDV_OK
                                                                                                  : KDV_ERR_CUDA;
  if (vec && (int64_t)num_heads * d_latent <= 0x7fffffff &&
      weight_map(&tmap, w_uk, (uint64_t)num_heads * d_latent, (uint64_t)d_nope, 64, PA_ROWS,
                 CU_TENSOR_MAP_SWIZZLE_128B)) {
    const dim3 g2((unsigned)((d_latent + PA_ROWS - 1) / PA_ROWS), (unsigned)num_heads);
    absorb_q_tma_kernel<<<g2, P_THREADS, absorb_tma_smem(d_nope), s>>>(
        tmap, rows / num_heads, num_heads, d_latent, d_nope, q_nope, q_nope_stride, q_dtype, q_lat, q_lat_stride,
        out_dtype);
    return cudaGetLastError() == cudaSuccess ? KDV_OK : KDV_ERR_CUDA;
  }
  const dim3 grid((unsigned)num_heads, (unsigned)((d_latent + THREADS - 1) / THREADS));
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

kdv_status kdv_absorb_q(int32_t rows, int32_t num_heads, int32_t d_latent, int32_t d_nope, const void* q_nope,
                        int64_t q_nope_stride, int32_t q_dtype, const void* w_uk, int32_t w_dtype, void* q_lat,
                        int64_t q_lat_stride, int32_t out_dtype, void* stream) {
  return kdv_absorb_q_ex(rows, num_heads, d_latent, d_nope, q_nope, q_nope_stride, q_dtype, w_uk, w_dtype, q_lat,
                         q_lat_stride, out_dtype, 0u, stream);
}

kdv_status kdv_unabsorb_o_ex(int32_t rows, int32_t num_heads, int32_t d_latent, int32_t d_v, const float* o_lat,
                             int64_t o_lat_stride, const void* w_uv, int32_t w_dtype, void* out, int64_t out_stride,
                             int32_t out_dtype, uint32_t flags, void* stream) {
  if ((flags & ~KDV_PROJ_STATIC_WEIGHTS) != 0) return KDV_ERR_INVALID_ARG;
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
            cudaSuccess ||
        cudaFuncSetAttribute(unabsorb_o_tma_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             (int)unabsorb_tma_smem(PU_MAX_DC)) != cudaSuccess)
      return KDV_ERR_CUDA;
    attr_set[dev] = true;
  }
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  CUtensorMap tmap;
  // tensor cores: bf16 weights, 128-column output tiles, 64-row K-blocks,
  // 16-byte aligned o_lat rows
  if (w_dtype == KDV_BF16 && d_v % 128 == 0 && d_latent % 64 == 0 && d_latent <= PU_MAX_DC &&
      (reinterpret_cast<uintptr_t>(w_uv) & 15) == 0 && (reinterpret_cast<uintptr_t>(o_lat) & 15) == 0 &&
      o_lat_stride % 4 == 0 && (int64_t)num_heads * d_latent <= 0x7fffffff &&
      weight_map(&tmap, w_uv, (uint64_t)num_heads * d_latent, (uint64_t)d_v, 64, 64, CU_TENSOR_MAP_SWIZZLE_128B))
    return launch_unabsorb_o_tc(tmap, rows, num_heads, d_latent, d_v, o_lat, o_lat_stride, out, out_stride, out_dtype,
                                (flags & KDV_PROJ_STATIC_WEIGHTS) != 0, s) == cudaSuccess ? KDV_OK : KDV_ERR_CUDA;
  if (w_dtype == KDV_BF16 && d_v % 8 == 0 && d_latent <= PU_MAX_DC &&
      (reinterpret_cast<uintptr_t>(w_uv) & 15) == 0 && (int64_t)num_heads * d_latent <= 0x7fffffff &&
      weight_map(&tmap, w_uv, (uint64_t)num_heads * d_latent, (uint64_t)d_v, PU_V, 256,
                 CU_TENSOR_MAP_SWIZZLE_NONE)) {
    const dim3 g2((unsigned)((d_v + PU_V - 1) / PU_V), (unsigned)num_heads);
    unabsorb_o_tma_kernel<<<g2, P_THREADS, unabsorb_tma_smem(d_latent), s>>>(
        tmap, rows / num_heads, num_heads, d_latent, d_v, o_lat, o_lat_stride,
        (reinterpret_cast<uintptr_t>(o_lat) & 15) == 0 && o_lat_stride % 8 == 0 && d_latent % 8 == 0 ? 1 : 0, out,
        out_stride, out_dtype);
    return cudaGetLastError() == cudaSuccess ? KDV_OK : KDV_ERR_CUDA;
  }
  const dim3 grid((unsigned)num_heads, (unsigned)((d_v + U_VB - 1) / U_VB));
  if (w_dtype == KDV_BF16)
    unabsorb_o_kernel<true><<<grid, U_THREADS, smem, s>>>(rows / num_heads, num_heads, d_latent, d_v, o_lat,
                                                          o_lat_stride, w_uv, w_dtype, out, out_stride, out_dtype);
  else
    unabsorb_o_kernel<false><<<grid, U_THREADS, smem, s>>>(rows / num_heads, num_heads, d_latent, d_v, o_lat,
                                                           o_lat_stride, w_uv, w_dtype, out, out_stride, out_dtype);
  return cudaGetLastError() == cudaSuccess ? KDV_OK : KDV_ERR_CUDA;
}

kdv_status kdv_unabsorb_o(int32_t rows, int32_t num_heads, int32_t d_latent, int32_t d_v, const float* o_lat,
                          int64_t o_lat_stride, const void* w_uv, int32_t w_dtype, void* out, int64_t out_stride,
                          int32_t out_dtype, void* stream) {
  return kdv_unabsorb_o_ex(rows, num_heads, d_latent, d_v, o_lat, o_lat_stride, w_uv, w_dtype, out, out_stride,
                           out_dtype, 0u, stream);
}

}  // extern "C"

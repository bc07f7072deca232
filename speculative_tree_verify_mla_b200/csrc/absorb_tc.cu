// absorb_tc.cu -- the two per-head projections around absorbed-form attention
// on the tensor cores (tcgen05.mma, TMEM accumulator, TMA-staged weights).
//
// The latent projection that the verify kernel absorbs (page "The
// Architecture of Diagnosis", section "Phase 1: Custom CUDA Kernels", item 2)
// leaves two small products per head h, with rows node-major (row = t*H+h):
//   q_lat[t,h] = W_UK[h] q_nope[t,h]      W_UK[h]: D_c x D_n, row-major
//   out[t,h]   = W_UV[h]^T o_lat[t,h]     W_UV[h]: D_c x D_v, row-major
// Both stream every weight once per call and do about 2*T flops per weight,
// so they are bound by HBM reading the weights; these kernels keep that
// stream going and leave the arithmetic to one MMA chain per CTA.
//
// Each CTA computes a 128-row slice of one head's output for all of that
// head's nodes, transposed: D[128 outputs][N nodes] = A[128][K] . B[N][K]^T
// with M = 128, N = the nodes of a pass rounded up to 16, in fp32 TMEM.
//   absorb:   A = 128 rows of W_UK[h] (K = D_n, K-major, TMA boxes of
//             [128 rows][64 k], 128-byte swizzle); B = the head's q_nope rows,
//             staged by the threads in the same K-major swizzled layout.
//   unabsorb: A = W_UV[h]^T, i.e. W_UV[h] read with v contiguous (MN-major):
//             TMA boxes of [64 c][64 v]; B = the head's o_lat rows (fp32)
//             split into bf16 hi = rn(o) and lo = rn(o - hi), stacked as
//             B rows [hi of the pass's nodes; lo of them], one MMA of twice
//             the nodes per K-step and the two column halves added in the
//             epilogue, so B carries ~16 significant bits and the product
//             stays at fp32-accumulation accuracy (W_UV is exact in bf16).
// The epilogue reads D with one TMEM lane per output row and one column per
// node, so a warp's stores for one node cover 32 consecutive outputs.
//
// Every wait is bounded (2 s); a CTA whose weights or MMAs never complete
// writes NaN to its outputs instead of waiting forever (these entry points
// take no device error flag).
//
// Launched as a programmatic dependent (the caller's "static weights" flag),
// a CTA starts its weight copy before the preceding kernel on the stream has
// finished and waits for that kernel (griddepcontrol.wait) only before it
// reads q_nope / o_lat or writes anything; launched normally the wait is a
// no-op. Each CTA also lets the next such launch begin at once.
#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include "kdv.h"
#include "sm100_ptx.cuh"

namespace kdv {
namespace {

using namespace ptx;

constexpr int TC_THREADS = 128;
constexpr int A_MAXN = 64;                 // absorb: nodes per pass
constexpr int U_MAXN = 32;                 // unabsorb: nodes per pass (hi + lo staging)
constexpr int BOX = 16384;                 // 128 x 128-byte rows
constexpr unsigned long long TC_WAIT_NS = 2000000000ull;

__device__ __forceinline__ unsigned long long tc_gtimer() {
  unsigned long long t;
  asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
  return t;
}
__device__ __forceinline__ bool tc_wait(uint32_t bar, uint32_t parity) {
  if (mbar_try_wait(bar, parity)) return true;
  const unsigned long long t0 = tc_gtimer();
  while (!mbar_try_wait(bar, parity))
    if (tc_gtimer() - t0 > TC_WAIT_NS) return false;
  return true;
}
__device__ __forceinline__ uint32_t align_1024(uint32_t a) { return (a + 1023u) & ~1023u; }
__device__ __forceinline__ uint32_t tmem_cols_for(int n) { return n <= 32 ? 32u : n <= 64 ? 64u : n <= 128 ? 128u : 256u; }

// Store column j of this thread's TMEM lane (row d of the slice) for node t.
__device__ __forceinline__ void store_out(void* out, int64_t idx, int dtype, float v) {
  if (dtype == KDV_BF16) static_cast<__nv_bfloat16*>(out)[idx] = __float2bfloat16_rn(v);
  else static_cast<float*>(out)[idx] = v;
}

// Read D (this warp's 32 lanes, columns [0, n)) and write node t's value to
// out[(t0 + t) * H + h][col0 + lane row]; with lo_col > 0, node t's value is
// the sum of columns t and lo_col + t.
__device__ __forceinline__ void epilogue(uint32_t tmem, int n, bool ok, void* out, int64_t o_stride, int o_dtype,
                                         int t0, int H, int h, int col0, int lo_col = 0) {
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const uint32_t lane_base = (uint32_t)(warp * 32) << 16;
  for (int c0 = 0; c0 < n; c0 += 32) {
    uint32_t v[32];
    tmem_ld32(tmem + lane_base + (uint32_t)c0, v);
    if (lo_col > 0) {
      uint32_t w[32];
      tmem_ld32(tmem + lane_base + (uint32_t)(lo_col + c0), w);
      tmem_wait_ld();
#pragma unroll
      for (int j = 0; j < 32; ++j) v[j] = __float_as_uint(__uint_as_float(v[j]) + __uint_as_float(w[j]));
    }
    tmem_wait_ld();
#pragma unroll
    for (int j = 0; j < 32; ++j) {
      const int t = c0 + j;
      if (t < n) {
        const int64_t row = (int64_t)(t0 + t) * H + h;
        store_out(out, row * o_stride + col0 + warp * 32 + lane, o_dtype,
                  ok ? __uint_as_float(v[j]) : __int_as_float(0x7fc00000));
      }
    }
  }
}

// q_lat = W_UK[h] q_nope. Grid (D_c / 128, H); D_n a multiple of 64, <= 256;
// q_nope bf16 with 16-byte aligned rows.
__global__ void __launch_bounds__(TC_THREADS)
absorb_q_tc_kernel(const __grid_constant__ CUtensorMap tmap_w, int32_t rows_per_head, int32_t H, int32_t D_c,
                   int32_t D_n, const __nv_bfloat16* __restrict__ q_nope, int64_t q_stride,
                   void* __restrict__ q_lat, int64_t o_stride, int o_dtype) {
  extern __shared__ unsigned char smem_raw[];
  __shared__ __align__(8) unsigned long long bars[2];
  __shared__ uint32_t tmem_slot;
  const uint32_t base = align_1024(smem_u32(smem_raw));
  const int nkb = D_n / 64;
  const uint32_t s_a = base;                       // nkb x [128 rows][64 k]
  const uint32_t s_b = base + nkb * BOX;           // nkb x [A_MAXN rows][64 k]
  const int h = blockIdx.y, d0 = blockIdx.x * 128;
  const int warp = threadIdx.x >> 5;
  const uint32_t full = smem_u32(&bars[0]), done = smem_u32(&bars[1]);
  if (threadIdx.x == 0) {
    mbar_init(full, 1);
    mbar_init(done, 1);
    fence_mbar_init();
    mbar_arrive_expect_tx(full, (uint32_t)nkb * BOX);
    for (int kb = 0; kb < nkb; ++kb) tma_load_2d(s_a + kb * BOX, &tmap_w, full, kb * 64, h * D_c + d0);
  }
  if (warp == 0) {
    tmem_alloc(smem_u32(&tmem_slot), tmem_cols_for(A_MAXN));
    tmem_relinquish();
  }
  if (threadIdx.x == 0) asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
  asm volatile("griddepcontrol.wait;" ::: "memory");
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = tmem_slot;
  bool ok = true;
  int pass = 0;
  for (int t0 = 0; t0 < rows_per_head; t0 += A_MAXN, ++pass) {
    const int n = min(A_MAXN, rows_per_head - t0), npad = (n + 15) & ~15;
    // B: node t's D_n dims as nkb swizzled rows of 128 bytes (zeros past
    // n); four items' loads go out before any (ordered) shared store
    const int total = npad * nkb * 8;
    for (int i0 = threadIdx.x; i0 < total; i0 += 4 * TC_THREADS) {
      uint4 v[4];
#pragma unroll
      for (int u = 0; u < 4; ++u) {
        const int i = i0 + u * TC_THREADS;
        const int ch = i & 7, kb = (i >> 3) % nkb, t = (i >> 3) / nkb;
        v[u] = make_uint4(0u, 0u, 0u, 0u);
        if (i < total && t < n)
          v[u] = *reinterpret_cast<const uint4*>(q_nope + ((int64_t)(t0 + t) * H + h) * q_stride + kb * 64 + ch * 8);
      }
#pragma unroll
      for (int u = 0; u < 4; ++u) {
        const int i = i0 + u * TC_THREADS;
        if (i >= total) break;
        const int ch = i & 7, kb = (i >> 3) % nkb, t = (i >> 3) / nkb;
        st_shared_v4(s_b + kb * (A_MAXN * 128) + t * 128 + ((ch ^ (t & 7)) << 4), v[u].x, v[u].y, v[u].z, v[u].w);
      }
    }
    fence_proxy_async_smem();
    __syncthreads();
    if (threadIdx.x == 0) {
      if (pass == 0) ok = tc_wait(full, 0);
      tc_fence_after();
      if (ok) {
        const uint32_t idesc = idesc_bf16_f32(128, npad, false, false);
        for (int kb = 0; kb < nkb; ++kb)
#pragma unroll
          for (int kk = 0; kk < 4; ++kk)
            mma_ss(tmem, sw128_desc(s_a + kb * BOX + kk * 32, 16, 1024),
                   sw128_desc(s_b + kb * (A_MAXN * 128) + kk * 32, 16, 1024), idesc, (kb > 0 || kk > 0) ? 1u : 0u);
      }
      tc_commit(done);
    }
    const bool landed = tc_wait(done, pass & 1);
    ok = __syncthreads_and(ok && landed) != 0;
    tc_fence_after();
    epilogue(tmem, n, ok, q_lat, o_stride, o_dtype, t0, H, h, d0);
    tc_fence_before();
    __syncthreads();                               // D and B free for the next pass
  }
  if (threadIdx.x == 0 && rows_per_head > 0 && !ok) tc_wait(full, 0);   // retire the weight copy
  if (warp == 0) {
    tc_fence_after();
    tmem_dealloc(tmem, tmem_cols_for(A_MAXN));
  }
}

// out = W_UV[h]^T o_lat. Grid (D_v / 128, H); D_c a multiple of 64, <= 512;
// o_lat fp32 with 16-byte aligned rows.
__global__ void __launch_bounds__(TC_THREADS)
unabsorb_o_tc_kernel(const __grid_constant__ CUtensorMap tmap_w, int32_t rows_per_head, int32_t H, int32_t D_c,
                     int32_t D_v, const float* __restrict__ o_lat, int64_t i_stride, void* __restrict__ out,
                     int64_t o_stride, int o_dtype) {
  extern __shared__ unsigned char smem_raw[];
  __shared__ __align__(8) unsigned long long bars[2];
  __shared__ uint32_t tmem_slot;
  const uint32_t base = align_1024(smem_u32(smem_raw));
  const int ncb = D_c / 64;
  constexpr int BB = 2 * U_MAXN * 128;             // one 64-c block of B: hi rows, then lo rows
  const uint32_t s_a = base;                       // ncb x ([64 c][64 v] x 2 v-blocks)
  const uint32_t s_b = base + ncb * BOX;           // ncb x [2 npad rows][64 c]
  const int h = blockIdx.y, v0 = blockIdx.x * 128;
  const int warp = threadIdx.x >> 5;
  const uint32_t full = smem_u32(&bars[0]), done = smem_u32(&bars[1]);
  if (threadIdx.x == 0) {
    mbar_init(full, 1);
    mbar_init(done, 1);
    fence_mbar_init();
    mbar_arrive_expect_tx(full, (uint32_t)ncb * BOX);
    for (int cb = 0; cb < ncb; ++cb)
      for (int vb = 0; vb < 2; ++vb)
        tma_load_2d(s_a + cb * BOX + vb * (BOX / 2), &tmap_w, full, v0 + vb * 64, h * D_c + cb * 64);
  }
  if (warp == 0) {
    tmem_alloc(smem_u32(&tmem_slot), tmem_cols_for(2 * U_MAXN));
    tmem_relinquish();
  }
  if (threadIdx.x == 0) asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
  asm volatile("griddepcontrol.wait;" ::: "memory");
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = tmem_slot;
  bool ok = true;
  int pass = 0;
  for (int t0 = 0; t0 < rows_per_head; t0 += U_MAXN, ++pass) {
    const int n = min(U_MAXN, rows_per_head - t0), npad = (n + 15) & ~15;
    // B: node t's D_c values as bf16 hi and lo parts, swizzled 128-byte
    // rows. Eight items' loads go out before any store (the shared stores
    // are ordered asm, so a load after one would wait for it).
    const int total = npad * ncb * 8;
    for (int i0 = threadIdx.x; i0 < total; i0 += 8 * TC_THREADS) {
      float4 xa[8], xb[8];
#pragma unroll
      for (int u = 0; u < 8; ++u) {
        const int i = i0 + u * TC_THREADS;
        const int ch = i & 7, cb = (i >> 3) % ncb, t = (i >> 3) / ncb;
        xa[u] = xb[u] = make_float4(0.f, 0.f, 0.f, 0.f);
        if (i < total && t < n) {
          const float* src = o_lat + ((int64_t)(t0 + t) * H + h) * i_stride + cb * 64 + ch * 8;
          xa[u] = *reinterpret_cast<const float4*>(src);
          xb[u] = *reinterpret_cast<const float4*>(src + 4);
        }
      }
#pragma unroll
      for (int u = 0; u < 8; ++u) {
        const int i = i0 + u * TC_THREADS;
        if (i >= total) break;
        const int ch = i & 7, cb = (i >> 3) % ncb, t = (i >> 3) / ncb;
        const float x[8] = {xa[u].x, xa[u].y, xa[u].z, xa[u].w, xb[u].x, xb[u].y, xb[u].z, xb[u].w};
        uint32_t hi[4], lo[4];
#pragma unroll
        for (int j = 0; j < 4; ++j) {
          const __nv_bfloat16 h0 = __float2bfloat16_rn(x[2 * j]), h1 = __float2bfloat16_rn(x[2 * j + 1]);
          const __nv_bfloat16 l0 = __float2bfloat16_rn(x[2 * j] - __bfloat162float(h0));
          const __nv_bfloat16 l1 = __float2bfloat16_rn(x[2 * j + 1] - __bfloat162float(h1));
          hi[j] = (uint32_t)__bfloat16_as_ushort(h0) | ((uint32_t)__bfloat16_as_ushort(h1) << 16);
          lo[j] = (uint32_t)__bfloat16_as_ushort(l0) | ((uint32_t)__bfloat16_as_ushort(l1) << 16);
        }
        const int tl = npad + t;                    // the lo row of node t
        st_shared_v4(s_b + cb * BB + t * 128 + ((ch ^ (t & 7)) << 4), hi[0], hi[1], hi[2], hi[3]);
        st_shared_v4(s_b + cb * BB + tl * 128 + ((ch ^ (tl & 7)) << 4), lo[0], lo[1], lo[2], lo[3]);
      }
    }
    fence_proxy_async_smem();
    __syncthreads();
    if (threadIdx.x == 0) {
      if (pass == 0) ok = tc_wait(full, 0);
      tc_fence_after();
      if (ok) {
        // A MN-major: 64-v blocks BOX/2 apart, 8-row (c) groups 1024 B apart,
        // 16 c per K-step = 2048 B
        const uint32_t idesc = idesc_bf16_f32(128, 2 * npad, true, false);
        for (int cb = 0; cb < ncb; ++cb)
#pragma unroll
          for (int kk = 0; kk < 4; ++kk) {
            const uint64_t adesc = sw128_desc(s_a + cb * BOX + kk * 2048, BOX / 2, 1024);
            mma_ss(tmem, adesc, sw128_desc(s_b + cb * BB + kk * 32, 16, 1024), idesc, (cb > 0 || kk > 0) ? 1u : 0u);
          }
      }
      tc_commit(done);
    }
    const bool landed = tc_wait(done, pass & 1);
    ok = __syncthreads_and(ok && landed) != 0;
    tc_fence_after();
    epilogue(tmem, n, ok, out, o_stride, o_dtype, t0, H, h, v0, npad);
    tc_fence_before();
    __syncthreads();
  }
  if (threadIdx.x == 0 && rows_per_head > 0 && !ok) tc_wait(full, 0);
  if (warp == 0) {
    tc_fence_after();
    tmem_dealloc(tmem, tmem_cols_for(2 * U_MAXN));
  }
}

}  // namespace

size_t absorb_tc_smem(int D_n) { return 1024 + (size_t)(D_n / 64) * (BOX + A_MAXN * 128); }
size_t unabsorb_tc_smem(int D_c) { return 1024 + (size_t)(D_c / 64) * (BOX + 2 * U_MAXN * 128); }

// Launch `kernel` with the programmatic-dependent attribute when `early`.
template <typename... Args>
static cudaError_t launch_maybe_early(bool early, void (*kernel)(Args...), dim3 grid, size_t smem, cudaStream_t s,
                                      Args... args) {
  if (!early) {
    kernel<<<grid, TC_THREADS, smem, s>>>(args...);
    return cudaGetLastError();
  }
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = dim3(TC_THREADS);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = s;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, kernel, args...);
}

cudaError_t launch_absorb_q_tc(const CUtensorMap& tmap, int32_t rows, int32_t H, int32_t D_c, int32_t D_n,
                               const void* q_nope, int64_t q_stride, void* q_lat, int64_t o_stride, int32_t o_dtype,
                               bool early_weights, cudaStream_t s) {
  static bool attr_set[64] = {};
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  if (dev >= 0 && dev < 64 && !attr_set[dev]) {
    e = cudaFuncSetAttribute(absorb_q_tc_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)absorb_tc_smem(256));
    if (e != cudaSuccess) return e;
    attr_set[dev] = true;
  }
  const dim3 grid((unsigned)(D_c / 128), (unsigned)H);
  return launch_maybe_early(early_weights, absorb_q_tc_kernel, grid, absorb_tc_smem(D_n), s, tmap, rows / H, H, D_c,
                            D_n, static_cast<const __nv_bfloat16*>(q_nope), q_stride, q_lat, o_stride, (int)o_dtype);
}

cudaError_t launch_unabsorb_o_tc(const CUtensorMap& tmap, int32_t rows, int32_t H, int32_t D_c, int32_t D_v,
                                 const float* o_lat, int64_t i_stride, void* out, int64_t o_stride, int32_t o_dtype,
                                 bool early_weights, cudaStream_t s) {
  static bool attr_set[64] = {};
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  if (dev >= 0 && dev < 64 && !attr_set[dev]) {
    e = cudaFuncSetAttribute(unabsorb_o_tc_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             (int)unabsorb_tc_smem(512));
    if (e != cudaSuccess) return e;
    attr_set[dev] = true;
  }
  const dim3 grid((unsigned)(D_v / 128), (unsigned)H);
  return launch_maybe_early(early_weights, unabsorb_o_tc_kernel, grid, unabsorb_tc_smem(D_c), s, tmap, rows / H, H,
                            D_c, D_v, o_lat, i_stride, out, o_stride, (int)o_dtype);
}

}  // namespace kdv

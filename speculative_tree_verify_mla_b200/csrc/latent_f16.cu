// latent_f16.cu -- the fp16 copy of the latent rows that the tensor-core
// kernel's P.V reads.
//
// The tensor-core verify kernel rounds the softmax numerators P to fp16 before
// P.V (in bf16 their rounding alone would cost ~1e-3 of the output's RMS), and
// a kind::f16 MMA needs V in the same type. Converting V inside the kernel is
// not an option on this part: while the tensor core streams shared memory,
// the load/store unit gets only ~5-10 B/clk of it, so a 16 KB stage read back
// through registers takes over a microsecond. This kernel therefore writes,
// before the verify launch, the c_kv part of every key the call will read --
// request b's logical keys 0 .. L_b+T_b-1, through the page table when there
// is one -- as fp16 rows [512] in logical order into the workspace, where the
// verify kernel's P.V side reads them with tiled TMA boxes. bf16 -> fp16 is
// exact for 2^-14 <= |x| < 65536; smaller values round to fp16 subnormals;
// |x| >= 65536 (or inf / NaN) is reported as KDV_DERR_RANGE.
//
// A paged pool can also be staged in the same pass: with `staged` given,
// the row's k_rope (D_r = 64 bf16, 128 bytes) is copied to staged row
// v16_base[b] + j, staged_off[b] = v16_base[b], and q_lat is written as fp16
// to q16 [total_rows][512]. The verify kernel then reads the request's keys
// with tiled TMA boxes instead of gathers: their latent dims from the fp16
// rows (Q.K^T over them in fp16: the same products as bf16 except where an
// input below 2^-14 in magnitude was rounded to an fp16 subnormal), their
// rope dims from the staged rows.
//
// HBM-bound: 1 KB read and 1 KB written per key; staging adds 128 B read and
// written per key (k_rope) and 1 KB read and written per query row (q_lat).
// One warp per key row, lane l owning dims [16 l, 16 l + 16) (and, for lanes
// 0-7, k_rope bytes [16 l, 16 l + 16)); each warp keeps four rows' loads in
// flight. The query rows follow, one warp per row over the whole grid.
#include <cuda_fp16.h>

#include "kdv_internal.cuh"
#include "sm100_ptx.cuh"

namespace kdv {
namespace {

constexpr int LF_THREADS = 256;
constexpr int LF_ROWS = 4;           // rows in flight per warp

// STAGED: staged, staged_off and q16 are given (a paged pool staged in this
// pass); otherwise all three are null and their code is compiled out
template <bool STAGED>
__global__ void __launch_bounds__(LF_THREADS)
latent_f16_kernel(const VerifyArgs a, const VerifyPlan p, __half* __restrict__ v16, uint8_t* __restrict__ staged,
                  int32_t* __restrict__ staged_off, __half* __restrict__ q16) {
  const int b = blockIdx.y;
  // Launched as a programmatic dependent of whatever kernel precedes it on
  // the stream (which may have written the pool or the page table): wait for
  // it before any access. Then let the attention grid launch: it reads the
  // fp16 rows only after this grid completes (griddepcontrol.wait), and
  // everything else it reads was written before this point.
  asm volatile("griddepcontrol.wait;" ::: "memory");
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
  if (STAGED && blockIdx.x == 0 && b == 0)
    for (int i = threadIdx.x; i <= p.B; i += LF_THREADS)
      staged_off[i] = i < p.B ? p.v16_base[i] : p.v16_base[p.B - 1] + p.L[p.B - 1] + p.T[p.B - 1];
  const int n = p.L[b] + p.T[b];
  const int64_t kv_base = a.kv_off[b];
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int wstride = gridDim.x * (LF_THREADS / 32);
  const char* kv = static_cast<const char*>(a.kv);
  uint32_t range = 0;
  bool bad_row = false;
  for (int j0 = (blockIdx.x * (LF_THREADS / 32) + warp) * LF_ROWS; j0 < n; j0 += wstride * LF_ROWS) {
    uint4 x[LF_ROWS][2], xr[LF_ROWS];
#pragma unroll
    for (int r = 0; r < LF_ROWS; ++r) {
      x[r][0] = x[r][1] = xr[r] = make_uint4(0u, 0u, 0u, 0u);
      const int j = j0 + r;
      if (j < n) {
        int64_t row = a.page_table != nullptr ? (int64_t)a.page_table[kv_base + j] : kv_base + j;
        if (row < 0 || row >= a.num_slots) {
          bad_row = true;
          continue;
        }
        const uint4* src = reinterpret_cast<const uint4*>(kv + row * (int64_t)((a.D_c + a.D_r) * 2) + lane * 32);
        x[r][0] = ptx::ldg_nc_v4(src);
        x[r][1] = ptx::ldg_nc_v4(src + 1);
        if (STAGED && lane < 8)
          xr[r] = ptx::ldg_nc_v4(reinterpret_cast<const uint4*>(kv + row * (int64_t)((a.D_c + a.D_r) * 2) + 1024 +
                                                                   lane * 16));
      }
    }
#pragma unroll
    for (int r = 0; r < LF_ROWS; ++r) {
      const int j = j0 + r;
      if (j < n) {
        uint4 y[2];
#pragma unroll
        for (int h = 0; h < 2; ++h) {
          const uint4 w = x[r][h];
          range |= ptx::bf16x2_beyond_f16(w.x) | ptx::bf16x2_beyond_f16(w.y) | ptx::bf16x2_beyond_f16(w.z) |
                   ptx::bf16x2_beyond_f16(w.w);
          y[h] = make_uint4(ptx::bf16x2_to_f16x2(w.x), ptx::bf16x2_to_f16x2(w.y), ptx::bf16x2_to_f16x2(w.z),
                            ptx::bf16x2_to_f16x2(w.w));
        }
        const int64_t out_row = (int64_t)p.v16_base[b] + j;
        if (v16 != nullptr) {
          uint4* dst = reinterpret_cast<uint4*>(v16 + out_row * 512 + lane * 16);
          dst[0] = y[0];
          dst[1] = y[1];
        }
        if (STAGED && lane < 8)
          reinterpret_cast<uint4*>(staged + out_row * (int64_t)(a.D_r * 2))[lane] = xr[r];
      }
    }
  }
  if (STAGED) {
    // q_lat as fp16: one warp per query row, over all CTAs of the grid
    const int64_t wid = ((int64_t)b * gridDim.x + blockIdx.x) * (LF_THREADS / 32) + warp;
    const int64_t nw = (int64_t)gridDim.x * gridDim.y * (LF_THREADS / 32);
    for (int64_t row = wid; row < p.total_rows; row += nw) {
      const uint4* src = reinterpret_cast<const uint4*>(static_cast<const char*>(a.q) + row * a.q_row_stride * 2 +
                                                        lane * 32);
      uint4 w[2] = {ptx::ldg_nc_v4(src), ptx::ldg_nc_v4(src + 1)};
      uint4* dst = reinterpret_cast<uint4*>(q16 + row * 512 + lane * 16);
#pragma unroll
      for (int h = 0; h < 2; ++h) {
        range |= ptx::bf16x2_beyond_f16(w[h].x) | ptx::bf16x2_beyond_f16(w[h].y) | ptx::bf16x2_beyond_f16(w[h].z) |
                 ptx::bf16x2_beyond_f16(w[h].w);
        dst[h] = make_uint4(ptx::bf16x2_to_f16x2(w[h].x), ptx::bf16x2_to_f16x2(w[h].y), ptx::bf16x2_to_f16x2(w[h].z),
                            ptx::bf16x2_to_f16x2(w[h].w));
      }
    }
  }
  if (__any_sync(0xffffffffu, range != 0) && lane == 0) record_error(a.d_err, KDV_DERR_RANGE);
  if (__any_sync(0xffffffffu, bad_row) && lane == 0)
    record_error(a.d_err, a.page_table != nullptr ? KDV_DERR_BAD_SLOT : KDV_DERR_BAD_LENGTH);
}

}  // namespace

cudaError_t launch_latent_f16(const VerifyArgs& a, const VerifyPlan& p, void* v16, void* staged, int32_t* staged_off,
                              void* q16, cudaStream_t stream) {
  const bool stage = staged != nullptr;
  if (a.D_c != 512 || (stage && a.D_r != 64) || (staged_off != nullptr) != stage || (q16 != nullptr) != stage)
    return cudaErrorInvalidValue;
  int max_n = 0;
  for (int b = 0; b < p.B; ++b) max_n = max_n > p.L[b] + p.T[b] ? max_n : p.L[b] + p.T[b];
  if (max_n == 0) return cudaSuccess;
  const int rows_per_cta = (LF_THREADS / 32) * LF_ROWS;
  // enough CTAs in flight to keep HBM busy, fewer for a short request; at
  // 200k keys a grid capped at 16 x 148 CTAs streams ~10% faster than one
  // capped at 8 x 148 (more waves of short-lived CTAs even out the rows per
  // CTA)
  int gx = (max_n + rows_per_cta - 1) / rows_per_cta;
  const int cap = (16 * 148 + p.B - 1) / p.B;
  if (gx > cap) gx = cap < 1 ? 1 : cap;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3((unsigned)gx, (unsigned)p.B);
  cfg.blockDim = dim3(LF_THREADS);
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, stage ? latent_f16_kernel<true> : latent_f16_kernel<false>, a, p, static_cast<__half*>(v16), static_cast<uint8_t*>(staged),
                            staged_off, static_cast<__half*>(q16));
}

}  // namespace kdv

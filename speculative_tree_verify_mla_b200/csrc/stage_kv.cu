// stage_kv.cu -- copy a batch's paged KV rows into a contiguous workspace.
//
// The staged alternative for paged KV (page_size 1, page "The Architecture of
// Diagnosis", section "The Discrepancy That Revealed the Truth", item 2):
// logical key j of request b, pool row page_table[kv_off[b] + j], is copied
// to staged row stage_base(b) + j, where stage_base(b) = sum over b' < b of
// (L_b' + T_b'). The verify kernel then reads the staged rows with tiled TMA
// boxes instead of four-row gathers. One warp copies one 1152-byte row as
// 16-byte vectors; block (x, b) covers 8 rows of request b.
#include <algorithm>

#include "kdv_internal.cuh"

namespace kdv {

cudaError_t launch_stage_kv(const VerifyArgs& a, const VerifyPlan& p, int32_t row_bytes, void* staged,
                            int32_t* staged_off, cudaStream_t stream);

namespace {

constexpr int STAGE_THREADS = 256;
constexpr int ROWS_PER_CTA = STAGE_THREADS / 32;

__global__ void __launch_bounds__(STAGE_THREADS)
stage_kv_kernel(const VerifyArgs a, const VerifyPlan p, int32_t row_bytes, uint8_t* __restrict__ staged,
                int32_t* __restrict__ staged_off) {
  const int b = blockIdx.y;
  int64_t base = 0;
  for (int i = 0; i < b; ++i) base += (int64_t)p.L[i] + p.T[i];
  const int64_t n_b = (int64_t)p.L[b] + p.T[b];
  if (blockIdx.x == 0 && threadIdx.x == 0) {
    staged_off[b] = (int32_t)base;
    if (b == p.B - 1) staged_off[b + 1] = (int32_t)(base + n_b);
  }
  const int64_t j = (int64_t)blockIdx.x * ROWS_PER_CTA + (threadIdx.x >> 5);
  if (j >= n_b) return;
  const int lane = threadIdx.x & 31;
  const int64_t k0 = a.kv_off[b];
  const bool range_ok = (int64_t)a.kv_off[b + 1] - k0 >= n_b;
  int32_t slot = range_ok ? a.page_table[k0 + j] : -1;
  if (!range_ok || slot < 0 || (int64_t)slot >= a.num_slots) {
    if (lane == 0) record_error(a.d_err, range_ok ? KDV_DERR_BAD_SLOT : KDV_DERR_BAD_LENGTH);
    slot = -1;
  }
  const int nvec = row_bytes / 16;
  uint4* dst = reinterpret_cast<uint4*>(staged + (base + j) * (int64_t)row_bytes);
  const uint4* src = reinterpret_cast<const uint4*>(static_cast<const uint8_t*>(a.kv) + (int64_t)(slot < 0 ? 0 : slot) * row_bytes);
  for (int v = lane; v < nvec; v += 32) dst[v] = slot < 0 ? make_uint4(0, 0, 0, 0) : __ldg(src + v);
}

}  // namespace

cudaError_t launch_stage_kv(const VerifyArgs& a, const VerifyPlan& p, int32_t row_bytes, void* staged,
                            int32_t* staged_off, cudaStream_t stream) {
  int64_t max_n = 0;
  for (int b = 0; b < p.B; ++b) max_n = std::max<int64_t>(max_n, (int64_t)p.L[b] + p.T[b]);
  const int64_t gx = (max_n + ROWS_PER_CTA - 1) / ROWS_PER_CTA;
  if (gx < 1 || gx > 0x7fffffff) return cudaErrorInvalidValue;
  const dim3 grid((unsigned)gx, (unsigned)p.B);
  stage_kv_kernel<<<grid, STAGE_THREADS, 0, stream>>>(a, p, row_bytes, static_cast<uint8_t*>(staged), staged_off);
  return cudaGetLastError();
}

}  // namespace kdv

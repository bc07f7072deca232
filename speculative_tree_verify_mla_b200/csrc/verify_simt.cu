// verify_simt.cu -- CUDA-core tree-verify attention for any latent shape.
//
// Same operation as the tensor-core kernel (absorbed q.k over D_c + D_r dims,
// softmax over the visible keys, p.c_kv over the D_c latent dims), for shapes
// the tensor-core kernel does not take (fp32 inputs, small or odd dims). One
// warp owns one query row; a CTA of 8 warps holds 8 rows of one request and
// stages 32 keys at a time in shared memory (converted to fp32), where
// lane k scores key k against its row and then every lane accumulates its
// D_c/32 output dims. Accumulation and softmax are fp32 with an online
// (running-max) rescale.
#include <cuda_bf16.h>

#include "kdv_internal.cuh"

namespace kdv {
namespace {

constexpr int KT = 32;                 // keys per shared-memory tile
constexpr int WARPS = SIMT_ROWS;       // one warp per query row
constexpr int MAX_DC_PER_LANE = 16;    // D_c <= 512

__device__ inline float to_f32(float x) { return x; }
__device__ inline float to_f32(__nv_bfloat16 x) { return __bfloat162float(x); }

__device__ inline float warp_max(float v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, o));
  return v;
}
__device__ inline float warp_sum(float v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  return v;
}

template <typename T>
__global__ void __launch_bounds__(WARPS * 32)
verify_simt_kernel(const VerifyArgs a, const VerifyPlan p) {
  extern __shared__ float smem[];
  const int D_c = a.D_c, D_q = a.D_c + a.D_r;
  const int KS = D_q + 1;                      // padded key row stride (floats)
  float* Ks = smem;                            // [KT][KS]
  float* Qs = smem + KT * KS;                  // [WARPS][D_q]
  __shared__ int key_ok[KT];

  const int item = blockIdx.x;
  const int b = plan_request(p, item);
  const int local = item - p.item_base[b];
  const int s = local / p.tiles[b];
  const int rt = local - s * p.tiles[b];
  const int L = p.L[b], Tn = p.T[b], H = p.H;
  const int n_keys = L + Tn;
  const int rows_b = Tn * H;
  const int k_lo = min(s * p.chunk[b], n_keys);
  const int k_hi = min(k_lo + p.chunk[b], n_keys);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

  if (threadIdx.x == 0) {
    if (a.prefix_len != nullptr && a.prefix_len[b] != L) record_error(a.d_err, KDV_DERR_BAD_LENGTH);
    if (a.tree_off != nullptr && a.tree_off[b] != p.tree_base[b]) record_error(a.d_err, KDV_DERR_BAD_LENGTH);
  }
  const int64_t kv_base = a.kv_off[b];
  // the request's key range must fit its kv_off slice; otherwise read nothing
  const bool range_ok = (int64_t)a.kv_off[b + 1] - kv_base >= (int64_t)n_keys;
  if (!range_ok && threadIdx.x == 0) record_error(a.d_err, KDV_DERR_BAD_LENGTH);
  const T* kv = static_cast<const T*>(a.kv);
  const T* q = static_cast<const T*>(a.q);

  // this warp's row
  const int r = rt * WARPS + warp;
  const bool row_ok = r < rows_b;
  const int t = row_ok ? r / H : 0;
  const uint64_t mask_t = row_ok ? a.mask[p.tree_base[b] + t] : 0ull;
  const int64_t row_global = (int64_t)p.tree_base[b] * H + r;
  for (int d = lane; d < D_q; d += 32)
    Qs[warp * D_q + d] = row_ok ? to_f32(q[row_global * a.q_row_stride + d]) : 0.f;

  float o[MAX_DC_PER_LANE];
#pragma unroll
  for (int i = 0; i < MAX_DC_PER_LANE; ++i) o[i] = 0.f;
  float m = -INFINITY, l = 0.f;

  for (int j0 = k_lo; j0 < k_hi; j0 += KT) {
    __syncthreads();
    if (threadIdx.x < KT) {
      const int j = j0 + threadIdx.x;
      int ok = 0;
      if (j < k_hi && range_ok) {
        const int64_t slot = a.page_table ? (int64_t)a.page_table[kv_base + j] : kv_base + j;
        ok = (slot >= 0 && slot < a.num_slots) ? 1 : 0;
        if (!ok) record_error(a.d_err, KDV_DERR_BAD_SLOT);
      }
      key_ok[threadIdx.x] = ok;
    }
    __syncthreads();
    for (int idx = threadIdx.x; idx < KT * D_q; idx += WARPS * 32) {
      const int k = idx / D_q, d = idx - k * D_q;
      const int j = j0 + k;
      float v = 0.f;
      if (key_ok[k]) {
        const int64_t slot = a.page_table ? (int64_t)a.page_table[kv_base + j] : kv_base + j;
        v = to_f32(kv[slot * D_q + d]);
      }
      Ks[k * KS + d] = v;
    }
    __syncthreads();
    if (!row_ok) continue;

    // lane scores key j0 + lane
    const int j = j0 + lane;
    bool vis = false;
    if (j < k_hi && key_ok[lane]) vis = (j < L) || ((mask_t >> (j - L)) & 1ull);
    float sc = -INFINITY;
    if (vis) {
      float acc = 0.f;
      const float* qr = Qs + warp * D_q;
      const float* kr = Ks + lane * KS;
      for (int d = 0; d < D_q; ++d) acc = fmaf(qr[d], kr[d], acc);
      sc = a.scale * acc;
    }
    const float m_new = fmaxf(m, warp_max(sc));
    if (m_new == -INFINITY) continue;          // nothing visible yet (warp-uniform)
    const float corr = expf(m - m_new);         // 0 when m == -inf
    const float pk = vis ? expf(sc - m_new) : 0.f;
    l = l * corr + warp_sum(pk);
#pragma unroll
    for (int i = 0; i < MAX_DC_PER_LANE; ++i) o[i] *= corr;
    for (int k = 0; k < KT; ++k) {
      const float pv = __shfl_sync(0xffffffffu, pk, k);
      if (pv == 0.f) continue;                  // warp-uniform
      const float* vr = Ks + k * KS;
#pragma unroll
      for (int i = 0; i < MAX_DC_PER_LANE; ++i) {
        const int d = lane + 32 * i;
        if (d < D_c) o[i] = fmaf(pv, vr[d], o[i]);
      }
    }
    m = m_new;
  }

  if (!row_ok) return;
  const int64_t orow = out_row_index(p, b, s, r);
  const float inv = l > 0.f ? 1.f / l : 0.f;
#pragma unroll
  for (int i = 0; i < MAX_DC_PER_LANE; ++i) {
    const int d = lane + 32 * i;
    if (d < D_c) a.o[orow * D_c + d] = o[i] * inv;
  }
  if (lane == 0 && a.lse != nullptr) a.lse[orow] = l > 0.f ? m + logf(l) : -INFINITY;
}

}  // namespace

cudaError_t launch_verify_simt(const VerifyArgs& a, const VerifyPlan& p, int32_t dtype,
                               cudaStream_t stream) {
  const int D_q = a.D_c + a.D_r;
  const size_t smem = (size_t)(KT * (D_q + 1) + WARPS * D_q) * sizeof(float);
  if (dtype == KDV_F32) {
    auto k = verify_simt_kernel<float>;
    cudaError_t e = cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    k<<<p.n_items, WARPS * 32, smem, stream>>>(a, p);
  } else {
    auto k = verify_simt_kernel<__nv_bfloat16>;
    cudaError_t e = cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    k<<<p.n_items, WARPS * 32, smem, stream>>>(a, p);
  }
  return cudaGetLastError();
}

}  // namespace kdv

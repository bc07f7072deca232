// tree_build.cu -- best-first draft-tree construction on the device.
//
// The GPU-resident builder of page "The Architecture of Diagnosis", section
// "Phase 1: Custom CUDA Kernels", item 1, which replaces a host heap that
// grows the draft tree best-first. A block drafter proposes K candidate
// tokens with log-probabilities for each of D future positions; a node is a
// path of candidate choices, its score the fp32 sum of the log-probabilities
// along it (one float add per edge, root first). The tree is what T steps of
// best-first expansion emit (take the frontier node first in (score
// descending, candidate path ascending) order, add its K children); with
// log-probabilities <= 0 that is the first T nodes of that order.
//
// One warp per request, no block barrier anywhere. Frontier entry i belongs
// to lane i % 32: its score image and path key live in that lane's registers
// (stripe i / 32), its depth, parent and token in shared memory, and every
// lane keeps the best of its own live entries. A round is
// then a warp-wide selection of the best lane-best under that total order
// (redux max over an order-preserving integer image of the score, redux min
// over the unique path key only when scores tie), after which the winner's
// lane retires it and rescans its own entries while the K lanes that own the
// next K frontier slots append the winner's children. The path key holds the
// choices as D base-(K+1) digits, most significant first, 0 past the path's
// end: numeric order is digit-by-digit order with a prefix first. A child's
// score that comes out NaN (+inf plus -inf) is read as -inf, like a NaN
// log-probability: a path with no defined score is never preferred.
#include <cuda_runtime.h>

#include <cmath>
#include <cstdint>

#include "kdv.h"

namespace kdv {
namespace {

constexpr int BUILD_THREADS = 32;     // one warp per request
constexpr int MAX_D = 16, MAX_K = 8, MAX_NODES = 64;
constexpr int MAX_FRONTIER = 1 + MAX_NODES * MAX_K;
constexpr int NSTRIPE = (MAX_FRONTIER + BUILD_THREADS - 1) / BUILD_THREADS;
constexpr unsigned FULL = 0xffffffffu;

struct BuildArgs {
  int32_t max_T, D, K;
  const int32_t* tree_off;
  const int32_t* root_token;
  const int32_t* cand_token;
  const float* cand_logp;
  int32_t* parent;
  int32_t* token;
  int32_t* depth;
  float* score;
  int32_t* d_err;
};

__device__ __forceinline__ void record_err(int32_t* d_err, int32_t code) {
  if (d_err != nullptr) atomicCAS(d_err, 0, code);
}

// Order-preserving image of a non-NaN score in [1, 2^32): x < y <=> img(x) <
// img(y), +0 and -0 equal. 0 stands for "no live entry".
__device__ __forceinline__ uint32_t score_img(float s) {
  const uint32_t u = __float_as_uint(s == 0.f ? 0.f : s);
  return (u & 0x80000000u) ? ~u : (u | 0x80000000u);
}
__device__ __forceinline__ float score_of(uint32_t img) {
  return __uint_as_float((img & 0x80000000u) ? (img & 0x7fffffffu) : ~img);
}

// (img, key) a ranks before b: score descending, then path key ascending
__device__ __forceinline__ bool before(uint32_t ia, unsigned long long ka, uint32_t ib, unsigned long long kb) {
  return ia > ib || (ia == ib && ka < kb);
}

__global__ void __launch_bounds__(BUILD_THREADS) tree_build_kernel(const BuildArgs a) {
  // frontier entries; entry i is touched by lane i % 32 only: score image
  // and path key in that lane's registers (stripe i / 32), the rest here
  __shared__ int32_t e_depth[MAX_FRONTIER], e_parent[MAX_FRONTIER], e_token[MAX_FRONTIER];
  uint32_t r_img[NSTRIPE];
  unsigned long long r_key[NSTRIPE];
#pragma unroll
  for (int st = 0; st < NSTRIPE; ++st) {
    r_img[st] = 0u;
    r_key[st] = 0ull;
  }
  __shared__ float s_logp[MAX_D * MAX_K];
  __shared__ int32_t s_tok[MAX_D * MAX_K];
  __shared__ unsigned long long s_place[MAX_D + 1];
  const int b = blockIdx.x, lane = threadIdx.x;
  const int D = a.D, K = a.K;
  const int t0 = a.tree_off[b];
  const int T = a.tree_off[b + 1] - t0;
  if (T < 1 || T > a.max_T) {                    // uniform over the warp
    if (lane == 0) record_err(a.d_err, KDV_DERR_BAD_LENGTH);
    return;
  }
  // ---- candidates into shared memory: every load issued before any use
  const int64_t cbase = (int64_t)b * D * K;
  constexpr int PER_LANE = MAX_D * MAX_K / BUILD_THREADS;
  float lp[PER_LANE];
  int32_t tk[PER_LANE];
#pragma unroll
  for (int r = 0; r < PER_LANE; ++r) {
    const int i = lane + r * BUILD_THREADS;
    if (i < D * K) {
      lp[r] = a.cand_logp[cbase + i];
      tk[r] = a.cand_token[cbase + i];
    }
  }
#pragma unroll
  for (int r = 0; r < PER_LANE; ++r) {
    const int i = lane + r * BUILD_THREADS;
    if (i < D * K) {
      if (isnan(lp[r])) {
        record_err(a.d_err, KDV_DERR_BAD_SCORE);
        lp[r] = -INFINITY;                           // a candidate never preferred
      }
      s_logp[i] = lp[r];
      s_tok[i] = tk[r];
    }
  }
  if (lane >= 1 && lane <= D) {                    // s_place[d] = (K+1)^(D-d)
    unsigned long long p = 1;
    for (int e = lane; e < D; ++e) p *= (unsigned long long)(K + 1);
    s_place[lane] = p;
  }
  // ---- the root: entry 0, lane 0
  uint32_t lb_img = 0;                             // this lane's best live entry
  unsigned long long lb_key = 0ull;
  int lb_dep = 0, lb_idx = -1;
  if (lane == 0) {
    r_img[0] = score_img(0.f);
    r_key[0] = 0ull;
    e_depth[0] = 0;
    e_parent[0] = -1;
    e_token[0] = a.root_token[b];
    lb_img = score_img(0.f);
    lb_idx = 0;
  }
  __syncwarp();                                    // candidates visible to every lane
  int n_front = 1;                                 // uniform over the warp
  int n = 0;
  for (; n < T; ++n) {
    // ---- the best live entry of the warp
    const uint32_t m = __reduce_max_sync(FULL, lb_img);
    if (m == 0u) break;                            // uniform: candidates ran out
    uint32_t win = __ballot_sync(FULL, lb_img == m);
    if (__popc(win) > 1) {                         // uniform: tied scores, unique keys decide
      const bool t = (win >> lane) & 1u;
      const uint32_t khi = t ? (uint32_t)(lb_key >> 32) : 0xffffffffu;
      const uint32_t mh = __reduce_min_sync(FULL, khi);
      const bool t2 = t && khi == mh;
      const uint32_t klo = t2 ? (uint32_t)lb_key : 0xffffffffu;
      const uint32_t ml = __reduce_min_sync(FULL, klo);
      win = __ballot_sync(FULL, t2 && klo == ml);
    }
    const int owner = __ffs(win) - 1;
    const unsigned long long bk = __shfl_sync(FULL, lb_key, owner);
    const int bi = __shfl_sync(FULL, lb_idx, owner);
    const int dep = __shfl_sync(FULL, lb_dep, owner);
    const float bs = score_of(m);
    // ---- the winner's lane emits node n, retires it and rescans its entries
    if (lane == owner) {
      a.parent[t0 + n] = e_parent[bi];
      a.token[t0 + n] = e_token[bi];
      if (a.depth) a.depth[t0 + n] = dep;
      if (a.score) a.score[t0 + n] = bs;
      const int bst = bi / BUILD_THREADS;
      uint32_t c_img[NSTRIPE];
      unsigned long long c_key[NSTRIPE];
      int c_st[NSTRIPE];
#pragma unroll
      for (int st = 0; st < NSTRIPE; ++st) {
        if (st == bst) r_img[st] = 0u;             // retire the emitted entry
        c_img[st] = r_img[st];
        c_key[st] = r_key[st];
        c_st[st] = st;
      }
      // pairwise tournament: 5 levels instead of a 16-long chain, over the
      // stripes the frontier has reached so far (the bound is warp-uniform)
      const int nst = (n_front + BUILD_THREADS - 1) / BUILD_THREADS;
#pragma unroll
      for (int w = 1; w < NSTRIPE; w *= 2) {
#pragma unroll
        for (int st = 0; st + w < NSTRIPE; st += 2 * w) {
          if (st + w < nst && before(c_img[st + w], c_key[st + w], c_img[st], c_key[st])) {
            c_img[st] = c_img[st + w];
            c_key[st] = c_key[st + w];
            c_st[st] = c_st[st + w];
          }
        }
      }
      lb_img = c_img[0];
      lb_key = c_key[0];
      lb_idx = lane + c_st[0] * BUILD_THREADS;
      lb_dep = lb_img != 0u ? e_depth[lb_idx] : 0;
    }
    // ---- the lanes owning slots n_front .. n_front+K-1 append the children
    if (dep < D) {                                 // uniform
      const int j = (lane - n_front) & (BUILD_THREADS - 1);
      if (j < K) {
        const int i = n_front + j;                 // i % 32 == lane
        float sc = bs + s_logp[dep * K + j];
        if (isnan(sc)) sc = -INFINITY;             // +inf + -inf: no defined score
        const uint32_t img = score_img(sc);
        const unsigned long long ky = bk + (unsigned long long)(j + 1) * s_place[dep + 1];
        const int ist = i / BUILD_THREADS;
#pragma unroll
        for (int st = 0; st < NSTRIPE; ++st)
          if (st == ist) {
            r_img[st] = img;
            r_key[st] = ky;
          }
        e_depth[i] = dep + 1;
        e_parent[i] = n;
        e_token[i] = s_tok[dep * K + j];
        if (lb_img == 0u || before(img, ky, lb_img, lb_key)) {
          lb_img = img;
          lb_key = ky;
          lb_idx = i;
          lb_dep = dep + 1;
        }
      }
      n_front += K;
    }
  }
  if (n < T) {                                     // budget above the number of paths
    if (lane == 0) record_err(a.d_err, KDV_DERR_BAD_LENGTH);
    for (int i = n + lane; i < T; i += BUILD_THREADS) {
      a.parent[t0 + i] = -1;
      a.token[t0 + i] = -1;
      if (a.depth) a.depth[t0 + i] = 0;
      if (a.score) a.score[t0 + i] = -INFINITY;
    }
  }
}

}  // namespace
}  // namespace kdv

using namespace kdv;

extern "C" {

kdv_status kdv_tree_build(const kdv_tree_build_params* p, void* stream) {
  if (p == nullptr) return KDV_ERR_INVALID_ARG;
  if (p->batch < 1 || p->batch > KDV_MAX_BATCH) return KDV_ERR_UNSUPPORTED;
  if (p->max_T < 1 || p->max_T > KDV_MAX_TREE) return KDV_ERR_UNSUPPORTED;
  if (p->depth < 0 || p->depth > MAX_D || p->topk < 1 || p->topk > MAX_K) return KDV_ERR_UNSUPPORTED;
  if (p->tree_off == nullptr || p->root_token == nullptr || p->parent == nullptr || p->token == nullptr)
    return KDV_ERR_INVALID_ARG;
  if (p->depth > 0 && (p->cand_token == nullptr || p->cand_logp == nullptr)) return KDV_ERR_INVALID_ARG;
  BuildArgs a;
  a.max_T = p->max_T;
  a.D = p->depth;
  a.K = p->topk;
  a.tree_off = p->tree_off;
  a.root_token = p->root_token;
  a.cand_token = p->cand_token;
  a.cand_logp = p->cand_logp;
  a.parent = p->parent;
  a.token = p->token;
  a.depth = p->depth_out;
  a.score = p->score;
  a.d_err = p->d_err;
  tree_build_kernel<<<p->batch, BUILD_THREADS, 0, static_cast<cudaStream_t>(stream)>>>(a);
  return cudaGetLastError() == cudaSuccess ? KDV_OK : KDV_ERR_CUDA;
}

}  // extern "C"

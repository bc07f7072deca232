// tree_build.cu -- best-first draft-tree construction on the device.
//
// The GPU-resident builder of page "The Architecture of Diagnosis", section
// "Phase 1: Custom CUDA Kernels", item 1, which replaces a host heap that
// grows the draft tree best-first. A block drafter proposes K candidate
// tokens with log-probabilities for each of D future positions; a node is a
// path of candidate choices, its score the fp32 sum of the log-probabilities
// along it (one float add per edge, root first). The tree is the first T
// nodes in (score descending, candidate path ascending) order, emitted in
// that order; with log-probabilities <= 0 this is exactly the best-first
// expansion (take the best frontier node, add its K children).
//
// One warp per request. The frontier (at most 1 + 64 * 8 entries) lives in
// shared memory; each of the T rounds is a warp-wide argmax over it under
// that total order (a unique path key breaks every tie, so the result does
// not depend on the reduction order), then K lanes append the winner's
// children -- no block barrier anywhere. The path key holds the choices as
// D base-(K+1) digits, most significant first, 0 past the path's end:
// numeric order is digit-by-digit order with a prefix first.
#include <cuda_runtime.h>

#include <cmath>

#include "kdv.h"

namespace kdv {
namespace {

constexpr int BUILD_THREADS = 32;     // one warp per request: no block barriers
constexpr int MAX_D = 16, MAX_K = 8, MAX_NODES = 64;
constexpr int MAX_FRONTIER = 1 + MAX_NODES * MAX_K;

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

// a ranks before b (score descending, then key ascending); an empty slot
// (idx < 0) ranks last
__device__ __forceinline__ bool before(float sa, unsigned long long ka, int ia, float sb, unsigned long long kb,
                                       int ib) {
  if (ia < 0) return false;
  if (ib < 0) return true;
  if (sa != sb) return sa > sb;
  return ka < kb;
}

__global__ void __launch_bounds__(BUILD_THREADS) tree_build_kernel(const BuildArgs a) {
  __shared__ float f_score[MAX_FRONTIER];
  __shared__ unsigned long long f_key[MAX_FRONTIER];
  __shared__ int32_t f_depth[MAX_FRONTIER], f_parent[MAX_FRONTIER], f_token[MAX_FRONTIER];
  __shared__ unsigned char f_live[MAX_FRONTIER];
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
  const int64_t cbase = (int64_t)b * D * K;
  for (int i = lane; i < D * K; i += BUILD_THREADS) {
    float lp = a.cand_logp[cbase + i];
    if (isnan(lp)) {
      record_err(a.d_err, KDV_DERR_BAD_SCORE);
      lp = -INFINITY;                              // a candidate never preferred
    }
    s_logp[i] = lp;
    s_tok[i] = a.cand_token[cbase + i];
  }
  if (lane == 0) {
    // s_place[d] = (K+1)^(D-d): the weight of the digit chosen at depth d
    unsigned long long p = 1;
    for (int d = D; d >= 1; --d) {
      s_place[d] = p;
      p *= (unsigned long long)(K + 1);
    }
    f_score[0] = 0.f;
    f_key[0] = 0ull;
    f_depth[0] = 0;
    f_parent[0] = -1;
    f_token[0] = a.root_token[b];
    f_live[0] = 1;
  }
  __syncwarp();
  int n_front = 1;                                 // uniform over the warp
  int n = 0;
  for (; n < T; ++n) {
    // ---- best live frontier entry: each lane scans a stripe, then shuffles
    float bs = 0.f;
    unsigned long long bk = 0ull;
    int bi = -1;
    // unrolled over the largest stripe so that a lane's loads issue together
#pragma unroll
    for (int st = 0; st < (MAX_FRONTIER + BUILD_THREADS - 1) / BUILD_THREADS; ++st) {
      const int i = lane + st * BUILD_THREADS;
      if (i < n_front) {
        const bool live = f_live[i];
        const float sc = f_score[i];
        const unsigned long long ky = f_key[i];
        if (live && before(sc, ky, i, bs, bk, bi)) {
          bs = sc;
          bk = ky;
          bi = i;
        }
      }
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) {
      const float os = __shfl_xor_sync(0xffffffffu, bs, o);
      const unsigned long long ok = __shfl_xor_sync(0xffffffffu, bk, o);
      const int oi = __shfl_xor_sync(0xffffffffu, bi, o);
      if (before(os, ok, oi, bs, bk, bi)) {
        bs = os;
        bk = ok;
        bi = oi;
      }
    }
    if (bi < 0) break;                             // uniform: candidates ran out
    // ---- emit node n, append its children
    const int dep = f_depth[bi];
    if (lane == 0) {
      a.parent[t0 + n] = f_parent[bi];
      a.token[t0 + n] = f_token[bi];
      if (a.depth) a.depth[t0 + n] = dep;
      if (a.score) a.score[t0 + n] = bs;
    }
    const bool kids = dep < D;
    if (kids && lane < K) {
      const int i = n_front + lane;
      f_score[i] = bs + s_logp[dep * K + lane];
      f_key[i] = bk + (unsigned long long)(lane + 1) * s_place[dep + 1];
      f_depth[i] = dep + 1;
      f_parent[i] = n;
      f_token[i] = s_tok[dep * K + lane];
      f_live[i] = 1;
    }
    __syncwarp();                                  // every read of the winner done
    if (lane == 0) f_live[bi] = 0;
    if (kids) n_front += K;
    __syncwarp();
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

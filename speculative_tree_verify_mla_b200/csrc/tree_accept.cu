// tree_accept.cu -- greedy tree acceptance on the device.
//
// The step after verification (page "The Architecture of Diagnosis", section
// "Phase 1: Custom CUDA Kernels", item 3): pick, without the host, the
// longest path of draft tokens that agrees with the target model's greedy
// choice at every step. Two launches:
//
//   argmax_partial_kernel  grid (chunks, rows): each CTA reduces CHUNK logits
//       of one row to one 64-bit key (orderable value << 32 | ~index), so a
//       plain unsigned max picks the largest value and, among equal values,
//       the lowest index. HBM-bound: it streams the logits once.
//   accept_tree_kernel     one CTA of 256 threads per request: the warps
//       finish the argmax over the chunk keys (one node per warp at a time),
//       then thread t <-> node t (warps 0-1) decides for every node
//       whether its root path is accepted (each node walks its own ancestors,
//       so no node waits on another), takes the deepest accepted node (lowest
//       index on ties), writes the path, the bonus token and optionally
//       commits the page table in place. It is launched as a programmatic
//       dependent of the argmax pass (its launch overlaps that pass) and
//       reads nothing before the pass has finished.
#include <cuda_runtime.h>

#include "kdv.h"

namespace kdv {
namespace {

constexpr int ARGMAX_THREADS = 256;
constexpr int CHUNK = 8192;          // logits per argmax CTA
constexpr int ACCEPT_THREADS = 256;  // 8 warps reduce the chunk keys; warps 0-1 hold the nodes
constexpr int MAX_NODES = 64;        // = KDV_MAX_TREE

__device__ __forceinline__ void record_err(int32_t* d_err, int32_t code) {
  if (d_err != nullptr) atomicCAS(d_err, 0, code);
}

// Key of one logit given its fp32 bit pattern: 0 for NaN; -0 counts as +0.
__device__ __forceinline__ unsigned long long logit_key(uint32_t bits, uint32_t idx) {
  if ((bits & 0x7fffffffu) > 0x7f800000u) return 0ull;            // NaN never wins
  if ((bits & 0x7fffffffu) == 0u) bits = 0u;                      // -0 == +0
  const uint32_t ord = (bits & 0x80000000u) ? ~bits : (bits | 0x80000000u);
  return ((unsigned long long)ord << 32) | (unsigned long long)(0xffffffffu - idx);
}

__device__ __forceinline__ unsigned long long umax64(unsigned long long a, unsigned long long b) {
  return a > b ? a : b;
}

template <bool BF16>
__global__ void __launch_bounds__(ARGMAX_THREADS)
argmax_partial_kernel(const void* __restrict__ logits, int64_t ld, int32_t vocab, int32_t chunks,
                      int vec, unsigned long long* __restrict__ part) {
  const int row = blockIdx.y, chunk = blockIdx.x;
  // the acceptance kernel may launch now; it waits for this grid to finish
  if (threadIdx.x == 0) asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
  const int64_t c0 = (int64_t)chunk * CHUNK;
  const int64_t c1 = c0 + CHUNK < vocab ? c0 + CHUNK : vocab;
  unsigned long long best = 0ull;
  const bool full = vec && c1 - c0 == CHUNK;
  if (full) {
    // a whole chunk: every thread issues all its 16-byte loads before using
    // any, so the CTA costs one memory round trip
    constexpr int LOADS = CHUNK * (BF16 ? 2 : 4) / 16 / ARGMAX_THREADS;
    constexpr int PER = BF16 ? 8 : 4;                 // logits per load
    const uint4* x4 = reinterpret_cast<const uint4*>(static_cast<const char*>(logits) +
                                                     ((int64_t)row * ld + c0) * (BF16 ? 2 : 4));
    uint4 u[LOADS];
#pragma unroll
    for (int k = 0; k < LOADS; ++k) u[k] = __ldg(x4 + k * ARGMAX_THREADS + threadIdx.x);
#pragma unroll
    for (int k = 0; k < LOADS; ++k) {
      const uint32_t idx0 = (uint32_t)(c0 + (int64_t)(k * ARGMAX_THREADS + threadIdx.x) * PER);
      const uint32_t w[4] = {u[k].x, u[k].y, u[k].z, u[k].w};
#pragma unroll
      for (int q = 0; q < 4; ++q) {
        if (BF16) {
          best = umax64(best, logit_key(w[q] << 16, idx0 + 2 * q));
          best = umax64(best, logit_key(w[q] & 0xffff0000u, idx0 + 2 * q + 1));
        } else {
          best = umax64(best, logit_key(w[q], idx0 + q));
        }
      }
    }
  } else if (BF16) {
    const uint16_t* x = static_cast<const uint16_t*>(logits) + (int64_t)row * ld;
    if (vec) {
      // 8 logits per 16-byte load; the row start is 16-byte aligned and CHUNK
      // is a multiple of 8, so every group starting before c1 is aligned
      for (int64_t g = c0 + 8 * threadIdx.x; g < c1; g += 8 * ARGMAX_THREADS) {
        if (g + 8 <= c1) {
          const uint4 u = __ldg(reinterpret_cast<const uint4*>(x + g));
          const uint32_t w[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
          for (int q = 0; q < 4; ++q) {
            best = umax64(best, logit_key(w[q] << 16, (uint32_t)(g + 2 * q)));
            best = umax64(best, logit_key(w[q] & 0xffff0000u, (uint32_t)(g + 2 * q + 1)));
          }
        } else {
          for (int64_t v = g; v < c1; ++v) best = umax64(best, logit_key((uint32_t)x[v] << 16, (uint32_t)v));
        }
      }
    } else {
      for (int64_t v = c0 + threadIdx.x; v < c1; v += ARGMAX_THREADS)
        best = umax64(best, logit_key((uint32_t)x[v] << 16, (uint32_t)v));
    }
  } else {
    const uint32_t* x = static_cast<const uint32_t*>(logits) + (int64_t)row * ld;
    if (vec) {
      for (int64_t g = c0 + 4 * threadIdx.x; g < c1; g += 4 * ARGMAX_THREADS) {
        if (g + 4 <= c1) {
          const uint4 u = __ldg(reinterpret_cast<const uint4*>(x + g));
          best = umax64(best, logit_key(u.x, (uint32_t)g));
          best = umax64(best, logit_key(u.y, (uint32_t)(g + 1)));
          best = umax64(best, logit_key(u.z, (uint32_t)(g + 2)));
          best = umax64(best, logit_key(u.w, (uint32_t)(g + 3)));
        } else {
          for (int64_t v = g; v < c1; ++v) best = umax64(best, logit_key(x[v], (uint32_t)v));
        }
      }
    } else {
      for (int64_t v = c0 + threadIdx.x; v < c1; v += ARGMAX_THREADS)
        best = umax64(best, logit_key(x[v], (uint32_t)v));
    }
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) best = umax64(best, __shfl_xor_sync(0xffffffffu, best, o));
  __shared__ unsigned long long s_best[ARGMAX_THREADS / 32];
  if ((threadIdx.x & 31) == 0) s_best[threadIdx.x >> 5] = best;
  __syncthreads();
  if (threadIdx.x == 0) {
    for (int w = 1; w < ARGMAX_THREADS / 32; ++w) best = umax64(best, s_best[w]);
    part[(int64_t)row * chunks + chunk] = best;
  }
}

struct AcceptArgs {
  int32_t max_T, vocab, chunks;
  const unsigned long long* part;   // [sumT][chunks] or NULL (targets given)
  const int32_t* target_in;
  const int32_t* token;
  const int32_t* parent;
  const int32_t* tree_off;
  int32_t* target_out;
  int32_t* accept_len;
  int32_t* accept_path;
  int32_t* bonus;
  int32_t* page_table;
  const int32_t* kv_off;
  const int32_t* prefix_len;
  int32_t* prefix_len_out;
  int32_t* d_err;
};

__global__ void __launch_bounds__(ACCEPT_THREADS) accept_tree_kernel(const AcceptArgs a) {
  __shared__ int32_t s_parent[MAX_NODES], s_token[MAX_NODES], s_target[MAX_NODES];
  __shared__ int32_t s_path[MAX_NODES];
  __shared__ unsigned long long s_key[ACCEPT_THREADS / 32];
  __shared__ int s_off_count;
  // launched as a programmatic dependent of the argmax pass: nothing is read
  // before that grid (and so all earlier work on the stream) has finished;
  // a no-op when launched normally
  asm volatile("griddepcontrol.wait;" ::: "memory");
  const int b = blockIdx.x, t = threadIdx.x, lane = t & 31, warp = t >> 5;
  const int t0 = a.tree_off[b];
  const int T = a.tree_off[b + 1] - t0;
  int32_t* path_out = a.accept_path + (int64_t)b * a.max_T;
  if (T < 1 || T > a.max_T) {                     // uniform over the block
    if (t == 0) {
      record_err(a.d_err, KDV_DERR_BAD_LENGTH);
      a.accept_len[b] = 0;
      if (a.bonus) a.bonus[b] = -1;
      if (a.prefix_len_out) a.prefix_len_out[b] = a.prefix_len[b];
    }
    if (t < a.max_T) path_out[t] = -1;
    return;
  }
  // ---- target of every node: warp w reduces the chunk keys of nodes w, w+8, ...
  if (a.part != nullptr) {
    for (int n = warp; n < T; n += ACCEPT_THREADS / 32) {
      const unsigned long long* kp = a.part + (int64_t)(t0 + n) * a.chunks;
      unsigned long long key = 0ull;
      for (int c = lane; c < a.chunks; c += 32) key = umax64(key, kp[c]);
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) key = umax64(key, __shfl_xor_sync(0xffffffffu, key, o));
      if (lane == 0) s_target[n] = key == 0ull ? 0 : (int32_t)(0xffffffffu - (uint32_t)(key & 0xffffffffull));
    }
  } else if (t < T) {
    const int32_t target = a.target_in[t0 + t];
    if (target < 0 || target >= a.vocab) record_err(a.d_err, KDV_DERR_BAD_TOKEN);
    s_target[t] = target;
  }
  // ---- per-node inputs (thread t <-> node t)
  bool bad_parent = false;
  if (t < T) {
    const int32_t p = a.parent[t0 + t];
    const int32_t tok = a.token[t0 + t];
    bad_parent = !(p == -1 || (p >= 0 && p < t));
    if (p != -1 && (tok < 0 || tok >= a.vocab)) record_err(a.d_err, KDV_DERR_BAD_TOKEN);
    s_parent[t] = p;
    s_token[t] = tok;
  }
  if (__syncthreads_or(bad_parent)) {
    if (t == 0) {
      record_err(a.d_err, KDV_DERR_BAD_PARENT);
      a.accept_len[b] = 0;
      if (a.bonus) a.bonus[b] = -1;
      if (a.prefix_len_out) a.prefix_len_out[b] = a.prefix_len[b];
    }
    if (t < T && a.target_out) a.target_out[t0 + t] = s_target[t];
    if (t < a.max_T) path_out[t] = -1;
    return;
  }
  if (t < T && a.target_out) a.target_out[t0 + t] = s_target[t];
  // ---- accepted iff every edge on the root path matches; key = (depth+1, -t)
  unsigned long long key = 0ull;
  int depth = 0;
  if (t < T) {
    bool ok = true;
    for (int u = t; s_parent[u] != -1; u = s_parent[u]) {   // parents precede children: <= 63 steps
      if (s_token[u] != s_target[s_parent[u]]) ok = false;
      ++depth;
    }
    if (ok) key = ((unsigned long long)(depth + 1) << 8) | (unsigned long long)(255 - t);
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) key = umax64(key, __shfl_xor_sync(0xffffffffu, key, o));
  if (lane == 0) s_key[warp] = key;
  __syncthreads();
  unsigned long long best = 0ull;
#pragma unroll
  for (int w = 0; w < ACCEPT_THREADS / 32; ++w) best = umax64(best, s_key[w]);
  const int end = 255 - (int)(best & 255ull);
  const int len = (int)(best >> 8);
  if (t == 0) {
    for (int u = end, i = len - 1; i >= 0; --i, u = s_parent[u]) s_path[i] = u;
    a.accept_len[b] = len;
    if (a.bonus) a.bonus[b] = s_target[end];
  }
  __syncthreads();
  if (t < a.max_T) path_out[t] = t < len ? s_path[t] : -1;
  if (a.prefix_len_out && t == 0) a.prefix_len_out[b] = a.prefix_len[b] + len;
  // ---- page commit: path slots first (in path order), then the others in node order
  if (a.page_table != nullptr) {
    const int64_t base = (int64_t)a.kv_off[b] + a.prefix_len[b];
    if (base + T > (int64_t)a.kv_off[b + 1] || a.prefix_len[b] < 0) {
      if (t == 0) record_err(a.d_err, KDV_DERR_BAD_LENGTH);
      return;                                    // uniform: every thread read the same values
    }
    // node t is on the path iff it is the path's entry at its own depth
    const bool on_path = t < T && depth < len && s_path[depth] == t;
    const bool off_path = t < T && !on_path;
    const unsigned ballot = __ballot_sync(0xffffffffu, off_path);
    if (t == 31) s_off_count = __popc(ballot);
    int32_t old = 0;
    if (t < T) old = a.page_table[base + t];
    __syncthreads();                             // every old slot read before any write
    const int below = __popc(ballot & ((1u << lane) - 1u)) + (warp == 1 ? s_off_count : 0);
    if (on_path) a.page_table[base + depth] = old;
    else if (off_path) a.page_table[base + len + below] = old;
  }
}

}  // namespace
}  // namespace kdv

using namespace kdv;

namespace {

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15) == 0; }

kdv_status check_accept(const kdv_accept_params* p) {
  if (p == nullptr) return KDV_ERR_INVALID_ARG;
  if (p->batch < 1 || p->batch > KDV_MAX_BATCH) return KDV_ERR_UNSUPPORTED;
  if (p->max_T < 1 || p->max_T > KDV_MAX_TREE) return KDV_ERR_UNSUPPORTED;
  if (p->total_nodes < p->batch || p->total_nodes > p->batch * p->max_T) return KDV_ERR_INVALID_ARG;
  if (p->vocab < 1) return KDV_ERR_INVALID_ARG;
  if (p->token == nullptr || p->parent == nullptr || p->tree_off == nullptr ||
      p->accept_len == nullptr || p->accept_path == nullptr)
    return KDV_ERR_INVALID_ARG;
  if (p->logits != nullptr) {
    if (p->dtype != KDV_BF16 && p->dtype != KDV_F32) return KDV_ERR_INVALID_ARG;
    if (p->logits_ld < p->vocab) return KDV_ERR_INVALID_ARG;
  } else if (p->target_in == nullptr) {
    return KDV_ERR_INVALID_ARG;
  }
  if (p->page_table != nullptr && (p->kv_off == nullptr || p->prefix_len == nullptr))
    return KDV_ERR_INVALID_ARG;
  if (p->prefix_len_out != nullptr && p->prefix_len == nullptr) return KDV_ERR_INVALID_ARG;
  return KDV_OK;
}

int32_t accept_chunks(const kdv_accept_params* p) { return (p->vocab + CHUNK - 1) / CHUNK; }

}  // namespace

extern "C" {

kdv_status kdv_tree_accept_workspace(const kdv_accept_params* p, size_t* bytes) {
  if (bytes == nullptr) return KDV_ERR_INVALID_ARG;
  const kdv_status st = check_accept(p);
  if (st != KDV_OK) return st;
  *bytes = p->logits == nullptr ? 0 : (size_t)p->total_nodes * accept_chunks(p) * sizeof(unsigned long long);
  return KDV_OK;
}

kdv_status kdv_tree_accept(const kdv_accept_params* p, void* stream) {
  size_t need = 0;
  kdv_status st = kdv_tree_accept_workspace(p, &need);
  if (st != KDV_OK) return st;
  if (need > 0 && (p->workspace == nullptr || p->workspace_bytes < need || !aligned16(p->workspace)))
    return KDV_ERR_WORKSPACE;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  AcceptArgs a;
  a.max_T = p->max_T;
  a.vocab = p->vocab;
  a.chunks = accept_chunks(p);
  a.part = nullptr;
  a.target_in = p->target_in;
  a.token = p->token;
  a.parent = p->parent;
  a.tree_off = p->tree_off;
  a.target_out = p->target_out;
  a.accept_len = p->accept_len;
  a.accept_path = p->accept_path;
  a.bonus = p->bonus;
  a.page_table = p->page_table;
  a.kv_off = p->kv_off;
  a.prefix_len = p->prefix_len;
  a.prefix_len_out = p->prefix_len_out;
  a.d_err = p->d_err;
  if (p->logits != nullptr) {
    unsigned long long* part = static_cast<unsigned long long*>(p->workspace);
    const size_t esz = p->dtype == KDV_BF16 ? 2 : 4;
    const int vec = aligned16(p->logits) && ((size_t)p->logits_ld * esz) % 16 == 0;
    const dim3 grid((unsigned)a.chunks, (unsigned)p->total_nodes);
    if (p->dtype == KDV_BF16)
      argmax_partial_kernel<true><<<grid, ARGMAX_THREADS, 0, s>>>(p->logits, p->logits_ld, p->vocab,
                                                                  a.chunks, vec, part);
    else
      argmax_partial_kernel<false><<<grid, ARGMAX_THREADS, 0, s>>>(p->logits, p->logits_ld, p->vocab,
                                                                   a.chunks, vec, part);
    if (cudaGetLastError() != cudaSuccess) return KDV_ERR_CUDA;
    a.part = part;
  }
  if (p->logits == nullptr) {
    accept_tree_kernel<<<p->batch, ACCEPT_THREADS, 0, s>>>(a);
    return cudaGetLastError() == cudaSuccess ? KDV_OK : KDV_ERR_CUDA;
  }
  // right behind the argmax pass: launch as its programmatic dependent
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3((unsigned)p->batch);
  cfg.blockDim = dim3(ACCEPT_THREADS);
  cfg.stream = s;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, accept_tree_kernel, a) == cudaSuccess ? KDV_OK : KDV_ERR_CUDA;
}

}  // extern "C"

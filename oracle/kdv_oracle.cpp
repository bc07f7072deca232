// kdv_oracle.cpp -- the CPU oracle for tree-verify MLA attention.
//
// TEST INFRASTRUCTURE ONLY. This file is the plain, slow, fp64 definition that
// the CUDA path is checked against. Only the tests, the smoke check and the
// benchmark's CPU-baseline leg load it; the product path never does. It shares
// no code, header, helper or constant with the CUDA library.
//
// What it computes (the pages never write the equations; they name the kernel
// as a fused multi-head latent attention that absorbs the latent projection
// and evaluates every draft-tree node in parallel under a visibility mask that
// follows the tree -- page "The Architecture of Diagnosis", section "Phase 1:
// Custom CUDA Kernels", item 2 -- and give the latent row as kv_lora_rank=512
// plus qk_rope_head_dim=64 -- page "From Diagnosis to Deployment", section
// "The Second Thread"). The plainest reading, standard MLA:
//
//   Anc*(t) = {t, parent[t], parent[parent[t]], ...}            (self included)
//   V(t)    = {0..L-1} U {L+u : u in Anc*(t)}                    (visible keys)
//   non-absorbed:  k_n[h,j] = c_kv[j]^T W_UK[h],  v[h,j] = c_kv[j]^T W_UV[h]
//                  s = scale*(q_nope.k_n + q_rope.k_rope[j]),  p = softmax_V(t)(s)
//                  out = sum_j p_j v[h,j],  lse = ln sum_{j in V(t)} exp(s_j)
//   absorbed:      q_lat = W_UK[h] q_nope,  s = scale*(q_lat.c_kv[j] + q_rope.k_rope[j])
//                  o_lat = sum_j p_j c_kv[j],  out = W_UV[h]^T o_lat
//   split/combine: a partition of V(t) into parts k gives (o_k, lse_k); then
//                  LSE = ln sum_k exp(lse_k), O = sum_k exp(lse_k - LSE) o_k
//                  (the prefix / tree-tail merge the page "The Three Acts of
//                  Engineering", reference [1], describes as one kernel for the
//                  long prefix and another for the small tree tail).
//
// Inputs are float32 storage holding the exact (bf16-rounded, for bf16 runs)
// values handed to the GPU; every sum here is a plain left-to-right loop in
// double. Softmax uses the two-pass maximum. Rows are spread over threads
// (rows are independent, so this reorders no arithmetic).
#include <algorithm>
#include <cmath>
#include <cstdint>
#include <cstring>
#include <limits>
#include <thread>
#include <vector>

namespace {

// Visible tree nodes of node t: walk parent[] from t to the root.
// Returns false when the walk leaves [0, T) or does not terminate in T steps.
bool ancestors(const int32_t* parent, int32_t T, int32_t t, std::vector<int32_t>& out) {
  out.clear();
  int32_t u = t;
  for (int32_t steps = 0; steps <= T; ++steps) {
    if (u < 0 || u >= T) return false;
    out.push_back(u);
    int32_t p = parent[u];
    if (p == -1) return true;
    if (p >= u) return false;   // parents come before children (discovery order)
    u = p;
  }
  return false;
}

template <class F>
void parallel_rows(int64_t n, int n_threads, F f) {
  if (n_threads <= 0) n_threads = (int)std::max(1u, std::thread::hardware_concurrency());
  if (n_threads > n) n_threads = (int)std::max<int64_t>(1, n);
  std::vector<std::thread> pool;
  for (int w = 0; w < n_threads; ++w) {
    pool.emplace_back([=]() {
      for (int64_t i = w; i < n; i += n_threads) f(i);
    });
  }
  for (auto& th : pool) th.join();
}

}  // namespace

extern "C" {

// Ancestor bitmask of one tree: bit u of mask[t] is set iff u is t or an
// ancestor of t; depth[t] = number of edges to the root. Returns 0, or -1 when
// parent[] is not a discovery-ordered forest (or T > 64).
int oracle_tree_mask(const int32_t* parent, int32_t T, uint64_t* mask, int32_t* depth) {
  if (T < 0 || T > 64) return -1;
  std::vector<int32_t> anc;
  for (int32_t t = 0; t < T; ++t) {
    if (!ancestors(parent, T, t, anc)) return -1;
    uint64_t m = 0;
    for (int32_t u : anc) m |= (uint64_t)1 << u;
    mask[t] = m;
    if (depth) depth[t] = (int32_t)anc.size() - 1;
  }
  return 0;
}

// Absorbed-form verify attention for ONE request, restricted to the logical
// key range [key_lo, key_hi) (a split; pass 0, L+T for the whole row).
//   q      : [T*H][D_c+D_r], row (t*H + h) = q_lat || q_rope
//   pool   : [*][D_c+D_r] latent rows c_kv || k_rope
//   logical key j lives in pool row page_table[j] (page_table != NULL) or
//   kv_base + j (page_table == NULL)
//   rows   : optional list of row indices to evaluate (n_rows of them);
//            NULL means all T*H rows in order
//   o      : [n_rows][D_c]   o_lat = sum_j p_j c_kv[j]
//   lse    : [n_rows]        natural-log sum of exp(s_j) over visible keys;
//            an empty visible set gives o = 0 and lse = -inf
// Returns 0, or -1 on a malformed tree / index.
int oracle_verify_absorbed(int32_t H, int32_t T, int32_t L, int32_t D_c, int32_t D_r,
                           double scale, const float* q, const float* pool, int64_t num_slots,
                           const int32_t* page_table, int64_t kv_base, const int32_t* parent,
                           int32_t key_lo, int32_t key_hi, const int32_t* rows, int64_t n_rows,
                           double* o, double* lse, int n_threads) {
  const int32_t D_q = D_c + D_r;
  const int32_t n_keys = L + T;
  if (key_lo < 0) key_lo = 0;
  if (key_hi > n_keys) key_hi = n_keys;
  // visibility of tree node keys per node
  std::vector<std::vector<char>> tree_vis(T, std::vector<char>(T, 0));
  std::vector<int32_t> anc;
  for (int32_t t = 0; t < T; ++t) {
    if (!ancestors(parent, T, t, anc)) return -1;
    for (int32_t u : anc) tree_vis[t][u] = 1;
  }
  // logical key -> pool row
  std::vector<int64_t> slot(n_keys);
  for (int32_t j = 0; j < n_keys; ++j) {
    int64_t s = page_table ? (int64_t)page_table[j] : kv_base + j;
    if (s < 0 || s >= num_slots) return -1;
    slot[j] = s;
  }
  if (rows == nullptr) n_rows = (int64_t)T * H;
  for (int64_t i = 0; i < n_rows; ++i) {
    int64_t r = rows ? rows[i] : i;
    if (r < 0 || r >= (int64_t)T * H) return -1;
  }
  parallel_rows(n_rows, n_threads, [&](int64_t i) {
    const int64_t r = rows ? rows[i] : i;
    const int32_t t = (int32_t)(r / H);
    const float* qr = q + r * D_q;
    // pass 1: logits of visible keys and their maximum
    std::vector<int32_t> keys;
    std::vector<double> s;
    double m = -std::numeric_limits<double>::infinity();
    for (int32_t j = key_lo; j < key_hi; ++j) {
      bool visible = (j < L) || tree_vis[t][j - L];
      if (!visible) continue;
      const float* kr = pool + slot[j] * D_q;
      double dot_lat = 0.0;
      for (int32_t c = 0; c < D_c; ++c) dot_lat += (double)qr[c] * (double)kr[c];
      double dot_rope = 0.0;
      for (int32_t c = D_c; c < D_q; ++c) dot_rope += (double)qr[c] * (double)kr[c];
      double sj = scale * (dot_lat + dot_rope);
      keys.push_back(j);
      s.push_back(sj);
      if (sj > m) m = sj;
    }
    double* orow = o + i * D_c;
    for (int32_t c = 0; c < D_c; ++c) orow[c] = 0.0;
    if (keys.empty()) {
      lse[i] = -std::numeric_limits<double>::infinity();
      return;
    }
    // pass 2: p_j = exp(s_j - m), l = sum p_j, o = sum p_j c_kv[j] / l
    double l = 0.0;
    for (size_t k = 0; k < keys.size(); ++k) {
      double p = std::exp(s[k] - m);
      l += p;
      const float* kr = pool + slot[keys[k]] * D_q;
      for (int32_t c = 0; c < D_c; ++c) orow[c] += p * (double)kr[c];
    }
    for (int32_t c = 0; c < D_c; ++c) orow[c] /= l;
    lse[i] = m + std::log(l);
  });
  return 0;
}

// Non-absorbed (explicit K and V) MLA attention for ONE request with a
// contiguous logical KV (c_kv [L+T][D_c], k_rope [L+T][D_r]).
//   q_nope [T*H][D_n], q_rope [T*H][D_r], W_UK [H][D_c][D_n], W_UV [H][D_c][D_v]
//   out [T*H][D_v], lse [T*H]
int oracle_verify_mla(int32_t H, int32_t T, int32_t L, int32_t D_c, int32_t D_r, int32_t D_n,
                      int32_t D_v, double scale, const float* q_nope, const float* q_rope,
                      const float* c_kv, const float* k_rope, const float* w_uk,
                      const float* w_uv, const int32_t* parent, double* out, double* lse,
                      int n_threads) {
  const int32_t n_keys = L + T;
  std::vector<std::vector<char>> tree_vis(T, std::vector<char>(T, 0));
  std::vector<int32_t> anc;
  for (int32_t t = 0; t < T; ++t) {
    if (!ancestors(parent, T, t, anc)) return -1;
    for (int32_t u : anc) tree_vis[t][u] = 1;
  }
  // explicit per-head keys and values: k_n[h][j][n], v[h][j][e]
  std::vector<double> k_n((size_t)H * n_keys * D_n), v((size_t)H * n_keys * D_v);
  parallel_rows((int64_t)H * n_keys, n_threads, [&](int64_t idx) {
    const int64_t h = idx / n_keys, j = idx % n_keys;
    const float* c = c_kv + j * D_c;
    for (int32_t n = 0; n < D_n; ++n) {
      double acc = 0.0;
      for (int32_t a = 0; a < D_c; ++a) acc += (double)c[a] * (double)w_uk[(h * D_c + a) * D_n + n];
      k_n[(h * n_keys + j) * D_n + n] = acc;
    }
    for (int32_t e = 0; e < D_v; ++e) {
      double acc = 0.0;
      for (int32_t a = 0; a < D_c; ++a) acc += (double)c[a] * (double)w_uv[(h * D_c + a) * D_v + e];
      v[(h * n_keys + j) * D_v + e] = acc;
    }
  });
  parallel_rows((int64_t)T * H, n_threads, [&](int64_t r) {
    const int32_t t = (int32_t)(r / H), h = (int32_t)(r % H);
    std::vector<int32_t> keys;
    std::vector<double> s;
    double m = -std::numeric_limits<double>::infinity();
    for (int32_t j = 0; j < n_keys; ++j) {
      if (!(j < L || tree_vis[t][j - L])) continue;
      double dn = 0.0;
      for (int32_t n = 0; n < D_n; ++n)
        dn += (double)q_nope[r * D_n + n] * k_n[((int64_t)h * n_keys + j) * D_n + n];
      double dr = 0.0;
      for (int32_t c = 0; c < D_r; ++c) dr += (double)q_rope[r * D_r + c] * (double)k_rope[(int64_t)j * D_r + c];
      double sj = scale * (dn + dr);
      keys.push_back(j);
      s.push_back(sj);
      if (sj > m) m = sj;
    }
    double l = 0.0;
    double* orow = out + r * D_v;
    for (int32_t e = 0; e < D_v; ++e) orow[e] = 0.0;
    for (size_t k = 0; k < keys.size(); ++k) {
      double p = std::exp(s[k] - m);
      l += p;
      for (int32_t e = 0; e < D_v; ++e) orow[e] += p * v[((int64_t)h * n_keys + keys[k]) * D_v + e];
    }
    for (int32_t e = 0; e < D_v; ++e) orow[e] /= l;
    lse[r] = m + std::log(l);
  });
  return 0;
}

// q_lat[r][a] = sum_n W_UK[h][a][n] q_nope[r][n], r = t*H + h.
void oracle_absorb_q(int32_t H, int64_t rows, int32_t D_c, int32_t D_n, const float* q_nope,
                     const float* w_uk, double* q_lat, int n_threads) {
  parallel_rows(rows, n_threads, [&](int64_t r) {
    const int64_t h = r % H;
    for (int32_t a = 0; a < D_c; ++a) {
      double acc = 0.0;
      for (int32_t n = 0; n < D_n; ++n)
        acc += (double)w_uk[(h * D_c + a) * D_n + n] * (double)q_nope[r * D_n + n];
      q_lat[r * D_c + a] = acc;
    }
  });
}

// out[r][e] = sum_a W_UV[h][a][e] o_lat[r][a], r = t*H + h.
void oracle_unabsorb_o(int32_t H, int64_t rows, int32_t D_c, int32_t D_v, const double* o_lat,
                       const float* w_uv, double* out, int n_threads) {
  parallel_rows(rows, n_threads, [&](int64_t r) {
    const int64_t h = r % H;
    for (int32_t e = 0; e < D_v; ++e) {
      double acc = 0.0;
      for (int32_t a = 0; a < D_c; ++a)
        acc += (double)w_uv[(h * D_c + a) * D_v + e] * o_lat[r * D_c + a];
      out[r * D_v + e] = acc;
    }
  });
}

// Merge S partial results per row: LSE = ln sum_k exp(lse_k),
// o = sum_k exp(lse_k - LSE) o_k. Parts with lse_k = -inf weigh nothing; a row
// whose parts are all empty gets o = 0, LSE = -inf.
//   o_part [S][rows][d], lse_part [S][rows]
void oracle_combine(int32_t S, int64_t rows, int32_t d, const double* o_part,
                    const double* lse_part, double* o, double* lse) {
  const double NEG_INF = -std::numeric_limits<double>::infinity();
  for (int64_t r = 0; r < rows; ++r) {
    double m = NEG_INF;
    for (int32_t k = 0; k < S; ++k) m = std::max(m, lse_part[(int64_t)k * rows + r]);
    double* orow = o + r * d;
    for (int32_t c = 0; c < d; ++c) orow[c] = 0.0;
    if (m == NEG_INF) {
      lse[r] = NEG_INF;
      continue;
    }
    double z = 0.0;
    for (int32_t k = 0; k < S; ++k) z += std::exp(lse_part[(int64_t)k * rows + r] - m);
    const double LSE = m + std::log(z);
    for (int32_t k = 0; k < S; ++k) {
      const double lk = lse_part[(int64_t)k * rows + r];
      if (lk == NEG_INF) continue;
      const double w = std::exp(lk - LSE);
      for (int32_t c = 0; c < d; ++c) orow[c] += w * o_part[((int64_t)k * rows + r) * d + c];
    }
    lse[r] = LSE;
  }
}

// ---------------------------------------------------------------------------
// Greedy tree acceptance: the step after verification, which keeps the longest
// run of draft tokens that the target model agrees with (page "The
// Architecture of Diagnosis", section "Phase 1: Custom CUDA Kernels", item 3:
// a device-side kernel picks the longest accepted prefix after verification).
// The page gives no formula; the reading used here:
//
//   target[t] = argmax_v logits[t][v]: the lowest v among equal maxima; NaN
//               entries never win; a row that is all NaN (or empty) gives 0.
//   accepted  : a root (parent -1) is accepted; node u with parent p is
//               accepted iff p is accepted and token[u] == target[p].
//   end       : the accepted node of greatest depth, the lowest index among
//               equal depths.
//   path      : end's ancestor chain, root first; len = depth(end) + 1.
//   bonus     : target[end], the target's own next token after the path.
//   commit    : (page-table KV) logical key L+i of the request becomes the slot
//               of path[i], for i < len -- the accepted nodes' KV rows move
//               to the front of the tree region without copying any row; the
//               other nodes' slots follow in node order.

// target[r] for `rows` rows of `vocab` values (row stride ld). The values are
// float32 storage (bf16 values are exact in it); plain comparisons decide.
void oracle_argmax(int64_t rows, int64_t vocab, const float* logits, int64_t ld,
                   int32_t* target) {
  for (int64_t r = 0; r < rows; ++r) {
    const float* x = logits + r * ld;
    int64_t best = -1;
    for (int64_t v = 0; v < vocab; ++v) {
      if (std::isnan(x[v])) continue;
      if (best < 0 || x[v] > x[best]) best = v;   // strict: equal values keep the lower v
    }
    target[r] = (int32_t)(best < 0 ? 0 : best);
  }
}

// Acceptance of ONE tree of T nodes. path must hold T entries; entries past
// len are set to -1. Returns 0, or -1 when parent[] is not a discovery-ordered
// forest (or T is not in [1, 64]).
int oracle_tree_accept(int32_t T, const int32_t* parent, const int32_t* token,
                       const int32_t* target, int32_t* path, int32_t* len, int32_t* bonus) {
  if (T < 1 || T > 64) return -1;
  std::vector<char> accepted(T, 0);
  std::vector<int32_t> depth(T, 0);
  for (int32_t u = 0; u < T; ++u) {
    const int32_t p = parent[u];
    if (p == -1) {
      accepted[u] = 1;
      depth[u] = 0;
    } else if (p >= 0 && p < u) {
      accepted[u] = accepted[p] && token[u] == target[p];
      depth[u] = depth[p] + 1;
    } else {
      return -1;
    }
  }
  int32_t end = -1;
  for (int32_t u = 0; u < T; ++u)
    if (accepted[u] && (end < 0 || depth[u] > depth[end])) end = u;
  const int32_t n = depth[end] + 1;
  for (int32_t i = 0; i < T; ++i) path[i] = -1;
  for (int32_t u = end, i = n - 1; i >= 0; --i, u = parent[u]) path[i] = u;
  *len = n;
  *bonus = target[end];
  return 0;
}

// Page-table commit of one request: pt is the request's logical->slot table
// ([L+T] entries). The tree region [L, L+T) is reordered: first the slots of
// the accepted path in path order, then the slots of the other nodes in node
// order, so the table stays a permutation and the rejected nodes' slots end
// up at [L+len, L+T) where the caller can recycle them.
void oracle_accept_commit(int32_t L, int32_t T, int32_t len, const int32_t* path, int32_t* pt) {
  std::vector<int32_t> old(pt + L, pt + L + T);
  std::vector<char> on_path(T, 0);
  int32_t k = 0;
  for (int32_t i = 0; i < len; ++i) {
    pt[L + k++] = old[path[i]];
    on_path[path[i]] = 1;
  }
  for (int32_t u = 0; u < T; ++u)
    if (!on_path[u]) pt[L + k++] = old[u];
}

}  // extern "C"

// ---------------------------------------------------------------------------
// Best-first draft-tree construction (page "The Architecture of Diagnosis",
// section "Phase 1: Custom CUDA Kernels", item 1: a GPU-resident builder
// replaces a host heap that grows the draft tree best-first). The page gives
// no scoring; the reading used here follows a block drafter that proposes K
// candidate tokens with log-probabilities for each of D future positions:
//
//   node   = root (depth 0, the last committed token) or a path of candidate
//            choices (j_1, ..., j_d), one per position 1..d (depth d <= D)
//   score  = fp32 sum of logp[i-1][j_i] along the path, accumulated root-first
//            (child = parent + logp, one float add)
//   order  = score descending, ties by the path compared digit by digit
//            (a prefix first, then the smaller candidate index)
//   tree   = the first T nodes in that order, emitted in that order with
//            parent = output index of the node's parent (-1 for the root).
// With every logp <= 0 a node never outranks its parent, so this is exactly
// what a best-first expansion (pop the best frontier node, push its K
// children) emits. Done here as that expansion with a linear frontier scan.
// A NaN log-probability is read as -inf (a candidate never preferred), and so
// is a NaN path score (+inf plus -inf along one path): both keep the order
// total.

namespace {
struct Cand { float score; uint64_t key; int32_t depth, parent, token; bool live; };
// true when a ranks before b
bool cand_before(const Cand& a, const Cand& b) {
  if (a.score != b.score) return a.score > b.score;
  return a.key < b.key;
}
}  // namespace

extern "C" {

// Returns the number of nodes emitted (T unless the candidates run out first),
// or -1 on bad sizes (T < 1, D > 16, K > 8).
int oracle_tree_build(int32_t T, int32_t D, int32_t K, int32_t root_token, const int32_t* cand_token,
                      const float* cand_logp, int32_t* parent, int32_t* token, int32_t* depth, float* score) {
  if (T < 1 || D < 0 || D > 16 || K < 1 || K > 8) return -1;
  std::vector<Cand> f;
  f.push_back(Cand{0.0f, 0u, 0, -1, root_token, true});
  int32_t n = 0;
  for (; n < T; ++n) {
    int best = -1;
    for (int i = 0; i < (int)f.size(); ++i)
      if (f[i].live && (best < 0 || cand_before(f[i], f[best]))) best = i;
    if (best < 0) break;
    Cand c = f[best];
    f[best].live = false;
    parent[n] = c.parent;
    token[n] = c.token;
    depth[n] = c.depth;
    score[n] = c.score;
    if (c.depth < D) {
      for (int32_t j = 0; j < K; ++j) {
        float lp = cand_logp[(int64_t)c.depth * K + j];
        if (std::isnan(lp)) lp = -std::numeric_limits<float>::infinity();   // never preferred
        float s = c.score + lp;
        // +inf + -inf: a path with no defined score is never preferred either
        if (std::isnan(s)) s = -std::numeric_limits<float>::infinity();
        // the path as D base-(K+1) digits, most significant first, 0 past
        // the end: numeric order = digit-by-digit order with a prefix first
        uint64_t place = 1;
        for (int32_t e = c.depth + 1; e < D; ++e) place *= (uint64_t)(K + 1);
        const uint64_t key = c.key + (uint64_t)(j + 1) * place;
        f.push_back(Cand{s, key, c.depth + 1, n, cand_token[(int64_t)c.depth * K + j], true});
      }
    }
  }
  return n;
}

}  // extern "C"

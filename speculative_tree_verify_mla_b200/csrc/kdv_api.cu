// kdv_api.cu -- the C ABI: argument checks, split planning, launches.
#include <cuda_runtime.h>

#include <algorithm>
#include <climits>
#include <cmath>
#include <cstring>

#include "kdv_internal.cuh"

using namespace kdv;

namespace {

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

int device_sm_count() {
  int dev = 0, n = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) { cudaGetLastError(); return 148; }
  if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || n <= 0) {
    cudaGetLastError();
    return 148;
  }
  return n;
}

// The tensor-core kernel: bf16, the Kimi / DeepSeek-V3 latent dims, and a
// positive softmax scale (its row maxima are taken over unscaled logits).
bool tc_shape_ok(const kdv_verify_params* p) {
  return p->dtype == KDV_BF16 && p->d_latent == 512 && p->d_rope == 64 && p->scale > 0.f;
}

bool is_tc(int impl) { return impl == KDV_IMPL_TC || impl == KDV_IMPL_TC_STAGED; }
// the 2-SM kernel, reading the pool directly or a staged copy
bool is_tc2(int impl) { return impl == KDV_IMPL_TC || impl == KDV_IMPL_TC_STAGED; }

// AUTO: the tensor-core kernel when its shape constraints hold, reading a
// paged pool through a staged contiguous copy (the fastest path, at the
// price of workspace for the copy); else SIMT.
int resolve_impl(const kdv_verify_params* p) {
  if (p->impl == KDV_IMPL_SIMT || is_tc(p->impl)) return p->impl;
  if (!tc_shape_ok(p)) return KDV_IMPL_SIMT;
  return p->page_table != nullptr ? KDV_IMPL_TC_STAGED : KDV_IMPL_TC;
}

// Host-side checks that need no device access.
kdv_status check_params(const kdv_verify_params* p, int impl) {
  if (p == nullptr) return KDV_ERR_INVALID_ARG;
  if (p->batch < 1) return KDV_ERR_INVALID_ARG;
  if (p->batch > KDV_MAX_BATCH) return KDV_ERR_UNSUPPORTED;
  if (p->num_heads < 1) return KDV_ERR_INVALID_ARG;
  if (p->dtype != KDV_BF16 && p->dtype != KDV_F32) return KDV_ERR_INVALID_ARG;
  if (p->impl < KDV_IMPL_AUTO || p->impl > KDV_IMPL_TC_STAGED) return KDV_ERR_INVALID_ARG;
  if (p->impl == KDV_IMPL_TC_1SM) return KDV_ERR_UNSUPPORTED;   // retired 1-SM-MMA variant
  if (p->d_latent < 1 || p->d_rope < 0) return KDV_ERR_INVALID_ARG;
  if (!std::isfinite(p->scale)) return KDV_ERR_INVALID_ARG;
  if (p->h_prefix_len == nullptr || p->h_tree_T == nullptr) return KDV_ERR_INVALID_ARG;
  for (int b = 0; b < p->batch; ++b) {
    if (p->h_prefix_len[b] < 0) return KDV_ERR_INVALID_ARG;
    if (p->h_tree_T[b] < 1) return KDV_ERR_INVALID_ARG;
    if (p->h_tree_T[b] > KDV_MAX_TREE) return KDV_ERR_UNSUPPORTED;
  }
  if (p->num_splits < 0) return KDV_ERR_INVALID_ARG;
  if (p->return_partials != 0 && p->return_partials != 1) return KDV_ERR_INVALID_ARG;
  if (p->return_partials && p->num_splits < 1) return KDV_ERR_INVALID_ARG;
  if (is_tc(impl)) {
    if (!tc_shape_ok(p)) return KDV_ERR_UNSUPPORTED;
  } else {
    if (p->d_latent > 512 || p->d_rope > 64) return KDV_ERR_UNSUPPORTED;
  }
  return KDV_OK;
}

kdv_status check_pointers(const kdv_verify_params* p, int impl) {
  const int64_t D_q = (int64_t)p->d_latent + p->d_rope;
  const int64_t stride = p->q_row_stride == 0 ? D_q : p->q_row_stride;
  if (stride < D_q) return KDV_ERR_INVALID_ARG;
  if (!p->q || !p->kv || !p->kv_off || !p->tree_off || !p->mask) return KDV_ERR_INVALID_ARG;
  if (p->num_slots < 0) return KDV_ERR_INVALID_ARG;
  if (p->return_partials) {
    if (!p->o_part || !p->lse_part) return KDV_ERR_INVALID_ARG;
  } else if (!p->o) {
    return KDV_ERR_INVALID_ARG;
  }
  const size_t esz = p->dtype == KDV_BF16 ? 2 : 4;
  if ((reinterpret_cast<uintptr_t>(p->q) % esz) || (reinterpret_cast<uintptr_t>(p->kv) % esz))
    return KDV_ERR_INVALID_ARG;
  if (is_tc(impl)) {
    // TMA needs 16-byte aligned bases and row pitches; the epilogue writes
    // o / o_part rows in 16-byte vectors
    if (!aligned16(p->q) || !aligned16(p->kv)) return KDV_ERR_INVALID_ARG;
    if ((stride * (int64_t)esz) % 16 != 0) return KDV_ERR_INVALID_ARG;
    if ((p->o && !aligned16(p->o)) || (p->o_part && !aligned16(p->o_part))) return KDV_ERR_INVALID_ARG;
    if (p->v16 && !aligned16(p->v16)) return KDV_ERR_INVALID_ARG;
  }
  float* outs[4] = {p->o, p->lse, p->o_part, p->lse_part};
  for (float* f : outs)
    if (f && (reinterpret_cast<uintptr_t>(f) & 3u)) return KDV_ERR_INVALID_ARG;
  return KDV_OK;
}

size_t align256(size_t n) { return (n + 255) & ~(size_t)255; }

// Partial rows of a plan (every request's S_b * T_b * H).
size_t plan_parts(const VerifyPlan& plan) {
  return (size_t)plan.part_base[plan.B - 1] + (size_t)plan.S[plan.B - 1] * plan.T[plan.B - 1] * plan.H;
}
// Bytes of o_k at the start of the workspace (256-aligned), then lse_k fp32.
size_t merge_o_bytes(const VerifyPlan& plan, int32_t d) {
  return align256(plan_parts(plan) * (size_t)d * (plan.part_f16 ? 2 : 4));
}
size_t merge_region_bytes(const VerifyPlan& plan, int32_t d) {
  return merge_o_bytes(plan, d) + plan_parts(plan) * sizeof(float);
}
// Keys a call reads, over all requests.
int64_t plan_keys(const VerifyPlan& plan) {
  int64_t n = 0;
  for (int b = 0; b < plan.B; ++b) n += (int64_t)plan.L[b] + plan.T[b];
  return n;
}
// Workspace layout: [merge partials (OUT_WORKSPACE)] [fp16 latent rows (TC)]
// [staged rows (TC_STAGED with a page table)], each region 256-byte aligned.
size_t v16_offset(const VerifyPlan& plan, int32_t d) {
  return plan.out_mode == OUT_WORKSPACE ? align256(merge_region_bytes(plan, d)) : 0;
}
size_t v16_bytes(const VerifyPlan& plan) { return (size_t)plan_keys(plan) * 512 * 2; }

// KDV_IMPL_TC_STAGED with a page table: the pool rows are first copied to a
// contiguous staged region of the workspace.
bool staged_paged(const kdv_verify_params* p, int impl) {
  return impl == KDV_IMPL_TC_STAGED && p->page_table != nullptr;
}

// Build the grid / split plan. Fills *ws_bytes with the workspace needed.
kdv_status make_plan(const kdv_verify_params* p, int impl, VerifyPlan* plan, size_t* ws_bytes) {
  std::memset(plan, 0, sizeof(*plan));
  const int B = p->batch, H = p->num_heads;
  const int rows_per_tile = is_tc2(impl) ? TC2_ROWS : SIMT_ROWS;
  plan->B = B;
  plan->H = H;
  plan->rows_per_tile = rows_per_tile;
  int64_t tree_acc = 0;
  for (int b = 0; b < B; ++b) {
    plan->L[b] = p->h_prefix_len[b];
    plan->T[b] = p->h_tree_T[b];
    plan->tree_base[b] = (int32_t)tree_acc;
    tree_acc += p->h_tree_T[b];
    const int64_t rows_b = (int64_t)p->h_tree_T[b] * H;
    const int64_t tiles = (rows_b + rows_per_tile - 1) / rows_per_tile;
    if (tiles > INT_MAX / 2 || rows_b > INT_MAX / 2) return KDV_ERR_UNSUPPORTED;
    plan->tiles[b] = (int32_t)tiles;
  }
  if (tree_acc * (int64_t)H > INT_MAX / 2) return KDV_ERR_UNSUPPORTED;
  plan->total_rows = (int32_t)(tree_acc * H);

  // splits per request
  const int sms = device_sm_count();
  // TC: one item is a 4-CTA cluster; clusters only fit within
  // a GPC, so one wave is what the occupancy query reports (fallback: the SM
  // count divided by the cluster size). SIMT: 8-warp CTAs, several per SM.
  double target_items = 4.0 * sms;
  if (is_tc2(impl)) {
    const int n = tc2_max_active_clusters();
    target_items = n > 0 ? n : sms / 4;
  }
  const int min_keys = is_tc(impl) ? 2 * TC_KEYS : 128;
  // Automatic splits: choose the chunk X (a multiple of SPLIT_ALIGN keys, at
  // least min_keys) that minimises a simple cost model of the kernel, in
  // units of keys processed by one work item:
  //   items(X) = sum_b tiles_b * ceil(n_b / X)
  //   one wave  (items <= clusters): the longest item, X + C
  //   more waves: (sum_b tiles_b * n_b + items * C) / clusters + (X + C) / 2
  // C = ITEM_OVERHEAD_KEYS is the fixed cost of an item (query load, pipeline
  // fill, epilogue and the partials it writes) measured on B200 as ~20 us
  // against ~7 us per 256 keys of steady-state work, i.e. ~740 keys.
  constexpr double ITEM_OVERHEAD_KEYS = 768.0;
  int64_t max_n = 1;
  double work_keys = 0.0;
  for (int b = 0; b < B; ++b) {
    max_n = std::max<int64_t>(max_n, (int64_t)plan->L[b] + plan->T[b]);
    work_keys += (double)plan->tiles[b] * ((double)plan->L[b] + plan->T[b]);
  }
  auto items_for = [&](int64_t X) {
    double n = 0.0;
    for (int b = 0; b < B; ++b)
      n += (double)plan->tiles[b] * (double)(((int64_t)plan->L[b] + plan->T[b] + X - 1) / X);
    return n;
  };
  auto cost = [&](int64_t X) {
    const double n = items_for(X), C = ITEM_OVERHEAD_KEYS;
    if (n <= target_items) return (double)X + C;
    return (work_keys + n * C) / target_items + 0.5 * ((double)X + C);
  };
  const int64_t align = SPLIT_ALIGN;
  const int64_t x_lo = std::max<int64_t>(min_keys, align);
  const int64_t x_hi = std::max<int64_t>(x_lo, ((max_n + align - 1) / align) * align);
  int64_t best_x = x_hi;
  double best_cost = cost(x_hi);
  for (double xf = (double)x_lo; xf < (double)x_hi; xf *= 1.05) {     // ~100 candidates
    const int64_t X = std::max(x_lo, ((int64_t)xf / align) * align);
    const double cx = cost(X);
    if (cx < best_cost) {
      best_cost = cx;
      best_x = X;
    }
  }
  const int64_t hi = best_x;
  const int64_t X = hi;
  for (int b = 0; b < B; ++b) {
    const int64_t n_b = (int64_t)plan->L[b] + plan->T[b];
    int64_t S;
    if (p->num_splits >= 1) {
      S = p->num_splits;
    } else {
      S = std::max<int64_t>(1, (n_b + X - 1) / X);
    }
    if (S > 4096) return KDV_ERR_UNSUPPORTED;
    const int64_t chunk = SPLIT_ALIGN * ((n_b + SPLIT_ALIGN * S - 1) / (SPLIT_ALIGN * S));
    plan->S[b] = (int32_t)S;
    plan->chunk[b] = (int32_t)std::max<int64_t>(chunk, SPLIT_ALIGN);
  }
  int64_t items = 0, parts = 0;
  bool all_one = true;
  for (int b = 0; b < B; ++b) {
    plan->item_base[b] = (int32_t)items;
    items += (int64_t)plan->tiles[b] * plan->S[b];
    plan->part_base[b] = (int32_t)parts;
    parts += (int64_t)plan->S[b] * plan->T[b] * H;
    if (plan->S[b] != 1) all_one = false;
    if (items > INT_MAX / 4 || parts > INT_MAX / 4) return KDV_ERR_UNSUPPORTED;
  }
  plan->item_base[B] = (int32_t)items;
  plan->n_items = (int32_t)items;
  int64_t v16_rows = 0;
  for (int b = 0; b < B; ++b) {
    plan->v16_base[b] = (int32_t)v16_rows;
    v16_rows += (int64_t)plan->L[b] + plan->T[b];
    if (v16_rows > INT_MAX / 2) return KDV_ERR_UNSUPPORTED;
  }
  *ws_bytes = 0;
  if (p->return_partials) {
    plan->out_mode = OUT_PARTIALS;
  } else if (all_one) {
    plan->out_mode = OUT_DIRECT;
  } else {
    // the merge's partials: fp16 o_k from the tensor-core kernel (its outputs
    // are convex combinations of c_kv values, which that kernel already
    // requires to lie in fp16's range), fp32 from the SIMT kernel
    plan->out_mode = OUT_WORKSPACE;
    plan->part_f16 = is_tc2(impl) ? 1 : 0;
    *ws_bytes = merge_region_bytes(*plan, p->d_latent);
  }
  if (is_tc2(impl) && p->v16 == nullptr) *ws_bytes = v16_offset(*plan, p->d_latent) + align256(v16_bytes(*plan));
  if (staged_paged(p, impl)) {
    // after the fp16 rows: staged row offsets [B+1], the staged k_rope rows
    // [keys][D_r], then q_lat in fp16 [total_rows][D_c]
    const size_t n_keys = (size_t)plan_keys(*plan);
    *ws_bytes = align256(*ws_bytes) + align256((size_t)(B + 1) * sizeof(int32_t)) +
                align256(n_keys * (size_t)p->d_rope * 2) + (size_t)plan->total_rows * p->d_latent * 2;
  }
  return KDV_OK;
}

kdv_status cuda_status(cudaError_t e) { return e == cudaSuccess ? KDV_OK : KDV_ERR_CUDA; }

}  // namespace

extern "C" {

const char* kdv_status_string(kdv_status s) {
  switch (s) {
    case KDV_OK: return "KDV_OK";
    case KDV_ERR_INVALID_ARG: return "KDV_ERR_INVALID_ARG: null, misaligned or out-of-range argument";
    case KDV_ERR_UNSUPPORTED: return "KDV_ERR_UNSUPPORTED: valid request the library does not implement";
    case KDV_ERR_WORKSPACE: return "KDV_ERR_WORKSPACE: workspace missing or too small";
    case KDV_ERR_CUDA: return "KDV_ERR_CUDA: a CUDA launch or runtime call failed";
  }
  return "KDV_ERR_UNKNOWN";
}

int32_t kdv_version(void) { return 123; }

kdv_status kdv_tree_mask_build(const int32_t* parent, const int32_t* tree_off, int32_t batch,
                               int32_t max_T, uint64_t* mask, int32_t* depth, int32_t* d_err,
                               void* stream) {
  if (parent == nullptr || mask == nullptr) return KDV_ERR_INVALID_ARG;
  if (batch < 1 || max_T < 1) return KDV_ERR_INVALID_ARG;
  if (max_T > KDV_MAX_TREE) return KDV_ERR_UNSUPPORTED;
  if (tree_off == nullptr && batch != 1) return KDV_ERR_INVALID_ARG;
  if (reinterpret_cast<uintptr_t>(mask) & 7u) return KDV_ERR_INVALID_ARG;
  return cuda_status(launch_mask_build(parent, tree_off, batch, max_T, mask, depth, d_err,
                                       static_cast<cudaStream_t>(stream)));
}

kdv_status kdv_verify_attn_workspace(const kdv_verify_params* p, size_t* bytes) {
  if (p == nullptr || bytes == nullptr) return KDV_ERR_INVALID_ARG;
  const int impl = resolve_impl(p);
  kdv_status st = check_params(p, impl);
  if (st != KDV_OK) return st;
  VerifyPlan plan;
  return make_plan(p, impl, &plan, bytes);
}

kdv_status kdv_verify_attn_plan(const kdv_verify_params* p, int32_t* splits, int32_t* grid_items) {
  if (p == nullptr) return KDV_ERR_INVALID_ARG;
  const int impl = resolve_impl(p);
  kdv_status st = check_params(p, impl);
  if (st != KDV_OK) return st;
  VerifyPlan plan;
  size_t bytes = 0;
  st = make_plan(p, impl, &plan, &bytes);
  if (st != KDV_OK) return st;
  if (splits)
    for (int b = 0; b < plan.B; ++b) splits[b] = plan.S[b];
  if (grid_items) *grid_items = plan.n_items;
  return KDV_OK;
}

kdv_status kdv_verify_attn_launches(const kdv_verify_params* p, int32_t* launches) {
  if (p == nullptr || launches == nullptr) return KDV_ERR_INVALID_ARG;
  const int impl = resolve_impl(p);
  kdv_status st = check_params(p, impl);
  if (st != KDV_OK) return st;
  VerifyPlan plan;
  size_t bytes = 0;
  st = make_plan(p, impl, &plan, &bytes);
  if (st != KDV_OK) return st;
  int32_t n = 1;                                                   // the attention kernel
  if ((is_tc2(impl) && p->v16 == nullptr) || staged_paged(p, impl)) ++n;   // the latent pass
  if (plan.out_mode == OUT_WORKSPACE) ++n;                        // the merge
  *launches = n;
  return KDV_OK;
}

kdv_status kdv_verify_attn(const kdv_verify_params* p, void* stream) {
  if (p == nullptr) return KDV_ERR_INVALID_ARG;
  const int impl = resolve_impl(p);
  kdv_status st = check_params(p, impl);
  if (st != KDV_OK) return st;
  st = check_pointers(p, impl);
  if (st != KDV_OK) return st;
  VerifyPlan plan;
  size_t need = 0;
  st = make_plan(p, impl, &plan, &need);
  if (st != KDV_OK) return st;
  if (need > 0) {
    if (p->workspace == nullptr || p->workspace_bytes < need || !aligned16(p->workspace))
      return KDV_ERR_WORKSPACE;
  }
  VerifyArgs a = {};
  a.q = p->q;
  a.q_row_stride = p->q_row_stride == 0 ? (int64_t)p->d_latent + p->d_rope : p->q_row_stride;
  a.kv = p->kv;
  a.num_slots = p->num_slots;
  a.page_table = p->page_table;
  a.kv_off = p->kv_off;
  a.tree_off = p->tree_off;
  a.prefix_len = p->prefix_len;
  a.mask = p->mask;
  a.D_c = p->d_latent;
  a.D_r = p->d_rope;
  a.scale = p->scale;
  a.d_err = p->d_err;
  a.wait_limit_ns = p->wait_limit_ns;
  float* ws_o = nullptr;
  float* ws_l = nullptr;
  if (plan.out_mode == OUT_DIRECT) {
    a.o = p->o;
    a.lse = p->lse;
  } else if (plan.out_mode == OUT_PARTIALS) {
    a.o = p->o_part;
    a.lse = p->lse_part;
  } else {
    ws_o = static_cast<float*>(p->workspace);
    ws_l = reinterpret_cast<float*>(static_cast<char*>(p->workspace) + merge_o_bytes(plan, p->d_latent));
    a.o = ws_o;
    a.lse = ws_l;
  }
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  // One pass over the pool rows the call reads: the fp16 latent rows of the
  // P.V operand (unless the caller gave them) and, for a staged paged pool,
  // the contiguous bf16 copy the kernel then reads with tiled boxes.
  const void* v16 = p->v16;
  void* own_v16 = nullptr;
  void* staged = nullptr;
  int32_t* staged_off = nullptr;
  void* q16 = nullptr;
  if (is_tc2(impl) && v16 == nullptr) {
    own_v16 = static_cast<char*>(p->workspace) + v16_offset(plan, p->d_latent);
    v16 = own_v16;
  }
  if (staged_paged(p, impl)) {
    char* region = static_cast<char*>(p->workspace) + v16_offset(plan, p->d_latent) +
                   (p->v16 == nullptr ? align256(v16_bytes(plan)) : 0);
    staged_off = reinterpret_cast<int32_t*>(region);
    staged = region + align256((size_t)(plan.B + 1) * sizeof(int32_t));
    q16 = static_cast<char*>(staged) + align256((size_t)plan_keys(plan) * p->d_rope * 2);
  }
  if (own_v16 != nullptr || staged != nullptr) {
    if (launch_latent_f16(a, plan, own_v16, staged, staged_off, q16, s) != cudaSuccess) return KDV_ERR_CUDA;
  }
  if (staged != nullptr) {
    // the keys in logical order: latent dims from the fp16 rows, k_rope
    // from the staged rows, queries' latent dims from q16
    a.kv = staged;
    a.num_slots = plan_keys(plan);
    a.page_table = nullptr;
    a.kv_off = staged_off;
    a.q16 = q16;
  }
  // The attention kernel may start while the latent pass still runs when
  // that pass writes only the fp16 rows (not a staged pool the S side reads).
  cudaError_t e = is_tc2(impl) ? launch_verify_tc2(a, plan, v16, plan_keys(plan),
                                                   own_v16 != nullptr && staged == nullptr, s)
                               : launch_verify_simt(a, plan, p->dtype, s);
  if (e != cudaSuccess) return KDV_ERR_CUDA;
  if (plan.out_mode == OUT_WORKSPACE)
    e = launch_combine_plan(ws_o, ws_l, plan, p->d_latent, p->o, p->lse, s);
  return cuda_status(e);
}

kdv_status kdv_latent_f16(const kdv_verify_params* p, void* v16, void* stream) {
  if (p == nullptr || v16 == nullptr || !aligned16(v16)) return KDV_ERR_INVALID_ARG;
  kdv_verify_params q = *p;
  q.impl = KDV_IMPL_TC;
  kdv_status st = check_params(&q, KDV_IMPL_TC);
  if (st != KDV_OK) return st;
  if (!q.kv || !q.kv_off || !aligned16(q.kv) || q.num_slots < 0) return KDV_ERR_INVALID_ARG;
  VerifyPlan plan;
  size_t need = 0;
  st = make_plan(&q, KDV_IMPL_TC, &plan, &need);
  if (st != KDV_OK) return st;
  VerifyArgs a;
  std::memset(&a, 0, sizeof(a));
  a.kv = q.kv;
  a.num_slots = q.num_slots;
  a.page_table = q.page_table;
  a.kv_off = q.kv_off;
  a.D_c = q.d_latent;
  a.D_r = q.d_rope;
  a.d_err = q.d_err;
  return cuda_status(launch_latent_f16(a, plan, v16, nullptr, nullptr, nullptr, static_cast<cudaStream_t>(stream)));
}

kdv_status kdv_combine(const float* o_part, const float* lse_part, int32_t S, int64_t rows,
                       int32_t d, float* o, float* lse, void* stream) {
  if (S < 1 || rows < 0 || d < 1) return KDV_ERR_INVALID_ARG;
  if (rows > 0 && (o_part == nullptr || lse_part == nullptr || o == nullptr))
    return KDV_ERR_INVALID_ARG;
  return cuda_status(launch_combine_uniform(o_part, lse_part, S, rows, d, o, lse,
                                            static_cast<cudaStream_t>(stream)));
}

}  // extern "C"

// kdv_internal.cuh -- shared declarations of the CUDA library (not part of the ABI).
#pragma once

#include <cuda_runtime.h>
#include <stdint.h>

#include "kdv.h"

namespace kdv {

// Split / grid plan computed on the host from the HOST length copies and
// passed to kernels by value (kernel parameters, ~5 KB). Work item i of the
// grid maps to request b with item_base[b] <= i < item_base[b+1]; inside the
// request, local = i - item_base[b] = split * tiles[b] + row_tile, so items
// that run side by side share one split's keys in L2.
struct VerifyPlan {
  int32_t B;
  int32_t H;
  int32_t n_items;
  int32_t rows_per_tile;
  int32_t out_mode;        // OUT_DIRECT / OUT_PARTIALS / OUT_WORKSPACE
  int32_t part_f16;        // OUT_WORKSPACE partials o_k stored as fp16 (TC kernel)
  int32_t total_rows;      // sumT * H
  int32_t item_base[KDV_MAX_BATCH + 1];
  int32_t L[KDV_MAX_BATCH];
  int32_t T[KDV_MAX_BATCH];
  int32_t S[KDV_MAX_BATCH];
  int32_t chunk[KDV_MAX_BATCH];
  int32_t tiles[KDV_MAX_BATCH];
  int32_t tree_base[KDV_MAX_BATCH];   // tree_off[b] (from the host T copies)
  int32_t part_base[KDV_MAX_BATCH];   // first workspace partial row of request b
  int32_t v16_base[KDV_MAX_BATCH];    // first fp16 latent row of request b (TC kernel)
};

enum OutMode : int32_t { OUT_DIRECT = 0, OUT_PARTIALS = 1, OUT_WORKSPACE = 2 };

// Everything a verify kernel reads or writes besides the plan.
struct VerifyArgs {
  const void* q;
  int64_t q_row_stride;
  const void* kv;
  int64_t num_slots;
  const int32_t* page_table;
  const int32_t* kv_off;
  const int32_t* tree_off;
  const int32_t* prefix_len;
  const uint64_t* mask;
  int32_t D_c;
  int32_t D_r;
  float scale;
  float* o;          // OUT_DIRECT: [rows][D_c]; OUT_PARTIALS: [S][rows][D_c]; OUT_WORKSPACE: ws
                     // (fp16 elements there when the plan's part_f16 is set)
  float* lse;        // matching lse array (may be null in OUT_DIRECT)
  int32_t* d_err;
  uint64_t wait_limit_ns;   // pipeline-wait bound of the TC kernel (0 = its default, 1 s)
  // Staged paged pool (TC kernel): q_lat as fp16 [total_rows][512], written
  // by the latent pass. When set, the S pair reads Q.K^T's latent dims in
  // fp16 -- the queries from here, the keys from the fp16 latent rows -- and
  // only k_rope from kv, which then holds [keys][D_r] bf16 rows.
  void* q16;
};

// Where the (request b, split s, local row r) result goes, in rows of D_c.
__host__ __device__ inline int64_t out_row_index(const VerifyPlan& p, int b, int s, int r) {
  const int64_t row_global = (int64_t)p.tree_base[b] * p.H + r;
  if (p.out_mode == OUT_DIRECT) return row_global;
  if (p.out_mode == OUT_PARTIALS) return (int64_t)s * p.total_rows + row_global;
  return (int64_t)p.part_base[b] + (int64_t)s * ((int64_t)p.T[b] * p.H) + r;
}

__device__ inline void record_error(int32_t* d_err, int32_t code) {
  if (d_err != nullptr) atomicCAS(d_err, 0, code);
}

// Find the request of work item `item` (B <= 128: a short scan).
__device__ inline int plan_request(const VerifyPlan& p, int item) {
  int b = 0;
  while (b + 1 < p.B && p.item_base[b + 1] <= item) ++b;
  return b;
}

// Launchers (each returns cudaGetLastError() of its launch).
cudaError_t launch_mask_build(const int32_t* parent, const int32_t* tree_off, int32_t batch,
                              int32_t max_T, uint64_t* mask, int32_t* depth, int32_t* d_err,
                              cudaStream_t stream);
cudaError_t launch_verify_simt(const VerifyArgs& a, const VerifyPlan& p, int32_t dtype,
                               cudaStream_t stream);
// v16: the fp16 latent rows written by launch_latent_f16 (request b's key j
// at row v16_base[b] + j). after_latent: the launch right before this one on
// `stream` is the latent pass that writes v16, and it writes nothing else
// this kernel reads; the kernel is then launched as its programmatic
// dependent and only the V loads wait for it (griddepcontrol.wait).
cudaError_t launch_verify_tc2(const VerifyArgs& a, const VerifyPlan& p, const void* v16, int64_t v16_rows,
                              bool after_latent, cudaStream_t stream);
// Writes the fp16 latent rows (v16, nullable) and, for a staged paged pool,
// the k_rope rows [keys][D_r] with their offsets (staged / staged_off) and
// q_lat as fp16 [total_rows][512] (q16): those three are all given or all
// null (else cudaErrorInvalidValue).
cudaError_t launch_latent_f16(const VerifyArgs& a, const VerifyPlan& p, void* v16, void* staged, int32_t* staged_off,
                              void* q16, cudaStream_t stream);
// Work items (4-CTA clusters) of the TC kernel that fit on the device at
// once, i.e. one wave; 0 when the query fails (no device).
int tc2_max_active_clusters();
cudaError_t launch_combine_uniform(const float* o_part, const float* lse_part, int32_t S,
                                   int64_t rows, int32_t d, float* o, float* lse,
                                   cudaStream_t stream);
// Merges the workspace partials of a plan: fp32 o_k, or fp16 o_k when
// p.part_f16 (then d must be 512). The fp16 merge is launched as a
// programmatic dependent of the launch before it on `stream`, which must be
// the tensor-core attention kernel that wrote the partials.
cudaError_t launch_combine_plan(const void* ws_o, const float* ws_lse, const VerifyPlan& p,
                                int32_t d, float* o, float* lse, cudaStream_t stream);

// TC kernel tile geometry (shared with the planner).
constexpr int TC2_ROWS = 256;  // query rows per work item of the 2-SM-MMA kernel
constexpr int TC_KEYS = 128;   // keys per S / P tile of the tensor-core kernel
constexpr int SPLIT_ALIGN = 128;  // split boundaries are multiples of this many keys
constexpr int SIMT_ROWS = 8;   // query rows per SIMT CTA (one warp per row)

}  // namespace kdv

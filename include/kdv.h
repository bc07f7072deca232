/*
 * kdv.h -- C ABI of the B200 (sm_100a) tree-verify MLA attention library.
 *
 * What the library computes. In a speculative-decoding verify step, every
 * node of a draft tree is evaluated in parallel; each node attends over the
 * KV cache under a visibility mask that follows the tree, in a fused
 * multi-head latent attention that absorbs the latent projection (page "The
 * Architecture of Diagnosis", section "Phase 1: Custom CUDA Kernels", item 2).
 * A latent KV row is c_kv[kv_lora_rank=512] || k_rope[qk_rope_head_dim=64],
 * 576 elements per token per layer (page "From Diagnosis to Deployment",
 * section "The Second Thread"). The KV cache is paged with page_size=1
 * (page "The Architecture of Diagnosis", section "The Discrepancy That
 * Revealed the Truth", item 2). A long prefix and the tree tail can be
 * evaluated separately and merged (page "The Three Acts of Engineering",
 * reference [1]); the merge is a log-sum-exp combine.
 *
 * Definitions used by every call (T = tree size, L = prefix length, H heads):
 *   Anc*(t) = {t, parent[t], parent[parent[t]], ...}       (self included)
 *   visible keys of node t: prefix keys 0..L-1 and tree keys L+u, u in Anc*(t)
 *   s[t,h,j] = scale * (q_lat[t,h] . c_kv[j] + q_rope[t,h] . k_rope[j])
 *   o_lat[t,h] = sum_j softmax_j(s) c_kv[j],  lse[t,h] = ln sum_j exp(s[t,h,j])
 *
 * Conventions.
 *   - Every call returns a kdv_status; 0 (KDV_OK) is success. No exceptions.
 *   - Array arguments are DEVICE pointers owned by the caller unless marked
 *     HOST. The library allocates no device memory: scratch space is the
 *     caller's `workspace`.
 *   - Calls are asynchronous on `stream` (a cudaStream_t; NULL = legacy
 *     default stream). Host-side argument checks run before any launch and
 *     return KDV_ERR_INVALID_ARG / KDV_ERR_UNSUPPORTED without touching the GPU.
 *   - Bad data that only the device can see (a parent[] entry out of range,
 *     a page-table slot >= num_slots, a device length that disagrees with the
 *     host copy) is reported through the optional int32 `d_err` flag (0 = ok,
 *     otherwise the first KDV_DERR_* code seen). The offending access is
 *     skipped and the kernel finishes normally; nothing traps.
 *   - Rows are node-major: global row = (tree_off[b] + t) * H + h.
 */
#ifndef KDV_H_
#define KDV_H_

#include <stddef.h>
#include <stdint.h>

#if defined(__GNUC__)
#define KDV_API __attribute__((visibility("default")))
#else
#define KDV_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
  KDV_OK = 0,
  KDV_ERR_INVALID_ARG = -1, /* null/misaligned pointer, bad size or stride     */
  KDV_ERR_UNSUPPORTED = -2, /* valid but not implemented (dims, T > 64, batch) */
  KDV_ERR_WORKSPACE = -3,   /* workspace missing or smaller than required     */
  KDV_ERR_CUDA = -4         /* a CUDA launch or runtime call failed           */
} kdv_status;

/* Codes written to *d_err by kernels (first error wins). */
#define KDV_DERR_BAD_PARENT 1  /* parent[i] not in {-1} U [0, i)            */
#define KDV_DERR_BAD_SLOT 2    /* page_table entry outside [0, num_slots)   */
#define KDV_DERR_BAD_LENGTH 3  /* device prefix_len differs from host copy  */
#define KDV_DERR_BAD_TOKEN 4   /* tree-accept: token id out of range        */
#define KDV_DERR_TIMEOUT 5     /* a bounded in-kernel wait ran out (1 s or
                                  wait_limit_ns); the kernel stopped early,
                                  its outputs are not valid                 */
#define KDV_DERR_BAD_SCORE 6   /* tree build: a NaN candidate log-probability
                                  (read as -inf)                            */
#define KDV_DERR_RANGE 7       /* verify (TC kernel): a c_kv value that P.V
                                  reads has |x| >= 65536, inf or NaN; it is
                                  outside fp16, the P.V operand type, and
                                  the affected outputs are not valid        */

/* Element type of q and kv. */
#define KDV_BF16 0
#define KDV_F32 1

/* Kernel family for kdv_verify_attn. AUTO picks the tensor-core kernel when
 * its shape constraints hold (bf16, d_latent=512, d_rope=64) -- through a
 * staged copy (TC_STAGED) when there is a page table -- else SIMT. TC runs
 * 2-SM tcgen05 MMAs on 4-CTA clusters (256 query rows per work item): Q.K^T
 * in bf16, P.V with P and V in fp16 (11 significant bits, so the rounding of
 * the softmax numerators costs ~1.5e-4 of the output's RMS instead of ~1e-3
 * in bf16). V is read from fp16 rows that the call writes first (see
 * kdv_latent_f16), so the c_kv values it reads must lie in fp16's range,
 * |x| < 65536 (KDV_DERR_RANGE otherwise); pool rows outside the requests'
 * keys are never read for P.V. TC reads a paged pool's keys in place with
 * TMA four-row gathers. Value 3 (a 1-SM-MMA variant of earlier versions) is
 * retired and returns KDV_ERR_UNSUPPORTED. */
#define KDV_IMPL_AUTO 0
#define KDV_IMPL_SIMT 1
#define KDV_IMPL_TC 2
#define KDV_IMPL_TC_1SM 3
/* TC_STAGED: the 2-SM kernel over a paged pool that reads every key with
 * tiled TMA boxes instead of four-row gathers: the pass that writes the fp16
 * rows (in logical order) also copies each key's k_rope into a contiguous
 * region of the workspace and writes q_lat in fp16, and Q.K^T then runs over
 * the latent dims in fp16 and over the rope dims in bf16. bf16 -> fp16 is
 * exact for 2^-14 <= |x| < 65536; smaller magnitudes round to fp16
 * subnormals (so results can differ from KDV_IMPL_TC by a few fp32 ulps), and
 * a q_lat value beyond that range sets KDV_DERR_RANGE, as a c_kv value does.
 * Faster for paged pools at the price of workspace = (sum of L_b + T_b) x
 * D_r x 2 + (sum of T_b) x H x D_c x 2 bytes more (plus the batch's
 * offsets, each region rounded up to 256 B); AUTO's choice for paged pools.
 * Without a page table it is KDV_IMPL_TC. */
#define KDV_IMPL_TC_STAGED 4

#define KDV_MAX_TREE 64    /* nodes per tree (one 64-bit mask word)          */
#define KDV_MAX_BATCH 128  /* requests per kdv_verify_attn call              */

/* Human-readable name of a status code (static string, never NULL). */
KDV_API const char* kdv_status_string(kdv_status s);

/* Library ABI version (major*100 + minor): 110 adds kdv_tree_accept,
 * kdv_tree_build, kdv_absorb_q / kdv_unabsorb_o and KDV_IMPL_TC_STAGED to
 * the 100 set (mask build, verify, no-alloc verify, combine); 120 adds
 * kdv_latent_f16, the wait_limit_ns and v16 fields of kdv_verify_params,
 * KDV_DERR_RANGE, and retires KDV_IMPL_TC_1SM; 121 adds kdv_absorb_q_ex /
 * kdv_unabsorb_o_ex; 122 adds kdv_verify_attn_launches; 123: KDV_IMPL_TC_STAGED
 * stages k_rope and q_lat in fp16 instead of whole bf16 rows (another
 * workspace size). */
KDV_API int32_t kdv_version(void);

/*
 * kdv_tree_mask_build -- parent[] to ancestor bitmask (bit-exact).
 * The tree visibility mask of page "The Architecture of Diagnosis", section
 * "Phase 1: Custom CUDA Kernels", item 2: bit u of mask[i] is set iff node u
 * is node i itself or one of its ancestors.
 *   parent   [sumT] int32, per-request local indices; parent[i] in {-1} U [0,i)
 *            (-1 marks a root; several roots form a forest)
 *   tree_off [batch+1] int32 CSR offsets into parent/mask, or NULL for a single
 *            request of max_T nodes (batch must then be 1)
 *   batch    >= 1;  max_T in [1, 64], an upper bound on every request's T
 *   mask     [sumT] uint64 out
 *   depth    [sumT] int32 out, nullable: edges to the root (root = 0)
 *   d_err    nullable; KDV_DERR_BAD_PARENT for a malformed parent[] (that
 *            node's mask is written as 0)
 */
KDV_API kdv_status kdv_tree_mask_build(const int32_t* parent, const int32_t* tree_off, int32_t batch,
                               int32_t max_T, uint64_t* mask, int32_t* depth, int32_t* d_err,
                               void* stream);

/*
 * Parameters of kdv_verify_attn (absorbed-form tree-verify attention).
 *
 * Key addressing: logical key j of request b (0 <= j < L_b + T_b) is pool row
 *   page_table[kv_off[b] + j]   when page_table != NULL (page_size = 1), or
 *   kv_off[b] + j               when page_table == NULL (contiguous).
 * Key L_b + u holds tree node u's own latent row (written by the caller).
 *
 * Splits: with S splits, split s of request b covers the logical keys
 *   [s*c_b, min((s+1)*c_b, L_b+T_b)),  c_b = 128 * ceil((L_b+T_b) / (128*S)),
 * so a split may be empty (o = 0, lse = -inf). num_splits = 0 lets the
 * library choose S per request to fill the GPU and merge the partials in the
 * workspace; num_splits >= 1 forces S for every request.
 */
typedef struct kdv_verify_params {
  int32_t batch;         /* B in [1, KDV_MAX_BATCH]                              */
  int32_t num_heads;     /* H >= 1                                               */
  int32_t d_latent;      /* D_c: 512 for the TC kernel; 1..512 for SIMT          */
  int32_t d_rope;        /* D_r: 64 for the TC kernel; 0..64 for SIMT            */
  float scale;           /* softmax scale on q.k (e.g. 1/sqrt(d_nope + d_rope))  */
  int32_t dtype;         /* KDV_BF16 or KDV_F32 (q and kv)                       */
  int32_t impl;          /* KDV_IMPL_AUTO / _SIMT / _TC / _TC_STAGED             */
  const void* q;         /* [sumT*H][q_row_stride], row = q_lat || q_rope        */
  int64_t q_row_stride;  /* elements between q rows; 0 means D_c + D_r           */
  const void* kv;        /* pool [num_slots][D_c + D_r], row = c_kv || k_rope    */
  int64_t num_slots;     /* rows in the pool                                     */
  const int32_t* page_table;   /* [kv_off[B]] slots, or NULL (contiguous)        */
  const int32_t* kv_off;       /* [B+1] device                                   */
  const int32_t* tree_off;     /* [B+1] device                                   */
  const int32_t* prefix_len;   /* [B] device, nullable: checked against host     */
  const int32_t* h_prefix_len; /* [B] HOST copy of L_b (used to plan the grid)   */
  const int32_t* h_tree_T;     /* [B] HOST copy of T_b in [1, 64]                */
  const uint64_t* mask;        /* [sumT] from kdv_tree_mask_build                */
  int32_t num_splits;          /* 0 = auto, >= 1 forced                          */
  int32_t return_partials;     /* 1: write o_part/lse_part, no merge (S forced)  */
  float* o;              /* [sumT*H][D_c] out (unused when return_partials)      */
  float* lse;            /* [sumT*H] out, nullable                               */
  float* o_part;         /* [S][sumT*H][D_c] out when return_partials            */
  float* lse_part;       /* [S][sumT*H] out when return_partials                 */
  void* workspace;       /* caller-owned scratch, >= kdv_verify_attn_workspace   */
  size_t workspace_bytes;
  int32_t* d_err;        /* nullable device error flag                           */
  uint64_t wait_limit_ns;  /* TC kernel: how long one pipeline wait inside the
                              kernel may take before the kernel gives up with
                              KDV_DERR_TIMEOUT (0 = 1 s). Every wait is
                              bounded; on giving up, the kernel still retires
                              its copies and MMAs in flight (waiting up to 1 s
                              for them) and exits normally, its outputs not
                              valid. A small value is for testing that path. */
  const void* v16;       /* TC kernel, nullable: the fp16 latent rows of this
                            call, as kdv_latent_f16 writes them for these
                            parameters (a caller that mirrors its latent cache
                            in fp16 keeps them up to date and saves the
                            conversion); NULL = the call writes them into its
                            workspace before the attention kernel runs        */
} kdv_verify_params;

/* Bytes of workspace kdv_verify_attn needs for these parameters (the plan
 * depends only on the host fields). Writes *bytes; may be 0. For the TC
 * kernel it includes the fp16 latent rows (sum_b (L_b + T_b) x 1 KB) unless
 * p->v16 is given. */
KDV_API kdv_status kdv_verify_attn_workspace(const kdv_verify_params* p, size_t* bytes);

/* The plan kdv_verify_attn would use for these parameters (host fields only):
 * splits[b] = S for request b (length batch, nullable) and *grid_items = the
 * number of work items (2-CTA clusters for the TC kernel, CTAs for SIMT),
 * nullable. Lets a caller size o_part for return_partials with the automatic
 * split count. */
KDV_API kdv_status kdv_verify_attn_plan(const kdv_verify_params* p, int32_t* splits,
                                        int32_t* grid_items);

/* How many kernels kdv_verify_attn launches for these parameters (host
 * fields only; writes *launches): the attention kernel, plus the fp16
 * latent-row pass when the TC kernel writes its own rows (or stages a paged
 * pool), plus the merge kernel when split partials are merged in the
 * workspace. For building CUDA graphs and counting launches. */
KDV_API kdv_status kdv_verify_attn_launches(const kdv_verify_params* p, int32_t* launches);

/*
 * kdv_verify_attn -- tree-verify MLA attention in absorbed form.
 * Absorbed Q.K^T over D_c + D_r dims, online softmax, P.V over the D_c latent
 * dims (V is the c_kv part of the same pool row), optional per-split LSE and
 * the split merge. Output o_lat is fp32 [sumT*H][D_c]; lse is the natural-log
 * log-sum-exp of the scaled logits. Requirements for the TC kernel: scale
 * > 0 (KDV_ERR_UNSUPPORTED otherwise; AUTO then picks the SIMT kernel); q, kv,
 * o and o_part 16-byte aligned; q_row_stride*elem and (D_c+D_r)*elem
 * multiples of 16 bytes (KDV_ERR_INVALID_ARG otherwise).
 */
KDV_API kdv_status kdv_verify_attn(const kdv_verify_params* p, void* stream);

/*
 * kdv_latent_f16 -- the fp16 copy of the latent rows that the tensor-core
 * kernel's P.V reads (this library's design, not the pages': its P.V runs
 * in fp16, whose 11 significant bits keep the rounding of the softmax
 * numerators ~8x below bf16's, and an MMA needs both operands in one type).
 * Writes the c_kv part (D_c = 512 dims) of every key the call reads --
 * request b's logical keys j = 0 .. L_b+T_b-1, through the page table when
 * there is one -- as fp16 to row sum_{b'<b}(L_b'+T_b') + j of
 * v16 [sum_b (L_b+T_b)][512] (device, 16-byte aligned). bf16 -> fp16 is
 * exact for 2^-14 <= |x| < 65536; smaller values round to subnormals.
 * Device errors: KDV_DERR_RANGE (|x| >= 65536, inf or NaN in a row it
 * reads), KDV_DERR_BAD_SLOT / KDV_DERR_BAD_LENGTH (a row outside the pool;
 * written as zeros). kdv_verify_attn calls it itself unless p->v16 is set.
 * Requires the TC shape (bf16, d_latent 512, d_rope 64); p->impl is ignored.
 */
KDV_API kdv_status kdv_latent_f16(const kdv_verify_params* p, void* v16, void* stream);

/*
 * kdv_verify_attn_noalloc -- kdv_verify_attn for callers that cannot allocate.
 * The pages describe nothing like it; it is a convenience of this library.
 * Some callers cannot give the library scratch memory: a serving engine that
 * reserved all free device memory for its KV-cache pool at start-up, a
 * plug-in whose host framework owns every device allocation, or a loop where
 * an allocation on the call path costs too much. This entry point computes
 * exactly what kdv_verify_attn computes, but keeps the split partials in a
 * scratch array compiled into the library (KDV_NOALLOC_SCRATCH_BYTES per
 * GPU, held by every GPU that loads the library until the process exits)
 * and ignores p->workspace / p->workspace_bytes. It allocates no memory.
 *   - Returns KDV_ERR_WORKSPACE when the split plan needs more scratch than
 *     KDV_NOALLOC_SCRATCH_BYTES (kdv_verify_attn_workspace tells the size;
 *     fewer splits or fewer requests per call fit).
 *   - The first call on a device looks up the array's device address with
 *     the device current; make that first call before any stream capture.
 *     The address is kept for the life of the process: after a
 *     cudaDeviceReset of that device it is stale, so do not call this entry
 *     point on a device that has been reset.
 *   - All calls share the one array and it keeps the previous call's
 *     contents (every byte a call reads, the same call writes first). Calls
 *     whose work overlaps on the GPU race on it: issue them on one stream or
 *     order them.
 */
#define KDV_NOALLOC_SCRATCH_BYTES (16 * 1024 * 1024)
KDV_API kdv_status kdv_verify_attn_noalloc(const kdv_verify_params* p, void* stream);

/*
 * kdv_combine -- log-sum-exp merge of S split partials (the prefix / tree-tail
 * merge of page "The Three Acts of Engineering", reference [1]):
 *   LSE = ln sum_k exp(lse_k),  o = sum_k exp(lse_k - LSE) o_k.
 * A part with lse_k = -inf weighs nothing; a row whose parts are all empty
 * gets o = 0 and LSE = -inf.
 *   o_part [S][rows][d] fp32, lse_part [S][rows] fp32, o [rows][d], lse [rows]
 *   (lse nullable). S >= 1, rows >= 0, d >= 1.
 */
KDV_API kdv_status kdv_combine(const float* o_part, const float* lse_part, int32_t S, int64_t rows,
                       int32_t d, float* o, float* lse, void* stream);

/*
 * Greedy tree acceptance -- the step after verification: keep the longest
 * run of draft tokens that the target model agrees with (page "The
 * Architecture of Diagnosis", section "Phase 1: Custom CUDA Kernels", item 3:
 * a device-side kernel selects the longest accepted prefix with no host
 * involvement). The page gives no formula; this library reads it as:
 *   target[t] = argmax_v logits[t][v]: the lowest v among equal maxima, NaN
 *               never wins, a row of only NaN gives 0. (Or taken as given
 *               from target_in when logits is NULL.)
 *   accepted  : a root (parent -1) is accepted; node u with parent p is
 *               accepted iff p is accepted and token[u] == target[p].
 *   end       : the accepted node of greatest depth (lowest index on ties);
 *   path      : end's ancestor chain, root first; accept_len = depth(end)+1;
 *   bonus     : target[end], the target model's next token after the path.
 * Page commit (optional, page_size = 1): the tree region [L, L+T) of the
 * request's page table is reordered in place so that logical key L+i holds
 * the slot of path[i] (i < accept_len) and the other nodes' slots follow in
 * node order -- the accepted KV rows move to the front without copying a row
 * (the non-contiguous KV commit of page "The Architecture of Diagnosis",
 * section "The Discrepancy That Revealed the Truth", item 2), and the
 * rejected nodes' slots end up at [L+accept_len, L+T) for reuse.
 */
typedef struct kdv_accept_params {
  int32_t batch;          /* B in [1, KDV_MAX_BATCH]                              */
  int32_t max_T;          /* [1, 64]: bound on every T_b, row stride of path     */
  int32_t total_nodes;    /* sumT = tree_off[B] (HOST value; rows of logits)     */
  int32_t vocab;          /* V >= 1: logits columns; tokens lie in [0, V)        */
  int32_t dtype;          /* KDV_BF16 or KDV_F32: element type of logits         */
  const void* logits;     /* [sumT][logits_ld] target logits, or NULL            */
  int64_t logits_ld;      /* elements between logits rows (>= vocab)             */
  const int32_t* target_in;   /* [sumT] target tokens, read when logits is NULL  */
  const int32_t* token;       /* [sumT] draft token of each node (roots: unused) */
  const int32_t* parent;      /* [sumT] local parent, -1 for a root              */
  const int32_t* tree_off;    /* [B+1] device CSR offsets                        */
  int32_t* target_out;        /* [sumT] out, nullable: target[t]                 */
  int32_t* accept_len;        /* [B] out: accepted nodes, root included          */
  int32_t* accept_path;       /* [B][max_T] out: local node ids root first, -1 pad */
  int32_t* bonus;             /* [B] out, nullable: target at the path's end     */
  int32_t* page_table;        /* nullable: [kv_off[B]] slots, committed in place */
  const int32_t* kv_off;      /* [B+1] device, required with page_table          */
  const int32_t* prefix_len;  /* [B] device, required with page_table or prefix_len_out */
  int32_t* prefix_len_out;    /* [B] out, nullable: prefix_len + accept_len (may
                                 be the prefix_len array itself)                 */
  void* workspace;            /* caller scratch, >= kdv_tree_accept_workspace    */
  size_t workspace_bytes;
  int32_t* d_err;             /* nullable device error flag                      */
} kdv_accept_params;

/* Bytes of workspace kdv_tree_accept needs (0 when logits is NULL). */
KDV_API kdv_status kdv_tree_accept_workspace(const kdv_accept_params* p, size_t* bytes);

/*
 * kdv_tree_accept -- argmax of the target logits at every node, greedy path
 * selection, and the optional page-table commit, all on the device.
 * Requirements: logits 16-byte aligned and logits_ld*elem a multiple of 16
 * bytes for the vector path (other layouts take a scalar path). Device-side
 * errors: KDV_DERR_BAD_PARENT (that request gets accept_len 0, path -1,
 * bonus -1, no commit), KDV_DERR_BAD_TOKEN (a draft or given target token
 * outside [0, V); it is compared as is), KDV_DERR_BAD_LENGTH (T_b outside
 * [1, max_T], or the page-table range of a request shorter than L_b + T_b:
 * no commit for that request).
 */
KDV_API kdv_status kdv_tree_accept(const kdv_accept_params* p, void* stream);

/*
 * The two per-head projections around absorbed-form attention (the latent
 * projection that page "The Architecture of Diagnosis", section "Phase 1:
 * Custom CUDA Kernels", item 2 says the verify kernel absorbs):
 *   kdv_absorb_q:   q_lat[row] = W_UK[h] q_nope[row]     (W_UK [H][D_c][D_n])
 *   kdv_unabsorb_o: out[row]   = W_UV[h]^T o_lat[row]    (W_UV [H][D_c][D_v])
 * Rows are node-major, row = t*H + h (rows must be a multiple of H). Weights
 * and q_nope are KDV_BF16 or KDV_F32; o_lat is fp32 (kdv_verify_attn's
 * output); out_dtype selects the output element type (KDV_BF16 rounds to
 * nearest even). Strides are in elements: q_lat may be written straight into
 * the first D_c columns of kdv_verify_attn's q rows (q_lat_stride = D_c +
 * D_r). Accumulation is fp32. Limits: D_n <= 512, D_c <= 4096 (absorb);
 * D_c <= 512, D_v <= 4096 (unabsorb); otherwise KDV_ERR_UNSUPPORTED.
 * bf16 weights with a 16-byte aligned base and rows a multiple of 16 bytes
 * (D_n resp. D_v a multiple of 8) take the TMA-staged kernels; anything else
 * takes the general kernels, with the same results up to fp32 summation
 * order. The TMA-staged kernels wait at most 2 s for their weight tile; if it
 * never lands they write NaN to their outputs (these entry points take no
 * device error flag).
 */
KDV_API kdv_status kdv_absorb_q(int32_t rows, int32_t num_heads, int32_t d_latent, int32_t d_nope,
                                const void* q_nope, int64_t q_nope_stride, int32_t q_dtype, const void* w_uk,
                                int32_t w_dtype, void* q_lat, int64_t q_lat_stride, int32_t out_dtype,
                                void* stream);
KDV_API kdv_status kdv_unabsorb_o(int32_t rows, int32_t num_heads, int32_t d_latent, int32_t d_v,
                                  const float* o_lat, int64_t o_lat_stride, const void* w_uv, int32_t w_dtype,
                                  void* out, int64_t out_stride, int32_t out_dtype, void* stream);

/*
 * kdv_absorb_q_ex / kdv_unabsorb_o_ex -- the same, with flags (0 = the calls
 * above). KDV_PROJ_STATIC_WEIGHTS promises that the weights are not written
 * by the kernel launched immediately before on `stream` (weights of a loaded
 * model are constant over the step). The TMA-staged kernels are then launched
 * as programmatic dependents of that kernel: their CTAs start copying weight
 * tiles while it finishes, and wait for it (griddepcontrol.wait) before they
 * read q_nope / o_lat or write any output, so every other stream-order
 * guarantee holds. The general kernels ignore the flag. Unknown flag bits:
 * KDV_ERR_INVALID_ARG.
 */
#define KDV_PROJ_STATIC_WEIGHTS 1u
KDV_API kdv_status kdv_absorb_q_ex(int32_t rows, int32_t num_heads, int32_t d_latent, int32_t d_nope,
                                   const void* q_nope, int64_t q_nope_stride, int32_t q_dtype, const void* w_uk,
                                   int32_t w_dtype, void* q_lat, int64_t q_lat_stride, int32_t out_dtype,
                                   uint32_t flags, void* stream);
KDV_API kdv_status kdv_unabsorb_o_ex(int32_t rows, int32_t num_heads, int32_t d_latent, int32_t d_v,
                                     const float* o_lat, int64_t o_lat_stride, const void* w_uv, int32_t w_dtype,
                                     void* out, int64_t out_stride, int32_t out_dtype, uint32_t flags, void* stream);

/*
 * kdv_tree_build -- best-first draft-tree construction on the device (the
 * GPU-resident builder of page "The Architecture of Diagnosis", section
 * "Phase 1: Custom CUDA Kernels", item 1, which replaces a host heap). The
 * page gives no scoring; this library reads it as: a block drafter proposes,
 * for each of D future positions, K candidate tokens with log-probabilities;
 * a node is a path of candidate choices (one per position, root = the last
 * committed token at depth 0); its score is the fp32 sum of the chosen
 * log-probabilities, added root first; the tree of request b is what a
 * best-first expansion emits in T_b steps (take the frontier node first in
 * (score descending, path ascending digit by digit with a prefix first)
 * order, add its K children), in emission order -- parents precede
 * children, so the output feeds kdv_tree_mask_build directly. With
 * log-probabilities <= 0 this is the first T_b nodes of that order. A NaN log-probability is read as -inf and
 * reported (KDV_DERR_BAD_SCORE); a path score that comes out NaN (+inf and
 * -inf on one path) is read as -inf, silently. A budget above the number of paths is
 * reported (KDV_DERR_BAD_LENGTH); the missing nodes get parent -1, token -1.
 */
typedef struct kdv_tree_build_params {
  int32_t batch;              /* B in [1, KDV_MAX_BATCH]                           */
  int32_t max_T;              /* [1, 64]: bound on every budget T_b                 */
  int32_t depth;              /* D in [0, 16]: draft positions with candidates      */
  int32_t topk;               /* K in [1, 8]: candidates per position               */
  const int32_t* tree_off;    /* [B+1] device: T_b = tree_off[b+1] - tree_off[b]    */
  const int32_t* root_token;  /* [B] token of each root                             */
  const int32_t* cand_token;  /* [B][D][K] candidate tokens                          */
  const float* cand_logp;     /* [B][D][K] their log-probabilities                   */
  int32_t* parent;            /* [sumT] out: request-local parent index, -1 = root   */
  int32_t* token;             /* [sumT] out                                          */
  int32_t* depth_out;         /* [sumT] out, nullable                                */
  float* score;               /* [sumT] out, nullable                                */
  int32_t* d_err;             /* nullable device error flag                          */
} kdv_tree_build_params;
KDV_API kdv_status kdv_tree_build(const kdv_tree_build_params* p, void* stream);

#ifdef __cplusplus
}
#endif

#endif /* KDV_H_ */

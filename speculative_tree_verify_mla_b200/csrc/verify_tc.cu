// verify_tc.cu -- tensor-core tree-verify MLA attention for sm_100a
// (tcgen05 MMAs with TMEM accumulators, TMA-staged KV tiles, 2-CTA clusters).
//
// Operation (page "The Architecture of Diagnosis", section "Phase 1: Custom
// CUDA Kernels", item 2; latent dims from page "From Diagnosis to
// Deployment", section "The Second Thread"): for every query row (t, h) of a
// draft tree, s_j = scale * (q_lat . c_kv[j] + q_rope . k_rope[j]) over the
// 576 latent dims, softmax over the keys visible to node t (the whole prefix
// plus t's ancestors-or-self in the tree), o_lat = sum_j p_j c_kv[j] over the
// 512 latent dims, and the log-sum-exp of the split.
//
// Why a CTA pair. The H x T query rows share one latent KV, so the work is a
// real dense contraction: 128 rows x 64 keys x 576 dims for S = Q K^T and
// 128 x 512 x 64 for O += P V per key tile. The fp32 O tile of 128 rows x 512
// dims fills all 512 TMEM columns of an SM, leaving no room for S, and
// splitting the 512 dims across SMs would recompute Q K^T. So each work item
// (128 rows of one request, one key split) runs on a 2-CTA cluster:
//
//   CTA 0 ("S side"): Q (128 x 576 bf16) lives in TMEM (288 columns) and is
//     the A operand of tcgen05.mma; KV tiles (64 keys x 576) arrive by TMA
//     into a 3-stage ring; S = Q K^T accumulates in one of three 64-column
//     TMEM buffers. Four softmax warps (one query row per thread) read S,
//     apply the tree mask, keep the running max and sum, and write P (bf16,
//     128 x 64, UMMA 128B-swizzled layout) straight into CTA 1's shared
//     memory over the cluster's distributed shared memory.
//   CTA 1 ("O side"): O (128 x 512 fp32) lives in all of TMEM; V tiles (the
//     first 512 columns of the same KV rows) arrive by TMA into a 2-stage
//     ring; O += P V runs as 2 MMAs of N=256 per 16 keys.
//
// Softmax uses a lazy rescale: the S side keeps a per-row reference max and
// only moves it (and asks the O side to rescale its O row) when a tile's max
// exceeds it by more than 2^8, so O is rarely touched between MMAs. Every
// wait is bounded (~1 s, then KDV_DERR_TIMEOUT and an orderly exit).
#include <cuda.h>
#include <cuda_bf16.h>

#include "kdv_internal.cuh"
#include "sm100_ptx.cuh"

namespace kdv {
namespace {

using namespace ptx;

constexpr int DQ = 576, DC = 512;
constexpr int ROWS = TC_ROWS;                       // 128 query rows per item
constexpr int KEYS = TC_KEYS;                       // 64 keys per tile
constexpr int BLOCK_BYTES = KEYS * 128;             // 64 keys x 64 dims bf16, swizzled
constexpr int QK_BLOCKS = DQ / 64;                  // 9
constexpr int PV_BLOCKS = DC / 64;                  // 8
constexpr int S_STAGES = 3;
constexpr int O_STAGES = 2;
constexpr int S_STAGE_BYTES = QK_BLOCKS * BLOCK_BYTES;  // 73728
constexpr int O_STAGE_BYTES = PV_BLOCKS * BLOCK_BYTES;  // 65536
constexpr int P_BYTES = ROWS * 128;                     // 128 rows x 64 keys bf16
constexpr int S_BUFS = 3;
constexpr uint32_t TMEM_COLS = 512;
constexpr uint32_t TMEM_Q_COL = 0;                      // 288 columns
constexpr uint32_t TMEM_S_COL = 288;                    // 3 x 64 columns
constexpr float TAU = 8.0f;                             // lazy-rescale threshold (log2)
constexpr float LOG2E = 1.4426950408889634f;
constexpr float LN2 = 0.6931471805599453f;
constexpr uint64_t TIMEOUT_NS = 1000000000ull;

// Shared-memory layout (offsets from a 1024-byte aligned base; the same in
// both CTAs so that mapa() addresses line up).
constexpr int OFF_STAGES = 0;
constexpr int OFF_P = O_STAGES * O_STAGE_BYTES;              // O side only
constexpr int OFF_MISC = S_STAGES * S_STAGE_BYTES;
static_assert(OFF_P + 2 * P_BYTES <= OFF_MISC, "P buffers overlap misc");
constexpr int OFF_ALPHA = OFF_MISC;                          // float [2][128]
constexpr int OFF_FLAG = OFF_ALPHA + 2 * ROWS * 4;           // u32 [2] (+pad)
constexpr int OFF_STAT_L = OFF_FLAG + 16;                    // float [128]
constexpr int OFF_STAT_M = OFF_STAT_L + ROWS * 4;            // float [128]
constexpr int OFF_BAR = OFF_STAT_M + ROWS * 4;               // u64 [NUM_BARS]
constexpr int NUM_BARS = 26;
constexpr int OFF_TMEM = OFF_BAR + NUM_BARS * 8;             // u32
constexpr int OFF_ABORT = OFF_TMEM + 4;                      // u32
constexpr int OFF_ISSUED = OFF_ABORT + 4;                    // u32 (O side)
constexpr int SMEM_USED = OFF_ISSUED + 8;
constexpr int SMEM_BYTES = SMEM_USED + 1024;                 // + alignment slack
static_assert(SMEM_BYTES <= 232448, "exceeds 227 KB of shared memory");

// Barrier slots. Each CTA initialises only its own side's slots; the S side
// arrives remotely on the O side's P_FULL / STATS and the O side on the S
// side's P_EMPTY, at the same slot offsets.
// S side
constexpr int B_KV_FULL = 0, B_KV_EMPTY = 3, B_S_FULL = 6, B_S_EMPTY = 9, B_P_EMPTY = 12,
              B_Q_READY = 14, B_S_DRAIN = 15;
// O side
constexpr int B_V_FULL = 16, B_V_EMPTY = 18, B_P_FULL = 20, B_STATS = 22, B_PV_DONE = 24;

constexpr uint32_t IDESC_QK = idesc_bf16_f32(128, 64, false, false);
constexpr uint32_t IDESC_PV = idesc_bf16_f32(128, 256, false, true);

constexpr int THREADS = 256;
constexpr int WG_FIRST_WARP = 4;      // warps 4..7: softmax (S side) / PV + epilogue (O side)

__device__ __forceinline__ uint64_t globaltimer() {
  uint64_t t;
  asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
  return t;
}

struct Ctx {
  uint32_t base;                 // aligned shared base (shared::cta address)
  volatile uint32_t* abort_flag;
  int32_t* d_err;
  __device__ uint32_t bar(int i) const { return base + OFF_BAR + 8 * i; }
};

// Bounded wait on phase `parity`. Returns false on timeout or when another
// role of this CTA already gave up (unless `drain`, which ignores the abort
// flag and only stops at the time limit: used to retire in-flight copies).
__device__ __noinline__ bool wait_bar(const Ctx& c, uint32_t bar, uint32_t parity, bool drain = false) {
  if (mbar_try_wait(bar, parity)) return true;
  const uint64_t t0 = globaltimer();
  for (uint32_t it = 1;; ++it) {
    if (mbar_try_wait(bar, parity)) return true;
    if ((it & 63) == 0) {
      if (!drain && *c.abort_flag) return false;
      if (globaltimer() - t0 > TIMEOUT_NS) {
        *c.abort_flag = 1;
        record_error(c.d_err, KDV_DERR_TIMEOUT);
        return false;
      }
    }
  }
}

__global__ void __launch_bounds__(THREADS, 1) __cluster_dims__(2, 1, 1)
verify_tc_kernel(const __grid_constant__ CUtensorMap tmap_kv, const VerifyArgs a, const VerifyPlan p) {
  extern __shared__ uint8_t smem_raw[];
  const uint32_t raw = smem_u32(smem_raw);
  const uint32_t base = (raw + 1023u) & ~1023u;
  uint8_t* smem = smem_raw + (base - raw);
  const uint32_t rank = cluster_ctarank();
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

  Ctx c;
  c.base = base;
  c.abort_flag = reinterpret_cast<volatile uint32_t*>(smem + OFF_ABORT);
  c.d_err = a.d_err;

  // ---- work item ---------------------------------------------------------
  const int item = blockIdx.x >> 1;
  const int b = plan_request(p, item);
  const int local = item - p.item_base[b];
  const int split = local / p.tiles[b];
  const int rt = local - split * p.tiles[b];
  const int H = p.H, L = p.L[b], Tn = p.T[b];
  const int n_keys = L + Tn;
  const int rows_b = Tn * H;
  const int row0 = rt * ROWS;
  const int k_lo = min(split * p.chunk[b], n_keys);
  const int k_hi = min(k_lo + p.chunk[b], n_keys);
  const int n_tiles = (k_hi - k_lo + KEYS - 1) / KEYS;
  const int64_t kv_base = a.kv_off[b];

  // ---- setup -------------------------------------------------------------
  if (threadIdx.x == 0) {
    *c.abort_flag = 0;
    if (rank == 0) {
      for (int i = 0; i < S_STAGES; ++i) {
        mbar_init(c.bar(B_KV_FULL + i), 1);
        mbar_init(c.bar(B_KV_EMPTY + i), 1);
      }
      for (int i = 0; i < S_BUFS; ++i) {
        mbar_init(c.bar(B_S_FULL + i), 1);
        mbar_init(c.bar(B_S_EMPTY + i), ROWS);
      }
      for (int i = 0; i < 2; ++i) mbar_init(c.bar(B_P_EMPTY + i), 1);
      mbar_init(c.bar(B_Q_READY), ROWS);
      mbar_init(c.bar(B_S_DRAIN), 1);
      // device-side consistency of the host plan
      if (a.prefix_len != nullptr && a.prefix_len[b] != L) record_error(a.d_err, KDV_DERR_BAD_LENGTH);
      if (a.tree_off != nullptr && a.tree_off[b] != p.tree_base[b]) record_error(a.d_err, KDV_DERR_BAD_LENGTH);
      if ((int64_t)a.kv_off[b + 1] - kv_base < (int64_t)n_keys) record_error(a.d_err, KDV_DERR_BAD_LENGTH);
      tma_prefetch_desc(&tmap_kv);
    } else {
      for (int i = 0; i < O_STAGES; ++i) {
        mbar_init(c.bar(B_V_FULL + i), 1);
        mbar_init(c.bar(B_V_EMPTY + i), 1);
      }
      for (int i = 0; i < 2; ++i) {
        mbar_init(c.bar(B_P_FULL + i), ROWS);
        mbar_init(c.bar(B_PV_DONE + i), 1);
      }
      mbar_init(c.bar(B_STATS), ROWS);
      tma_prefetch_desc(&tmap_kv);
    }
    fence_mbar_init();
  }
  if (warp == 2) {
    tmem_alloc(base + OFF_TMEM, TMEM_COLS);
    tmem_relinquish();
  }
  __syncwarp();
  tc_fence_before();
  cluster_sync();
  tc_fence_after();
  const uint32_t tmem = *reinterpret_cast<volatile uint32_t*>(smem + OFF_TMEM);

  if (rank == 0) {
    // ======================================================= S side (CTA 0)
    if (warp == 0 && lane == 0) {
      // ---------------- KV producer: 64 keys x 576 dims per stage
      int issued = 0;
      for (int i = 0; i < n_tiles; ++i) {
        const int st = i % S_STAGES;
        if (!wait_bar(c, c.bar(B_KV_EMPTY + st), ((i / S_STAGES) & 1) ^ 1)) break;
        mbar_arrive_expect_tx(c.bar(B_KV_FULL + st), S_STAGE_BYTES);
        const int32_t y = (int32_t)(kv_base + k_lo + i * KEYS);
        const uint32_t dst = base + OFF_STAGES + st * S_STAGE_BYTES;
        for (int blk = 0; blk < QK_BLOCKS; ++blk)
          tma_load_2d(dst + blk * BLOCK_BYTES, &tmap_kv, c.bar(B_KV_FULL + st), blk * 64, y);
        issued = i + 1;
      }
      // retire copies still in flight (normally none: the MMA consumed them)
      for (int i = max(0, issued - S_STAGES); i < issued; ++i)
        wait_bar(c, c.bar(B_KV_FULL + i % S_STAGES), (i / S_STAGES) & 1, true);
    } else if (warp == 1 && lane == 0) {
      // ---------------- QK^T MMA issuer
      bool ok = n_tiles == 0 || wait_bar(c, c.bar(B_Q_READY), 0);
      tc_fence_after();
      for (int i = 0; ok && i < n_tiles; ++i) {
        const int st = i % S_STAGES, sb = i % S_BUFS;
        if (!wait_bar(c, c.bar(B_KV_FULL + st), (i / S_STAGES) & 1)) break;
        if (!wait_bar(c, c.bar(B_S_EMPTY + sb), ((i / S_BUFS) & 1) ^ 1)) break;
        tc_fence_after();
        const uint32_t d = tmem + TMEM_S_COL + sb * KEYS;
        const uint32_t stage = base + OFF_STAGES + st * S_STAGE_BYTES;
#pragma unroll 4
        for (int kk = 0; kk < DQ / 16; ++kk) {
          const uint64_t bdesc = sw128_desc(stage + (kk >> 2) * BLOCK_BYTES + (kk & 3) * 32, 16, 1024);
          mma_ts(d, tmem + TMEM_Q_COL + kk * 8, bdesc, IDESC_QK, kk > 0 ? 1u : 0u);
        }
        tc_commit(c.bar(B_S_FULL + sb));
        tc_commit(c.bar(B_KV_EMPTY + st));
      }
      // all issued MMAs complete before TMEM is freed
      tc_commit(c.bar(B_S_DRAIN));
      wait_bar(c, c.bar(B_S_DRAIN), 0, true);
    } else if (warp >= WG_FIRST_WARP) {
      // ---------------- softmax warpgroup: thread <-> query row
      const int sp = warp & 3;                       // TMEM sub-partition of this warp
      const int r = sp * 32 + lane;                  // row within the tile
      const int row = row0 + r;
      const bool valid = row < rows_b;
      const uint32_t lane_base = (uint32_t)(sp * 32) << 16;
      // Q row -> TMEM columns [0, 288) (bf16 pairs, element 2i in the low half)
      {
        const uint4* qrow = reinterpret_cast<const uint4*>(
            static_cast<const __nv_bfloat16*>(a.q) + ((int64_t)p.tree_base[b] * H + row) * a.q_row_stride);
#pragma unroll 1
        for (int cb = 0; cb < DQ / 64; ++cb) {
          uint32_t v[32];
#pragma unroll
          for (int k = 0; k < 8; ++k) {
            uint4 u = valid ? __ldg(qrow + cb * 8 + k) : make_uint4(0, 0, 0, 0);
            v[4 * k + 0] = u.x;
            v[4 * k + 1] = u.y;
            v[4 * k + 2] = u.z;
            v[4 * k + 3] = u.w;
          }
          tmem_st32(tmem + lane_base + TMEM_Q_COL + cb * 32, v);
        }
        tmem_wait_st();
        tc_fence_before();
        mbar_arrive(c.bar(B_Q_READY));
      }
      const uint64_t mask_t = valid ? a.mask[p.tree_base[b] + row / H] : 0ull;
      const float sl2 = a.scale * LOG2E;
      float m_run = -INFINITY, l_run = 0.f;
      const uint32_t peer_p = mapa(base + OFF_P, 1);
      const uint32_t peer_alpha = mapa(base + OFF_ALPHA, 1);
      const uint32_t peer_flag = mapa(base + OFF_FLAG, 1);
      const uint32_t peer_pfull = mapa(c.bar(B_P_FULL), 1);
      bool ok = true;
      for (int i = 0; i < n_tiles; ++i) {
        const int sb = i % S_BUFS;
        ok = ok && wait_bar(c, c.bar(B_S_FULL + sb), (i / S_BUFS) & 1);
        const bool wok = __all_sync(0xffffffffu, ok);     // tcgen05.ld is warp-aligned
        uint32_t sv[64];
        if (wok) {
          __syncwarp();
          tc_fence_after();
          tmem_ld32(tmem + lane_base + TMEM_S_COL + sb * KEYS, *reinterpret_cast<uint32_t(*)[32]>(sv));
          tmem_ld32(tmem + lane_base + TMEM_S_COL + sb * KEYS + 32, *reinterpret_cast<uint32_t(*)[32]>(sv + 32));
          tmem_wait_ld();
          tc_fence_before();
          mbar_arrive(c.bar(B_S_EMPTY + sb));
        } else {
#pragma unroll
          for (int k = 0; k < 64; ++k) sv[k] = 0u;
        }
        ok = ok && wok;
        // scores in log2 units with the tree / range mask
        const int key0 = k_lo + i * KEYS;
        float x[64];
        float m_tile = -INFINITY;
#pragma unroll
        for (int k = 0; k < 64; ++k) {
          const int j = key0 + k;
          bool vis = valid && j < k_hi;
          if (j >= L) vis = vis && ((mask_t >> ((j - L) & 63)) & 1ull);
          x[k] = vis ? __uint_as_float(sv[k]) * sl2 : -INFINITY;
          m_tile = fmaxf(m_tile, x[k]);
        }
        float alpha = 1.f;
        bool need = false;
        if (m_tile > m_run + TAU || (m_run == -INFINITY && m_tile != -INFINITY)) {
          if (m_run != -INFINITY) {
            alpha = ex2(m_run - m_tile);
            l_run *= alpha;
            need = true;
          }
          m_run = m_tile;
        }
        const float m_use = m_run == -INFINITY ? 0.f : m_run;
        uint32_t pk[32];
        float lsum = 0.f;
#pragma unroll
        for (int k = 0; k < 32; ++k) {
          const float p0 = ex2(x[2 * k] - m_use);
          const float p1 = ex2(x[2 * k + 1] - m_use);
          lsum += p0 + p1;
          pk[k] = pack_bf16x2(p0, p1);
        }
        l_run += lsum;
        // hand P (and the rescale factor) to the O side
        const int pb = i & 1;
        ok = ok && wait_bar(c, c.bar(B_P_EMPTY + pb), ((i >> 1) & 1) ^ 1);
        if (ok) {
          const uint32_t prow = peer_p + pb * P_BYTES + r * 128;
#pragma unroll
          for (int cc = 0; cc < 8; ++cc)
            st_cluster_v4(prow + ((cc ^ (r & 7)) << 4), pk[4 * cc], pk[4 * cc + 1], pk[4 * cc + 2], pk[4 * cc + 3]);
          st_cluster_f32(peer_alpha + (pb * ROWS + r) * 4, alpha);
        }
        const bool any = named_bar_or(1, 128, need);
        if (ok) {
          if (r == 0) st_cluster_u32(peer_flag + pb * 4, any ? 1u : 0u);
          mbar_arrive_remote(peer_pfull + pb * 8);
        }
      }
      // final row statistics for the O side's epilogue
      st_cluster_f32(mapa(base + OFF_STAT_L, 1) + r * 4, l_run);
      st_cluster_f32(mapa(base + OFF_STAT_M, 1) + r * 4, m_run);
      mbar_arrive_remote(mapa(c.bar(B_STATS), 1));
    }
  } else {
    // ======================================================= O side (CTA 1)
    if (warp == 0 && lane == 0) {
      // ---------------- V producer: 64 keys x 512 dims per stage
      int issued = 0;
      for (int i = 0; i < n_tiles; ++i) {
        const int st = i % O_STAGES;
        if (!wait_bar(c, c.bar(B_V_EMPTY + st), ((i / O_STAGES) & 1) ^ 1)) break;
        mbar_arrive_expect_tx(c.bar(B_V_FULL + st), O_STAGE_BYTES);
        const int32_t y = (int32_t)(kv_base + k_lo + i * KEYS);
        const uint32_t dst = base + OFF_STAGES + st * O_STAGE_BYTES;
        for (int blk = 0; blk < PV_BLOCKS; ++blk)
          tma_load_2d(dst + blk * BLOCK_BYTES, &tmap_kv, c.bar(B_V_FULL + st), blk * 64, y);
        issued = i + 1;
      }
      for (int i = max(0, issued - O_STAGES); i < issued; ++i)
        wait_bar(c, c.bar(B_V_FULL + i % O_STAGES), (i / O_STAGES) & 1, true);
    } else if (warp >= WG_FIRST_WARP) {
      const int sp = warp & 3;
      const int r = sp * 32 + lane;
      const int row = row0 + r;
      const bool valid = row < rows_b;
      const uint32_t lane_base = (uint32_t)(sp * 32) << 16;
      const bool issuer = (warp == WG_FIRST_WARP && lane == 0);
      const uint32_t peer_pempty = mapa(c.bar(B_P_EMPTY), 0);
      const volatile uint32_t* flag = reinterpret_cast<const volatile uint32_t*>(smem + OFF_FLAG);
      const volatile float* alpha_s = reinterpret_cast<const volatile float*>(smem + OFF_ALPHA);
      volatile uint32_t* issued_s = reinterpret_cast<volatile uint32_t*>(smem + OFF_ISSUED);
      bool ok = true;
      int issued = 0;
      for (int i = 0; i < n_tiles; ++i) {
        const int pb = i & 1;
        ok = ok && wait_bar(c, c.bar(B_P_FULL + pb), (i >> 1) & 1);
        const bool rescale = ok && flag[pb] != 0 && i > 0;
        if (rescale) ok = wait_bar(c, c.bar(B_PV_DONE + ((i - 1) & 1)), ((i - 1) >> 1) & 1);
        // rescale O rows before this tile's MMAs (rare: the S side moved a row max)
        if (__all_sync(0xffffffffu, ok) && __any_sync(0xffffffffu, rescale)) {
          __syncwarp();
          tc_fence_after();
          const float al = alpha_s[pb * ROWS + r];
#pragma unroll 1
          for (int cb = 0; cb < DC / 32; ++cb) {
            uint32_t v[32];
            tmem_ld32(tmem + lane_base + cb * 32, v);
            tmem_wait_ld();
#pragma unroll
            for (int k = 0; k < 32; ++k) v[k] = __float_as_uint(__uint_as_float(v[k]) * al);
            tmem_st32(tmem + lane_base + cb * 32, v);
          }
          tmem_wait_st();
          tc_fence_before();
        }
        // every row has read flag/alpha (and rescaled) before P or O move on
        __syncwarp();
        const bool fail = named_bar_or(2, 128, !ok || *c.abort_flag != 0);
        ok = ok && !fail;
        if (issuer && ok) {
          bool released = false;
          if (rescale) {
            mbar_arrive_remote(peer_pempty + ((i - 1) & 1) * 8);
            released = true;
          }
          const int st = i % O_STAGES;
          if (wait_bar(c, c.bar(B_V_FULL + st), (i / O_STAGES) & 1)) {
            tc_fence_after();
            const uint32_t pbuf = base + OFF_P + pb * P_BYTES;
            const uint32_t vst = base + OFF_STAGES + st * O_STAGE_BYTES;
#pragma unroll
            for (int kk = 0; kk < KEYS / 16; ++kk) {
              const uint64_t adesc = sw128_desc(pbuf + kk * 32, 16, 1024);
#pragma unroll
              for (int nh = 0; nh < 2; ++nh) {
                // V block: K (keys) rows of 128 B, 8-key groups 1024 B apart (SBO),
                // 64-dim column blocks BLOCK_BYTES apart (LBO), N = 256 dims
                const uint64_t bdesc = sw128_desc(vst + nh * 4 * BLOCK_BYTES + kk * 2048, BLOCK_BYTES, 1024);
                mma_ss(tmem + nh * 256, adesc, bdesc, IDESC_PV, (i > 0 || kk > 0) ? 1u : 0u);
              }
            }
            tc_commit(c.bar(B_PV_DONE + pb));
            tc_commit(c.bar(B_V_EMPTY + st));
            issued = i + 1;
            // release the previous P buffer once its MMAs are done
            if (i > 0 && !released) {
              if (wait_bar(c, c.bar(B_PV_DONE + ((i - 1) & 1)), ((i - 1) >> 1) & 1))
                mbar_arrive_remote(peer_pempty + ((i - 1) & 1) * 8);
            }
          }
        }
      }
      // ---------------- epilogue: o = O / l, lse = ln2 * (m + log2 l)
      if (issuer) *issued_s = (uint32_t)issued;
      __syncwarp();
      named_bar_sync(2, 128);
      const int n_issued = (int)*issued_s;
      bool have_o = n_issued > 0;
      if (have_o) {
        const int i = n_issued - 1;
        have_o = wait_bar(c, c.bar(B_PV_DONE + (i & 1)), (i >> 1) & 1, true);
      }
      have_o = __all_sync(0xffffffffu, have_o);
      __syncwarp();
      ok = ok && n_issued == n_tiles;
      tc_fence_after();
      ok = wait_bar(c, c.bar(B_STATS), 0) && ok;
      const float l = *reinterpret_cast<volatile float*>(smem + OFF_STAT_L + r * 4);
      const float m = *reinterpret_cast<volatile float*>(smem + OFF_STAT_M + r * 4);
      const float inv = (l > 0.f && ok) ? 1.f / l : 0.f;
      const float lse = (l > 0.f && ok) ? (m + __log2f(l)) * LN2 : -INFINITY;
      const int64_t orow = out_row_index(p, b, split, row);
      float* orow_ptr = a.o + orow * DC;
#pragma unroll 1
      for (int cb = 0; cb < DC / 32; ++cb) {
        uint32_t v[32];
        if (have_o) {
          tmem_ld32(tmem + lane_base + cb * 32, v);
          tmem_wait_ld();
        } else {
#pragma unroll
          for (int k = 0; k < 32; ++k) v[k] = 0u;
        }
        if (valid) {
#pragma unroll
          for (int k = 0; k < 8; ++k) {
            float4 f;
            f.x = __uint_as_float(v[4 * k + 0]) * inv;
            f.y = __uint_as_float(v[4 * k + 1]) * inv;
            f.z = __uint_as_float(v[4 * k + 2]) * inv;
            f.w = __uint_as_float(v[4 * k + 3]) * inv;
            *reinterpret_cast<float4*>(orow_ptr + cb * 32 + 4 * k) = f;
          }
        }
      }
      if (valid && a.lse != nullptr) a.lse[orow] = lse;
    }
  }

  // ---- teardown: peers done with our shared memory; TMEM idle -------------
  __syncwarp();
  tc_fence_before();
  cluster_sync();
  if (warp == 2) {
    tc_fence_after();
    tmem_dealloc(tmem, TMEM_COLS);
  }
}

typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                                  const cuuint64_t*, const cuuint32_t*, const cuuint32_t*,
                                  CUtensorMapInterleave, CUtensorMapSwizzle, CUtensorMapL2promotion,
                                  CUtensorMapFloatOOBfill);

EncodeTiledFn encode_fn() {
  static EncodeTiledFn fn = nullptr;
  if (fn == nullptr) {
    void* ptr = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &ptr, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<EncodeTiledFn>(ptr);
  }
  return fn;
}

}  // namespace

cudaError_t launch_verify_tc(const VerifyArgs& a, const VerifyPlan& p, cudaStream_t stream) {
  EncodeTiledFn enc = encode_fn();
  if (enc == nullptr) return cudaErrorNotSupported;
  if (a.num_slots < 1 || a.num_slots > (int64_t)0x7fffffff) return cudaErrorInvalidValue;
  CUtensorMap tmap;
  const cuuint64_t dims[2] = {(cuuint64_t)DQ, (cuuint64_t)a.num_slots};
  const cuuint64_t strides[1] = {(cuuint64_t)DQ * 2};
  const cuuint32_t box[2] = {64, (cuuint32_t)KEYS};
  const cuuint32_t estr[2] = {1, 1};
  CUresult r = enc(&tmap, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(a.kv), dims, strides, box,
                   estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                   CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  if (r != CUDA_SUCCESS) return cudaErrorInvalidValue;
  static bool attr_set[64] = {};
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  if (dev < 0 || dev >= 64 || !attr_set[dev]) {
    e = cudaFuncSetAttribute(verify_tc_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, SMEM_BYTES);
    if (e != cudaSuccess) return e;
    if (dev >= 0 && dev < 64) attr_set[dev] = true;
  }
  verify_tc_kernel<<<2 * p.n_items, THREADS, SMEM_BYTES, stream>>>(tmap, a, p);
  return cudaGetLastError();
}

}  // namespace kdv

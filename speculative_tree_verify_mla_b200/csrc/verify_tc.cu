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
// real dense contraction: per 128-key tile, S = Q K^T is 128 rows x 128 keys
// x 576 dims and O += P V is 128 x 512 x 128. The fp32 O tile of 128 rows x
// 512 dims fills all 512 TMEM columns of an SM, leaving no room for S, and
// splitting the 512 dims across SMs would recompute Q K^T. So each work item
// (128 rows of one request, one key split) runs on a 2-CTA cluster:
//
//   CTA 0 ("S side"): q_lat (128 x 512 bf16) lives in TMEM (256 columns) and
//     q_rope (128 x 64) in shared memory; KV arrives by TMA as 16 KB blocks
//     (128 keys x 64 dims, 128B-swizzled), three blocks per barrier, through a
//     4-stage ring (one wait per 48 KB, not per block); S = Q K^T
//     (M=128, N=128, K=576) accumulates in one of two 128-column TMEM
//     buffers. Four softmax warps (one query row per thread) read S, apply the
//     tree mask, keep the running max and sum, and push P (bf16, 128 x 128, in
//     the UMMA 128B-swizzled layout) into CTA 1's shared memory with st.async,
//     whose bytes complete a barrier there.
//   CTA 1 ("O side"): O (128 x 512 fp32) lives in all of TMEM; V (the first
//     512 columns of the same KV rows) arrives by TMA as 32-key stages through
//     a 4-stage ring; O += P V runs as 2 MMAs of N=256 per 16 keys.
//
// N=128 for Q K^T because a tcgen05.mma of N=64 issues at half the tensor
// rate of N>=128 on this part (measured); 128-key tiles keep each MMA large.
//
// Softmax uses a lazy rescale: the S side keeps a per-row reference max and
// only moves it (sending the factor with P, so the O side rescales that row
// of O between MMAs) when a tile's max exceeds it by more than 2^8. Every
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
constexpr int KEYS = TC_KEYS;                       // 128 keys per S / P tile
constexpr int VKEYS = 32;                           // keys per V stage (O side)
constexpr int KBLOCK_BYTES = KEYS * 128;            // 128 keys x 64 dims bf16, swizzled
constexpr int VBLOCK_BYTES = VKEYS * 128;           // 32 keys x 64 dims
constexpr int QBLOCK_BYTES = ROWS * 128;            // 128 rows x 64 dims
constexpr int QK_BLOCKS = DQ / 64;                  // 9 (8 latent + 1 rope)
constexpr int QLAT_BLOCKS = 8;
constexpr int PV_BLOCKS = DC / 64;                  // 8
constexpr int STAGE_BLOCKS = 3;                     // 16 KB blocks per S-side ring stage
constexpr int KV_STAGES = 4;                        // S-side ring: 4 stages x 48 KB
constexpr int KV_SLOTS = KV_STAGES * STAGE_BLOCKS;  // 16 KB block slots in the ring
constexpr int Q_STAGES = 3;                         // stages holding q_lat at start-up
constexpr int STAGES_PER_TILE = QK_BLOCKS / STAGE_BLOCKS;
static_assert(QK_BLOCKS % STAGE_BLOCKS == 0 && QLAT_BLOCKS <= Q_STAGES * STAGE_BLOCKS, "stage geometry");
constexpr int V_STAGES = 4;
constexpr int NP = 2;                               // P slots in flight
constexpr int V_STAGE_BYTES = PV_BLOCKS * VBLOCK_BYTES;  // 32768
constexpr int P_BYTES = ROWS * KEYS * 2;                 // 128 rows x 128 keys bf16
constexpr int P_KBLOCK_BYTES = ROWS * 128;               // 64 keys of P
constexpr int P_MSG_BYTES = P_BYTES + ROWS * 4;          // P + per-row rescale factor
constexpr int P_SLOT_BYTES = 33792;                      // P_MSG_BYTES rounded to 1 KB
constexpr int STATS_BYTES = 2 * ROWS * 4;                // final l and m per row
constexpr int S_BUFS = 2;
constexpr uint32_t TMEM_COLS = 512;
constexpr uint32_t TMEM_QLAT_COL = 0;                   // 256 columns
constexpr uint32_t TMEM_S_COL = 256;                    // 2 x 128 columns
constexpr float TAU = 8.0f;                             // lazy-rescale threshold (log2)
constexpr float LOG2E = 1.4426950408889634f;
constexpr float LN2 = 0.6931471805599453f;
constexpr uint64_t TIMEOUT_NS = 1000000000ull;

// Shared-memory layout, offsets from a 1024-byte aligned base. Both CTAs use
// the same offsets so that mapa() addresses of one side line up with the
// other side's buffers.
//   S side: [0, 196608) KV ring (4 stages x 3 blocks of 16 KB; q_lat occupies
//           the first 8 blocks at start-up),
//           [196608, 212992) q_rope.
//   O side: [0, 131072) V ring (4 x 32 KB); P slots; final stats.
constexpr int OFF_RING = 0;
constexpr int OFF_QROPE = KV_SLOTS * KBLOCK_BYTES;           // S side
constexpr int OFF_P = V_STAGES * V_STAGE_BYTES;              // O side
constexpr int OFF_STATS = OFF_P + NP * P_SLOT_BYTES;         // O side: float l[128], m[128]
constexpr int OFF_MISC = OFF_QROPE + QBLOCK_BYTES;
static_assert(OFF_STATS + STATS_BYTES <= OFF_MISC, "O-side buffers overlap misc");
constexpr int OFF_BAR = OFF_MISC;                            // u64 [NUM_BARS]
constexpr int NUM_BARS = 48;
constexpr int OFF_TMEM = OFF_BAR + NUM_BARS * 8;             // u32
constexpr int OFF_ABORT = OFF_TMEM + 4;                      // u32
constexpr int SMEM_USED = OFF_ABORT + 12;
constexpr int SMEM_BYTES = SMEM_USED + 1024;                 // + alignment slack
static_assert(SMEM_BYTES <= 232448, "exceeds 227 KB of shared memory");

// Barrier slots. Each CTA initialises only its own side's slots; remote
// arrivals / completions land at the same slot offsets in the other CTA.
// S side
constexpr int B_KV_FULL = 0, B_KV_EMPTY = 12, B_S_FULL = 24, B_S_EMPTY = 26, B_P_EMPTY = 28,  // KV: 4 used
              B_QROPE_FULL = 30, B_Q_READY = 31, B_S_DRAIN = 32;
// O side
constexpr int B_V_FULL = 33, B_V_EMPTY = 37, B_P_FULL = 41, B_READY = 43, B_PV_DONE = 45,
              B_STATS = 47;
constexpr int B_O_DRAIN = 30;          // O side reuses an S-only slot number
static_assert(B_STATS < NUM_BARS, "barrier slots");

constexpr uint32_t IDESC_QK = idesc_bf16_f32(128, 128, false, false);
constexpr uint32_t IDESC_PV = idesc_bf16_f32(128, 256, false, true);

constexpr int THREADS = 256;
constexpr int WG_FIRST_WARP = 4;      // warps 4..7: softmax (S side) / rescale + epilogue (O side)

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
// flag and only stops at the time limit: used to retire in-flight work).
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

// Warp-wide bounded wait: lane 0 polls the barrier and the warp then syncs,
// so one thread per warp (not 32) spins on the barrier while the TMA engine
// and the tensor core share this SM's shared memory. __syncwarp orders lane
// 0's acquire before the other lanes' reads. Call with the full warp.
__device__ __forceinline__ bool wait_warp(const Ctx& c, uint32_t bar, uint32_t parity, bool drain = false) {
  bool ok = true;
  if ((threadIdx.x & 31) == 0) ok = wait_bar(c, bar, parity, drain);
  ok = __shfl_sync(0xffffffffu, ok ? 1 : 0, 0) != 0;
  __syncwarp();
  return ok;
}

__global__ void __launch_bounds__(THREADS, 1) __cluster_dims__(2, 1, 1)
verify_tc_kernel(const __grid_constant__ CUtensorMap tmap_kv, const __grid_constant__ CUtensorMap tmap_v,
                 const __grid_constant__ CUtensorMap tmap_q, const VerifyArgs a, const VerifyPlan p) {
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
      for (int i = 0; i < KV_STAGES; ++i) {
        mbar_init(c.bar(B_KV_FULL + i), 1);
        mbar_init(c.bar(B_KV_EMPTY + i), 1);
      }
      for (int i = 0; i < S_BUFS; ++i) {
        mbar_init(c.bar(B_S_FULL + i), 1);
        mbar_init(c.bar(B_S_EMPTY + i), ROWS);
      }
      for (int i = 0; i < NP; ++i) mbar_init(c.bar(B_P_EMPTY + i), 1);
      mbar_init(c.bar(B_QROPE_FULL), 1);
      mbar_init(c.bar(B_Q_READY), ROWS);
      mbar_init(c.bar(B_S_DRAIN), 1);
      // device-side consistency of the host plan
      if (a.prefix_len != nullptr && a.prefix_len[b] != L) record_error(a.d_err, KDV_DERR_BAD_LENGTH);
      if (a.tree_off != nullptr && a.tree_off[b] != p.tree_base[b]) record_error(a.d_err, KDV_DERR_BAD_LENGTH);
      if ((int64_t)a.kv_off[b + 1] - kv_base < (int64_t)n_keys) record_error(a.d_err, KDV_DERR_BAD_LENGTH);
      tma_prefetch_desc(&tmap_kv);
      tma_prefetch_desc(&tmap_q);
    } else {
      for (int i = 0; i < V_STAGES; ++i) {
        mbar_init(c.bar(B_V_FULL + i), 1);
        mbar_init(c.bar(B_V_EMPTY + i), 1);
      }
      for (int i = 0; i < NP; ++i) {
        mbar_init(c.bar(B_P_FULL + i), 1);
        mbar_init(c.bar(B_READY + i), ROWS);
        mbar_init(c.bar(B_PV_DONE + i), 1);
      }
      mbar_init(c.bar(B_STATS), 1);
      mbar_init(c.bar(B_O_DRAIN), 1);
      // arm the first use of every P slot and the stats message: the S side's
      // st.async bytes complete these phases
      for (int i = 0; i < NP; ++i) mbar_arrive_expect_tx(c.bar(B_P_FULL + i), P_MSG_BYTES);
      mbar_arrive_expect_tx(c.bar(B_STATS), STATS_BYTES);
      tma_prefetch_desc(&tmap_v);
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
      // ---------------- producer. Stage use number pos goes to ring stage
      // pos % 4: q_lat fills uses 0-2 (stages 0-2), KV stage g (three dim-
      // blocks of tile g/3) is use g + 3.
      const int n_stg = n_tiles * STAGES_PER_TILE;
      int issued = 0;
      if (n_tiles > 0) {
        const int32_t qy = (int32_t)((int64_t)p.tree_base[b] * H + row0);
        for (int st = 0; st < Q_STAGES; ++st) {
          const int nb = min(STAGE_BLOCKS, QLAT_BLOCKS - st * STAGE_BLOCKS);
          mbar_arrive_expect_tx(c.bar(B_KV_FULL + st), nb * QBLOCK_BYTES);
          for (int e = 0; e < nb; ++e) {
            const int blk = st * STAGE_BLOCKS + e;
            tma_load_2d(base + OFF_RING + blk * KBLOCK_BYTES, &tmap_q, c.bar(B_KV_FULL + st), blk * 64, qy);
          }
        }
        mbar_arrive_expect_tx(c.bar(B_QROPE_FULL), QBLOCK_BYTES);
        tma_load_2d(base + OFF_QROPE, &tmap_q, c.bar(B_QROPE_FULL), QLAT_BLOCKS * 64, qy);
      }
      for (int g = 0; g < n_stg; ++g) {
        const int pos = g + Q_STAGES, st = pos % KV_STAGES;
        if (!wait_bar(c, c.bar(B_KV_EMPTY + st), ((pos / KV_STAGES) & 1) ^ 1)) break;
        mbar_arrive_expect_tx(c.bar(B_KV_FULL + st), STAGE_BLOCKS * KBLOCK_BYTES);
        const int tile = g / STAGES_PER_TILE, blk0 = (g % STAGES_PER_TILE) * STAGE_BLOCKS;
        const int32_t y = (int32_t)(kv_base + k_lo + tile * KEYS);
        for (int e = 0; e < STAGE_BLOCKS; ++e)
          tma_load_2d(base + OFF_RING + (st * STAGE_BLOCKS + e) * KBLOCK_BYTES, &tmap_kv, c.bar(B_KV_FULL + st),
                      (blk0 + e) * 64, y);
        issued = g + 1;
      }
      // retire copies still in flight (normally none: the MMA consumed them)
      if (n_tiles > 0) wait_bar(c, c.bar(B_QROPE_FULL), 0, true);
      for (int g = max(0, issued - KV_STAGES); g < issued; ++g) {
        const int pos = g + Q_STAGES;
        wait_bar(c, c.bar(B_KV_FULL + pos % KV_STAGES), (pos / KV_STAGES) & 1, true);
      }
    } else if (warp == 1 && lane == 0) {
      // ---------------- QK^T MMA issuer: S[128 x 128] = Q[128 x 576] . K^T
      bool ok = n_tiles == 0 || (wait_bar(c, c.bar(B_Q_READY), 0) && wait_bar(c, c.bar(B_QROPE_FULL), 0));
      tc_fence_after();
      // the q_lat staging stages (0-2) are free once Q is in TMEM
      if (ok && n_tiles > 0)
        for (int st = 0; st < Q_STAGES; ++st) mbar_arrive(c.bar(B_KV_EMPTY + st));
      for (int i = 0; ok && i < n_tiles; ++i) {
        const int sb = i % S_BUFS;
        if (!wait_bar(c, c.bar(B_S_EMPTY + sb), ((i / S_BUFS) & 1) ^ 1)) break;
        tc_fence_after();
        const uint32_t d = tmem + TMEM_S_COL + sb * KEYS;
        for (int gs = 0; ok && gs < STAGES_PER_TILE; ++gs) {
          const int pos = i * STAGES_PER_TILE + gs + Q_STAGES, st = pos % KV_STAGES;
          if (!wait_bar(c, c.bar(B_KV_FULL + st), (pos / KV_STAGES) & 1)) { ok = false; break; }
          tc_fence_after();
#pragma unroll
          for (int e = 0; e < STAGE_BLOCKS; ++e) {
            const int blk = gs * STAGE_BLOCKS + e;
            const uint32_t kb = base + OFF_RING + (st * STAGE_BLOCKS + e) * KBLOCK_BYTES;
#pragma unroll
            for (int kk = 0; kk < 4; ++kk) {
              const uint64_t bdesc = sw128_desc(kb + kk * 32, 16, 1024);
              const uint32_t acc = (blk > 0 || kk > 0) ? 1u : 0u;
              if (blk < QLAT_BLOCKS)
                mma_ts(d, tmem + TMEM_QLAT_COL + (blk * 4 + kk) * 8, bdesc, IDESC_QK, acc);
              else
                mma_ss(d, sw128_desc(base + OFF_QROPE + kk * 32, 16, 1024), bdesc, IDESC_QK, acc);
            }
          }
          tc_commit(c.bar(B_KV_EMPTY + st));
        }
        if (!ok) break;
        tc_commit(c.bar(B_S_FULL + sb));
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
      bool ok = true;
      if (n_tiles > 0) {
        // q_lat row (TMA-staged, 128B-swizzled, first 8 ring blocks) -> TMEM columns [0, 256)
        for (int st = 0; st < Q_STAGES; ++st) ok = wait_warp(c, c.bar(B_KV_FULL + st), 0) && ok;
        if (__all_sync(0xffffffffu, ok)) {
#pragma unroll 1
          for (int blk = 0; blk < QLAT_BLOCKS; ++blk) {
            uint32_t v[32];
            const uint8_t* rowp = smem + OFF_RING + blk * KBLOCK_BYTES + r * 128;
#pragma unroll
            for (int ch = 0; ch < 8; ++ch) {
              const uint4 u4 = *reinterpret_cast<const uint4*>(rowp + ((ch ^ (r & 7)) << 4));
              v[4 * ch + 0] = u4.x;
              v[4 * ch + 1] = u4.y;
              v[4 * ch + 2] = u4.z;
              v[4 * ch + 3] = u4.w;
            }
            __syncwarp();
            tmem_st32(tmem + lane_base + TMEM_QLAT_COL + blk * 32, v);
          }
          tmem_wait_st();
        }
        tc_fence_before();
        mbar_arrive(c.bar(B_Q_READY));
      }
      const uint64_t mask_t = valid ? a.mask[p.tree_base[b] + row / H] : 0ull;
      const float sl2 = a.scale * LOG2E;
      float m_run = -INFINITY, l_run = 0.f;
      const uint32_t peer_p = mapa(base + OFF_P, 1);
      const uint32_t peer_pfull = mapa(c.bar(B_P_FULL), 1);
      for (int i = 0; i < n_tiles; ++i) {
        const int sb = i % S_BUFS;
        ok = wait_warp(c, c.bar(B_S_FULL + sb), (i / S_BUFS) & 1) && ok;
        const bool wok = __all_sync(0xffffffffu, ok);     // tcgen05.ld is warp-aligned
        uint32_t sv[KEYS];
        if (wok) {
          __syncwarp();
          tc_fence_after();
          const uint32_t sa = tmem + lane_base + TMEM_S_COL + sb * KEYS;
          tmem_ld32(sa, *reinterpret_cast<uint32_t(*)[32]>(sv));
          tmem_ld32(sa + 32, *reinterpret_cast<uint32_t(*)[32]>(sv + 32));
          tmem_ld32(sa + 64, *reinterpret_cast<uint32_t(*)[32]>(sv + 64));
          tmem_ld32(sa + 96, *reinterpret_cast<uint32_t(*)[32]>(sv + 96));
          tmem_wait_ld();
          tc_fence_before();
          mbar_arrive(c.bar(B_S_EMPTY + sb));
        } else {
#pragma unroll
          for (int k = 0; k < KEYS; ++k) sv[k] = 0u;
        }
        ok = ok && wok;
        // scores in log2 units with the tree / range mask (in place)
        const int key0 = k_lo + i * KEYS;
        float m_tile = -INFINITY;
        if (valid && key0 + KEYS <= min(L, k_hi)) {
          // whole tile inside the prefix: every key visible
#pragma unroll
          for (int k = 0; k < KEYS; ++k) {
            const float xk = __uint_as_float(sv[k]) * sl2;
            sv[k] = __float_as_uint(xk);
            m_tile = fmaxf(m_tile, xk);
          }
        } else {
          // visibility of the tile's keys as 32-bit words: prefix keys
          // inside the split, tree keys L+u with bit u of the row's ancestor
          // mask, nothing at or past the split's end (keeps S in registers)
          const int n_pre = max(0, min(KEYS, min(L, k_hi) - key0));
          const int n_lim = max(0, min(KEYS, k_hi - key0));
          uint32_t vw[KEYS / 32];
#pragma unroll
          for (int w = 0; w < KEYS / 32; ++w) {
            const int lo = 32 * w;
            const uint32_t pre = n_pre >= lo + 32 ? 0xffffffffu : (n_pre <= lo ? 0u : (1u << (n_pre - lo)) - 1u);
            const uint32_t lim = n_lim >= lo + 32 ? 0xffffffffu : (n_lim <= lo ? 0u : (1u << (n_lim - lo)) - 1u);
            const int sft = key0 + lo - L;
            uint32_t tree = 0u;
            if (sft >= 0 && sft < 64) tree = (uint32_t)(mask_t >> sft);
            else if (sft < 0 && sft > -32) tree = (uint32_t)(mask_t << (-sft));
            vw[w] = valid ? ((pre | tree) & lim) : 0u;
          }
#pragma unroll
          for (int k = 0; k < KEYS; ++k) {
            const bool vis = (vw[k >> 5] >> (k & 31)) & 1u;
            const float xk = vis ? __uint_as_float(sv[k]) * sl2 : -INFINITY;
            sv[k] = __float_as_uint(xk);
            m_tile = fmaxf(m_tile, xk);
          }
        }
        float alpha = 1.f;
        if (m_tile > m_run + TAU || (m_run == -INFINITY && m_tile != -INFINITY)) {
          if (m_run != -INFINITY) {
            alpha = ex2(m_run - m_tile);
            l_run *= alpha;
          }
          m_run = m_tile;
        }
        const float m_use = m_run == -INFINITY ? 0.f : m_run;
        // hand P (and the rescale factor) to the O side with async stores
        const int slot = i % NP;
        ok = wait_warp(c, c.bar(B_P_EMPTY + slot), ((i / NP) & 1) ^ 1) && ok;
        const uint32_t pslot = peer_p + slot * P_SLOT_BYTES;
        const uint32_t pbar = peer_pfull + slot * 8;
        float lsum = 0.f;
#pragma unroll
        for (int ch = 0; ch < KEYS / 8; ++ch) {          // 16-byte pieces of 8 keys
          uint32_t w[4];
#pragma unroll
          for (int q = 0; q < 4; ++q) {
            const float p0 = ex2(__uint_as_float(sv[8 * ch + 2 * q]) - m_use);
            const float p1 = ex2(__uint_as_float(sv[8 * ch + 2 * q + 1]) - m_use);
            lsum += p0 + p1;
            w[q] = pack_bf16x2(p0, p1);
          }
          const int kb = ch >> 3, piece = ch & 7;
          if (ok)
            st_async_v4(pslot + kb * P_KBLOCK_BYTES + r * 128 + ((piece ^ (r & 7)) << 4), w[0], w[1], w[2],
                        w[3], pbar);
        }
        l_run += lsum;
        if (ok) st_async_f32(pslot + P_BYTES + r * 4, alpha, pbar);
      }
      // final row statistics for the O side's epilogue
      const uint32_t peer_stats = mapa(base + OFF_STATS, 1);
      const uint32_t peer_sbar = mapa(c.bar(B_STATS), 1);
      st_async_f32(peer_stats + r * 4, l_run, peer_sbar);
      st_async_f32(peer_stats + ROWS * 4 + r * 4, m_run, peer_sbar);
    }
  } else {
    // ======================================================= O side (CTA 1)
    if (warp == 0 && lane == 0) {
      // ---------------- V producer: 32 keys x 512 dims per stage
      int issued = 0;
      const int n_sub = (KEYS / VKEYS) * n_tiles;
      for (int u = 0; u < n_sub; ++u) {
        const int st = u % V_STAGES;
        if (!wait_bar(c, c.bar(B_V_EMPTY + st), ((u / V_STAGES) & 1) ^ 1)) break;
        mbar_arrive_expect_tx(c.bar(B_V_FULL + st), V_STAGE_BYTES);
        const int32_t y = (int32_t)(kv_base + k_lo + u * VKEYS);
        const uint32_t dst = base + OFF_RING + st * V_STAGE_BYTES;
        for (int blk = 0; blk < PV_BLOCKS; ++blk)
          tma_load_2d(dst + blk * VBLOCK_BYTES, &tmap_v, c.bar(B_V_FULL + st), blk * 64, y);
        issued = u + 1;
      }
      for (int u = max(0, issued - V_STAGES); u < issued; ++u)
        wait_bar(c, c.bar(B_V_FULL + u % V_STAGES), (u / V_STAGES) & 1, true);
    } else if (warp == 1 && lane == 0) {
      // ---------------- PV MMA issuer: O[128 x 512] += P[128 x 128] . V[128 x 512]
      for (int i = 0; i < n_tiles; ++i) {
        const int slot = i % NP;
        if (!wait_bar(c, c.bar(B_READY + slot), (i / NP) & 1)) break;
        fence_proxy_async_smem();          // P arrived by st.async; the MMA reads it
        bool ok = true;
        const uint32_t pbuf = base + OFF_P + slot * P_SLOT_BYTES;
        for (int h = 0; ok && h < KEYS / VKEYS; ++h) {
          const int u = (KEYS / VKEYS) * i + h, st = u % V_STAGES;
          if (!wait_bar(c, c.bar(B_V_FULL + st), (u / V_STAGES) & 1)) { ok = false; break; }
          tc_fence_after();
          const uint32_t vst = base + OFF_RING + st * V_STAGE_BYTES;
#pragma unroll
          for (int kk = 0; kk < VKEYS / 16; ++kk) {
            const int k = (VKEYS / 16) * h + kk;       // 16-key step within the tile
            const uint64_t adesc = sw128_desc(pbuf + (k >> 2) * P_KBLOCK_BYTES + (k & 3) * 32, 16, 1024);
#pragma unroll
            for (int nh = 0; nh < 2; ++nh) {
              // V: K (keys) rows of 128 B, 8-key groups 1024 B apart (SBO),
              // 64-dim column blocks VBLOCK_BYTES apart (LBO), N = 256 dims
              const uint64_t bdesc = sw128_desc(vst + nh * 4 * VBLOCK_BYTES + kk * 2048, VBLOCK_BYTES, 1024);
              mma_ss(tmem + nh * 256, adesc, bdesc, IDESC_PV, (i > 0 || k > 0) ? 1u : 0u);
            }
          }
          tc_commit(c.bar(B_V_EMPTY + st));
        }
        if (!ok) break;
        tc_commit(c.bar(B_PV_DONE + slot));
      }
      tc_commit(c.bar(B_O_DRAIN));
      wait_bar(c, c.bar(B_O_DRAIN), 0, true);
    } else if (warp == 2 && lane == 0) {
      // ---------------- P-slot releaser: after tile i's MMAs, re-arm its slot
      // and tell the S side it may overwrite it
      const uint32_t peer_pempty = mapa(c.bar(B_P_EMPTY), 0);
      for (int i = 0; i < n_tiles; ++i) {
        const int slot = i % NP;
        if (!wait_bar(c, c.bar(B_PV_DONE + slot), (i / NP) & 1)) break;
        if (i + NP < n_tiles) {
          // relaxed: the MMAs that read the slot are complete (commit observed),
          // and the slot's next bytes arrive by complete_tx; a release-ordered
          // remote arrive costs ~4x more on this part (measured)
          mbar_arrive_expect_tx(c.bar(B_P_FULL + slot), P_MSG_BYTES);
          mbar_arrive_remote_relaxed(peer_pempty + slot * 8);
        }
      }
    } else if (warp >= WG_FIRST_WARP) {
      // ---------------- rescale + epilogue warpgroup: thread <-> output row
      const int sp = warp & 3;
      const int r = sp * 32 + lane;
      const int row = row0 + r;
      const bool valid = row < rows_b;
      const uint32_t lane_base = (uint32_t)(sp * 32) << 16;
      bool ok = true;
      for (int i = 0; i < n_tiles; ++i) {
        const int slot = i % NP;
        ok = wait_warp(c, c.bar(B_P_FULL + slot), (i / NP) & 1) && ok;
        const float al = *reinterpret_cast<volatile float*>(smem + OFF_P + slot * P_SLOT_BYTES + P_BYTES + r * 4);
        const bool need = ok && i > 0 && al != 1.f;
        if (__any_sync(0xffffffffu, need)) {
          // O must be quiescent: wait for tile i-1's MMAs, then scale the rows
          ok = wait_warp(c, c.bar(B_PV_DONE + (i - 1) % NP), ((i - 1) / NP) & 1) && ok;
          if (__all_sync(0xffffffffu, ok)) {
            __syncwarp();
            tc_fence_after();
            const float f = need ? al : 1.f;
#pragma unroll 1
            for (int cb = 0; cb < DC / 32; ++cb) {
              uint32_t v[32];
              tmem_ld32(tmem + lane_base + cb * 32, v);
              tmem_wait_ld();
#pragma unroll
              for (int k = 0; k < 32; ++k) v[k] = __float_as_uint(__uint_as_float(v[k]) * f);
              tmem_st32(tmem + lane_base + cb * 32, v);
            }
            tmem_wait_st();
            tc_fence_before();
          }
        }
        if (ok) mbar_arrive(c.bar(B_READY + slot));
      }
      // ---------------- epilogue: o = O / l, lse = ln2 * (m + log2 l)
      bool have_o = n_tiles > 0;
      if (have_o) {
        const int i = n_tiles - 1;
        have_o = wait_warp(c, c.bar(B_PV_DONE + i % NP), (i / NP) & 1, !ok);
      }
      have_o = __all_sync(0xffffffffu, have_o);
      ok = wait_warp(c, c.bar(B_STATS), 0) && ok && have_o == (n_tiles > 0);
      __syncwarp();
      tc_fence_after();
      const float l = *reinterpret_cast<volatile float*>(smem + OFF_STATS + r * 4);
      const float m = *reinterpret_cast<volatile float*>(smem + OFF_STATS + ROWS * 4 + r * 4);
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
  if (p.total_rows < 1) return cudaErrorInvalidValue;
  auto make = [&](CUtensorMap* m, const void* ptr, uint64_t rows, uint64_t pitch_elems, uint32_t box_rows) {
    const cuuint64_t dims[2] = {(cuuint64_t)DQ, (cuuint64_t)rows};
    const cuuint64_t strides[1] = {(cuuint64_t)pitch_elems * 2};
    const cuuint32_t box[2] = {64, box_rows};
    const cuuint32_t estr[2] = {1, 1};
    return enc(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(ptr), dims, strides, box, estr,
               CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
               CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  };
  CUtensorMap tmap_kv, tmap_v, tmap_q;
  if (make(&tmap_kv, a.kv, (uint64_t)a.num_slots, DQ, KEYS) != CUDA_SUCCESS ||
      make(&tmap_v, a.kv, (uint64_t)a.num_slots, DQ, VKEYS) != CUDA_SUCCESS ||
      make(&tmap_q, a.q, (uint64_t)p.total_rows, (uint64_t)a.q_row_stride, ROWS) != CUDA_SUCCESS)
    return cudaErrorInvalidValue;
  static bool attr_set[64] = {};
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  if (dev < 0 || dev >= 64 || !attr_set[dev]) {
    e = cudaFuncSetAttribute(verify_tc_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, SMEM_BYTES);
    if (e != cudaSuccess) return e;
    if (dev >= 0 && dev < 64) attr_set[dev] = true;
  }
  verify_tc_kernel<<<2 * p.n_items, THREADS, SMEM_BYTES, stream>>>(tmap_kv, tmap_v, tmap_q, a, p);
  return cudaGetLastError();
}

int tc1_max_active_clusters() {
  static int cached[64] = {};
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) { cudaGetLastError(); return 0; }
  if (cached[dev] > 0) return cached[dev];
  if (cudaFuncSetAttribute(verify_tc_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, SMEM_BYTES) != cudaSuccess) {
    cudaGetLastError();
    return 0;
  }
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(2 * 64);
  cfg.blockDim = dim3(THREADS);
  cfg.dynamicSmemBytes = SMEM_BYTES;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = 2;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  int n = 0;
  if (cudaOccupancyMaxActiveClusters(&n, verify_tc_kernel, &cfg) != cudaSuccess) { cudaGetLastError(); return 0; }
  cached[dev] = n;
  return n;
}

}  // namespace kdv

// verify_tc2.cu -- tensor-core tree-verify MLA attention on 2-SM MMAs
// (tcgen05.mma cta_group::2, TMEM accumulators, TMA-staged operands).
//
// The operation (page "The Architecture of Diagnosis",
// section "Phase 1: Custom CUDA Kernels", item 2; latent dims from page "From
// Diagnosis to Deployment", section "The Second Thread"): per query row,
// s_j = scale (q_lat . c_kv[j] + q_rope . k_rope[j]), a softmax over the keys
// the row's tree node may see, o_lat = sum_j p_j c_kv[j], and the split's LSE.
//
// Why 2-SM pairs. Staging a 128-key x 576-dim KV tile for one 128-row MMA
// needs about as many shared-memory bytes per cycle for the TMA writes as the
// tensor core reads back, and together they exceed what one SM's shared
// memory delivers. In a cta_group::2 MMA the B operand is split across the
// two SMs of a pair, so each SM stages and reads only half of it.
//
// One work item = 256 query rows of one request and one key split, on a
// 4-CTA cluster:
//   CTA 0 + CTA 1 ("S pair"): S = Q K^T with M=256 (rows 0-127 in CTA 0,
//     128-255 in CTA 1), N=256 keys, K=576, both operands in shared memory.
//     Each CTA keeps its rows' q (q_lat || q_rope, 144 KB) in shared memory
//     for the whole item and stages the KV rows of its half of the keys (128
//     of every 256) through a 16 KB x 5 ring, one 64-dim K-block per stage;
//     the next tile's rows are prefetched into L2 meanwhile. TMEM holds two
//     S buffers of 256 columns, so the MMAs of tile i+1 (issued by CTA 0)
//     run while the softmax warps drain tile i. Two softmax warpgroups per
//     CTA (one row per thread, keys 0-127 and 128-255 of the tile) agree on
//     the row maximum (a barrier vote; an exchange through shared memory
//     only when some row's reference max may move), and each pushes its fp16
//     P half to the partner CTA on the O side with st.async, the second
//     warpgroup half a P tile behind the first so that one's exp2 work
//     overlaps the other's pushes.
//   CTA 2 + CTA 3 ("O pair"): O += P V with M=256, N=256 (two MMAs per 16
//     keys), K=16, per 128-key P tile. O (128 rows x 512 fp32) fills each
//     CTA's TMEM; each CTA stages 256 of the 512 V dims (the half of each
//     N=256 column range the MMA expects from it) through a 16 KB x 5 ring,
//     with TMA boxes from the call's fp16 copy of the latent rows (below),
//     and takes P tiles into 4 slots. CTA 2 issues the MMAs.
//
// Precision of P.V. The softmax numerators P are rounded to a 16-bit type
// before the P.V MMA, and that rounding is the kernel's dominant error. In
// bf16 (8 significant bits) it leaves a normalised mean error near 1e-3 of
// the output's RMS; in fp16 (11 bits) about 1.3e-4. A kind::f16 MMA takes A
// and B of one type, so V is read as fp16 too, from rows that
// latent_f16.cu writes before this kernel (which may be launched as that
// pass's programmatic dependent; only the V loads wait for it) (bf16 -> fp16 is exact for
// every latent value with 2^-14 <= |x| < 65536). V cannot be converted here:
// while the tensor core streams shared memory the load/store unit gets only
// ~5-10 B/clk of it (measured), so reading a 16 KB stage back through
// registers would take over a microsecond. P is at most 2^TAU = 256 by the
// lazy rescale rule, well inside fp16's range.
//
// Every MMA is N=256: with the TMA stream running beside it, N=128 MMAs on
// this part leave ~35 cycles per instruction unhidden, N=256 ones do not
// (measured). Cross-CTA arrivals are relaxed (see arrive_on).
//
// Softmax: one query row per thread; the running max moves only when a
// tile's max exceeds it by more than TAU (in log2 units), and then O is
// rescaled on the O side before the next P tile ("lazy rescale"). Every wait
// is bounded (TIMEOUT_NS, then KDV_DERR_TIMEOUT and an orderly exit). The
// split epilogue writes o = O / l and lse = ln 2 * (m + log2 l).
#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_fp16.h>

#include <algorithm>
#include <cstring>

#include "kdv_internal.cuh"
#include "sm100_ptx.cuh"
#ifdef KDV_TRACE
#include "kdv_trace.h"
#endif

namespace kdv {
namespace {

using namespace ptx;

constexpr int DQ = 576, DC = 512;
constexpr int ROWS = 128;                           // rows per CTA (256 per pair)
constexpr int STILE = 2 * TC_KEYS;                  // 256 keys per S tile (QK^T N)
constexpr int KEYS = TC_KEYS;                       // 128 keys per P tile
constexpr int HKEYS = STILE / 2;                    // keys of an S tile staged per S CTA
constexpr int VKEYS = 32;                           // keys per V stage
constexpr int KBLOCK_BYTES = HKEYS * 128;           // 128 keys x 64 dims, swizzled (16 KB)
constexpr int VBLOCK_BYTES = VKEYS * 128;           // 32 keys x 64 dims (4 KB)
constexpr int QBLOCK_BYTES = ROWS * 128;            // 128 rows x 64 dims (16 KB)
constexpr int QK_BLOCKS = DQ / 64;                  // 9 (8 latent + 1 rope)
constexpr int V_LOCAL_BLOCKS = 4;                   // V dim-blocks per O CTA per stage
constexpr int KV_STAGES = 5;                        // KV ring: one 16 KB K-block per stage
constexpr int V_STAGES = 5;
constexpr int V_STAGE_BYTES = V_LOCAL_BLOCKS * VBLOCK_BYTES;  // 16 KB
constexpr int NP = 4;                               // P slots per O CTA (slots 2j+hw: one pair per warpgroup)
constexpr int P_BYTES = ROWS * KEYS * 2;
constexpr int P_KCHUNK_BYTES = ROWS * 16;           // 8 keys of all 128 rows (interleaved core matrices)
constexpr int P_MSG_BYTES = P_BYTES + ROWS * 4;
constexpr int P_SLOT_BYTES = 33792;
constexpr int STATS_BYTES = 2 * ROWS * 4;
constexpr uint32_t TMEM_COLS = 512;               // S side: S buffer b at columns [256 b, 256 b + 256)
constexpr float TAU = 8.0f;
constexpr float LOG2E = 1.4426950408889634f;
constexpr float LN2 = 0.6931471805599453f;
constexpr uint64_t TIMEOUT_NS = 1000000000ull;

// Shared-memory layout (same offsets in all four CTAs; mapa() relies on it).
//   S CTAs: [0, 147456) the CTA's 128 query rows, q_lat || q_rope, as nine
//           128B-swizzled K-blocks of 64 dims (the A operand of Q.K^T, read
//           by every tile); [147456, 229376) KV ring (5 x 16 KB, one K-block
//           of the CTA's 128 keys per stage); row-max / row-sum exchange.
//   O CTAs: [0, 81920) V ring (5 x 16 KB); 4 P slots; final stats.
constexpr int OFF_Q = 0;
constexpr int OFF_KV = OFF_Q + QK_BLOCKS * QBLOCK_BYTES;
constexpr int OFF_XCHG = OFF_KV + KV_STAGES * KBLOCK_BYTES;   // float [2][2][128] + [128] (S side)
constexpr int XCHG_BYTES = 3 * ROWS * 4;   // [2 hw][128] row maxima + [128] row sums
constexpr int OFF_VRING = 0;
constexpr int OFF_P = OFF_VRING + V_STAGES * V_STAGE_BYTES;
constexpr int OFF_STATS = OFF_P + NP * P_SLOT_BYTES;
constexpr int EPI_STAGE_BYTES = 16384;                         // per epilogue warp, over V ring + P slots
static_assert(OFF_VRING + 8 * EPI_STAGE_BYTES <= OFF_STATS, "epilogue staging overlaps the row statistics");
constexpr int OFF_MISC = OFF_XCHG + XCHG_BYTES > OFF_STATS + STATS_BYTES ? OFF_XCHG + XCHG_BYTES : OFF_STATS + STATS_BYTES;
static_assert(OFF_STATS + STATS_BYTES <= OFF_MISC, "O-side buffers overlap misc");
constexpr int OFF_BAR = OFF_MISC;
constexpr int NUM_BARS = 56;
constexpr int OFF_TMEM = OFF_BAR + NUM_BARS * 8;
constexpr int OFF_ABORT = OFF_TMEM + 4;
// teardown records: [0] some CTA of the cluster aborted (written by that CTA
// into all four); [1..4] per rescale warp, the first P tile it did not see
// arrive; [5..8] per rescale warp, whether it saw the row statistics arrive
constexpr int OFF_TEAR = OFF_ABORT + 4;
constexpr int SMEM_USED = OFF_TEAR + 9 * 4;
constexpr int SMEM_BYTES = SMEM_USED + 1024;
static_assert(SMEM_BYTES <= 232448, "exceeds 227 KB of shared memory");

// Barrier slots (each CTA initialises the slots its role uses).
// S pair. KV_FULL, S_EMPTY and Q_FULL are used in CTA 0 only (the MMA
// issuer's barriers; both CTAs' bytes count there); the others in both.
constexpr int B_KV_FULL = 0, B_KV_EMPTY = B_KV_FULL + KV_STAGES, B_S_FULL = B_KV_EMPTY + KV_STAGES,
              B_S_EMPTY = B_S_FULL + 2, B_P_EMPTY = B_S_EMPTY + 2, B_Q_FULL = B_P_EMPTY + NP,
              B_S_DRAIN = B_Q_FULL + QK_BLOCKS;
// O pair. V_FULL, READY and O_DRAIN in CTA 2 only.
constexpr int B_V_FULL = B_S_DRAIN + 1, B_V_EMPTY = B_V_FULL + V_STAGES, B_P_FULL = B_V_EMPTY + V_STAGES,
              B_READY = B_P_FULL + NP, B_PV_DONE = B_READY + NP, B_STATS = B_PV_DONE + NP,
              B_O_DRAIN = B_STATS + 1;
static_assert(B_O_DRAIN < NUM_BARS, "barrier slots");

constexpr uint16_t S_PAIR = 0x3, O_PAIR = 0xC;     // cluster CTA masks
constexpr uint32_t IDESC_QK = idesc_bf16_f32(256, 256, false, false);
constexpr uint32_t IDESC_QK16 = idesc_f16_f32(256, 256, false, false);   // latent dims in fp16 (staged pool)
constexpr uint32_t IDESC_PV = idesc_f16_f32(256, 256, false, true);   // fp16 P and V

constexpr int THREADS = 384;
constexpr int WG_FIRST_WARP = 4;      // warps 4-7: softmax keys 0-127 / O-side rescale + epilogue
constexpr int WG2_FIRST_WARP = 8;     // warps 8-11: softmax keys 128-255 (S side)

__device__ __forceinline__ uint64_t globaltimer() {
  uint64_t t;
  asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
  return t;
}

#ifdef KDV_TRACE
// Tracing build (kdv_trace.h): CTA c writes the global timer at stage s
// into kdv_trace_buf[c * KDV_TRACE_SLOTS + s].
__device__ unsigned long long kdv_trace_buf[KDV_TRACE_CTAS * KDV_TRACE_SLOTS];
__device__ __forceinline__ void trace_stamp(int slot) {
  if (blockIdx.x < KDV_TRACE_CTAS) kdv_trace_buf[blockIdx.x * KDV_TRACE_SLOTS + slot] = globaltimer();
}
#define KDV_STAMP(slot) trace_stamp(slot)
#else
#define KDV_STAMP(slot) ((void)0)
#endif

__device__ __forceinline__ uint32_t ld_shared_u32(uint32_t addr) {
  uint32_t v;
  asm volatile("ld.volatile.shared.u32 %0, [%1];" : "=r"(v) : "r"(addr) : "memory");
  return v;
}
__device__ __forceinline__ void st_shared_u32(uint32_t addr, uint32_t v) {
  asm volatile("st.volatile.shared.u32 [%0], %1;" :: "r"(addr), "r"(v) : "memory");
}

// Per-CTA wait context. It must stay in registers: a copy in local memory
// (which a reference passed to an out-of-line function forces) turns every
// wait into a load through the load/store unit, which the streaming tensor
// core leaves a few B/clk of the SM's shared-memory/L1 bandwidth -- enough to
// stall the MMA issuer hundreds of cycles per ring stage.
struct Ctx {
  uint32_t base;
  int32_t* d_err;
  uint64_t limit;        // ns a pipeline wait may take (drain waits always get TIMEOUT_NS)
  __device__ uint32_t bar(int i) const { return base + OFF_BAR + 8 * i; }
  __device__ uint32_t abort_addr() const { return base + OFF_ABORT; }
};

// The part of a bounded wait that runs once the first probe failed: it takes
// scalars only, so calling it out of line keeps nothing of the caller in memory.
__device__ __noinline__ bool wait_bar_slow(uint32_t bar, uint32_t parity, uint32_t abort_addr, int32_t* d_err,
                                           uint64_t lim, bool drain) {
  const uint64_t t0 = globaltimer();
  for (uint32_t it = 1;; ++it) {
    if (mbar_try_wait(bar, parity)) return true;
    if ((it & 63) == 0) {
      if (!drain && ld_shared_u32(abort_addr) != 0) return false;
      if (globaltimer() - t0 > lim) {
        st_shared_u32(abort_addr, 1u);
        record_error(d_err, KDV_DERR_TIMEOUT);
        return false;
      }
    }
  }
}

// Bounded wait for phase `parity` of `bar`. A pipeline wait gives up after
// c.limit ns (recording KDV_DERR_TIMEOUT and raising this CTA's abort flag)
// or as soon as the flag is up; a drain wait -- one that retires this CTA's
// own copies and MMAs before it exits -- ignores the flag and waits up to
// TIMEOUT_NS.
__device__ __forceinline__ bool wait_bar(const Ctx& c, uint32_t bar, uint32_t parity, bool drain = false) {
  if (mbar_try_wait(bar, parity)) return true;
  return wait_bar_slow(bar, parity, c.abort_addr(), c.d_err, drain ? TIMEOUT_NS : c.limit, drain);
}

// Wait for phase `parity` of `bar` until the globaltimer reaches `deadline`.
__device__ __noinline__ bool wait_until(uint32_t bar, uint32_t parity, uint64_t deadline) {
  while (!mbar_try_wait(bar, parity))
    if (globaltimer() > deadline) return false;
  return true;
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

// Arrive on barrier `bar` (local offset) of CTA `rank`: a local arrive when
// it is this CTA, else a relaxed remote arrive. Every cross-CTA arrival in
// this kernel is relaxed. Each follows work the arriving thread has already
// completed -- tcgen05.ld / tcgen05.st it waited for (tcgen05.wait), bytes
// that reached its CTA through complete_tx, or its own shared-memory stores
// of a V stage -- and, where the pair's MMA will read shared memory of the
// arriving CTA, a fence.proxy.async that orders that CTA's writes before
// async-proxy reads. A release-ordered remote arrive costs ~1800 cycles on
// this part against ~440 for a relaxed one (measured), enough to starve the
// pipeline.
__device__ __forceinline__ void arrive_on(uint32_t bar, uint32_t rank, uint32_t my_rank) {
  if (rank == my_rank) mbar_arrive(bar);
  else mbar_arrive_remote_relaxed(mapa(bar, rank));
}

// Pool row of logical key j (paged KV, page_size 1). Keys past the split's
// end (the tail of a partial tile, masked out by the softmax) reuse the last
// key's row, so every row read is one the caller handed in; a slot outside
// [0, num_slots) is reported and replaced by row 0.
__device__ __forceinline__ int32_t paged_slot(const VerifyArgs& a, int64_t kv_base, int j, int k_hi) {
  const int jj = j < k_hi ? j : k_hi - 1;
  int32_t s = a.page_table[kv_base + jj];
  if (s < 0 || (int64_t)s >= a.num_slots) {
    record_error(a.d_err, KDV_DERR_BAD_SLOT);
    s = 0;
  }
  return s;
}

// PAGED: the keys gathered through the page table (bf16); LAT16: a staged
// pool, Q.K^T's latent dims read in fp16 (never both)
template <bool PAGED, bool LAT16>
__global__ void __launch_bounds__(THREADS, 1) __cluster_dims__(4, 1, 1)
verify_tc2_kernel(const __grid_constant__ CUtensorMap tmap_kv, const __grid_constant__ CUtensorMap tmap_v,
                  const __grid_constant__ CUtensorMap tmap_q, const __grid_constant__ CUtensorMap tmap_o,
                  const __grid_constant__ CUtensorMap tmap_l16, const __grid_constant__ CUtensorMap tmap_q16,
                  const int o_tma, const VerifyArgs a, const VerifyPlan p) {
  extern __shared__ uint8_t smem_raw[];
  const uint32_t raw = smem_u32(smem_raw);
  const uint32_t base = (raw + 1023u) & ~1023u;
  uint8_t* smem = smem_raw + (base - raw);
  const uint32_t rank = cluster_ctarank();
  const bool s_side = rank < 2;
  const uint32_t half = rank & 1;                 // which 128 rows (and which operand half)
  const bool leader = half == 0;                  // CTA 0 / CTA 2 issue the pair's MMAs
  const uint32_t lead_rank = rank & ~1u;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

  Ctx c;
  c.base = base;
  c.d_err = a.d_err;
  c.limit = a.wait_limit_ns > 0 ? a.wait_limit_ns : TIMEOUT_NS;

  // ---- work item ---------------------------------------------------------
  const int item = blockIdx.x >> 2;
  const int b = plan_request(p, item);
  const int local = item - p.item_base[b];
  const int split = local / p.tiles[b];
  const int rt = local - split * p.tiles[b];
  const int H = p.H, L = p.L[b], Tn = p.T[b];
  const int n_keys = L + Tn;
  const int rows_b = Tn * H;
  const int row0 = rt * (2 * ROWS) + (int)half * ROWS;   // this CTA's first row
  const int k_lo = min(split * p.chunk[b], n_keys);
  const int k_hi = min(k_lo + p.chunk[b], n_keys);
  const int n_stiles = (k_hi - k_lo + STILE - 1) / STILE;
  auto stile_key = [&](int i) { return k_lo + i * STILE; };
  const int n_ptiles = 2 * n_stiles;
  const int64_t kv_base = a.kv_off[b];
  constexpr bool lat16 = LAT16 && !PAGED;

  // ---- setup -------------------------------------------------------------
  if (threadIdx.x == 0) {
    st_shared_u32(c.abort_addr(), 0u);
    reinterpret_cast<volatile uint32_t*>(smem + OFF_TEAR)[0] = 0;
    if (s_side) {
      for (int i = 0; i < KV_STAGES; ++i) {
        mbar_init(c.bar(B_KV_FULL + i), 1);              // the leader's expect_tx (both CTAs' bytes)
        mbar_init(c.bar(B_KV_EMPTY + i), 1);
      }
      for (int i = 0; i < 2; ++i) {
        mbar_init(c.bar(B_S_FULL + i), 1);
        mbar_init(c.bar(B_S_EMPTY + i), 16);             // every softmax warp of both S CTAs
      }
      for (int i = 0; i < NP; ++i) mbar_init(c.bar(B_P_EMPTY + i), 1);
      for (int i = 0; i < QK_BLOCKS; ++i) mbar_init(c.bar(B_Q_FULL + i), 1);
      mbar_init(c.bar(B_S_DRAIN), 1);
      tma_prefetch_desc(&tmap_kv);
      tma_prefetch_desc(&tmap_q);
    } else {
      for (int i = 0; i < V_STAGES; ++i) {
        mbar_init(c.bar(B_V_FULL + i), 1);               // the leader's expect_tx (both CTAs' bytes)
        mbar_init(c.bar(B_V_EMPTY + i), 1);
      }
      for (int i = 0; i < NP; ++i) {
        mbar_init(c.bar(B_P_FULL + i), 1);
        mbar_init(c.bar(B_READY + i), 8);                // the rescale warps of both O CTAs
        mbar_init(c.bar(B_PV_DONE + i), 1);
      }
      mbar_init(c.bar(B_STATS), 1);
      mbar_init(c.bar(B_O_DRAIN), 1);
      for (int i = 0; i < NP; ++i) mbar_arrive_expect_tx(c.bar(B_P_FULL + i), P_MSG_BYTES);
      mbar_arrive_expect_tx(c.bar(B_STATS), STATS_BYTES);
      tma_prefetch_desc(&tmap_v);
    }
    fence_mbar_init();
  }
  if (warp == 2) {
    tmem_alloc2(base + OFF_TMEM, TMEM_COLS);
    tmem_relinquish2();
  }
  __syncwarp();
  tc_fence_before();
  cluster_sync();
  tc_fence_after();
  const uint32_t tmem = *reinterpret_cast<volatile uint32_t*>(smem + OFF_TMEM);
  if (threadIdx.x == 0) KDV_STAMP(KDV_TRACE_SETUP);

  if (s_side && leader && warp == 2 && lane == 0) {
    // device copies of the lengths against the host copies the plan used
    if (a.prefix_len != nullptr && a.prefix_len[b] != L) record_error(a.d_err, KDV_DERR_BAD_LENGTH);
    if (a.tree_off != nullptr && a.tree_off[b] != p.tree_base[b]) record_error(a.d_err, KDV_DERR_BAD_LENGTH);
    if ((int64_t)a.kv_off[b + 1] - kv_base < (int64_t)n_keys) record_error(a.d_err, KDV_DERR_BAD_LENGTH);
  }
  if (s_side) {
    // ======================================================= S pair
    if (warp == 0 && (PAGED || lane == 0)) {
      // ---------------- producer (both S CTAs): this CTA's 128 query rows
      // (nine K-blocks, kept for the whole item) and its 128 of every 256 KV
      // rows, one K-block per ring stage; everything counts on the leader's
      // barriers. Contiguous KV: TMA boxes, and the next tile's rows are
      // prefetched into L2 while this tile streams. Paged KV: TMA four-row
      // gathers through the page table, lane l taking keys 4l..4l+3 of the
      // CTA's 128 (plain loads or cp.async would go through the load/store
      // unit, which the streaming tensor core leaves only a few B/clk of
      // shared-memory bandwidth).
      const int n_stg = n_stiles * QK_BLOCKS;
      int issued = 0;
      // paged KV: lane l looks up keys 4l..4l+3 of this CTA's 128 one tile
      // ahead, so the page-table latency stays off the path
      int32_t slot[4] = {0, 0, 0, 0}, nslot[4] = {0, 0, 0, 0};
      if (PAGED && n_stiles > 0) {
        const int j0 = stile_key(0) + (int)half * HKEYS + 4 * lane;
#pragma unroll
        for (int q = 0; q < 4; ++q) nslot[q] = paged_slot(a, kv_base, j0 + q, k_hi);
      }
      // The query K-blocks go out interleaved with the first KV stages
      // (q_k just before KV stage k while the ring fills, then the rest), so the first tile's MMAs
      // start once block 0 of both has landed rather than after all of q.
      const int32_t qy = (int32_t)((int64_t)p.tree_base[b] * H + row0);
      int q_issued = 0;
      auto issue_q = [&](int upto) {
        if (lane == 0)
          for (; q_issued < upto; ++q_issued) {
            if (leader) mbar_arrive_expect_tx(c.bar(B_Q_FULL + q_issued), 2 * QBLOCK_BYTES);
            tma_load_2d_pair(base + OFF_Q + q_issued * QBLOCK_BYTES,
                             lat16 && q_issued < QK_BLOCKS - 1 ? &tmap_q16 : &tmap_q,
                             mapa(c.bar(B_Q_FULL + q_issued), lead_rank), q_issued * 64, qy);
          }
      };
      // A free ring stage is waited for like a drain (no abort check, 1 s):
      // both producers of the pair watch the same multicast commits, so they
      // issue the same stages -- the leader's drain below covers the pair's
      // loads only if neither producer goes on after the other stopped.
      for (int g = 0; g < n_stg; ++g) {
        const int st = g % KV_STAGES;
        const uint32_t eparity = ((g / KV_STAGES) & 1) ^ 1;
        if (!(PAGED ? wait_warp(c, c.bar(B_KV_EMPTY + st), eparity, true)
                    : wait_bar(c, c.bar(B_KV_EMPTY + st), eparity, true)))
          break;
        const int tile = g / QK_BLOCKS, blk = g % QK_BLOCKS;
        if (g < KV_STAGES) issue_q(g + 1);
        const uint32_t dst = base + OFF_KV + st * KBLOCK_BYTES;
        if (leader && lane == 0) mbar_arrive_expect_tx(c.bar(B_KV_FULL + st), 2 * KBLOCK_BYTES);
        const uint32_t fb = mapa(c.bar(B_KV_FULL + st), lead_rank);
        if (PAGED) {
          if (blk == 0) {
#pragma unroll
            for (int q = 0; q < 4; ++q) slot[q] = nslot[q];
            if (tile + 1 < n_stiles) {
              const int j0 = stile_key(tile + 1) + (int)half * HKEYS + 4 * lane;
#pragma unroll
              for (int q = 0; q < 4; ++q) nslot[q] = paged_slot(a, kv_base, j0 + q, k_hi);
            }
          }
          tma_gather4_pair(dst + lane * 512, &tmap_kv, fb, blk * 64, slot[0], slot[1], slot[2], slot[3]);
        } else {
          const int32_t y = (int32_t)(kv_base + stile_key(tile) + (int)half * HKEYS);
          // staged pool: latent K-blocks from the fp16 rows, the rope block
          // from the staged k_rope rows (its columns start at 0 there)
          auto kv_map = [&](int e) { return lat16 && e < QK_BLOCKS - 1 ? &tmap_l16 : &tmap_kv; };
          auto kv_x = [&](int e) { return lat16 && e == QK_BLOCKS - 1 ? 0 : e * 64; };
          if (blk == 0 && tile + 1 < n_stiles)
            for (int e = 0; e < QK_BLOCKS; ++e) tma_prefetch_l2(kv_map(e), kv_x(e), y + STILE);
          tma_load_2d_pair(dst, kv_map(blk), fb, kv_x(blk), y);
        }
        issued = g + 1;
        if (g == KV_STAGES - 1) issue_q(QK_BLOCKS);
      }
      if (leader && lane == 0) {
        // retire copies in flight (both halves count on the leader's barriers)
        for (int blk = 0; blk < q_issued; ++blk) wait_bar(c, c.bar(B_Q_FULL + blk), 0, true);
        for (int g = max(0, issued - KV_STAGES); g < issued; ++g)
          wait_bar(c, c.bar(B_KV_FULL + g % KV_STAGES), (g / KV_STAGES) & 1, true);
      }
      // every load of this S CTA is issued: a programmatic dependent (the
      // merge kernel) may launch as far as this CTA is concerned
      asm volatile("griddepcontrol.launch_dependents;");
    } else if (warp == 1 && lane == 0 && leader) {
      // ---------------- pair MMA issuer: S[256 x 256] = Q[256 x 576] . K^T,
      // both operands in shared memory, into the two TMEM S buffers in turn:
      // the MMAs of tile i+1 run while the softmax warps drain tile i. The
      // first tile waits for each query K-block as it lands.
      bool ok = true;
      for (int i = 0; ok && i < n_stiles; ++i) {
        const int sb = i & 1;
        if (!wait_bar(c, c.bar(B_S_EMPTY + sb), ((i >> 1) & 1) ^ 1)) break;
        tc_fence_after();
        const uint32_t d = tmem + (uint32_t)(sb * 256);
        for (int blk = 0; blk < QK_BLOCKS; ++blk) {
          const int g = i * QK_BLOCKS + blk, st = g % KV_STAGES;
          if ((i == 0 && !wait_bar(c, c.bar(B_Q_FULL + blk), 0)) ||
              !wait_bar(c, c.bar(B_KV_FULL + st), (g / KV_STAGES) & 1)) {
            ok = false;
            break;
          }
          tc_fence_after();
          const uint32_t qb = base + OFF_Q + blk * QBLOCK_BYTES;
          const uint32_t kb = base + OFF_KV + st * KBLOCK_BYTES;
#pragma unroll
          for (int kk = 0; kk < 4; ++kk)
            mma2_ss(d, sw128_desc(qb + kk * 32, 16, 1024), sw128_desc(kb + kk * 32, 16, 1024),
                    lat16 && blk < QK_BLOCKS - 1 ? IDESC_QK16 : IDESC_QK, (blk > 0 || kk > 0) ? 1u : 0u);
          tc_commit2_mc(c.bar(B_KV_EMPTY + st), S_PAIR);
        }
        if (!ok) break;
        tc_commit2_mc(c.bar(B_S_FULL + sb), S_PAIR);
        if (i == 0) KDV_STAMP(KDV_TRACE_S_MMA_T0);
        if (i == 1) KDV_STAMP(KDV_TRACE_S_MMA_T1);
        if (i == n_stiles - 1) KDV_STAMP(KDV_TRACE_S_MMA_LAST);
      }
      tc_commit2_mc(c.bar(B_S_DRAIN), (uint16_t)(1u << rank));
      wait_bar(c, c.bar(B_S_DRAIN), 0, true);
    } else if (warp >= WG_FIRST_WARP) {
      // ---------------- softmax warpgroups (both S CTAs): thread <-> row;
      // warpgroup hw takes keys [128*hw, 128*hw + 128) of every S tile
      const int hw = warp >= WG2_FIRST_WARP ? 1 : 0;
      const int sp = warp & 3;
      const int r = sp * 32 + lane;
      const int row = row0 + r;
      const bool valid = row < rows_b;
      const uint32_t lane_base = (uint32_t)(sp * 32) << 16;
      // [2 hw][128] row maxima (+ [128] final sums); one buffer suffices:
      // every tile's vote is a barrier between one exchange's reads and the
      // next exchange's writes
      float* xchg = reinterpret_cast<float*>(smem + OFF_XCHG);
      bool ok = true;
      const uint64_t mask_t = valid ? a.mask[p.tree_base[b] + row / H] : 0ull;
      // a warp whose 32 rows all lie past the request's last row (the tail
      // of its last row tile) sends zeros and does no softmax work
      const bool warp_rows = __any_sync(0xffffffffu, valid);
      const float sl2 = a.scale * LOG2E;
      float m_run = -INFINITY, l_part = 0.f;
      const uint32_t o_rank = 2 + half;                       // this CTA's O partner
      const uint32_t pslot0 = mapa(base + OFF_P, o_rank);
      const uint32_t pbar0 = mapa(c.bar(B_P_FULL), o_rank);
      for (int i = 0; i < n_stiles; ++i) {
        ok = wait_warp(c, c.bar(B_S_FULL + (i & 1)), (i >> 1) & 1) && ok;
        if (i == 0 && warp == WG_FIRST_WARP && lane == 0) KDV_STAMP(KDV_TRACE_SM0_T0_READY);
        const bool wok = __all_sync(0xffffffffu, ok);
        uint32_t sv[KEYS];
        if (wok) {
          __syncwarp();
          tc_fence_after();
          // one 128-column load: the S half arrives in a single TMEM round trip
          tmem_ld128(tmem + lane_base + (uint32_t)((i & 1) * 256 + hw * KEYS), sv);
          tmem_wait_ld();
          tc_fence_before();
          __syncwarp();
          if (lane == 0) arrive_on(c.bar(B_S_EMPTY + (i & 1)), lead_rank, rank);
        } else {
#pragma unroll
          for (int k = 0; k < KEYS; ++k) sv[k] = 0u;
        }
        ok = ok && wok;
        const int key0 = stile_key(i) + hw * KEYS;
        float m_half = -INFINITY;
        // the row max over raw logits, scaled once after: the scale is
        // positive (checked on the host), so max(s) * sl2 = max(s * sl2),
        // and the exp2 arguments below take the scale in one FMA
        if (valid && key0 + KEYS <= min(L, k_hi)) {
#pragma unroll
          for (int k = 0; k < KEYS; ++k) m_half = fmaxf(m_half, __uint_as_float(sv[k]));
        } else if (warp_rows) {
          // visibility of the tile's 128 keys as four 32-bit words: prefix
          // keys (j < L) inside the split, tree keys j = L+u with bit u of
          // the row's ancestor mask, nothing at or past the split's end
          const int n_pre = max(0, min(KEYS, min(L, k_hi) - key0));
          const int n_lim = max(0, min(KEYS, k_hi - key0));
          uint32_t vw[KEYS / 32];
#pragma unroll
          for (int w = 0; w < KEYS / 32; ++w) {
            const int lo = 32 * w;
            const uint32_t pre = n_pre >= lo + 32 ? 0xffffffffu : (n_pre <= lo ? 0u : (1u << (n_pre - lo)) - 1u);
            const uint32_t lim = n_lim >= lo + 32 ? 0xffffffffu : (n_lim <= lo ? 0u : (1u << (n_lim - lo)) - 1u);
            const int sft = key0 + lo - L;              // tree index of the word's first key
            uint32_t tree = 0u;
            if (sft >= 0 && sft < 64) tree = (uint32_t)(mask_t >> sft);
            else if (sft < 0 && sft > -32) tree = (uint32_t)(mask_t << (-sft));
            vw[w] = valid ? ((pre | tree) & lim) : 0u;
          }
#pragma unroll
          for (int k = 0; k < KEYS; ++k) {
            const bool vis = (vw[k >> 5] >> (k & 31)) & 1u;
            const float xk = vis ? __uint_as_float(sv[k]) : -INFINITY;
            sv[k] = __float_as_uint(xk);
            m_half = fmaxf(m_half, xk);
          }
        }
        m_half *= sl2;
        // Row max of the whole 256-key tile from both warpgroups -- needed
        // only if some row's reference max may move. One barrier vote
        // decides: when no half-tile max exceeds its row's m_run + TAU (and
        // no row sees its first finite logit), neither does the full-tile
        // max, so the exchange through shared memory (load/store-unit work
        // that the streaming tensor core starves) is skipped. Either way
        // both warpgroups take the same decision as with the exchange.
        const bool moves = m_half > m_run + TAU || (m_run == -INFINITY && m_half != -INFINITY);
        float m_tile = m_half;
        if (named_bar_or(1, 2 * 128, moves)) {
          volatile float* xm = xchg;
          xm[hw * ROWS + r] = m_half;
          named_bar_sync(1, 2 * 128);
          m_tile = fmaxf(m_half, xm[(hw ^ 1) * ROWS + r]);
        }
        float alpha = 1.f;
        if (m_tile > m_run + TAU || (m_run == -INFINITY && m_tile != -INFINITY)) {
          if (m_run != -INFINITY) {
            alpha = ex2(m_run - m_tile);
            l_part *= alpha;
          }
          m_run = m_tile;
        }
        const float m_use = m_run == -INFINITY ? 0.f : m_run;
        // P tile pt = 2i + hw goes to O-side slot pt % NP (the O side
        // consumes P tiles in order, slot by slot)
        const int pt = 2 * i + hw, pslot_i = pt % NP;
        const uint32_t pslot = pslot0 + pslot_i * P_SLOT_BYTES;
        const uint32_t pbar = pbar0 + pslot_i * 8;
        ok = wait_warp(c, c.bar(B_P_EMPTY + pslot_i), ((pt / NP) & 1) ^ 1) && ok;
        // The two warpgroups are staggered by half a P tile: warpgroup 1
        // starts once warpgroup 0 has pushed its first 64 keys, so one
        // warpgroup's exp2 work overlaps the other's DSMEM pushes instead of
        // both computing, then both pushing.
        // row sum in two lanes (even and odd keys), added once at the end;
        // the exp2 arguments two at a time (packed FMA)
        float2 lsum2 = make_float2(0.f, 0.f);
        const float2 sl2x2 = make_float2(sl2, sl2), negm = make_float2(-m_use, -m_use);
        if (hw == 1) named_bar_sync(2, 2 * 128);
        if (warp_rows) {
#pragma unroll
          for (int ch = 0; ch < KEYS / 8; ++ch) {
            uint32_t w[4];
#pragma unroll
            for (int q = 0; q < 4; ++q) {
              const float2 x = fma_f32x2(make_float2(__uint_as_float(sv[8 * ch + 2 * q]),
                                                     __uint_as_float(sv[8 * ch + 2 * q + 1])), sl2x2, negm);
              const float2 pp = make_float2(ex2(x.x), ex2(x.y));
              lsum2 = add_f32x2(lsum2, pp);
              w[q] = pack_f16x2(pp.x, pp.y);
            }
            // no-swizzle K-major layout: keys 8ch..8ch+7 of row r at ch*2048 + r*16,
            // so a warp's 32 rows fill 512 contiguous bytes per store
            if (ok) st_async_v4(pslot + ch * P_KCHUNK_BYTES + r * 16, w[0], w[1], w[2], w[3], pbar);
            if (hw == 0 && ch == KEYS / 16 - 1) named_bar_arrive(2, 2 * 128);
          }
        } else {
          if (hw == 0) named_bar_arrive(2, 2 * 128);
          if (ok) {
#pragma unroll 1
            for (int ch = 0; ch < KEYS / 8; ++ch) st_async_v4(pslot + ch * P_KCHUNK_BYTES + r * 16, 0u, 0u, 0u, 0u, pbar);
          }
        }
        l_part += lsum2.x + lsum2.y;
        // the O side rescales O before P tile 2i (slot 0); P tile 2i+1 needs none
        if (ok) st_async_f32(pslot + P_BYTES + r * 4, hw == 0 ? alpha : 1.f, pbar);
        if (i == 0 && warp == WG_FIRST_WARP && lane == 0) KDV_STAMP(KDV_TRACE_SM0_T0_DONE);
      }
      if (warp == WG_FIRST_WARP && lane == 0) KDV_STAMP(KDV_TRACE_SM0_DONE);
      if (warp == WG2_FIRST_WARP && lane == 0) KDV_STAMP(KDV_TRACE_SM1_DONE);
      // final row statistics (sum of both halves) for the O side's epilogue
      volatile float* xs = xchg + 2 * ROWS;
      named_bar_sync(1, 2 * 128);
      if (hw == 1) xs[r] = l_part;
      named_bar_sync(1, 2 * 128);
      if (hw == 0) {
        const float l = l_part + xs[r];
        const uint32_t peer_stats = mapa(base + OFF_STATS, o_rank);
        const uint32_t peer_sbar = mapa(c.bar(B_STATS), o_rank);
        st_async_f32(peer_stats + r * 4, l, peer_sbar);
        st_async_f32(peer_stats + ROWS * 4 + r * 4, m_run, peer_sbar);
      }
    }
  } else {
    // ======================================================= O pair
    if (warp == 0 && lane == 0) {
      // ---------------- V producer (both O CTAs): this CTA's 256 of the 512
      // fp16 dims of every 32 keys, read from the call's fp16 latent rows
      // (contiguous per request, whatever the pool's layout) and counted on
      // the leader's V_FULL; local block lb holds dims
      // 64*((lb/2)*4 + half*2 + lb%2), 128B-swizzled. Rows past the request's
      // keys are other requests' rows or past the end (read as zeros): finite
      // either way, and masked out by P = 0.
      int issued = 0;
      const int n_sub = (STILE / VKEYS) * n_stiles;
      // The fp16 rows may still be being written by the latent pass this
      // grid was launched to overlap (programmatic dependent launch): wait
      // for that grid's completion before the first V load. A no-op when the
      // grid was launched normally.
      asm volatile("griddepcontrol.wait;" ::: "memory");
      asm volatile("fence.proxy.async.global;" ::: "memory");
      KDV_STAMP(KDV_TRACE_V_READY);
      for (int u = 0; u < n_sub; ++u) {
        const int st = u % V_STAGES;
        if (!wait_bar(c, c.bar(B_V_EMPTY + st), ((u / V_STAGES) & 1) ^ 1, true)) break;
        if (leader) mbar_arrive_expect_tx(c.bar(B_V_FULL + st), 2 * V_STAGE_BYTES);
        const int key0 = stile_key(u / (STILE / VKEYS)) + (u % (STILE / VKEYS)) * VKEYS;
        const uint32_t dst = base + OFF_VRING + st * V_STAGE_BYTES;
        const uint32_t fb = mapa(c.bar(B_V_FULL + st), lead_rank);
        const int32_t y = p.v16_base[b] + key0;
        for (int lb = 0; lb < V_LOCAL_BLOCKS; ++lb) {
          const int gb = (lb >> 1) * 4 + (int)half * 2 + (lb & 1);
          tma_load_2d_pair(dst + lb * VBLOCK_BYTES, &tmap_v, fb, gb * 64, y);
        }
        issued = u + 1;
      }
      if (leader)
        for (int u = max(0, issued - V_STAGES); u < issued; ++u)
          wait_bar(c, c.bar(B_V_FULL + u % V_STAGES), (u / V_STAGES) & 1, true);
    } else if (warp == 1 && lane == 0 && leader) {
      // ---------------- pair MMA issuer: O[256 x 512] += P[256 x 128] . V[128 x 512]
      for (int i = 0; i < n_ptiles; ++i) {
        const int slot = i % NP;
        if (!wait_bar(c, c.bar(B_READY + slot), (i / NP) & 1)) break;
        bool ok = true;
        const uint32_t pbuf = base + OFF_P + slot * P_SLOT_BYTES;
        for (int h = 0; ok && h < KEYS / VKEYS; ++h) {
          const int u = (KEYS / VKEYS) * i + h, st = u % V_STAGES;
          if (!wait_bar(c, c.bar(B_V_FULL + st), (u / V_STAGES) & 1)) { ok = false; break; }
          tc_fence_after();
          const uint32_t vst = base + OFF_VRING + st * V_STAGE_BYTES;
#pragma unroll
          for (int kk = 0; kk < VKEYS / 16; ++kk) {
            const int k = (VKEYS / 16) * h + kk;
            const uint64_t adesc = interleave_desc(pbuf + k * 2 * P_KCHUNK_BYTES, P_KCHUNK_BYTES, 128);
#pragma unroll
            for (int nh = 0; nh < 2; ++nh) {
              // this CTA's 128 of the 256 columns: two 64-dim blocks, LBO apart
              const uint64_t bdesc = sw128_desc(vst + nh * 2 * VBLOCK_BYTES + kk * 2048, VBLOCK_BYTES, 1024);
              mma2_ss(tmem + nh * 256, adesc, bdesc, IDESC_PV, (i > 0 || k > 0) ? 1u : 0u);
            }
          }
          tc_commit2_mc(c.bar(B_V_EMPTY + st), O_PAIR);
        }
        if (!ok) break;
        tc_commit2_mc(c.bar(B_PV_DONE + slot), O_PAIR);
        if (i == 0) KDV_STAMP(KDV_TRACE_PV_T0);
        if (i == n_ptiles - 1) KDV_STAMP(KDV_TRACE_PV_LAST);
      }
      tc_commit2_mc(c.bar(B_O_DRAIN), (uint16_t)(1u << rank));
      wait_bar(c, c.bar(B_O_DRAIN), 0, true);
    } else if (warp == 3 && lane == 0) {
      // ---------------- P-slot releaser (both O CTAs)
      const uint32_t peer_pempty = mapa(c.bar(B_P_EMPTY), half);
      for (int i = 0; i < n_ptiles; ++i) {
        const int slot = i % NP;
        if (!wait_bar(c, c.bar(B_PV_DONE + slot), (i / NP) & 1)) break;
        if (i + NP < n_ptiles) {
          mbar_arrive_expect_tx(c.bar(B_P_FULL + slot), P_MSG_BYTES);
          mbar_arrive_remote_relaxed(peer_pempty + slot * 8);
        }
      }
    } else if (warp >= WG_FIRST_WARP) {
      // ---------------- rescale (warps 4-7) and epilogue (warps 4-11), both
      // O CTAs: thread <-> row; warpgroup eh stores columns [256*eh, 256*eh+256)
      const int ew = warp - WG_FIRST_WARP;
      const int eh = ew >> 2;
      const int sp = warp & 3;
      const int r = sp * 32 + lane;
      const int row = row0 + r;
      const bool valid = row < rows_b;
      const uint32_t lane_base = (uint32_t)(sp * 32) << 16;
      bool bad = false;
      if (eh == 0) {
        bool ok = true;
        int first_miss = n_ptiles;          // first P tile this warp did not see arrive
        for (int i = 0; i < n_ptiles; ++i) {
          const int slot = i % NP;
          const bool got = wait_warp(c, c.bar(B_P_FULL + slot), (i / NP) & 1);
          if (i == 0 && warp == WG_FIRST_WARP && lane == 0) KDV_STAMP(KDV_TRACE_O_P0);
          if (!got && first_miss == n_ptiles) first_miss = i;
          ok = got && ok;
          fence_proxy_async_smem();      // P arrived by st.async; the pair's MMA reads it
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
          __syncwarp();
          if (ok && lane == 0) arrive_on(c.bar(B_READY + slot), lead_rank, rank);
        }
        // the final MMAs and the row statistics (waited in order: every
        // earlier phase of these barriers is already known to be complete)
        bool have_o = n_ptiles > 0;
        if (have_o) {
          const int i = n_ptiles - 1;
          have_o = wait_warp(c, c.bar(B_PV_DONE + i % NP), (i / NP) & 1, !ok);
        }
        have_o = __all_sync(0xffffffffu, have_o);
        const bool got_stats = wait_warp(c, c.bar(B_STATS), 0);
        ok = got_stats && ok && have_o == (n_ptiles > 0);
        bad = !ok;
        if (lane == 0) {
          volatile uint32_t* tear = reinterpret_cast<volatile uint32_t*>(smem + OFF_TEAR);
          tear[1 + sp] = (uint32_t)first_miss;
          tear[5 + sp] = got_stats ? 1u : 0u;
        }
      }
      // warps 8-11 learn of the final MMA and the statistics through this barrier
      bad = named_bar_or(1, 2 * 128, bad);
      const bool have_o = n_ptiles > 0 && !bad;
      tc_fence_after();
      // the merge kernel that follows (a programmatic dependent) may launch
      // now; it waits for this grid to complete before it reads the partials
      asm volatile("griddepcontrol.launch_dependents;");
      if (warp == WG_FIRST_WARP && lane == 0) KDV_STAMP(KDV_TRACE_EPILOGUE);
      // ---------------- epilogue: o = O / l, lse = ln2 * (m + log2 l)
      const float l = *reinterpret_cast<volatile float*>(smem + OFF_STATS + r * 4);
      const float m = *reinterpret_cast<volatile float*>(smem + OFF_STATS + ROWS * 4 + r * 4);
      const float inv = (l > 0.f && !bad) ? 1.f / l : 0.f;
      const float lse = (l > 0.f && !bad) ? (m + __log2f(l)) * LN2 : -INFINITY;
      const int64_t orow = out_row_index(p, b, split, row);
      // Whole-warp rows go out through TMA stores of 4 KB boxes staged
      // 128B-swizzled in the V ring and P slots (free once the last PV is
      // done; 16 KB per warp, four boxes in flight): 32 rows x 32 fp32
      // columns, or, for the internal merge's fp16 partials, 32 rows x 64
      // fp16 columns. A warp straddling the end of the request stores row by
      // row.
      const int wrow0 = row0 + sp * 32;
      const bool warp_full = o_tma != 0 && !bad && wrow0 + 32 <= rows_b;
      const int64_t wy = out_row_index(p, b, split, wrow0);
      const uint32_t stage = base + OFF_VRING + ew * EPI_STAGE_BYTES;
      // 64 columns per step: two TMEM loads, one wait; then one fp16 box or
      // two fp32 boxes (staging buffer cb & 3, four boxes in flight)
      auto put_box = [&](int cb, int col, const uint32_t (&v)[32]) {
        if (warp_full) {
          const uint32_t buf = stage + (cb & 3) * 4096;
          if (cb >= 4) {
            if (lane == 0) bulk_wait_group_read<3>();
            __syncwarp();
          }
#pragma unroll
          for (int q = 0; q < 8; ++q)
            st_shared_v4(buf + lane * 128 + ((q ^ (lane & 7)) << 4), v[4 * q], v[4 * q + 1], v[4 * q + 2],
                         v[4 * q + 3]);
          fence_proxy_async_smem();
          __syncwarp();
          if (lane == 0) {
            tma_store_2d(&tmap_o, buf, col, (int32_t)wy);
            bulk_commit_group();
          }
        } else if (valid) {
          // 128 bytes of this row: 32 fp32 or 64 fp16 columns
          uint4* dst = p.part_f16 ? reinterpret_cast<uint4*>(reinterpret_cast<__half*>(a.o) + orow * DC + col)
                                  : reinterpret_cast<uint4*>(a.o + orow * DC + col);
#pragma unroll
          for (int q = 0; q < 8; ++q) dst[q] = make_uint4(v[4 * q], v[4 * q + 1], v[4 * q + 2], v[4 * q + 3]);
        }
      };
#pragma unroll 1
      for (int ck = 0; ck < 4; ++ck) {
        const int col = eh * 256 + ck * 64;
        uint32_t t0[32], t1[32];
        if (have_o) {
          tmem_ld32(tmem + lane_base + col, t0);
          tmem_ld32(tmem + lane_base + col + 32, t1);
          tmem_wait_ld();
        } else {
#pragma unroll
          for (int k = 0; k < 32; ++k) t0[k] = t1[k] = 0u;
        }
        if (p.part_f16) {
          uint32_t v[32];
#pragma unroll
          for (int k = 0; k < 16; ++k) {
            v[k] = pack_f16x2(__uint_as_float(t0[2 * k]) * inv, __uint_as_float(t0[2 * k + 1]) * inv);
            v[16 + k] = pack_f16x2(__uint_as_float(t1[2 * k]) * inv, __uint_as_float(t1[2 * k + 1]) * inv);
          }
          put_box(ck, col, v);
        } else {
#pragma unroll
          for (int k = 0; k < 32; ++k) {
            t0[k] = __float_as_uint(__uint_as_float(t0[k]) * inv);
            t1[k] = __float_as_uint(__uint_as_float(t1[k]) * inv);
          }
          put_box(2 * ck, col, t0);
          put_box(2 * ck + 1, col + 32, t1);
        }
      }
      if (warp == WG_FIRST_WARP && lane == 0) KDV_STAMP(KDV_TRACE_STORED);
      if (warp_full && lane == 0) bulk_wait_group_read<0>();
      __syncwarp();
      if (eh == 0 && valid && a.lse != nullptr) a.lse[orow] = lse;
    }
  }

  // ---- teardown ----------------------------------------------------------
  if (warp == WG_FIRST_WARP && lane == 0) KDV_STAMP(KDV_TRACE_TEARDOWN);
  // After an abort (a wait that ran out) the O side stops waiting for P
  // tiles, so st.async bytes from the S pair could still be in flight toward
  // an O CTA when it reaches this point. So: a CTA whose abort flag is up
  // tells all four CTAs; after the cluster barrier, if any CTA aborted, each
  // O CTA waits -- in order, against one deadline -- for every P-tile phase
  // and the statistics that none of its rescale warps saw arrive, and a
  // second barrier keeps every CTA resident until then. (Every phase the
  // drain waits for is at most the barrier's current one: a later phase of
  // a slot needs the MMAs of this one, which need all rescale warps to have
  // seen it.) The normal path costs one CTA barrier.
  volatile uint32_t* tear = reinterpret_cast<volatile uint32_t*>(smem + OFF_TEAR);
  __syncwarp();
  __syncthreads();
  if (threadIdx.x < 4 && ld_shared_u32(c.abort_addr()) != 0) st_cluster_u32(mapa(base + OFF_TEAR, threadIdx.x), 1u);
  tc_fence_before();
  cluster_sync();
  if (tear[0] != 0) {
    if (!s_side && threadIdx.x == 0 && n_ptiles > 0) {
      int from = 0;
      bool stats = false;
      for (int w = 0; w < 4; ++w) {
        from = max(from, (int)tear[1 + w]);
        stats = stats || tear[5 + w] != 0;
      }
      const uint64_t deadline = globaltimer() + TIMEOUT_NS;
      for (int i = from; i < n_ptiles; ++i) wait_until(c.bar(B_P_FULL + i % NP), (i / NP) & 1, deadline);
      if (!stats) wait_until(c.bar(B_STATS), 0, deadline);
    }
    cluster_sync();
  }
  if (warp == 2) {
    tc_fence_after();
    tmem_dealloc2(tmem, TMEM_COLS);
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

cudaError_t launch_verify_tc2(const VerifyArgs& a, const VerifyPlan& p, const void* v16, int64_t v16_rows,
                              bool after_latent, cudaStream_t stream) {
  EncodeTiledFn enc = encode_fn();
  if (enc == nullptr) return cudaErrorNotSupported;
  if (a.num_slots < 1 || a.num_slots > (int64_t)0x7fffffff) return cudaErrorInvalidValue;
  if (p.total_rows < 1) return cudaErrorInvalidValue;
  // 16-bit [rows][cols] with a row pitch, in 64-column boxes of box_rows rows
  auto make = [&](CUtensorMap* m, const void* ptr, uint64_t rows, uint64_t pitch_elems, uint32_t box_rows,
                  uint64_t cols = DQ, CUtensorMapDataType dt = CU_TENSOR_MAP_DATA_TYPE_BFLOAT16) {
    const cuuint64_t dims[2] = {(cuuint64_t)cols, (cuuint64_t)rows};
    const cuuint64_t strides[1] = {(cuuint64_t)pitch_elems * 2};
    const cuuint32_t box[2] = {64, box_rows};
    const cuuint32_t estr[2] = {1, 1};
    return enc(m, dt, 2, const_cast<void*>(ptr), dims, strides, box, estr,
               CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
               CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  };
  CUtensorMap tmap_kv, tmap_v, tmap_q, tmap_o, tmap_l16, tmap_q16;
  const bool paged = a.page_table != nullptr;
  if (v16 == nullptr || v16_rows < 1 || v16_rows > (int64_t)0x7fffffff) return cudaErrorInvalidValue;
  // V: the fp16 latent rows [v16_rows][512] in 32-row boxes
  {
    const cuuint64_t dims[2] = {(cuuint64_t)DC, (cuuint64_t)v16_rows};
    const cuuint64_t strides[1] = {(cuuint64_t)DC * 2};
    const cuuint32_t box[2] = {64, VKEYS};
    const cuuint32_t estr[2] = {1, 1};
    if (enc(&tmap_v, CU_TENSOR_MAP_DATA_TYPE_FLOAT16, 2, const_cast<void*>(v16), dims, strides, box, estr,
            CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
            CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
      return cudaErrorInvalidValue;
  }
  if (make(&tmap_q, a.q, (uint64_t)p.total_rows, (uint64_t)a.q_row_stride, ROWS) != CUDA_SUCCESS)
    return cudaErrorInvalidValue;
  if (a.q16 != nullptr) {
    // staged pool: kv holds only k_rope [keys][D_r]; the keys' latent dims
    // come from the fp16 rows, the queries' from q16, both in 128-row boxes
    if (paged || a.D_r != 64 ||
        make(&tmap_kv, a.kv, (uint64_t)a.num_slots, (uint64_t)a.D_r, HKEYS, (uint64_t)a.D_r) != CUDA_SUCCESS ||
        make(&tmap_l16, v16, (uint64_t)v16_rows, DC, HKEYS, DC, CU_TENSOR_MAP_DATA_TYPE_FLOAT16) != CUDA_SUCCESS ||
        make(&tmap_q16, a.q16, (uint64_t)p.total_rows, DC, ROWS, DC, CU_TENSOR_MAP_DATA_TYPE_FLOAT16) != CUDA_SUCCESS)
      return cudaErrorInvalidValue;
  } else {
    if (make(&tmap_kv, a.kv, (uint64_t)a.num_slots, DQ, paged ? 1 : HKEYS) != CUDA_SUCCESS)
      return cudaErrorInvalidValue;
    tmap_l16 = tmap_kv;     // unused
    tmap_q16 = tmap_q;
  }
  // output rows for the epilogue's TMA stores
  int64_t out_rows = 0;
  for (int b = 0; b < p.B; ++b)
    if (p.T[b] > 0) out_rows = std::max<int64_t>(out_rows, out_row_index(p, b, p.S[b] - 1, p.T[b] * p.H - 1) + 1);
  int o_tma = 0;
  std::memset(&tmap_o, 0, sizeof(tmap_o));
  if (out_rows > 0 && out_rows <= (int64_t)0x7fffffff && (reinterpret_cast<uintptr_t>(a.o) & 15) == 0) {
    // fp32 [rows][512] in 32x32 boxes, or the fp16 merge partials in 64x32 boxes
    const cuuint64_t dims[2] = {(cuuint64_t)DC, (cuuint64_t)out_rows};
    const cuuint64_t strides[1] = {(cuuint64_t)DC * (p.part_f16 ? 2 : 4)};
    const cuuint32_t box[2] = {p.part_f16 ? 64u : 32u, 32};
    const cuuint32_t estr[2] = {1, 1};
    o_tma = enc(&tmap_o, p.part_f16 ? CU_TENSOR_MAP_DATA_TYPE_FLOAT16 : CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 2, a.o,
                dims, strides, box, estr,
                CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_NONE,
                CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS ? 1 : 0;
  }
  static bool attr_set[64] = {};
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  using KernelFn = decltype(&verify_tc2_kernel<false, false>);
  const KernelFn kernels[3] = {verify_tc2_kernel<false, false>, verify_tc2_kernel<true, false>,
                               verify_tc2_kernel<false, true>};
  if (dev < 0 || dev >= 64 || !attr_set[dev]) {
    for (int i = 0; e == cudaSuccess && i < 3; ++i)
      e = cudaFuncSetAttribute(kernels[i], cudaFuncAttributeMaxDynamicSharedMemorySize, SMEM_BYTES);
    if (e != cudaSuccess) return e;
    if (dev >= 0 && dev < 64) attr_set[dev] = true;
  }
  const KernelFn kern = kernels[paged ? 1 : a.q16 != nullptr ? 2 : 0];
  if (paged || !after_latent) {
    kern<<<4 * p.n_items, THREADS, SMEM_BYTES, stream>>>(tmap_kv, tmap_v, tmap_q, tmap_o, tmap_l16, tmap_q16, o_tma, a, p);
    return cudaGetLastError();
  }
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(4 * p.n_items);
  cfg.blockDim = dim3(THREADS);
  cfg.dynamicSmemBytes = SMEM_BYTES;
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, kern, tmap_kv, tmap_v, tmap_q, tmap_o, tmap_l16, tmap_q16, o_tma, a, p);
}

#ifdef KDV_TRACE
}  // namespace kdv

extern "C" {
KDV_API kdv_status kdv_trace_clear(void* stream) {
  void* ptr = nullptr;
  if (cudaGetSymbolAddress(&ptr, kdv::kdv_trace_buf) != cudaSuccess) return KDV_ERR_CUDA;
  return cudaMemsetAsync(ptr, 0, sizeof(kdv::kdv_trace_buf), static_cast<cudaStream_t>(stream)) == cudaSuccess
             ? KDV_OK
             : KDV_ERR_CUDA;
}
KDV_API kdv_status kdv_trace_read(uint64_t* host_dst, int64_t n_words) {
  if (n_words < 0 || n_words > (int64_t)KDV_TRACE_CTAS * KDV_TRACE_SLOTS) return KDV_ERR_INVALID_ARG;
  if (n_words == 0) return KDV_OK;
  if (host_dst == nullptr) return KDV_ERR_INVALID_ARG;
  return cudaMemcpyFromSymbol(host_dst, kdv::kdv_trace_buf, (size_t)n_words * 8) == cudaSuccess ? KDV_OK
                                                                                             : KDV_ERR_CUDA;
}
}  // extern "C"

namespace kdv {
#endif

int tc2_max_active_clusters() {
  static int cached[64] = {};
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) { cudaGetLastError(); return 0; }
  if (cached[dev] > 0) return cached[dev];
  if (cudaFuncSetAttribute(verify_tc2_kernel<false, false>, cudaFuncAttributeMaxDynamicSharedMemorySize, SMEM_BYTES) != cudaSuccess) {
    cudaGetLastError();
    return 0;
  }
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(4 * 64);
  cfg.blockDim = dim3(THREADS);
  cfg.dynamicSmemBytes = SMEM_BYTES;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = 4;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  int n = 0;
  if (cudaOccupancyMaxActiveClusters(&n, verify_tc2_kernel<false, false>, &cfg) != cudaSuccess) { cudaGetLastError(); return 0; }
  cached[dev] = n;
  return n;
}

}  // namespace kdv

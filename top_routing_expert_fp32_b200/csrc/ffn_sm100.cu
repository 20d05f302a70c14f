// Grouped gated expert FFN on the 5th-generation tensor cores (tcgen05, sm_100a).
//   GEMM1: H[r] = act(X_perm[r] W1_e) (.) (X_perm[r] W2_e)     (act and product fused)
//   GEMM2: Y[r] = H[r] W3_e
// for every row r of expert e's segment [offsets[e], offsets[e+1]) -- LLMs-from-scratch
// ch.12, 12.1 (f_e(x) = [SiLU(x W1_e) (.) (x W2_e)] W3_e); Grok-1 book ch.5, 5.3.5 (GeGLU
// variant, x W_value times GELU(x W_gate)) and 5.3.2 (weights stacked [E, D, F] / [E, F, D]).
//
// Design (one persistent CTA per SM, 10 warps):
//   warp 0 lane 0 : TMA producer. Per k-block of 64: one 128x64 A box (X_perm or H rows,
//                   K-major, 128-byte swizzle) and four 64x64 B boxes from the 3-D weight
//                   tensor [E][K][N] (N contiguous = MN-major B, 128-byte swizzle). GEMM1 takes
//                   two boxes from W1 and two from W2 for the same 128 output columns, so one
//                   N=256 MMA produces both up-projections side by side.
//   warp 1        : allocates 512 TMEM columns (two 128x256 fp32 accumulators); lane 0 issues
//                   tcgen05.mma (M=128, N=256, K=16, bf16 -> fp32) and commits to barriers.
//   warps 2..9    : epilogue, two warps per TMEM lane quarter taking alternate 32-column
//                   chunks. tcgen05.ld of the accumulator rows (one row per thread), act in
//                   fp32, bf16 rounding, masked 16-byte stores (rows past the expert's segment
//                   are never written). The accumulator is double buffered, so the epilogue
//                   of tile i overlaps the main loop of tile i+1.
// CTA pairs (cta_group::2, M=256) split A by rows and B by columns between the two CTAs; wide
// pairs issue two N=256 MMAs per k-step into one 512-column accumulator (not double-buffered:
// the epilogue hands the lower 256 columns back first, and the next tile's MMAs into them start
// on the k-blocks already loaded). A last round of wide tiles that would keep at most half of
// the pairs busy runs as half tiles (one MMA per k-step, half the output columns). Single-CTA
// launches run only the CTAs that an even split of the rounds needs.
// Tiles: per expert ceil(M_e/128) row blocks x ceil(N/NT) column blocks. The column blocks
// are cut into groups of G; tiles run group by group, inside a group expert by expert, then
// column block, with row blocks innermost (consecutive CTAs share a weight column block
// through L2). G = all column blocks gives plain expert-by-expert order; a small G makes the
// CTAs resident at any moment work on several experts at once, so experts with few rows
// (bound by streaming their weights) run beside experts with many rows (bound by the MMAs).
// Per-expert row counts are read from device memory: the host never learns them.
// Scheduling: tiles are handed out in order by a global counter (one atomic per tile, taken
// by the TMA producer of the CTA, or of the pair's first CTA, a few k-blocks before the end of
// the current tile's loads) and passed to
// the MMA issuer and the epilogue (and to the second CTA of a pair) through a small ring of
// tile ids in shared memory. The tiles in flight are therefore always a window of
// consecutive tiles: the row blocks that share a weight column block run together, and a
// weight block or an expert's rows are read from DRAM about once, however unevenly the tiles
// progress. The counter and a count of finished CTAs live in the workspace header (zeroed by
// moe_workspace_init); the last CTA to finish resets both to zero, also after an error.
// Every barrier wait is bounded in time; on a timeout the CTA records
// MOE_DEVERR_WAIT_TIMEOUT, unwinds, drains its MMAs and frees its TMEM.
#include <algorithm>
#include <cmath>
#include <cstdio>
#include <cstdlib>
#include <cstring>
#include <mutex>

#include "common.cuh"
#include "internal.h"

namespace moe {
namespace {

constexpr int kRows = 128;                         // rows of A (and accumulator lanes) per CTA
constexpr int BN = 256;                            // UMMA N
constexpr int BK = 64;                             // k-block: one 128-byte swizzle row of bf16
constexpr int UK = 16;                             // K of one tcgen05.mma kind::f16
constexpr int kABytes = kRows * BK * 2;            // 16 KB
constexpr int kBoxBytes = 64 * BK * 2;             // 8 KB: 64 columns x 64 k-rows
constexpr int kAccCols = 256;
constexpr int kTmemCols = 512;
constexpr int kEpiWarps = 8;                       // two per TMEM lane quarter
constexpr int kThreads = 64 + 32 * kEpiWarps;      // producer warp, MMA warp, epilogue
constexpr int kMaxE = 64;
constexpr int kRing = 4;                           // tile ids in flight between the roles
constexpr int kGrabAhead = 4;                      // k-blocks before a tile's end to take the next id
constexpr int kStoreStage = 32 * 64;               // per epilogue warp: 32 rows x 32 bf16

// Per-variant shape: a single CTA computes 128-row tiles with the whole B; a CTA pair
// computes 256-row tiles, each CTA holding its 128 A rows and half of the B columns. A wide
// pair issues two N=256 MMAs per k-step into one 512-column accumulator (all of TMEM, so the
// accumulator is not double-buffered): each CTA then moves 48 KB per k-block for twice the
// FLOPs of the 32 KB of a plain pair, 25 % fewer bytes from L2 per FLOP.
template <bool PAIR, bool WIDE>
struct Shape {
  static_assert(PAIR || !WIDE, "wide tiles are CTA pairs");
  static constexpr int kTileRows = PAIR ? 256 : 128;
  static constexpr int kMmas = WIDE ? 2 : 1;                         // N=256 MMAs per k-step
  static constexpr int kAccBufs = WIDE ? 1 : 2;                      // accumulators in TMEM
  static constexpr int kBBoxes = PAIR ? 2 * kMmas : 4;               // 64-col B boxes per CTA
  static constexpr int kStages = PAIR ? (WIDE ? 4 : 6) : 4;  // fills the 227 KB of shared memory
  static constexpr int kBBytes = kBBoxes * kBoxBytes;
  static constexpr int kStageBytes = kABytes + kBBytes;
  static constexpr int kTxBytes = PAIR ? 2 * kStageBytes : kStageBytes;  // per stage, both CTAs
  static constexpr int kSmemBytes = kStages * kStageBytes + kEpiWarps * kStoreStage +
                                    1024 /*align*/ + 1024 /*barriers*/;
  static_assert(kSmemBytes <= 227 * 1024, "shared memory per CTA");
  // Instruction descriptor, kind::f16: D fp32, A bf16, B bf16, A K-major, B MN-major,
  // N = 256, M = tile rows.
  static constexpr uint32_t kIdesc = (1u << 4) | (1u << 7) | (1u << 10) | (0u << 15) |
                                     (1u << 16) | (static_cast<uint32_t>(BN >> 3) << 17) |
                                     (static_cast<uint32_t>(kTileRows >> 4) << 24);
  // Single-CTA tiles whose rows all fit in 64 (an expert's last row block) use M = 64: the
  // accumulator then holds row 16q + l in TMEM lane 32q + l (lanes 0-15 of each quarter).
  static constexpr uint32_t kIdesc64 = (1u << 4) | (1u << 7) | (1u << 10) | (0u << 15) |
                                       (1u << 16) | (static_cast<uint32_t>(BN >> 3) << 17) |
                                       (static_cast<uint32_t>(64 >> 4) << 24);
};

struct GemmParams {
  const int32_t* offsets;  // [E+1] expert segments of the A rows
  __nv_bfloat16* out;      // [rows, n_out]
  int E;
  int K;                   // reduction length (D for GEMM1, F for GEMM2)
  int n_out;               // output columns (F for GEMM1, D for GEMM2)
  int n_group;             // column blocks per tile group (>= 1)
  int l2_a;                // L2 eviction priority of the A rows (+1 last, 0 normal, -1 first)
  int l2_b;                // and of the expert weights
  int* err;
  int* sched;              // [2]: next tile to hand out, CTAs (or pairs) finished; zero at rest
  int static_order;        // 1: CTA (pair) u takes tiles u, u + units, ... (no counter)
  int halves;              // wide tiles split in two: 0 never, 1 a short last round, 2 all
  uint64_t timeout_ns;
};

// Stores a 32-bit value into the shared memory of a CTA of this cluster (address from
// mapa_shared); ordered before a later release.cluster arrival of the same thread.
__device__ __forceinline__ void st_dsmem_u32(uint32_t cluster_addr, uint32_t v) {
  asm volatile("st.shared::cluster.u32 [%0], %1;" ::"r"(cluster_addr), "r"(v) : "memory");
}

// Every CTA (the first CTA of every pair) calls this once, last: the one that finishes last
// returns the tile counter and the finished count to zero for the next launch.
__device__ __forceinline__ void sched_finish(int* sched, int ctas) {
  __threadfence();
  if (atomicAdd(&sched[1], 1) == ctas - 1) {
    atomicExch(&sched[0], 0);
    atomicExch(&sched[1], 0);
  }
}

template <bool DUAL, int ACT, bool PAIR, bool WIDE>
__global__ void __launch_bounds__(kThreads, 1)
    grouped_gemm_sm100(const __grid_constant__ CUtensorMap tmA,
                       const __grid_constant__ CUtensorMap tmB0,
                       const __grid_constant__ CUtensorMap tmB1, const GemmParams p) {
  using S = Shape<PAIR, WIDE>;
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  const uint32_t raw_addr = smem_u32(smem_raw);
  uint8_t* smem = smem_raw + ((1024u - (raw_addr & 1023u)) & 1023u);
  uint8_t* sA = smem;
  uint8_t* sB = smem + S::kStages * kABytes;
  uint8_t* sT = sB + S::kStages * S::kBBytes;  // [kEpiWarps][32 rows][64 B] store staging
  uint64_t* full = reinterpret_cast<uint64_t*>(sT + kEpiWarps * kStoreStage);
  uint64_t* empty = full + S::kStages;
  uint64_t* tfull = empty + S::kStages;
  uint64_t* tempty = tfull + 2;
  uint64_t* drain = tempty + 2;
  uint64_t* ring_full = drain + 1;            // [kRing] a tile id is in its slot
  uint64_t* ring_empty = ring_full + kRing;   // [kRing] every consumer has read the slot
  uint32_t* s_tmem = reinterpret_cast<uint32_t*>(ring_empty + kRing);
  volatile int* s_ring = reinterpret_cast<volatile int*>(s_tmem + 1);  // [kRing] tile ids
  int* s_mstart = const_cast<int*>(s_ring) + kRing;    // [E+1] first row block of expert e
  int* s_seg = s_mstart + (kMaxE + 1);                 // [E+1]

  constexpr int NT = (DUAL ? 128 : 256) * S::kMmas;  // output columns per tile
  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const int n_blocks = (p.n_out + NT - 1) / NT;
  const int num_kb = (p.K + BK - 1) / BK;
  const uint32_t rank = PAIR ? cluster_ctarank() : 0u;  // 0 = the CTA that issues the MMAs
  const bool mma_cta = rank == 0;
  const int cta_unit = PAIR ? static_cast<int>(blockIdx.x >> 1) : static_cast<int>(blockIdx.x);
  const int units = PAIR ? static_cast<int>(gridDim.x >> 1) : static_cast<int>(gridDim.x);
  pdl_wait();  // offsets, the A rows and the tile counter come from the previous kernels
  pdl_trigger();

  if (threadIdx.x == 0) {
    int acc = 0;
    for (int e = 0; e <= p.E; ++e) s_seg[e] = p.offsets[e];
    for (int e = 0; e < p.E; ++e) {
      s_mstart[e] = acc;
      const int m = s_seg[e + 1] - s_seg[e];
      acc += (m + S::kTileRows - 1) / S::kTileRows;
    }
    s_mstart[p.E] = acc;
  }
  __syncthreads();
  const int m_total = s_mstart[p.E];
  const int total_tiles = m_total * n_blocks;
  const int group = min(max(p.n_group, 1), n_blocks);
  const int group_tiles = m_total * group;
  // Wide tiles of a last round that would keep at most half of the pairs busy are split
  // into two half tiles (one N=256 MMA each, NT/2 output columns), so that the round takes
  // half a tile's time: ids [0, first_half) are whole tiles in the order below, id
  // first_half + 2j + h is half h of tile first_half + j.
  int split = 0;
  if (WIDE) {
    if (p.halves == 2) {
      split = total_tiles;
    } else if (p.halves == 1) {
      const int r = total_tiles % units;
      if (2 * r <= units) split = r;
    }
  }
  const int first_half = total_tiles - split;
  const int work = total_tiles + split;  // tile ids handed out
  // Single CTAs: only ceil(work / rounds) of them take tiles, rounds = ceil(work / units), so
  // that every active CTA gets `rounds` tiles or one fewer and no last round runs on a few
  // CTAs while the rest wait. Streaming (HBM-bound) tiles then share the bandwidth evenly to
  // the end; compute-bound tiles take the same number of rounds either way.
  const int rounds = (work + units - 1) / units;
  const int active = PAIR ? units : (rounds > 0 ? (work + rounds - 1) / rounds : 0);
  // CTAs (pairs) beyond the active ones take no tile id; they only count themselves
  // finished. Uniform over the block and over the pair.
  if (cta_unit >= active || cta_unit >= work) {
    if (threadIdx.x == 0 && mma_cta) sched_finish(p.sched, units);
    return;
  }

  if (threadIdx.x == 0) {
    for (int s = 0; s < S::kStages; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], 1);
    }
    for (int a = 0; a < 2; ++a) {
      mbar_init(&tfull[a], 1);
      mbar_init(&tempty[a], (PAIR ? 2 : 1) * kEpiWarps);  // per epilogue warp (of both CTAs)
    }
    for (int r = 0; r < kRing; ++r) {
      mbar_init(&ring_full[r], 1);
      // consumers of a tile id: the MMA issuer and the epilogue warps, plus (pairs) the
      // second CTA's producer and its epilogue warps
      mbar_init(&ring_empty[r], PAIR ? 2 * (1 + kEpiWarps) : 1 + kEpiWarps);
    }
    mbar_init(drain, 1);
    fence_barrier_init();
    prefetch_tensormap(&tmA);
    prefetch_tensormap(&tmB0);
    if (DUAL) prefetch_tensormap(&tmB1);
  }
  if (warp == 1) {
    if (PAIR) {
      tmem_alloc_pair(s_tmem, kTmemCols);
      tmem_relinquish_pair();
    } else {
      tmem_alloc(s_tmem, kTmemCols);
      tmem_relinquish();
    }
  }
  tc_fence_before_sync();
  __syncwarp();
  if (PAIR) cluster_sync_all();  // barriers and TMEM of both CTAs ready before any remote use
  else __syncthreads();
  tc_fence_after_sync();
  const uint32_t tmem_base = *s_tmem;

  // tile -> (expert, row block, column block). Group c holds g column blocks (g = group but
  // for a shorter last group); inside it expert e owns g * m_tiles(e) consecutive tiles.
  auto decode = [&](int tile, int& e, int& m_blk, int& n_blk) {
    const int c = tile / group_tiles;
    const int g = min(group, n_blocks - c * group);
    int local = tile - c * group_tiles;
    e = 0;
    while (e < p.E - 1 && local >= s_mstart[e + 1] * g) ++e;
    local -= s_mstart[e] * g;
    const int m_tiles = s_mstart[e + 1] - s_mstart[e];
    const int n_in = local / m_tiles;
    m_blk = local - n_in * m_tiles;
    n_blk = c * group + n_in;
  };
  // Tile id -> its tile and the first output column; *mmas = N=256 MMAs per k-step.
  auto decode_id = [&](int id, int& e, int& m_blk, int& n0, int& mmas) {
    int base = id, h = -1;
    if (WIDE && id >= first_half) {
      base = first_half + ((id - first_half) >> 1);
      h = (id - first_half) & 1;
    }
    int n_blk;
    decode(base, e, m_blk, n_blk);
    n0 = n_blk * NT + (h > 0 ? NT / 2 : 0);
    mmas = h >= 0 ? 1 : S::kMmas;
  };

  // Next tile id from the ring (consumers). The second CTA of a pair receives the ids from
  // the first CTA (remote store + release.cluster arrival), so it waits with cluster scope
  // and returns its slot with a remote arrival.
  int r_slot = 0;
  uint32_t r_phase = 0;
  auto ring_take = [&](int& t) -> bool {
    const bool ok = (PAIR && !mma_cta)
                        ? mbar_wait_cluster(&ring_full[r_slot], r_phase, p.timeout_ns)
                        : mbar_wait(&ring_full[r_slot], r_phase, p.timeout_ns);
    if (ok) t = s_ring[r_slot];
    return ok;
  };
  auto ring_release = [&]() {
    if (PAIR && !mma_cta) mbar_arrive_cluster(mapa_shared(smem_u32(&ring_empty[r_slot]), 0));
    else mbar_arrive(&ring_empty[r_slot]);
  };
  auto ring_advance = [&]() {
    if (++r_slot == kRing) {
      r_slot = 0;
      r_phase ^= 1u;
    }
  };

  if (warp == 0) {
    if (lane == 0) {  // ---------------------------------------------------- TMA producer
      int stage = 0;
      uint32_t phase = 0;
      bool ok = true;
      const uint64_t pol_a = l2_policy(p.l2_a);
      const uint64_t pol_b = l2_policy(p.l2_b);
      // The first CTA takes tile ids from the counter and publishes them; the
      // second CTA of a pair takes them from the ring.
      int next = !mma_cta ? 0 : (p.static_order ? cta_unit : atomicAdd(&p.sched[0], 1));
      bool first_tile = true;
      while (ok) {
        int tile = next;
        if (mma_cta) {
          // Pairs: the second CTA returns slots with release.cluster arrivals; acquire at
          // cluster scope before storing the next id into its shared memory.
          const bool free_slot =
              PAIR ? mbar_wait_cluster(&ring_empty[r_slot], r_phase ^ 1u, p.timeout_ns)
                   : mbar_wait(&ring_empty[r_slot], r_phase ^ 1u, p.timeout_ns);
          if (!free_slot) {
            record_error(p.err, MOE_DEVERR_WAIT_TIMEOUT);
            break;
          }
          s_ring[r_slot] = tile;
          if (PAIR) st_dsmem_u32(mapa_shared(smem_u32(const_cast<int*>(&s_ring[r_slot])), 1),
                                 static_cast<uint32_t>(tile));
          mbar_arrive(&ring_full[r_slot]);
          if (PAIR) mbar_arrive_cluster(mapa_shared(smem_u32(&ring_full[r_slot]), 1));
          ring_advance();
          if (tile >= work) break;
          if (p.static_order) next = tile + active;
        } else {
          if (!ring_take(tile)) {
            record_error(p.err, MOE_DEVERR_WAIT_TIMEOUT);
            break;
          }
          ring_release();
          ring_advance();
          if (tile >= work) break;
        }
        int e, m_blk, n0, mmas;
        decode_id(tile, e, m_blk, n0, mmas);
        const int row0 = s_seg[e] + m_blk * S::kTileRows + static_cast<int>(rank) * kRows;
        // The next tile id is taken when this tile's loads start (its latency hides behind
        // them), except during a CTA's first tile: then it is taken a few k-blocks before the
        // tile's last loads. Taking it at the start of the first tile let the CTAs that
        // launch first hold two tiles each, so with fewer tiles than CTAs the late CTAs found
        // the counter exhausted and the grid ran the tiles in two rounds (the decode
        // down-projection at 210 us instead of 140 us).
        const int grab_kb = !first_tile ? 0 : (num_kb > kGrabAhead ? num_kb - kGrabAhead : 0);
        first_tile = false;
        for (int kb = 0; kb < num_kb; ++kb) {
          if (mma_cta && !p.static_order && kb == grab_kb) next = atomicAdd(&p.sched[0], 1);
          if (!mbar_wait(&empty[stage], phase ^ 1u, p.timeout_ns)) {
            record_error(p.err, MOE_DEVERR_WAIT_TIMEOUT);
            ok = false;
            break;
          }
          uint8_t* a_dst = sA + stage * kABytes;
          uint8_t* b_dst = sB + stage * S::kBBytes;
          const int k0 = kb * BK;
          if (PAIR) {
            // Both CTAs' bytes are counted on the MMA CTA's barrier.
            const uint32_t bar = mapa_shared(smem_u32(&full[stage]), 0);
            if (mma_cta)
              mbar_arrive_expect_tx(&full[stage],
                                    mmas == S::kMmas ? S::kTxBytes
                                                     : 2 * (kABytes + 2 * mmas * kBoxBytes));
            tma_load_2d_pair_hint(a_dst, &tmA, bar, k0, row0, pol_a);
            // MMA h of the k-step reads boxes 2h, 2h+1 of each CTA.
            for (int h = 0; h < mmas; ++h) {
              uint8_t* bh = b_dst + 2 * h * kBoxBytes;
              if (DUAL) {  // CTA 0 holds W1 columns [n0 + 128h, +128), CTA 1 the same of W2
                const CUtensorMap* m = rank == 0 ? &tmB0 : &tmB1;
                tma_load_3d_pair_hint(bh, m, bar, n0 + 128 * h, k0, e, pol_b);
                tma_load_3d_pair_hint(bh + kBoxBytes, m, bar, n0 + 128 * h + 64, k0, e, pol_b);
              } else {     // CTA r holds columns [n0 + 256h + 128r, +128)
                const int nc = n0 + 256 * h + static_cast<int>(rank) * 128;
                tma_load_3d_pair_hint(bh, &tmB0, bar, nc, k0, e, pol_b);
                tma_load_3d_pair_hint(bh + kBoxBytes, &tmB0, bar, nc + 64, k0, e, pol_b);
              }
            }
          } else {
            mbar_arrive_expect_tx(&full[stage], S::kTxBytes);
            tma_load_2d_hint(a_dst, &tmA, &full[stage], k0, row0, pol_a);
            if (DUAL) {
              tma_load_3d_hint(b_dst, &tmB0, &full[stage], n0, k0, e, pol_b);
              tma_load_3d_hint(b_dst + kBoxBytes, &tmB0, &full[stage], n0 + 64, k0, e, pol_b);
              tma_load_3d_hint(b_dst + 2 * kBoxBytes, &tmB1, &full[stage], n0, k0, e, pol_b);
              tma_load_3d_hint(b_dst + 3 * kBoxBytes, &tmB1, &full[stage], n0 + 64, k0, e, pol_b);
            } else {
#pragma unroll
              for (int j = 0; j < 4; ++j)
                tma_load_3d_hint(b_dst + j * kBoxBytes, &tmB0, &full[stage], n0 + 64 * j, k0, e,
                                 pol_b);
            }
          }
          if (++stage == S::kStages) {
            stage = 0;
            phase ^= 1u;
          }
        }
      }
    }
  } else if (warp == 1) {
    if (lane == 0 && mma_cta) {  // ------------------------------------------- MMA issuer
      int stage = 0;
      uint32_t phase = 0;
      bool ok = true;
      for (int it = 0; ok; ++it) {
        int tile = 0;
        if (!ring_take(tile)) {
          record_error(p.err, MOE_DEVERR_WAIT_TIMEOUT);
          break;
        }
        ring_release();
        ring_advance();
        if (tile >= work) break;
        const int mmas = WIDE && tile >= first_half ? 1 : S::kMmas;  // a half tile: one MMA
        const int acc = it % S::kAccBufs;
        const uint32_t acc_phase = static_cast<uint32_t>(it / S::kAccBufs) & 1u;
        // Wide tiles: tempty[0] / tempty[1] free the lower / upper 256 accumulator columns
        // (both are waited for on every tile, half tiles included, so that no epilogue warp
        // can arrive for a tile before every warp has arrived for the one before).
        if (!mbar_wait(&tempty[acc], acc_phase ^ 1u, p.timeout_ns)) {
          record_error(p.err, MOE_DEVERR_WAIT_TIMEOUT);
          ok = false;
          break;
        }
        tc_fence_after_sync();
        const uint32_t d_tmem = tmem_base + static_cast<uint32_t>(acc * kAccCols);
        uint32_t idesc = S::kIdesc;
        if (!PAIR) {
          int e, m_blk, n_blk;
          decode(tile, e, m_blk, n_blk);
          if (s_seg[e + 1] - s_seg[e] - m_blk * kRows <= 64) idesc = S::kIdesc64;
        }
        // The MMAs of k-block kb (MMA h writes accumulator columns [256h, 256h + 256)).
        auto issue = [&](int kb, int st, int h_lo, int h_hi) {
          const uint32_t a_addr = smem_u32(sA + st * kABytes);
          const uint32_t b_addr = smem_u32(sB + st * S::kBBytes);
#pragma unroll
          for (int kk = 0; kk < BK / UK; ++kk) {
            // A: K-major SW128, advance 16 elements = 32 bytes inside the swizzle row.
            const uint64_t ad = smem_desc_sw128(a_addr + kk * 32, 16, 1024);
            // B: MN-major SW128, 64-column blocks kBoxBytes apart (LBO), 8-row k groups
            // 1024 bytes apart (SBO); advance 16 k-rows = 2048 bytes. MMA h (wide tiles)
            // reads boxes 2h, 2h+1.
            for (int h = h_lo; h < h_hi; ++h) {
              const uint64_t bd =
                  smem_desc_sw128(b_addr + 2 * h * kBoxBytes + kk * 2048, kBoxBytes, 1024);
              const uint32_t dh = d_tmem + static_cast<uint32_t>(256 * h);
              if (PAIR) umma_bf16_ss_pair(dh, ad, bd, idesc, (kb | kk) != 0 ? 1u : 0u);
              else umma_bf16_ss(dh, ad, bd, idesc, (kb | kk) != 0 ? 1u : 0u);
            }
          }
        };
        auto free_stage = [&](int st) {  // once these MMAs have read it (both CTAs)
          if (PAIR) umma_commit_pair(&empty[st], 0x3);
          else umma_commit(&empty[st]);
        };
        int kb = 0;
        if (WIDE) {
          // The epilogue hands back the lower half of the accumulator before the upper one.
          // Meanwhile the lower-half MMAs of the first k-blocks already in the ring run; their
          // stages are freed once the upper-half MMAs have read them too.
          const int pre = min(num_kb, S::kStages);
          int st = stage;
          uint32_t ph = phase;
          for (int j = 0; j < pre; ++j) {
            if (!mbar_wait(&full[st], ph, p.timeout_ns)) {
              record_error(p.err, MOE_DEVERR_WAIT_TIMEOUT);
              ok = false;
              break;
            }
            tc_fence_after_sync();
            issue(j, st, 0, 1);
            if (++st == S::kStages) {
              st = 0;
              ph ^= 1u;
            }
          }
          if (ok && !mbar_wait(&tempty[1], acc_phase ^ 1u, p.timeout_ns)) {
            record_error(p.err, MOE_DEVERR_WAIT_TIMEOUT);
            ok = false;
          }
          if (!ok) break;
          tc_fence_after_sync();
          for (; kb < pre; ++kb) {
            issue(kb, stage, 1, mmas);
            free_stage(stage);
            if (++stage == S::kStages) {
              stage = 0;
              phase ^= 1u;
            }
          }
        }
        for (; kb < num_kb; ++kb) {
          if (!mbar_wait(&full[stage], phase, p.timeout_ns)) {
            record_error(p.err, MOE_DEVERR_WAIT_TIMEOUT);
            ok = false;
            break;
          }
          tc_fence_after_sync();
          issue(kb, stage, 0, mmas);
          free_stage(stage);
          if (++stage == S::kStages) {
            stage = 0;
            phase ^= 1u;
          }
        }
        if (ok) {  // accumulator complete
          if (PAIR) umma_commit_pair(&tfull[acc], 0x3);
          else umma_commit(&tfull[acc]);
        }
      }
      // Every MMA issued by this thread has completed once `drain` flips.
      if (PAIR) umma_commit_pair(drain, 0x1);
      else umma_commit(drain);
      if (!mbar_wait(drain, 0, p.timeout_ns)) record_error(p.err, MOE_DEVERR_WAIT_TIMEOUT);
    }
  } else {  // ------------------------------------------------------------------ epilogue
    const int q = warp & 3;  // this warp may access TMEM lanes [32q, 32q+32)
    // The two warps of a lane quarter take alternate 32-column chunks of the accumulator.
    const int c_first = (warp - 2) / 4;
    const uint32_t tempty_mma0 = PAIR ? mapa_shared(smem_u32(&tempty[0]), 0) : 0u;
    for (int it = 0;; ++it) {
      int tile = 0;
      const bool got = ring_take(tile);
      if (__any_sync(0xffffffffu, !got)) {
        if (lane == 0) record_error(p.err, MOE_DEVERR_WAIT_TIMEOUT);
        break;
      }
      __syncwarp();
      if (lane == 0) ring_release();
      ring_advance();
      if (tile >= work) break;
      const int acc = it % S::kAccBufs;
      const uint32_t acc_phase = static_cast<uint32_t>(it / S::kAccBufs) & 1u;
      // The accumulator is ready only after the tile's whole main loop: suspend rather than
      // spin while the MMAs run (eight warps polling would take issue slots and power).
      const bool ok = mbar_wait_suspend(&tfull[acc], acc_phase, p.timeout_ns);
      if (__any_sync(0xffffffffu, !ok)) {
        if (lane == 0) record_error(p.err, MOE_DEVERR_WAIT_TIMEOUT);
        break;
      }
      __syncwarp();
      tc_fence_after_sync();
      int e, m_blk, n0, mmas;
      decode_id(tile, e, m_blk, n0, mmas);
      const int first_row = m_blk * S::kTileRows + static_cast<int>(rank) * kRows;
      const int rows = min(kRows, s_seg[e + 1] - s_seg[e] - first_row);
      // Row held by TMEM lane 32q + l (M = 64 tiles use lanes 0-15 of each quarter).
      const bool half = !PAIR && rows <= 64;
      auto tile_row = [&](int l) { return half ? (l < 16 ? 16 * q + l : kRows) : q * 32 + l; };
      const int64_t row0 = static_cast<int64_t>(s_seg[e]) + first_row;
      const uint32_t t_row =
          tmem_base + (static_cast<uint32_t>(q * 32) << 16) + static_cast<uint32_t>(acc * kAccCols);
      // The accumulator is handed back to the MMA issuer as soon as this warp's last
      // tcgen05.ld from it has completed; the last chunk's activation and stores follow. Wide
      // tiles hand back their lower 256 columns (barrier tempty[0]) once the warp's loads from
      // them are done, and the upper ones (tempty[1]) after its last load.
      auto release_acc = [&](int part) {
        tc_fence_before_sync();
        __syncwarp();
        if (lane == 0) {
          if (PAIR) mbar_arrive_cluster(tempty_mma0 + static_cast<uint32_t>((acc + part) * 8));
          else mbar_arrive(&tempty[acc + part]);
        }
      };
      // After the warp's last load: the whole accumulator (wide tiles: the upper half, and the
      // lower half too for a half tile, which has not released it yet).
      auto release_all = [&]() {
        if (WIDE && mmas == 1) release_acc(0);
        release_acc(WIDE ? 1 : 0);
      };
      // Output columns [n0 + 32c, +32) of the warp's 32 rows: each lane holds its row's 64 bytes.
      // They pass through the warp's 2 KB of shared memory so that each global store
      // instruction writes 8 whole 64-byte row segments (4 lanes per row) instead of 32
      // scattered 16-byte pieces. Segment v of row l sits in slot v ^ ((l >> 1) & 3), which
      // keeps both the row-wise writes and the segment-wise reads free of bank conflicts.
      uint8_t* stage = sT + (warp - 2) * kStoreStage;
      auto store_chunk = [&](const uint32_t (&w)[16], int c) {
        uint4* mine = reinterpret_cast<uint4*>(stage + lane * 64);
#pragma unroll
        for (int v = 0; v < 4; ++v)
          mine[v ^ ((lane >> 1) & 3)] = make_uint4(w[4 * v], w[4 * v + 1], w[4 * v + 2], w[4 * v + 3]);
        __syncwarp();
        const int sg = lane & 3;
        const int col = n0 + c * 32 + sg * 8;
#pragma unroll
        for (int i = 0; i < 4; ++i) {
          const int l = 8 * i + (lane >> 2);
          const uint4 val = reinterpret_cast<const uint4*>(stage + l * 64)[sg ^ ((l >> 1) & 3)];
          const int r = tile_row(l);
          if (r < rows && col < p.n_out)
            *reinterpret_cast<uint4*>(p.out + (row0 + r) * p.n_out + col) = val;
        }
        __syncwarp();  // the next chunk overwrites the staging rows
      };
      // The TMEM loads are software-pipelined: the next piece's tcgen05.ld is issued before
      // this piece's math, so its latency hides behind the math (tcgen05.wait::ld waits for
      // every load the thread has in flight, hence the two statically indexed buffers).
      if (DUAL) {
        // Output columns [32c, 32c + 32) of the tile: x W1 in accumulator columns
        // 256h + 32(c mod 4) and x W2 128 further, h = c / 4 (wide tiles have two halves);
        // each chunk is read as two 16-column pieces.
        const int n_c = (4 * mmas - c_first + 1) / 2;  // this warp's chunks
        auto piece_col = [&](int cc, int half) {
          const int c = c_first + 2 * cc;
          return static_cast<uint32_t>(256 * (c >> 2) + 32 * (c & 3) + 16 * half);
        };
        auto act_pack = [&](const uint32_t (&ra)[16], const uint32_t (&rb)[16], uint32_t* w) {
#pragma unroll
          for (int i = 0; i < 8; ++i) {
            const float h0 = activation<ACT>(__uint_as_float(ra[2 * i])) * __uint_as_float(rb[2 * i]);
            const float h1 =
                activation<ACT>(__uint_as_float(ra[2 * i + 1])) * __uint_as_float(rb[2 * i + 1]);
            w[i] = pack_bf16x2(h0, h1);
          }
        };
        uint32_t ra0[16], rb0[16], ra1[16], rb1[16];
        tmem_ld_16cols(t_row + piece_col(0, 0), ra0);        // x W1 (activated branch)
        tmem_ld_16cols(t_row + piece_col(0, 0) + 128, rb0);  // x W2 (linear branch)
#pragma unroll 1
        for (int cc = 0; cc < n_c; ++cc) {
          uint32_t w[16];
          tmem_ld_wait();
          tmem_ld_16cols(t_row + piece_col(cc, 1), ra1);
          tmem_ld_16cols(t_row + piece_col(cc, 1) + 128, rb1);
          act_pack(ra0, rb0, w);
          tmem_ld_wait();
          if (mmas == 2 && 2 * (cc + 1) == n_c) release_acc(0);  // the lower half is read
          if (cc + 1 < n_c) {
            tmem_ld_16cols(t_row + piece_col(cc + 1, 0), ra0);
            tmem_ld_16cols(t_row + piece_col(cc + 1, 0) + 128, rb0);
          } else {
            release_all();
          }
          act_pack(ra1, rb1, w + 8);
          store_chunk(w, c_first + 2 * cc);
        }
      } else {  // accumulator column j is output column n0 + j
        const int n_c = (8 * mmas - c_first + 1) / 2;  // this warp's chunks (even)
        auto pack = [&](const uint32_t (&ra)[32], uint32_t (&w)[16]) {
#pragma unroll
          for (int i = 0; i < 16; ++i)
            w[i] = pack_bf16x2(__uint_as_float(ra[2 * i]), __uint_as_float(ra[2 * i + 1]));
        };
        uint32_t ra0[32], ra1[32];
        tmem_ld_32cols(t_row + c_first * 32, ra0);
#pragma unroll 1
        for (int cc = 0; cc < n_c; cc += 2) {
          uint32_t w[16];
          tmem_ld_wait();
          tmem_ld_32cols(t_row + (c_first + 2 * (cc + 1)) * 32, ra1);
          pack(ra0, w);
          store_chunk(w, c_first + 2 * cc);
          tmem_ld_wait();
          if (mmas == 2 && 2 * (cc + 2) == n_c) release_acc(0);  // the lower half is read
          if (cc + 2 < n_c) tmem_ld_32cols(t_row + (c_first + 2 * (cc + 2)) * 32, ra0);
          else release_all();
          pack(ra1, w);
          store_chunk(w, c_first + 2 * (cc + 1));
        }
      }
    }
  }

  __syncwarp();  // role branches leave warps 0 and 1 divergent; the barrier below is .aligned
  if (PAIR) cluster_sync_all();  // no CTA of the pair leaves while the other may signal it
  else __syncthreads();
  if (warp == 1) {
    __syncwarp();
    tc_fence_after_sync();
    if (PAIR) tmem_dealloc_pair(tmem_base, kTmemCols);
    else tmem_dealloc(tmem_base, kTmemCols);
  }
  if (threadIdx.x == 0 && mma_cta) sched_finish(p.sched, units);
}

// ------------------------------------------------------------------ host side

using EncodeTiledFn = CUresult (*)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*,
                                   const cuuint64_t*, const cuuint64_t*, const cuuint32_t*,
                                   const cuuint32_t*, CUtensorMapInterleave, CUtensorMapSwizzle,
                                   CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn encode_fn() {
  static EncodeTiledFn fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* ptr = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &ptr, cudaEnableDefault, &q) ==
            cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<EncodeTiledFn>(ptr);
  });
  return fn;
}

// Rows x cols bf16 matrix (cols contiguous), box = 64 columns x box_rows rows, 128-B swizzle.
bool make_map_2d(CUtensorMap* m, const void* ptr, uint64_t cols, uint64_t rows, uint32_t box_rows) {
  const cuuint64_t dims[2] = {cols, rows};
  const cuuint64_t strides[1] = {cols * 2};
  const cuuint32_t box[2] = {64, box_rows};
  const cuuint32_t estr[2] = {1, 1};
  return encode_fn()(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(ptr), dims, strides,
                     box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                     CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                     CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// Stacked weights [E][K][N] (N contiguous), box = 64 columns x 64 k-rows x 1 expert.
bool make_map_3d(CUtensorMap* m, const void* ptr, uint64_t n, uint64_t k, uint64_t E) {
  const cuuint64_t dims[3] = {n, k, E};
  const cuuint64_t strides[2] = {n * 2, n * k * 2};
  const cuuint32_t box[3] = {64, 64, 1};
  const cuuint32_t estr[3] = {1, 1, 1};
  return encode_fn()(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(ptr), dims, strides,
                     box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                     CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                     CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// Clusters of two that fit on the device at once for this kernel (cached per kernel).
template <typename Kern>
int max_pair_clusters(Kern kern, int smem) {
  static int cached = 0;
  if (cached > 0) return cached;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(2 * num_sms());
  cfg.blockDim = dim3(kThreads);
  cfg.dynamicSmemBytes = smem;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = 2;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  int n = 0;
  if (cudaOccupancyMaxActiveClusters(&n, kern, &cfg) != cudaSuccess || n <= 0) {
    (void)cudaGetLastError();
    n = num_sms() / 2;
  }
  cached = n;
  return n;
}

template <bool DUAL, int ACT, bool PAIR, bool WIDE>
cudaError_t launch_gemm(const CUtensorMap& a, const CUtensorMap& b0, const CUtensorMap& b1,
                        const GemmParams& gp, int64_t tiles_upper, cudaStream_t stream) {
  using S = Shape<PAIR, WIDE>;
  auto kern = grouped_gemm_sm100<DUAL, ACT, PAIR, WIDE>;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, S::kSmemBytes);
  if (e != cudaSuccess) return e;
  if (!PAIR) {
    const int grid = static_cast<int>(std::max<int64_t>(1, std::min<int64_t>(num_sms(), tiles_upper)));
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(grid);
    cfg.blockDim = dim3(kThreads);
    cfg.dynamicSmemBytes = S::kSmemBytes;
    cfg.stream = stream;
    cudaLaunchAttribute attr[1];
    cfg.attrs = attr;
    cfg.numAttrs = pdl_attr(&attr[0]);
    e = cudaLaunchKernelEx(&cfg, kern, a, b0, b1, gp);
    return e != cudaSuccess ? e : cudaGetLastError();
  }
  const int clusters = static_cast<int>(
      std::max<int64_t>(1, std::min<int64_t>(max_pair_clusters(kern, S::kSmemBytes), tiles_upper)));
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(2 * clusters);
  cfg.blockDim = dim3(kThreads);
  cfg.dynamicSmemBytes = S::kSmemBytes;
  cfg.stream = stream;
  cudaLaunchAttribute attr[2];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = 2;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1 + pdl_attr(&attr[1]);
  e = cudaLaunchKernelEx(&cfg, kern, a, b0, b1, gp);
  return e != cudaSuccess ? e : cudaGetLastError();
}

// Tile shape: CTA pairs (256-row tiles) pay off when experts hold many rows; 128-row tiles
// waste less on small or skewed experts. Without capacity the routing of a large batch is
// close to balanced, so R/E >= 384 rows already fill pair tiles; under a capacity the per-expert
// counts are skewed below the cap, and pairs need 768. MOE_GEMM_TILE_ROWS=128|256 overrides.
bool use_pairs(const moe_problem& p) {
  if (const char* env = std::getenv("MOE_GEMM_TILE_ROWS")) {
    if (std::strcmp(env, "256") == 0) return true;
    if (std::strcmp(env, "128") == 0) return false;
  }
  const int64_t R = p.N * p.k;
  int64_t per_expert = R / p.E;
  if (p.capacity_factor > 0.0) {
    const int64_t C = static_cast<int64_t>(std::ceil(p.capacity_factor * static_cast<double>(p.N) *
                                                     static_cast<double>(p.k) / static_cast<double>(p.E)));
    per_expert = std::min(per_expert, C);
  }
  return per_expert >= (p.capacity_factor > 0.0 ? 768 : 384);
}

// Column blocks per tile group. Experts that hold many rows (CTA-pair tiles) keep the
// expert-by-expert order, which keeps an expert's A rows in L2 across its column blocks.
// Otherwise groups of kGroup blocks mix experts of all sizes among the resident CTAs.
// MOE_GEMM_NGROUP=<n> overrides (testing and tuning).
int column_group(bool pairs, int64_t n_blocks) {
  constexpr int kGroup = 8;
  if (const char* env = std::getenv("MOE_GEMM_NGROUP")) {
    const int g = std::atoi(env);
    if (g > 0) return static_cast<int>(std::min<int64_t>(g, n_blocks));
  }
  return static_cast<int>(pairs ? n_blocks : std::min<int64_t>(kGroup, n_blocks));
}

// Tile order: handed out in order by the workspace counter (default), or the static
// round-robin CTA u -> tiles u, u + units, ... (MOE_GEMM_SCHED=static; tuning and comparison).
int static_order() {
  const char* env = std::getenv("MOE_GEMM_SCHED");
  return env != nullptr && std::strcmp(env, "static") == 0 ? 1 : 0;
}

// Half tiles (wide tiles only): the tiles of a last round that would keep at most half of the
// pairs busy run as two half-width tiles each (default, 1); MOE_GEMM_HALVES=0 never splits,
// MOE_GEMM_HALVES=all splits every tile (testing).
int halves_mode() {
  if (const char* env = std::getenv("MOE_GEMM_HALVES")) {
    if (std::strcmp(env, "0") == 0) return 0;
    if (std::strcmp(env, "all") == 0) return 2;
  }
  return 1;
}

// L2 priorities of the GEMM operands: an expert's A rows are read again by every column block
// of that expert, its weights by the few row blocks running at the same time. Default: A rows
// evict_last, weights evict_normal. MOE_GEMM_L2=<a>,<b> (each -1, 0 or 1) overrides.
void l2_priorities(int* a, int* b) {
  *a = 1;
  *b = 0;
  if (const char* env = std::getenv("MOE_GEMM_L2")) {
    int x = 0, y = 0;
    if (std::sscanf(env, "%d,%d", &x, &y) == 2) {
      *a = std::max(-1, std::min(1, x));
      *b = std::max(-1, std::min(1, y));
    }
  }
}

// CTA-pair tiles twice as wide (two MMAs into one 512-column accumulator, not double-buffered):
// 25 % fewer bytes from L2 per FLOP against an epilogue that no longer overlaps the next
// tile's main loop. Measured faster for both projections on the mixtral and grok1 shapes.
// MOE_GEMM_WIDE=0|1 overrides (testing and tuning).
bool use_wide() {
  if (const char* env = std::getenv("MOE_GEMM_WIDE")) {
    if (std::strcmp(env, "1") == 0) return true;
    if (std::strcmp(env, "0") == 0) return false;
  }
  return true;
}

template <bool DUAL, int ACT>
cudaError_t launch_shape(const moe_problem& p, const CUtensorMap& a, const CUtensorMap& b0,
                         const CUtensorMap& b1, GemmParams gp, int n_tile,
                         cudaStream_t stream) {
  const int64_t R = p.N * p.k;
  const bool pairs = use_pairs(p);
  const bool wide = pairs && use_wide();
  if (wide) n_tile *= 2;
  const int64_t n_blocks = (gp.n_out + n_tile - 1) / n_tile;
  gp.n_group = column_group(pairs, n_blocks);
  gp.static_order = static_order();
  gp.halves = wide ? halves_mode() : 0;
  l2_priorities(&gp.l2_a, &gp.l2_b);
  if (pairs) {
    const int64_t tiles = ((R + 255) / 256 + p.E) * n_blocks;
    // half tiles: up to twice as many ids as tiles
    if (wide)
      return launch_gemm<DUAL, ACT, true, true>(a, b0, b1, gp, gp.halves ? 2 * tiles : tiles,
                                                stream);
    return launch_gemm<DUAL, ACT, true, false>(a, b0, b1, gp, tiles, stream);
  }
  const int64_t tiles = ((R + 127) / 128 + p.E) * n_blocks;
  return launch_gemm<DUAL, ACT, false, false>(a, b0, b1, gp, tiles, stream);
}

}  // namespace

bool make_tensor_map_2d_bf16(CUtensorMap* m, const void* ptr, uint64_t cols, uint64_t rows,
                             uint32_t box_cols, uint32_t box_rows) {
  if (encode_fn() == nullptr) return false;
  const cuuint64_t dims[2] = {cols, rows};
  const cuuint64_t strides[1] = {cols * 2};
  const cuuint32_t box[2] = {box_cols, box_rows};
  const cuuint32_t estr[2] = {1, 1};
  return encode_fn()(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(ptr), dims, strides,
                     box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                     CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                     CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

bool make_tensor_map_3d_u8(CUtensorMap* m, const void* ptr, uint64_t n, uint64_t k, uint64_t E,
                           uint32_t box_n, uint32_t box_k) {
  if (encode_fn() == nullptr) return false;
  const cuuint64_t dims[3] = {n, k, E};
  const cuuint64_t strides[2] = {n, n * k};
  const cuuint32_t box[3] = {box_n, box_k, 1};
  const cuuint32_t estr[3] = {1, 1, 1};
  return encode_fn()(m, CU_TENSOR_MAP_DATA_TYPE_UINT8, 3, const_cast<void*>(ptr), dims, strides,
                     box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                     CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                     CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

bool make_tensor_map_3d_u8_sw64(CUtensorMap* m, const void* ptr, uint64_t inner, uint64_t rows,
                                uint64_t E, uint32_t box_inner, uint32_t box_rows) {
  if (encode_fn() == nullptr) return false;
  const cuuint64_t dims[3] = {inner, rows, E};
  const cuuint64_t strides[2] = {inner, inner * rows};
  const cuuint32_t box[3] = {box_inner, box_rows, 1};
  const cuuint32_t estr[3] = {1, 1, 1};
  return encode_fn()(m, CU_TENSOR_MAP_DATA_TYPE_UINT8, 3, const_cast<void*>(ptr), dims, strides,
                     box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_64B,
                     CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                     CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

cudaError_t launch_ffn_up_sm100(const moe_problem& p, const void* X_perm, const int32_t* offsets,
                                const void* W1, const void* W2, void* H, int* err, int* sched,
                                uint64_t timeout_ns, cudaStream_t stream) {
  const int64_t R = p.N * p.k;
  if (R == 0) return cudaSuccess;
  if (encode_fn() == nullptr) return cudaErrorNotSupported;
  CUtensorMap tA, tW1, tW2;
  if (!make_map_2d(&tA, X_perm, p.D, R, kRows) || !make_map_3d(&tW1, W1, p.F, p.D, p.E) ||
      !make_map_3d(&tW2, W2, p.F, p.D, p.E))
    return cudaErrorInvalidValue;
  GemmParams g;
  g.offsets = offsets;
  g.out = static_cast<__nv_bfloat16*>(H);
  g.E = p.E;
  g.K = static_cast<int>(p.D);
  g.n_out = static_cast<int>(p.F);
  g.err = err;
  g.sched = sched;
  g.timeout_ns = timeout_ns;
  switch (p.activation) {
    case MOE_ACT_SILU:
      return launch_shape<true, MOE_ACT_SILU>(p, tA, tW1, tW2, g, 128, stream);
    case MOE_ACT_GELU_ERF:
      return launch_shape<true, MOE_ACT_GELU_ERF>(p, tA, tW1, tW2, g, 128, stream);
    default:
      return launch_shape<true, MOE_ACT_GELU_TANH>(p, tA, tW1, tW2, g, 128, stream);
  }
}

cudaError_t launch_ffn_down_sm100(const moe_problem& p, const void* H, const int32_t* offsets,
                                  const void* W3, void* Y, int* err, int* sched,
                                  uint64_t timeout_ns, cudaStream_t stream) {
  const int64_t R = p.N * p.k;
  if (R == 0) return cudaSuccess;
  if (encode_fn() == nullptr) return cudaErrorNotSupported;
  CUtensorMap tA, tW3;
  if (!make_map_2d(&tA, H, p.F, R, kRows) || !make_map_3d(&tW3, W3, p.D, p.F, p.E))
    return cudaErrorInvalidValue;
  GemmParams g;
  g.offsets = offsets;
  g.out = static_cast<__nv_bfloat16*>(Y);
  g.E = p.E;
  g.K = static_cast<int>(p.F);
  g.n_out = static_cast<int>(p.D);
  g.err = err;
  g.sched = sched;
  g.timeout_ns = timeout_ns;
  return launch_shape<false, MOE_ACT_SILU>(p, tA, tW3, tW3, g, 256, stream);
}

}  // namespace moe

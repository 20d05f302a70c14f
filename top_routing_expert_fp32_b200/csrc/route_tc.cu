// Router for bf16 activations on the tensor cores: logits z = X W_r (+ bias) with fp32-level
// accuracy, then softmax, top-k and gates, all in one kernel.
//   Grok-1 book ch.5, 5.2 (router logits kept in fp32, softmax, TopK) and 5.2.3 (gates);
//   MoE formula-to-code walkthrough 1.1-1.2; LLMs-from-scratch ch.12, 12.1.
//
// Precision. The fp32 router weights are split into three bf16 terms, w = w0 + w1 + w2 with
// w0 = bf16(w), w1 = bf16(w - w0), w2 = bf16(w - w0 - w1) (the "bf16x3" decomposition of
// Henry, Tang and Heinecke, "Leveraging the bfloat16 Artificial Intelligence Datatype For
// Higher-Precision Computations", ARITH 2019). The three terms carry 24 significant bits, as
// many as the fp32 value; what is left over is below 2^-24 |w|. X is bf16 already, so every
// product x * w_i is exact in fp32, and one bf16 MMA with fp32 accumulation over the
// concatenated [w0 | w1 | w2] columns gives the three partial dot products; they are added
// smallest first, z = (z2 + z1) + z0.
//
// Kernel (one launch per call; two with more than 16 experts): route_tc_kernel, clusters of S CTAs (S = 1, 2, 4 or 8),
// persistent over 128-token tiles; CTA r of a cluster accumulates the r-th slice of D
// (split-K), so that a batch of few tiles still spreads over the SMs. Warp 0 issues the TMA
// loads of X and a bulk copy of the k-block's fp32 W_r slice (64 x E, contiguous) into the
// stage; warps 6-9 turn that slice into the B operand (the three bf16 terms, in the
// 128-byte-swizzled K-major layout the MMA reads; row i * Ep + e holds term i of expert e,
// padding rows are zero) from shared memory, so no global latency sits between the
// k-blocks; with more than 16 experts a small kernel writes the three terms once per call
// instead ([3 Ep, rounded up to 16][D] bf16 in the workspace) and warp 0 loads each k-block's
// B by TMA beside X, so the loop no longer waits on the conversion; warp 1 issues the
// tcgen05.mma, warps 2-5 are the epilogue: CTA r owns tokens [r*128/S, (r+1)*128/S) of the
// tile; every epilogue thread stores its row's partial logits into the owner's shared memory
// (a slot per source CTA, remote stores) and arrives there (release.cluster), and the owner
// adds the S slots of its rows in slice order from its own shared memory, adds the bias and
// takes the routing decision. No global round trip, no remote loads, no atomics; the result
// does not depend on timing.
// Every barrier wait is bounded in time; on a timeout the CTA records MOE_DEVERR_WAIT_TIMEOUT,
// unwinds, drains its MMAs and frees its tensor memory.
#include <algorithm>
#include <cstdlib>

#include "common.cuh"
#include "internal.h"
#include "select.cuh"

namespace moe {
namespace {

constexpr int kRows = 128;        // tokens per tile = accumulator lanes
constexpr int BK = 64;            // k-block: one 128-byte swizzle row of bf16
constexpr int UK = 16;            // K of one tcgen05.mma kind::f16
constexpr int kThreads = 320;
constexpr int kEpiThreads = 128;   // warps 2-5
constexpr int kConvThreads = 128;  // warps 6-9: the B operand from the staged W_r slice
constexpr int kConvWarps = kConvThreads / 32;
constexpr int kABytes = kRows * BK * 2;  // 16 KB
constexpr int kMaxStages = 8;
constexpr int kMaxCluster = 8;
constexpr int kAccStride = 256;   // TMEM columns between the two accumulators
constexpr int kTmemCols = 512;
constexpr int kSmemLimit = 227 * 1024;
constexpr int kUnitTarget = 148;  // CTAs wanted per launch (one per SM of a B200)
constexpr int kMaxEc = 64;

struct TcArgs {
  const float* W_r;        // [D][E] fp32
  const float* bias;       // [E] or nullptr
  float* logits_out;       // [N][E] or nullptr
  int32_t* idx;            // [N][k]
  float* gate;             // [N][k]
  float* colsum_partial;   // [gridDim.x][E] or nullptr
  const float* noise;      // [N][E] (mode != TOPK) or nullptr
  float* zl_partial;       // [gridDim.x] sums of (log Z)^2, or nullptr
  int mode;                // MOE_ROUTE_*
  int64_t N;
  int64_t tiles;
  int D, E, k, renorm;
  int Ep;                  // E rounded up to 8 (TMEM load granularity)
  int NB;                  // MMA N: 3 * Ep rounded up to 16
  int zstride;             // floats per row of the partial-logit buffer (Ep + 4)
  int num_kb, S, num_clusters, stages;
  int prepared;            // 1: B comes by TMA from the operand written by route_operand_kernel
  uint32_t stage_bytes, b_off, w_off, zbuf_off, sz_off, bar_off;
  int* err;
  uint64_t timeout_ns;
};

// Three bf16 terms of w (w = t0 + t1 + t2 to 24 significant bits): t0 = bf16(w), and the
// remainders w - t0 and (w - t0) - t1 are exact in fp32.
__device__ __forceinline__ void split3(float w, float& t0, float& t1, float& t2) {
  t0 = __bfloat162float(__float2bfloat16_rn(w));
  const float r1 = w - t0;
  t1 = __bfloat162float(__float2bfloat16_rn(r1));
  t2 = r1 - t1;  // rounded to bf16 when packed
}

// The router's B operand for all of D, once per call: row n = i Ep + e holds term i of expert
// e's column of W_r (k contiguous, the K-major rows a 128-byte-swizzled TMA box of 64 k
// delivers to shared memory as the MMA reads them); rows e >= E of each term and rows past
// 3 Ep are zero. One thread per element, consecutive threads along k.
__global__ void route_operand_kernel(const float* __restrict__ W_r, int D, int E, int Ep, int NB,
                                     __nv_bfloat16* __restrict__ out) {
  pdl_wait();  // W_r and the workspace belong to the previous kernels until here
  pdl_trigger();
  const int64_t total = static_cast<int64_t>(NB) * D;
  for (int64_t i = blockIdx.x * static_cast<int64_t>(blockDim.x) + threadIdx.x; i < total;
       i += static_cast<int64_t>(gridDim.x) * blockDim.x) {
    const int n = static_cast<int>(i / D);
    const int d = static_cast<int>(i - static_cast<int64_t>(n) * D);
    const int term = n / Ep, e = n - term * Ep;
    float v = 0.f;
    if (term < 3 && e < E) {
      float t0, t1, t2;
      split3(__ldg(W_r + static_cast<int64_t>(d) * E + e), t0, t1, t2);
      v = term == 0 ? t0 : (term == 1 ? t1 : t2);
    }
    out[i] = __float2bfloat16_rn(v);
  }
}

// EB: the experts the epilogue holds in registers per token (8, 16, 32 or 64; >= E).
template <int EB>
__global__ void __launch_bounds__(kThreads, 1)
    route_tc_kernel(const __grid_constant__ CUtensorMap tmX,
                    const __grid_constant__ CUtensorMap tmB, const TcArgs a) {
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  const uint32_t raw_addr = smem_u32(smem_raw);
  uint8_t* smem = smem_raw + ((1024u - (raw_addr & 1023u)) & 1023u);
  float* zbuf = reinterpret_cast<float*>(smem + a.zbuf_off);   // [128][zstride] own partials
  float* s_z = reinterpret_cast<float*>(smem + a.sz_off);      // [128/S][E+1] summed logits
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + a.bar_off);
  uint64_t* empty = full + kMaxStages;
  uint64_t* tfull = empty + kMaxStages;
  uint64_t* tempty = tfull + 2;
  uint64_t* zready = tempty + 2;  // the S partials of this CTA's rows have been stored here
  uint64_t* zfree = zready + 1;   // the owners have read the partials this CTA stored
  uint64_t* drain = zfree + 1;
  uint64_t* wfull = drain + 1;    // [kMaxStages] the k-block's fp32 W_r slice has landed
  uint32_t* s_tmem = reinterpret_cast<uint32_t*>(wfull + kMaxStages);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const int S = a.S;
  const uint32_t rank = cluster_ctarank();
  const int64_t first_tile = blockIdx.x / S;  // the cluster index; same for every CTA of it
  // k-blocks [kb0, kb1) of this CTA: an even share, at least one since S <= num_kb.
  const int kb0 = static_cast<int>((static_cast<int64_t>(rank) * a.num_kb) / S);
  const int kb1 = static_cast<int>((static_cast<int64_t>(rank + 1) * a.num_kb) / S);
  const bool has_k = kb1 > kb0;

  if (threadIdx.x == 0) {
    for (int s = 0; s < a.stages; ++s) {
      // the X copy (with its bytes) and the B writers, or the X and B copies
      mbar_init(&full[s], a.prepared ? 1 : 1 + kConvWarps);
      mbar_init(&empty[s], 1);
      mbar_init(&wfull[s], 1);
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(&tfull[b], 1);
      mbar_init(&tempty[b], 4);  // one arrival per epilogue warp
    }
    // zready: one arrival per pushed row (T owned rows x S source CTAs = 128); zfree: one per
    // owned row read, from the owner threads of the S CTAs (S x T = 128).
    mbar_init(zready, kRows);
    mbar_init(zfree, kRows);
    mbar_init(drain, 1);
    fence_barrier_init();
    prefetch_tensormap(&tmX);
    if (a.prepared) prefetch_tensormap(&tmB);
  }
  if (warp == 1) {
    tmem_alloc(s_tmem, kTmemCols);
    tmem_relinquish();
  }
  tc_fence_before_sync();
  __syncwarp();
  cluster_sync_all();  // every CTA's barriers exist before any remote arrival
  tc_fence_after_sync();
  const uint32_t tmem_base = *s_tmem;
  // X box, plus the B box (NB rows of 128 bytes) when B comes by TMA
  const uint32_t tx_bytes = static_cast<uint32_t>(kABytes + (a.prepared ? a.NB * 128 : 0));
  pdl_wait();  // X, W_r and the outputs belong to the previous kernels until here
  pdl_trigger();

  if (warp == 0) {
    if (lane == 0) {  // ------------------------------------------------------ TMA producer
      int stage = 0;
      uint32_t phase = 0;
      bool ok = true;
      for (int64_t tile = first_tile; ok && tile < a.tiles; tile += a.num_clusters) {
        for (int kb = kb0; kb < kb1; ++kb) {
          if (!mbar_wait(&empty[stage], phase ^ 1u, a.timeout_ns)) {
            record_error(a.err, MOE_DEVERR_WAIT_TIMEOUT);
            ok = false;
            break;
          }
          uint8_t* dst = smem + stage * a.stage_bytes;
          mbar_arrive_expect_tx(&full[stage], tx_bytes);
          tma_load_2d(dst, &tmX, &full[stage], kb * BK, static_cast<int>(tile * kRows));
          if (a.prepared) {
            tma_load_2d(dst + a.b_off, &tmB, &full[stage], kb * BK, 0);
          } else {
            // W_r rows [kb*64, kb*64 + rows) are one contiguous run of rows * E floats (a
            // multiple of 32 bytes, since D % 8 == 0); the B writers convert it.
            const int wrows = min(BK, a.D - kb * BK);
            const uint32_t wbytes = static_cast<uint32_t>(wrows * a.E * 4);
            mbar_arrive_expect_tx(&wfull[stage], wbytes);
            bulk_g2s(dst + a.w_off, a.W_r + static_cast<int64_t>(kb) * BK * a.E, wbytes,
                     &wfull[stage]);
          }
          if (++stage == a.stages) {
            stage = 0;
            phase ^= 1u;
          }
        }
      }
    }
  } else if (warp == 1) {
    if (lane == 0) {  // ---------------------------------------------------------- MMA issuer
      // kind::f16: D fp32 (bit 4), A bf16 (bits 7-9), B bf16 (bits 10-12), both K-major,
      // N >> 3 at bit 17, M >> 4 at bit 24.
      const uint32_t idesc = (1u << 4) | (1u << 7) | (1u << 10) |
                             (static_cast<uint32_t>(a.NB >> 3) << 17) |
                             (static_cast<uint32_t>(kRows >> 4) << 24);
      int stage = 0;
      uint32_t phase = 0;
      bool ok = true;
      int it = 0;
      for (int64_t tile = first_tile; ok && tile < a.tiles; tile += a.num_clusters, ++it) {
        const int acc = it & 1;
        const uint32_t acc_phase = static_cast<uint32_t>(it >> 1) & 1u;
        if (!mbar_wait(&tempty[acc], acc_phase ^ 1u, a.timeout_ns)) {
          record_error(a.err, MOE_DEVERR_WAIT_TIMEOUT);
          ok = false;
          break;
        }
        tc_fence_after_sync();
        const uint32_t d_tmem = tmem_base + static_cast<uint32_t>(acc * kAccStride);
        for (int kb = kb0; kb < kb1; ++kb) {
          if (!mbar_wait(&full[stage], phase, a.timeout_ns)) {
            record_error(a.err, MOE_DEVERR_WAIT_TIMEOUT);
            ok = false;
            break;
          }
          tc_fence_after_sync();
          const uint32_t a_addr = smem_u32(smem + stage * a.stage_bytes);
          const uint32_t b_addr = a_addr + a.b_off;
#pragma unroll
          for (int kk = 0; kk < BK / UK; ++kk) {
            // Both operands K-major SW128: advance 16 elements = 32 bytes in the swizzle row.
            const uint64_t ad = smem_desc_sw128(a_addr + kk * 32, 16, 1024);
            const uint64_t bd = smem_desc_sw128(b_addr + kk * 32, 16, 1024);
            umma_bf16_ss(d_tmem, ad, bd, idesc, (kb > kb0 || kk > 0) ? 1u : 0u);
          }
          umma_commit(&empty[stage]);  // frees the stage once these MMAs have read it
          if (++stage == a.stages) {
            stage = 0;
            phase ^= 1u;
          }
        }
        if (ok) umma_commit(&tfull[acc]);  // with no k-block this arrives at once
      }
      umma_commit(drain);  // flips once every MMA issued above has completed
      if (!mbar_wait(drain, 0, a.timeout_ns)) record_error(a.err, MOE_DEVERR_WAIT_TIMEOUT);
    }
  } else if (warp >= 6) {  // ------------------------------------------ B operand writers
    if (!a.prepared) {  // (with the prepared operand B comes by TMA: nothing to convert)
      // Item (c, e): 8 consecutive k of expert e's W_r column (a 16-byte chunk c of the
      // 128-byte K-major rows), split into its three bf16 terms, stored in rows e, Ep + e and
      // 2 Ep + e at the 128-byte-swizzled position of chunk c (chunk c ^ (row & 7)). Lanes take
      // consecutive e, so the fp32 reads are coalesced and each 8-lane phase of the 16-byte
      // stores hits 8 distinct chunks.
      const int ct = threadIdx.x - (kThreads - kConvThreads);
      const int E = a.E;
      const int items = 8 * E;
      // Padding rows (e in [E, Ep) of each term, and rows past 3 Ep) stay zero: written once.
      const int pad_rows = a.NB - 3 * E;
      for (int s = 0; s < a.stages; ++s) {
        uint8_t* b = smem + s * a.stage_bytes + a.b_off;
        for (int i = ct; i < pad_rows * 8; i += kConvThreads) {
          const int pr = i >> 3, c = i & 7;
          int n;  // the pr-th padding row
          if (pr < 3 * (a.Ep - E)) n = (pr / (a.Ep - E)) * a.Ep + E + pr % (a.Ep - E);
          else n = 3 * a.Ep + (pr - 3 * (a.Ep - E));
          *reinterpret_cast<uint4*>(b + n * 128 + ((c ^ (n & 7)) << 4)) = make_uint4(0u, 0u, 0u, 0u);
        }
      }
      int stage = 0;
      uint32_t phase = 0;
      bool ok = true;
      for (int64_t tile = first_tile; ok && tile < a.tiles; tile += a.num_clusters) {
        for (int kb = kb0; kb < kb1; ++kb) {
          // The slice lands after the producer has seen this stage free (empty), so waiting for
          // it also orders these stores after the MMAs that read the stage's previous B.
          if (!mbar_wait(&wfull[stage], phase, a.timeout_ns)) {
            if (lane == 0) record_error(a.err, MOE_DEVERR_WAIT_TIMEOUT);
            ok = false;
            break;
          }
          uint8_t* b = smem + stage * a.stage_bytes + a.b_off;
          const float* wf = reinterpret_cast<const float*>(smem + stage * a.stage_bytes + a.w_off);
          const int wrows = min(BK, a.D - kb * BK);
          // Item (c, e) -> its three 16-byte chunks of B.
          auto convert_store = [&](int i, const float (&wv)[8]) {
            const int c = i / E, e = i - c * E;
            float t0[8], t1[8], t2[8];
  #pragma unroll
            for (int j = 0; j < 8; ++j) split3(wv[j], t0[j], t1[j], t2[j]);
            const uint4 v0 = make_uint4(pack_bf16x2(t0[0], t0[1]), pack_bf16x2(t0[2], t0[3]),
                                        pack_bf16x2(t0[4], t0[5]), pack_bf16x2(t0[6], t0[7]));
            const uint4 v1 = make_uint4(pack_bf16x2(t1[0], t1[1]), pack_bf16x2(t1[2], t1[3]),
                                        pack_bf16x2(t1[4], t1[5]), pack_bf16x2(t1[6], t1[7]));
            const uint4 v2 = make_uint4(pack_bf16x2(t2[0], t2[1]), pack_bf16x2(t2[2], t2[3]),
                                        pack_bf16x2(t2[4], t2[5]), pack_bf16x2(t2[6], t2[7]));
            const int n0 = e, n1 = a.Ep + e, n2 = 2 * a.Ep + e;
            *reinterpret_cast<uint4*>(b + n0 * 128 + ((c ^ (n0 & 7)) << 4)) = v0;
            *reinterpret_cast<uint4*>(b + n1 * 128 + ((c ^ (n1 & 7)) << 4)) = v1;
            *reinterpret_cast<uint4*>(b + n2 * 128 + ((c ^ (n2 & 7)) << 4)) = v2;
          };
          if (items <= kConvThreads) {  // E <= 16: at most one item per thread
            if (ct < items) {
              const int c = ct / E, e = ct - c * E;
              float wv[8];
  #pragma unroll
              for (int j = 0; j < 8; ++j) {
                const int d = c * 8 + j;
                wv[j] = d < wrows ? wf[d * E + e] : 0.f;
              }
              convert_store(ct, wv);
            }
          }
          // Larger E: kBatch items per thread at a time, all their loads first (independent
          // chains for the scheduler; E = 64 gives each thread 4 items per k-block).
          constexpr int kBatch = 4;
          for (int i0 = items <= kConvThreads ? items : ct; i0 < items;
               i0 += kBatch * kConvThreads) {
            float w[kBatch][8];
  #pragma unroll
            for (int u = 0; u < kBatch; ++u) {
              const int i = i0 + u * kConvThreads;
              const int c = i / E, e = i - c * E;
  #pragma unroll
              for (int j = 0; j < 8; ++j) {
                const int d = c * 8 + j;
                w[u][j] = (i < items && d < wrows) ? wf[d * E + e] : 0.f;
              }
            }
  #pragma unroll
            for (int u = 0; u < kBatch; ++u) {
              const int i = i0 + u * kConvThreads;
              if (i >= items) break;
              convert_store(i, w[u]);
            }
          }
          fence_proxy_async_smem();  // generic-proxy stores before the MMA (async proxy) reads
          __syncwarp();
          if (lane == 0) mbar_arrive(&full[stage]);
          if (++stage == a.stages) {
            stage = 0;
            phase ^= 1u;
          }
        }
      }
    }
  } else {  // ------------------------------------------------------------------- epilogue
    // Thread row = q*32 + lane reads TMEM lane `row` (tile row = token). With S = 1 it owns
    // that token outright; with S > 1 every row's partial goes to shared memory and the
    // thread whose row lies in this CTA's share [rank*T, rank*T + T) adds the S partials.
    const int q = warp & 3;
    const int row = q * 32 + lane;
    const int et = threadIdx.x - 64;  // 0..127, for the per-expert column sums
    const int T = kRows / S;
    const int share0 = static_cast<int>(rank) * T;
    const bool owner = row >= share0 && row < share0 + T;
    const int E = a.E;
    float colsum_acc = 0.f;
    float zl_acc = 0.f;
    int it = 0;
    for (int64_t tile = first_tile; tile < a.tiles; tile += a.num_clusters, ++it) {
      const int acc = it & 1;
      const uint32_t acc_phase = static_cast<uint32_t>(it >> 1) & 1u;
      bool ok = mbar_wait(&tfull[acc], acc_phase, a.timeout_ns);
      // The owners must have read this CTA's pushes of the previous tile before they are
      // overwritten.
      if (S > 1 && ok && it > 0)
        ok = mbar_wait_cluster(zfree, static_cast<uint32_t>(it - 1) & 1u, a.timeout_ns);
      // Leave together: the four epilogue warps share named barriers below.
      if (named_bar_any(1, kEpiThreads, !ok)) {
        if (et == 0) record_error(a.err, MOE_DEVERR_WAIT_TIMEOUT);
        break;
      }
      __syncwarp();
      tc_fence_after_sync();
      // 1. Accumulator -> registers, the three terms added smallest first.
      float z[EB];
      const uint32_t t_row = tmem_base + (static_cast<uint32_t>(q * 32) << 16) +
                             static_cast<uint32_t>(acc * kAccStride);
#pragma unroll
      for (int g = 0; g < EB; g += 8) {
        if (g < a.Ep && has_k) {
          uint32_t r0[8], r1[8], r2[8];
          tmem_ld_8cols(t_row + g, r0);
          tmem_ld_8cols(t_row + a.Ep + g, r1);
          tmem_ld_8cols(t_row + 2 * a.Ep + g, r2);
          tmem_ld_wait();
#pragma unroll
          for (int i = 0; i < 8; ++i)
            z[g + i] = (__uint_as_float(r2[i]) + __uint_as_float(r1[i])) + __uint_as_float(r0[i]);
        } else {
#pragma unroll
          for (int i = 0; i < 8; ++i) z[g + i] = 0.f;
        }
      }
      tc_fence_before_sync();
      __syncwarp();
      if (lane == 0) mbar_arrive(&tempty[acc]);  // the MMA warp may reuse this accumulator
      if (S > 1) {
        // 2. Push this row's partial to its owner q (slot [rank][row - q T] of q's receive
        //    buffer), arrive on q's zready; then each owner adds the S slots of its rows in
        //    slice order, locally.
        const int q = row / T;
        const uint32_t dst = mapa_shared(
            smem_u32(zbuf) + static_cast<uint32_t>(((static_cast<int>(rank) * T + row - q * T) *
                                                    a.zstride) * 4),
            static_cast<uint32_t>(q));
#pragma unroll
        for (int c = 0; c < EB; c += 4)
          if (c < a.Ep) st_dsmem_f4(dst + c * 4u, make_float4(z[c], z[c + 1], z[c + 2], z[c + 3]));
        mbar_arrive_cluster(mapa_shared(smem_u32(zready), static_cast<uint32_t>(q)));
        ok = mbar_wait_cluster(zready, static_cast<uint32_t>(it) & 1u, a.timeout_ns);
        if (named_bar_any(1, kEpiThreads, !ok)) {
          if (et == 0) record_error(a.err, MOE_DEVERR_WAIT_TIMEOUT);
          break;
        }
        if (owner) {
          const float* slot = zbuf + (row - share0) * a.zstride;  // slice r: + r T zstride
#pragma unroll
          for (int c = 0; c < EB; c += 4) {
            if (c < a.Ep) {
              float4 acc4 = *reinterpret_cast<const float4*>(slot + c);
#pragma unroll
              for (int r = 1; r < kMaxCluster; ++r) {
                if (r < S) {
                  const float4 w = *reinterpret_cast<const float4*>(slot + r * T * a.zstride + c);
                  acc4.x += w.x;
                  acc4.y += w.y;
                  acc4.z += w.z;
                  acc4.w += w.w;
                }
              }
              z[c] = acc4.x;
              z[c + 1] = acc4.y;
              z[c + 2] = acc4.z;
              z[c + 3] = acc4.w;
            } else {
              z[c] = z[c + 1] = z[c + 2] = z[c + 3] = 0.f;
            }
          }
          // Another tile follows: tell every source CTA its slot of this row has been read.
          if (tile + a.num_clusters < a.tiles)
            for (int r = 0; r < S; ++r)
              mbar_arrive_cluster(mapa_shared(smem_u32(zfree), static_cast<uint32_t>(r)));
        }
      }
      // 3. Bias and the routing decision for the owned tokens.
      const int64_t t = tile * kRows + row;
      if (owner && t < a.N) {
#pragma unroll
        for (int e = 0; e < EB; ++e)
          if (e < E && a.bias != nullptr) z[e] += __ldg(a.bias + e);
        if (a.logits_out != nullptr)
#pragma unroll
          for (int e = 0; e < EB; ++e)
            if (e < E) a.logits_out[t * E + e] = z[e];
        // The decision runs from the token's row of shared memory (loops over E, not unrolled
        // per expert and per choice: compact code, and the same arithmetic as the SIMT
        // routers); with the balance statistic the row is left holding the probabilities.
        float* zt = s_z + (row - share0) * (E + 1);  // column E: (log Z)^2 of the token
#pragma unroll
        for (int e = 0; e < EB; ++e)
          if (e < E) zt[e] = z[e];
        float lse = 0.f;
        select_token(zt, E, a.k, a.renorm, a.mode, a.noise != nullptr ? a.noise + t * E : nullptr,
                     a.idx + t * a.k, a.gate + t * a.k, a.colsum_partial != nullptr,
                     a.zl_partial != nullptr ? &lse : nullptr);
        zt[E] = lse * lse;
      }
      if (a.colsum_partial != nullptr || a.zl_partial != nullptr) {  // sums in token order
        named_bar_sync(1, kEpiThreads);
        const int64_t left = a.N - (tile * kRows + share0);
        const int valid = left < T ? static_cast<int>(left > 0 ? left : 0) : T;
        if (a.colsum_partial != nullptr && et < E)
          for (int i = 0; i < valid; ++i) colsum_acc += s_z[i * (E + 1) + et];
        if (a.zl_partial != nullptr && et == 0)
          for (int i = 0; i < valid; ++i) zl_acc += s_z[i * (E + 1) + E];
        named_bar_sync(1, kEpiThreads);
      }
    }
    if (a.colsum_partial != nullptr && et < E)
      a.colsum_partial[static_cast<int64_t>(blockIdx.x) * E + et] = colsum_acc;
    if (a.zl_partial != nullptr && et == 0) a.zl_partial[blockIdx.x] = zl_acc;
  }

  __syncwarp();  // role branches leave warps 0 and 1 divergent; the barriers below are .aligned
  __syncthreads();
  if (warp == 1) {
    __syncwarp();
    tc_fence_after_sync();
    tmem_dealloc(tmem_base, kTmemCols);
  }
  __syncwarp();
  cluster_sync_all();  // no CTA leaves while a peer may still read its shared memory
}

constexpr uint32_t kBarBytes = 512;  // mbarriers and the TMEM address

struct TcShape {
  int Ep, NB, zstride, num_kb, S, num_clusters, stages;
  int64_t tiles;
  uint32_t stage_bytes, b_off, w_off, zbuf_off, sz_off, bar_off, smem_bytes;
};

// More than 16 experts: the B operand is written once per call and loaded by TMA.
bool prepared_operand(int E) { return E > 16; }

TcShape tc_shape(int64_t N, int D, int E) {
  TcShape s{};
  s.Ep = (E + 7) / 8 * 8;
  s.NB = (3 * s.Ep + 15) / 16 * 16;
  s.zstride = s.Ep + 4;  // rows 16 bytes apart in the bank map: conflict-free float4 stores
  s.num_kb = (D + BK - 1) / BK;
  s.tiles = (N + kRows - 1) / kRows;
  // Cluster size: the largest power of two <= 8 that keeps tiles * S within one CTA per SM and
  // leaves every CTA at least one k-block.
  const int64_t want = std::max<int64_t>(1, kUnitTarget / std::max<int64_t>(1, s.tiles));
  s.S = 1;
  while (s.S * 2 <= kMaxCluster && s.S * 2 <= want && s.S * 2 <= s.num_kb) s.S *= 2;
  if (const char* env = std::getenv("MOE_ROUTE_CLUSTER")) {  // testing and tuning
    const int v = std::atoi(env);
    if (v == 1 || v == 2 || v == 4 || v == 8) {
      s.S = v;
      while (s.S > 1 && s.S > s.num_kb) s.S /= 2;  // every CTA keeps at least one k-block
    }
  }
  s.num_clusters = static_cast<int>(
      std::max<int64_t>(1, std::min<int64_t>(s.tiles, kUnitTarget / s.S)));
  // Shared memory: [stages][A 16 KB | B (bf16 terms) | W (fp32 slice, 64 x E; not with the
  // prepared operand)] [partials 128 x zstride] [summed logits] [barriers]; A and B
  // 1024-byte aligned.
  const uint32_t b_bytes = static_cast<uint32_t>((s.NB * BK * 2 + 1023) / 1024 * 1024);
  const uint32_t w_bytes =
      prepared_operand(E) ? 0u : static_cast<uint32_t>((BK * E * 4 + 1023) / 1024 * 1024);
  s.b_off = kABytes;
  s.w_off = kABytes + b_bytes;
  s.stage_bytes = kABytes + b_bytes + w_bytes;
  // Partials are exchanged only between the CTAs of a cluster (S > 1).
  const uint32_t zbuf_bytes = s.S > 1 ? static_cast<uint32_t>(kRows * s.zstride * 4) : 0u;
  const uint32_t sz_bytes = static_cast<uint32_t>(((kRows / s.S) * (E + 1) * 4 + 15) / 16 * 16);
  const uint32_t fixed = 1024 /*align*/ + kBarBytes + zbuf_bytes + sz_bytes;
  s.stages = static_cast<int>(
      std::min<uint32_t>(kMaxStages, (kSmemLimit - fixed) / s.stage_bytes));
  s.zbuf_off = static_cast<uint32_t>(s.stages) * s.stage_bytes;
  s.sz_off = s.zbuf_off + zbuf_bytes;
  s.bar_off = s.sz_off + sz_bytes;
  s.smem_bytes = s.bar_off + kBarBytes + 1024;
  return s;
}

}  // namespace

bool route_tc_supported(const moe_problem& p) {
  return p.dtype == MOE_DTYPE_BF16 && p.E <= kMaxEc;
}

size_t route_tc_operand_bytes(const moe_problem& p) {
  if (!route_tc_supported(p) || !prepared_operand(p.E) || p.E < 1) return 0;
  const TcShape s = tc_shape(1, static_cast<int>(p.D), p.E);
  return static_cast<size_t>(s.NB) * static_cast<size_t>(p.D) * 2;
}

cudaError_t launch_route_tc(const moe_problem& p, const void* X, const float* W_r,
                            const float* bias, const float* noise, float* logits_out,
                            int32_t* idx, float* gate, float* colsum_partial, float* zl_partial,
                            void* operand, int* grid_out, int* err, uint64_t timeout_ns,
                            cudaStream_t stream) {
  const TcShape s = tc_shape(p.N, static_cast<int>(p.D), p.E);
  *grid_out = 0;
  if (p.N == 0) return cudaSuccess;
  if (s.stages < 2) return cudaErrorInvalidConfiguration;
  const int D = static_cast<int>(p.D);
  const bool prepared = prepared_operand(p.E);
  if (prepared && operand == nullptr) return cudaErrorInvalidValue;
  CUtensorMap tX, tB;
  if (!make_tensor_map_2d_bf16(&tX, X, static_cast<uint64_t>(D), static_cast<uint64_t>(p.N), 64,
                               kRows))
    return cudaErrorInvalidValue;
  tB = tX;  // unused unless prepared
  cudaError_t e = cudaSuccess;
  if (prepared) {
    // The B operand [NB][D] bf16, rows 128 bytes apart in each 64-k box (128-byte swizzle).
    if (!make_tensor_map_2d_bf16(&tB, operand, static_cast<uint64_t>(D),
                                 static_cast<uint64_t>(s.NB), 64, static_cast<uint32_t>(s.NB)))
      return cudaErrorInvalidValue;
    const int64_t total = static_cast<int64_t>(s.NB) * D;
    const int blocks = static_cast<int>(std::min<int64_t>((total + 255) / 256, 4 * num_sms()));
    cudaLaunchConfig_t ocfg = {};
    ocfg.gridDim = dim3(static_cast<unsigned>(std::max(blocks, 1)));
    ocfg.blockDim = dim3(256);
    ocfg.stream = stream;
    cudaLaunchAttribute oattr[1];
    ocfg.attrs = oattr;
    ocfg.numAttrs = pdl_attr(&oattr[0]);
    e = cudaLaunchKernelEx(&ocfg, route_operand_kernel, W_r, D, p.E, s.Ep, s.NB,
                           static_cast<__nv_bfloat16*>(operand));
    if (e != cudaSuccess) return e;
  }
  TcArgs a;
  a.W_r = W_r;
  a.bias = bias;
  a.logits_out = logits_out;
  a.idx = idx;
  a.gate = gate;
  a.colsum_partial = colsum_partial;
  a.noise = noise;
  a.zl_partial = zl_partial;
  a.mode = p.routing_mode;
  a.N = p.N;
  a.tiles = s.tiles;
  a.D = D;
  a.E = p.E;
  a.k = p.k;
  a.renorm = p.renormalize;
  a.Ep = s.Ep;
  a.NB = s.NB;
  a.zstride = s.zstride;
  a.num_kb = s.num_kb;
  a.S = s.S;
  a.num_clusters = s.num_clusters;
  a.stages = s.stages;
  a.prepared = prepared ? 1 : 0;
  a.stage_bytes = s.stage_bytes;
  a.b_off = s.b_off;
  a.w_off = s.w_off;
  a.zbuf_off = s.zbuf_off;
  a.sz_off = s.sz_off;
  a.bar_off = s.bar_off;
  a.err = err;
  a.timeout_ns = timeout_ns;
  void (*kern)(const CUtensorMap, const CUtensorMap, const TcArgs) =
      s.Ep <= 8 ? route_tc_kernel<8>
                : (s.Ep <= 16 ? route_tc_kernel<16> : (s.Ep <= 32 ? route_tc_kernel<32> : route_tc_kernel<64>));
  e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize,
                           static_cast<int>(s.smem_bytes));
  if (e != cudaSuccess) return e;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(static_cast<unsigned>(s.num_clusters * s.S));
  cfg.blockDim = dim3(kThreads);
  cfg.dynamicSmemBytes = s.smem_bytes;
  cfg.stream = stream;
  cudaLaunchAttribute attr[2];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = static_cast<unsigned>(s.S);
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1 + pdl_attr(&attr[1]);
  e = cudaLaunchKernelEx(&cfg, kern, tX, tB, a);
  if (e != cudaSuccess) return e;
  *grid_out = s.num_clusters * s.S;
  return cudaGetLastError();
}

}  // namespace moe

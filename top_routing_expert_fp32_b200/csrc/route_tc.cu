// Router logits on the tensor cores for bf16 activations: z = X W_r (+ bias) with fp32-level
// accuracy, where X is [N, D] bf16 and W_r is [D, E] fp32.
//   Grok-1 book ch.5, 5.2 (router logits kept in fp32); MoE formula-to-code walkthrough 1.1.
//
// The fp32 router weights are split into three bf16 terms, w = w0 + w1 + w2 with
// w0 = bf16(w), w1 = bf16(w - w0), w2 = bf16(w - w0 - w1) (the "bf16x3" decomposition of
// Henry, Tang and Heinecke, "Leveraging the bfloat16 Artificial Intelligence Datatype For
// Higher-Precision Computations", ARITH 2019). The three terms carry 24 significant bits,
// as many as the fp32 value; what is left over is below 2^-24 |w|. X is bf16 already, so
// every product x * w_i is exact in fp32 and one bf16 MMA with fp32 accumulation over the
// concatenated [w0 | w1 | w2] columns gives all three partial dot products. The epilogue adds
// them smallest first: z = (z2 + z1) + z0.
//
// Kernels:
//   split_wr_kernel  : W_r [D][E] fp32 -> Wt [NB][D] bf16 (K-major B operand), row
//                      i * Ep + e holding term i of expert e; padding rows are zero.
//   route_tc_kernel  : persistent, one CTA per SM, 6 warps (TMA producer, MMA issuer, 4
//                      epilogue warps). A work unit is a 128-token tile and a slice of the
//                      D range (split-K when there are fewer tiles than SMs). Each unit's
//                      partial logits go to zpart[slice][token][Ep]; the selection kernel
//                      adds the slices in slice order (deterministic, no atomics).
// Every barrier wait is bounded in time; on a timeout the CTA records MOE_DEVERR_WAIT_TIMEOUT,
// drains its MMAs and frees its tensor memory.
#include <algorithm>

#include "common.cuh"
#include "internal.h"

namespace moe {
namespace {

constexpr int kRows = 128;         // tokens per tile = accumulator lanes
constexpr int BK = 64;             // k-block: one 128-byte swizzle row of bf16
constexpr int UK = 16;             // K of one tcgen05.mma kind::f16
constexpr int kThreads = 192;
constexpr int kMaxNB = 192;        // 3 terms x 64 experts
constexpr int kABytes = kRows * BK * 2;           // 16 KB
constexpr int kBBytesMax = kMaxNB * BK * 2;       // 24 KB
constexpr int kStageBytes = kABytes + kBBytesMax;  // 40 KB
constexpr int kStages = 5;
constexpr int kAccStride = 256;    // TMEM columns between the two accumulators
constexpr int kTmemCols = 512;
constexpr int kSmemBytes = kStages * kStageBytes + 1024 /*align*/ + 256 /*barriers*/;
constexpr int kUnitTarget = 148;   // work units wanted per launch (one per SM of a B200)

struct TcParams {
  float* zpart;       // [S][N][Ep]
  int64_t N;
  int Ep;             // experts padded to a multiple of 8 (TMEM load granularity)
  int NB;             // MMA N: 3 * Ep padded to a multiple of 16
  int num_kb;         // k-blocks over D
  int kps;            // k-blocks per slice
  int S;              // slices
  int64_t units;      // tiles * S
  int* err;
  uint64_t timeout_ns;
};

__global__ void __launch_bounds__(kThreads, 1)
    route_tc_kernel(const __grid_constant__ CUtensorMap tmX, const __grid_constant__ CUtensorMap tmW,
                    const TcParams p) {
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  const uint32_t raw_addr = smem_u32(smem_raw);
  uint8_t* smem = smem_raw + ((1024u - (raw_addr & 1023u)) & 1023u);
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + kStages * kStageBytes);
  uint64_t* empty = full + kStages;
  uint64_t* tfull = empty + kStages;
  uint64_t* tempty = tfull + 2;
  uint64_t* drain = tempty + 2;
  uint32_t* s_tmem = reinterpret_cast<uint32_t*>(drain + 1);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  if (static_cast<int64_t>(blockIdx.x) >= p.units) return;  // uniform over the block

  if (threadIdx.x == 0) {
    for (int s = 0; s < kStages; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], 1);
    }
    for (int a = 0; a < 2; ++a) {
      mbar_init(&tfull[a], 1);
      mbar_init(&tempty[a], 4);  // one arrival per epilogue warp
    }
    mbar_init(drain, 1);
    fence_barrier_init();
    prefetch_tensormap(&tmX);
    prefetch_tensormap(&tmW);
  }
  if (warp == 1) {
    tmem_alloc(s_tmem, kTmemCols);
    tmem_relinquish();
  }
  tc_fence_before_sync();
  __syncthreads();
  tc_fence_after_sync();
  const uint32_t tmem_base = *s_tmem;
  const uint32_t tx_bytes = static_cast<uint32_t>(kABytes + p.NB * BK * 2);

  if (warp == 0) {
    if (lane == 0) {  // ------------------------------------------------------ TMA producer
      int stage = 0;
      uint32_t phase = 0;
      bool ok = true;
      for (int64_t u = blockIdx.x; ok && u < p.units; u += gridDim.x) {
        const int64_t tile = u / p.S;
        const int s = static_cast<int>(u - tile * p.S);
        const int kb0 = s * p.kps;
        const int kb1 = min(kb0 + p.kps, p.num_kb);
        for (int kb = kb0; kb < kb1; ++kb) {
          if (!mbar_wait(&empty[stage], phase ^ 1u, p.timeout_ns)) {
            record_error(p.err, MOE_DEVERR_WAIT_TIMEOUT);
            ok = false;
            break;
          }
          uint8_t* a_dst = smem + stage * kStageBytes;
          mbar_arrive_expect_tx(&full[stage], tx_bytes);
          tma_load_2d(a_dst, &tmX, &full[stage], kb * BK, static_cast<int>(tile * kRows));
          tma_load_2d(a_dst + kABytes, &tmW, &full[stage], kb * BK, 0);
          if (++stage == kStages) {
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
                             (static_cast<uint32_t>(p.NB >> 3) << 17) |
                             (static_cast<uint32_t>(kRows >> 4) << 24);
      int stage = 0;
      uint32_t phase = 0;
      bool ok = true;
      int it = 0;
      for (int64_t u = blockIdx.x; ok && u < p.units; u += gridDim.x, ++it) {
        const int64_t tile = u / p.S;
        const int s = static_cast<int>(u - tile * p.S);
        const int kb0 = s * p.kps;
        const int kb1 = min(kb0 + p.kps, p.num_kb);
        const int acc = it & 1;
        const uint32_t acc_phase = static_cast<uint32_t>(it >> 1) & 1u;
        if (!mbar_wait(&tempty[acc], acc_phase ^ 1u, p.timeout_ns)) {
          record_error(p.err, MOE_DEVERR_WAIT_TIMEOUT);
          ok = false;
          break;
        }
        tc_fence_after_sync();
        const uint32_t d_tmem = tmem_base + static_cast<uint32_t>(acc * kAccStride);
        for (int kb = kb0; kb < kb1; ++kb) {
          if (!mbar_wait(&full[stage], phase, p.timeout_ns)) {
            record_error(p.err, MOE_DEVERR_WAIT_TIMEOUT);
            ok = false;
            break;
          }
          tc_fence_after_sync();
          const uint32_t a_addr = smem_u32(smem + stage * kStageBytes);
          const uint32_t b_addr = a_addr + kABytes;
#pragma unroll
          for (int kk = 0; kk < BK / UK; ++kk) {
            // Both operands K-major SW128: advance 16 elements = 32 bytes in the swizzle row.
            const uint64_t ad = smem_desc_sw128(a_addr + kk * 32, 16, 1024);
            const uint64_t bd = smem_desc_sw128(b_addr + kk * 32, 16, 1024);
            umma_bf16_ss(d_tmem, ad, bd, idesc, (kb > kb0 || kk > 0) ? 1u : 0u);
          }
          umma_commit(&empty[stage]);  // frees the stage once these MMAs have read it
          if (++stage == kStages) {
            stage = 0;
            phase ^= 1u;
          }
        }
        if (ok) umma_commit(&tfull[acc]);
      }
      umma_commit(drain);  // flips once every MMA issued above has completed
      if (!mbar_wait(drain, 0, p.timeout_ns)) record_error(p.err, MOE_DEVERR_WAIT_TIMEOUT);
    }
  } else {  // ------------------------------------------------------------------- epilogue
    const int q = warp & 3;  // this warp may access TMEM lanes [32q, 32q+32)
    int it = 0;
    for (int64_t u = blockIdx.x; u < p.units; u += gridDim.x, ++it) {
      const int64_t tile = u / p.S;
      const int s = static_cast<int>(u - tile * p.S);
      const int acc = it & 1;
      const uint32_t acc_phase = static_cast<uint32_t>(it >> 1) & 1u;
      const bool ok = mbar_wait(&tfull[acc], acc_phase, p.timeout_ns);
      if (__any_sync(0xffffffffu, !ok)) {
        if (lane == 0) record_error(p.err, MOE_DEVERR_WAIT_TIMEOUT);
        break;
      }
      __syncwarp();
      tc_fence_after_sync();
      const int64_t t = tile * kRows + q * 32 + lane;
      const bool valid = t < p.N;
      float* zrow = p.zpart + (static_cast<int64_t>(s) * p.N + (valid ? t : 0)) * p.Ep;
      const uint32_t t_row = tmem_base + (static_cast<uint32_t>(q * 32) << 16) +
                             static_cast<uint32_t>(acc * kAccStride);
#pragma unroll 1
      for (int g = 0; g < p.Ep; g += 8) {
        uint32_t r0[8], r1[8], r2[8];
        tmem_ld_8cols(t_row + g, r0);                // w0 term
        tmem_ld_8cols(t_row + p.Ep + g, r1);         // w1 term
        tmem_ld_8cols(t_row + 2 * p.Ep + g, r2);     // w2 term
        tmem_ld_wait();
        if (valid) {
          float z[8];
#pragma unroll
          for (int i = 0; i < 8; ++i)
            z[i] = (__uint_as_float(r2[i]) + __uint_as_float(r1[i])) + __uint_as_float(r0[i]);
          reinterpret_cast<float4*>(zrow + g)[0] = make_float4(z[0], z[1], z[2], z[3]);
          reinterpret_cast<float4*>(zrow + g)[1] = make_float4(z[4], z[5], z[6], z[7]);
        }
      }
      tc_fence_before_sync();
      __syncwarp();
      if (lane == 0) mbar_arrive(&tempty[acc]);
    }
  }

  __syncwarp();  // role branches leave warps 0 and 1 divergent; the barrier below is .aligned
  __syncthreads();
  if (warp == 1) {
    __syncwarp();
    tc_fence_after_sync();
    tmem_dealloc(tmem_base, kTmemCols);
  }
}

// Wt[i * Ep + e][d] = term i of W_r[d][e] (zero for e >= E and for rows >= 3 * Ep).
// A block converts 64 rows of W_r (contiguous in memory) through shared memory.
constexpr int kSplitRows = 64;
constexpr int kSplitThreads = 256;

__global__ void __launch_bounds__(kSplitThreads)
    split_wr_kernel(const float* __restrict__ W_r, __nv_bfloat16* __restrict__ Wt, int D, int E,
                    int Ep, int NB) {
  __shared__ float s_w[kSplitRows * 64];
  const int d0 = blockIdx.x * kSplitRows;
  const int rows = min(kSplitRows, D - d0);
  for (int i = threadIdx.x; i < rows * E; i += kSplitThreads)
    s_w[i] = W_r[static_cast<int64_t>(d0) * E + i];
  __syncthreads();
  // Output element (n, d0 + dd): consecutive threads take consecutive dd (coalesced rows).
  for (int i = threadIdx.x; i < NB * kSplitRows; i += kSplitThreads) {
    const int n = i / kSplitRows;
    const int dd = i - n * kSplitRows;
    if (dd >= rows) continue;
    const int term = n / Ep;
    const int e = n - term * Ep;
    float v = 0.f;
    if (term < 3 && e < E) {
      const float w = s_w[dd * E + e];
      const float w0 = __bfloat162float(__float2bfloat16_rn(w));
      const float r1 = w - w0;  // exact: w0 holds w's leading 8 significant bits
      const float w1 = __bfloat162float(__float2bfloat16_rn(r1));
      const float r2 = r1 - w1;  // exact for the same reason
      v = term == 0 ? w0 : (term == 1 ? w1 : __bfloat162float(__float2bfloat16_rn(r2)));
    }
    Wt[static_cast<int64_t>(n) * D + d0 + dd] = __float2bfloat16_rn(v);
  }
}

struct TcShape {
  int Ep, NB, num_kb, kps, S;
  int64_t tiles;
};

TcShape tc_shape(int64_t N, int D, int E) {
  TcShape s;
  s.Ep = (E + 7) / 8 * 8;
  s.NB = (3 * s.Ep + 15) / 16 * 16;
  s.num_kb = (D + BK - 1) / BK;
  s.tiles = (N + kRows - 1) / kRows;
  // Slices per tile: as many as keep tiles * S within one unit per SM.
  const int want = static_cast<int>(
      std::min<int64_t>(s.num_kb, std::max<int64_t>(1, kUnitTarget / std::max<int64_t>(1, s.tiles))));
  s.kps = (s.num_kb + want - 1) / want;
  s.S = (s.num_kb + s.kps - 1) / s.kps;  // no empty slice
  return s;
}

}  // namespace

bool route_tc_supported(const moe_problem& p) {
  return p.dtype == MOE_DTYPE_BF16 && p.E <= 64;
}

size_t route_tc_wt_bytes(const moe_problem& p) {
  if (!route_tc_supported(p)) return 0;
  const TcShape s = tc_shape(p.N, static_cast<int>(p.D), p.E);
  return static_cast<size_t>(s.NB) * static_cast<size_t>(p.D) * 2;
}

size_t route_tc_zpart_bytes(const moe_problem& p) {
  if (!route_tc_supported(p)) return 0;
  const TcShape s = tc_shape(p.N, static_cast<int>(p.D), p.E);
  return static_cast<size_t>(s.S) * static_cast<size_t>(p.N) * s.Ep * sizeof(float);
}

cudaError_t launch_route_tc_logits(const moe_problem& p, const void* X, const float* W_r,
                                   __nv_bfloat16* Wt, float* zpart, int* S_out, int* Ep_out,
                                   int* err, uint64_t timeout_ns, cudaStream_t stream) {
  const TcShape s = tc_shape(p.N, static_cast<int>(p.D), p.E);
  *S_out = s.S;
  *Ep_out = s.Ep;
  if (p.N == 0) return cudaSuccess;
  const int D = static_cast<int>(p.D);
  split_wr_kernel<<<(D + kSplitRows - 1) / kSplitRows, kSplitThreads, 0, stream>>>(
      W_r, Wt, D, p.E, s.Ep, s.NB);
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  CUtensorMap tX, tW;
  if (!make_tensor_map_2d_bf16(&tX, X, static_cast<uint64_t>(D), static_cast<uint64_t>(p.N), 64,
                               kRows) ||
      !make_tensor_map_2d_bf16(&tW, Wt, static_cast<uint64_t>(D), static_cast<uint64_t>(s.NB), 64,
                               static_cast<uint32_t>(s.NB)))
    return cudaErrorInvalidValue;
  TcParams tp;
  tp.zpart = zpart;
  tp.N = p.N;
  tp.Ep = s.Ep;
  tp.NB = s.NB;
  tp.num_kb = s.num_kb;
  tp.kps = s.kps;
  tp.S = s.S;
  tp.units = s.tiles * s.S;
  tp.err = err;
  tp.timeout_ns = timeout_ns;
  e = cudaFuncSetAttribute(route_tc_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, kSmemBytes);
  if (e != cudaSuccess) return e;
  const int grid = static_cast<int>(std::max<int64_t>(1, std::min<int64_t>(num_sms(), tp.units)));
  route_tc_kernel<<<grid, kThreads, kSmemBytes, stream>>>(tX, tW, tp);
  return cudaGetLastError();
}

}  // namespace moe

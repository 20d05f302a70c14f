// Grouped gated expert FFN with 8-bit expert weights for experts that hold few rows (the
// decode-sized layer), on the tcgen05 tensor cores with the weights as the TMEM operand.
//   GEMM1: H[r] = act(x_r W1_e) (.) (x_r W2_e)      GEMM2: Y[r] = H[r] W3_e
// with W = q * s, q int8 and s one fp32 scale per expert and output column (Grok-1 book ch.5,
// 5.3.3 and 5.3.5: weight = weight * scales before each expert matmul).
//
// The product is computed transposed, D^T = W^T X^T: the M = 128 output columns of a tile are
// the MMA's rows and its N <= 64 token rows the MMA's columns. Converter warps turn the int8
// weights into bf16 (exactly) and store them with tcgen05.st straight into tensor memory,
// where tcgen05.mma takes its A operand from; the token rows come from shared memory as the B
// operand. The converted weights therefore never touch shared memory, the traffic that bounds
// the shared-memory variant of this layer when the batch is small and the weights dominate.
// In the epilogue each thread owns one output column (its TMEM lane): the column scale is a
// register and a warp stores 32 consecutive columns of a row.
//
// One persistent CTA per SM, 14 warps:
//   warp 0 lane 0 : TMA producer. Per k-block of 64: the tile's token rows (64x64 bf16,
//                   K-major, 128-byte swizzle) and one or two 64x128 int8 weight boxes.
//   warps 6..13   : converters. Warp w takes TMEM lanes [32 (w % 4), +32) (output columns) and
//                   half of the k-block's rows; each thread converts its column's 32 weights
//                   of each matrix to 16 bf16 pairs and stores them with one tcgen05.st.
//   warp 1        : TMEM allocation (512 columns: two accumulator sets of 2 x 64 columns and
//                   four 64-column weight stages); lane 0 issues the MMAs (A from TMEM).
//   warps 2..5    : epilogue, double-buffered against the next tile.
// Every barrier wait is bounded in time; on a timeout the CTA records MOE_DEVERR_WAIT_TIMEOUT,
// unwinds, drains its MMAs and frees its TMEM.
#include <algorithm>
#include <cstdlib>
#include <cstring>

#include "common.cuh"
#include "internal.h"

namespace moe {
namespace {

constexpr int kNT = 128;                  // output columns per tile = MMA M = TMEM lanes
constexpr int kRT = 64;                   // token rows per tile = largest MMA N
constexpr int BK = 64;
constexpr int UK = 16;
constexpr int kXBytes = kRT * BK * 2;     // 8 KB: token rows of a k-block
constexpr int kQBox = BK * kNT;           // 8 KB: 64 k-rows x 128 int8 columns
constexpr int kStageBytes = kXBytes + 2 * kQBox;  // 24 KB
constexpr int kAccCols = 2 * kRT;         // one accumulator set: W1 and W2 products
constexpr int kACols = 2 * (BK / 2);      // one TMEM weight stage: two matrices x 32 columns
constexpr int kAColBase = 2 * kAccCols;   // TMEM weight stages after the two accumulator sets
constexpr int kAMatBytes = kNT * BK * 2;  // 16 KB: one converted matrix in shared memory
constexpr int kThreads = 448;
constexpr int kConvWarps = 8;
constexpr int kMaxE = 64;
constexpr int kGroup = 8;

// ASMEM: the converted weights are the A operand in shared memory (K-major, 128-byte swizzle,
// one 128-byte row per output column); otherwise in tensor memory.
template <bool ASMEM>
struct W8tShape {
  static constexpr int kStages = ASMEM ? 5 : 8;    // TMA ring (token rows + int8 weights)
  static constexpr int kAStages = ASMEM ? 3 : 4;   // converted-weight stages
  static constexpr int kAStageBytes = ASMEM ? 2 * kAMatBytes : 0;
  static constexpr int kTmemCols = ASMEM ? 2 * kAccCols : 512;
  static constexpr int kSmemBytes =
      kStages * kStageBytes + kAStages * kAStageBytes + 1024 /*align*/ + 1024 /*barriers*/;
};
static_assert(kAColBase + 4 * kACols <= 512, "TMEM budget");
static_assert(W8tShape<true>::kSmemBytes <= 227 * 1024, "shared memory budget");
static_assert(W8tShape<false>::kSmemBytes <= 227 * 1024, "shared memory budget");

struct W8tParams {
  const int32_t* offsets;  // [E+1]
  const float* s0;         // scales of W1 (GEMM1) or W3 (GEMM2): [E][n_out]
  const float* s1;         // scales of W2 (GEMM1 only)
  __nv_bfloat16* out;      // [rows, n_out]
  int E;
  int K;
  int n_out;
  int* err;
  uint64_t timeout_ns;
};

// Two int8 weights (q0, q1: low bytes of the registers) -> their bf16 pair, exactly: the byte,
// biased to q + 128, becomes the low mantissa byte of 2^23 + q + 128; subtracting 2^23 + 128
// leaves q, whose upper 16 bits are its bf16 encoding.
__device__ __forceinline__ uint32_t i8x2_to_bf16x2(uint32_t b0, uint32_t b1) {
  const float f0 = __uint_as_float((b0 ^ 0x80u) | 0x4B000000u) - 8388736.0f;
  const float f1 = __uint_as_float((b1 ^ 0x80u) | 0x4B000000u) - 8388736.0f;
  return __byte_perm(__float_as_uint(f0), __float_as_uint(f1), 0x7632);
}

// Four int8 (one 32-bit word, k ascending) -> two bf16 pairs (k0,k1), (k2,k3), exactly (the
// same construction as i8x2_to_bf16x2, four bytes at a time).
__device__ __forceinline__ void i8x4_to_bf16x4(uint32_t w, uint32_t& lo, uint32_t& hi) {
  const uint32_t u = w ^ 0x80808080u;
  const float f0 = __uint_as_float(__byte_perm(u, 0x4B000000u, 0x7650)) - 8388736.0f;
  const float f1 = __uint_as_float(__byte_perm(u, 0x4B000000u, 0x7651)) - 8388736.0f;
  const float f2 = __uint_as_float(__byte_perm(u, 0x4B000000u, 0x7652)) - 8388736.0f;
  const float f3 = __uint_as_float(__byte_perm(u, 0x4B000000u, 0x7653)) - 8388736.0f;
  lo = __byte_perm(__float_as_uint(f0), __float_as_uint(f1), 0x7632);
  hi = __byte_perm(__float_as_uint(f2), __float_as_uint(f3), 0x7632);
}

// PACKED: weights K-contiguous ([E][n][k]), boxes of 64 k-bytes x 128 n-rows, 64-byte swizzle;
// otherwise the page's layout ([E][k][n]), boxes of 128 n-bytes x 64 k-rows, 128-byte swizzle.
template <bool DUAL, int ACT, bool PACKED, bool ASMEM>
__global__ void __launch_bounds__(kThreads, 1)
    grouped_gemm_w8t(const __grid_constant__ CUtensorMap tmX,
                     const __grid_constant__ CUtensorMap tmQ0,
                     const __grid_constant__ CUtensorMap tmQ1, const W8tParams p) {
  using C = W8tShape<ASMEM>;
  constexpr int kStages = C::kStages;
  constexpr int kAStages = C::kAStages;
  constexpr int kTmemCols = C::kTmemCols;
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  const uint32_t raw_addr = smem_u32(smem_raw);
  uint8_t* smem = smem_raw + ((1024u - (raw_addr & 1023u)) & 1023u);
  uint8_t* aring = smem + kStages * kStageBytes;  // converted weights (ASMEM)
  uint64_t* full = reinterpret_cast<uint64_t*>(aring + kAStages * C::kAStageBytes);
  uint64_t* empty = full + kStages;
  uint64_t* afull = empty + kStages;   // converted weights ready (converters -> MMA)
  uint64_t* aempty = afull + kAStages;  // weight stage read by the MMAs (MMA -> converters)
  uint64_t* tfull = aempty + kAStages;
  uint64_t* tempty = tfull + 2;
  uint64_t* drain = tempty + 2;
  uint32_t* s_tmem = reinterpret_cast<uint32_t*>(drain + 1);
  int* s_mstart = reinterpret_cast<int*>(s_tmem + 1);  // [E+1]
  int* s_seg = s_mstart + (kMaxE + 1);                 // [E+1]

  constexpr int NM = DUAL ? 2 : 1;  // weight matrices per k-block
  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const int n_blocks = (p.n_out + kNT - 1) / kNT;
  const int num_kb = (p.K + BK - 1) / BK;

  if (threadIdx.x == 0) {
    int acc = 0;
    for (int e = 0; e <= p.E; ++e) s_seg[e] = p.offsets[e];
    for (int e = 0; e < p.E; ++e) {
      s_mstart[e] = acc;
      acc += (s_seg[e + 1] - s_seg[e] + kRT - 1) / kRT;
    }
    s_mstart[p.E] = acc;
  }
  __syncthreads();
  const int m_total = s_mstart[p.E];
  const int total_tiles = m_total * n_blocks;
  if (static_cast<int>(blockIdx.x) >= total_tiles) return;  // uniform over the block
  const int group = min(kGroup, n_blocks);
  const int group_tiles = m_total * group;

  if (threadIdx.x == 0) {
    for (int s = 0; s < kStages; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], 1);
    }
    for (int a = 0; a < kAStages; ++a) {
      mbar_init(&afull[a], kConvWarps);
      mbar_init(&aempty[a], 1);
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(&tfull[b], 1);
      mbar_init(&tempty[b], 4);
    }
    mbar_init(drain, 1);
    fence_barrier_init();
    prefetch_tensormap(&tmX);
    prefetch_tensormap(&tmQ0);
    prefetch_tensormap(&tmQ1);
  }
  if (warp == 1) {
    tmem_alloc(s_tmem, kTmemCols);
    tmem_relinquish();
  }
  tc_fence_before_sync();
  __syncthreads();
  tc_fence_after_sync();
  const uint32_t tmem_base = *s_tmem;

  // tile -> (expert, row block of 64, column block of 128), column blocks in groups of kGroup
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

  if (warp == 0) {
    if (lane == 0) {  // ------------------------------------------------------ TMA producer
      int stage = 0;
      uint32_t phase = 0;
      bool ok = true;
      for (int tile = blockIdx.x; ok && tile < total_tiles; tile += gridDim.x) {
        int e, m_blk, n_blk;
        decode(tile, e, m_blk, n_blk);
        const int row0 = s_seg[e] + m_blk * kRT;
        const int n0 = n_blk * kNT;
        for (int kb = 0; kb < num_kb; ++kb) {
          if (!mbar_wait(&empty[stage], phase ^ 1u, p.timeout_ns)) {
            record_error(p.err, MOE_DEVERR_WAIT_TIMEOUT);
            ok = false;
            break;
          }
          uint8_t* st = smem + stage * kStageBytes;
          mbar_arrive_expect_tx(&full[stage], kXBytes + NM * kQBox);
          tma_load_2d(st, &tmX, &full[stage], kb * BK, row0);
          const int qc0 = PACKED ? kb * BK : n0;  // box coordinates (inner, rows)
          const int qc1 = PACKED ? n0 : kb * BK;
          tma_load_3d(st + kXBytes, &tmQ0, &full[stage], qc0, qc1, e);
          if (DUAL) tma_load_3d(st + kXBytes + kQBox, &tmQ1, &full[stage], qc0, qc1, e);
          if (++stage == kStages) {
            stage = 0;
            phase ^= 1u;
          }
        }
      }
    }
  } else if (warp >= 6) {  // ---------------------------------------------------- converters
    // Thread (quarter q, lane) holds output column n = 32 q + lane; this warp converts k-rows
    // [32 kh, 32 kh + 32) of each k-block. Byte (k, n) of a 128-byte-swizzled staging box sits
    // at k*128 + (((n >> 4) ^ (k & 7)) << 4) + (n & 15).
    const int q = warp & 3;
    const int kh = (warp - 6) >> 2;
    const int n = 32 * q + lane;
    const uint32_t t_lane = static_cast<uint32_t>(32 * q) << 16;
    int stage = 0, astage = 0;
    uint32_t phase = 0, aphase = 0;
    bool ok = true;
    for (int tile = blockIdx.x; ok && tile < total_tiles; tile += gridDim.x) {
      for (int kb = 0; kb < num_kb; ++kb) {
        ok = mbar_wait(&full[stage], phase, p.timeout_ns) &&
             mbar_wait(&aempty[astage], aphase ^ 1u, p.timeout_ns);
        if (__any_sync(0xffffffffu, !ok)) {
          if (lane == 0) record_error(p.err, MOE_DEVERR_WAIT_TIMEOUT);
          ok = false;
          break;
        }
        const uint8_t* qs = smem + stage * kStageBytes + kXBytes;
#pragma unroll
        for (int m = 0; m < NM; ++m) {
          uint32_t r[16];
          const uint8_t* box = qs + m * kQBox;
          if (PACKED) {
            // Row n holds the k-block's 64 weights of column n (64 bytes); 16-byte unit c of
            // row n sits at unit c ^ ((n >> 1) & 3). This warp's 32 k are units 2 kh, 2 kh + 1.
#pragma unroll
            for (int u = 0; u < 2; ++u) {
              const int c = 2 * kh + u;
              const uint4 w = *reinterpret_cast<const uint4*>(box + n * 64 +
                                                              ((c ^ ((n >> 1) & 3)) << 4));
              i8x4_to_bf16x4(w.x, r[8 * u + 0], r[8 * u + 1]);
              i8x4_to_bf16x4(w.y, r[8 * u + 2], r[8 * u + 3]);
              i8x4_to_bf16x4(w.z, r[8 * u + 4], r[8 * u + 5]);
              i8x4_to_bf16x4(w.w, r[8 * u + 6], r[8 * u + 7]);
            }
          } else {
#pragma unroll
            for (int j = 0; j < 16; ++j) {
              const int k = 32 * kh + 2 * j;
              const uint32_t b0 = box[k * 128 + ((((n >> 4) ^ (k & 7))) << 4) + (n & 15)];
              const uint32_t b1 =
                  box[(k + 1) * 128 + ((((n >> 4) ^ ((k + 1) & 7))) << 4) + (n & 15)];
              r[j] = i8x2_to_bf16x2(b0, b1);
            }
          }
          if (ASMEM) {
            // Row n of matrix m: 64 k as 128 bytes; this warp's 32 k are 16-byte chunks 4 kh ..
            // 4 kh + 3, chunk c stored at c ^ (n & 7) (the 128-byte swizzle).
            uint8_t* arow = aring + astage * C::kAStageBytes + m * kAMatBytes + n * 128;
#pragma unroll
            for (int j = 0; j < 4; ++j)
              *reinterpret_cast<uint4*>(arow + (((4 * kh + j) ^ (n & 7)) << 4)) =
                  make_uint4(r[4 * j], r[4 * j + 1], r[4 * j + 2], r[4 * j + 3]);
          } else {
            tmem_st_16cols(
                tmem_base + t_lane +
                    static_cast<uint32_t>(kAColBase + astage * kACols + m * 32 + kh * 16),
                r);
          }
        }
        if (ASMEM) {
          fence_proxy_async_smem();  // these generic-proxy writes -> the tensor core's reads
        } else {
          tmem_st_wait();
        }
        tc_fence_before_sync();
        __syncwarp();
        if (lane == 0) mbar_arrive(&afull[astage]);
        if (++stage == kStages) {
          stage = 0;
          phase ^= 1u;
        }
        if (++astage == kAStages) {
          astage = 0;
          aphase ^= 1u;
        }
      }
    }
  } else if (warp == 1) {
    if (lane == 0) {  // ---------------------------------------------------------- MMA issuer
      int stage = 0, astage = 0;
      uint32_t phase = 0, aphase = 0;
      bool ok = true;
      int it = 0;
      for (int tile = blockIdx.x; ok && tile < total_tiles; tile += gridDim.x, ++it) {
        const int acc = it & 1;
        const uint32_t acc_phase = static_cast<uint32_t>(it >> 1) & 1u;
        if (!mbar_wait(&tempty[acc], acc_phase ^ 1u, p.timeout_ns)) {
          record_error(p.err, MOE_DEVERR_WAIT_TIMEOUT);
          ok = false;
          break;
        }
        tc_fence_after_sync();
        int e, m_blk, n_blk;
        decode(tile, e, m_blk, n_blk);
        const int rows = min(kRT, s_seg[e + 1] - s_seg[e] - m_blk * kRT);
        const int nmma = max(16, (rows + 15) / 16 * 16);  // MMA N: the tile's rows, rounded up
        // kind::f16: D fp32, A bf16 (from TMEM), B bf16 K-major, N >> 3 at bit 17, M >> 4 at 24.
        const uint32_t idesc = (1u << 4) | (1u << 7) | (1u << 10) |
                               (static_cast<uint32_t>(nmma >> 3) << 17) |
                               (static_cast<uint32_t>(kNT >> 4) << 24);
        const uint32_t d_tmem = tmem_base + static_cast<uint32_t>(acc * kAccCols);
        for (int kb = 0; kb < num_kb; ++kb) {
          if (!mbar_wait(&full[stage], phase, p.timeout_ns) ||
              !mbar_wait(&afull[astage], aphase, p.timeout_ns)) {
            record_error(p.err, MOE_DEVERR_WAIT_TIMEOUT);
            ok = false;
            break;
          }
          tc_fence_after_sync();
          const uint32_t x_addr = smem_u32(smem + stage * kStageBytes);
          const uint32_t a_col = tmem_base + static_cast<uint32_t>(kAColBase + astage * kACols);
          const uint32_t a_addr = smem_u32(aring + astage * C::kAStageBytes);
#pragma unroll
          for (int kk = 0; kk < BK / UK; ++kk) {
            const uint64_t bd = smem_desc_sw128(x_addr + kk * 32, 16, 1024);
#pragma unroll
            for (int m = 0; m < NM; ++m) {
              if (ASMEM)
                umma_bf16_ss(d_tmem + static_cast<uint32_t>(m * kRT),
                             smem_desc_sw128(a_addr + m * kAMatBytes + kk * 32, 16, 1024), bd,
                             idesc, (kb | kk) != 0 ? 1u : 0u);
              else
                umma_bf16_ts(d_tmem + static_cast<uint32_t>(m * kRT),
                             a_col + static_cast<uint32_t>(m * 32 + kk * 8), bd, idesc,
                             (kb | kk) != 0 ? 1u : 0u);
            }
          }
          umma_commit(&empty[stage]);    // token rows and int8 stage free,
          umma_commit(&aempty[astage]);  // converted weights free, once these MMAs are done
          if (++stage == kStages) {
            stage = 0;
            phase ^= 1u;
          }
          if (++astage == kAStages) {
            astage = 0;
            aphase ^= 1u;
          }
        }
        if (ok) umma_commit(&tfull[acc]);
      }
      umma_commit(drain);
      if (!mbar_wait(drain, 0, p.timeout_ns)) record_error(p.err, MOE_DEVERR_WAIT_TIMEOUT);
    }
  } else if (warp >= 2) {  // ----------------------------------------------------- epilogue
    // This thread's TMEM lane is output column n0 + 32 q + lane; accumulator column r is token
    // row r of the tile.
    const int q = warp & 3;
    int it = 0;
    for (int tile = blockIdx.x; tile < total_tiles; tile += gridDim.x, ++it) {
      const int acc = it & 1;
      const uint32_t acc_phase = static_cast<uint32_t>(it >> 1) & 1u;
      const bool ok = mbar_wait_suspend(&tfull[acc], acc_phase, p.timeout_ns);
      if (__any_sync(0xffffffffu, !ok)) {
        if (lane == 0) record_error(p.err, MOE_DEVERR_WAIT_TIMEOUT);
        break;
      }
      __syncwarp();
      tc_fence_after_sync();
      int e, m_blk, n_blk;
      decode(tile, e, m_blk, n_blk);
      const int rows = min(kRT, s_seg[e + 1] - s_seg[e] - m_blk * kRT);
      const int col = n_blk * kNT + 32 * q + lane;
      const bool valid = col < p.n_out;
      const float sc0 = valid ? __ldg(p.s0 + static_cast<int64_t>(e) * p.n_out + col) : 0.f;
      const float sc1 =
          (DUAL && valid) ? __ldg(p.s1 + static_cast<int64_t>(e) * p.n_out + col) : 0.f;
      __nv_bfloat16* ocol =
          p.out + (static_cast<int64_t>(s_seg[e]) + m_blk * kRT) * p.n_out + col;
      const uint32_t t_row = tmem_base + (static_cast<uint32_t>(32 * q) << 16) +
                             static_cast<uint32_t>(acc * kAccCols);
#pragma unroll 1
      for (int c = 0; c * 16 < rows; ++c) {  // 16 token rows per chunk
        uint32_t ra[16], rb[16];
        tmem_ld_16cols(t_row + c * 16, ra);
        if (DUAL) tmem_ld_16cols(t_row + kRT + c * 16, rb);
        tmem_ld_wait();
        if (valid) {
#pragma unroll
          for (int i = 0; i < 16; ++i) {
            const int r = c * 16 + i;
            if (r < rows) {
              const float a = __uint_as_float(ra[i]) * sc0;
              const float h = DUAL ? activation<ACT>(a) * (__uint_as_float(rb[i]) * sc1) : a;
              ocol[static_cast<int64_t>(r) * p.n_out] = __float2bfloat16_rn(h);
            }
          }
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

template <bool DUAL, int ACT, bool PACKED, bool ASMEM>
cudaError_t launch_w8t_shape(const CUtensorMap& x, const CUtensorMap& q0, const CUtensorMap& q1,
                             const W8tParams& wp, int64_t tiles_upper, cudaStream_t stream) {
  auto kern = grouped_gemm_w8t<DUAL, ACT, PACKED, ASMEM>;
  constexpr int smem = W8tShape<ASMEM>::kSmemBytes;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
  if (e != cudaSuccess) return e;
  const int grid = static_cast<int>(std::max<int64_t>(1, std::min<int64_t>(num_sms(), tiles_upper)));
  kern<<<grid, kThreads, smem, stream>>>(x, q0, q1, wp);
  return cudaGetLastError();
}

// Where the converted weights go: tensor memory (the default; measured faster on the decode
// layer, 308 against 329 us for the up-projection) or shared memory. MOE_W8T_A=smem|tmem
// overrides.
bool w8t_a_in_smem() {
  if (const char* env = std::getenv("MOE_W8T_A")) {
    if (std::strcmp(env, "tmem") == 0) return false;
    if (std::strcmp(env, "smem") == 0) return true;
  }
  return false;
}

template <bool DUAL, int ACT, bool PACKED>
cudaError_t launch_w8t(const CUtensorMap& x, const CUtensorMap& q0, const CUtensorMap& q1,
                       const W8tParams& wp, int64_t tiles_upper, cudaStream_t stream) {
  return w8t_a_in_smem()
             ? launch_w8t_shape<DUAL, ACT, PACKED, true>(x, q0, q1, wp, tiles_upper, stream)
             : launch_w8t_shape<DUAL, ACT, PACKED, false>(x, q0, q1, wp, tiles_upper, stream);
}

}  // namespace

// Weight boxes: the page's layout [E][K][n_out] -> 128 n x 64 k (128-byte swizzle); packed
// [E][n_out][K] -> 64 k x 128 n (64-byte swizzle).
bool make_weight_map(CUtensorMap* m, const int8_t* q, int64_t K, int64_t n_out, int64_t E,
                     bool packed) {
  return packed ? make_tensor_map_3d_u8_sw64(m, q, K, n_out, E, BK, kNT)
                : make_tensor_map_3d_u8(m, q, n_out, K, E, kNT, BK);
}

cudaError_t launch_ffn_up_w8t(const moe_problem& p, const void* X_perm, const int32_t* offsets,
                              const int8_t* W1q, const float* S1, const int8_t* W2q,
                              const float* S2, void* H, bool packed, int* err,
                              uint64_t timeout_ns, cudaStream_t stream) {
  const int64_t R = p.N * p.k;
  if (R == 0) return cudaSuccess;
  CUtensorMap tX, tQ1, tQ2;
  if (!make_tensor_map_2d_bf16(&tX, X_perm, p.D, R, 64, kRT) ||
      !make_weight_map(&tQ1, W1q, p.D, p.F, p.E, packed) ||
      !make_weight_map(&tQ2, W2q, p.D, p.F, p.E, packed))
    return cudaErrorInvalidValue;
  W8tParams w;
  w.offsets = offsets;
  w.s0 = S1;
  w.s1 = S2;
  w.out = static_cast<__nv_bfloat16*>(H);
  w.E = p.E;
  w.K = static_cast<int>(p.D);
  w.n_out = static_cast<int>(p.F);
  w.err = err;
  w.timeout_ns = timeout_ns;
  const int64_t tiles = ((R + kRT - 1) / kRT + p.E) * ((p.F + kNT - 1) / kNT);
#define MOE_W8T_UP(ACT_)                                                                   \
  return packed ? launch_w8t<true, ACT_, true>(tX, tQ1, tQ2, w, tiles, stream)             \
                : launch_w8t<true, ACT_, false>(tX, tQ1, tQ2, w, tiles, stream)
  switch (p.activation) {
    case MOE_ACT_SILU:
      MOE_W8T_UP(MOE_ACT_SILU);
    case MOE_ACT_GELU_ERF:
      MOE_W8T_UP(MOE_ACT_GELU_ERF);
    default:
      MOE_W8T_UP(MOE_ACT_GELU_TANH);
  }
#undef MOE_W8T_UP
}

cudaError_t launch_ffn_down_w8t(const moe_problem& p, const void* H, const int32_t* offsets,
                                const int8_t* W3q, const float* S3, void* Y, bool packed,
                                int* err, uint64_t timeout_ns, cudaStream_t stream) {
  const int64_t R = p.N * p.k;
  if (R == 0) return cudaSuccess;
  CUtensorMap tX, tQ3;
  if (!make_tensor_map_2d_bf16(&tX, H, p.F, R, 64, kRT) ||
      !make_weight_map(&tQ3, W3q, p.F, p.D, p.E, packed))
    return cudaErrorInvalidValue;
  W8tParams w;
  w.offsets = offsets;
  w.s0 = S3;
  w.s1 = nullptr;
  w.out = static_cast<__nv_bfloat16*>(Y);
  w.E = p.E;
  w.K = static_cast<int>(p.F);
  w.n_out = static_cast<int>(p.D);
  w.err = err;
  w.timeout_ns = timeout_ns;
  const int64_t tiles = ((R + kRT - 1) / kRT + p.E) * ((p.D + kNT - 1) / kNT);
  return packed ? launch_w8t<false, MOE_ACT_SILU, true>(tX, tQ3, tQ3, w, tiles, stream)
                : launch_w8t<false, MOE_ACT_SILU, false>(tX, tQ3, tQ3, w, tiles, stream);
}

namespace {

// dst[e][j][i] = src[e][i][j] for an [E][k][n] byte tensor: 32x32 tiles through shared memory.
__global__ void __launch_bounds__(256)
    pack_w8_kernel(const int8_t* __restrict__ src, int8_t* __restrict__ dst, int64_t k, int64_t n) {
  __shared__ int8_t tile[32][33];
  const int64_t e = blockIdx.z;
  const int64_t i0 = static_cast<int64_t>(blockIdx.y) * 32;  // k
  const int64_t j0 = static_cast<int64_t>(blockIdx.x) * 32;  // n
  const int tx = threadIdx.x & 31, ty = threadIdx.x >> 5;    // 32 x 8 threads
  const int8_t* s = src + e * k * n;
  int8_t* d = dst + e * k * n;
  for (int r = ty; r < 32; r += 8)
    if (i0 + r < k && j0 + tx < n) tile[r][tx] = s[(i0 + r) * n + j0 + tx];
  __syncthreads();
  for (int r = ty; r < 32; r += 8)
    if (j0 + r < n && i0 + tx < k) d[(j0 + r) * k + i0 + tx] = tile[tx][r];
}

}  // namespace

cudaError_t launch_pack_w8(const int8_t* src, int8_t* dst, int64_t E, int64_t k, int64_t n,
                           cudaStream_t stream) {
  if (E == 0 || k == 0 || n == 0) return cudaSuccess;
  const dim3 grid(static_cast<unsigned>((n + 31) / 32), static_cast<unsigned>((k + 31) / 32),
                  static_cast<unsigned>(E));
  pack_w8_kernel<<<grid, 256, 0, stream>>>(src, dst, k, n);
  return cudaGetLastError();
}

}  // namespace moe

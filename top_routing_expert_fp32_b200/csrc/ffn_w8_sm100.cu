// Grouped gated expert FFN with 8-bit expert weights on the tcgen05 tensor cores (sm_100a).
//   GEMM1: H[r] = act(X_perm[r] W1_e) (.) (X_perm[r] W2_e)      GEMM2: Y[r] = H[r] W3_e
// with W = q * s, q int8 and s one fp32 scale per expert and output column. The Grok-1 book
// (ch.5, 5.3.3 and 5.3.5) dequantizes before each expert matmul ("weight = weight * scales");
// with the scale shared by a whole output column it commutes with the contraction:
//   x . (q[:, n] * s[n]) = s[n] * (x . q[:, n]),
// so the tensor cores multiply bf16 activations by q converted exactly to bf16 (|q| <= 128
// needs 8 significant bits) and the epilogue applies s[n] in fp32. The weights cross HBM as
// int8: half the bytes of the bf16 layer, which is what bounds small (decode-sized) batches.
//
// Design (one persistent CTA per SM, 18 warps, 128-row tiles; an expert's last row block of
// at most 64 rows uses M = 64 MMAs and a 64-row A box):
//   warp 0        : TMA producers. Lane 0: per k-block one bf16 A box (128 or 64 rows,
//                   K-major, 128-byte swizzle) into a 4-stage ring that the MMA frees. Lane 1:
//                   two 64x128 int8 B boxes (128-byte swizzle) into a 6-stage ring that the
//                   converters free as soon as they have read it, so the weight stream runs
//                   ahead of the MMA (what keeps HBM busy when the layer is bound by it).
//   warps 6..17   : converters. int8 -> bf16 into one of two 32 KB buffers in the MN-major
//                   128-byte-swizzled layout the MMA reads (four 64-column boxes), then an
//                   async-proxy fence and an arrival. Each 8-lane phase of a 16-byte store hits
//                   8 distinct 16-byte units (no bank conflicts): shared-memory bandwidth
//                   (TMA writes, converter reads and writes, MMA reads) bounds this kernel.
//   warp 1        : TMEM allocation (512 columns, two 128x256 fp32 accumulators); lane 0
//                   issues tcgen05.mma once a converted buffer is ready, and its completion
//                   frees both the stage and the buffer.
//   warps 2..5    : epilogue: tcgen05.ld (16 columns at a time), scale, (act and product),
//                   bf16, masked stores; double-buffered against the next tile's main loop.
// Tiles are enumerated as in the bf16 grouped GEMM (column blocks in groups of 8, experts,
// column block, row blocks innermost). Every barrier wait is bounded in time; on a timeout the
// CTA records MOE_DEVERR_WAIT_TIMEOUT, unwinds, drains its MMAs and frees its TMEM.
#include <algorithm>
#include <cmath>

#include "common.cuh"
#include "internal.h"

namespace moe {
namespace {

constexpr int kRows = 128;
constexpr int BN = 256;                      // MMA N
constexpr int BK = 64;
constexpr int UK = 16;
constexpr int kABytes = kRows * BK * 2;      // 16 KB
constexpr int kB8Box = 64 * 128;             // 8 KB: 64 k-rows x 128 int8 columns
constexpr int kB8Bytes = 2 * kB8Box;         // 16 KB
constexpr int kA64Bytes = 64 * BK * 2;       // 8 KB: the A box of an M = 64 tile
constexpr int kB16Box = 64 * 64 * 2;         // 8 KB: 64 k-rows x 64 bf16 columns
constexpr int kB16Bytes = 4 * kB16Box;       // 32 KB
constexpr int kAStages = 4;                  // A ring: freed by the MMA
constexpr int kBStages = 6;                  // int8 ring: freed as soon as converted
constexpr int kB16Bufs = 2;                  // converted B buffers
constexpr int kThreads = 576;
constexpr int kConvThreads = 384;            // warps 6..17
constexpr int kTmemCols = 512;
constexpr int kAccCols = 256;
constexpr int kMaxE = 64;
constexpr int kGroup = 8;                    // column blocks per tile group
constexpr int kSmemBytes = kAStages * kABytes + kBStages * kB8Bytes + kB16Bufs * kB16Bytes +
                           1024 /*align*/ + 1024 /*barriers*/;

constexpr uint32_t kIdesc = (1u << 4) | (1u << 7) | (1u << 10) | (1u << 16) |
                            (static_cast<uint32_t>(BN >> 3) << 17) |
                            (static_cast<uint32_t>(kRows >> 4) << 24);
constexpr uint32_t kIdesc64 = (1u << 4) | (1u << 7) | (1u << 10) | (1u << 16) |
                              (static_cast<uint32_t>(BN >> 3) << 17) |
                              (static_cast<uint32_t>(64 >> 4) << 24);

struct W8Params {
  const int32_t* offsets;  // [E+1]
  const float* s0;         // scales of the first B (W1 or W3): [E][n_out]
  const float* s1;         // scales of the second B (W2), GEMM1 only
  __nv_bfloat16* out;      // [rows, n_out]
  int E;
  int K;
  int n_out;
  int* err;
  uint64_t timeout_ns;
};

// Four int8 (one 32-bit word) -> four bf16 (two 32-bit words), exactly. Each byte, biased to
// u = q + 128, becomes the low mantissa byte of the float 2^23 + u; subtracting 2^23 + 128
// leaves q as a float whose upper 16 bits are its bf16 encoding (q has at most 8 significant
// bits, so nothing is rounded).
__device__ __forceinline__ void i8x4_to_bf16x4(uint32_t w, uint32_t& lo, uint32_t& hi) {
  const uint32_t u = w ^ 0x80808080u;
  const float f0 = __uint_as_float(__byte_perm(u, 0x4B000000u, 0x7650)) - 8388736.0f;
  const float f1 = __uint_as_float(__byte_perm(u, 0x4B000000u, 0x7651)) - 8388736.0f;
  const float f2 = __uint_as_float(__byte_perm(u, 0x4B000000u, 0x7652)) - 8388736.0f;
  const float f3 = __uint_as_float(__byte_perm(u, 0x4B000000u, 0x7653)) - 8388736.0f;
  lo = __byte_perm(__float_as_uint(f0), __float_as_uint(f1), 0x7632);
  hi = __byte_perm(__float_as_uint(f2), __float_as_uint(f3), 0x7632);
}

template <bool DUAL, int ACT>
__global__ void __launch_bounds__(kThreads, 1)
    grouped_gemm_w8(const __grid_constant__ CUtensorMap tmA,
                    const __grid_constant__ CUtensorMap tmA64,
                    const __grid_constant__ CUtensorMap tmB0,
                    const __grid_constant__ CUtensorMap tmB1, const W8Params p) {
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  const uint32_t raw_addr = smem_u32(smem_raw);
  uint8_t* smem = smem_raw + ((1024u - (raw_addr & 1023u)) & 1023u);
  uint8_t* a_base = smem;
  uint8_t* b8_base = a_base + kAStages * kABytes;
  uint8_t* b16_base = b8_base + kBStages * kB8Bytes;
  uint64_t* afull = reinterpret_cast<uint64_t*>(b16_base + kB16Bufs * kB16Bytes);
  uint64_t* aempty = afull + kAStages;
  uint64_t* bfull = aempty + kAStages;  // int8 stage landed (TMA -> converters)
  uint64_t* bempty = bfull + kBStages;  // int8 stage read (converters -> producer)
  uint64_t* cfull = bempty + kBStages;  // converted buffer ready (converters -> MMA)
  uint64_t* cempty = cfull + kB16Bufs;  // converted buffer consumed (MMA -> converters)
  uint64_t* tfull = cempty + kB16Bufs;
  uint64_t* tempty = tfull + 2;
  uint64_t* drain = tempty + 2;
  uint32_t* s_tmem = reinterpret_cast<uint32_t*>(drain + 1);
  int* s_mstart = reinterpret_cast<int*>(s_tmem + 1);  // [E+1]
  int* s_seg = s_mstart + (kMaxE + 1);                 // [E+1]

  constexpr int NT = DUAL ? 128 : 256;  // output columns per tile
  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const int n_blocks = (p.n_out + NT - 1) / NT;
  const int num_kb = (p.K + BK - 1) / BK;

  if (threadIdx.x == 0) {
    int acc = 0;
    for (int e = 0; e <= p.E; ++e) s_seg[e] = p.offsets[e];
    for (int e = 0; e < p.E; ++e) {
      s_mstart[e] = acc;
      acc += (s_seg[e + 1] - s_seg[e] + kRows - 1) / kRows;
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
    for (int s = 0; s < kAStages; ++s) {
      mbar_init(&afull[s], 1);
      mbar_init(&aempty[s], 1);
    }
    for (int s = 0; s < kBStages; ++s) {
      mbar_init(&bfull[s], 1);
      mbar_init(&bempty[s], kConvThreads / 32);
    }
    for (int b = 0; b < kB16Bufs; ++b) {
      mbar_init(&cfull[b], kConvThreads / 32);
      mbar_init(&cempty[b], 1);
    }
    for (int a = 0; a < 2; ++a) {
      mbar_init(&tfull[a], 1);
      mbar_init(&tempty[a], 4);
    }
    mbar_init(drain, 1);
    fence_barrier_init();
    prefetch_tensormap(&tmA);
    prefetch_tensormap(&tmA64);
    prefetch_tensormap(&tmB0);
    prefetch_tensormap(&tmB1);
  }
  if (warp == 1) {
    tmem_alloc(s_tmem, kTmemCols);
    tmem_relinquish();
  }
  tc_fence_before_sync();
  __syncthreads();
  tc_fence_after_sync();
  const uint32_t tmem_base = *s_tmem;

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
    // Lane 0 streams the A tiles, lane 1 the int8 weights: the weights run ahead of the MMA by
    // up to kBStages k-blocks, bounded only by the converters.
    if (lane < 2) {  // ---------------------------------------------------- TMA producers
      const bool weights = lane == 1;
      const int nst = weights ? kBStages : kAStages;
      uint64_t* emptyb = weights ? bempty : aempty;
      int stage = 0;
      uint32_t phase = 0;
      bool ok = true;
      for (int tile = blockIdx.x; ok && tile < total_tiles; tile += gridDim.x) {
        int e, m_blk, n_blk;
        decode(tile, e, m_blk, n_blk);
        const int row0 = s_seg[e] + m_blk * kRows;
        const bool rows64 = s_seg[e + 1] - row0 <= 64;  // M = 64 tile: load only its rows
        const int n0 = n_blk * NT;
        for (int kb = 0; kb < num_kb; ++kb) {
          if (!mbar_wait(&emptyb[stage], phase ^ 1u, p.timeout_ns)) {
            record_error(p.err, MOE_DEVERR_WAIT_TIMEOUT);
            ok = false;
            break;
          }
          if (!weights) {
            uint8_t* st = a_base + stage * kABytes;
            mbar_arrive_expect_tx(&afull[stage], rows64 ? kA64Bytes : kABytes);
            tma_load_2d(st, rows64 ? &tmA64 : &tmA, &afull[stage], kb * BK, row0);
          } else {
            uint8_t* st = b8_base + stage * kB8Bytes;
            mbar_arrive_expect_tx(&bfull[stage], kB8Bytes);
            if (DUAL) {  // W1 and W2 columns [n0, n0 + 128)
              tma_load_3d(st, &tmB0, &bfull[stage], n0, kb * BK, e);
              tma_load_3d(st + kB8Box, &tmB1, &bfull[stage], n0, kb * BK, e);
            } else {     // W3 columns [n0, n0 + 256)
              tma_load_3d(st, &tmB0, &bfull[stage], n0, kb * BK, e);
              tma_load_3d(st + kB8Box, &tmB0, &bfull[stage], n0 + 128, kb * BK, e);
            }
          }
          if (++stage == nst) {
            stage = 0;
            phase ^= 1u;
          }
        }
      }
    }
  } else if (warp >= 6) {  // ---------------------------------------------------- converters
    // Item (staging box sb, k-row, 16-byte unit c16): 16 int8 at columns 16*c16 .. +16 of the
    // staging row become 16 bf16, the units 2*(c16 & 3) and +1 of row k in bf16 box
    // 2*sb + (c16 >> 2). Both layouts use the 128-byte swizzle: the 16-byte unit c of row k
    // sits at unit c ^ (k & 7).
    const int ct = threadIdx.x - 192;
    // This thread converts the same three pieces of every k-block: offsets computed once.
    constexpr int kPieces = 3;  // ceil(1024 / kConvThreads)
    int src_off[kPieces], dst_off0[kPieces], dst_off1[kPieces];
    bool hi_first[kPieces], has[kPieces];
#pragma unroll
    for (int u = 0; u < kPieces; ++u) {
      const int i = ct + u * kConvThreads;
      has[u] = i < 1024;
      const int sb = (i >> 9) & 1;
      const int k = (i >> 3) & 63;
      const int c16 = i & 7;
      const int sw = k & 7;
      src_off[u] = sb * kB8Box + k * 128 + ((c16 ^ sw) << 4);
      const int dst = (2 * sb + (c16 >> 2)) * kB16Box + k * 128;
      const int cb = 2 * (c16 & 3);
      // Lanes of the upper box store their odd unit first, so that in each 8-lane phase (one
      // row, both boxes) the two boxes' units have opposite parity.
      hi_first[u] = (c16 >> 2) != 0;
      dst_off0[u] = dst + (((hi_first[u] ? cb + 1 : cb) ^ sw) << 4);
      dst_off1[u] = dst + (((hi_first[u] ? cb : cb + 1) ^ sw) << 4);
    }
    int stage = 0, buf = 0;
    uint32_t phase = 0, bphase = 0;
    bool ok = true;
    for (int tile = blockIdx.x; ok && tile < total_tiles; tile += gridDim.x) {
      for (int kb = 0; kb < num_kb; ++kb) {
        ok = mbar_wait_suspend(&bfull[stage], phase, p.timeout_ns) &&
             mbar_wait_suspend(&cempty[buf], bphase ^ 1u, p.timeout_ns);
        if (__any_sync(0xffffffffu, !ok)) {
          if (lane == 0) record_error(p.err, MOE_DEVERR_WAIT_TIMEOUT);
          ok = false;
          break;
        }
        const uint8_t* b8 = b8_base + stage * kB8Bytes;
        uint8_t* b16 = b16_base + buf * kB16Bytes;
#pragma unroll
        for (int u = 0; u < kPieces; ++u) {
          if (has[u]) {
            const uint4 w = *reinterpret_cast<const uint4*>(b8 + src_off[u]);
            uint4 v0, v1;
            i8x4_to_bf16x4(w.x, v0.x, v0.y);
            i8x4_to_bf16x4(w.y, v0.z, v0.w);
            i8x4_to_bf16x4(w.z, v1.x, v1.y);
            i8x4_to_bf16x4(w.w, v1.z, v1.w);
            *reinterpret_cast<uint4*>(b16 + dst_off0[u]) = hi_first[u] ? v1 : v0;
            *reinterpret_cast<uint4*>(b16 + dst_off1[u]) = hi_first[u] ? v0 : v1;
          }
        }
        fence_proxy_async_smem();  // these generic-proxy writes -> the tensor core's reads
        __syncwarp();
        if (lane == 0) {
          mbar_arrive(&bempty[stage]);  // this warp's reads of the int8 stage are done
          mbar_arrive(&cfull[buf]);
        }
        if (++stage == kBStages) {
          stage = 0;
          phase ^= 1u;
        }
        if (++buf == kB16Bufs) {
          buf = 0;
          bphase ^= 1u;
        }
      }
    }
  } else if (warp == 1) {
    if (lane == 0) {  // ---------------------------------------------------------- MMA issuer
      int stage = 0, buf = 0;
      uint32_t phase = 0, bphase = 0;
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
        const uint32_t d_tmem = tmem_base + static_cast<uint32_t>(acc * kAccCols);
        int e, m_blk, n_blk;
        decode(tile, e, m_blk, n_blk);
        const uint32_t idesc = (s_seg[e + 1] - s_seg[e] - m_blk * kRows <= 64) ? kIdesc64 : kIdesc;
        for (int kb = 0; kb < num_kb; ++kb) {
          if (!mbar_wait(&afull[stage], phase, p.timeout_ns) ||
              !mbar_wait(&cfull[buf], bphase, p.timeout_ns)) {
            record_error(p.err, MOE_DEVERR_WAIT_TIMEOUT);
            ok = false;
            break;
          }
          tc_fence_after_sync();
          const uint32_t a_addr = smem_u32(a_base + stage * kABytes);
          const uint32_t b_addr = smem_u32(b16_base + buf * kB16Bytes);
#pragma unroll
          for (int kk = 0; kk < BK / UK; ++kk) {
            const uint64_t ad = smem_desc_sw128(a_addr + kk * 32, 16, 1024);
            const uint64_t bd = smem_desc_sw128(b_addr + kk * 2048, kB16Box, 1024);
            umma_bf16_ss(d_tmem, ad, bd, idesc, (kb | kk) != 0 ? 1u : 0u);
          }
          umma_commit(&aempty[stage]);  // A stage and converted buffer both free once these
          umma_commit(&cempty[buf]);    // MMAs have read them
          if (++stage == kAStages) {
            stage = 0;
            phase ^= 1u;
          }
          if (++buf == kB16Bufs) {
            buf = 0;
            bphase ^= 1u;
          }
        }
        if (ok) umma_commit(&tfull[acc]);
      }
      umma_commit(drain);
      if (!mbar_wait(drain, 0, p.timeout_ns)) record_error(p.err, MOE_DEVERR_WAIT_TIMEOUT);
    }
  } else if (warp >= 2) {  // ----------------------------------------------------- epilogue
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
      const int first_row = m_blk * kRows;
      const int rows = min(kRows, s_seg[e + 1] - s_seg[e] - first_row);
      const bool half = rows <= 64;  // M = 64: row 16q + l sits in TMEM lane 32q + l
      const int r = half ? (lane < 16 ? 16 * q + lane : kRows) : q * 32 + lane;
      const bool valid = r < rows;
      const int64_t grow = static_cast<int64_t>(s_seg[e]) + first_row + r;
      const int n0 = n_blk * NT;
      __nv_bfloat16* orow = p.out + grow * p.n_out + n0;
      const float* sc0 = p.s0 + static_cast<int64_t>(e) * p.n_out + n0;
      const float* sc1 = DUAL ? p.s1 + static_cast<int64_t>(e) * p.n_out + n0 : nullptr;
      const uint32_t t_row =
          tmem_base + (static_cast<uint32_t>(q * 32) << 16) + static_cast<uint32_t>(acc * kAccCols);
      constexpr int kChunks = DUAL ? 8 : 16;  // 16 output columns each
#pragma unroll 1
      for (int c = 0; c < kChunks; ++c) {
        uint32_t ra[16], rb[16];
        tmem_ld_16cols(t_row + c * 16, ra);
        if (DUAL) tmem_ld_16cols(t_row + 128 + c * 16, rb);
        tmem_ld_wait();
        if (valid) {
          uint32_t w[8];
#pragma unroll
          for (int i = 0; i < 8; ++i) {
            float h[2];
#pragma unroll
            for (int h2 = 0; h2 < 2; ++h2) {
              const int col = c * 16 + 2 * i + h2;
              const bool in = n0 + col < p.n_out;
              const float s0 = in ? __ldg(sc0 + col) : 0.f;
              const float a = __uint_as_float(ra[2 * i + h2]) * s0;
              if (DUAL) {
                const float s1 = in ? __ldg(sc1 + col) : 0.f;
                h[h2] = activation<ACT>(a) * (__uint_as_float(rb[2 * i + h2]) * s1);
              } else {
                h[h2] = a;
              }
            }
            w[i] = pack_bf16x2(h[0], h[1]);
          }
#pragma unroll
          for (int v = 0; v < 2; ++v)
            if (n0 + c * 16 + v * 8 < p.n_out)
              reinterpret_cast<uint4*>(orow + c * 16)[v] =
                  make_uint4(w[4 * v], w[4 * v + 1], w[4 * v + 2], w[4 * v + 3]);
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

template <bool DUAL, int ACT>
cudaError_t launch_w8(const CUtensorMap& a, const CUtensorMap& a64, const CUtensorMap& b0,
                      const CUtensorMap& b1, const W8Params& wp, int64_t tiles_upper,
                      cudaStream_t stream) {
  auto kern = grouped_gemm_w8<DUAL, ACT>;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, kSmemBytes);
  if (e != cudaSuccess) return e;
  const int grid = static_cast<int>(std::max<int64_t>(1, std::min<int64_t>(num_sms(), tiles_upper)));
  kern<<<grid, kThreads, kSmemBytes, stream>>>(a, a64, b0, b1, wp);
  return cudaGetLastError();
}

}  // namespace

cudaError_t launch_ffn_up_w8(const moe_problem& p, const void* X_perm, const int32_t* offsets,
                             const int8_t* W1q, const float* S1, const int8_t* W2q,
                             const float* S2, void* H, int* err, uint64_t timeout_ns,
                             cudaStream_t stream) {
  const int64_t R = p.N * p.k;
  if (R == 0) return cudaSuccess;
  CUtensorMap tA, tA64, tW1, tW2;
  if (!make_tensor_map_2d_bf16(&tA, X_perm, p.D, R, 64, kRows) ||
      !make_tensor_map_2d_bf16(&tA64, X_perm, p.D, R, 64, 64) ||
      !make_tensor_map_3d_u8(&tW1, W1q, p.F, p.D, p.E, 128, 64) ||
      !make_tensor_map_3d_u8(&tW2, W2q, p.F, p.D, p.E, 128, 64))
    return cudaErrorInvalidValue;
  W8Params w;
  w.offsets = offsets;
  w.s0 = S1;
  w.s1 = S2;
  w.out = static_cast<__nv_bfloat16*>(H);
  w.E = p.E;
  w.K = static_cast<int>(p.D);
  w.n_out = static_cast<int>(p.F);
  w.err = err;
  w.timeout_ns = timeout_ns;
  const int64_t tiles = ((R + kRows - 1) / kRows + p.E) * ((p.F + 127) / 128);
  switch (p.activation) {
    case MOE_ACT_SILU:
      return launch_w8<true, MOE_ACT_SILU>(tA, tA64, tW1, tW2, w, tiles, stream);
    case MOE_ACT_GELU_ERF:
      return launch_w8<true, MOE_ACT_GELU_ERF>(tA, tA64, tW1, tW2, w, tiles, stream);
    default:
      return launch_w8<true, MOE_ACT_GELU_TANH>(tA, tA64, tW1, tW2, w, tiles, stream);
  }
}

cudaError_t launch_ffn_down_w8(const moe_problem& p, const void* H, const int32_t* offsets,
                               const int8_t* W3q, const float* S3, void* Y, int* err,
                               uint64_t timeout_ns, cudaStream_t stream) {
  const int64_t R = p.N * p.k;
  if (R == 0) return cudaSuccess;
  CUtensorMap tA, tA64, tW3;
  if (!make_tensor_map_2d_bf16(&tA, H, p.F, R, 64, kRows) ||
      !make_tensor_map_2d_bf16(&tA64, H, p.F, R, 64, 64) ||
      !make_tensor_map_3d_u8(&tW3, W3q, p.D, p.F, p.E, 128, 64))
    return cudaErrorInvalidValue;
  W8Params w;
  w.offsets = offsets;
  w.s0 = S3;
  w.s1 = nullptr;
  w.out = static_cast<__nv_bfloat16*>(Y);
  w.E = p.E;
  w.K = static_cast<int>(p.F);
  w.n_out = static_cast<int>(p.D);
  w.err = err;
  w.timeout_ns = timeout_ns;
  const int64_t tiles = ((R + kRows - 1) / kRows + p.E) * ((p.D + 255) / 256);
  return launch_w8<false, MOE_ACT_SILU>(tA, tA64, tW3, tW3, w, tiles, stream);
}

}  // namespace moe

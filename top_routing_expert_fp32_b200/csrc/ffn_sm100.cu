// Grouped gated expert FFN on the 5th-generation tensor cores (tcgen05, sm_100a).
//   GEMM1: H[r] = act(X_perm[r] W1_e) (.) (X_perm[r] W2_e)     (act and product fused)
//   GEMM2: Y[r] = H[r] W3_e
// for every row r of expert e's segment [offsets[e], offsets[e+1]) -- LLMs-from-scratch
// ch.12, 12.1 (f_e(x) = [SiLU(x W1_e) (.) (x W2_e)] W3_e); Grok-1 book ch.5, 5.3.5 (GeGLU
// variant, x W_value times GELU(x W_gate)) and 5.3.2 (weights stacked [E, D, F] / [E, F, D]).
//
// Design (one persistent CTA per SM, 6 warps):
//   warp 0 lane 0 : TMA producer. Per k-block of 64: one 128x64 A box (X_perm or H rows,
//                   K-major, 128-byte swizzle) and four 64x64 B boxes from the 3-D weight
//                   tensor [E][K][N] (N contiguous = MN-major B, 128-byte swizzle). GEMM1 takes
//                   two boxes from W1 and two from W2 for the same 128 output columns, so one
//                   N=256 MMA produces both up-projections side by side.
//   warp 1        : allocates 512 TMEM columns (two 128x256 fp32 accumulators); lane 0 issues
//                   tcgen05.mma (M=128, N=256, K=16, bf16 -> fp32) and commits to barriers.
//   warps 2..5    : epilogue. tcgen05.ld of the accumulator rows (one row per thread), act in
//                   fp32, bf16 rounding, masked 16-byte stores (rows past the expert's segment
//                   are never written). The accumulator is double buffered, so the epilogue
//                   of tile i overlaps the main loop of tile i+1.
// Tiles: per expert ceil(M_e/128) row blocks x ceil(N/NT) column blocks, enumerated expert by
// expert with row blocks innermost (consecutive CTAs share a weight column block through L2).
// Per-expert row counts are read from device memory: the host never learns them.
// Every barrier wait is bounded in time; on a timeout the CTA records
// MOE_DEVERR_WAIT_TIMEOUT, unwinds, drains its MMAs and frees its TMEM.
#include <algorithm>
#include <mutex>

#include "common.cuh"
#include "internal.h"

namespace moe {
namespace {

constexpr int BM = 128;                            // tile rows (UMMA M)
constexpr int BN = 256;                            // UMMA N
constexpr int BK = 64;                             // k-block: one 128-byte swizzle row of bf16
constexpr int UK = 16;                             // K of one tcgen05.mma kind::f16
constexpr int kStages = 4;
constexpr int kABytes = BM * BK * 2;               // 16 KB
constexpr int kBoxBytes = 64 * BK * 2;             // 8 KB: 64 columns x 64 k-rows
constexpr int kBBytes = 4 * kBoxBytes;             // 32 KB
constexpr int kStageBytes = kABytes + kBBytes;     // 48 KB
constexpr int kAccCols = 256;
constexpr int kTmemCols = 512;
constexpr int kThreads = 192;
constexpr int kMaxE = 64;
constexpr int kSmemBytes = kStages * kStageBytes + 1024 /*align*/ + 1024 /*barriers etc*/;

// Instruction descriptor, kind::f16: D fp32, A bf16, B bf16, A K-major, B MN-major,
// N = 256, M = 128.
constexpr uint32_t kIdesc = (1u << 4) | (1u << 7) | (1u << 10) | (0u << 15) | (1u << 16) |
                            (static_cast<uint32_t>(BN >> 3) << 17) |
                            (static_cast<uint32_t>(BM >> 4) << 24);

struct GemmParams {
  const int32_t* offsets;  // [E+1] expert segments of the A rows
  __nv_bfloat16* out;      // [rows, n_out]
  int E;
  int K;                   // reduction length (D for GEMM1, F for GEMM2)
  int n_out;               // output columns (F for GEMM1, D for GEMM2)
  int* err;
  uint64_t timeout_ns;
};

template <bool DUAL, int ACT>
__global__ void __launch_bounds__(kThreads, 1)
    grouped_gemm_sm100(const __grid_constant__ CUtensorMap tmA,
                       const __grid_constant__ CUtensorMap tmB0,
                       const __grid_constant__ CUtensorMap tmB1, const GemmParams p) {
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  const uint32_t raw_addr = smem_u32(smem_raw);
  uint8_t* smem = smem_raw + ((1024u - (raw_addr & 1023u)) & 1023u);
  uint8_t* sA = smem;
  uint8_t* sB = smem + kStages * kABytes;
  uint64_t* full = reinterpret_cast<uint64_t*>(sB + kStages * kBBytes);
  uint64_t* empty = full + kStages;
  uint64_t* tfull = empty + kStages;
  uint64_t* tempty = tfull + 2;
  uint64_t* drain = tempty + 2;
  uint32_t* s_tmem = reinterpret_cast<uint32_t*>(drain + 1);
  int* s_tile_start = reinterpret_cast<int*>(s_tmem + 1);  // [E+1]
  int* s_seg = s_tile_start + (kMaxE + 1);                 // [E+1]

  constexpr int NT = DUAL ? 128 : 256;  // output columns per tile
  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const int n_blocks = (p.n_out + NT - 1) / NT;
  const int num_kb = (p.K + BK - 1) / BK;

  if (threadIdx.x == 0) {
    int acc = 0;
    for (int e = 0; e <= p.E; ++e) s_seg[e] = p.offsets[e];
    for (int e = 0; e < p.E; ++e) {
      s_tile_start[e] = acc;
      const int m = s_seg[e + 1] - s_seg[e];
      acc += ((m + BM - 1) / BM) * n_blocks;
    }
    s_tile_start[p.E] = acc;
  }
  __syncthreads();
  const int total_tiles = s_tile_start[p.E];
  if (static_cast<int>(blockIdx.x) >= total_tiles) return;  // uniform: before any allocation

  if (threadIdx.x == 0) {
    for (int s = 0; s < kStages; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], 1);
    }
    for (int a = 0; a < 2; ++a) {
      mbar_init(&tfull[a], 1);
      mbar_init(&tempty[a], 128);
    }
    mbar_init(drain, 1);
    fence_barrier_init();
    prefetch_tensormap(&tmA);
    prefetch_tensormap(&tmB0);
    if (DUAL) prefetch_tensormap(&tmB1);
  }
  if (warp == 1) {
    tmem_alloc(s_tmem, kTmemCols);
    tmem_relinquish();
  }
  tc_fence_before_sync();
  __syncthreads();
  tc_fence_after_sync();
  const uint32_t tmem_base = *s_tmem;

  // tile -> (expert, row block, column block)
  auto decode = [&](int tile, int& e, int& m_blk, int& n_blk) {
    e = 0;
    while (e < p.E - 1 && tile >= s_tile_start[e + 1]) ++e;
    const int local = tile - s_tile_start[e];
    const int m_tiles = (s_seg[e + 1] - s_seg[e] + BM - 1) / BM;
    n_blk = local / m_tiles;
    m_blk = local - n_blk * m_tiles;
  };

  if (warp == 0) {
    if (lane == 0) {  // ---------------------------------------------------- TMA producer
      int stage = 0;
      uint32_t phase = 0;
      bool ok = true;
      for (int tile = blockIdx.x; ok && tile < total_tiles; tile += gridDim.x) {
        int e, m_blk, n_blk;
        decode(tile, e, m_blk, n_blk);
        const int row0 = s_seg[e] + m_blk * BM;
        const int n0 = n_blk * NT;
        for (int kb = 0; kb < num_kb; ++kb) {
          if (!mbar_wait(&empty[stage], phase ^ 1u, p.timeout_ns)) {
            record_error(p.err, MOE_DEVERR_WAIT_TIMEOUT);
            ok = false;
            break;
          }
          mbar_arrive_expect_tx(&full[stage], kStageBytes);
          uint8_t* a_dst = sA + stage * kABytes;
          uint8_t* b_dst = sB + stage * kBBytes;
          const int k0 = kb * BK;
          tma_load_2d(a_dst, &tmA, &full[stage], k0, row0);
          if (DUAL) {
            tma_load_3d(b_dst, &tmB0, &full[stage], n0, k0, e);
            tma_load_3d(b_dst + kBoxBytes, &tmB0, &full[stage], n0 + 64, k0, e);
            tma_load_3d(b_dst + 2 * kBoxBytes, &tmB1, &full[stage], n0, k0, e);
            tma_load_3d(b_dst + 3 * kBoxBytes, &tmB1, &full[stage], n0 + 64, k0, e);
          } else {
#pragma unroll
            for (int j = 0; j < 4; ++j)
              tma_load_3d(b_dst + j * kBoxBytes, &tmB0, &full[stage], n0 + 64 * j, k0, e);
          }
          if (++stage == kStages) {
            stage = 0;
            phase ^= 1u;
          }
        }
      }
    }
  } else if (warp == 1) {
    if (lane == 0) {  // ---------------------------------------------------- MMA issuer
      int stage = 0;
      uint32_t phase = 0;
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
        for (int kb = 0; kb < num_kb; ++kb) {
          if (!mbar_wait(&full[stage], phase, p.timeout_ns)) {
            record_error(p.err, MOE_DEVERR_WAIT_TIMEOUT);
            ok = false;
            break;
          }
          tc_fence_after_sync();
          const uint32_t a_addr = smem_u32(sA + stage * kABytes);
          const uint32_t b_addr = smem_u32(sB + stage * kBBytes);
#pragma unroll
          for (int kk = 0; kk < BK / UK; ++kk) {
            // A: K-major SW128, advance 16 elements = 32 bytes inside the swizzle row.
            const uint64_t ad = smem_desc_sw128(a_addr + kk * 32, 16, 1024);
            // B: MN-major SW128, 64-column blocks kBoxBytes apart (LBO), 8-row k groups
            // 1024 bytes apart (SBO); advance 16 k-rows = 2048 bytes.
            const uint64_t bd = smem_desc_sw128(b_addr + kk * 2048, kBoxBytes, 1024);
            umma_bf16_ss(d_tmem, ad, bd, kIdesc, (kb | kk) != 0 ? 1u : 0u);
          }
          umma_commit(&empty[stage]);  // frees the smem stage once these MMAs have read it
          if (++stage == kStages) {
            stage = 0;
            phase ^= 1u;
          }
        }
        if (ok) umma_commit(&tfull[acc]);  // accumulator complete
      }
      // Every MMA issued by this thread has completed once `drain` flips.
      umma_commit(drain);
      if (!mbar_wait(drain, 0, p.timeout_ns)) record_error(p.err, MOE_DEVERR_WAIT_TIMEOUT);
    }
  } else {  // ------------------------------------------------------------------ epilogue
    const int q = warp & 3;  // this warp may access TMEM lanes [32q, 32q+32)
    const int r = q * 32 + lane;
    int it = 0;
    for (int tile = blockIdx.x; tile < total_tiles; tile += gridDim.x, ++it) {
      const int acc = it & 1;
      const uint32_t acc_phase = static_cast<uint32_t>(it >> 1) & 1u;
      const bool ok = mbar_wait(&tfull[acc], acc_phase, p.timeout_ns);
      if (__any_sync(0xffffffffu, !ok)) {
        if (lane == 0) record_error(p.err, MOE_DEVERR_WAIT_TIMEOUT);
        break;
      }
      tc_fence_after_sync();
      int e, m_blk, n_blk;
      decode(tile, e, m_blk, n_blk);
      const int rows = min(BM, s_seg[e + 1] - s_seg[e] - m_blk * BM);
      const bool valid = r < rows;
      const int64_t grow = static_cast<int64_t>(s_seg[e]) + m_blk * BM + r;
      const int n0 = n_blk * NT;
      __nv_bfloat16* orow = p.out + grow * p.n_out + n0;
      const uint32_t t_row =
          tmem_base + (static_cast<uint32_t>(q * 32) << 16) + static_cast<uint32_t>(acc * kAccCols);
      if (DUAL) {
#pragma unroll 1
        for (int c = 0; c < 4; ++c) {
          uint32_t ra[32], rb[32];
          tmem_ld_32cols(t_row + c * 32, ra);        // x W1 (activated branch)
          tmem_ld_32cols(t_row + 128 + c * 32, rb);  // x W2 (linear branch)
          tmem_ld_wait();
          if (valid) {
            uint32_t w[16];
#pragma unroll
            for (int i = 0; i < 16; ++i) {
              const float h0 = activation<ACT>(__uint_as_float(ra[2 * i])) * __uint_as_float(rb[2 * i]);
              const float h1 =
                  activation<ACT>(__uint_as_float(ra[2 * i + 1])) * __uint_as_float(rb[2 * i + 1]);
              w[i] = pack_bf16x2(h0, h1);
            }
#pragma unroll
            for (int v = 0; v < 4; ++v)
              if (n0 + c * 32 + v * 8 < p.n_out)
                reinterpret_cast<uint4*>(orow + c * 32)[v] =
                    make_uint4(w[4 * v], w[4 * v + 1], w[4 * v + 2], w[4 * v + 3]);
          }
        }
      } else {
#pragma unroll 1
        for (int c = 0; c < 8; ++c) {
          uint32_t ra[32];
          tmem_ld_32cols(t_row + c * 32, ra);
          tmem_ld_wait();
          if (valid) {
            uint32_t w[16];
#pragma unroll
            for (int i = 0; i < 16; ++i)
              w[i] = pack_bf16x2(__uint_as_float(ra[2 * i]), __uint_as_float(ra[2 * i + 1]));
#pragma unroll
            for (int v = 0; v < 4; ++v)
              if (n0 + c * 32 + v * 8 < p.n_out)
                reinterpret_cast<uint4*>(orow + c * 32)[v] =
                    make_uint4(w[4 * v], w[4 * v + 1], w[4 * v + 2], w[4 * v + 3]);
          }
        }
      }
      tc_fence_before_sync();
      mbar_arrive(&tempty[acc]);
    }
  }

  __syncthreads();
  if (warp == 1) {
    __syncwarp();
    tc_fence_after_sync();
    tmem_dealloc(tmem_base, kTmemCols);
  }
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

template <bool DUAL, int ACT>
cudaError_t launch_gemm(const CUtensorMap& a, const CUtensorMap& b0, const CUtensorMap& b1,
                        const GemmParams& gp, int grid, cudaStream_t stream) {
  auto kern = grouped_gemm_sm100<DUAL, ACT>;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, kSmemBytes);
  if (e != cudaSuccess) return e;
  kern<<<grid, kThreads, kSmemBytes, stream>>>(a, b0, b1, gp);
  return cudaGetLastError();
}

}  // namespace

cudaError_t launch_ffn_up_sm100(const moe_problem& p, const void* X_perm, const int32_t* offsets,
                                const void* W1, const void* W2, void* H, int* err,
                                uint64_t timeout_ns, cudaStream_t stream) {
  const int64_t R = p.N * p.k;
  if (R == 0) return cudaSuccess;
  if (encode_fn() == nullptr) return cudaErrorNotSupported;
  CUtensorMap tA, tW1, tW2;
  if (!make_map_2d(&tA, X_perm, p.D, R, BM) || !make_map_3d(&tW1, W1, p.F, p.D, p.E) ||
      !make_map_3d(&tW2, W2, p.F, p.D, p.E))
    return cudaErrorInvalidValue;
  const int64_t row_blocks = (R + BM - 1) / BM + p.E;  // upper bound over any split of R
  GemmParams g;
  g.offsets = offsets;
  g.out = static_cast<__nv_bfloat16*>(H);
  g.E = p.E;
  g.K = static_cast<int>(p.D);
  g.n_out = static_cast<int>(p.F);
  g.err = err;
  g.timeout_ns = timeout_ns;
  const int grid = static_cast<int>(std::min<int64_t>(num_sms(), row_blocks * ((p.F + 127) / 128)));
  switch (p.activation) {
    case MOE_ACT_SILU:
      return launch_gemm<true, MOE_ACT_SILU>(tA, tW1, tW2, g, grid, stream);
    case MOE_ACT_GELU_ERF:
      return launch_gemm<true, MOE_ACT_GELU_ERF>(tA, tW1, tW2, g, grid, stream);
    default:
      return launch_gemm<true, MOE_ACT_GELU_TANH>(tA, tW1, tW2, g, grid, stream);
  }
}

cudaError_t launch_ffn_down_sm100(const moe_problem& p, const void* H, const int32_t* offsets,
                                  const void* W3, void* Y, int* err, uint64_t timeout_ns,
                                  cudaStream_t stream) {
  const int64_t R = p.N * p.k;
  if (R == 0) return cudaSuccess;
  if (encode_fn() == nullptr) return cudaErrorNotSupported;
  CUtensorMap tA, tW3;
  if (!make_map_2d(&tA, H, p.F, R, BM) || !make_map_3d(&tW3, W3, p.D, p.F, p.E))
    return cudaErrorInvalidValue;
  const int64_t row_blocks = (R + BM - 1) / BM + p.E;
  GemmParams g;
  g.offsets = offsets;
  g.out = static_cast<__nv_bfloat16*>(Y);
  g.E = p.E;
  g.K = static_cast<int>(p.F);
  g.n_out = static_cast<int>(p.D);
  g.err = err;
  g.timeout_ns = timeout_ns;
  const int grid = static_cast<int>(std::min<int64_t>(num_sms(), row_blocks * ((p.D + 255) / 256)));
  return launch_gemm<false, MOE_ACT_SILU>(tA, tW3, tW3, g, grid, stream);
}

}  // namespace moe

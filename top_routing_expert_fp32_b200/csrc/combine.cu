// Combine: out[t] = sum_j [not dropped] * gate[t,j] * Y[offsets[idx[t,j]] + pos[t,j]].
//   Grok-1 book ch.5, 5.3.5 (gate-weighted sum over the k expert outputs); LLMs-from-scratch
//   ch.12, 12.2 (a token accumulates its k contributions; never overwrite); MoE series 2.2
//   (an overflowed slot contributes nothing; a token with every slot dropped gets 0; case A:
//   with renorm_kept, a token that lost some slots spreads the whole weight over the kept
//   ones, gate / sum of kept gates).
//
// One warp per token; each lane owns 16-byte column chunks of the row. The k rows are read
// with 16-byte loads, accumulated in fp32 in ascending j (fixed order, no atomics), and
// rounded once to the output dtype. HBM-bound: reads the kept Y rows once, writes out once.
#include "common.cuh"
#include "internal.h"

namespace moe {
namespace {

constexpr int kWarps = 8;  // tokens per block
constexpr int kThreads = 32 * kWarps;

template <typename T>
struct Vec16;
template <>
struct Vec16<__nv_bfloat16> {
  static constexpr int kElems = 8;
  __device__ static void unpack(const uint4& v, float (&f)[8]) {
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      const uint32_t w = (&v.x)[i];
      f[2 * i] = bf16_bits_to_float(w & 0xFFFFu);
      f[2 * i + 1] = bf16_bits_to_float(w >> 16);
    }
  }
  __device__ static uint4 pack(const float (&f)[8]) {
    uint4 v;
#pragma unroll
    for (int i = 0; i < 4; ++i) (&v.x)[i] = pack_bf16x2(f[2 * i], f[2 * i + 1]);
    return v;
  }
};
template <>
struct Vec16<float> {
  static constexpr int kElems = 4;
  __device__ static void unpack(const uint4& v, float (&f)[4]) {
#pragma unroll
    for (int i = 0; i < 4; ++i) f[i] = __uint_as_float((&v.x)[i]);
  }
  __device__ static uint4 pack(const float (&f)[4]) {
    uint4 v;
#pragma unroll
    for (int i = 0; i < 4; ++i) (&v.x)[i] = __float_as_uint(f[i]);
    return v;
  }
};

// wpt warps per token (1, or kWarps for batches too small to fill the GPU), kWarps / wpt
// tokens per block, no block-wide barrier. Lanes 0..k-1 of each warp read the token's records
// (expert, position, drop flag, gate) and the warp shares them by shuffles; every lane then
// streams 16-byte chunks of the k rows, kBatch chunks of all k rows loaded before any is used
// (about 8 loads in flight per lane).
template <typename T, int KMAX, int WPT>
__global__ void __launch_bounds__(kThreads)
    combine_kernel(const uint4* __restrict__ Y, const int32_t* __restrict__ idx,
                   const float* __restrict__ gate, const int32_t* __restrict__ offsets,
                   const int32_t* __restrict__ pos, const uint8_t* __restrict__ dropped,
                   uint4* __restrict__ out, int64_t N, int k, int E, int64_t chunks_per_row,
                   bool renorm_kept, int* err) {
  constexpr int wpt = WPT;
  constexpr int V = Vec16<T>::kElems;
  constexpr int kBatch = KMAX >= 8 ? 1 : 8 / KMAX;
  const int lane = threadIdx.x & 31;
  const int warp = threadIdx.x >> 5;
  const int64_t t = static_cast<int64_t>(blockIdx.x) * (kWarps / wpt) + warp / wpt;
  const int64_t first = 32 * (warp % wpt) + lane;  // this lane's first chunk
  const int64_t step = 32 * wpt;
  pdl_wait();  // Y and the routing come from the previous kernels
  pdl_trigger();
  if (t >= N) return;  // uniform over the warp
  int64_t my_row = -1;
  float my_g = 0.f;
  if (lane < k) {
    const int64_t rec = t * k + lane;
    const int e = idx[rec];
    bool keep = dropped == nullptr || dropped[rec] == 0;
    if (e < 0 || e >= E) {
      record_error(err, MOE_DEVERR_BAD_INDEX);
      keep = false;
    }
    if (keep) {
      // A kept record's row lies inside its expert's segment; a position outside it (a
      // dropped record passed without its flag, or a corrupt pos) is reported and skipped,
      // so no row past the segment, or past the end of Y, is ever read.
      const int32_t ps = pos[rec];
      const int32_t seg0 = offsets[e];
      if (ps < 0 || ps >= offsets[e + 1] - seg0) {
        record_error(err, MOE_DEVERR_BAD_INDEX);
        keep = false;
      } else {
        my_row = static_cast<int64_t>(seg0) + ps;
      }
    }
    my_g = gate[rec];
  }
  int64_t row[KMAX];
  float g[KMAX];
#pragma unroll
  for (int j = 0; j < KMAX; ++j) {
    row[j] = __shfl_sync(0xffffffffu, my_row, j);
    g[j] = __shfl_sync(0xffffffffu, my_g, j);
    if (j >= k) row[j] = -1;
  }
  if (renorm_kept) {  // MoE series 2.2 case A: the kept gates share the whole weight
    float kept_sum = 0.f;
    int kept = 0;
#pragma unroll
    for (int j = 0; j < KMAX; ++j)
      if (row[j] >= 0) {
        kept_sum += g[j];
        ++kept;
      }
    if (kept > 0 && kept < k) {
#pragma unroll
      for (int j = 0; j < KMAX; ++j)
        if (row[j] >= 0) g[j] = g[j] / kept_sum;
    }
  }
  for (int64_t c0 = first; c0 < chunks_per_row; c0 += step * kBatch) {
    uint4 yv[kBatch][KMAX];
#pragma unroll
    for (int b = 0; b < kBatch; ++b) {
      const int64_t c = c0 + b * step;
#pragma unroll
      for (int j = 0; j < KMAX; ++j) {
        yv[b][j] = make_uint4(0u, 0u, 0u, 0u);
        if (c < chunks_per_row && row[j] >= 0) yv[b][j] = __ldg(Y + row[j] * chunks_per_row + c);
      }
    }
#pragma unroll
    for (int b = 0; b < kBatch; ++b) {
      const int64_t c = c0 + b * step;
      if (c >= chunks_per_row) break;
      float acc[V];
#pragma unroll
      for (int i = 0; i < V; ++i) acc[i] = 0.f;
#pragma unroll
      for (int j = 0; j < KMAX; ++j) {
        if (row[j] < 0) continue;
        float y[V];
        Vec16<T>::unpack(yv[b][j], y);
#pragma unroll
        for (int i = 0; i < V; ++i) acc[i] = fmaf(g[j], y[i], acc[i]);
      }
      out[t * chunks_per_row + c] = Vec16<T>::pack(acc);
    }
  }
}

}  // namespace

cudaError_t launch_combine(const moe_problem& p, const void* Y, const int32_t* idx,
                           const float* gate, const int32_t* offsets, const int32_t* pos,
                           const uint8_t* dropped, void* out, int* err, cudaStream_t stream) {
  if (p.N == 0) return cudaSuccess;
  const int64_t elem = p.dtype == MOE_DTYPE_BF16 ? 2 : 4;
  const int64_t chunks = p.D * elem / 16;
  // A warp per token once there are enough tokens for 16 warps per SM (about 64 KB of loads
  // in flight per SM), else a block of kWarps warps per token.
  const int wpt = p.N >= static_cast<int64_t>(num_sms()) * 16 ? 1 : kWarps;
  const int tpb = kWarps / wpt;
  const dim3 grid(static_cast<unsigned>((p.N + tpb - 1) / tpb));
  const uint4* y = static_cast<const uint4*>(Y);
  uint4* o = static_cast<uint4*>(out);
  const bool rk = p.drop_policy == MOE_DROP_RENORM_KEPT && dropped != nullptr;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = dim3(kThreads);
  cfg.dynamicSmemBytes = 0;
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  cfg.attrs = attr;
  cfg.numAttrs = pdl_attr(&attr[0]);
  cudaError_t e = cudaSuccess;
#define MOE_COMBINE(T, KM)                                                                     \
  do {                                                                                         \
    if (wpt == 1)                                                                              \
      e = cudaLaunchKernelEx(&cfg, combine_kernel<T, KM, 1>, y, idx, gate, offsets, pos,       \
                             dropped, o, p.N, p.k, p.E, chunks, rk, err);                      \
    else                                                                                       \
      e = cudaLaunchKernelEx(&cfg, combine_kernel<T, KM, kWarps>, y, idx, gate, offsets, pos,  \
                             dropped, o, p.N, p.k, p.E, chunks, rk, err);                      \
  } while (0)
  if (p.dtype == MOE_DTYPE_BF16) {
    if (p.k <= 1) MOE_COMBINE(__nv_bfloat16, 1);
    else if (p.k <= 2) MOE_COMBINE(__nv_bfloat16, 2);
    else if (p.k <= 4) MOE_COMBINE(__nv_bfloat16, 4);
    else MOE_COMBINE(__nv_bfloat16, 8);
  } else {
    if (p.k <= 1) MOE_COMBINE(float, 1);
    else if (p.k <= 2) MOE_COMBINE(float, 2);
    else if (p.k <= 4) MOE_COMBINE(float, 4);
    else MOE_COMBINE(float, 8);
  }
#undef MOE_COMBINE
  return e != cudaSuccess ? e : cudaGetLastError();
}

}  // namespace moe

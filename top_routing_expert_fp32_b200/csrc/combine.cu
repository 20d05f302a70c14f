// Combine: out[t] = sum_j [not dropped] * gate[t,j] * Y[offsets[idx[t,j]] + pos[t,j]].
//   Grok-1 book ch.5, 5.3.5 (gate-weighted sum over the k expert outputs); LLMs-from-scratch
//   ch.12, 12.2 (a token accumulates its k contributions; never overwrite); MoE series 2.2
//   (an overflowed slot contributes nothing; a token with every slot dropped gets 0; case A:
//   with renorm_kept, a token that lost some slots spreads the whole weight over the kept
//   ones, gate / sum of kept gates).
//
// One block per token, each thread owns 16-byte column chunks of the row. The k rows are read
// with 16-byte loads, accumulated in fp32 in ascending j (fixed order, no atomics), and
// rounded once to the output dtype. HBM-bound: reads the kept Y rows once, writes out once.
#include "common.cuh"
#include "internal.h"

namespace moe {
namespace {

constexpr int kThreads = 128;
constexpr int kMaxK = 8;

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

template <typename T, int KMAX, bool BATCH>
__global__ void __launch_bounds__(kThreads)
    combine_kernel(const uint4* __restrict__ Y, const int32_t* __restrict__ idx,
                   const float* __restrict__ gate, const int32_t* __restrict__ offsets,
                   const int32_t* __restrict__ pos, const uint8_t* __restrict__ dropped,
                   uint4* __restrict__ out, int64_t N, int k, int E, int64_t chunks_per_row,
                   bool renorm_kept, int* err) {
  constexpr int V = Vec16<T>::kElems;
  __shared__ int64_t s_row[kMaxK];
  __shared__ float s_g[kMaxK];
  const int64_t t = blockIdx.x;
  if (threadIdx.x < k) {
    const int j = threadIdx.x;
    const int64_t rec = t * k + j;
    const int e = idx[rec];
    bool keep = dropped == nullptr || dropped[rec] == 0;
    if (e < 0 || e >= E) {
      record_error(err, MOE_DEVERR_BAD_INDEX);
      keep = false;
    }
    s_row[j] = keep ? static_cast<int64_t>(offsets[e]) + pos[rec] : -1;
    s_g[j] = gate[rec];
  }
  __syncthreads();
  if (renorm_kept && threadIdx.x == 0) {
    float kept_sum = 0.f;
    int kept = 0;
    for (int j = 0; j < k; ++j)
      if (s_row[j] >= 0) {
        kept_sum += s_g[j];
        ++kept;
      }
    if (kept > 0 && kept < k)
      for (int j = 0; j < k; ++j)
        if (s_row[j] >= 0) s_g[j] = s_g[j] / kept_sum;
  }
  if (renorm_kept) __syncthreads();
  // With BATCH (long rows), kBatch chunks per thread are loaded (all k rows) before any is
  // used, so a thread keeps about 8 16-byte loads in flight instead of one round trip per
  // chunk; short rows keep the register count (and occupancy) of one chunk at a time.
  constexpr int kBatch = (!BATCH || KMAX >= 8) ? 1 : 8 / KMAX;
  for (int64_t c0 = threadIdx.x; c0 < chunks_per_row; c0 += kThreads * kBatch) {
    uint4 yv[kBatch][KMAX];
#pragma unroll
    for (int b = 0; b < kBatch; ++b) {
      const int64_t c = c0 + b * kThreads;
#pragma unroll
      for (int j = 0; j < KMAX; ++j) {
        yv[b][j] = make_uint4(0u, 0u, 0u, 0u);
        if (j < k && c < chunks_per_row && s_row[j] >= 0)
          yv[b][j] = __ldg(Y + s_row[j] * chunks_per_row + c);
      }
    }
#pragma unroll
    for (int b = 0; b < kBatch; ++b) {
      const int64_t c = c0 + b * kThreads;
      if (c >= chunks_per_row) break;
      float acc[V];
#pragma unroll
      for (int i = 0; i < V; ++i) acc[i] = 0.f;
#pragma unroll
      for (int j = 0; j < KMAX; ++j) {
        if (j >= k || s_row[j] < 0) continue;
        float y[V];
        Vec16<T>::unpack(yv[b][j], y);
        const float g = s_g[j];
#pragma unroll
        for (int i = 0; i < V; ++i) acc[i] = fmaf(g, y[i], acc[i]);
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
  const dim3 grid(static_cast<unsigned>(p.N));
  const uint4* y = static_cast<const uint4*>(Y);
  uint4* o = static_cast<uint4*>(out);
  const bool batch = chunks >= 4 * kThreads;
  const bool rk = p.drop_policy == MOE_DROP_RENORM_KEPT && dropped != nullptr;
#define MOE_COMBINE(T, KM)                                                                     \
  do {                                                                                         \
    if (batch)                                                                                 \
      combine_kernel<T, KM, true><<<grid, kThreads, 0, stream>>>(y, idx, gate, offsets, pos,   \
                                                                 dropped, o, p.N, p.k, p.E,    \
                                                                 chunks, rk, err);             \
    else                                                                                       \
      combine_kernel<T, KM, false><<<grid, kThreads, 0, stream>>>(y, idx, gate, offsets, pos,  \
                                                                  dropped, o, p.N, p.k, p.E,   \
                                                                  chunks, rk, err);            \
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
  return cudaGetLastError();
}

}  // namespace moe

// Grouped gated expert FFN in fp32 on CUDA cores (fp32 problems):
//   H[r] = act(X_perm[r] W1_e) (.) (X_perm[r] W2_e),   Y[r] = H[r] W3_e
// for every row r of expert e's segment [offsets[e], offsets[e+1]) (LLMs-from-scratch ch.12,
// 12.1; Grok-1 book ch.5, 5.3.5). Full fp32 FMA accumulation in ascending d / f, so results
// stay within fp32 rounding of the exact values. One thread per output element; threads of a
// block cover consecutive columns so weight rows are read coalesced, the activation row is a
// broadcast. Intended for small fp32 layers; bf16 layers use the tensor-core path.
#include <algorithm>

#include "common.cuh"
#include "internal.h"

namespace moe {
namespace {

constexpr int kThreads = 128;

__device__ __forceinline__ int expert_of_row(const int32_t* __restrict__ offsets, int E,
                                             int64_t row) {
  int e = 0;
  while (e < E - 1 && row >= offsets[e + 1]) ++e;
  return e;
}

template <int ACT>
__global__ void __launch_bounds__(kThreads)
    ffn1_f32_kernel(const float* __restrict__ Xp, const int32_t* __restrict__ offsets, int E,
                    const float* __restrict__ W1, const float* __restrict__ W2,
                    float* __restrict__ H, int64_t D, int64_t F) {
  const int64_t rows = offsets[E];
  const int64_t f = static_cast<int64_t>(blockIdx.x) * kThreads + threadIdx.x;
  for (int64_t row = blockIdx.y; row < rows; row += gridDim.y) {
    if (f >= F) continue;
    const int e = expert_of_row(offsets, E, row);
    const float* x = Xp + row * D;
    const float* w1 = W1 + static_cast<int64_t>(e) * D * F + f;
    const float* w2 = W2 + static_cast<int64_t>(e) * D * F + f;
    float a = 0.f, b = 0.f;
    for (int64_t d = 0; d < D; ++d) {
      const float xd = x[d];
      a = fmaf(xd, __ldg(w1 + d * F), a);
      b = fmaf(xd, __ldg(w2 + d * F), b);
    }
    H[row * F + f] = activation<ACT>(a) * b;
  }
}

__global__ void __launch_bounds__(kThreads)
    ffn2_f32_kernel(const float* __restrict__ H, const int32_t* __restrict__ offsets, int E,
                    const float* __restrict__ W3, float* __restrict__ Y, int64_t D, int64_t F) {
  const int64_t rows = offsets[E];
  const int64_t c = static_cast<int64_t>(blockIdx.x) * kThreads + threadIdx.x;
  for (int64_t row = blockIdx.y; row < rows; row += gridDim.y) {
    if (c >= D) continue;
    const int e = expert_of_row(offsets, E, row);
    const float* h = H + row * F;
    const float* w3 = W3 + static_cast<int64_t>(e) * F * D + c;
    float y = 0.f;
    for (int64_t f = 0; f < F; ++f) y = fmaf(h[f], __ldg(w3 + f * D), y);
    Y[row * D + c] = y;
  }
}

}  // namespace

cudaError_t launch_ffn_up_f32(const moe_problem& p, const void* X_perm, const int32_t* offsets,
                              const void* W1, const void* W2, void* H, cudaStream_t stream) {
  const int64_t R = p.N * p.k;
  if (R == 0) return cudaSuccess;
  const unsigned gy = static_cast<unsigned>(std::min<int64_t>(R, 65535));
  const dim3 g1(static_cast<unsigned>((p.F + kThreads - 1) / kThreads), gy);
  const float* xp = static_cast<const float*>(X_perm);
  const float* w1 = static_cast<const float*>(W1);
  const float* w2 = static_cast<const float*>(W2);
  float* h = static_cast<float*>(H);
  switch (p.activation) {
    case MOE_ACT_SILU:
      ffn1_f32_kernel<MOE_ACT_SILU><<<g1, kThreads, 0, stream>>>(xp, offsets, p.E, w1, w2, h, p.D, p.F);
      break;
    case MOE_ACT_GELU_ERF:
      ffn1_f32_kernel<MOE_ACT_GELU_ERF><<<g1, kThreads, 0, stream>>>(xp, offsets, p.E, w1, w2, h, p.D, p.F);
      break;
    default:
      ffn1_f32_kernel<MOE_ACT_GELU_TANH><<<g1, kThreads, 0, stream>>>(xp, offsets, p.E, w1, w2, h, p.D, p.F);
      break;
  }
  return cudaGetLastError();
}

cudaError_t launch_ffn_down_f32(const moe_problem& p, const void* H, const int32_t* offsets,
                                const void* W3, void* Y, cudaStream_t stream) {
  const int64_t R = p.N * p.k;
  if (R == 0) return cudaSuccess;
  const unsigned gy = static_cast<unsigned>(std::min<int64_t>(R, 65535));
  const dim3 g2(static_cast<unsigned>((p.D + kThreads - 1) / kThreads), gy);
  ffn2_f32_kernel<<<g2, kThreads, 0, stream>>>(static_cast<const float*>(H), offsets, p.E,
                                               static_cast<const float*>(W3),
                                               static_cast<float*>(Y), p.D, p.F);
  return cudaGetLastError();
}

}  // namespace moe

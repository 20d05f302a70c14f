// Router: fp32 logits x.W_r (+bias), softmax over the E experts, top-k with lower-index
// tie-breaking, gates with or without renormalisation over the selected set.
//   Grok-1 book ch.5, 5.2 (fp32 router, softmax, TopK) and 5.2.3 (two gate variants);
//   MoE formula-to-code walkthrough 1.1-1.2; LLMs-from-scratch ch.12, 12.1.
//
// Layout of the work: a warp owns a group of G tokens and a block of EB experts (G*EB = 64
// fp32 accumulators per lane). Lanes split the model dimension D into 16-byte chunks, so each
// warp-wide load of X is one contiguous 512-byte segment per token; W_r rows are read through
// L1. The 64 per-lane partial sums are reduced across the warp with a 5-step butterfly that
// leaves 2 finished logits per lane. One thread per token then does softmax + top-k + gates
// from shared memory. Blocks are persistent over token tiles and keep one fixed-order partial
// sum of the softmax probabilities per expert (for the balance-loss statistic), which a second
// tiny kernel adds up in block order -- deterministic, no atomics.
#include <algorithm>

#include "common.cuh"
#include "internal.h"

namespace moe {
namespace {

constexpr int kThreads = 128;  // 4 warps
constexpr int kMaxTok = 64;    // tokens per tile (upper bound)
constexpr int kMaxE = 64;
constexpr int kMaxBlocks = 1184;  // persistent-grid cap (8 blocks x 148 SMs); device independent

struct RouteArgs {
  const void* X;
  const float* W_r;
  const float* bias;
  const float* logits_in;  // X == nullptr: given logits
  float* logits_out;       // may be nullptr
  int32_t* idx;
  float* gate;
  float* colsum_partial;  // [gridDim.x][E] or nullptr
  int* err;
  int64_t N;
  int D;
  int E;
  int k;
  int renorm;
  int nwe;  // warps per token group (expert blocks)
};

// 16 bytes of X: 8 bf16 or 4 fp32 values.
template <typename XT>
struct XVec;
template <>
struct XVec<__nv_bfloat16> {
  static constexpr int kElems = 8;
  __device__ static float get(const uint4& v, int j) {
    const uint32_t w = (&v.x)[j >> 1];
    return bf16_bits_to_float((j & 1) ? (w >> 16) : (w & 0xFFFFu));
  }
  __device__ static float one(const void* X, int64_t i) {
    return bf16_bits_to_float(static_cast<const uint16_t*>(X)[i]);
  }
};
template <>
struct XVec<float> {
  static constexpr int kElems = 4;
  __device__ static float get(const uint4& v, int j) { return __uint_as_float((&v.x)[j]); }
  __device__ static float one(const void* X, int64_t i) {
    return static_cast<const float*>(X)[i];
  }
};

// W_r[d][e0 .. e0+EB) with zero padding past E.
template <int EB, bool VECW>
__device__ __forceinline__ void load_w(const float* __restrict__ W_r, int d, int e0, int E,
                                       float (&w)[EB]) {
  const float* row = W_r + static_cast<int64_t>(d) * E + e0;
  if constexpr (VECW) {
#pragma unroll
    for (int q = 0; q < EB / 4; ++q) {
      if (e0 + 4 * q < E) {
        const float4 v = __ldg(reinterpret_cast<const float4*>(row) + q);
        w[4 * q + 0] = v.x;
        w[4 * q + 1] = v.y;
        w[4 * q + 2] = v.z;
        w[4 * q + 3] = v.w;
      } else {
        w[4 * q + 0] = w[4 * q + 1] = w[4 * q + 2] = w[4 * q + 3] = 0.f;
      }
    }
  } else {
#pragma unroll
    for (int e = 0; e < EB; ++e) w[e] = (e0 + e < E) ? __ldg(row + e) : 0.f;
  }
}

template <typename XT, int EB, bool VECW>
__global__ void __launch_bounds__(kThreads) route_kernel(RouteArgs a) {
  constexpr int G = 64 / EB;
  constexpr int V = XVec<XT>::kElems;
  __shared__ float s_z[kMaxTok][kMaxE + 1];

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const int nwe = a.nwe;
  const int ntg = 4 / nwe;
  const int tpc = ntg * G;  // tokens per tile
  const int E = a.E;
  float colsum_acc = 0.f;   // thread e < E: this block's running sum of p_e

  for (int64_t tile = blockIdx.x; tile * tpc < a.N; tile += gridDim.x) {
    const int64_t t_tile = tile * tpc;
    if (a.X != nullptr) {
      const int tg = warp / nwe;
      const int eb = warp % nwe;
      if (tg < ntg) {
        const int64_t t0 = t_tile + static_cast<int64_t>(tg) * G;
        const int e0 = eb * EB;
        const int D = a.D;
        float acc[G][EB];
#pragma unroll
        for (int g = 0; g < G; ++g)
#pragma unroll
          for (int e = 0; e < EB; ++e) acc[g][e] = 0.f;

        const int nvec = D / V;
        for (int c = lane; c < nvec; c += 32) {
          const int d0 = c * V;
          uint4 xv[G];
#pragma unroll
          for (int g = 0; g < G; ++g) {
            if (t0 + g < a.N) {
              const XT* row = static_cast<const XT*>(a.X) + (t0 + g) * static_cast<int64_t>(D);
              xv[g] = __ldg(reinterpret_cast<const uint4*>(row + d0));
            } else {
              xv[g] = make_uint4(0u, 0u, 0u, 0u);
            }
          }
#pragma unroll
          for (int j = 0; j < V; ++j) {
            float w[EB];
            load_w<EB, VECW>(a.W_r, d0 + j, e0, E, w);
#pragma unroll
            for (int g = 0; g < G; ++g) {
              const float x = XVec<XT>::get(xv[g], j);
#pragma unroll
              for (int e = 0; e < EB; ++e) acc[g][e] = fmaf(x, w[e], acc[g][e]);
            }
          }
        }
        for (int d = nvec * V + lane; d < D; d += 32) {  // D not a multiple of V
          float w[EB];
          load_w<EB, VECW>(a.W_r, d, e0, E, w);
#pragma unroll
          for (int g = 0; g < G; ++g) {
            const float x =
                (t0 + g < a.N) ? XVec<XT>::one(a.X, (t0 + g) * static_cast<int64_t>(D) + d) : 0.f;
#pragma unroll
            for (int e = 0; e < EB; ++e) acc[g][e] = fmaf(x, w[e], acc[g][e]);
          }
        }

        // Butterfly reduce-scatter of the 64 partials: after the step with lane offset o the
        // lanes with bit o set keep the upper half. Lane l ends with entries 2l and 2l+1.
        float v[64];
#pragma unroll
        for (int i = 0; i < 64; ++i) v[i] = acc[i / EB][i % EB];
#pragma unroll
        for (int s = 0; s < 5; ++s) {
          const int o = 16 >> s;
          const int half = 32 >> s;
          const bool upper = (lane & o) != 0;
#pragma unroll
          for (int i = 0; i < half; ++i) {
            const float send = upper ? v[i] : v[i + half];
            const float keep = upper ? v[i + half] : v[i];
            v[i] = keep + __shfl_xor_sync(0xffffffffu, send, o);
          }
        }
#pragma unroll
        for (int q = 0; q < 2; ++q) {
          const int i = 2 * lane + q;
          const int g = i / EB;
          const int e = e0 + i % EB;
          if (e < E) s_z[tg * G + g][e] = v[q] + (a.bias != nullptr ? __ldg(a.bias + e) : 0.f);
        }
      }
    } else {
      for (int i = threadIdx.x; i < tpc * E; i += kThreads) {
        const int tl = i / E;
        const int e = i % E;
        const int64_t t = t_tile + tl;
        if (t < a.N) s_z[tl][e] = a.logits_in[t * E + e];
      }
    }
    __syncthreads();

    // One thread per token: softmax, top-k, gates (and probabilities for the statistic).
    const int tl = threadIdx.x;
    const int64_t t = t_tile + tl;
    if (tl < tpc && t < a.N) {
      float* z = s_z[tl];
      if (a.logits_out != nullptr && a.X != nullptr)
        for (int e = 0; e < E; ++e) a.logits_out[t * E + e] = z[e];
      float zmax = z[0];
      for (int e = 1; e < E; ++e) zmax = z[e] > zmax ? z[e] : zmax;
      uint64_t chosen = 0;
      int sel[8];
#pragma unroll
      for (int j = 0; j < 8; ++j) {
        sel[j] = 0;
        if (j < a.k) {
          int best = -1;
          for (int e = 0; e < E; ++e) {
            if ((chosen >> e) & 1ull) continue;
            if (best < 0 || z[e] > z[best]) best = e;  // strict: equal keeps the lower index
          }
          chosen |= 1ull << best;
          sel[j] = best;
        }
      }
      float s_all = 0.f;
      for (int e = 0; e < E; ++e) s_all += expf(z[e] - zmax);
      float s_sel = 0.f;
#pragma unroll
      for (int j = 0; j < 8; ++j)
        if (j < a.k) s_sel += expf(z[sel[j]] - zmax);
      const float denom = a.renorm ? s_sel : s_all;
#pragma unroll
      for (int j = 0; j < 8; ++j) {
        if (j < a.k) {
          a.idx[t * a.k + j] = sel[j];
          a.gate[t * a.k + j] = expf(z[sel[j]] - zmax) / denom;
        }
      }
      if (a.colsum_partial != nullptr)
        for (int e = 0; e < E; ++e) z[e] = expf(z[e] - zmax) / s_all;
    }
    __syncthreads();
    if (a.colsum_partial != nullptr && threadIdx.x < E) {
      const int64_t valid64 = a.N - t_tile;
      const int valid = valid64 < tpc ? static_cast<int>(valid64) : tpc;
      for (int i = 0; i < valid; ++i) colsum_acc += s_z[i][threadIdx.x];
    }
    __syncthreads();
  }
  if (a.colsum_partial != nullptr && threadIdx.x < E)
    a.colsum_partial[static_cast<int64_t>(blockIdx.x) * E + threadIdx.x] = colsum_acc;
}

// prob_colsum[e] = sum over blocks, in block order, of the per-block partials.
__global__ void colsum_reduce_kernel(const float* __restrict__ partial, int nblocks, int E,
                                     float* __restrict__ out) {
  const int e = threadIdx.x;
  if (e >= E) return;
  float s = 0.f;
  for (int b = 0; b < nblocks; ++b) s += partial[static_cast<int64_t>(b) * E + e];
  out[e] = s;
}

int expert_block(int E) { return E <= 4 ? 4 : (E <= 8 ? 8 : 16); }

template <typename XT>
cudaError_t launch_typed(const RouteArgs& a, int grid, int EB, bool vecw, cudaStream_t s) {
  if (EB == 4) {
    if (vecw) route_kernel<XT, 4, true><<<grid, kThreads, 0, s>>>(a);
    else route_kernel<XT, 4, false><<<grid, kThreads, 0, s>>>(a);
  } else if (EB == 8) {
    if (vecw) route_kernel<XT, 8, true><<<grid, kThreads, 0, s>>>(a);
    else route_kernel<XT, 8, false><<<grid, kThreads, 0, s>>>(a);
  } else {
    if (vecw) route_kernel<XT, 16, true><<<grid, kThreads, 0, s>>>(a);
    else route_kernel<XT, 16, false><<<grid, kThreads, 0, s>>>(a);
  }
  return cudaGetLastError();
}

}  // namespace

int route_num_blocks(int64_t N, int E) {
  const int EB = expert_block(E);
  const int nwe = (E + EB - 1) / EB;
  const int tpc = (4 / nwe) * (64 / EB);
  const int64_t tiles = (N + tpc - 1) / tpc;
  return static_cast<int>(std::max<int64_t>(1, std::min<int64_t>(tiles, kMaxBlocks)));
}

cudaError_t launch_route(const moe_problem& p, const void* X, const float* W_r, const float* bias,
                         float* logits, int32_t* idx, float* gate, float* colsum_partial,
                         float* prob_colsum, int* err, cudaStream_t stream) {
  if (p.N == 0) return cudaSuccess;
  RouteArgs a;
  a.X = X;
  a.W_r = W_r;
  a.bias = bias;
  a.logits_in = X == nullptr ? logits : nullptr;
  a.logits_out = X != nullptr ? logits : nullptr;
  a.idx = idx;
  a.gate = gate;
  a.colsum_partial = prob_colsum != nullptr ? colsum_partial : nullptr;
  a.err = err;
  a.N = p.N;
  a.D = static_cast<int>(p.D);
  a.E = p.E;
  a.k = p.k;
  a.renorm = p.renormalize;
  const int EB = expert_block(p.E);
  a.nwe = (p.E + EB - 1) / EB;
  const bool vecw = (p.E % 4) == 0;
  const int grid = route_num_blocks(p.N, p.E);
  cudaError_t e = p.dtype == MOE_DTYPE_BF16
                      ? launch_typed<__nv_bfloat16>(a, grid, EB, vecw, stream)
                      : launch_typed<float>(a, grid, EB, vecw, stream);
  if (e != cudaSuccess) return e;
  if (prob_colsum != nullptr) {
    colsum_reduce_kernel<<<1, kMaxE, 0, stream>>>(colsum_partial, grid, p.E, prob_colsum);
    e = cudaGetLastError();
  }
  return e;
}

}  // namespace moe

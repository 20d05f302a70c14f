// Router: fp32 logits x.W_r (+bias), softmax over the E experts, top-k with lower-index
// tie-breaking, gates with or without renormalisation over the selected set.
//   Grok-1 book ch.5, 5.2 (fp32 router, softmax, TopK) and 5.2.3 (two gate variants);
//   MoE formula-to-code walkthrough 1.1-1.2; LLMs-from-scratch ch.12, 12.1.
//
// bf16 X: the logits run on the tensor cores (route_tc.cu) and this file's selection kernel
// finishes. fp32 X: two logit kernels, chosen by E (both fp32 FMA with fp32 accumulation):
//   narrow (E <= 16, bound by reading X): persistent 512-thread blocks, one per SM, with W_r
//     resident in shared memory; a warp owns G = 32/EB tokens and a slice of D, lanes stream
//     16-byte chunks of X, a butterfly leaves one finished partial per lane, and the K slices
//     are added in a fixed order through shared memory.
//   wide (E > 16, bound by fp32 FMA throughput): a block computes a 128-token x 64-expert
//     tile as a small SGEMM over D in 32-wide slices staged through shared memory, each
//     thread an 8x8 register tile, two K halves added in a fixed order.
// Then one thread per token does softmax + top-k + gates from shared memory. Blocks are
// persistent over token tiles and keep a fixed-order partial sum of the softmax probabilities
// per expert (for the balance-loss statistic); a second tiny kernel adds the partials in block
// order -- deterministic, no atomics. With X == nullptr the logits are an input and only the
// selection runs.
#include <algorithm>

#include "common.cuh"
#include "internal.h"
#include "select.cuh"

namespace moe {
namespace {

constexpr int kMaxE = 64;
constexpr int kMaxBlocks = 1184;  // persistent-grid cap; device independent (workspace sizing)

struct RouteArgs {
  const void* X;
  const float* W_r;
  const float* bias;
  const float* logits_in;  // X == nullptr: given logits
  float* logits_out;       // may be nullptr
  int32_t* idx;
  float* gate;
  float* colsum_partial;  // [gridDim.x][E] or nullptr
  const float* noise;     // [N][E] (routing_mode != TOPK) or nullptr
  int mode;               // MOE_ROUTE_*
  float* zl_partial;      // [gridDim.x]: per-block sum of (log Z)^2, or nullptr
  int64_t N;
  int D;
  int E;
  int k;
  int renorm;
};

// 16 bytes of X: 4 fp32 values.
template <typename XT>
struct XVec;
template <>
struct XVec<float> {
  static constexpr int kElems = 4;
  __device__ static float get(const uint4& v, int j) { return __uint_as_float((&v.x)[j]); }
  __device__ static float one(const void* X, int64_t i) {
    return static_cast<const float*>(X)[i];
  }
};

__device__ __forceinline__ uint4 ld_stream(const void* p) {
  uint4 v;
  asm volatile("ld.global.nc.L1::no_allocate.v4.u32 {%0, %1, %2, %3}, [%4];"
               : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w)
               : "l"(p));
  return v;
}

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

// Softmax, top-k and gates for the tokens of one tile whose logits are in s_z (row stride
// kMaxE + 1). One thread per token; afterwards s_z holds the probabilities if colsum is
// wanted. `colsum_acc` (thread e < E) accumulates this block's per-expert probability sum in
// token order.
// (log Z)^2 of token row i is parked in the row's spare column kMaxE (E <= kMaxE).
__device__ __forceinline__ void select_tile(const RouteArgs& a, float (*s_z)[kMaxE + 1],
                                            int tpc, int64_t t_tile, float& colsum_acc,
                                            float& zl_acc) {
  const int E = a.E;
  const int tl = threadIdx.x;
  const int64_t t = t_tile + tl;
  if (tl < tpc && t < a.N) {
    float* z = s_z[tl];
    if (a.logits_out != nullptr)
      for (int e = 0; e < E; ++e) a.logits_out[t * E + e] = z[e];
    float lse = 0.f;
    select_token(z, E, a.k, a.renorm, a.mode, a.noise != nullptr ? a.noise + t * E : nullptr,
                 a.idx + t * a.k, a.gate + t * a.k, a.colsum_partial != nullptr,
                 a.zl_partial != nullptr ? &lse : nullptr);
    z[kMaxE] = lse * lse;
  }
  __syncthreads();
  const int64_t valid64 = a.N - t_tile;
  const int valid = valid64 < tpc ? static_cast<int>(valid64) : tpc;
  if (a.colsum_partial != nullptr && static_cast<int>(threadIdx.x) < E)
    for (int i = 0; i < valid; ++i) colsum_acc += s_z[i][threadIdx.x];
  if (a.zl_partial != nullptr && threadIdx.x == 0)
    for (int i = 0; i < valid; ++i) zl_acc += s_z[i][kMaxE];
  __syncthreads();
}

__device__ __forceinline__ void write_colsum(const RouteArgs& a, float colsum_acc, float zl_acc) {
  if (a.colsum_partial != nullptr && static_cast<int>(threadIdx.x) < a.E)
    a.colsum_partial[static_cast<int64_t>(blockIdx.x) * a.E + threadIdx.x] = colsum_acc;
  if (a.zl_partial != nullptr && threadIdx.x == 0) a.zl_partial[blockIdx.x] = zl_acc;
}

// ------------------------------------------------------------------ narrow: E <= 16
//
// Persistent, one 512-thread block per SM. W_r (D x EB fp32, zero padded to EB experts) is
// copied once into shared memory, laid out so that lane l's rows are contiguous with lane
// l+1's (conflict-free 16-byte reads). A warp owns G tokens and a K slice; lanes take 16-byte
// chunks of X (prefetched one step ahead), accumulate G x EB partial logits, and a butterfly
// leaves one finished partial per lane. KS warps (KS = 1..16, chosen for enough parallelism)
// share a token group; their partials are added in a fixed order through shared memory.

constexpr int kNarrowThreads = 512;
constexpr int kNarrowWarps = kNarrowThreads / 32;
constexpr size_t kNarrowMaxSmemBytes = 227 * 1024;  // W_r must fit with the logit tile

template <int EB>
struct NarrowShape {
  static constexpr int G = 32 / EB;  // tokens per warp (G*EB = 32 accumulators per lane)
};

// Shared-memory index (in float4 units) of W_r[d][4q..4q+3] for the chunk layout used below:
// d = 8*c + j, chunk c = 32*i + l.
template <int EB>
__device__ __forceinline__ int w_slot(int d, int q) {
  const int c = d >> 3, j = d & 7;
  const int i = c >> 5, l = c & 31;
  return (((i * 8 + j) * (EB / 4) + q) << 5) + l;
}

template <typename XT, int EB>
__global__ void __launch_bounds__(kNarrowThreads, 1) route_narrow_kernel(RouteArgs a, int KS) {
  constexpr int G = NarrowShape<EB>::G;
  constexpr int V = XVec<XT>::kElems;  // X elements per 16-byte chunk
  static_assert(V == 8 || V == 4, "chunk");
  extern __shared__ __align__(16) float n_smem[];
  float4* s_w = reinterpret_cast<float4*>(n_smem);
  const int D = a.D;
  const int E = a.E;
  const int nchunk8 = (D + 7) / 8;                   // chunks of 8 rows of W_r
  const int w_f4 = ((nchunk8 + 31) / 32) * 32 * 8 * (EB / 4);
  float* s_part = n_smem + 4 * w_f4;                 // [warps][32]
  auto s_z = reinterpret_cast<float (*)[kMaxE + 1]>(s_part + kNarrowWarps * 32);  // [tokens][E]
  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;

  // W_r -> shared memory (zero rows past D and columns past E), kFill 16-byte loads in
  // flight per thread so the copy costs a few L2 round trips, not one per element.
  {
    constexpr int kFill = 8;
    const bool vec = (E % 4) == 0;
    for (int base = threadIdx.x; base < w_f4; base += kNarrowThreads * kFill) {
      float4 v[kFill];
#pragma unroll
      for (int u = 0; u < kFill; ++u) {
        const int idx = base + u * kNarrowThreads;
        v[u] = make_float4(0.f, 0.f, 0.f, 0.f);
        if (idx < w_f4) {
          const int q = (idx >> 5) % (EB / 4);
          const int rest = (idx >> 5) / (EB / 4);  // i*8 + j
          const int d = ((rest >> 3) * 32 + (idx & 31)) * 8 + (rest & 7);
          if (d < D && 4 * q < E) {
            const float* src = a.W_r + static_cast<int64_t>(d) * E + 4 * q;
            if (vec) {
              v[u] = __ldg(reinterpret_cast<const float4*>(src));
            } else {
              float t4[4];
#pragma unroll
              for (int c = 0; c < 4; ++c) t4[c] = (4 * q + c < E) ? __ldg(src + c) : 0.f;
              v[u] = make_float4(t4[0], t4[1], t4[2], t4[3]);
            }
          }
        }
      }
#pragma unroll
      for (int u = 0; u < kFill; ++u) {
        const int idx = base + u * kNarrowThreads;
        if (idx < w_f4) s_w[idx] = v[u];
      }
    }
  }
  __syncthreads();

  const int groups_per_block = kNarrowWarps / KS;  // token groups handled together
  const int tg = warp / KS;                          // this warp's group within the block
  const int ks = warp % KS;                          // this warp's K slice
  const int tpb = groups_per_block * G;              // tokens per block step
  float colsum_acc = 0.f;
  float zl_acc = 0.f;
  const int nvec = D / V;  // 16-byte chunks of an X row

  for (int64_t step = blockIdx.x; step * tpb < a.N; step += gridDim.x) {
    const int64_t t0 = step * tpb + static_cast<int64_t>(tg) * G;
    float acc[G][EB];
#pragma unroll
    for (int g = 0; g < G; ++g)
#pragma unroll
      for (int e = 0; e < EB; ++e) acc[g][e] = 0.f;

    // This lane's chunks: c = 32*(ks + KS*i) + lane (in units of V elements).
    auto chunk_at = [&](int i) { return 32 * (ks + KS * i) + lane; };
    auto load_x = [&](int c, uint4 (&xv)[G]) {
#pragma unroll
      for (int g = 0; g < G; ++g)
        xv[g] = (c < nvec && t0 + g < a.N)
                    ? ld_stream(static_cast<const XT*>(a.X) + (t0 + g) * static_cast<int64_t>(D) +
                                static_cast<int64_t>(c) * V)
                    : make_uint4(0u, 0u, 0u, 0u);
    };
    uint4 cur[G], nxt[G];
    int c = chunk_at(0);
    load_x(c, cur);
    for (int i = 0; chunk_at(i) - lane < nvec; ++i) {
      const int cn = chunk_at(i + 1);
      load_x(cn, nxt);  // prefetch the next chunk while this one is consumed
      if (c < nvec) {
#pragma unroll
        for (int j = 0; j < V; ++j) {
          const int d = c * V + j;
          float w[EB];
#pragma unroll
          for (int q = 0; q < EB / 4; ++q) {
            const float4 f = s_w[w_slot<EB>(d, q)];
            w[4 * q] = f.x;
            w[4 * q + 1] = f.y;
            w[4 * q + 2] = f.z;
            w[4 * q + 3] = f.w;
          }
#pragma unroll
          for (int g = 0; g < G; ++g) {
            const float x = XVec<XT>::get(cur[g], j);
#pragma unroll
            for (int e = 0; e < EB; ++e) acc[g][e] = fmaf(x, w[e], acc[g][e]);
          }
        }
      }
#pragma unroll
      for (int g = 0; g < G; ++g) cur[g] = nxt[g];
      c = cn;
    }
    // Tail of D past the last full 16-byte chunk (D % V != 0): ragged scalar rows.
    for (int d = nvec * V + 32 * ks + lane; d < D; d += 32 * KS) {
      float w[EB];
#pragma unroll
      for (int q = 0; q < EB / 4; ++q) {
        const float4 f = s_w[w_slot<EB>(d, q)];
        w[4 * q] = f.x;
        w[4 * q + 1] = f.y;
        w[4 * q + 2] = f.z;
        w[4 * q + 3] = f.w;
      }
#pragma unroll
      for (int g = 0; g < G; ++g) {
        const float x =
            (t0 + g < a.N) ? XVec<XT>::one(a.X, (t0 + g) * static_cast<int64_t>(D) + d) : 0.f;
#pragma unroll
        for (int e = 0; e < EB; ++e) acc[g][e] = fmaf(x, w[e], acc[g][e]);
      }
    }
    // Butterfly reduce-scatter of the 32 partials: lane l ends with entry l.
    float v[32];
#pragma unroll
    for (int i = 0; i < 32; ++i) v[i] = acc[i / EB][i % EB];
#pragma unroll
    for (int s = 0; s < 5; ++s) {
      const int o = 16 >> s;
      const int half = 16 >> s;
      const bool upper = (lane & o) != 0;
#pragma unroll
      for (int i = 0; i < half; ++i) {
        const float send = upper ? v[i] : v[i + half];
        const float keep = upper ? v[i + half] : v[i];
        v[i] = keep + __shfl_xor_sync(0xffffffffu, send, o);
      }
    }
    s_part[warp * 32 + lane] = v[0];
    __syncthreads();
    if (ks == 0) {  // first warp of the group adds the KS slices in order
      float z = s_part[warp * 32 + lane];
      for (int r = 1; r < KS; ++r) z += s_part[(warp + r) * 32 + lane];
      const int g = lane / EB, e = lane % EB;
      if (e < E) s_z[tg * G + g][e] = z + (a.bias != nullptr ? __ldg(a.bias + e) : 0.f);
    }
    __syncthreads();
    select_tile(a, s_z, tpb, step * tpb, colsum_acc, zl_acc);
  }
  write_colsum(a, colsum_acc, zl_acc);
}

// ------------------------------------------------------------------ wide: 16 < E <= 64
//
// A block computes 128 tokens x 64 experts over D in 32-wide slices staged through shared
// memory (X converted to fp32 once and stored transposed, W_r slice as is, double buffered).
// 256 threads = 2 K halves x 128; each thread holds an 8x8 register tile made of two 4-token
// and two 4-expert halves so that every shared-memory read of a quarter warp is a contiguous
// 128-byte line. The two K halves are added in a fixed order at the end.

constexpr int kWideThreads = 256;
constexpr int kWT = 128;  // tokens per tile
constexpr int kWBK = 32;  // D slice per stage
constexpr int kXStride = kWT + 4;
constexpr int kWideSmemFloats = 2 * kWBK * kXStride + 2 * kWBK * kMaxE;

template <typename XT, bool VECW>
__global__ void __launch_bounds__(kWideThreads) route_wide_kernel(RouteArgs a) {
  constexpr int V = XVec<XT>::kElems;
  extern __shared__ __align__(16) float w_smem[];
  static_assert(kWT * (kMaxE + 1) <= kWideSmemFloats, "logit tile must fit the staging");
  auto s_x = reinterpret_cast<float (*)[kWBK][kXStride]>(w_smem);                    // [buf][d][tok]
  auto s_w = reinterpret_cast<float (*)[kWBK][kMaxE]>(w_smem + 2 * kWBK * kXStride);  // [buf][d][e]
  auto s_z = reinterpret_cast<float (*)[kMaxE + 1]>(w_smem);                         // [tok][e]
  const int tid = threadIdx.x;
  const int kh = tid >> 7;          // K half: slice rows [16*kh, 16*kh+16)
  const int ty = (tid & 127) >> 3;  // tokens 4ty..4ty+3 and 64+4ty..
  const int tx = tid & 7;           // experts 4tx..4tx+3 and 32+4tx..
  const int D = a.D;
  const int E = a.E;
  float colsum_acc = 0.f;
  float zl_acc = 0.f;
  constexpr int kChunks = kWBK / V;                      // 16-byte chunks per token per slice
  constexpr int kXLoads = kWT * kChunks / kWideThreads;  // 2 (bf16) or 4 (fp32)
  const int nslices = (D + kWBK - 1) / kWBK;

  for (int64_t tile = blockIdx.x; tile * kWT < a.N; tile += gridDim.x) {
    const int64_t t0 = tile * kWT;
    uint4 xr[kXLoads];
    float4 wr[2];
    auto load_slice = [&](int s) {
      const int d_base = s * kWBK;
#pragma unroll
      for (int q = 0; q < kXLoads; ++q) {
        const int li = tid + q * kWideThreads;
        const int tok = li % kWT;
        const int ch = li / kWT;
        const int d0 = d_base + ch * V;
        xr[q] = make_uint4(0u, 0u, 0u, 0u);
        if (t0 + tok < a.N && d0 < D)  // D % V == 0, so a started chunk is complete
          xr[q] = ld_stream(static_cast<const XT*>(a.X) + (t0 + tok) * static_cast<int64_t>(D) + d0);
      }
#pragma unroll
      for (int q = 0; q < 2; ++q) {
        const int li = tid + q * kWideThreads;  // 512 float4 = 32 rows x 64 experts
        const int row = li >> 4;
        const int col = (li & 15) * 4;
        const int d = d_base + row;
        float4 v = make_float4(0.f, 0.f, 0.f, 0.f);
        if (d < D) {
          const float* wrow = a.W_r + static_cast<int64_t>(d) * E;
          if (VECW) {
            if (col < E) v = __ldg(reinterpret_cast<const float4*>(wrow + col));
          } else {
            float t4[4];
#pragma unroll
            for (int j = 0; j < 4; ++j) t4[j] = (col + j < E) ? __ldg(wrow + col + j) : 0.f;
            v = make_float4(t4[0], t4[1], t4[2], t4[3]);
          }
        }
        wr[q] = v;
      }
    };
    auto store_slice = [&](int buf) {
#pragma unroll
      for (int q = 0; q < kXLoads; ++q) {
        const int li = tid + q * kWideThreads;
        const int tok = li % kWT;
        const int ch = li / kWT;
#pragma unroll
        for (int j = 0; j < V; ++j) s_x[buf][ch * V + j][tok] = XVec<XT>::get(xr[q], j);
      }
#pragma unroll
      for (int q = 0; q < 2; ++q) {
        const int li = tid + q * kWideThreads;
        *reinterpret_cast<float4*>(&s_w[buf][li >> 4][(li & 15) * 4]) = wr[q];
      }
    };

    float acc[8][8];
#pragma unroll
    for (int i = 0; i < 8; ++i)
#pragma unroll
      for (int j = 0; j < 8; ++j) acc[i][j] = 0.f;

    load_slice(0);
    store_slice(0);
    __syncthreads();
    for (int s = 0; s < nslices; ++s) {
      const int buf = s & 1;
      if (s + 1 < nslices) load_slice(s + 1);  // global loads in flight during the FMAs
#pragma unroll
      for (int kk = 16 * kh; kk < 16 * kh + 16; ++kk) {
        const float4 x0 = *reinterpret_cast<const float4*>(&s_x[buf][kk][4 * ty]);
        const float4 x1 = *reinterpret_cast<const float4*>(&s_x[buf][kk][64 + 4 * ty]);
        const float4 w0 = *reinterpret_cast<const float4*>(&s_w[buf][kk][4 * tx]);
        const float4 w1 = *reinterpret_cast<const float4*>(&s_w[buf][kk][32 + 4 * tx]);
        const float xs[8] = {x0.x, x0.y, x0.z, x0.w, x1.x, x1.y, x1.z, x1.w};
        const float ws[8] = {w0.x, w0.y, w0.z, w0.w, w1.x, w1.y, w1.z, w1.w};
#pragma unroll
        for (int i = 0; i < 8; ++i)
#pragma unroll
          for (int j = 0; j < 8; ++j) acc[i][j] = fmaf(xs[i], ws[j], acc[i][j]);
      }
      if (s + 1 < nslices) store_slice(buf ^ 1);
      __syncthreads();
    }
    // K half 1 parks its partial tile in s_z; K half 0 adds its own (fixed order).
    auto tok_of = [&](int i) { return i < 4 ? 4 * ty + i : 64 + 4 * ty + (i - 4); };
    auto exp_of = [&](int j) { return j < 4 ? 4 * tx + j : 32 + 4 * tx + (j - 4); };
    if (kh == 1) {
#pragma unroll
      for (int i = 0; i < 8; ++i)
#pragma unroll
        for (int j = 0; j < 8; ++j) s_z[tok_of(i)][exp_of(j)] = acc[i][j];
    }
    __syncthreads();
    if (kh == 0) {
#pragma unroll
      for (int i = 0; i < 8; ++i)
#pragma unroll
        for (int j = 0; j < 8; ++j) {
          const int e = exp_of(j);
          const float b = (a.bias != nullptr && e < E) ? __ldg(a.bias + e) : 0.f;
          s_z[tok_of(i)][e] = (acc[i][j] + s_z[tok_of(i)][e]) + b;
        }
    }
    __syncthreads();
    select_tile(a, s_z, kWT, t0, colsum_acc, zl_acc);
  }
  write_colsum(a, colsum_acc, zl_acc);
}

// ------------------------------------------------------------------ routing from given logits

constexpr int kSelThreads = 64;

__global__ void __launch_bounds__(kSelThreads) route_select_kernel(RouteArgs a) {
  __shared__ float s_z[kSelThreads][kMaxE + 1];
  float colsum_acc = 0.f;
  float zl_acc = 0.f;
  const int E = a.E;
  for (int64_t tile = blockIdx.x; tile * kSelThreads < a.N; tile += gridDim.x) {
    const int64_t t0 = tile * kSelThreads;
    for (int i = threadIdx.x; i < kSelThreads * E; i += kSelThreads) {
      const int tl = i / E;
      const int e = i % E;
      if (t0 + tl < a.N) s_z[tl][e] = a.logits_in[(t0 + tl) * E + e];
    }
    __syncthreads();
    select_tile(a, s_z, kSelThreads, t0, colsum_acc, zl_acc);
  }
  write_colsum(a, colsum_acc, zl_acc);
}

// z_loss = (sum over blocks, in block order, of the per-block sums of (log Z)^2) / N.
__global__ void zloss_reduce_kernel(const float* __restrict__ partial, int nblocks, int64_t N,
                                    float* __restrict__ out) {
  if (threadIdx.x != 0) return;
  float s = 0.f;
  for (int b = 0; b < nblocks; ++b) s += partial[b];
  out[0] = N > 0 ? s / static_cast<float>(N) : 0.f;
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

enum class Kind { kNarrow, kWide, kSelect };

int expert_block(int E) { return E <= 4 ? 4 : (E <= 8 ? 8 : 16); }

size_t narrow_smem_bytes(int D, int EB) {
  const int nchunk8 = (D + 7) / 8;
  const size_t w_f4 = static_cast<size_t>((nchunk8 + 31) / 32) * 32 * 8 * (EB / 4);
  const size_t tpb_max = static_cast<size_t>(kNarrowWarps) * (32 / EB);
  return w_f4 * 16 + kNarrowWarps * 32 * 4 + tpb_max * (kMaxE + 1) * 4;
}

Kind kind_of(const void* X, int E, int D) {
  if (X == nullptr) return Kind::kSelect;
  if (E <= 16 && narrow_smem_bytes(D, expert_block(E)) <= kNarrowMaxSmemBytes)
    return Kind::kNarrow;
  return Kind::kWide;
}

// K split of the narrow kernel: as many warps per token group as keep every SM's 16 warps busy.
int narrow_ks(int64_t N, int E) {
  const int64_t groups = (N + (32 / expert_block(E)) - 1) / (32 / expert_block(E));
  const int64_t warps = static_cast<int64_t>(num_sms()) * kNarrowWarps;
  int ks = 1;
  while (ks < kNarrowWarps && groups * ks * 2 <= warps) ks *= 2;
  return ks;
}

template <typename XT>
cudaError_t launch_narrow(const RouteArgs& a, int EB, int ks, cudaStream_t s) {
  const int tpb = (kNarrowWarps / ks) * (32 / EB);
  const int64_t steps = (a.N + tpb - 1) / tpb;
  const int grid = static_cast<int>(
      std::max<int64_t>(1, std::min<int64_t>(std::min<int64_t>(steps, num_sms()), kMaxBlocks)));
  const size_t smem = narrow_smem_bytes(a.D, EB);
  cudaError_t e = cudaSuccess;
  if (EB == 4) {
    e = cudaFuncSetAttribute(route_narrow_kernel<XT, 4>, cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(smem));
    if (e == cudaSuccess) route_narrow_kernel<XT, 4><<<grid, kNarrowThreads, smem, s>>>(a, ks);
  } else if (EB == 8) {
    e = cudaFuncSetAttribute(route_narrow_kernel<XT, 8>, cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(smem));
    if (e == cudaSuccess) route_narrow_kernel<XT, 8><<<grid, kNarrowThreads, smem, s>>>(a, ks);
  } else {
    e = cudaFuncSetAttribute(route_narrow_kernel<XT, 16>, cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(smem));
    if (e == cudaSuccess) route_narrow_kernel<XT, 16><<<grid, kNarrowThreads, smem, s>>>(a, ks);
  }
  return e != cudaSuccess ? e : cudaGetLastError();
}

template <typename XT>
cudaError_t launch_wide(const RouteArgs& a, int grid, bool vecw, cudaStream_t s) {
  const int smem = kWideSmemFloats * 4;
  cudaError_t e;
  if (vecw) {
    e = cudaFuncSetAttribute(route_wide_kernel<XT, true>, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
    if (e == cudaSuccess) route_wide_kernel<XT, true><<<grid, kWideThreads, smem, s>>>(a);
  } else {
    e = cudaFuncSetAttribute(route_wide_kernel<XT, false>, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
    if (e == cudaSuccess) route_wide_kernel<XT, false><<<grid, kWideThreads, smem, s>>>(a);
  }
  return e != cudaSuccess ? e : cudaGetLastError();
}

}  // namespace

int route_num_blocks(int64_t N, int E) {
  // Every router grid is capped at kMaxBlocks (workspace sizing, device independent).
  (void)N;
  (void)E;
  return kMaxBlocks;
}

cudaError_t launch_route(const moe_problem& p, const void* X, const float* W_r, const float* bias,
                         const float* noise, float* logits, int32_t* idx, float* gate,
                         float* colsum_partial, float* prob_colsum, float* zl_partial,
                         float* z_loss, void* operand, int* err, uint64_t timeout_ns,
                         cudaStream_t stream) {
  if (p.N == 0) return cudaSuccess;
  RouteArgs a;
  a.noise = p.routing_mode != MOE_ROUTE_TOPK ? noise : nullptr;
  a.mode = p.routing_mode;
  a.zl_partial = z_loss != nullptr ? zl_partial : nullptr;
  a.X = X;
  a.W_r = W_r;
  a.bias = bias;
  a.logits_in = X == nullptr ? logits : nullptr;
  a.logits_out = X != nullptr ? logits : nullptr;
  a.idx = idx;
  a.gate = gate;
  a.colsum_partial = prob_colsum != nullptr ? colsum_partial : nullptr;
  a.N = p.N;
  a.D = static_cast<int>(p.D);
  a.E = p.E;
  a.k = p.k;
  a.renorm = p.renormalize;
  const Kind kind = kind_of(X, p.E, a.D);
  int grid = 1;
  cudaError_t e = cudaSuccess;
  if (X != nullptr && route_tc_supported(p)) {
    // bf16 activations: one tensor-core kernel computes the logits and routes.
    e = launch_route_tc(p, X, W_r, bias, a.noise, a.logits_out, idx, gate, a.colsum_partial,
                        a.zl_partial, operand, &grid, err, timeout_ns, stream);
  } else if (kind == Kind::kSelect) {
    grid = static_cast<int>(std::max<int64_t>(
        1, std::min<int64_t>((p.N + kSelThreads - 1) / kSelThreads, kMaxBlocks)));
    route_select_kernel<<<grid, kSelThreads, 0, stream>>>(a);
    e = cudaGetLastError();
  } else if (kind == Kind::kNarrow) {
    const int EB = expert_block(p.E);
    const int ks = narrow_ks(p.N, p.E);
    const int tpb = (kNarrowWarps / ks) * (32 / EB);
    grid = static_cast<int>(std::max<int64_t>(
        1, std::min<int64_t>(std::min<int64_t>((p.N + tpb - 1) / tpb, num_sms()), kMaxBlocks)));
    e = launch_narrow<float>(a, EB, ks, stream);  // fp32 X (bf16 X takes the tensor cores)
  } else {
    grid = static_cast<int>(
        std::max<int64_t>(1, std::min<int64_t>((p.N + kWT - 1) / kWT, kMaxBlocks)));
    const bool vecw = (p.E % 4) == 0;
    e = launch_wide<float>(a, grid, vecw, stream);
  }
  if (e != cudaSuccess) return e;
  if (prob_colsum != nullptr) {
    colsum_reduce_kernel<<<1, kMaxE, 0, stream>>>(colsum_partial, grid, p.E, prob_colsum);
    e = cudaGetLastError();
    if (e != cudaSuccess) return e;
  }
  if (z_loss != nullptr) {
    zloss_reduce_kernel<<<1, 32, 0, stream>>>(zl_partial, grid, p.N, z_loss);
    e = cudaGetLastError();
  }
  return e;
}

}  // namespace moe

// Dispatch: expert load histogram, capacity, slot-major position assignment, drop mask,
// expert-contiguous row map, and the permutation of token rows into expert order.
//   MoE formula-to-code walkthrough 1.3 (load = bincount of the routed experts), 3.1
//   (capacity), 3.2 (dispatch with a dropped mask); LLMs-from-scratch ch.12, 12.2 (N*k
//   dispatch records); MoE series (GShard/Mixtral/Switch) 2.2 (overflow).
//
// Record order: slot-major r = j*N + t (all rank-0 records in token order, then rank 1 ...)
// or token-major r = t*k + j (the walkthrough's loop, 3.2), per the problem's capacity_order.
// pos(t,j) = number of earlier records (in that order) routed to the same expert.
//   pass 1 (count): records are split into chunks of kDispatchChunk; each block counts its
//                   chunk per expert (integer shared-memory counters: order-free, exact).
//   pass 2 (assign): each block sums the counts of the chunks before it (a few hundred ints),
//                   then walks its chunk in tiles of 1024 records; inside a tile, warps rank
//                   equal experts with __match_any_sync, and a per-expert scan over the 32
//                   warps orders the warps. The result is the stable counting-sort rank --
//                   bit-exact and independent of scheduling.
// Gather: one warp per block; lane 0 streams 16-KB pieces of rows global -> shared -> global
// with bulk copies (cp.async.bulk), keeping up to kGatherStages pieces in flight.
#include <algorithm>

#include "common.cuh"
#include "internal.h"

namespace moe {
namespace {

constexpr int kMaxE = 64;
constexpr int kAssignThreads = 1024;  // 32 warps: one tile = one chunk
constexpr int kCountThreads = 256;

// Token and rank of the r-th record in the visiting order.
__device__ __forceinline__ void record_at(int64_t r, int64_t N, int k, bool token_major,
                                          int64_t& t, int64_t& j) {
  if (token_major) {
    t = r / k;
    j = r - t * k;
  } else {
    j = r / N;
    t = r - j * N;
  }
}

__global__ void __launch_bounds__(kCountThreads)
    count_kernel(const int32_t* __restrict__ idx, int64_t N, int k, int E, int64_t R,
                 bool token_major, int32_t* __restrict__ counts, int* err) {
  __shared__ int hist[kMaxE];
  for (int e = threadIdx.x; e < E; e += blockDim.x) hist[e] = 0;
  __syncthreads();
  const int64_t r0 = static_cast<int64_t>(blockIdx.x) * kDispatchChunk;
  const int64_t r1 = std::min<int64_t>(r0 + kDispatchChunk, R);
  constexpr int kPer = kDispatchChunk / kCountThreads;  // records per thread, loaded together
  int ev[kPer];
#pragma unroll
  for (int u = 0; u < kPer; ++u) {
    const int64_t r = r0 + threadIdx.x + static_cast<int64_t>(u) * kCountThreads;
    ev[u] = -1;
    if (r < r1) {
      int64_t t, j;
      record_at(r, N, k, token_major, t, j);
      ev[u] = idx[t * k + j];
      if (ev[u] < 0 || ev[u] >= E) {
        record_error(err, MOE_DEVERR_BAD_INDEX);
        ev[u] = -1;
      }
    }
  }
#pragma unroll
  for (int u = 0; u < kPer; ++u)
    if (ev[u] >= 0) atomicAdd(&hist[ev[u]], 1);
  __syncthreads();
  for (int e = threadIdx.x; e < E; e += blockDim.x)
    counts[static_cast<int64_t>(blockIdx.x) * E + e] = hist[e];
}

__global__ void __launch_bounds__(kAssignThreads)
    assign_kernel(const int32_t* __restrict__ idx, int64_t N, int k, int E, int64_t R,
                  bool token_major, int64_t C, int nchunks, const int32_t* __restrict__ counts,
                  int32_t* __restrict__ load, int32_t* __restrict__ offsets,
                  int32_t* __restrict__ pos, uint8_t* __restrict__ dropped,
                  int32_t* __restrict__ row_token) {
  __shared__ int s_base[kMaxE];   // records of expert e in earlier chunks
  __shared__ int s_off[kMaxE + 1];  // first row of expert e in the expert-contiguous order
  __shared__ int s_wpre[32][kMaxE];  // per-warp running prefix of the current tile

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  if (threadIdx.x < E) {
    const int e = threadIdx.x;
    int base = 0, total = 0;
    for (int c = 0; c < nchunks; ++c) {
      const int v = counts[static_cast<int64_t>(c) * E + e];
      if (c < static_cast<int>(blockIdx.x)) base += v;
      total += v;
    }
    s_base[e] = base;
    s_wpre[0][e] = total;  // temporary: totals, consumed below
  }
  __syncthreads();
  if (threadIdx.x == 0) {
    int run = 0;
    for (int e = 0; e < E; ++e) {
      s_off[e] = run;
      const int64_t tot = s_wpre[0][e];
      run += static_cast<int>(tot < C ? tot : C);
    }
    s_off[E] = run;
    if (blockIdx.x == 0) {
      for (int e = 0; e < E; ++e) {
        load[e] = s_wpre[0][e];
        offsets[e] = s_off[e];
      }
      offsets[E] = run;
    }
  }
  __syncthreads();

  int running = 0;  // thread e < E: records of expert e seen in earlier tiles of this chunk
  const int64_t r0 = static_cast<int64_t>(blockIdx.x) * kDispatchChunk;
  const int64_t r1 = std::min<int64_t>(r0 + kDispatchChunk, R);
  const unsigned lt_mask = (1u << lane) - 1u;
  for (int64_t tile = r0; tile < r1; tile += kAssignThreads) {
    for (int i = threadIdx.x; i < 32 * kMaxE; i += kAssignThreads) (&s_wpre[0][0])[i] = 0;
    __syncthreads();
    const int64_t r = tile + threadIdx.x;
    const bool valid = r < r1;
    int64_t j = 0, t = 0;
    int e = -1;
    if (valid) {
      record_at(r, N, k, token_major, t, j);
      e = idx[t * k + j];
      if (e < 0 || e >= E) e = -1;  // recorded by the count pass
    }
    const unsigned peers = __match_any_sync(0xffffffffu, valid ? e : -2);
    const int rank = __popc(peers & lt_mask);
    if (valid && e >= 0 && rank == 0) s_wpre[warp][e] = __popc(peers);
    __syncthreads();
    if (threadIdx.x < E) {
      const int ee = threadIdx.x;
      int run = running;
      for (int w = 0; w < 32; ++w) {
        const int c = s_wpre[w][ee];
        s_wpre[w][ee] = run;
        run += c;
      }
      running = run;
    }
    __syncthreads();
    if (valid) {
      const int64_t rec = t * k + j;
      if (e >= 0) {
        const int p = s_base[e] + s_wpre[warp][e] + rank;
        const bool drop = p >= C;
        pos[rec] = p;
        dropped[rec] = drop ? 1 : 0;
        if (!drop && row_token != nullptr) row_token[s_off[e] + p] = static_cast<int32_t>(t);
      } else {
        pos[rec] = -1;
        dropped[rec] = 1;
      }
    }
    __syncthreads();
  }
}

constexpr int kGatherMaxStages = 16;
constexpr uint32_t kMaxPieceBytes = 16384;
constexpr uint32_t kGatherSmem = 64 * 1024;
constexpr uint64_t kGatherTimeoutNs = 2000000000ull;

// One warp per block. A row is copied in pieces of piece_bytes (= the row when it is at most
// 16 KB); piece q = blockIdx.x + i*gridDim.x covers bytes [(q % P) * piece_bytes, ...) of row
// q / P. `stages` pieces (64 KB of shared memory / piece size, at most 16) are in flight.
__global__ void __launch_bounds__(32)
    gather_kernel(const uint8_t* __restrict__ X, const int32_t* __restrict__ row_token,
                  const int32_t* __restrict__ offsets, int E, uint32_t row_bytes,
                  uint32_t piece_bytes, int stages, uint8_t* __restrict__ X_perm, int* err) {
  extern __shared__ __align__(128) uint8_t g_smem[];
  __shared__ __align__(8) uint64_t bars[kGatherMaxStages];
  const int lane = threadIdx.x;
  const int64_t rows = offsets[E];
  const int64_t P = (row_bytes + piece_bytes - 1) / piece_bytes;
  const int64_t total = rows * P;
  if (static_cast<int64_t>(blockIdx.x) >= total) return;
  const int64_t n = (total - blockIdx.x + gridDim.x - 1) / gridDim.x;  // pieces of this block

  if (lane == 0) {
    for (int s = 0; s < stages; ++s) mbar_init(&bars[s], 1);
    fence_barrier_init();
  }
  __syncwarp();

  auto piece = [&](int64_t i, int64_t& row, uint32_t& off, uint32_t& bytes) {
    const int64_t q = blockIdx.x + i * gridDim.x;
    row = q / P;
    off = static_cast<uint32_t>((q - row * P) * piece_bytes);
    const uint32_t rest = row_bytes - off;
    bytes = rest < piece_bytes ? rest : piece_bytes;
  };
  // Token of the row of load index i, fetched 32 at a time by the whole warp.
  int tok_batch = -1;
  int64_t batch_base = -1;
  auto token_of = [&](int64_t i) -> int {
    const int64_t b = i & ~static_cast<int64_t>(31);
    if (b != batch_base) {
      batch_base = b;
      const int64_t li = b + lane;
      tok_batch = 0;
      if (li < n) {
        int64_t row;
        uint32_t off, bytes;
        piece(li, row, off, bytes);
        tok_batch = row_token[row];
      }
    }
    return __shfl_sync(0xffffffffu, tok_batch, static_cast<int>(i - b));
  };
  auto issue_load = [&](int64_t i) {
    int64_t row;
    uint32_t off, bytes;
    piece(i, row, off, bytes);
    const int tok = token_of(i);
    if (lane == 0) {
      const int s = static_cast<int>(i % stages);
      mbar_arrive_expect_tx(&bars[s], bytes);
      bulk_g2s(g_smem + static_cast<uint32_t>(s) * piece_bytes,
               X + static_cast<int64_t>(tok) * row_bytes + off, bytes, &bars[s]);
    }
  };

  const int64_t pro = n < stages ? n : stages;
  for (int64_t i = 0; i < pro; ++i) issue_load(i);
  int64_t issued = pro;  // loads [0, issued) have been issued
  int64_t i = 0;
  bool ok = true;
  for (; i < n; ++i) {
    const int s = static_cast<int>(i % stages);
    const uint32_t parity = static_cast<uint32_t>((i / stages) & 1);
    if (lane == 0) ok = mbar_wait(&bars[s], parity, kGatherTimeoutNs);
    ok = __shfl_sync(0xffffffffu, ok ? 1 : 0, 0) != 0;
    if (!ok) {
      if (lane == 0) record_error(err, MOE_DEVERR_WAIT_TIMEOUT);
      break;
    }
    if (lane == 0) {
      int64_t row;
      uint32_t off, bytes;
      piece(i, row, off, bytes);
      bulk_s2g(X_perm + row * row_bytes + off, g_smem + static_cast<uint32_t>(s) * piece_bytes,
               bytes);
      bulk_commit();
    }
    const int64_t nxt = i - 1 + stages;  // refill the stage read by store i-1
    if (i >= 1 && nxt < n) {
      if (lane == 0) bulk_wait_read<1>();
      __syncwarp();
      issue_load(nxt);
      issued = nxt + 1;
    }
  }
  if (lane == 0) {
    bulk_wait_all();
    // After a timeout, loads [i, issued) may still be landing in shared memory: wait for
    // each of them (bounded) before the block exits.
    for (int64_t L = i; !ok && L < issued; ++L)
      (void)mbar_wait(&bars[L % stages], static_cast<uint32_t>((L / stages) & 1),
                      kGatherTimeoutNs / 16);
  }
}

// dst[i] = src[index[i]] for i < n_rows: one warp per row, 16-byte words when the row length
// allows (else 4-byte words). An index outside [0, n_src) is recorded as MOE_DEVERR_BAD_INDEX
// and its row is zero-filled instead of read.
__global__ void __launch_bounds__(256)
    gather_rows_kernel(const uint8_t* __restrict__ src, int64_t n_src,
                       const int32_t* __restrict__ index, int64_t n_rows, int64_t row_bytes,
                       uint8_t* __restrict__ dst, int* err) {
  const int lane = threadIdx.x & 31;
  const int64_t wpb = blockDim.x >> 5;
  const int64_t nwarps = static_cast<int64_t>(gridDim.x) * wpb;
  const bool wide = (row_bytes & 15) == 0;
  for (int64_t i = blockIdx.x * wpb + (threadIdx.x >> 5); i < n_rows; i += nwarps) {
    const int64_t r = index[i];
    uint8_t* d = dst + i * row_bytes;
    const bool bad = r < 0 || r >= n_src;
    if (bad && lane == 0) record_error(err, MOE_DEVERR_BAD_INDEX);
    const uint8_t* s = src + (bad ? 0 : r) * row_bytes;
    if (wide) {
      const int64_t words = row_bytes >> 4;
      for (int64_t j = lane; j < words; j += 32)
        reinterpret_cast<uint4*>(d)[j] =
            bad ? make_uint4(0, 0, 0, 0) : __ldg(reinterpret_cast<const uint4*>(s) + j);
    } else {
      const int64_t words = row_bytes >> 2;
      for (int64_t j = lane; j < words; j += 32)
        reinterpret_cast<uint32_t*>(d)[j] =
            bad ? 0u : __ldg(reinterpret_cast<const uint32_t*>(s) + j);
    }
  }
}

// ------------------------------------------------------------------ fused dispatch
//
// Count, slot assignment and gather in one cooperative launch (every block resident at
// once). Phase 1: blocks b < nchunks count chunk b (kDispatchChunk records) per expert (as
// count_kernel). Grid barrier. Phase 2: block b takes the b-th of G equal slices of the
// records; an expert's records before the slice are the counts of the earlier chunks plus a
// recount of the slice's own chunk up to the slice start; inside the slice, warps rank equal
// experts with __match_any_sync and a per-expert scan over the warps orders them (the stable
// counting-sort rank, as assign_kernel). The block writes its records' positions, drop flags
// and row map (block 0 also load and offsets) and copies the X rows of its kept records to
// X_perm straight away (one warp per row, 16-byte words, four loads in flight per lane): no
// second barrier, and every block has copy work. Counts another block wrote are read at L2
// (ld.global.cg). The barrier counters live in the workspace header (zero at rest); the last
// block to finish returns them to zero, also after the barrier timed out. Bit-exact with the
// three-kernel path.

constexpr int kFusedThreads = 512;

struct FusedArgs {
  const int32_t* idx;
  const uint8_t* X;        // nullptr: no gather (phase 3 and its barrier are skipped)
  uint8_t* X_perm;
  int32_t* counts;         // [nchunks][E]
  int32_t* load;
  int32_t* offsets;
  int32_t* pos;
  uint8_t* dropped;
  int32_t* row_token;
  int* err;
  int* bar;                // [2]: barrier arrivals (one or two per block), blocks finished
  int64_t N, R, C;
  int k, E, nchunks;
  bool token_major;
  uint32_t row_words;      // 16-byte words per row
  uint64_t timeout_ns;
};

// Arrive on the grid barrier and wait until `target` arrivals have been made (bounded).
// Returns false to every thread of the block when the wait ran out.
__device__ bool grid_barrier(int* bar, int target, uint64_t timeout_ns, int* err) {
  __shared__ int s_ok;
  __syncthreads();
  if (threadIdx.x == 0) {
    __threadfence();  // this block's writes before its arrival
    atomicAdd(bar, 1);
    int ok = 1;
    const uint64_t t0 = globaltimer_ns();
    while (true) {
      int v;
      asm volatile("ld.acquire.gpu.global.b32 %0, [%1];" : "=r"(v) : "l"(bar) : "memory");
      if (v >= target) break;
      if (globaltimer_ns() - t0 > timeout_ns) {
        ok = 0;
        record_error(err, MOE_DEVERR_WAIT_TIMEOUT);
        break;
      }
    }
    __threadfence();
    s_ok = ok;
  }
  __syncthreads();
  return s_ok != 0;
}

__global__ void __launch_bounds__(kFusedThreads) dispatch_fused_kernel(FusedArgs a) {
  __shared__ int hist[kMaxE];
  __shared__ int s_base[kMaxE];
  __shared__ int s_tot[kMaxE];
  __shared__ int s_off[kMaxE + 1];
  __shared__ int s_wpre[kFusedThreads / 32][kMaxE];
  __shared__ int s_row[kFusedThreads];      // X_perm row of each record of the tile (-1: none)
  __shared__ int32_t s_tok[kFusedThreads];  // and its token
  const int E = a.E;
  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  constexpr int kWarps = kFusedThreads / 32;
  const int G = static_cast<int>(gridDim.x);
  bool ok = true;
  pdl_wait();  // idx (and X) come from the previous kernels
  pdl_trigger();

  // Phase 1: per-chunk histograms.
  for (int c = blockIdx.x; c < a.nchunks; c += G) {
    for (int e = threadIdx.x; e < E; e += kFusedThreads) hist[e] = 0;
    __syncthreads();
    const int64_t r0 = static_cast<int64_t>(c) * kDispatchChunk;
    const int64_t r1 = std::min<int64_t>(r0 + kDispatchChunk, a.R);
    for (int64_t r = r0 + threadIdx.x; r < r1; r += kFusedThreads) {
      int64_t t, j;
      record_at(r, a.N, a.k, a.token_major, t, j);
      const int e = a.idx[t * a.k + j];
      if (e < 0 || e >= E) record_error(a.err, MOE_DEVERR_BAD_INDEX);
      else atomicAdd(&hist[e], 1);
    }
    __syncthreads();
    for (int e = threadIdx.x; e < E; e += kFusedThreads)
      a.counts[static_cast<int64_t>(c) * E + e] = hist[e];
    __syncthreads();
  }
  ok = grid_barrier(a.bar, G, a.timeout_ns, a.err);

  // Phase 2: this block's slice [s0, s1) of the records.
  const int64_t slice = (a.R + G - 1) / G;
  const int64_t s0 = std::min<int64_t>(a.R, static_cast<int64_t>(blockIdx.x) * slice);
  const int64_t s1 = std::min<int64_t>(a.R, s0 + slice);
  if (ok && s0 < s1) {
    const int c0 = static_cast<int>(s0 / kDispatchChunk);
    for (int e = threadIdx.x; e < E; e += kFusedThreads) hist[e] = 0;
    __syncthreads();
    // Recount the records of chunk c0 before s0.
    for (int64_t r = static_cast<int64_t>(c0) * kDispatchChunk + threadIdx.x; r < s0;
         r += kFusedThreads) {
      int64_t t, j;
      record_at(r, a.N, a.k, a.token_major, t, j);
      const int e = a.idx[t * a.k + j];
      if (e >= 0 && e < E) atomicAdd(&hist[e], 1);
    }
    if (threadIdx.x < E) {
      const int e = threadIdx.x;
      int base = 0, total = 0;
      for (int cc = 0; cc < a.nchunks; ++cc) {
        const int v = __ldcg(a.counts + static_cast<int64_t>(cc) * E + e);
        if (cc < c0) base += v;
        total += v;
      }
      s_base[e] = base;
      s_tot[e] = total;
    }
    __syncthreads();
    if (threadIdx.x < E) s_base[threadIdx.x] += hist[threadIdx.x];
    if (threadIdx.x == 0) {
      int run = 0;
      for (int e = 0; e < E; ++e) {
        s_off[e] = run;
        const int64_t tot = s_tot[e];
        run += static_cast<int>(tot < a.C ? tot : a.C);
      }
      s_off[E] = run;
      if (blockIdx.x == 0) {
        for (int e = 0; e < E; ++e) {
          a.load[e] = s_tot[e];
          a.offsets[e] = s_off[e];
        }
        a.offsets[E] = run;
      }
    }
    __syncthreads();
    int running = 0;  // thread e < E: records of expert e in earlier tiles of this slice
    const unsigned lt_mask = (1u << lane) - 1u;
    const uint32_t words = a.row_words;
    for (int64_t tile = s0; tile < s1; tile += kFusedThreads) {
      for (int i = threadIdx.x; i < kWarps * kMaxE; i += kFusedThreads) (&s_wpre[0][0])[i] = 0;
      __syncthreads();
      const int64_t r = tile + threadIdx.x;
      const bool valid = r < s1;
      int64_t j = 0, t = 0;
      int e = -1;
      if (valid) {
        record_at(r, a.N, a.k, a.token_major, t, j);
        e = a.idx[t * a.k + j];
        if (e < 0 || e >= E) e = -1;  // recorded in phase 1
      }
      const unsigned peers = __match_any_sync(0xffffffffu, valid ? e : -2);
      const int rank = __popc(peers & lt_mask);
      if (valid && e >= 0 && rank == 0) s_wpre[warp][e] = __popc(peers);
      __syncthreads();
      if (threadIdx.x < E) {
        const int ee = threadIdx.x;
        int run = running;
        for (int w = 0; w < kWarps; ++w) {
          const int cnt = s_wpre[w][ee];
          s_wpre[w][ee] = run;
          run += cnt;
        }
        running = run;
      }
      __syncthreads();
      int my_row = -1;
      if (valid) {
        const int64_t rec = t * a.k + j;
        if (e >= 0) {
          const int p = s_base[e] + s_wpre[warp][e] + rank;
          const bool drop = p >= a.C;
          a.pos[rec] = p;
          a.dropped[rec] = drop ? 1 : 0;
          if (!drop) {
            my_row = s_off[e] + p;
            a.row_token[my_row] = static_cast<int32_t>(t);
          }
        } else {
          a.pos[rec] = -1;
          a.dropped[rec] = 1;
        }
      }
      if (a.X != nullptr) {
        // Copy the kept rows of this tile, spread over all warps of the block.
        s_row[threadIdx.x] = my_row;
        s_tok[threadIdx.x] = static_cast<int32_t>(t);
        __syncthreads();
        const int n_here = static_cast<int>(std::min<int64_t>(kFusedThreads, s1 - tile));
        for (int i = warp; i < n_here; i += kWarps) {
          const int row = s_row[i];
          if (row < 0) continue;
          const int64_t tok = s_tok[i];
          const uint4* src = reinterpret_cast<const uint4*>(a.X) + tok * words;
          uint4* dst = reinterpret_cast<uint4*>(a.X_perm) + static_cast<int64_t>(row) * words;
          uint32_t w = lane;
          for (; w + 96 < words; w += 128) {
            const uint4 v0 = __ldg(src + w), v1 = __ldg(src + w + 32),
                        v2 = __ldg(src + w + 64), v3 = __ldg(src + w + 96);
            dst[w] = v0;
            dst[w + 32] = v1;
            dst[w + 64] = v2;
            dst[w + 96] = v3;
          }
          for (; w < words; w += 32) dst[w] = __ldg(src + w);
        }
      }
      __syncthreads();
    }
  }

  // Last block out returns the barrier counters to zero for the next launch.
  __syncthreads();
  if (threadIdx.x == 0) {
    __threadfence();
    if (atomicAdd(&a.bar[1], 1) == G - 1) {
      atomicExch(&a.bar[0], 0);
      atomicExch(&a.bar[1], 0);
    }
  }
}

}  // namespace

cudaError_t launch_gather_rows(const void* src, int64_t n_src, const int32_t* index,
                               int64_t n_rows, int64_t row_bytes, void* dst, int* err,
                               cudaStream_t stream) {
  if (n_rows == 0) return cudaSuccess;
  const int64_t blocks = std::min<int64_t>((n_rows + 7) / 8, int64_t(num_sms()) * 8);
  gather_rows_kernel<<<static_cast<unsigned>(blocks), 256, 0, stream>>>(
      static_cast<const uint8_t*>(src), n_src, index, n_rows, row_bytes,
      static_cast<uint8_t*>(dst), err);
  return cudaGetLastError();
}

int dispatch_num_chunks(int64_t records) {
  return static_cast<int>(std::max<int64_t>(1, (records + kDispatchChunk - 1) / kDispatchChunk));
}

cudaError_t launch_slot_assign(const moe_problem& p, int64_t capacity, const int32_t* idx,
                               int32_t* chunk_counts, int32_t* load, int32_t* offsets,
                               int32_t* pos, uint8_t* dropped, int32_t* row_token, int* err,
                               cudaStream_t stream) {
  const int64_t R = p.N * p.k;
  if (R == 0) {
    cudaError_t e = cudaMemsetAsync(load, 0, sizeof(int32_t) * p.E, stream);
    if (e != cudaSuccess) return e;
    return cudaMemsetAsync(offsets, 0, sizeof(int32_t) * (p.E + 1), stream);
  }
  const int nchunks = dispatch_num_chunks(R);
  const bool token_major = p.capacity_order == MOE_ORDER_TOKEN_MAJOR;
  count_kernel<<<nchunks, kCountThreads, 0, stream>>>(idx, p.N, p.k, p.E, R, token_major,
                                                     chunk_counts, err);
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  assign_kernel<<<nchunks, kAssignThreads, 0, stream>>>(idx, p.N, p.k, p.E, R, token_major,
                                                       capacity, nchunks, chunk_counts, load,
                                                       offsets, pos, dropped, row_token);
  return cudaGetLastError();
}

cudaError_t launch_gather(const moe_problem& p, const void* X, const int32_t* row_token,
                          const int32_t* offsets, void* X_perm, int* err, cudaStream_t stream) {
  const int64_t R = p.N * p.k;
  if (R == 0) return cudaSuccess;
  const uint32_t elem = p.dtype == MOE_DTYPE_BF16 ? 2u : 4u;
  const uint32_t row_bytes = static_cast<uint32_t>(p.D) * elem;
  const uint32_t piece = row_bytes < kMaxPieceBytes ? row_bytes : kMaxPieceBytes;
  const int stages = static_cast<int>(std::min<uint32_t>(kGatherMaxStages, kGatherSmem / piece));
  const int64_t P = (row_bytes + piece - 1) / piece;
  const int64_t max_pieces = R * P;
  const int grid = static_cast<int>(std::min<int64_t>(max_pieces, int64_t(num_sms()) * 3));
  const size_t smem = static_cast<size_t>(stages) * piece;
  cudaError_t e = cudaFuncSetAttribute(
      gather_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(kGatherSmem));
  if (e != cudaSuccess) return e;
  gather_kernel<<<grid, 32, smem, stream>>>(static_cast<const uint8_t*>(X), row_token, offsets,
                                            p.E, row_bytes, piece, stages,
                                            static_cast<uint8_t*>(X_perm), err);
  return cudaGetLastError();
}

// Blocks of the fused dispatch that fit on the device at once (cached per device).
int fused_max_blocks() {
  static int cache[64] = {0};
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return 0;
  if (cache[dev] == 0) {
    int per_sm = 0;
    if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, dispatch_fused_kernel,
                                                      kFusedThreads, 0) != cudaSuccess ||
        per_sm <= 0) {
      (void)cudaGetLastError();
      per_sm = -1;
    }
    cache[dev] = per_sm > 0 ? per_sm * num_sms() : -1;
  }
  return cache[dev] > 0 ? cache[dev] : 0;
}

cudaError_t launch_dispatch_fused(const moe_problem& p, int64_t capacity, const int32_t* idx,
                                  int32_t* chunk_counts, int32_t* load, int32_t* offsets,
                                  int32_t* pos, uint8_t* dropped, int32_t* row_token,
                                  const void* X, void* X_perm, int* err, int* bar,
                                  uint64_t timeout_ns, cudaStream_t stream) {
  const int64_t R = p.N * p.k;
  const int nchunks = dispatch_num_chunks(R);
  const uint32_t elem = p.dtype == MOE_DTYPE_BF16 ? 2u : 4u;
  const int max_blocks = fused_max_blocks();
  if (R == 0 || max_blocks < 1 || (static_cast<int64_t>(p.D) * elem) % 16 != 0) {
    // Nothing to fuse (or no resident grid): the three-kernel path.
    cudaError_t e = launch_slot_assign(p, capacity, idx, chunk_counts, load, offsets, pos,
                                       dropped, row_token, err, stream);
    if (e != cudaSuccess || X == nullptr) return e;
    return launch_gather(p, X, row_token, offsets, X_perm, err, stream);
  }
  FusedArgs a;
  a.idx = idx;
  a.X = static_cast<const uint8_t*>(X);
  a.X_perm = static_cast<uint8_t*>(X_perm);
  a.counts = chunk_counts;
  a.load = load;
  a.offsets = offsets;
  a.pos = pos;
  a.dropped = dropped;
  a.row_token = row_token;
  a.err = err;
  a.bar = bar;
  a.N = p.N;
  a.R = R;
  a.C = capacity;
  a.k = p.k;
  a.E = p.E;
  a.nchunks = nchunks;
  a.token_major = p.capacity_order == MOE_ORDER_TOKEN_MAJOR;
  a.row_words = static_cast<uint32_t>(static_cast<int64_t>(p.D) * elem / 16);
  a.timeout_ns = timeout_ns;
  // With rows to copy, a block per 96 KB of rows up to every resident block (the copy spread
  // over the device; small batches keep the grid barrier small); without, one block per 512
  // records. At least one block per chunk.
  const int64_t copy_bytes = R * static_cast<int64_t>(p.D) * elem;
  const int64_t want = std::max<int64_t>(
      nchunks, X != nullptr ? (copy_bytes + 98303) / 98304 : (R + kFusedThreads - 1) / kFusedThreads);
  // At most two blocks per SM (room for a kernel of another stream beside it); with more
  // chunks than blocks, blocks loop over chunks (still one launch).
  const int grid = static_cast<int>(
      std::min<int64_t>(want, std::min<int64_t>(max_blocks, 2 * static_cast<int64_t>(num_sms()))));
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(static_cast<unsigned>(std::max(grid, 1)));
  cfg.blockDim = dim3(kFusedThreads);
  cfg.dynamicSmemBytes = 0;
  cfg.stream = stream;
  cudaLaunchAttribute attr[2];
  attr[0].id = cudaLaunchAttributeCooperative;
  attr[0].val.cooperative = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1 + pdl_attr(&attr[1]);
  cudaError_t e = cudaLaunchKernelEx(&cfg, dispatch_fused_kernel, a);
  if (e != cudaSuccess && cfg.numAttrs > 1) {  // no dependent launch with a cooperative one here
    (void)cudaGetLastError();
    cfg.numAttrs = 1;
    e = cudaLaunchKernelEx(&cfg, dispatch_fused_kernel, a);
  }
  return e != cudaSuccess ? e : cudaGetLastError();
}

}  // namespace moe

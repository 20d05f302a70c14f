// Host-side launchers of the kernels behind the C ABI. All pointers are device pointers;
// every launcher enqueues on `stream` and returns the CUDA error of the launch.
#pragma once

#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stddef.h>
#include <stdint.h>

#include <string>

#include <nvtx3/nvToolsExt.h>

#include "../../include/moe.h"

namespace moe {

// NVTX range around the enqueueing of one stage (route, dispatch, expert up/down, combine),
// seen by profilers that attach to NVTX (ncu --nvtx, nsys); header-only, a no-op otherwise.
struct NvtxRange {
  explicit NvtxRange(const char* name) { nvtxRangePushA(name); }
  ~NvtxRange() { nvtxRangePop(); }
  NvtxRange(const NvtxRange&) = delete;
  NvtxRange& operator=(const NvtxRange&) = delete;
};

// Upper bound on router partial-sum blocks (the launcher never exceeds it).
int route_num_blocks(int64_t N, int E);

// Router logits + softmax + top-k + gates. X == nullptr: `logits` is an input.
// colsum_partial: [route_num_blocks][E] floats (or nullptr when prob_colsum is nullptr).
// noise: [N][E] (p.routing_mode != TOPK). zl_partial: [route_num_blocks] floats, used when
// z_loss (device scalar) is requested. operand: route_tc_operand_bytes(p) bytes of workspace
// (256-byte aligned) for the tensor-core router's bf16 operand, or nullptr when that is 0.
cudaError_t launch_route(const moe_problem& p, const void* X, const float* W_r, const float* bias,
                         const float* noise, float* logits, int32_t* idx, float* gate,
                         float* colsum_partial, float* prob_colsum, float* zl_partial,
                         float* z_loss, void* operand, int* err, uint64_t timeout_ns,
                         cudaStream_t stream);

// Tensor-core router for bf16 X (logits from a three-term bf16 split of W_r, made in the same
// kernel, then the routing decision). colsum_partial may be nullptr; *grid_out = blocks that
// wrote a colsum partial row.
// With more than 16 experts the three bf16 terms of W_r are written once per call by a small
// kernel into `operand` ([3 Ep rounded up to 16][D] bf16, route_tc_operand_bytes(p) bytes) and
// loaded by TMA; with fewer the router splits each W_r slice itself in shared memory.
bool route_tc_supported(const moe_problem& p);
size_t route_tc_operand_bytes(const moe_problem& p);
cudaError_t launch_route_tc(const moe_problem& p, const void* X, const float* W_r,
                            const float* bias, const float* noise, float* logits_out,
                            int32_t* idx, float* gate, float* colsum_partial, float* zl_partial,
                            void* operand, int* grid_out, int* err, uint64_t timeout_ns,
                            cudaStream_t stream);

// 2-D bf16 tensor map (cols contiguous, row stride cols * 2 bytes), box box_cols x box_rows,
// 128-byte swizzle, out-of-range elements read as zero.
bool make_tensor_map_2d_bf16(CUtensorMap* m, const void* ptr, uint64_t cols, uint64_t rows,
                             uint32_t box_cols, uint32_t box_rows);

// 3-D uint8 tensor map over stacked [E][k][n] bytes (n contiguous), box box_n x box_k x 1,
// 128-byte swizzle (box_n must be 128).
bool make_tensor_map_3d_u8(CUtensorMap* m, const void* ptr, uint64_t n, uint64_t k, uint64_t E,
                           uint32_t box_n, uint32_t box_k);

// 3-D uint8 tensor map over stacked [E][rows][inner] bytes with a 64-byte swizzle (box_inner
// must be 64): the K-contiguous (packed) 8-bit expert weights.
bool make_tensor_map_3d_u8_sw64(CUtensorMap* m, const void* ptr, uint64_t inner, uint64_t rows,
                                uint64_t E, uint32_t box_inner, uint32_t box_rows);

// Repack 8-bit expert weights [E][k][n] (n contiguous) into [E][n][k] (k contiguous).
cudaError_t launch_pack_w8(const int8_t* src, int8_t* dst, int64_t E, int64_t k, int64_t n,
                           cudaStream_t stream);

// Grouped expert GEMMs with 8-bit weights (W = q * s, s per expert and output column),
// bf16 activations, tcgen05 tensor cores; 128-row tiles on single CTAs.
cudaError_t launch_ffn_up_w8(const moe_problem& p, const void* X_perm, const int32_t* offsets,
                             const int8_t* W1q, const float* S1, const int8_t* W2q,
                             const float* S2, void* H, int* err, uint64_t timeout_ns,
                             cudaStream_t stream);
cudaError_t launch_ffn_down_w8(const moe_problem& p, const void* H, const int32_t* offsets,
                               const int8_t* W3q, const float* S3, void* Y, int* err,
                               uint64_t timeout_ns, cudaStream_t stream);
// The same two GEMMs for experts holding few rows: computed transposed with the converted
// weights as the tensor-memory operand (64-row tiles).
// `packed`: the weights are K-contiguous ([E][n][k], from launch_pack_w8).
cudaError_t launch_ffn_up_w8t(const moe_problem& p, const void* X_perm, const int32_t* offsets,
                              const int8_t* W1q, const float* S1, const int8_t* W2q,
                              const float* S2, void* H, bool packed, int* err,
                              uint64_t timeout_ns, cudaStream_t stream);
cudaError_t launch_ffn_down_w8t(const moe_problem& p, const void* H, const int32_t* offsets,
                                const int8_t* W3q, const float* S3, void* Y, bool packed,
                                int* err, uint64_t timeout_ns, cudaStream_t stream);

// Records are processed in chunks of this many for the slot assignment.
constexpr int kDispatchChunk = 1024;

int dispatch_num_chunks(int64_t records);

// Histogram + prefix sums + slot-major capacity positions (+ row -> token map).
cudaError_t launch_slot_assign(const moe_problem& p, int64_t capacity, const int32_t* idx,
                               int32_t* chunk_counts, int32_t* load, int32_t* offsets,
                               int32_t* pos, uint8_t* dropped, int32_t* row_token, int* err,
                               cudaStream_t stream);

// Count, slot assignment and (when X != nullptr) the gather in one cooperative launch.
// bar: two ints of the workspace header, zero at rest (returned to zero by the kernel).
// Falls back to launch_slot_assign + launch_gather when no resident grid is available.
cudaError_t launch_dispatch_fused(const moe_problem& p, int64_t capacity, const int32_t* idx,
                                  int32_t* chunk_counts, int32_t* load, int32_t* offsets,
                                  int32_t* pos, uint8_t* dropped, int32_t* row_token,
                                  const void* X, void* X_perm, int* err, int* bar,
                                  uint64_t timeout_ns, cudaStream_t stream);

// X_perm[row] = X[row_token[row]] for row < offsets[E] (bulk-copy staged through shared memory).
cudaError_t launch_gather(const moe_problem& p, const void* X, const int32_t* row_token,
                          const int32_t* offsets, void* X_perm, int* err, cudaStream_t stream);

// dst[i] = src[index[i]] for i < n_rows (rows of row_bytes bytes, a multiple of 4; 16-byte
// aligned pointers). Out-of-range indices: MOE_DEVERR_BAD_INDEX in *err, row zero-filled.
cudaError_t launch_gather_rows(const void* src, int64_t n_src, const int32_t* index,
                               int64_t n_rows, int64_t row_bytes, void* dst, int* err,
                               cudaStream_t stream);

// Grouped expert GEMMs, bf16 operands, tcgen05 tensor cores.
//   up:   H = act(X_perm W1_e) (.) (X_perm W2_e)      down: Y = H W3_e
// sched: two ints of the workspace header, zero at rest (the in-order tile counter and the
// count of finished CTAs; the kernel returns them to zero when it ends).
cudaError_t launch_ffn_up_sm100(const moe_problem& p, const void* X_perm, const int32_t* offsets,
                                const void* W1, const void* W2, void* H, int* err, int* sched,
                                uint64_t timeout_ns, cudaStream_t stream);
cudaError_t launch_ffn_down_sm100(const moe_problem& p, const void* H, const int32_t* offsets,
                                  const void* W3, void* Y, int* err, int* sched,
                                  uint64_t timeout_ns, cudaStream_t stream);

// The same two steps in fp32 on CUDA cores.
cudaError_t launch_ffn_up_f32(const moe_problem& p, const void* X_perm, const int32_t* offsets,
                              const void* W1, const void* W2, void* H, cudaStream_t stream);
cudaError_t launch_ffn_down_f32(const moe_problem& p, const void* H, const int32_t* offsets,
                                const void* W3, void* Y, cudaStream_t stream);

// Gate-weighted combine of each token's k expert rows.
cudaError_t launch_combine(const moe_problem& p, const void* Y, const int32_t* idx,
                           const float* gate, const int32_t* offsets, const int32_t* pos,
                           const uint8_t* dropped, void* out, int* err, cudaStream_t stream);

// Failure-detection self-test: one bounded wait on a barrier nothing completes; records
// MOE_DEVERR_WAIT_TIMEOUT in *err after timeout_ns and returns.
cudaError_t launch_wait_timeout_probe(int* err, uint64_t timeout_ns, cudaStream_t stream);

int num_sms();

// Whether the layer's kernels are launched as programmatic dependents of the previous kernel
// in the stream (cudaLaunchAttributeProgrammaticStreamSerialization; each kernel waits in
// pdl_wait() before touching global memory). Off unless MOE_PDL=1 (read once per process).
bool pdl_enabled();

// Fills attr with the programmatic-dependent-launch attribute when enabled; returns the
// number of attributes written (0 or 1).
int pdl_attr(cudaLaunchAttribute* attr);

// Message returned by moe_last_error() on the calling thread.
void set_last_error(const std::string& msg);

}  // namespace moe

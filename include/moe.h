/*
 * moe.h -- C ABI of the B200 (sm_100a) Mixture-of-Experts FFN forward library.
 *
 * The layer (one data-parallel hot path, single GPU):
 *   logits = X W_r (+bias) in fp32 -> softmax over E -> top-k -> gates (optionally
 *   renormalised over the selected set) -> per-expert load -> capacity
 *   max(ceil(CF*N*k/E), min_capacity) with a slot-major or token-major drop mask ->
 *   expert-contiguous permutation of the N*k records -> per-expert gated FFN
 *   [act(x W1_e) (.) (x W2_e)] W3_e -> gate-weighted sum back to the N tokens.
 *
 * Sources, cited by page title and section:
 *   - Grok-1 book ch.5 "MoE routing & experts": 5.2 (fp32 router x.W_r, softmax, TopK),
 *     5.2.3 (softmax then top-k, no renormalisation), 5.3.2 (expert weights stacked with a
 *     leading expert dimension), 5.3.5 (GeGLU expert, gate-weighted sum over k).
 *   - LLMs-from-scratch ch.12 "MoE": 12.1 (X:[B,T,D], W_r:[D,E], top-k softmax over the
 *     selected set, f_e(x) = [SiLU(x W1_e) (.) (x W2_e)] W3_e, W1,W2:[D,F], W3:[F,D]),
 *     12.2 (flatten to [N,D], N*k dispatch records, accumulate the k contributions).
 *   - MoE formula-to-code walkthrough: 1.1 (stable softmax), 1.2 (top-k ordered by
 *     descending score, renormalisation), 1.3 (expert load), 2.1 (balance loss), 3.1
 *     (capacity), 3.2 (dispatch with a dropped mask), 3.3 (drop rate).
 *   - MoE series (GShard/Mixtral/Switch): 2.1 (capacity with min_capacity), 2.2 (an
 *     overflowed slot contributes nothing; case A: the kept expert takes the whole weight).
 *
 * Conventions shared by every entry point:
 *   - Array pointers are DEVICE pointers unless the entry point says otherwise. The caller
 *     allocates and owns every buffer, including the workspace; the library never
 *     allocates device memory.
 *   - Layouts are dense row-major. X [N,D]; W_r [D,E] fp32; bias [E] fp32; W1, W2 [E,D,F]
 *     (W1 = activated branch, Grok "linear"; W2 = linear branch, Grok "linear_v");
 *     W3 [E,F,D] (Grok "linear_1"); logits [N,E] fp32; topk_idx [N,k] int32 (rank 0 = the
 *     largest logit); topk_gate [N,k] fp32; load [E] int32; offsets [E+1] int32;
 *     pos [N,k] int32; dropped [N,k] uint8; row_token [N*k] int32; X_perm [N*k,D];
 *     H [N*k,F]; Y [N*k,D]; out [N,D].
 *   - X, W1..W3, X_perm, H, Y and out all have the problem's dtype (fp32 or bf16).
 *   - Every device pointer must be 16-byte aligned.
 *   - `stream` is a cudaStream_t (NULL = legacy default stream). Work is enqueued
 *     asynchronously; nothing synchronises the host except where stated.
 *   - Errors: arguments are checked on the host before anything is enqueued; a bad
 *     argument returns MOE_ERR_INVALID_ARG and a shape outside the kernels' support returns
 *     MOE_ERR_UNSUPPORTED, in both cases with nothing enqueued. A failed CUDA call returns
 *     MOE_ERR_CUDA (work enqueued before it by the same call stays enqueued).
 *     moe_last_error() gives a message for the calling thread.
 *   - Workspace: a device buffer of moe_workspace_size() bytes, 256-byte aligned, owned by
 *     the caller. Its first 256 bytes hold the device error word and the expert GEMMs'
 *     tile counters (which every GEMM launch returns to zero): zero them once with
 *     moe_workspace_init() before the first use. Calls that share a workspace must be
 *     ordered on one stream (they reuse its scratch regions).
 *   - Determinism: identical inputs give bitwise identical outputs; no floating-point
 *     atomics are used anywhere.
 *   - Kernels that wait on an on-chip barrier give up after a bounded time and record a
 *     code in the workspace's device error word (see moe_get_device_error).
 *   - Requires an sm_100a GPU (B200).
 */
#ifndef MOE_B200_H
#define MOE_B200_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
  MOE_OK = 0,
  MOE_ERR_INVALID_ARG = 1,
  MOE_ERR_UNSUPPORTED = 2,
  MOE_ERR_CUDA = 3,
  MOE_ERR_DEVICE = 4 /* a kernel recorded a device-side error (see moe_get_device_error) */
} moe_status;

enum { MOE_DTYPE_F32 = 0, MOE_DTYPE_BF16 = 1 };
enum { MOE_ACT_SILU = 0, MOE_ACT_GELU_ERF = 1, MOE_ACT_GELU_TANH = 2 };
/* Order in which routing records take capacity positions (walkthrough 3.2; MoE series 2.2). */
enum { MOE_ORDER_SLOT_MAJOR = 0, MOE_ORDER_TOKEN_MAJOR = 1 };
/* Weights of a token's kept slots when another of its slots was dropped (MoE series 2.2). */
enum { MOE_DROP_ZERO = 0, MOE_DROP_RENORM_KEPT = 1 };
/* Expert selection (moe_route_ex / moe_forward_ex; the other entry points need TOPK):
 *   TOPK           the k largest logits.
 *   NOISY_TOPK     Grok-1 book 5.2.2 (Switch's noisy top-k): z' = z + noise (fp32); the k
 *                  largest z' are selected and the gates come from softmax(z').
 *   GSHARD_RANDOM  MoE series 3: the first expert is the largest z; each later one is the
 *                  largest z' = z + noise (fp32) among the experts not chosen yet; the gates
 *                  come from softmax(z) (over the selected set when renormalize = 1, which is
 *                  GShard's w_i = P_i / (P_0 + P_1) for top-2). */
enum { MOE_ROUTE_TOPK = 0, MOE_ROUTE_NOISY_TOPK = 1, MOE_ROUTE_GSHARD_RANDOM = 2 };

/* Device error codes written to the workspace error word. */
enum {
  MOE_DEVERR_NONE = 0,
  MOE_DEVERR_WAIT_TIMEOUT = 1, /* a pipeline barrier wait exceeded its time bound */
  MOE_DEVERR_BAD_INDEX = 2     /* an expert index outside [0,E) reached a kernel */
};

/* The problem statement (LLMs-from-scratch 12.1; walkthrough 3.1; Grok-1 book 5.2.3).
 *   N               tokens (B*T flattened), >= 0
 *   D, F            model width and expert FFN width, >= 1
 *   E               experts, 1..64
 *   k               experts per token, 1..min(E, 8)
 *   capacity_factor CF; <= 0 means no capacity (every record is kept)
 *   renormalize     0: gate = softmax over all E (Grok-1); 1: gate renormalised over the
 *                   selected k (Mixtral / walkthrough 1.2)
 *   activation      MOE_ACT_* applied to x W1 (SiLU, exact-erf GELU, tanh GELU)
 *   dtype           MOE_DTYPE_* of X, W1..W3 and every activation buffer
 *   capacity_order  MOE_ORDER_SLOT_MAJOR: all rank-0 records in token order take positions
 *                   first, then rank 1, ... (every token's first choice has priority);
 *                   MOE_ORDER_TOKEN_MAJOR: token by token, each token's slots in rank order
 *                   (the walkthrough's dispatch loop, 3.2)
 *   drop_policy     MOE_DROP_ZERO: a dropped slot contributes nothing and the kept slots keep
 *                   their gates; MOE_DROP_RENORM_KEPT: when a token has dropped and kept
 *                   slots, the kept gates are divided by their sum (GShard case A, MoE series
 *                   2.2: (w1, w2) -> (1, 0) when the second expert overflows)
 *   routing_mode    MOE_ROUTE_* (selection variant; needs a noise array unless TOPK)
 *   min_capacity    >= 0; the capacity is max(ceil(CF*N*k/E), min_capacity) (MoE series 2.1)
 * bf16 problems need D and F to be multiples of 8 (16-byte rows for the tensor-memory
 * copies); fp32 problems need D and F to be multiples of 4. */
typedef struct {
  int64_t N;
  int64_t D;
  int64_t F;
  int32_t E;
  int32_t k;
  double capacity_factor;
  int32_t renormalize;
  int32_t activation;
  int32_t dtype;
  int32_t capacity_order;
  int32_t drop_policy;
  int32_t routing_mode;
  int64_t min_capacity;
  int32_t reserved; /* must be 0 */
} moe_problem;

/* Host only. C = max(ceil(CF * N * k / E), min_capacity), the first term evaluated in double
 * left to right (walkthrough 3.1; MoE series 2.1); C = N*k when CF <= 0. */
moe_status moe_capacity(const moe_problem* p, int64_t* C);

/* Host only. Bytes of workspace every entry point below accepts for problem p (one size for
 * all of them). The workspace holds the device error word, scratch counters, the router's
 * bf16 operand (bf16 X with more than 16 experts: the three bf16 terms of W_r, written by each
 * router call) and, for moe_forward, the intermediate buffers (routing results, X_perm, H,
 * Y). */
moe_status moe_workspace_size(const moe_problem* p, size_t* bytes);

/* Router + softmax + top-k + gates (Grok-1 book 5.2, 5.2.3; walkthrough 1.1, 1.2;
 * LLMs-from-scratch 12.1).
 *   X != NULL : logits = fp32(X) . W_r (+ bias), fp32 accumulation; written to `logits`
 *               when `logits` != NULL. bf16 X runs on the tensor cores with W_r split into
 *               three bf16 terms (products exact, sums in fp32); fp32 X on fp32 FMA.
 *   X == NULL : `logits` is read as an INPUT [N,E] (routing from given fp32 logits).
 *   topk_idx  : the k experts with the largest fp32 logits, in descending order; equal
 *               logits are ordered by lower expert index.
 *   topk_gate : renormalize=0: softmax(logits)[idx]; renormalize=1: softmax of the selected
 *               logits (= probs[idx] / sum of the selected probs).
 *   prob_colsum (optional, [E]): sum over tokens of the full softmax, for the balance loss
 *               (walkthrough 2.1); summed in a fixed order.
 *   W_r may be NULL only when X is NULL. bias (optional, [E] fp32) is added to computed
 *   logits; given logits (X == NULL) are used as they are.
 * Workspace: moe_workspace_size bytes. */
moe_status moe_route(const moe_problem* p, const void* X, const float* W_r, const float* bias,
                     float* logits, int32_t* topk_idx, float* topk_gate, float* prob_colsum,
                     void* ws, size_t ws_bytes, void* stream);

/* moe_route with the training-time selection variants (p->routing_mode) and the z-loss.
 *   noise   [N,E] fp32, device; the caller's random draws (e.g. N(0, sigma^2) for noisy
 *           top-k, Grok-1 book 5.2.2; GShard's perturbation, MoE series 3). Required unless
 *           routing_mode is MOE_ROUTE_TOPK (then ignored).
 *   z_loss  optional [1] fp32, device: mean over tokens of (log sum_e exp(logits_te))^2 on the
 *           unperturbed logits (the z-loss of Grok-1 book 5.2.2 before its coefficient);
 *           summed in a fixed order.
 *   prob_colsum reports the softmax the gates come from (of z' under NOISY_TOPK).
 * Everything else as moe_route. */
moe_status moe_route_ex(const moe_problem* p, const void* X, const float* W_r, const float* bias,
                        const float* noise, float* logits, int32_t* topk_idx, float* topk_gate,
                        float* prob_colsum, float* z_loss, void* ws, size_t ws_bytes,
                        void* stream);

/* Load histogram, capacity, slot assignment and permutation (walkthrough 1.3, 3.1, 3.2;
 * LLMs-from-scratch 12.2; MoE series 2.2).
 *   load[e]      = number of records (t,j) with topk_idx[t,j] == e (before capacity).
 *   pos[t,j]     = rank of record (t,j) among expert e's records, records taken in
 *                  p->capacity_order: slot-major (all j=0 records in token order, then all
 *                  j=1 records, ...) or token-major (t ascending, j ascending within t).
 *   dropped[t,j] = pos[t,j] >= C.
 *   offsets      = exclusive prefix sum of min(load_e, C); offsets[E] = kept records.
 *   row_token[offsets[e] + pos[t,j]] = t for every kept record; entries past offsets[E]
 *                  are not written.
 *   X_perm[row]  = X[row_token[row]] for row < offsets[E] (skipped when X or X_perm is NULL);
 *                  rows past offsets[E] are not written.
 * topk_idx values must lie in [0,E); a value outside is recorded as MOE_DEVERR_BAD_INDEX
 * and that record is treated as dropped. Bit-exact and deterministic. */
moe_status moe_dispatch(const moe_problem* p, const void* X, const int32_t* topk_idx,
                        int32_t* load, int32_t* offsets, int32_t* pos, uint8_t* dropped,
                        int32_t* row_token, void* X_perm, void* ws, size_t ws_bytes,
                        void* stream);

/* moe_dispatch for callers that cannot give the library any device memory of their own:
 * code that may no longer call cudaMalloc once it runs (an allocation synchronises the device
 * and can stall every stream of a serving loop), or a host whose device memory is all owned by
 * its own pool and lent out only as the tensors it computes on. Same arguments, results and
 * guarantees as moe_dispatch, minus the workspace: the per-chunk expert counters live in a
 * fixed 64 KiB array inside the library (held on every GPU that loads the library until the
 * process exits). There is no counterpart on the pages; this is a deployment variant.
 *   - row_token is required (it is an output here, not workspace).
 *   - Limit: ceil(N*k / 1024) * E <= 16384 counters (e.g. N*k <= 262144 records at E = 64);
 *     larger problems return MOE_ERR_UNSUPPORTED -- use moe_dispatch.
 *   - The first call on each device looks up the array's device address
 *     (cudaGetSymbolAddress) and, under CUDA's lazy module loading, may load this library's
 *     kernels into the device's context, which takes device memory the driver allocates
 *     itself. Make that first call during set-up, before any stream capture and before the
 *     code that must not allocate starts. After cudaDeviceReset the device gets a new
 *     context and the next call looks the address up again.
 *   - Every call shares the one array: calls that may overlap on the GPU (different streams,
 *     or different host threads on one device) race and must be serialised by the caller.
 *     Each call rewrites every counter it reads, so no clearing is needed between calls.
 *   - Out-of-range expert indices are treated as dropped but not reported, and neither is a
 *     gather whose bounded wait on its copy barrier ran out (X_perm may then be partly
 *     written): there is no workspace error word on this path. Callers that need those
 *     reports use moe_dispatch.
 * Allocates nothing: no cudaMalloc, cudaFree or allocating library routine. */
moe_status moe_dispatch_noalloc(const moe_problem* p, const void* X, const int32_t* topk_idx,
                                int32_t* load, int32_t* offsets, int32_t* pos, uint8_t* dropped,
                                int32_t* row_token, void* X_perm, void* stream);

/* Grouped gated expert FFN on the expert-contiguous rows (LLMs-from-scratch 12.1; Grok-1
 * book 5.3.5): for each expert e and each row r in [offsets[e], offsets[e+1]):
 *   H[r] = act(X_perm[r] W1_e) (.) (X_perm[r] W2_e),   Y[r] = H[r] W3_e.
 * bf16: tcgen05 tensor-core GEMMs with fp32 accumulation, act and product in fp32, H and Y
 * rounded to bf16. fp32: CUDA-core fp32 FMA throughout. offsets stay on the device (the
 * host never learns the per-expert counts). Rows past offsets[E] are not written. */
moe_status moe_expert_ffn(const moe_problem* p, const void* X_perm, const int32_t* offsets,
                          const void* W1, const void* W2, const void* W3, void* H, void* Y,
                          void* ws, size_t ws_bytes, void* stream);

/* First half of moe_expert_ffn (GEMM1 with the gating fused into its epilogue):
 *   H[r] = act(X_perm[r] W1_e) (.) (X_perm[r] W2_e)   for r in [offsets[e], offsets[e+1]).
 * Same precision, layout and row rules as moe_expert_ffn. */
moe_status moe_expert_up(const moe_problem* p, const void* X_perm, const int32_t* offsets,
                         const void* W1, const void* W2, void* H, void* ws, size_t ws_bytes,
                         void* stream);

/* Second half of moe_expert_ffn (GEMM2): Y[r] = H[r] W3_e for r in [offsets[e], offsets[e+1]). */
moe_status moe_expert_down(const moe_problem* p, const void* H, const int32_t* offsets,
                           const void* W3, void* Y, void* ws, size_t ws_bytes, void* stream);

/* Gate-weighted combine (Grok-1 book 5.3.5; LLMs-from-scratch 12.2; MoE series 2.2):
 *   out[t] = sum_{j=0..k-1} [!dropped[t,j]] * g[t,j] * Y[offsets[topk_idx[t,j]] + pos[t,j]]
 * with g = topk_gate, except under MOE_DROP_RENORM_KEPT for a token with both dropped and kept
 * slots: g[t,j] = topk_gate[t,j] / (sum of its kept slots' gates, fp32, ascending j).
 * Accumulated in fp32 in ascending j, rounded once to the output dtype; a token whose slots
 * are all dropped gets 0. `dropped` may be NULL only without a capacity
 * (capacity_factor <= 0: nothing is dropped); with a capacity it is required
 * (MOE_ERR_INVALID_ARG otherwise). A kept record whose expert index or position falls outside
 * its expert's segment [offsets[e], offsets[e+1]) contributes nothing and is not read; no
 * workspace is passed here, so it is not reported (moe_forward reports it as
 * MOE_DEVERR_BAD_INDEX). No atomics. */
moe_status moe_combine(const moe_problem* p, const void* Y, const int32_t* topk_idx,
                       const float* topk_gate, const int32_t* offsets, const int32_t* pos,
                       const uint8_t* dropped, void* out, void* stream);

/* The whole layer: moe_route -> moe_dispatch -> moe_expert_ffn -> moe_combine, enqueued on
 * one stream with no host synchronisation. Intermediates live in the workspace; each of
 * the optional export pointers (logits .. prob_colsum) may be NULL, otherwise the
 * corresponding intermediate is also written there. */
moe_status moe_forward(const moe_problem* p, const void* X, const float* W_r, const float* bias,
                       const void* W1, const void* W2, const void* W3, void* out, float* logits,
                       int32_t* topk_idx, float* topk_gate, int32_t* load, int32_t* offsets,
                       int32_t* pos, uint8_t* dropped, float* prob_colsum, void* ws,
                       size_t ws_bytes, void* stream);

/* ---- 8-bit expert weights (Grok-1 book 5.3.3 and 5.3.5: weight = weight * scales before
 * each expert matmul). Layouts as the bf16 weights, stored as int8: W1q, W2q [E,D,F], W3q
 * [E,F,D]; one fp32 scale per expert and output column: S1, S2 [E,F], S3 [E,D]; the expert
 * uses W[e][k][n] = Wq[e][k][n] * S[e][n]. Activations (X, X_perm, H, Y, out) are bf16
 * (p->dtype must be MOE_DTYPE_BF16) and D, F must be multiples of 16, else
 * MOE_ERR_UNSUPPORTED. The tensor cores multiply bf16 activations by the exact bf16 value of q
 * with fp32 accumulation and the scale is applied to the fp32 sum (x.(q s) = s (x.q) for a
 * per-column s), so the weights cross HBM as int8. Pointers: device memory, 16-byte aligned.
 * Same results rules, workspace and error behaviour as the bf16 entry points. */
moe_status moe_expert_up_w8(const moe_problem* p, const void* X_perm, const int32_t* offsets,
                            const int8_t* W1q, const float* S1, const int8_t* W2q,
                            const float* S2, void* H, void* ws, size_t ws_bytes, void* stream);
moe_status moe_expert_down_w8(const moe_problem* p, const void* H, const int32_t* offsets,
                              const int8_t* W3q, const float* S3, void* Y, void* ws,
                              size_t ws_bytes, void* stream);
/* moe_forward with 8-bit expert weights (router, dispatch and combine unchanged). */
moe_status moe_forward_w8(const moe_problem* p, const void* X, const float* W_r,
                          const float* bias, const int8_t* W1q, const float* S1,
                          const int8_t* W2q, const float* S2, const int8_t* W3q, const float* S3,
                          void* out, float* logits, int32_t* topk_idx, float* topk_gate,
                          int32_t* load, int32_t* offsets, int32_t* pos, uint8_t* dropped,
                          float* prob_colsum, void* ws, size_t ws_bytes, void* stream);

/* Load-time repacking of the 8-bit expert weights with the reduction dimension contiguous:
 * W1p, W2p [E,F,D] from W1q, W2q [E,D,F]; W3p [E,D,F] from W3q [E,F,D] (an exact byte
 * transpose of each expert's matrix, Wp[e][n][k] = Wq[e][k][n]). Same shape rules as
 * moe_expert_up_w8; the caller owns all six device buffers (16-byte aligned, no overlap).
 * Enqueued on `stream`; returns MOE_ERR_INVALID_ARG / MOE_ERR_UNSUPPORTED / MOE_ERR_CUDA. */
moe_status moe_pack_w8(const moe_problem* p, const int8_t* W1q, const int8_t* W2q,
                       const int8_t* W3q, int8_t* W1p, int8_t* W2p, int8_t* W3p, void* stream);
/* moe_expert_up_w8 / moe_expert_down_w8 / moe_forward_w8 on weights repacked by moe_pack_w8
 * (scales unchanged). Same results: each output element is the same fp32 sum of the same
 * products, taken by the kernel that computes each expert transposed (weights as the
 * tensor-memory operand), which is also the one the unpacked entry points pick for
 * decode-sized batches. */
moe_status moe_expert_up_w8p(const moe_problem* p, const void* X_perm, const int32_t* offsets,
                             const int8_t* W1p, const float* S1, const int8_t* W2p,
                             const float* S2, void* H, void* ws, size_t ws_bytes, void* stream);
moe_status moe_expert_down_w8p(const moe_problem* p, const void* H, const int32_t* offsets,
                               const int8_t* W3p, const float* S3, void* Y, void* ws,
                               size_t ws_bytes, void* stream);
moe_status moe_forward_w8p(const moe_problem* p, const void* X, const float* W_r,
                           const float* bias, const int8_t* W1p, const float* S1,
                           const int8_t* W2p, const float* S2, const int8_t* W3p,
                           const float* S3, void* out, float* logits, int32_t* topk_idx,
                           float* topk_gate, int32_t* load, int32_t* offsets, int32_t* pos,
                           uint8_t* dropped, float* prob_colsum, void* ws, size_t ws_bytes,
                           void* stream);

/* moe_forward with the training-time selection variants (p->routing_mode, noise as in
 * moe_route_ex) and the optional z_loss output. */
moe_status moe_forward_ex(const moe_problem* p, const void* X, const float* W_r,
                          const float* bias, const float* noise, const void* W1, const void* W2,
                          const void* W3, void* out, float* logits, int32_t* topk_idx,
                          float* topk_gate, int32_t* load, int32_t* offsets, int32_t* pos,
                          uint8_t* dropped, float* prob_colsum, float* z_loss, void* ws,
                          size_t ws_bytes, void* stream);

/* moe_forward with HOST activations: X_host [N,D] and out_host [N,D] are host pointers
 * (page-locked memory gives asynchronous copies), the weights and W_r/bias are device
 * pointers. Enqueues the host->device copy of X, the forward, and the device->host copy
 * of out on `stream`, then waits for the stream, so out_host is valid on return. Uses
 * the workspace (moe_workspace_size_host bytes: moe_workspace_size plus the device copies of
 * X and out, double-buffered for moe_forward_host_many). Without capacity (capacity_factor <= 0) and with N >= 1024 the
 * batch runs as two halves, the copies of one half overlapping the other half's layer on an
 * internal copy stream; each token's output is then the layer on its own half-batch (the same
 * result up to the rounding of the router's split of D). Needs routing_mode = TOPK. */
moe_status moe_forward_host(const moe_problem* p, const void* X_host, const float* W_r,
                            const float* bias, const void* W1, const void* W2, const void* W3,
                            void* out_host, void* ws, size_t ws_bytes, void* stream);

/* A sequence of host batches through the layer, for serving loops: batch b's X is
 * X_host + b*N*D*s and its output goes to out_host + b*N*D*s (both [n_batches, N, D], pinned
 * host memory for asynchronous copies; the caller owns them). Each batch is a complete
 * moe_forward call on its N tokens (capacity per batch) and its output equals moe_forward's bit
 * for bit. Device buffers for X and the output are double-buffered in the workspace
 * (moe_workspace_size_host), with input copies on one internal copy stream and output copies on
 * another, so batch b+1's input copy and batch b-1's output copy overlap batch b's layer on
 * `stream`. Returns after every output copy has completed (the stream is synchronised).
 * n_batches == 0 or N == 0 is a no-op. Errors as moe_forward_host; after a failure the outputs
 * of batches from the failing one on are unspecified. Plain top-k routing only. */
moe_status moe_forward_host_many(const moe_problem* p, int64_t n_batches, const void* X_host,
                                 const float* W_r, const float* bias, const void* W1,
                                 const void* W2, const void* W3, void* out_host, void* ws,
                                 size_t ws_bytes, void* stream);

/* Host only. Workspace bytes for moe_forward_host and moe_forward_host_many (moe_workspace_size
 * plus 4*N*D*sizeof(element), each part 256-byte aligned). */
moe_status moe_workspace_size_host(const moe_problem* p, size_t* bytes);

/* Row gather: dst[i] = src[index[i]] for i < n_rows, rows of row_bytes bytes. The local
 * reorder steps of expert parallelism (Grok-1 book 5.6: tokens travel by all-to-all to the
 * device holding their expert and back; MoE series 4.1): rows received from every source rank
 * are put in expert-major order before the expert GEMMs, and the expert outputs back in
 * source-rank order before the return exchange. src: [n_src_rows, row_bytes] (may be NULL when
 * n_src_rows == 0), index: [n_rows] int32, dst: [n_rows, row_bytes]; device memory, src/dst
 * 16-byte aligned, dst not overlapping src. row_bytes: a positive multiple of 4 (16-byte
 * words when it is a multiple of 16). An index outside [0, n_src_rows) sets
 * MOE_DEVERR_BAD_INDEX in the workspace's error word (moe_get_device_error) and its dst row
 * is zero-filled; nothing outside the buffers is read or written. ws: any workspace (at
 * least 256 bytes; only its error word is used). Enqueued on `stream`. */
moe_status moe_gather_rows(const void* src, int64_t n_src_rows, const int32_t* index,
                           int64_t n_rows, int64_t row_bytes, void* dst, void* ws,
                           size_t ws_bytes, void* stream);

/* Host only: the layer's diagnostics, in fp64 from host copies of its [E] and [N,k] outputs.
 * Balance loss (MoE formula-to-code walkthrough 2.1-2.3; MoE series 7.3):
 *   loss = E * sum_e f_e * P_e,  f_e = load[e] / (N*k),  P_e = prob_colsum[e] / N,
 * with load from moe_dispatch (records per expert before capacity) and prob_colsum from
 * moe_route (the column sums of the full softmax); uniform routing gives exactly 1 for any k.
 * Drop rate (walkthrough 3.3): dropped records / (N*k) over the routing slots, dropped [N,k]
 * from moe_dispatch. Pointers are host pointers; N == 0 gives 0. Errors: MOE_ERR_INVALID_ARG
 * for a NULL pointer or an invalid problem. */
moe_status moe_balance_loss(const moe_problem* p, const int32_t* load, const float* prob_colsum,
                            double* loss);
moe_status moe_drop_rate(const moe_problem* p, const uint8_t* dropped, double* rate);

/* Failure-detection self-test; it changes no result. Enqueues one kernel that waits on a
 * barrier that nothing completes (the state of a pipeline wait whose producer has stopped),
 * bounded by timeout_us of wall time, with the same bounded wait the pipeline kernels use. It
 * then records MOE_DEVERR_WAIT_TIMEOUT in the workspace's error word and returns:
 * moe_get_device_error reports the code and clears it, and the context stays usable. ws: any
 * workspace (at least 256 bytes). timeout_us in [1, 10^7], else MOE_ERR_INVALID_ARG. */
moe_status moe_selftest_wait_timeout(void* ws, size_t ws_bytes, int64_t timeout_us,
                                     void* stream);

/* Zero the device error word of a new workspace (asynchronous, on `stream`). */
moe_status moe_workspace_init(void* ws, size_t ws_bytes, void* stream);

/* Synchronises `stream`, then reads the device error word of workspace `ws` into *code
 * (MOE_DEVERR_*) and clears it. Returns MOE_ERR_DEVICE when the word was non-zero. */
moe_status moe_get_device_error(void* ws, void* stream, int32_t* code);

/* Static strings. */
const char* moe_status_string(moe_status s);
const char* moe_last_error(void);

/* Library version (major*10000 + minor*100 + patch). */
int32_t moe_version(void);

#ifdef __cplusplus
}
#endif

#endif /* MOE_B200_H */

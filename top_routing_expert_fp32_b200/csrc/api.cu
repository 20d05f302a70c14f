// C ABI of the MoE FFN forward library (declared in include/moe.h): argument validation,
// workspace layout, and the enqueueing of the kernels in the pages' order
// (route -> dispatch -> expert FFN -> combine).
#include <cmath>
#include <cstdint>
#include <cstdlib>
#include <cstring>
#include <mutex>
#include <string>

#include "../../include/moe.h"
#include "internal.h"

namespace moe {

int num_sms() {
  static int cache[64] = {0};
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return 148;
  if (cache[dev] == 0) {
    int n = 0;
    if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || n <= 0)
      n = 148;
    cache[dev] = n;
  }
  return cache[dev];
}

// Off by default: measured on decode- and mixtral-shaped layers, launching each kernel as a
// programmatic dependent of the previous one was slower (decode back-to-back 476 -> 505 us)
// or no faster. MOE_PDL=1 turns it on.
bool pdl_enabled() {
  static const bool on = [] {
    const char* env = std::getenv("MOE_PDL");
    return env != nullptr && std::strcmp(env, "1") == 0;
  }();
  return on;
}

int pdl_attr(cudaLaunchAttribute* attr) {
  if (!pdl_enabled()) return 0;
  attr->id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr->val.programmaticStreamSerializationAllowed = 1;
  return 1;
}

}  // namespace moe

namespace {

using namespace moe;

thread_local std::string g_last_error;

moe_status fail(moe_status s, const std::string& msg) {
  g_last_error = msg;
  return s;
}

moe_status cuda_fail(cudaError_t e, const char* where) {
  return fail(MOE_ERR_CUDA, std::string(where) + ": " + cudaGetErrorString(e));
}

uint64_t wait_timeout_ns() {
  static uint64_t ns = 0;
  static std::once_flag once;
  std::call_once(once, [] {
    uint64_t ms = 2000;
    if (const char* s = std::getenv("MOE_WAIT_TIMEOUT_MS")) {
      const long long v = std::atoll(s);
      if (v > 0) ms = static_cast<uint64_t>(v);
    }
    ns = ms * 1000000ull;
  });
  return ns;
}

size_t align256(size_t x) { return (x + 255) & ~static_cast<size_t>(255); }

// The workspace header (its first 256 bytes, zeroed by moe_workspace_init): int 0 is the
// device error word, ints 16 and 17 the grouped GEMMs' tile counter and finished count (zero
// at rest; each GEMM launch returns them to zero when it ends).
constexpr int kSchedInt = 16;
int* sched_of(int* header) { return header + kSchedInt; }
// Ints 20 and 21: the fused dispatch's grid-barrier arrivals and finished count (zero at rest).
constexpr int kDispatchBarInt = 20;
int* dispatch_bar_of(int* header) { return header + kDispatchBarInt; }

size_t elem_size(const moe_problem& p) { return p.dtype == MOE_DTYPE_BF16 ? 2 : 4; }

// Device workspace regions (byte offsets from the workspace base).
struct Layout {
  size_t err, colsum_part, zl_part, route_op, counts, idx, gate, pos, dropped, load, offsets,
      row_token, xperm, h, y;
  size_t total;       // moe_forward and every other entry point
  size_t xin, xout;   // moe_forward_host / moe_forward_host_many
  size_t xin2, xout2; // second buffers of moe_forward_host_many
  size_t total_host;
};

Layout make_layout(const moe_problem& p) {
  Layout L{};
  size_t o = 0;
  auto take = [&](size_t bytes) {
    const size_t at = o;
    o = align256(o + bytes);
    return at;
  };
  const size_t R = static_cast<size_t>(p.N) * static_cast<size_t>(p.k);
  const size_t es = elem_size(p);
  L.err = take(256);
  L.colsum_part = take(sizeof(float) * static_cast<size_t>(route_num_blocks(p.N, p.E)) * p.E);
  L.zl_part = take(sizeof(float) * static_cast<size_t>(route_num_blocks(p.N, p.E)));
  L.route_op = take(route_tc_operand_bytes(p));
  L.counts = take(sizeof(int32_t) * static_cast<size_t>(dispatch_num_chunks(R)) * p.E);
  L.idx = take(sizeof(int32_t) * R);
  L.gate = take(sizeof(float) * R);
  L.pos = take(sizeof(int32_t) * R);
  L.dropped = take(R);
  L.load = take(sizeof(int32_t) * p.E);
  L.offsets = take(sizeof(int32_t) * (p.E + 1));
  L.row_token = take(sizeof(int32_t) * R);
  L.xperm = take(es * R * static_cast<size_t>(p.D));
  L.h = take(es * R * static_cast<size_t>(p.F));
  L.y = take(es * R * static_cast<size_t>(p.D));
  L.total = o;
  L.xin = take(es * static_cast<size_t>(p.N) * static_cast<size_t>(p.D));
  L.xout = take(es * static_cast<size_t>(p.N) * static_cast<size_t>(p.D));
  L.xin2 = take(es * static_cast<size_t>(p.N) * static_cast<size_t>(p.D));
  L.xout2 = take(es * static_cast<size_t>(p.N) * static_cast<size_t>(p.D));
  L.total_host = o;
  return L;
}

moe_status check_problem(const moe_problem* p) {
  if (p == nullptr) return fail(MOE_ERR_INVALID_ARG, "problem is NULL");
  if (p->reserved != 0) return fail(MOE_ERR_INVALID_ARG, "reserved field must be 0");
  if (p->N < 0) return fail(MOE_ERR_INVALID_ARG, "N < 0");
  if (p->D < 1 || p->F < 1) return fail(MOE_ERR_INVALID_ARG, "D and F must be >= 1");
  if (p->E < 1) return fail(MOE_ERR_INVALID_ARG, "E < 1");
  if (p->k < 1 || p->k > p->E) return fail(MOE_ERR_INVALID_ARG, "k must be in [1, E]");
  if (p->E > 64) return fail(MOE_ERR_UNSUPPORTED, "E > 64");
  if (p->k > 8) return fail(MOE_ERR_UNSUPPORTED, "k > 8");
  if (p->dtype != MOE_DTYPE_F32 && p->dtype != MOE_DTYPE_BF16)
    return fail(MOE_ERR_INVALID_ARG, "unknown dtype");
  if (p->activation < MOE_ACT_SILU || p->activation > MOE_ACT_GELU_TANH)
    return fail(MOE_ERR_INVALID_ARG, "unknown activation");
  if (p->renormalize != 0 && p->renormalize != 1)
    return fail(MOE_ERR_INVALID_ARG, "renormalize must be 0 or 1");
  if (std::isnan(p->capacity_factor)) return fail(MOE_ERR_INVALID_ARG, "capacity_factor is NaN");
  if (p->capacity_order != MOE_ORDER_SLOT_MAJOR && p->capacity_order != MOE_ORDER_TOKEN_MAJOR)
    return fail(MOE_ERR_INVALID_ARG, "unknown capacity_order");
  if (p->drop_policy != MOE_DROP_ZERO && p->drop_policy != MOE_DROP_RENORM_KEPT)
    return fail(MOE_ERR_INVALID_ARG, "unknown drop_policy");
  if (p->min_capacity < 0) return fail(MOE_ERR_INVALID_ARG, "min_capacity < 0");
  if (p->routing_mode < MOE_ROUTE_TOPK || p->routing_mode > MOE_ROUTE_GSHARD_RANDOM)
    return fail(MOE_ERR_INVALID_ARG, "unknown routing_mode");
  if (p->N * static_cast<int64_t>(p->k) > INT32_MAX)
    return fail(MOE_ERR_UNSUPPORTED, "N*k exceeds 2^31-1 records");
  if (p->D > (1 << 24) || p->F > (1 << 24)) return fail(MOE_ERR_UNSUPPORTED, "D or F > 2^24");
  const int64_t vec = p->dtype == MOE_DTYPE_BF16 ? 8 : 4;
  if (p->D % vec != 0 || p->F % vec != 0)
    return fail(MOE_ERR_UNSUPPORTED,
                p->dtype == MOE_DTYPE_BF16 ? "bf16 needs D and F multiples of 8"
                                           : "fp32 needs D and F multiples of 4");
  return MOE_OK;
}

bool aligned(const void* ptr, uintptr_t a) { return (reinterpret_cast<uintptr_t>(ptr) % a) == 0; }

moe_status need(const void* ptr, const char* name, uintptr_t align = 16) {
  if (ptr == nullptr) return fail(MOE_ERR_INVALID_ARG, std::string(name) + " is NULL");
  if (!aligned(ptr, align))
    return fail(MOE_ERR_INVALID_ARG, std::string(name) + " is not " + std::to_string(align) +
                                         "-byte aligned");
  return MOE_OK;
}

moe_status opt(const void* ptr, const char* name, uintptr_t align = 16) {
  return ptr == nullptr ? MOE_OK : need(ptr, name, align);
}

#define MOE_TRY(expr)              \
  do {                             \
    const moe_status _s = (expr);  \
    if (_s != MOE_OK) return _s;   \
  } while (0)

#define MOE_CUDA(expr, where)                        \
  do {                                               \
    const cudaError_t _e = (expr);                   \
    if (_e != cudaSuccess) return cuda_fail(_e, where); \
  } while (0)

moe_status check_ws(const moe_problem& p, const void* ws, size_t ws_bytes, bool host) {
  MOE_TRY(need(ws, "ws", 256));
  const Layout L = make_layout(p);
  const size_t want = host ? L.total_host : L.total;
  if (ws_bytes < want)
    return fail(MOE_ERR_INVALID_ARG,
                "workspace too small: " + std::to_string(ws_bytes) + " < " + std::to_string(want));
  return MOE_OK;
}

moe_status check_sm100() {
  int dev = 0, major = 0, minor = 0;
  MOE_CUDA(cudaGetDevice(&dev), "cudaGetDevice");
  MOE_CUDA(cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev), "attr");
  MOE_CUDA(cudaDeviceGetAttribute(&minor, cudaDevAttrComputeCapabilityMinor, dev), "attr");
  if (major != 10 || minor != 0)
    return fail(MOE_ERR_UNSUPPORTED, "requires an sm_100a (B200) GPU");
  return MOE_OK;
}

int64_t capacity_of(const moe_problem& p) {
  const int64_t R = p.N * static_cast<int64_t>(p.k);
  if (p.capacity_factor <= 0.0) return R;
  const int64_t c = static_cast<int64_t>(
      std::ceil(p.capacity_factor * static_cast<double>(p.N) * static_cast<double>(p.k) /
                static_cast<double>(p.E)));
  return c > p.min_capacity ? c : p.min_capacity;
}

template <typename T>
T* at(void* ws, size_t off) {
  return reinterpret_cast<T*>(static_cast<uint8_t*>(ws) + off);
}

moe_status run_up(const moe_problem& p, const void* X_perm, const int32_t* offsets,
                  const void* W1, const void* W2, void* H, int* err, cudaStream_t stream) {
  NvtxRange range("moe expert up");
  if (p.dtype == MOE_DTYPE_BF16) {
    MOE_TRY(check_sm100());
    MOE_CUDA(launch_ffn_up_sm100(p, X_perm, offsets, W1, W2, H, err, sched_of(err),
                                 wait_timeout_ns(), stream),
             "expert up-projection (tcgen05)");
  } else {
    MOE_CUDA(launch_ffn_up_f32(p, X_perm, offsets, W1, W2, H, stream), "expert up-projection");
  }
  return MOE_OK;
}

moe_status run_down(const moe_problem& p, const void* H, const int32_t* offsets, const void* W3,
                    void* Y, int* err, cudaStream_t stream) {
  NvtxRange range("moe expert down");
  if (p.dtype == MOE_DTYPE_BF16) {
    MOE_TRY(check_sm100());
    MOE_CUDA(launch_ffn_down_sm100(p, H, offsets, W3, Y, err, sched_of(err), wait_timeout_ns(),
                                   stream),
             "expert down-projection (tcgen05)");
  } else {
    MOE_CUDA(launch_ffn_down_f32(p, H, offsets, W3, Y, stream), "expert down-projection");
  }
  return MOE_OK;
}

// Expert weights: bf16/fp32 (W1..W3) or 8-bit with per-column scales (Q1..Q3, S1..S3).
struct Experts {
  const void* W1 = nullptr;
  const void* W2 = nullptr;
  const void* W3 = nullptr;
  const int8_t* Q1 = nullptr;
  const int8_t* Q2 = nullptr;
  const int8_t* Q3 = nullptr;
  const float* S1 = nullptr;
  const float* S2 = nullptr;
  const float* S3 = nullptr;
  bool packed = false;  // 8-bit weights K-contiguous (moe_pack_w8)
  bool w8() const { return Q1 != nullptr; }
};

// 8-bit experts: the tensor-memory-operand kernel for experts with few rows (decode-sized
// batches, R/E <= 64), the shared-memory kernel otherwise. MOE_W8_KERNEL=tmem|smem overrides.
bool use_w8t(const moe_problem& p) {
  if (const char* env = std::getenv("MOE_W8_KERNEL")) {
    if (std::strcmp(env, "tmem") == 0) return true;
    if (std::strcmp(env, "smem") == 0) return false;
  }
  return p.N * p.k <= 64 * static_cast<int64_t>(p.E);
}

// packed: K-contiguous weights from moe_pack_w8 (always the tensor-memory-operand kernel).
moe_status run_up_w8(const moe_problem& p, const void* X_perm, const int32_t* offsets,
                     const int8_t* Q1, const float* S1, const int8_t* Q2, const float* S2,
                     void* H, bool packed, int* err, cudaStream_t stream) {
  NvtxRange range("moe expert up (8-bit)");
  MOE_TRY(check_sm100());
  if (packed || use_w8t(p))
    MOE_CUDA(launch_ffn_up_w8t(p, X_perm, offsets, Q1, S1, Q2, S2, H, packed, err,
                               wait_timeout_ns(), stream),
             "expert up-projection, 8-bit weights (tcgen05, TMEM operand)");
  else
    MOE_CUDA(launch_ffn_up_w8(p, X_perm, offsets, Q1, S1, Q2, S2, H, err, wait_timeout_ns(),
                              stream),
             "expert up-projection, 8-bit weights (tcgen05)");
  return MOE_OK;
}

moe_status run_down_w8(const moe_problem& p, const void* H, const int32_t* offsets,
                       const int8_t* Q3, const float* S3, void* Y, bool packed, int* err,
                       cudaStream_t stream) {
  NvtxRange range("moe expert down (8-bit)");
  MOE_TRY(check_sm100());
  if (packed || use_w8t(p))
    MOE_CUDA(launch_ffn_down_w8t(p, H, offsets, Q3, S3, Y, packed, err, wait_timeout_ns(),
                                 stream),
             "expert down-projection, 8-bit weights (tcgen05, TMEM operand)");
  else
    MOE_CUDA(launch_ffn_down_w8(p, H, offsets, Q3, S3, Y, err, wait_timeout_ns(), stream),
             "expert down-projection, 8-bit weights (tcgen05)");
  return MOE_OK;
}

moe_status run_ffn(const moe_problem& p, const void* X_perm, const int32_t* offsets,
                   const Experts& w, void* H, void* Y, int* err, cudaStream_t stream) {
  if (!w.w8()) {
    MOE_TRY(run_up(p, X_perm, offsets, w.W1, w.W2, H, err, stream));
    return run_down(p, H, offsets, w.W3, Y, err, stream);
  }
  MOE_TRY(run_up_w8(p, X_perm, offsets, w.Q1, w.S1, w.Q2, w.S2, H, w.packed, err, stream));
  return run_down_w8(p, H, offsets, w.Q3, w.S3, Y, w.packed, err, stream);
}

// Extra shape rule of the 8-bit expert path: bf16 activations, and D, F multiples of 16
// (16-byte rows of int8 weights for the tensor-memory copies).
moe_status check_w8(const moe_problem& p) {
  if (p.dtype != MOE_DTYPE_BF16)
    return fail(MOE_ERR_UNSUPPORTED, "8-bit expert weights need bf16 activations");
  if (p.D % 16 != 0 || p.F % 16 != 0)
    return fail(MOE_ERR_UNSUPPORTED, "8-bit expert weights need D and F multiples of 16");
  return MOE_OK;
}

// Entry points without a noise argument: only plain top-k selection.
moe_status need_topk(const moe_problem& p) {
  if (p.routing_mode != MOE_ROUTE_TOPK)
    return fail(MOE_ERR_INVALID_ARG,
                "routing_mode needs a noise array: use moe_route_ex / moe_forward_ex");
  return MOE_OK;
}

moe_status route_impl(const moe_problem& p, const void* X, const float* W_r, const float* bias,
                      const float* noise, float* logits, int32_t* topk_idx, float* topk_gate,
                      float* prob_colsum, float* z_loss, void* ws, cudaStream_t s) {
  NvtxRange range("moe route");
  const Layout L = make_layout(p);
  if (p.N == 0) {
    if (prob_colsum) MOE_CUDA(cudaMemsetAsync(prob_colsum, 0, sizeof(float) * p.E, s), "memset");
    if (z_loss) MOE_CUDA(cudaMemsetAsync(z_loss, 0, sizeof(float), s), "memset");
    return MOE_OK;
  }
  MOE_CUDA(launch_route(p, X, W_r, bias, noise, logits, topk_idx, topk_gate,
                        at<float>(ws, L.colsum_part), prob_colsum, at<float>(ws, L.zl_part), z_loss,
                        at<void>(ws, L.route_op), at<int>(ws, L.err), wait_timeout_ns(), s),
           "route");
  return MOE_OK;
}

moe_status forward_impl(const moe_problem& p, const void* X, const float* W_r, const float* bias,
                        const float* noise, const Experts& w, void* out, float* logits,
                        int32_t* topk_idx, float* topk_gate, int32_t* load, int32_t* offsets,
                        int32_t* pos, uint8_t* dropped, float* prob_colsum, float* z_loss,
                        void* ws, cudaStream_t stream) {
  const Layout L = make_layout(p);
  int* err = at<int>(ws, L.err);
  int32_t* idx = topk_idx ? topk_idx : at<int32_t>(ws, L.idx);
  float* gate = topk_gate ? topk_gate : at<float>(ws, L.gate);
  int32_t* ld = load ? load : at<int32_t>(ws, L.load);
  int32_t* off = offsets ? offsets : at<int32_t>(ws, L.offsets);
  int32_t* ps = pos ? pos : at<int32_t>(ws, L.pos);
  uint8_t* dr = dropped ? dropped : at<uint8_t>(ws, L.dropped);
  int32_t* row_token = at<int32_t>(ws, L.row_token);
  void* xperm = at<void>(ws, L.xperm);
  void* h = at<void>(ws, L.h);
  void* y = at<void>(ws, L.y);
  if (p.N == 0) {
    MOE_CUDA(launch_slot_assign(p, 0, idx, at<int32_t>(ws, L.counts), ld, off, ps, dr, row_token,
                                err, stream),
             "dispatch");
    if (prob_colsum) MOE_CUDA(cudaMemsetAsync(prob_colsum, 0, sizeof(float) * p.E, stream), "memset");
    if (z_loss) MOE_CUDA(cudaMemsetAsync(z_loss, 0, sizeof(float), stream), "memset");
    return MOE_OK;
  }
  MOE_TRY(route_impl(p, X, W_r, bias, noise, logits, idx, gate, prob_colsum, z_loss, ws, stream));
  {
    NvtxRange range("moe dispatch");
    MOE_CUDA(launch_dispatch_fused(p, capacity_of(p), idx, at<int32_t>(ws, L.counts), ld, off,
                                   ps, dr, row_token, X, xperm, err, dispatch_bar_of(err),
                                   wait_timeout_ns(), stream),
             "dispatch");
  }
  MOE_TRY(run_ffn(p, xperm, off, w, h, y, err, stream));
  NvtxRange range("moe combine");
  MOE_CUDA(launch_combine(p, y, idx, gate, off, ps, dr, out, err, stream), "combine");
  return MOE_OK;
}

}  // namespace

extern "C" {

moe_status moe_capacity(const moe_problem* p, int64_t* C) {
  MOE_TRY(check_problem(p));
  if (C == nullptr) return fail(MOE_ERR_INVALID_ARG, "C is NULL");
  *C = capacity_of(*p);
  return MOE_OK;
}

moe_status moe_workspace_size(const moe_problem* p, size_t* bytes) {
  MOE_TRY(check_problem(p));
  if (bytes == nullptr) return fail(MOE_ERR_INVALID_ARG, "bytes is NULL");
  *bytes = make_layout(*p).total;
  return MOE_OK;
}

moe_status moe_workspace_size_host(const moe_problem* p, size_t* bytes) {
  MOE_TRY(check_problem(p));
  if (bytes == nullptr) return fail(MOE_ERR_INVALID_ARG, "bytes is NULL");
  *bytes = make_layout(*p).total_host;
  return MOE_OK;
}

moe_status moe_route(const moe_problem* p, const void* X, const float* W_r, const float* bias,
                     float* logits, int32_t* topk_idx, float* topk_gate, float* prob_colsum,
                     void* ws, size_t ws_bytes, void* stream) {
  MOE_TRY(check_problem(p));
  MOE_TRY(check_ws(*p, ws, ws_bytes, false));
  if (X != nullptr) {
    MOE_TRY(need(X, "X"));
    MOE_TRY(need(W_r, "W_r"));
    MOE_TRY(opt(logits, "logits", 4));
  } else {
    MOE_TRY(need(logits, "logits (input when X is NULL)", 4));
  }
  MOE_TRY(opt(bias, "bias", 4));
  MOE_TRY(need(topk_idx, "topk_idx", 4));
  MOE_TRY(need(topk_gate, "topk_gate", 4));
  MOE_TRY(opt(prob_colsum, "prob_colsum", 4));
  MOE_TRY(need_topk(*p));
  return route_impl(*p, X, W_r, bias, nullptr, logits, topk_idx, topk_gate, prob_colsum, nullptr,
                    ws, static_cast<cudaStream_t>(stream));
}

moe_status moe_route_ex(const moe_problem* p, const void* X, const float* W_r, const float* bias,
                        const float* noise, float* logits, int32_t* topk_idx, float* topk_gate,
                        float* prob_colsum, float* z_loss, void* ws, size_t ws_bytes,
                        void* stream) {
  MOE_TRY(check_problem(p));
  MOE_TRY(check_ws(*p, ws, ws_bytes, false));
  if (X != nullptr) {
    MOE_TRY(need(X, "X"));
    MOE_TRY(need(W_r, "W_r"));
    MOE_TRY(opt(logits, "logits", 4));
  } else {
    MOE_TRY(need(logits, "logits (input when X is NULL)", 4));
  }
  MOE_TRY(opt(bias, "bias", 4));
  if (p->routing_mode != MOE_ROUTE_TOPK && p->N > 0) MOE_TRY(need(noise, "noise", 4));
  MOE_TRY(need(topk_idx, "topk_idx", 4));
  MOE_TRY(need(topk_gate, "topk_gate", 4));
  MOE_TRY(opt(prob_colsum, "prob_colsum", 4));
  MOE_TRY(opt(z_loss, "z_loss", 4));
  return route_impl(*p, X, W_r, bias, noise, logits, topk_idx, topk_gate, prob_colsum, z_loss,
                    ws, static_cast<cudaStream_t>(stream));
}

moe_status moe_dispatch(const moe_problem* p, const void* X, const int32_t* topk_idx,
                        int32_t* load, int32_t* offsets, int32_t* pos, uint8_t* dropped,
                        int32_t* row_token, void* X_perm, void* ws, size_t ws_bytes,
                        void* stream) {
  MOE_TRY(check_problem(p));
  MOE_TRY(check_ws(*p, ws, ws_bytes, false));
  MOE_TRY(need(topk_idx, "topk_idx", 4));
  MOE_TRY(need(load, "load", 4));
  MOE_TRY(need(offsets, "offsets", 4));
  MOE_TRY(need(pos, "pos", 4));
  MOE_TRY(need(dropped, "dropped", 1));
  MOE_TRY(opt(row_token, "row_token", 4));
  const bool gather = X != nullptr && X_perm != nullptr;
  if ((X == nullptr) != (X_perm == nullptr))
    return fail(MOE_ERR_INVALID_ARG, "X and X_perm must both be given or both be NULL");
  if (gather) {
    MOE_TRY(need(X, "X"));
    MOE_TRY(need(X_perm, "X_perm"));
  }
  const Layout L = make_layout(*p);
  const cudaStream_t s = static_cast<cudaStream_t>(stream);
  int* err = at<int>(ws, L.err);
  int32_t* rt = row_token ? row_token : at<int32_t>(ws, L.row_token);
  NvtxRange range("moe dispatch");
  MOE_CUDA(launch_dispatch_fused(*p, capacity_of(*p), topk_idx, at<int32_t>(ws, L.counts), load,
                                 offsets, pos, dropped, rt, gather ? X : nullptr,
                                 gather ? X_perm : nullptr, err, dispatch_bar_of(err),
                                 wait_timeout_ns(), s),
           "dispatch");
  return MOE_OK;
}

moe_status moe_expert_ffn(const moe_problem* p, const void* X_perm, const int32_t* offsets,
                          const void* W1, const void* W2, const void* W3, void* H, void* Y,
                          void* ws, size_t ws_bytes, void* stream) {
  MOE_TRY(check_problem(p));
  MOE_TRY(check_ws(*p, ws, ws_bytes, false));
  MOE_TRY(need(X_perm, "X_perm"));
  MOE_TRY(need(offsets, "offsets", 4));
  MOE_TRY(need(W1, "W1"));
  MOE_TRY(need(W2, "W2"));
  MOE_TRY(need(W3, "W3"));
  MOE_TRY(need(H, "H"));
  MOE_TRY(need(Y, "Y"));
  if (p->N == 0) return MOE_OK;
  const Layout L = make_layout(*p);
  Experts w;
  w.W1 = W1;
  w.W2 = W2;
  w.W3 = W3;
  return run_ffn(*p, X_perm, offsets, w, H, Y, at<int>(ws, L.err),
                 static_cast<cudaStream_t>(stream));
}

moe_status moe_expert_up(const moe_problem* p, const void* X_perm, const int32_t* offsets,
                         const void* W1, const void* W2, void* H, void* ws, size_t ws_bytes,
                         void* stream) {
  MOE_TRY(check_problem(p));
  MOE_TRY(check_ws(*p, ws, ws_bytes, false));
  MOE_TRY(need(X_perm, "X_perm"));
  MOE_TRY(need(offsets, "offsets", 4));
  MOE_TRY(need(W1, "W1"));
  MOE_TRY(need(W2, "W2"));
  MOE_TRY(need(H, "H"));
  if (p->N == 0) return MOE_OK;
  const Layout L = make_layout(*p);
  return run_up(*p, X_perm, offsets, W1, W2, H, at<int>(ws, L.err),
                static_cast<cudaStream_t>(stream));
}

moe_status moe_expert_down(const moe_problem* p, const void* H, const int32_t* offsets,
                           const void* W3, void* Y, void* ws, size_t ws_bytes, void* stream) {
  MOE_TRY(check_problem(p));
  MOE_TRY(check_ws(*p, ws, ws_bytes, false));
  MOE_TRY(need(H, "H"));
  MOE_TRY(need(offsets, "offsets", 4));
  MOE_TRY(need(W3, "W3"));
  MOE_TRY(need(Y, "Y"));
  if (p->N == 0) return MOE_OK;
  const Layout L = make_layout(*p);
  return run_down(*p, H, offsets, W3, Y, at<int>(ws, L.err), static_cast<cudaStream_t>(stream));
}

moe_status moe_combine(const moe_problem* p, const void* Y, const int32_t* topk_idx,
                       const float* topk_gate, const int32_t* offsets, const int32_t* pos,
                       const uint8_t* dropped, void* out, void* stream) {
  MOE_TRY(check_problem(p));
  MOE_TRY(need(Y, "Y"));
  MOE_TRY(need(topk_idx, "topk_idx", 4));
  MOE_TRY(need(topk_gate, "topk_gate", 4));
  MOE_TRY(need(offsets, "offsets", 4));
  MOE_TRY(need(pos, "pos", 4));
  // Under a capacity some records may be dropped, and only the flags say which.
  if (p->capacity_factor > 0.0)
    MOE_TRY(need(dropped, "dropped (required when capacity_factor > 0)", 1));
  else
    MOE_TRY(opt(dropped, "dropped", 1));
  MOE_TRY(need(out, "out"));
  NvtxRange range("moe combine");
  MOE_CUDA(launch_combine(*p, Y, topk_idx, topk_gate, offsets, pos, dropped, out, nullptr,
                          static_cast<cudaStream_t>(stream)),
           "combine");
  return MOE_OK;
}

moe_status moe_forward(const moe_problem* p, const void* X, const float* W_r, const float* bias,
                       const void* W1, const void* W2, const void* W3, void* out, float* logits,
                       int32_t* topk_idx, float* topk_gate, int32_t* load, int32_t* offsets,
                       int32_t* pos, uint8_t* dropped, float* prob_colsum, void* ws,
                       size_t ws_bytes, void* stream) {
  MOE_TRY(check_problem(p));
  MOE_TRY(check_ws(*p, ws, ws_bytes, false));
  MOE_TRY(need(X, "X"));
  MOE_TRY(need(W_r, "W_r"));
  MOE_TRY(opt(bias, "bias", 4));
  MOE_TRY(need(W1, "W1"));
  MOE_TRY(need(W2, "W2"));
  MOE_TRY(need(W3, "W3"));
  MOE_TRY(need(out, "out"));
  MOE_TRY(opt(logits, "logits", 4));
  MOE_TRY(opt(topk_idx, "topk_idx", 4));
  MOE_TRY(opt(topk_gate, "topk_gate", 4));
  MOE_TRY(opt(load, "load", 4));
  MOE_TRY(opt(offsets, "offsets", 4));
  MOE_TRY(opt(pos, "pos", 4));
  MOE_TRY(opt(dropped, "dropped", 1));
  MOE_TRY(opt(prob_colsum, "prob_colsum", 4));
  Experts w;
  w.W1 = W1;
  w.W2 = W2;
  w.W3 = W3;
  MOE_TRY(need_topk(*p));
  return forward_impl(*p, X, W_r, bias, nullptr, w, out, logits, topk_idx, topk_gate, load,
                      offsets, pos, dropped, prob_colsum, nullptr, ws,
                      static_cast<cudaStream_t>(stream));
}

moe_status moe_forward_ex(const moe_problem* p, const void* X, const float* W_r,
                          const float* bias, const float* noise, const void* W1, const void* W2,
                          const void* W3, void* out, float* logits, int32_t* topk_idx,
                          float* topk_gate, int32_t* load, int32_t* offsets, int32_t* pos,
                          uint8_t* dropped, float* prob_colsum, float* z_loss, void* ws,
                          size_t ws_bytes, void* stream) {
  MOE_TRY(check_problem(p));
  MOE_TRY(check_ws(*p, ws, ws_bytes, false));
  MOE_TRY(need(X, "X"));
  MOE_TRY(need(W_r, "W_r"));
  MOE_TRY(opt(bias, "bias", 4));
  if (p->routing_mode != MOE_ROUTE_TOPK && p->N > 0) MOE_TRY(need(noise, "noise", 4));
  MOE_TRY(need(W1, "W1"));
  MOE_TRY(need(W2, "W2"));
  MOE_TRY(need(W3, "W3"));
  MOE_TRY(need(out, "out"));
  MOE_TRY(opt(logits, "logits", 4));
  MOE_TRY(opt(topk_idx, "topk_idx", 4));
  MOE_TRY(opt(topk_gate, "topk_gate", 4));
  MOE_TRY(opt(load, "load", 4));
  MOE_TRY(opt(offsets, "offsets", 4));
  MOE_TRY(opt(pos, "pos", 4));
  MOE_TRY(opt(dropped, "dropped", 1));
  MOE_TRY(opt(prob_colsum, "prob_colsum", 4));
  MOE_TRY(opt(z_loss, "z_loss", 4));
  Experts w;
  w.W1 = W1;
  w.W2 = W2;
  w.W3 = W3;
  return forward_impl(*p, X, W_r, bias, noise, w, out, logits, topk_idx, topk_gate, load,
                      offsets, pos, dropped, prob_colsum, z_loss, ws,
                      static_cast<cudaStream_t>(stream));
}

// Non-blocking streams per device for the host copies of moe_forward_host[_many] (created on
// first use, kept for the life of the process): `which` 0 carries host-to-device copies (and
// both directions in moe_forward_host), 1 device-to-host copies.
cudaError_t copy_stream(cudaStream_t* out, int which = 0) {
  static cudaStream_t streams[64][2] = {};
  static std::mutex mu;
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  if (dev < 0 || dev >= 64) return cudaErrorInvalidDevice;
  std::lock_guard<std::mutex> lock(mu);
  if (streams[dev][which] == nullptr) {
    e = cudaStreamCreateWithFlags(&streams[dev][which], cudaStreamNonBlocking);
    if (e != cudaSuccess) return e;
  }
  *out = streams[dev][which];
  return cudaSuccess;
}

// Tokens per half below which moe_forward_host does not split the batch.
constexpr int64_t kMinHalfTokens = 512;

moe_status moe_forward_host(const moe_problem* p, const void* X_host, const float* W_r,
                            const float* bias, const void* W1, const void* W2, const void* W3,
                            void* out_host, void* ws, size_t ws_bytes, void* stream) {
  MOE_TRY(check_problem(p));
  MOE_TRY(check_ws(*p, ws, ws_bytes, true));
  MOE_TRY(need_topk(*p));
  if (p->N > 0) {
    MOE_TRY(need(X_host, "X_host", 1));
    MOE_TRY(need(out_host, "out_host", 1));
  }
  MOE_TRY(need(W_r, "W_r"));
  MOE_TRY(opt(bias, "bias", 4));
  MOE_TRY(need(W1, "W1"));
  MOE_TRY(need(W2, "W2"));
  MOE_TRY(need(W3, "W3"));
  const Layout L = make_layout(*p);
  const cudaStream_t s = static_cast<cudaStream_t>(stream);
  const size_t bytes = elem_size(*p) * static_cast<size_t>(p->N) * static_cast<size_t>(p->D);
  void* xin = at<void>(ws, L.xin);
  void* xout = at<void>(ws, L.xout);
  Experts w;
  w.W1 = W1;
  w.W2 = W2;
  w.W3 = W3;
  // Without capacity every token's output depends on that token alone, so the batch runs as
  // two halves: the copy of the second half's X overlaps the first half's layer, and the copy
  // of the first half's output overlaps the second half's layer. With capacity the positions
  // depend on the whole batch, which then runs as one.
  const bool split = p->capacity_factor <= 0.0 && p->N >= 2 * kMinHalfTokens;
  if (!split) {
    if (bytes > 0) MOE_CUDA(cudaMemcpyAsync(xin, X_host, bytes, cudaMemcpyHostToDevice, s), "H2D");
    MOE_TRY(forward_impl(*p, xin, W_r, bias, nullptr, w, xout, nullptr, nullptr, nullptr,
                         nullptr, nullptr, nullptr, nullptr, nullptr, nullptr, ws, s));
    if (bytes > 0) MOE_CUDA(cudaMemcpyAsync(out_host, xout, bytes, cudaMemcpyDeviceToHost, s), "D2H");
    MOE_CUDA(cudaStreamSynchronize(s), "cudaStreamSynchronize");
    return MOE_OK;
  }
  cudaStream_t cs = nullptr;
  MOE_CUDA(copy_stream(&cs), "copy stream");
  const size_t row = elem_size(*p) * static_cast<size_t>(p->D);
  const int64_t n_half[2] = {p->N / 2, p->N - p->N / 2};
  const int64_t t_first[2] = {0, p->N / 2};
  cudaEvent_t ev[6] = {};  // start, in0, in1, done0, done1, out
  moe_status st = MOE_OK;
  for (int i = 0; i < 6 && st == MOE_OK; ++i)
    if (cudaEventCreateWithFlags(&ev[i], cudaEventDisableTiming) != cudaSuccess)
      st = fail(MOE_ERR_CUDA, "cudaEventCreateWithFlags");
  auto step = [&](cudaError_t e, const char* what) {
    if (st == MOE_OK && e != cudaSuccess) st = cuda_fail(e, what);
  };
  if (st == MOE_OK) {
    // The copies follow whatever the caller's stream has queued before this call.
    step(cudaEventRecord(ev[0], s), "event");
    step(cudaStreamWaitEvent(cs, ev[0], 0), "wait");
    for (int h = 0; h < 2; ++h) {
      step(cudaMemcpyAsync(static_cast<uint8_t*>(xin) + t_first[h] * row,
                           static_cast<const uint8_t*>(X_host) + t_first[h] * row,
                           n_half[h] * row, cudaMemcpyHostToDevice, cs),
           "H2D");
      step(cudaEventRecord(ev[1 + h], cs), "event");
    }
    for (int h = 0; h < 2 && st == MOE_OK; ++h) {
      moe_problem ph = *p;
      ph.N = n_half[h];
      step(cudaStreamWaitEvent(s, ev[1 + h], 0), "wait");
      if (st == MOE_OK)
        st = forward_impl(ph, static_cast<uint8_t*>(xin) + t_first[h] * row, W_r, bias, nullptr,
                          w, static_cast<uint8_t*>(xout) + t_first[h] * row, nullptr, nullptr,
                          nullptr, nullptr, nullptr, nullptr, nullptr, nullptr, nullptr, ws, s);
      step(cudaEventRecord(ev[3 + h], s), "event");
      step(cudaStreamWaitEvent(cs, ev[3 + h], 0), "wait");
      step(cudaMemcpyAsync(static_cast<uint8_t*>(out_host) + t_first[h] * row,
                           static_cast<const uint8_t*>(xout) + t_first[h] * row, n_half[h] * row,
                           cudaMemcpyDeviceToHost, cs),
           "D2H");
    }
    step(cudaEventRecord(ev[5], cs), "event");
    step(cudaStreamWaitEvent(s, ev[5], 0), "wait");
    step(cudaStreamSynchronize(s), "cudaStreamSynchronize");
  }
  for (int i = 0; i < 6; ++i)
    if (ev[i] != nullptr) cudaEventDestroy(ev[i]);
  return st;
}

moe_status moe_forward_host_many(const moe_problem* p, int64_t n_batches, const void* X_host,
                                 const float* W_r, const float* bias, const void* W1,
                                 const void* W2, const void* W3, void* out_host, void* ws,
                                 size_t ws_bytes, void* stream) {
  MOE_TRY(check_problem(p));
  if (n_batches < 0) return fail(MOE_ERR_INVALID_ARG, "n_batches < 0");
  MOE_TRY(check_ws(*p, ws, ws_bytes, true));
  MOE_TRY(need_topk(*p));
  if (p->N > 0 && n_batches > 0) {
    MOE_TRY(need(X_host, "X_host", 1));
    MOE_TRY(need(out_host, "out_host", 1));
  }
  MOE_TRY(need(W_r, "W_r"));
  MOE_TRY(opt(bias, "bias", 4));
  MOE_TRY(need(W1, "W1"));
  MOE_TRY(need(W2, "W2"));
  MOE_TRY(need(W3, "W3"));
  if (p->N == 0 || n_batches == 0) return MOE_OK;
  const Layout L = make_layout(*p);
  const cudaStream_t s = static_cast<cudaStream_t>(stream);
  const size_t bytes = elem_size(*p) * static_cast<size_t>(p->N) * static_cast<size_t>(p->D);
  void* xin[2] = {at<void>(ws, L.xin), at<void>(ws, L.xin2)};
  void* xout[2] = {at<void>(ws, L.xout), at<void>(ws, L.xout2)};
  cudaStream_t cs_in = nullptr, cs_out = nullptr;
  MOE_CUDA(copy_stream(&cs_in, 0), "copy stream");
  MOE_CUDA(copy_stream(&cs_out, 1), "copy stream");
  Experts w;
  w.W1 = W1;
  w.W2 = W2;
  w.W3 = W3;
  // Batch b uses buffer pair b % 2. Its input copy waits until batch b-2's layer has read that
  // buffer, its layer until batch b-2's output copy has read the output buffer, so the input
  // copy of batch b+1 and the output copy of batch b-1 run under batch b's layer.
  cudaEvent_t ev[7] = {};  // start, in_done[2], comp_done[2], out_done[2]
  cudaEvent_t* in_done = ev + 1;
  cudaEvent_t* comp_done = ev + 3;
  cudaEvent_t* out_done = ev + 5;
  moe_status st = MOE_OK;
  for (int i = 0; i < 7 && st == MOE_OK; ++i)
    if (cudaEventCreateWithFlags(&ev[i], cudaEventDisableTiming) != cudaSuccess)
      st = fail(MOE_ERR_CUDA, "cudaEventCreateWithFlags");
  auto step = [&](cudaError_t e, const char* what) {
    if (st == MOE_OK && e != cudaSuccess) st = cuda_fail(e, what);
  };
  int64_t issued = 0;  // batches whose output copy was enqueued
  if (st == MOE_OK) {
    // The copies follow whatever the caller's stream has queued before this call.
    step(cudaEventRecord(ev[0], s), "event");
    step(cudaStreamWaitEvent(cs_in, ev[0], 0), "wait");
    step(cudaStreamWaitEvent(cs_out, ev[0], 0), "wait");
    for (int64_t b = 0; b < n_batches && st == MOE_OK; ++b) {
      const int slot = static_cast<int>(b & 1);
      const uint8_t* xh = static_cast<const uint8_t*>(X_host) + static_cast<size_t>(b) * bytes;
      uint8_t* oh = static_cast<uint8_t*>(out_host) + static_cast<size_t>(b) * bytes;
      if (b >= 2) step(cudaStreamWaitEvent(cs_in, comp_done[slot], 0), "wait");
      step(cudaMemcpyAsync(xin[slot], xh, bytes, cudaMemcpyHostToDevice, cs_in), "H2D");
      step(cudaEventRecord(in_done[slot], cs_in), "event");
      step(cudaStreamWaitEvent(s, in_done[slot], 0), "wait");
      if (b >= 2) step(cudaStreamWaitEvent(s, out_done[slot], 0), "wait");
      if (st == MOE_OK)
        st = forward_impl(*p, xin[slot], W_r, bias, nullptr, w, xout[slot], nullptr, nullptr,
                          nullptr, nullptr, nullptr, nullptr, nullptr, nullptr, nullptr, ws, s);
      step(cudaEventRecord(comp_done[slot], s), "event");
      step(cudaStreamWaitEvent(cs_out, comp_done[slot], 0), "wait");
      step(cudaMemcpyAsync(oh, xout[slot], bytes, cudaMemcpyDeviceToHost, cs_out), "D2H");
      step(cudaEventRecord(out_done[slot], cs_out), "event");
      if (st == MOE_OK) issued = b + 1;
    }
  }
  // Join: the caller's stream waits for every enqueued output copy, then the host waits.
  for (int i = 0; i < 2 && i < issued; ++i) cudaStreamWaitEvent(s, out_done[i], 0);
  if (issued > 0 || st != MOE_OK) {
    const cudaError_t e = cudaStreamSynchronize(s);
    if (st == MOE_OK && e != cudaSuccess) st = cuda_fail(e, "cudaStreamSynchronize");
    if (st != MOE_OK) {  // after an error, wait for the copy streams too before returning
      cudaStreamSynchronize(cs_in);
      cudaStreamSynchronize(cs_out);
    }
  }
  for (int i = 0; i < 7; ++i)
    if (ev[i] != nullptr) cudaEventDestroy(ev[i]);
  return st;
}

moe_status moe_expert_up_w8(const moe_problem* p, const void* X_perm, const int32_t* offsets,
                            const int8_t* W1q, const float* S1, const int8_t* W2q,
                            const float* S2, void* H, void* ws, size_t ws_bytes, void* stream) {
  MOE_TRY(check_problem(p));
  MOE_TRY(check_w8(*p));
  MOE_TRY(check_ws(*p, ws, ws_bytes, false));
  MOE_TRY(need(X_perm, "X_perm"));
  MOE_TRY(need(offsets, "offsets", 4));
  MOE_TRY(need(W1q, "W1q"));
  MOE_TRY(need(S1, "S1"));
  MOE_TRY(need(W2q, "W2q"));
  MOE_TRY(need(S2, "S2"));
  MOE_TRY(need(H, "H"));
  if (p->N == 0) return MOE_OK;
  const Layout L = make_layout(*p);
  return run_up_w8(*p, X_perm, offsets, W1q, S1, W2q, S2, H, false, at<int>(ws, L.err),
                   static_cast<cudaStream_t>(stream));
}

moe_status moe_expert_down_w8(const moe_problem* p, const void* H, const int32_t* offsets,
                              const int8_t* W3q, const float* S3, void* Y, void* ws,
                              size_t ws_bytes, void* stream) {
  MOE_TRY(check_problem(p));
  MOE_TRY(check_w8(*p));
  MOE_TRY(check_ws(*p, ws, ws_bytes, false));
  MOE_TRY(need(H, "H"));
  MOE_TRY(need(offsets, "offsets", 4));
  MOE_TRY(need(W3q, "W3q"));
  MOE_TRY(need(S3, "S3"));
  MOE_TRY(need(Y, "Y"));
  if (p->N == 0) return MOE_OK;
  const Layout L = make_layout(*p);
  return run_down_w8(*p, H, offsets, W3q, S3, Y, false, at<int>(ws, L.err),
                     static_cast<cudaStream_t>(stream));
}

}  // extern "C"

namespace {

moe_status forward_w8_impl(const moe_problem* p, const void* X, const float* W_r,
                           const float* bias, const int8_t* W1q, const float* S1,
                           const int8_t* W2q, const float* S2, const int8_t* W3q,
                           const float* S3, void* out, float* logits, int32_t* topk_idx,
                           float* topk_gate, int32_t* load, int32_t* offsets, int32_t* pos,
                           uint8_t* dropped, float* prob_colsum, void* ws, size_t ws_bytes,
                           void* stream, bool packed) {
  MOE_TRY(check_problem(p));
  MOE_TRY(check_w8(*p));
  MOE_TRY(check_ws(*p, ws, ws_bytes, false));
  MOE_TRY(need(X, "X"));
  MOE_TRY(need(W_r, "W_r"));
  MOE_TRY(opt(bias, "bias", 4));
  MOE_TRY(need(W1q, "W1q"));
  MOE_TRY(need(S1, "S1"));
  MOE_TRY(need(W2q, "W2q"));
  MOE_TRY(need(S2, "S2"));
  MOE_TRY(need(W3q, "W3q"));
  MOE_TRY(need(S3, "S3"));
  MOE_TRY(need(out, "out"));
  MOE_TRY(opt(logits, "logits", 4));
  MOE_TRY(opt(topk_idx, "topk_idx", 4));
  MOE_TRY(opt(topk_gate, "topk_gate", 4));
  MOE_TRY(opt(load, "load", 4));
  MOE_TRY(opt(offsets, "offsets", 4));
  MOE_TRY(opt(pos, "pos", 4));
  MOE_TRY(opt(dropped, "dropped", 1));
  MOE_TRY(opt(prob_colsum, "prob_colsum", 4));
  Experts w;
  w.Q1 = W1q;
  w.Q2 = W2q;
  w.Q3 = W3q;
  w.S1 = S1;
  w.S2 = S2;
  w.S3 = S3;
  w.packed = packed;
  MOE_TRY(need_topk(*p));
  return forward_impl(*p, X, W_r, bias, nullptr, w, out, logits, topk_idx, topk_gate, load,
                      offsets, pos, dropped, prob_colsum, nullptr, ws,
                      static_cast<cudaStream_t>(stream));
}

}  // namespace

extern "C" {

moe_status moe_forward_w8(const moe_problem* p, const void* X, const float* W_r,
                          const float* bias, const int8_t* W1q, const float* S1,
                          const int8_t* W2q, const float* S2, const int8_t* W3q, const float* S3,
                          void* out, float* logits, int32_t* topk_idx, float* topk_gate,
                          int32_t* load, int32_t* offsets, int32_t* pos, uint8_t* dropped,
                          float* prob_colsum, void* ws, size_t ws_bytes, void* stream) {
  return forward_w8_impl(p, X, W_r, bias, W1q, S1, W2q, S2, W3q, S3, out, logits, topk_idx,
                         topk_gate, load, offsets, pos, dropped, prob_colsum, ws, ws_bytes,
                         stream, false);
}

moe_status moe_forward_w8p(const moe_problem* p, const void* X, const float* W_r,
                           const float* bias, const int8_t* W1p, const float* S1,
                           const int8_t* W2p, const float* S2, const int8_t* W3p,
                           const float* S3, void* out, float* logits, int32_t* topk_idx,
                           float* topk_gate, int32_t* load, int32_t* offsets, int32_t* pos,
                           uint8_t* dropped, float* prob_colsum, void* ws, size_t ws_bytes,
                           void* stream) {
  return forward_w8_impl(p, X, W_r, bias, W1p, S1, W2p, S2, W3p, S3, out, logits, topk_idx,
                         topk_gate, load, offsets, pos, dropped, prob_colsum, ws, ws_bytes,
                         stream, true);
}

moe_status moe_pack_w8(const moe_problem* p, const int8_t* W1q, const int8_t* W2q,
                       const int8_t* W3q, int8_t* W1p, int8_t* W2p, int8_t* W3p, void* stream) {
  MOE_TRY(check_problem(p));
  MOE_TRY(check_w8(*p));
  MOE_TRY(need(W1q, "W1q"));
  MOE_TRY(need(W2q, "W2q"));
  MOE_TRY(need(W3q, "W3q"));
  MOE_TRY(need(W1p, "W1p"));
  MOE_TRY(need(W2p, "W2p"));
  MOE_TRY(need(W3p, "W3p"));
  MOE_TRY(check_sm100());
  const cudaStream_t s = static_cast<cudaStream_t>(stream);
  MOE_CUDA(launch_pack_w8(W1q, W1p, p->E, p->D, p->F, s), "pack W1");
  MOE_CUDA(launch_pack_w8(W2q, W2p, p->E, p->D, p->F, s), "pack W2");
  MOE_CUDA(launch_pack_w8(W3q, W3p, p->E, p->F, p->D, s), "pack W3");
  return MOE_OK;
}

moe_status moe_expert_up_w8p(const moe_problem* p, const void* X_perm, const int32_t* offsets,
                             const int8_t* W1p, const float* S1, const int8_t* W2p,
                             const float* S2, void* H, void* ws, size_t ws_bytes, void* stream) {
  MOE_TRY(check_problem(p));
  MOE_TRY(check_w8(*p));
  MOE_TRY(check_ws(*p, ws, ws_bytes, false));
  MOE_TRY(need(X_perm, "X_perm"));
  MOE_TRY(need(offsets, "offsets", 4));
  MOE_TRY(need(W1p, "W1p"));
  MOE_TRY(need(S1, "S1"));
  MOE_TRY(need(W2p, "W2p"));
  MOE_TRY(need(S2, "S2"));
  MOE_TRY(need(H, "H"));
  if (p->N == 0) return MOE_OK;
  const Layout L = make_layout(*p);
  return run_up_w8(*p, X_perm, offsets, W1p, S1, W2p, S2, H, true, at<int>(ws, L.err),
                   static_cast<cudaStream_t>(stream));
}

moe_status moe_expert_down_w8p(const moe_problem* p, const void* H, const int32_t* offsets,
                               const int8_t* W3p, const float* S3, void* Y, void* ws,
                               size_t ws_bytes, void* stream) {
  MOE_TRY(check_problem(p));
  MOE_TRY(check_w8(*p));
  MOE_TRY(check_ws(*p, ws, ws_bytes, false));
  MOE_TRY(need(H, "H"));
  MOE_TRY(need(offsets, "offsets", 4));
  MOE_TRY(need(W3p, "W3p"));
  MOE_TRY(need(S3, "S3"));
  MOE_TRY(need(Y, "Y"));
  if (p->N == 0) return MOE_OK;
  const Layout L = make_layout(*p);
  return run_down_w8(*p, H, offsets, W3p, S3, Y, true, at<int>(ws, L.err),
                     static_cast<cudaStream_t>(stream));
}

moe_status moe_gather_rows(const void* src, int64_t n_src_rows, const int32_t* index,
                           int64_t n_rows, int64_t row_bytes, void* dst, void* ws,
                           size_t ws_bytes, void* stream) {
  if (n_rows < 0 || n_src_rows < 0)
    return fail(MOE_ERR_INVALID_ARG, "n_rows and n_src_rows must be >= 0");
  if (row_bytes <= 0 || row_bytes % 4 != 0)
    return fail(MOE_ERR_INVALID_ARG, "row_bytes must be a positive multiple of 4");
  MOE_TRY(need(ws, "ws", 256));
  if (ws_bytes < 256) return fail(MOE_ERR_INVALID_ARG, "workspace smaller than 256 bytes");
  if (n_rows == 0) return MOE_OK;
  MOE_TRY(need(index, "index", 4));
  MOE_TRY(need(dst, "dst"));
  if (n_src_rows > 0) MOE_TRY(need(src, "src"));
  MOE_CUDA(launch_gather_rows(src, n_src_rows, index, n_rows, row_bytes, dst,
                              static_cast<int*>(ws), static_cast<cudaStream_t>(stream)),
           "gather rows");
  return MOE_OK;
}

moe_status moe_balance_loss(const moe_problem* p, const int32_t* load, const float* prob_colsum,
                            double* loss) {
  MOE_TRY(check_problem(p));
  if (load == nullptr || prob_colsum == nullptr || loss == nullptr)
    return fail(MOE_ERR_INVALID_ARG, "load, prob_colsum and loss must not be NULL");
  *loss = 0.0;
  if (p->N == 0) return MOE_OK;
  const double records = static_cast<double>(p->N) * static_cast<double>(p->k);
  const double tokens = static_cast<double>(p->N);
  double sum = 0.0;
  for (int32_t e = 0; e < p->E; ++e)  // f_e = share of the records, P_e = mean probability
    sum += (static_cast<double>(load[e]) / records) * (static_cast<double>(prob_colsum[e]) / tokens);
  *loss = static_cast<double>(p->E) * sum;
  return MOE_OK;
}

moe_status moe_drop_rate(const moe_problem* p, const uint8_t* dropped, double* rate) {
  MOE_TRY(check_problem(p));
  if (rate == nullptr) return fail(MOE_ERR_INVALID_ARG, "rate must not be NULL");
  *rate = 0.0;
  const int64_t records = p->N * static_cast<int64_t>(p->k);
  if (records == 0) return MOE_OK;
  if (dropped == nullptr) return fail(MOE_ERR_INVALID_ARG, "dropped must not be NULL");
  int64_t n = 0;
  for (int64_t r = 0; r < records; ++r) n += dropped[r] != 0 ? 1 : 0;
  *rate = static_cast<double>(n) / static_cast<double>(records);
  return MOE_OK;
}

moe_status moe_selftest_wait_timeout(void* ws, size_t ws_bytes, int64_t timeout_us,
                                     void* stream) {
  MOE_TRY(need(ws, "ws", 256));
  if (ws_bytes < 256) return fail(MOE_ERR_INVALID_ARG, "workspace smaller than 256 bytes");
  if (timeout_us < 1 || timeout_us > 10000000)
    return fail(MOE_ERR_INVALID_ARG, "timeout_us must be in [1, 1e7]");
  MOE_CUDA(launch_wait_timeout_probe(static_cast<int*>(ws),
                                     static_cast<uint64_t>(timeout_us) * 1000ull,
                                     static_cast<cudaStream_t>(stream)),
           "wait-timeout self-test");
  return MOE_OK;
}

moe_status moe_workspace_init(void* ws, size_t ws_bytes, void* stream) {
  MOE_TRY(need(ws, "ws", 256));
  if (ws_bytes < 256) return fail(MOE_ERR_INVALID_ARG, "workspace smaller than 256 bytes");
  MOE_CUDA(cudaMemsetAsync(ws, 0, 256, static_cast<cudaStream_t>(stream)), "memset");
  return MOE_OK;
}

moe_status moe_get_device_error(void* ws, void* stream, int32_t* code) {
  if (ws == nullptr || code == nullptr) return fail(MOE_ERR_INVALID_ARG, "ws or code is NULL");
  const cudaStream_t s = static_cast<cudaStream_t>(stream);
  MOE_CUDA(cudaStreamSynchronize(s), "cudaStreamSynchronize");
  int32_t v = 0;
  MOE_CUDA(cudaMemcpy(&v, ws, sizeof(v), cudaMemcpyDeviceToHost), "read error word");
  *code = v;
  if (v != 0) {
    MOE_CUDA(cudaMemset(ws, 0, sizeof(v)), "clear error word");
    return fail(MOE_ERR_DEVICE, "device error code " + std::to_string(v));
  }
  return MOE_OK;
}

const char* moe_status_string(moe_status s) {
  switch (s) {
    case MOE_OK: return "ok";
    case MOE_ERR_INVALID_ARG: return "invalid argument";
    case MOE_ERR_UNSUPPORTED: return "unsupported problem";
    case MOE_ERR_CUDA: return "CUDA error";
    case MOE_ERR_DEVICE: return "device-side error";
  }
  return "unknown status";
}

const char* moe_last_error(void) { return g_last_error.c_str(); }

int32_t moe_version(void) { return 120; }

}  // extern "C"

namespace moe {

// Lets entry points defined in other files report through moe_last_error().
void set_last_error(const std::string& msg) { g_last_error = msg; }

}  // namespace moe

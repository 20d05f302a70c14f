// moe_dispatch_noalloc: the dispatch step for callers that cannot hand the library any
// device memory of its own -- for example code that runs after its process has stopped
// allocating (a serving loop that forbids cudaMalloc because it synchronises the device and
// can stall every stream), or a host that owns all device memory through its own pool and
// only lends out the tensors it computes on.
//
// It runs the same count and slot-assignment kernels (and, optionally, the gather) as
// moe_dispatch, but the per-chunk expert counters they need live in the fixed array below
// instead of a caller-provided workspace. The array is part of the library image: every GPU
// that loads the library keeps it until the process exits.
#include <mutex>
#include <string>

#include "../../include/moe.h"
#include "internal.h"

namespace {

// Per-chunk expert counters: ceil(N*k / 1024) * E int32 values must fit.
constexpr int kScratchInts = 16384;  // 64 KiB
static __device__ __align__(256) int32_t g_dispatch_counts[kScratchInts];

// The calling thread's current CUDA context (driver handle), or nullptr if it cannot be read.
CUcontext current_context() {
  using GetCurrent = CUresult (*)(CUcontext*);
  static GetCurrent fn = [] {
    void* ptr = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuCtxGetCurrent", &ptr, cudaEnableDefault, &q) !=
            cudaSuccess ||
        q != cudaDriverEntryPointSuccess)
      return static_cast<GetCurrent>(nullptr);
    return reinterpret_cast<GetCurrent>(ptr);
  }();
  CUcontext c = nullptr;
  if (fn == nullptr || fn(&c) != CUDA_SUCCESS) return nullptr;
  return c;
}

// Device address of g_dispatch_counts, looked up once per device (and context) with that
// device current. In host code the symbol itself is only a host-side stand-in, never a device
// address. The address belongs to the context the module was loaded into: after
// cudaDeviceReset the device gets a new primary context, whose handle differs, and the
// address is looked up again.
cudaError_t scratch_address(int32_t** out) {
  static std::mutex mu;
  static int32_t* addr[64] = {nullptr};
  static CUcontext ctx[64] = {nullptr};
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  if (dev < 0 || dev >= 64) return cudaErrorInvalidDevice;
  const CUcontext cur = current_context();  // nullptr before the device's first runtime call
  std::lock_guard<std::mutex> lock(mu);
  if (addr[dev] == nullptr || cur == nullptr || ctx[dev] != cur) {
    void* p = nullptr;
    e = cudaGetSymbolAddress(&p, g_dispatch_counts);  // sets up the primary context if needed
    if (e != cudaSuccess) return e;
    addr[dev] = static_cast<int32_t*>(p);
    ctx[dev] = current_context();
  }
  *out = addr[dev];
  return cudaSuccess;
}

moe_status noalloc_fail(moe_status s, const std::string& msg) {
  moe::set_last_error("moe_dispatch_noalloc: " + msg);
  return s;
}

bool misaligned(const void* p, uintptr_t a) { return (reinterpret_cast<uintptr_t>(p) % a) != 0; }

}  // namespace

extern "C" moe_status moe_dispatch_noalloc(const moe_problem* p, const void* X,
                                           const int32_t* topk_idx, int32_t* load,
                                           int32_t* offsets, int32_t* pos, uint8_t* dropped,
                                           int32_t* row_token, void* X_perm, void* stream) {
  size_t ws_bytes = 0;
  // Same problem checks as every other entry point (host only, allocates nothing).
  const moe_status st = moe_workspace_size(p, &ws_bytes);
  if (st != MOE_OK) return st;
  if (topk_idx == nullptr || load == nullptr || offsets == nullptr || pos == nullptr ||
      dropped == nullptr || row_token == nullptr)
    return noalloc_fail(MOE_ERR_INVALID_ARG,
                        "topk_idx, load, offsets, pos, dropped and row_token are required");
  if (misaligned(topk_idx, 4) || misaligned(load, 4) || misaligned(offsets, 4) ||
      misaligned(pos, 4) || misaligned(row_token, 4))
    return noalloc_fail(MOE_ERR_INVALID_ARG, "int32 arrays must be 4-byte aligned");
  if ((X == nullptr) != (X_perm == nullptr))
    return noalloc_fail(MOE_ERR_INVALID_ARG, "X and X_perm must both be given or both be NULL");
  if (X != nullptr && (misaligned(X, 16) || misaligned(X_perm, 16)))
    return noalloc_fail(MOE_ERR_INVALID_ARG, "X and X_perm must be 16-byte aligned");
  const int64_t records = p->N * static_cast<int64_t>(p->k);
  const int64_t need = static_cast<int64_t>(moe::dispatch_num_chunks(records)) * p->E;
  if (need > kScratchInts)
    return noalloc_fail(MOE_ERR_UNSUPPORTED,
                        "ceil(N*k/1024)*E = " + std::to_string(need) +
                            " exceeds the fixed scratch of " + std::to_string(kScratchInts) +
                            " counters; use moe_dispatch with a workspace");
  int32_t* counts = nullptr;
  cudaError_t e = scratch_address(&counts);
  if (e != cudaSuccess)
    return noalloc_fail(MOE_ERR_CUDA, std::string("cudaGetSymbolAddress: ") + cudaGetErrorString(e));
  // The count kernel overwrites every counter it later reads, so nothing needs clearing.
  int64_t C = records;
  if (p->capacity_factor > 0.0) {
    const moe_status cs = moe_capacity(p, &C);
    if (cs != MOE_OK) return cs;
  }
  const cudaStream_t s = static_cast<cudaStream_t>(stream);
  e = moe::launch_slot_assign(*p, C, topk_idx, counts, load, offsets, pos, dropped, row_token,
                              nullptr, s);
  if (e == cudaSuccess && X != nullptr)
    e = moe::launch_gather(*p, X, row_token, offsets, X_perm, nullptr, s);
  if (e != cudaSuccess)
    return noalloc_fail(MOE_ERR_CUDA, std::string("launch: ") + cudaGetErrorString(e));
  return MOE_OK;
}

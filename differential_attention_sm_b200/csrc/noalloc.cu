// noalloc.cu — V2 single-token decode for callers that cannot allocate
// device memory.
//
// diffattn_v2_decode needs a caller-provided scratch workspace for its
// split-KV partial results.  Some callers cannot provide one: code that runs
// where cudaMalloc is not allowed or not wanted (a serving loop that must
// never block the device on an allocation, a plug-in inside a host framework
// that owns every device buffer, a runtime with a fixed memory budget set at
// start-up).  This entry point runs the same split-KV kernels with their
// scratch placed in one statically allocated device array,
// g_decode_scratch (DA_NOALLOC_SCRATCH_BYTES = 8 MiB), and calls no
// allocating routine.
//
// Set-up: the device address of the array is looked up with
// cudaGetSymbolAddress the first time the entry point runs on a device (with
// that device current) and cached for that device and its current CUDA
// context; that first call should come before any stream capture.  A call
// made under another context of the same device (after cudaDeviceReset has
// replaced the primary context, or under a context the caller created with
// the driver API) looks the address up again for that context.  In host
// code the array's name is only a host-side stand-in, so the kernels always
// receive the looked-up address.
// Shared state: every call on a device uses the same array and leaves its
// contents behind.  Nothing in it has to start at zero (each partial the
// combine step reads is written earlier in the same call), but calls whose
// execution overlaps on the GPU (different streams, or concurrent host
// threads) race on the array and must be serialised by the caller.
#include <cuda.h>
#include <cuda_runtime.h>

#include <cstdint>
#include <mutex>

#include "diffattn.h"
#include "kernels.h"

namespace {

constexpr size_t kScratchBytes = DA_NOALLOC_SCRATCH_BYTES;
constexpr int kPlanSMs = 148;   // same split planning basis as diffattn_v2_decode
constexpr int kMaxDevices = 64;

static __device__ __align__(256) unsigned char g_decode_scratch[kScratchBytes];

// The looked-up address of g_decode_scratch per device, with the CUDA
// context it belongs to.
struct ScratchEntry {
  CUcontext ctx = nullptr;
  void* addr = nullptr;
};
ScratchEntry g_scratch[kMaxDevices];
std::mutex g_scratch_mu;

typedef CUresult (*CtxGetCurrentFn)(CUcontext*);

CtxGetCurrentFn ctx_get_current_fn() {
  static CtxGetCurrentFn fn = []() -> CtxGetCurrentFn {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuCtxGetCurrent", &p, cudaEnableDefault, &q) != cudaSuccess ||
        q != cudaDriverEntryPointSuccess)
      return nullptr;
    return reinterpret_cast<CtxGetCurrentFn>(p);
  }();
  return fn;
}

// Device address of g_decode_scratch in the current device's current context
// (looked up on the first call in each context).
int scratch_address(void** out) {
  int dev = -1;
  if (cudaGetDevice(&dev) != cudaSuccess) return DA_ERR_CUDA;
  if (dev < 0 || dev >= kMaxDevices) return DA_ERR_UNSUPPORTED;
  CtxGetCurrentFn get_ctx = ctx_get_current_fn();
  if (!get_ctx) return DA_ERR_CUDA;
  CUcontext ctx = nullptr;
  if (get_ctx(&ctx) != CUDA_SUCCESS) return DA_ERR_CUDA;
  std::lock_guard<std::mutex> lock(g_scratch_mu);
  ScratchEntry& e = g_scratch[dev];
  if (ctx == nullptr || e.ctx != ctx || e.addr == nullptr) {
    // the lookup also binds the runtime's context to this thread if none was
    void* addr = nullptr;
    if (cudaGetSymbolAddress(&addr, g_decode_scratch) != cudaSuccess || addr == nullptr)
      return DA_ERR_CUDA;
    if (get_ctx(&ctx) != CUDA_SUCCESS || ctx == nullptr) return DA_ERR_CUDA;
    e.ctx = ctx;
    e.addr = addr;
  }
  *out = e.addr;
  return DA_OK;
}

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

}  // namespace

extern "C" DA_API int diffattn_v2_decode_noalloc(const void* q, const void* k_cache,
                                                 const void* v_cache, const int* cache_lens,
                                                 int max_len, void* out, int batch,
                                                 int n_q_heads, int n_kv_heads,
                                                 const float* lambda, int* dev_status,
                                                 void* stream) {
  if (!q || !k_cache || !v_cache || !out || !lambda) return DA_ERR_INVALID_ARG;
  if (batch < 1 || max_len < 1 || n_q_heads < 2 || n_kv_heads < 1) return DA_ERR_INVALID_ARG;
  if (n_q_heads % n_kv_heads != 0) return DA_ERR_INVALID_ARG;
  const int group = n_q_heads / n_kv_heads;
  if (group % 2 != 0) return DA_ERR_INVALID_ARG;
  if (group > 8) return DA_ERR_UNSUPPORTED;
  if ((long long)batch * max_len >= (1LL << 31) ||
      (long long)max_len * n_kv_heads * 128 >= (1LL << 31))
    return DA_ERR_UNSUPPORTED;
  if (!aligned16(q) || !aligned16(k_cache) || !aligned16(v_cache) || !aligned16(out))
    return DA_ERR_ALIGNMENT;
  // Sizes whose partial results cannot fit in the fixed scratch are refused.
  da::V2DecodePlan plan =
      da::plan_v2_decode_capped(batch, n_kv_heads, max_len, kPlanSMs, kScratchBytes);
  if (plan.n_items == 0) return DA_ERR_UNSUPPORTED;
  void* scratch = nullptr;
  int rc = scratch_address(&scratch);
  if (rc != DA_OK) return rc;
  int dev = 0, sms = 0;
  if (cudaGetDevice(&dev) != cudaSuccess ||
      cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess ||
      sms < 1)
    return DA_ERR_CUDA;
  plan.grid = plan.n_items < sms ? plan.n_items : sms;
  CUtensorMap tk, tv;
  if (da::make_tmap_bf16_4d(&tk, k_cache, 128, n_kv_heads, max_len, batch, 64, 1, 64, 1) ||
      da::make_tmap_bf16_4d(&tv, v_cache, 128, n_kv_heads, max_len, batch, 64, 1, 64, 1))
    return DA_ERR_CUDA;
  cudaError_t e = da::launch_v2_decode(tk, tv, q, cache_lens, max_len, 0, out, batch, n_q_heads,
                                       n_kv_heads, lambda, plan, scratch, dev_status,
                                       static_cast<cudaStream_t>(stream));
  return e == cudaSuccess ? DA_OK : DA_ERR_CUDA;
}

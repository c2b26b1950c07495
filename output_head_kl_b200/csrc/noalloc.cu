// kdkl_forward_noalloc: the forward for callers that cannot allocate device
// memory.  Some callers cannot hand the library a workspace: a loss hook whose
// host framework passes only inputs and outputs, a runtime that pre-plans every
// device byte at start-up and forbids later allocations, or a latency-critical
// loop that must not call cudaMalloc because it may synchronise the device.
// This entry point needs nothing from them beyond inputs and outputs: its
// scratch is one file-scope device array, kStaticScratchBytes long, that every
// GPU loading the library holds until the process exits.
#include <cstdio>
#include <mutex>

#include "../../include/kdkl.h"
#include "kdkl_internal.h"

namespace {

constexpr size_t kStaticScratchBytes = size_t(32) << 20;  // 32 MiB per device
constexpr int kMaxDevices = 64;

__device__ __align__(256) unsigned char g_static_scratch[kStaticScratchBytes];

// The array's address is looked up once per device and primary context: a new
// context (after cudaDeviceReset, say) loads the module again, so the array may
// move, and the lookup is then redone.
typedef CUresult (*CtxGetCurrentFn)(CUcontext*);

CtxGetCurrentFn ctx_get_current() {
  static CtxGetCurrentFn fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPointByVersion("cuCtxGetCurrent", &p, 12000, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<CtxGetCurrentFn>(p);
  });
  return fn;
}

std::mutex g_mu;
void* g_scratch_addr[kMaxDevices] = {nullptr};
CUcontext g_scratch_ctx[kMaxDevices] = {nullptr};

kdkl_status reject(kdkl_status st, const char* msg) {
  kdkl::set_last_error(msg);
  return st;
}

}  // namespace

extern "C" kdkl_status kdkl_forward_noalloc(const void* hidden, const void* W, const int32_t* topk_idx,
                                            const float* topk_logit, const uint8_t* mask, int64_t N, int32_t d,
                                            int32_t V, int32_t K, float tau, float* loss, float* lse,
                                            void* stream) {
  // Shapes the forward rejects anyway: let it report them (it returns before any launch).
  if (kdkl_workspace_bytes(N, d, V, K, 0) == 0)
    return kdkl_forward(hidden, W, topk_idx, topk_logit, mask, N, d, V, K, tau, loss, lse, nullptr, 0, stream);
  const size_t need = kdkl::make_layout(N, d, V, K, 0).gbuf;
  if (need > kStaticScratchBytes) {
    char msg[256];
    snprintf(msg, sizeof(msg),
             "kdkl_forward_noalloc: N=%lld, K=%d need %zu bytes of scratch; the built-in scratch holds %zu "
             "(use kdkl_forward with a caller workspace)",
             (long long)N, K, need, kStaticScratchBytes);
    return reject(KDKL_ERR_UNSUPPORTED, msg);
  }
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return reject(KDKL_ERR_UNSUPPORTED, "kdkl_forward_noalloc: no CUDA device");
  if (dev < 0 || dev >= kMaxDevices) return reject(KDKL_ERR_UNSUPPORTED, "kdkl_forward_noalloc: device index too large");
  // The current context, if this thread has one yet (a thread whose only CUDA call so
  // far is cudaGetDevice may not): without one the lookup below runs, which binds it.
  CUcontext ctx = nullptr;
  CtxGetCurrentFn get_ctx = ctx_get_current();
  if (get_ctx && get_ctx(&ctx) != CUDA_SUCCESS) ctx = nullptr;
  void* scratch = nullptr;
  {
    // Set-up, once per device and context, with that device current: the host-side
    // name of the array is not a device address, so ask the runtime for this device's copy.
    std::lock_guard<std::mutex> lk(g_mu);
    if (!g_scratch_addr[dev] || !ctx || g_scratch_ctx[dev] != ctx) {
      void* p = nullptr;
      const cudaError_t e = cudaGetSymbolAddress(&p, g_static_scratch);
      if (e != cudaSuccess || p == nullptr) {
        char msg[256];
        snprintf(msg, sizeof(msg), "kdkl_forward_noalloc: cudaGetSymbolAddress failed: %s", cudaGetErrorString(e));
        return reject(KDKL_ERR_CUDA, msg);
      }
      if (get_ctx && get_ctx(&ctx) != CUDA_SUCCESS) ctx = nullptr;
      g_scratch_addr[dev] = p;
      g_scratch_ctx[dev] = ctx;
    }
    scratch = g_scratch_addr[dev];
  }
  // The forward clears the scratch's header words itself and overwrites every
  // other scratch byte it later reads, so leftovers of an earlier call do not matter.
  return kdkl_forward(hidden, W, topk_idx, topk_logit, mask, N, d, V, K, tau, loss, lse, scratch,
                      kStaticScratchBytes, stream);
}

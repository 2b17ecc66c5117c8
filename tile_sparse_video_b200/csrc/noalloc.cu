// vsa_coarse_topk_noalloc: steps 2 and 3 without any caller-supplied or
// library-allocated workspace.
//
// Some callers cannot call cudaMalloc: a host application that owns all device
// memory through its own pool and hands plugins no allocator, or a latency-
// critical loop where cudaMalloc's implicit device-wide synchronisation would
// stall unrelated streams.  For them this entry point keeps the pooled-mean
// scratch (the only scratch memory of vsa_coarse_topk) in a fixed-size array in
// the library's own device memory.
//
// The array is a file-scope __device__ variable: every GPU that loads this
// module holds its kStaticScratchBytes until the process exits.  Host code
// cannot use the array's name as a device address (it names a host-side
// stand-in), so the first call on each device, with that device current,
// resolves the real address with cudaGetSymbolAddress and caches it (again
// when a later call finds another CUDA context current, as after a reset).  That
// first call on a device therefore does a one-time runtime query; make it
// before any stream capture.
//
// All calls share the array and it keeps the last call's contents.  Nothing in
// it needs to start at zero: the pooling kernel overwrites every value it later
// reads.  Calls whose executions overlap on the GPU (different streams, or
// different threads) race on the array and must be serialised by the caller.
#include <cuda.h>

#include <mutex>

#include "vsa_internal.h"

namespace {

constexpr size_t kStaticScratchBytes = size_t(16) << 20;   // 16 MiB
static __device__ __align__(256) float g_static_scratch[kStaticScratchBytes / sizeof(float)];

constexpr int kMaxDevices = 64;
std::mutex g_scratch_mu;
void* g_scratch_addr[kMaxDevices] = {};
CUcontext g_scratch_ctx[kMaxDevices] = {};   // context current when the address was taken

typedef CUresult (*CtxGetCurrentFn)(CUcontext*);

// The driver's cuCtxGetCurrent, found through the runtime (the library links
// no driver stub); nullptr when the driver does not provide it.
CtxGetCurrentFn ctx_get_current_fn() {
  static CtxGetCurrentFn fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuCtxGetCurrent", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<CtxGetCurrentFn>(p);
  });
  return fn;
}

// Device address of g_static_scratch on `device`, which must be current.  The
// address is cached with the context it was taken in and taken again when
// another context is current (a reset device gets a new primary context).
vsa_status static_scratch(int device, void** out) {
  if (device < 0 || device >= kMaxDevices)
    return vsa::fail(VSA_ERR_UNSUPPORTED, "device ordinal beyond the static scratch table");
  CUcontext ctx = nullptr;
  if (CtxGetCurrentFn get = ctx_get_current_fn()) get(&ctx);
  std::lock_guard<std::mutex> lock(g_scratch_mu);
  if (g_scratch_addr[device] == nullptr || g_scratch_ctx[device] != ctx) {
    void* p = nullptr;
    const cudaError_t e = cudaGetSymbolAddress(&p, g_static_scratch);
    if (e != cudaSuccess || p == nullptr)
      return vsa::fail(VSA_ERR_CUDA, std::string("cudaGetSymbolAddress of the static scratch: ") +
                                         cudaGetErrorString(e));
    g_scratch_addr[device] = p;
    g_scratch_ctx[device] = ctx;
  }
  *out = g_scratch_addr[device];
  return VSA_OK;
}

}  // namespace

extern "C" vsa_status vsa_coarse_topk_noalloc(vsa_plan p, const void* q_t, const void* k_t,
                                              const void* v_t, int B, int H, int D, float scale,
                                              int k, float* o_coarse, int32_t* topk_idx,
                                              float* topk_score, void* stream) {
  if (p == nullptr) return vsa::fail(VSA_ERR_INVALID_ARG, "plan is NULL");
  if (p->device < 0)
    return vsa::fail(VSA_ERR_INVALID_ARG, "host-only plan (device = -1) cannot launch");
  int cur = -1;
  const cudaError_t e = cudaGetDevice(&cur);
  if (e != cudaSuccess) return vsa::fail(VSA_ERR_CUDA, cudaGetErrorString(e));
  if (cur != p->device)
    return vsa::fail(VSA_ERR_INVALID_ARG, "current CUDA device differs from the plan's device");
  size_t need = 0;
  const vsa_status st = vsa_workspace_size(p, B, H, D, k, &need);
  if (st != VSA_OK) return st;
  if (need > kStaticScratchBytes)
    return vsa::fail(VSA_ERR_WORKSPACE,
                     "vsa_coarse_topk_noalloc needs " + std::to_string(need) +
                         " bytes of scratch (3*B*H*T*D*4); its static scratch holds " +
                         std::to_string(kStaticScratchBytes) + " bytes");
  void* scratch = nullptr;
  const vsa_status s2 = static_scratch(p->device, &scratch);
  if (s2 != VSA_OK) return s2;
  return vsa_coarse_topk(p, q_t, k_t, v_t, B, H, D, scale, k, o_coarse, topk_idx, topk_score,
                         scratch, kStaticScratchBytes, stream);
}

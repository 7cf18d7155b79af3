// ivc_noalloc.cu — ivc_ps_project without a caller-provided workspace.
//
// Some callers cannot call cudaMalloc at the point where they run the
// connector: for example a plugin inside an inference engine whose device
// memory is planned ahead and which must not allocate while it enqueues
// work, or a latency-critical loop that cannot afford the device-wide
// synchronisation an allocation may cause. For them this file keeps the
// scratch memory that ivc_ps_project needs (row statistics and the MLP's
// hidden activations) in one file-scope device array of fixed size,
// IVC_NOALLOC_SCRATCH_BYTES. Every GPU that loads the library holds that
// array until the process exits.
//
// In host code `g_noalloc_scratch` only names a host-side stand-in for the
// array, not its device address: the address is obtained once per device,
// with that device current, through cudaGetSymbolAddress and then passed to
// the kernels like any workspace pointer.
#include <cuda.h>
#include <cuda_runtime.h>

#include <mutex>

#include "ivc.h"

static __device__ __align__(256) unsigned char g_noalloc_scratch[IVC_NOALLOC_SCRATCH_BYTES];

namespace {

constexpr int kMaxDevices = 64;

typedef CUresult (*CtxGetCurrentFn)(CUcontext*);

// The driver's current context (nullptr if it cannot be queried).
CUcontext current_context() {
  static CtxGetCurrentFn fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPointByVersion("cuCtxGetCurrent", &p, 12000, cudaEnableDefault, &q) ==
            cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<CtxGetCurrentFn>(p);
  });
  CUcontext c = nullptr;
  if (fn == nullptr || fn(&c) != CUDA_SUCCESS) return nullptr;
  return c;
}

// Device address of g_noalloc_scratch on `dev` (the current device), looked
// up on the first call for that device and again whenever the device's
// current context has changed since (after cudaDeviceReset the array lives in
// a new context, at an address that may differ). Returns nullptr on failure.
void* scratch_address(int dev) {
  static std::mutex mu;
  static void* addr[kMaxDevices] = {};
  static CUcontext ctx_of[kMaxDevices] = {};
  if (dev < 0 || dev >= kMaxDevices) return nullptr;
  const CUcontext ctx = current_context();
  std::lock_guard<std::mutex> lock(mu);
  if (addr[dev] == nullptr || ctx == nullptr || ctx != ctx_of[dev]) {
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_noalloc_scratch) != cudaSuccess) return nullptr;
    addr[dev] = p;
    ctx_of[dev] = ctx;
  }
  return addr[dev];
}

}  // namespace

extern "C" int ivc_ps_project_noalloc(const void* x, int T, int C, float scale, int flags,
                                      const ivc_mlp* m, void* y, ivc_stream_t stream) {
  if (!m || T < 0) return IVC_EINVAL;
  // The LayerNorm fold must already be in the caller's memory (ivc_mlp_fold),
  // so that the only scratch left is the statistics and hidden activations.
  if (!m->fold_colsum || !m->fold_W0 || !m->fold_bias) return IVC_EINVAL;
  const int op = scale == 0.5f ? IVC_OP_PS_PROJECT_HALF : IVC_OP_PS_PROJECT_QUARTER;
  if (scale != 0.5f && scale != 0.25f) return IVC_EINVAL;
  const size_t need = ivc_workspace_size(op, T, C, m, nullptr, nullptr);
  if (need == 0) return IVC_EUNSUPPORTED;
  if (need > IVC_NOALLOC_SCRATCH_BYTES) return IVC_EWORKSPACE;
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return IVC_ECUDA;
  void* ws = scratch_address(dev);
  if (ws == nullptr) return IVC_ECUDA;
  // The array keeps the previous call's contents: the status word at its start
  // must begin each call at zero. Nothing else in the scratch is read before
  // this call writes it.
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  if (T > 0 && cudaMemsetAsync(ws, 0, sizeof(int), s) != cudaSuccess) return IVC_ECUDA;
  return ivc_ps_project(x, T, C, scale, flags, m, y, ws, IVC_NOALLOC_SCRATCH_BYTES, stream);
}

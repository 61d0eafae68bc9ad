// Step entry point for callers that cannot allocate device memory themselves.
//
// dion_step_batched takes a caller-allocated workspace.  Some callers have no way
// to get one: a plug-in or extension handed only the model's buffers by a host
// program whose allocator it cannot reach, or a training loop whose device memory is
// sized once at start-up and that must not allocate afterwards.  For them,
// dion_step_batched_noalloc runs the same step with its scratch taken from a fixed
// array in device memory that is part of this library (DION_STATIC_SCRATCH_BYTES per
// GPU, held from the moment the library's module is loaded on a GPU until the process
// exits).
#include <cuda.h>
#include <cuda_runtime.h>

#include <mutex>

#include "../../include/dion.h"
#include "internal.h"

namespace {

__device__ __align__(256) unsigned char g_scratch[DION_STATIC_SCRATCH_BYTES];

constexpr int kMaxDevices = 64;

// Per device: the device address of g_scratch and the context it was looked up in.
// A context has a process-unique id (cuCtxGetId), so a context created after a reset
// never matches the cached one even if the driver reuses the handle's value.
struct ScratchAddr {
  void* ptr;
  unsigned long long ctx_id;
};
ScratchAddr g_scratch_addr[kMaxDevices] = {};
std::mutex g_scratch_mu;

using PfnCtxGetCurrent = CUresult (*)(CUcontext*);
using PfnCtxGetId = CUresult (*)(CUcontext, unsigned long long*);

struct CtxFns {
  PfnCtxGetCurrent get_current = nullptr;
  PfnCtxGetId get_id = nullptr;
};

const CtxFns& ctx_fns() {
  static const CtxFns fns = [] {
    CtxFns f;
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuCtxGetCurrent", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      f.get_current = reinterpret_cast<PfnCtxGetCurrent>(p);
    p = nullptr;
    if (cudaGetDriverEntryPoint("cuCtxGetId", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      f.get_id = reinterpret_cast<PfnCtxGetId>(p);
    return f;
  }();
  return fns;
}

// Id of the context current on this thread; 0 when none is current (yet).
dion_status current_ctx_id(unsigned long long* id) {
  const CtxFns& f = ctx_fns();
  if (!f.get_current || !f.get_id)
    return dion::set_error(DION_ERR_CUDA, "cuCtxGetCurrent / cuCtxGetId unavailable");
  CUcontext ctx = nullptr;
  if (f.get_current(&ctx) != CUDA_SUCCESS)
    return dion::set_error(DION_ERR_CUDA, "cuCtxGetCurrent failed");
  *id = 0;
  if (ctx && f.get_id(ctx, id) != CUDA_SUCCESS)
    return dion::set_error(DION_ERR_CUDA, "cuCtxGetId failed");
  return DION_OK;
}

// Device address of g_scratch in the current device's context, looked up on the first
// call on a device and again whenever that device's context has changed.  (In host
// code g_scratch names a host-side shadow, never the device array.)
dion_status scratch_for_current_device(void** out) {
  int dev = -1;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess)
    return dion::set_error(DION_ERR_CUDA, "cudaGetDevice: %s", cudaGetErrorString(e));
  if (dev < 0 || dev >= kMaxDevices)
    return dion::set_error(DION_ERR_DEVICE, "device %d out of range", dev);
  unsigned long long id = 0;
  dion_status st = current_ctx_id(&id);
  if (st != DION_OK) return st;
  std::lock_guard<std::mutex> lock(g_scratch_mu);
  ScratchAddr& a = g_scratch_addr[dev];
  if (!a.ptr || id == 0 || a.ctx_id != id) {
    void* p = nullptr;
    e = cudaGetSymbolAddress(&p, g_scratch);  // makes the device's context current if needed
    if (e != cudaSuccess || p == nullptr)
      return dion::set_error(DION_ERR_CUDA, "cudaGetSymbolAddress(static scratch): %s",
                             cudaGetErrorString(e));
    if (id == 0 && (st = current_ctx_id(&id)) != DION_OK) return st;
    a.ptr = p;
    a.ctx_id = id;
  }
  *out = a.ptr;
  return DION_OK;
}

}  // namespace

static dion_status noalloc_impl(dion_handle h, const dion_bucket_ptrs* ptrs, int32_t nbuckets,
                                float lr, int32_t* d_status, void* stream) {
  size_t need = 0;
  dion_status st = dion::plan_workspace_bytes(h, &need);
  if (st != DION_OK) return st;
  if (need > (size_t)DION_STATIC_SCRATCH_BYTES)
    return dion::set_error(DION_ERR_WORKSPACE_TOO_SMALL,
                           "this plan needs %zu bytes of scratch; the built-in scratch holds %zu "
                           "(use dion_step_batched with a caller workspace)",
                           need, (size_t)DION_STATIC_SCRATCH_BYTES);
  void* scratch = nullptr;
  st = scratch_for_current_device(&scratch);
  if (st != DION_OK) return st;
  return dion_step_batched(h, ptrs, nbuckets, lr, scratch, DION_STATIC_SCRATCH_BYTES, d_status,
                           stream);
}

extern "C" dion_status dion_step_batched_noalloc(dion_handle h, const dion_bucket_ptrs* ptrs,
                                                 int32_t nbuckets, float lr, int32_t* d_status,
                                                 void* stream) {
  try {  // no C++ exception leaves the library (the lock can throw)
    return noalloc_impl(h, ptrs, nbuckets, lr, d_status, stream);
  } catch (...) {
    return dion::set_error(DION_ERR_HOST, "dion_step_batched_noalloc: host-side failure");
  }
}

// Step entry point for callers that cannot allocate device memory themselves.
//
// dion_step_batched takes a caller-allocated workspace.  Some callers have no way
// to get one: code that runs while a stream is being captured into a CUDA graph
// (cudaMalloc is not allowed then), plug-ins that receive only the model's buffers
// from a host program whose allocator they cannot reach, or loops that forbid any
// allocation after start-up.  For them, dion_step_batched_noalloc runs the same
// step with its scratch taken from a fixed array in device memory that is part of
// this library (DION_STATIC_SCRATCH_BYTES per GPU, held from the moment the library
// first touches a GPU until the process exits).
#include <cuda_runtime.h>

#include <mutex>

#include "../../include/dion.h"
#include "internal.h"

namespace {

__device__ __align__(256) unsigned char g_scratch[DION_STATIC_SCRATCH_BYTES];

constexpr int kMaxDevices = 64;
void* g_scratch_ptr[kMaxDevices] = {};
std::mutex g_scratch_mu;

// Device address of g_scratch on the current device, looked up once per device.
// (In host code g_scratch names a host-side shadow, never the device array.)
dion_status scratch_for_current_device(void** out) {
  int dev = -1;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess)
    return dion::set_error(DION_ERR_CUDA, "cudaGetDevice: %s", cudaGetErrorString(e));
  if (dev < 0 || dev >= kMaxDevices)
    return dion::set_error(DION_ERR_DEVICE, "device %d out of range", dev);
  std::lock_guard<std::mutex> lock(g_scratch_mu);
  if (!g_scratch_ptr[dev]) {
    void* p = nullptr;
    e = cudaGetSymbolAddress(&p, g_scratch);
    if (e != cudaSuccess || p == nullptr)
      return dion::set_error(DION_ERR_CUDA, "cudaGetSymbolAddress(static scratch): %s",
                             cudaGetErrorString(e));
    g_scratch_ptr[dev] = p;
  }
  *out = g_scratch_ptr[dev];
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

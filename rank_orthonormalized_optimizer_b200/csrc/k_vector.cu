// The step of the vector (1-D) parameters: AdamW or Lion over a list of fp32 tensors.
//
// Dion takes only the 2-D weight matrices; biases and normalisation gains go to AdamW
// or Lion (rivista.ai, "Dion e la fine del monopolio di Adam negli optimizer AI
// distribuiti", paragraph 5).  The article does not write the two rules down; they are
// taken as published: AdamW from "Decoupled Weight Decay Regularization" (Loshchilov and
// Hutter; decay first, then the bias-corrected Adam step) and Lion from "Symbolic
// Discovery of Optimization Algorithms" (Chen et al.; the sign of b1 m + (1 - b1) g).
//
// The work is a stream over HBM with no reuse: AdamW reads x, g, m, v and writes x, m,
// v (28 bytes per element), Lion reads x, g, m and writes x, m (20 bytes).  Every
// tensor is cut into chunks of kChunk elements; one launch covers up to kPerLaunch
// tensors whose pointers and chunk offsets travel in the kernel's parameters, and a
// grid of a few CTAs per SM walks the chunks (chunk c, c + grid, ...).  A chunk whose
// four arrays are 16-byte aligned at its start moves float4s, four per thread in flight
// per array; others go element by element.
#include <cuda_runtime.h>

#include <cmath>
#include <cstdint>

#include "../../include/dion.h"
#include "internal.h"

namespace {

constexpr int kPerLaunch = 128;  // 7.2 KB of kernel parameters (sm_70+ takes up to 32 KB)
constexpr int kChunk = 8192;  // elements per work item (a multiple of 4 * kThreads)
constexpr int kThreads = 256;
constexpr int kCtasPerSm = 8;

struct VecT {
  float* x;
  const float* g;
  float* m;
  float* v;
  int64_t numel;
  int64_t chunk0;  // first chunk of this tensor in the launch
  int vec4;        // x, g, m (and v) 16-byte aligned
};

struct VecLaunch {
  VecT t[kPerLaunch];
  int n;
  int rule;
  int64_t chunks;
  float b1, b2, omb1, omb2;  // betas and 1 - beta, each rounded to fp32
  float decay;               // 1 - lr wd
  float lr;
  float step_size;           // AdamW: lr / (1 - b1^t)
  float inv_sqrt_bc2;        // AdamW: 1 / sqrt(1 - b2^t)
  float eps;
};

thread_local int32_t tl_vec_launches = 0;

__device__ __forceinline__ void adamw1(const VecLaunch& L, float& x, float g, float& m, float& v) {
  x *= L.decay;
  m = fmaf(L.b1, m, L.omb1 * g);
  v = fmaf(L.b2, v, L.omb2 * g * g);
  const float den = fmaf(sqrtf(v), L.inv_sqrt_bc2, L.eps);
  x = fmaf(-L.step_size, m / den, x);
}

__device__ __forceinline__ void lion1(const VecLaunch& L, float& x, float g, float& m) {
  // c = b1 m + (1 - b1) g with every product and the sum rounded (no contraction)
  const float c = __fadd_rn(__fmul_rn(L.b1, m), __fmul_rn(L.omb1, g));
  const float s = isnan(c) ? c : (float)((c > 0.f) - (c < 0.f));
  x = fmaf(-L.lr, s, x * L.decay);
  m = fmaf(L.b2, m, L.omb2 * g);
}

__device__ __forceinline__ void step1(const VecLaunch& L, const VecT& T, int64_t i) {
  float x = T.x[i], m = T.m[i];
  const float g = T.g[i];
  if (L.rule == DION_VEC_ADAMW) {
    float v = T.v[i];
    adamw1(L, x, g, m, v);
    T.v[i] = v;
  } else {
    lion1(L, x, g, m);
  }
  T.x[i] = x;
  T.m[i] = m;
}

template <int RULE>
__device__ __forceinline__ void chunk4(const VecLaunch& L, const VecT& T, int64_t e0, int64_t n4) {
  const float4* __restrict__ g4 = reinterpret_cast<const float4*>(T.g + e0);
  float4* __restrict__ x4 = reinterpret_cast<float4*>(T.x + e0);
  float4* __restrict__ m4 = reinterpret_cast<float4*>(T.m + e0);
  float4* __restrict__ v4 = RULE == DION_VEC_ADAMW ? reinterpret_cast<float4*>(T.v + e0) : nullptr;
  constexpr int U = 4;  // float4s of each array in flight per thread
  for (int64_t base = threadIdx.x; base < n4; base += (int64_t)U * kThreads) {
    float4 x[U], g[U], m[U], v[U];
#pragma unroll
    for (int u = 0; u < U; ++u) {
      const int64_t i = base + (int64_t)u * kThreads;
      if (i < n4) {
        x[u] = x4[i];
        g[u] = g4[i];
        m[u] = m4[i];
        if (RULE == DION_VEC_ADAMW) v[u] = v4[i];
      }
    }
#pragma unroll
    for (int u = 0; u < U; ++u) {
      const int64_t i = base + (int64_t)u * kThreads;
      if (i >= n4) continue;
      float* xs = &x[u].x;
      float* ms = &m[u].x;
      float* vs = &v[u].x;
      const float* gs = &g[u].x;
#pragma unroll
      for (int q = 0; q < 4; ++q) {
        if (RULE == DION_VEC_ADAMW) adamw1(L, xs[q], gs[q], ms[q], vs[q]);
        else lion1(L, xs[q], gs[q], ms[q]);
      }
      x4[i] = x[u];
      m4[i] = m[u];
      if (RULE == DION_VEC_ADAMW) v4[i] = v[u];
    }
  }
}

__global__ void __launch_bounds__(kThreads) k_vec_step(const __grid_constant__ VecLaunch L) {
  for (int64_t c = blockIdx.x; c < L.chunks; c += gridDim.x) {
    // the tensor owning chunk c: the last one whose first chunk is <= c
    int lo = 0, hi = L.n - 1;
    while (lo < hi) {
      const int mid = (lo + hi + 1) >> 1;
      if (L.t[mid].chunk0 <= c) lo = mid;
      else hi = mid - 1;
    }
    const VecT& T = L.t[lo];
    const int64_t e0 = (c - T.chunk0) * kChunk;
    const int64_t e1 = min(T.numel, e0 + (int64_t)kChunk);
    int64_t done = e0;
    if (T.vec4) {
      const int64_t n4 = (e1 - e0) / 4;
      if (L.rule == DION_VEC_ADAMW) chunk4<DION_VEC_ADAMW>(L, T, e0, n4);
      else chunk4<DION_VEC_LION>(L, T, e0, n4);
      done = e0 + 4 * n4;
    }
    for (int64_t i = done + threadIdx.x; i < e1; i += kThreads) step1(L, T, i);
  }
}

bool aligned4(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 3u) == 0; }
bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

dion_status check_options(const dion_vec_options* o) {
  if (!o) return dion::set_error(DION_ERR_INVALID_ARG, "options are NULL");
  if (o->rule != DION_VEC_ADAMW && o->rule != DION_VEC_LION)
    return dion::set_error(DION_ERR_INVALID_ARG, "rule %d is neither AdamW (0) nor Lion (1)",
                           o->rule);
  if (!std::isfinite(o->lr)) return dion::set_error(DION_ERR_INVALID_ARG, "lr is not finite");
  if (!(o->beta1 >= 0.f && o->beta1 < 1.f) || !(o->beta2 >= 0.f && o->beta2 < 1.f))
    return dion::set_error(DION_ERR_INVALID_ARG, "betas must lie in [0, 1)");
  if (!(o->weight_decay >= 0.f) || !std::isfinite(o->weight_decay))
    return dion::set_error(DION_ERR_INVALID_ARG, "weight_decay must be finite and >= 0");
  if (o->rule == DION_VEC_ADAMW) {
    if (!(o->eps > 0.f) || !std::isfinite(o->eps))
      return dion::set_error(DION_ERR_INVALID_ARG, "eps must be finite and > 0");
    if (o->step < 1) return dion::set_error(DION_ERR_INVALID_ARG, "step must be >= 1");
  }
  return DION_OK;
}

dion_status check_tensor(const dion_vec_tensor& t, int i, int rule) {
  if (t.numel < 0) return dion::set_error(DION_ERR_INVALID_ARG, "tensor %d: numel < 0", i);
  if (t.numel == 0) return DION_OK;
  if (!t.x || !t.g || !t.m || (rule == DION_VEC_ADAMW && !t.v))
    return dion::set_error(DION_ERR_INVALID_ARG, "tensor %d: a NULL pointer", i);
  if (!aligned4(t.x) || !aligned4(t.g) || !aligned4(t.m) ||
      (rule == DION_VEC_ADAMW && !aligned4(t.v)))
    return dion::set_error(DION_ERR_MISALIGNED, "tensor %d: pointers must be 4-byte aligned", i);
  if (t.numel > (INT64_MAX / 2) / kChunk * kChunk)
    return dion::set_error(DION_ERR_INVALID_ARG, "tensor %d: numel too large", i);
  return DION_OK;
}

dion_status check_device_sm100(int* sms) {
  int dev = -1;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess)
    return dion::set_error(DION_ERR_CUDA, "cudaGetDevice: %s", cudaGetErrorString(e));
  int major = 0, minor = 0;
  cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev);
  cudaDeviceGetAttribute(&minor, cudaDevAttrComputeCapabilityMinor, dev);
  if (major != 10 || minor != 0)
    return dion::set_error(DION_ERR_DEVICE,
                           "device %d is sm_%d%d; this library is built for sm_100a (B200)", dev,
                           major, minor);
  *sms = 0;
  cudaDeviceGetAttribute(sms, cudaDevAttrMultiProcessorCount, dev);
  if (*sms <= 0) *sms = 148;
  return DION_OK;
}

void fill_scalars(VecLaunch& L, const dion_vec_options& o) {
  L.rule = o.rule;
  L.b1 = o.beta1;
  L.b2 = o.beta2;
  L.omb1 = 1.0f - o.beta1;
  L.omb2 = 1.0f - o.beta2;
  L.decay = (float)(1.0 - (double)o.lr * (double)o.weight_decay);
  L.lr = o.lr;
  L.eps = o.eps;
  if (o.rule == DION_VEC_ADAMW) {
    const double t = (double)o.step;
    const double bc1 = 1.0 - std::pow((double)o.beta1, t);
    const double bc2 = 1.0 - std::pow((double)o.beta2, t);
    L.step_size = (float)((double)o.lr / bc1);
    L.inv_sqrt_bc2 = (float)(1.0 / std::sqrt(bc2));
  } else {
    L.step_size = 0.f;
    L.inv_sqrt_bc2 = 0.f;
  }
}

dion_status vec_step_impl(const dion_vec_tensor* tensors, int32_t ntensors,
                          const dion_vec_options* o, void* stream) {
  tl_vec_launches = 0;
  dion_status st = check_options(o);
  if (st != DION_OK) return st;
  if (ntensors < 0) return dion::set_error(DION_ERR_INVALID_ARG, "ntensors < 0");
  if (ntensors > 0 && !tensors) return dion::set_error(DION_ERR_INVALID_ARG, "tensors is NULL");
  for (int32_t i = 0; i < ntensors; ++i)
    if ((st = check_tensor(tensors[i], i, o->rule)) != DION_OK) return st;
  int sms = 0;
  if ((st = check_device_sm100(&sms)) != DION_OK) return st;
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  VecLaunch L;
  fill_scalars(L, *o);
  int32_t i = 0;
  while (i < ntensors) {
    L.n = 0;
    L.chunks = 0;
    for (; i < ntensors && L.n < kPerLaunch; ++i) {
      const dion_vec_tensor& t = tensors[i];
      if (t.numel == 0) continue;
      VecT& T = L.t[L.n++];
      T.x = t.x;
      T.g = t.g;
      T.m = t.m;
      T.v = o->rule == DION_VEC_ADAMW ? t.v : nullptr;
      T.numel = t.numel;
      T.chunk0 = L.chunks;
      T.vec4 = aligned16(t.x) && aligned16(t.g) && aligned16(t.m) &&
               (o->rule != DION_VEC_ADAMW || aligned16(t.v));
      L.chunks += (t.numel + kChunk - 1) / kChunk;
    }
    if (L.n == 0) break;
    const int64_t cap = (int64_t)sms * kCtasPerSm;
    const unsigned grid = (unsigned)(L.chunks < cap ? L.chunks : cap);
    k_vec_step<<<grid, kThreads, 0, s>>>(L);
    cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess)
      return dion::set_error(DION_ERR_CUDA, "k_vec_step: %s", cudaGetErrorString(e));
    ++tl_vec_launches;
  }
  return DION_OK;
}

}  // namespace

extern "C" {

dion_status dion_vec_default_options(int32_t rule, dion_vec_options* o) {
  if (!o) return dion::set_error(DION_ERR_INVALID_ARG, "options are NULL");
  if (rule == DION_VEC_ADAMW) {
    *o = dion_vec_options{DION_VEC_ADAMW, 1e-3f, 0.9f, 0.999f, 1e-8f, 0.01f, 1};
  } else if (rule == DION_VEC_LION) {
    *o = dion_vec_options{DION_VEC_LION, 1e-4f, 0.9f, 0.99f, 0.f, 0.f, 1};
  } else {
    return dion::set_error(DION_ERR_INVALID_ARG, "rule %d is neither AdamW (0) nor Lion (1)",
                           rule);
  }
  return DION_OK;
}

dion_status dion_vec_step(const dion_vec_tensor* tensors, int32_t ntensors,
                          const dion_vec_options* o, void* stream) {
  return vec_step_impl(tensors, ntensors, o, stream);
}

int32_t dion_vec_last_launch_count(void) { return tl_vec_launches; }

}  // extern "C"

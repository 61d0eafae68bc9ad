// Device helpers shared by the kernels of the batched Dion step (sm_100a).
#pragma once

#include <cuda_runtime.h>
#include <cuda_bf16.h>
#include <stdint.h>

#include "../../include/dion.h"

namespace dion {

// Per-matrix flag bits kept in the workspace during a step; they are the
// public DION_MAT_* bits, copied to the caller's status array at the end.
constexpr int32_t F_FALLBACK = DION_MAT_FALLBACK;
constexpr int32_t F_CHOLQR2 = DION_MAT_CHOLQR2;
constexpr int32_t F_NONFINITE = DION_MAT_NONFINITE;
constexpr int32_t F_TIMEOUT = DION_MAT_TIMEOUT;
constexpr int32_t F_ZERO_COL = DION_MAT_ZERO_COLUMN;
constexpr int32_t F_PUBLIC = 0xFFFF;  // bits reported to the caller
// Internal bits of the shifted Cholesky-QR iteration that replaces Householder QR for
// flagged matrices when r > 256 (never reported):
constexpr int32_t F_SMORE = 1 << 16;    // this iterate is not orthonormal yet
constexpr int32_t F_SDONE = 1 << 17;    // the iterate in P is the final P
constexpr int32_t F_SFAIL = 1 << 18;    // a factorisation failed: Householder QR takes over
constexpr int32_t F_SITER = 1 << 19;    // P holds an iterate (P0 R^-1, R upper triangular)
constexpr int32_t F_SNOSHIFT = 1 << 20; // well conditioned now: no shift from here on
// Per-matrix statistics of the factorisation, ST floats each: min and max of diag(L),
// the largest diagonal entry of the Gram (shifted iteration), the shift last added.
constexpr int ST = 4;

typedef __nv_bfloat16 bf16;

template <typename T> struct Cvt;
template <> struct Cvt<float> {
  static __device__ __forceinline__ float load(const float* p) { return *p; }
  static __device__ __forceinline__ float to_f(float v) { return v; }
  static __device__ __forceinline__ float from_f(float v) { return v; }
};
template <> struct Cvt<bf16> {
  static __device__ __forceinline__ float load(const bf16* p) { return __bfloat162float(*p); }
  static __device__ __forceinline__ float to_f(bf16 v) { return __bfloat162float(v); }
  static __device__ __forceinline__ bf16 from_f(float v) { return __float2bfloat16_rn(v); }
};

__device__ __forceinline__ bool finitef(float v) { return isfinite(v); }

// x = h + m + l with h, m, l bf16: each part is the bf16 rounding of what the
// earlier parts left over, so h + m + l carries about 24 significant bits of x.
__device__ __forceinline__ void split3_bf16(float v, bf16& h, bf16& m, bf16& l) {
  h = __float2bfloat16_rn(v);
  const float r1 = v - __bfloat162float(h);
  m = __float2bfloat16_rn(r1);
  l = __float2bfloat16_rn(r1 - __bfloat162float(m));
}

// Positive floats order like their bit patterns; used for atomic min/max.
__device__ __forceinline__ void atomic_max_pos(float* a, float v) {
  atomicMax(reinterpret_cast<int*>(a), __float_as_int(v));
}
__device__ __forceinline__ void atomic_min_pos(float* a, float v) {
  atomicMin(reinterpret_cast<int*>(a), __float_as_int(v));
}

template <int NT>
__device__ __forceinline__ float block_sum(float v, float* red) {
  for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  const int w = threadIdx.x >> 5, l = threadIdx.x & 31;
  __syncthreads();
  if (l == 0) red[w] = v;
  __syncthreads();
  float t = 0.f;
  if (threadIdx.x < 32) {
    t = (l < NT / 32) ? red[l] : 0.f;
    for (int o = 16; o > 0; o >>= 1) t += __shfl_xor_sync(0xffffffffu, t, o);
    if (l == 0) red[0] = t;
  }
  __syncthreads();
  return red[0];
}

template <int NT>
__device__ __forceinline__ float block_max(float v, float* red) {
  for (int o = 16; o > 0; o >>= 1) v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, o));
  const int w = threadIdx.x >> 5, l = threadIdx.x & 31;
  __syncthreads();
  if (l == 0) red[w] = v;
  __syncthreads();
  if (threadIdx.x < 32) {
    float t = (l < NT / 32) ? red[l] : -INFINITY;
    for (int o = 16; o > 0; o >>= 1) t = fmaxf(t, __shfl_xor_sync(0xffffffffu, t, o));
    if (l == 0) red[0] = t;
  }
  __syncthreads();
  return red[0];
}

}  // namespace dion

// Streaming and layout kernels of the batched Dion step: B = M + G in GEMM
// precision, the previous Q in GEMM layout, the final P and its GEMM copy,
// Q = colnorm(R) with the update operands, and the per-matrix status words.
#include "common.cuh"
#include "internal.h"

namespace dion {

// SM count of the first device asked (the library runs on B200s only); initialised once,
// thread-safely, by the static local's initialiser
static int sm_count() {
  static const int sms = [] {
    int dev = 0, n = 0;
    cudaGetDevice(&dev);
    cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev);
    return n > 0 ? n : 148;
  }();
  return sms;
}

// ---------------------------------------------------------------- B = M + G
// Step 1 of the Dion step (error-feedback buffer plus this step's gradient),
// written once in the precision the contractions read.  Pure HBM stream:
// 8 bytes read and 2 (bf16) or 4 (fp32) bytes written per element.
template <bool BF16, int U>
__global__ void __launch_bounds__(256) k_form_b(const float4* __restrict__ M,
                                                 const float4* __restrict__ G,
                                                 void* __restrict__ B, int64_t n4) {
  const int64_t stride = (int64_t)gridDim.x * blockDim.x;
  for (int64_t base = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; base < n4;
       base += stride * U) {
    float4 a[U], g[U];
#pragma unroll
    for (int u = 0; u < U; ++u) {
      const int64_t i = base + u * stride;
      if (i < n4) {
        a[u] = __ldcs(M + i);
        g[u] = __ldcs(G + i);
      }
    }
#pragma unroll
    for (int u = 0; u < U; ++u) {
      const int64_t i = base + u * stride;
      if (i < n4) {
        float4 c = make_float4(a[u].x + g[u].x, a[u].y + g[u].y, a[u].z + g[u].z,
                               a[u].w + g[u].w);
        if (BF16) {
          __nv_bfloat162 lo = __floats2bfloat162_rn(c.x, c.y);
          __nv_bfloat162 hi = __floats2bfloat162_rn(c.z, c.w);
          uint2 pk;
          pk.x = *reinterpret_cast<uint32_t*>(&lo);
          pk.y = *reinterpret_cast<uint32_t*>(&hi);
          reinterpret_cast<uint2*>(B)[i] = pk;
        } else {
          reinterpret_cast<float4*>(B)[i] = c;
        }
      }
    }
  }
}

// B = M + G kept to fp32 accuracy as three bf16 parts [3][elems] (for the fp32
// contractions on bf16 tensor cores): 8 bytes read, 6 written per element.
__global__ void __launch_bounds__(256) k_form_b_split(const float4* __restrict__ M,
                                                       const float4* __restrict__ G,
                                                       bf16* __restrict__ Bs, int64_t n4,
                                                       int64_t stride) {
  const int64_t step = (int64_t)gridDim.x * blockDim.x;
  for (int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; i < n4; i += step) {
    const float4 a = __ldcs(M + i), g = __ldcs(G + i);
    const float v[4] = {a.x + g.x, a.y + g.y, a.z + g.z, a.w + g.w};
    __align__(8) bf16 h[4], m[4], l[4];
#pragma unroll
    for (int q = 0; q < 4; ++q) split3_bf16(v[q], h[q], m[q], l[q]);
    reinterpret_cast<uint2*>(Bs)[i] = *reinterpret_cast<const uint2*>(h);
    reinterpret_cast<uint2*>(Bs + stride)[i] = *reinterpret_cast<const uint2*>(m);
    reinterpret_cast<uint2*>(Bs + 2 * stride)[i] = *reinterpret_cast<const uint2*>(l);
  }
}

cudaError_t launch_form_b_split(const float* M, const float* G, void* Bs, int64_t elems,
                                cudaStream_t s) {
  const int64_t n4 = elems / 4;
  int64_t grid = (n4 + 255) / 256;
  if (grid > (int64_t)sm_count() * 8) grid = (int64_t)sm_count() * 8;
  if (grid < 1) grid = 1;
  k_form_b_split<<<(unsigned)grid, 256, 0, s>>>((const float4*)M, (const float4*)G, (bf16*)Bs, n4,
                                                elems);
  return cudaGetLastError();
}

cudaError_t launch_form_b(const float* M, const float* G, void* Bg, bool use_bf16, int64_t elems,
                          cudaStream_t s) {
  const int64_t n4 = elems / 4;
  int64_t want = (n4 + 255) / 256;
  int64_t grid = (int64_t)sm_count() * 4;
  if (want < grid) grid = want < 1 ? 1 : want;
  if (use_bf16)
    k_form_b<true, 4><<<(unsigned)grid, 256, 0, s>>>((const float4*)M, (const float4*)G, Bg, n4);
  else
    k_form_b<false, 4><<<(unsigned)grid, 256, 0, s>>>((const float4*)M, (const float4*)G, Bg, n4);
  return cudaGetLastError();
}

// ------------------------------------------------- previous Q into GEMM layout
// Qg[b][j][i] = Q[b][i][j]: the n x r factor transposed to r x n so that the
// contraction B Q reads both operands along n (the reduction axis).  64 x 64 tiles:
// float4 loads along r, 4-element stores along n.
template <typename T, bool SPLIT>
__global__ void __launch_bounds__(256) k_prep_q(const float* __restrict__ Q, T* __restrict__ Qg,
                                                 int64_t n, int64_t r, int64_t split_stride) {
  __shared__ float tile[64][65];
  const int64_t b = blockIdx.z;
  const float* q = Q + b * n * r;
  T* qg = Qg + b * n * r;
  const int64_t j0 = (int64_t)blockIdx.x * 64, i0 = (int64_t)blockIdx.y * 64;
  const int tid = threadIdx.x;
  for (int e = tid; e < 64 * 16; e += 256) {       // 64 rows (i) x 16 float4 (j)
    const int y = e / 16, x4 = e % 16;
    const int64_t i = i0 + y, j = j0 + 4 * x4;
    float4 v = make_float4(0.f, 0.f, 0.f, 0.f);
    if (i < n && j < r) v = *reinterpret_cast<const float4*>(q + i * r + j);  // r % 16 == 0
    tile[4 * x4 + 0][y] = v.x;
    tile[4 * x4 + 1][y] = v.y;
    tile[4 * x4 + 2][y] = v.z;
    tile[4 * x4 + 3][y] = v.w;
  }
  __syncthreads();
  for (int e = tid; e < 64 * 16; e += 256) {       // 64 rows (j) x 16 groups of 4 (i)
    const int y = e / 16, x4 = e % 16;
    const int64_t j = j0 + y, i = i0 + 4 * x4;
    if (j >= r || i >= n) continue;
    T* dst = qg + j * n + i;
    if (SPLIT) {  // three bf16 parts, each plane [count][r][n]
      for (int q2 = 0; q2 < 4 && i + q2 < n; ++q2) {
        bf16 h, m, l;
        split3_bf16(tile[y][4 * x4 + q2], h, m, l);
        reinterpret_cast<bf16*>(dst)[q2] = h;
        reinterpret_cast<bf16*>(dst)[q2 + split_stride] = m;
        reinterpret_cast<bf16*>(dst)[q2 + 2 * split_stride] = l;
      }
    } else if (i + 3 < n) {
      if (sizeof(T) == 2) {
        __nv_bfloat162 lo = __floats2bfloat162_rn(tile[y][4 * x4], tile[y][4 * x4 + 1]);
        __nv_bfloat162 hi = __floats2bfloat162_rn(tile[y][4 * x4 + 2], tile[y][4 * x4 + 3]);
        uint2 pk;
        pk.x = *reinterpret_cast<uint32_t*>(&lo);
        pk.y = *reinterpret_cast<uint32_t*>(&hi);
        *reinterpret_cast<uint2*>(dst) = pk;  // n % 8 == 0: 8-byte aligned
      } else {
        *reinterpret_cast<float4*>(dst) =
            make_float4(tile[y][4 * x4], tile[y][4 * x4 + 1], tile[y][4 * x4 + 2], tile[y][4 * x4 + 3]);
      }
    } else {
      for (int q2 = 0; q2 < 4 && i + q2 < n; ++q2) dst[q2] = Cvt<T>::from_f(tile[y][4 * x4 + q2]);
    }
  }
}

cudaError_t launch_prep_q(const float* Q, void* Qg, bool use_bf16, int count, int64_t n, int64_t r,
                          cudaStream_t s) {
  dim3 grid((unsigned)((r + 63) / 64), (unsigned)((n + 63) / 64), (unsigned)count);
  if (use_bf16)
    k_prep_q<bf16, false><<<grid, 256, 0, s>>>(Q, (bf16*)Qg, n, r, 0);
  else
    k_prep_q<float, false><<<grid, 256, 0, s>>>(Q, (float*)Qg, n, r, 0);
  return cudaGetLastError();
}

cudaError_t launch_prep_q_split(const float* Q, void* Qs, int count, int64_t n, int64_t r,
                                cudaStream_t s) {
  dim3 grid((unsigned)((r + 63) / 64), (unsigned)((n + 63) / 64), (unsigned)count);
  k_prep_q<bf16, true><<<grid, 256, 0, s>>>(Q, (bf16*)Qs, n, r, (int64_t)count * n * r);
  return cudaGetLastError();
}

// ------------------------------------------------ three-way bf16 split of fp32
// dst[i], dst[i + stride], dst[i + 2 stride] = the bf16 parts of src[i], for the
// split-operand tensor-core contractions of the orthonormalisation.
__global__ void __launch_bounds__(256) k_split3(const float* __restrict__ src,
                                                 bf16* __restrict__ dst, int64_t n,
                                                 int64_t stride) {
  for (int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; i < n;
       i += (int64_t)gridDim.x * blockDim.x) {
    bf16 h, m, l;
    split3_bf16(src[i], h, m, l);
    dst[i] = h;
    dst[i + stride] = m;
    dst[i + 2 * stride] = l;
  }
}

cudaError_t launch_split3(const float* src, void* dst, int64_t n, int64_t dst_stride,
                          cudaStream_t s) {
  int64_t grid = (n + 255) / 256;
  if (grid > (int64_t)sm_count() * 8) grid = (int64_t)sm_count() * 8;
  if (grid < 1) grid = 1;
  k_split3<<<(unsigned)grid, 256, 0, s>>>(src, (bf16*)dst, n, dst_stride);
  return cudaGetLastError();
}

// ---------------------------------------------------------- flags and status
__global__ void k_init_flags(int32_t* flags, float* stats, int* sched, float* rmmc, int count,
                             int32_t init_bits) {
  const int b = blockIdx.x * blockDim.x + threadIdx.x;
  if (b < 16) sched[b] = 0;
  if (b < count) {
    flags[b] = init_bits;
    stats[ST * b] = 3.0e38f;     // running min of diag(L)
    stats[ST * b + 1] = 0.f;     // running max of diag(L)
    stats[ST * b + 2] = 0.f;
    stats[ST * b + 3] = 0.f;
    rmmc[b] = 0.f;               // max |M' - M|, max-ed into by the update
    rmmc[count + b] = 0.f;       // max |M|
  }
}

cudaError_t launch_init_flags(int32_t* flags, float* stats, int* sched, float* rmmc, int count,
                              int32_t init_bits, cudaStream_t s) {
  const int n = count > 16 ? count : 16;
  k_init_flags<<<(n + 255) / 256, 256, 0, s>>>(flags, stats, sched, rmmc, count, init_bits);
  return cudaGetLastError();
}

// CurvaDion's statistic from the update's maxima (the relative maximum momentum change):
// RMMC = max |M' - M| / max |M|, and the gate bit where it exceeds the threshold.
__global__ void k_write_status(const int32_t* flags, float* rmmc, float tau, int32_t* st,
                               int count) {
  const int b = blockIdx.x * blockDim.x + threadIdx.x;
  if (b >= count) return;
  const float num = rmmc[b], den = rmmc[count + b];
  const float v = den > 0.f ? num / den : (num > 0.f ? INFINITY : 0.f);
  rmmc[2 * count + b] = v;
  if (st) st[b] = (flags[b] & F_PUBLIC) | (v > tau ? DION_MAT_HIGH_RMMC : 0);
}

cudaError_t launch_write_status(const int32_t* flags, float* rmmc, float rmmc_threshold,
                                int32_t* d_status, int count, cudaStream_t s) {
  k_write_status<<<(count + 255) / 256, 256, 0, s>>>(flags, rmmc, rmmc_threshold, d_status,
                                                     count);
  return cudaGetLastError();
}

// ------------------------------------------------ row-sharded step: P0 gather
// In a row-sharded step every rank holds rows [row0, row0 + m) of each matrix's P0.
// When a matrix needs the Householder fallback the whole P0 is assembled by summing,
// over ranks, m_full x r buffers that hold only the rank's own rows (zero elsewhere).
// Its rows go into `full` (zeroed beforehand); P0 is read in fp32, or as the sum of its
// three bf16 parts when P0s is not null (planes `plane` elements apart).
__global__ void k_rows_to_full(const float* __restrict__ P0, const bf16* __restrict__ P0s,
                               int64_t plane, float* __restrict__ full, int64_t m,
                               int64_t m_full, int64_t row0, int64_t r) {
  const int64_t b = blockIdx.y;
  const int64_t mr = m * r;
  for (int64_t e = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; e < mr;
       e += (int64_t)gridDim.x * blockDim.x) {
    const int64_t src = b * mr + e;
    const float v = P0s ? (__bfloat162float(P0s[src]) + __bfloat162float(P0s[src + plane])) +
                              __bfloat162float(P0s[src + 2 * plane])
                        : P0[src];
    full[b * m_full * r + row0 * r + e] = v;
  }
}

cudaError_t launch_rows_to_full(const float* P0, const void* P0s, float* full, int count,
                                int64_t m, int64_t m_full, int64_t row0, int64_t r,
                                cudaStream_t s) {
  int64_t gx = (m * r + 255) / 256;
  if (gx > 64) gx = 64;
  k_rows_to_full<<<dim3((unsigned)gx, (unsigned)count), 256, 0, s>>>(
      P0, (const bf16*)P0s, (int64_t)count * m * r, full, m, m_full, row0, r);
  return cudaGetLastError();
}

// P[b] (m x r) = rows [row0, row0 + m) of full[b] (m_full x r), for the matrices
// flagged F_FALLBACK only (the others keep their Cholesky-QR result).
__global__ void k_rows_from_full(const float* __restrict__ full, float* __restrict__ P,
                                 const int32_t* __restrict__ flags, int64_t m,
                                 int64_t m_full, int64_t row0, int64_t r) {
  const int64_t b = blockIdx.y;
  if (!(flags[b] & F_FALLBACK)) return;
  const int64_t mr = m * r;
  for (int64_t e = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; e < mr;
       e += (int64_t)gridDim.x * blockDim.x)
    P[b * mr + e] = full[b * m_full * r + row0 * r + e];
}

cudaError_t launch_rows_from_full(const float* full, float* P, const int32_t* flags, int count,
                                  int64_t m, int64_t m_full, int64_t row0, int64_t r,
                                  cudaStream_t s) {
  int64_t gx = (m * r + 255) / 256;
  if (gx > 64) gx = 64;
  k_rows_from_full<<<dim3((unsigned)gx, (unsigned)count), 256, 0, s>>>(full, P, flags, m,
                                                                        m_full, row0, r);
  return cudaGetLastError();
}

// *out = the number of matrices with (flags & mask) != 0, as a float (one block; the
// count is exact far beyond 65535 matrices).
__global__ void __launch_bounds__(256) k_count_flags(const int32_t* flags, int count,
                                                     int32_t mask, float* out) {
  __shared__ float red[32];
  float c = 0.f;
  for (int b = threadIdx.x; b < count; b += 256) c += (flags[b] & mask) ? 1.f : 0.f;
  c = block_sum<256>(c, red);
  if (threadIdx.x == 0) *out = c;
}

cudaError_t launch_count_flags(const int32_t* flags, int count, int32_t mask, float* out,
                               cudaStream_t s) {
  k_count_flags<<<1, 256, 0, s>>>(flags, count, mask, out);
  return cudaGetLastError();
}

// ------------------------------------------------ fp32 P from its split (inspection)
// The first Cholesky-QR pass on the tensor path writes P only as its three-way bf16
// split x0 + x1 + x2; each part is the rounding of what the earlier ones left, so the
// fp32 sum (x0 + x1) + x2 is the fp32 P exactly.
__global__ void k_p_from_split(float* __restrict__ P, const bf16* __restrict__ Ps, int64_t plane,
                               const int32_t* __restrict__ flags, int64_t mr) {
  const int64_t b = blockIdx.y;
  if (flags[b] & (F_FALLBACK | F_CHOLQR2)) return;  // their fp32 P is the finalize's
  for (int64_t e = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; e < mr;
       e += (int64_t)gridDim.x * blockDim.x) {
    const int64_t i = b * mr + e;
    P[i] = (__bfloat162float(Ps[i]) + __bfloat162float(Ps[i + plane])) +
           __bfloat162float(Ps[i + 2 * plane]);
  }
}

cudaError_t launch_p_from_split(float* P, const void* Ps, int64_t plane, const int32_t* flags,
                                int count, int64_t m, int64_t r, cudaStream_t s) {
  int64_t gx = (m * r + 255) / 256;
  if (gx > 64) gx = 64;
  k_p_from_split<<<dim3((unsigned)gx, (unsigned)count), 256, 0, s>>>(P, (const bf16*)Ps, plane,
                                                                      flags, m * r);
  return cudaGetLastError();
}

// ------------------------------------------------------------- final P
// P holds the first Cholesky-QR pass or the fallback's result; P2 the
// second pass.  Picks per matrix, then writes the GEMM copy Pg (bf16 mode).
// pg_ready: the first pass already wrote Pg, so only matrices that took the second
// pass or the fallback are touched.
// MODE 0: fp32 only; 1: + bf16 copy; 2: + three-way bf16 split (planes of count*m*r)
template <int MODE>
__global__ void k_finalize_p(float* __restrict__ P, const float* __restrict__ P2,
                             void* __restrict__ Pg, const int32_t* __restrict__ flags,
                             int64_t mr4, int64_t plane, int pg_ready) {
  const int64_t b = blockIdx.y;
  const int32_t f = flags[b];
  const bool take2 = (f & F_CHOLQR2) && !(f & F_FALLBACK);
  if (!take2 && MODE == 0) return;
  if (pg_ready && !take2 && !(f & F_FALLBACK)) return;
  float4* p = reinterpret_cast<float4*>(P) + b * mr4;
  const float4* p2 = reinterpret_cast<const float4*>(P2) + b * mr4;
  for (int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; i < mr4;
       i += (int64_t)gridDim.x * blockDim.x) {
    float4 v = take2 ? p2[i] : p[i];
    if (take2) p[i] = v;
    if (MODE == 2) {
      const float vv[4] = {v.x, v.y, v.z, v.w};
      __align__(8) bf16 h[4], m[4], l[4];
#pragma unroll
      for (int q = 0; q < 4; ++q) split3_bf16(vv[q], h[q], m[q], l[q]);
      bf16* o = reinterpret_cast<bf16*>(Pg);
      reinterpret_cast<uint2*>(o)[b * mr4 + i] = *reinterpret_cast<const uint2*>(h);
      reinterpret_cast<uint2*>(o + plane)[b * mr4 + i] = *reinterpret_cast<const uint2*>(m);
      reinterpret_cast<uint2*>(o + 2 * plane)[b * mr4 + i] = *reinterpret_cast<const uint2*>(l);
    } else if (MODE == 1) {
      __nv_bfloat162 lo = __floats2bfloat162_rn(v.x, v.y);
      __nv_bfloat162 hi = __floats2bfloat162_rn(v.z, v.w);
      uint2 pk;
      pk.x = *reinterpret_cast<uint32_t*>(&lo);
      pk.y = *reinterpret_cast<uint32_t*>(&hi);
      reinterpret_cast<uint2*>(Pg)[b * mr4 + i] = pk;
    }
  }
}

cudaError_t launch_finalize_p(const float* P2, void* Pg, int mode, const int32_t* flags,
                              int count, int64_t m, int64_t r, float* P, bool pg_ready,
                              cudaStream_t s) {
  const int64_t mr4 = m * r / 4;
  int64_t gx = (mr4 + 255) / 256;
  if (gx > 64) gx = 64;
  dim3 grid((unsigned)gx, (unsigned)count);
  const int64_t plane = (int64_t)count * m * r;
  if (mode == 2)
    k_finalize_p<2><<<grid, 256, 0, s>>>(P, P2, Pg, flags, mr4, plane, pg_ready ? 1 : 0);
  else if (mode == 1)
    k_finalize_p<1><<<grid, 256, 0, s>>>(P, P2, Pg, flags, mr4, plane, pg_ready ? 1 : 0);
  else
    k_finalize_p<0><<<grid, 256, 0, s>>>(P, P2, Pg, flags, mr4, plane, 0);
  return cudaGetLastError();
}

// ------------------------------------------------------------- Q = colnorm(R)
// Step 6: each column of R (n x r) divided by its 2-norm over the n rows.
// Deterministic two-stage reduction: every block sums the squares of a fixed
// row range in a fixed order, then the per-range sums are added in range order.
// A zero column gives a zero Q column and F_ZERO_COL.
// Vectorised by 4 columns (r % 16 == 0); 256 threads = (256 / (r/4)) row lanes.
__global__ void __launch_bounds__(256) k_colnorm_partial(const float* __restrict__ R,
                                                          float* __restrict__ part, int64_t n,
                                                          int64_t r, int nsplit) {
  extern __shared__ float4 red4[];  // [lanes][r/4]
  const int64_t b = blockIdx.y;
  const int split = blockIdx.x;
  const int vc = (int)(r / 4);
  const int64_t rows = (n + nsplit - 1) / nsplit;
  const int64_t i0 = split * rows, i1 = (i0 + rows < n) ? i0 + rows : n;
  const float4* rb = reinterpret_cast<const float4*>(R + b * n * r);
  const int lanes = vc >= 256 ? 1 : 256 / vc;  // row lanes
  for (int c0 = 0; c0 < vc; c0 += 256) {
    const int t = threadIdx.x;
    const int col = c0 + (vc >= 256 ? t : t % vc);
    const int lane = vc >= 256 ? 0 : t / vc;
    float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
    if (col < vc && lane < lanes) {
#pragma unroll 4
      for (int64_t i = i0 + lane; i < i1; i += lanes) {
        const float4 v = __ldcs(rb + i * vc + col);
        acc.x = fmaf(v.x, v.x, acc.x);
        acc.y = fmaf(v.y, v.y, acc.y);
        acc.z = fmaf(v.z, v.z, acc.z);
        acc.w = fmaf(v.w, v.w, acc.w);
      }
    }
    if (lane < lanes && col < vc) red4[lane * (vc >= 256 ? 256 : vc) + (col - c0)] = acc;
    __syncthreads();
    if (lane == 0 && col < vc) {
      float4 s4 = red4[col - c0];
      for (int l = 1; l < lanes; ++l) {
        const float4 o = red4[l * vc + (col - c0)];
        s4.x += o.x; s4.y += o.y; s4.z += o.z; s4.w += o.w;
      }
      reinterpret_cast<float4*>(part + (b * nsplit + split) * r)[col] = s4;
    }
    __syncthreads();
  }
}

// Many partials (one per 32 rows of R, from B^T P): add them once per column, in
// row-block order, into partial 0, so that the apply kernel's blocks read one value.
__global__ void __launch_bounds__(256) k_colnorm_fold(float* __restrict__ part, int64_t r,
                                                       int nsplit) {
  const int64_t b = blockIdx.y;
  const int64_t j = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
  if (j >= r) return;
  float* pb = part + b * nsplit * r;
  float ss = 0.f;
  for (int s2 = 0; s2 < nsplit; ++s2) ss += pb[s2 * r + j];
  pb[j] = ss;
}

// MODE 0: Q only; 1: + bf16 R and Q; 2: + three-way bf16 splits of R and Q
template <int MODE>
__global__ void __launch_bounds__(256) k_colnorm_apply(const float* __restrict__ R,
                                                        float* __restrict__ Q,
                                                        void* __restrict__ Rg,
                                                        void* __restrict__ Qg,
                                                        const float* __restrict__ part,
                                                        int32_t* __restrict__ flags, int64_t n,
                                                        int64_t r, int nsplit, int64_t part_bs,
                                                        int64_t rows_per_block) {
  extern __shared__ __align__(16) float norm_s[];  // r floats
  const int64_t b = blockIdx.y;
  bool zero = false;
  for (int64_t j = threadIdx.x; j < r; j += blockDim.x) {
    float ss = 0.f;
    for (int s2 = 0; s2 < nsplit; ++s2) ss += part[b * part_bs + s2 * r + j];
    const float nrm = sqrtf(ss);
    norm_s[j] = nrm;
    zero |= !(nrm > 0.f);
  }
  zero = __syncthreads_or(zero);
  if (zero && blockIdx.x == 0 && threadIdx.x == 0) atomicOr(flags + b, F_ZERO_COL);
  const int64_t vc = r / 4;
  const int64_t i0 = blockIdx.x * rows_per_block;
  const int64_t i1 = (i0 + rows_per_block < n) ? i0 + rows_per_block : n;
  const int64_t e0 = (b * n + i0) * vc, e1 = (b * n + i1) * vc;
  const float4* R4 = reinterpret_cast<const float4*>(R);
  float4* Q4 = reinterpret_cast<float4*>(Q);
  // the thread's column group advances by blockDim % vc per iteration (no division)
  const int vci = (int)vc, step = (int)(blockDim.x % vc);
  int jg = (int)(threadIdx.x % vc);
  for (int64_t e = e0 + threadIdx.x; e < e1; e += blockDim.x) {
    const int j = jg * 4;
    jg += step;
    if (jg >= vci) jg -= vci;
    const float4 rv = R4[e];
    const float4 nv = *reinterpret_cast<const float4*>(norm_s + j);
    const float n0 = nv.x, n1 = nv.y, n2 = nv.z, n3 = nv.w;
    float4 qv;
    qv.x = n0 > 0.f ? rv.x / n0 : 0.f;
    qv.y = n1 > 0.f ? rv.y / n1 : 0.f;
    qv.z = n2 > 0.f ? rv.z / n2 : 0.f;
    qv.w = n3 > 0.f ? rv.w / n3 : 0.f;
    Q4[e] = qv;
    if (MODE == 2) {
      const int64_t plane = (int64_t)gridDim.y * n * vc;  // in float4 units
      const float rr[4] = {rv.x, rv.y, rv.z, rv.w}, qq[4] = {qv.x, qv.y, qv.z, qv.w};
      __align__(8) bf16 rh[4], rm[4], rl[4], qh[4], qm[4], ql[4];
#pragma unroll
      for (int q = 0; q < 4; ++q) {
        split3_bf16(rr[q], rh[q], rm[q], rl[q]);
        split3_bf16(qq[q], qh[q], qm[q], ql[q]);
      }
      uint2* R2 = reinterpret_cast<uint2*>(Rg);
      uint2* Q2 = reinterpret_cast<uint2*>(Qg);
      R2[e] = *reinterpret_cast<const uint2*>(rh);
      R2[e + plane] = *reinterpret_cast<const uint2*>(rm);
      R2[e + 2 * plane] = *reinterpret_cast<const uint2*>(rl);
      Q2[e] = *reinterpret_cast<const uint2*>(qh);
      Q2[e + plane] = *reinterpret_cast<const uint2*>(qm);
      Q2[e + 2 * plane] = *reinterpret_cast<const uint2*>(ql);
    } else if (MODE == 1) {
      __nv_bfloat162 r01 = __floats2bfloat162_rn(rv.x, rv.y), r23 = __floats2bfloat162_rn(rv.z, rv.w);
      __nv_bfloat162 q01 = __floats2bfloat162_rn(qv.x, qv.y), q23 = __floats2bfloat162_rn(qv.z, qv.w);
      uint2 rp, qp;
      rp.x = *reinterpret_cast<uint32_t*>(&r01); rp.y = *reinterpret_cast<uint32_t*>(&r23);
      qp.x = *reinterpret_cast<uint32_t*>(&q01); qp.y = *reinterpret_cast<uint32_t*>(&q23);
      reinterpret_cast<uint2*>(Rg)[e] = rp;
      reinterpret_cast<uint2*>(Qg)[e] = qp;
    }
  }
}

int colnorm_splits(int count, int64_t n) {
  // planned on the host before any device is touched: sized for B200's 148 SMs
  int64_t ns = (8 * 148 + count - 1) / count;
  if (ns > 256) ns = 256;
  if (ns > (n + 15) / 16) ns = (n + 15) / 16;
  if (ns < 1) ns = 1;
  return (int)ns;
}

cudaError_t launch_colnorm(const float* R, float* Q, void* Rg, void* Qg, int mode, float* part,
                           int nsplit, bool part_ready, int32_t* flags, int count, int64_t n,
                           int64_t r, cudaStream_t s) {
  const int64_t vc = r / 4;
  if (!part_ready) {
    const size_t red_bytes = (size_t)(vc >= 256 ? 256 : 256 / vc * vc) * sizeof(float4);
    k_colnorm_partial<<<dim3((unsigned)nsplit, (unsigned)count), 256, red_bytes, s>>>(R, part, n,
                                                                                    r, nsplit);
  } else {
    k_colnorm_fold<<<dim3((unsigned)((r + 255) / 256), (unsigned)count), 256, 0, s>>>(part, r,
                                                                                   nsplit);
  }
  const int64_t part_bs = (int64_t)nsplit * r;  // partials of one matrix
  if (part_ready) nsplit = 1;                    // folded into the first
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  const int64_t target_blocks = 8 * (int64_t)sm_count();
  int64_t per_mat = (target_blocks + count - 1) / count;
  int64_t rows = (n + per_mat - 1) / per_mat;
  if (rows < 4) rows = 4;
  const int64_t gx = (n + rows - 1) / rows;
  const size_t smem = (size_t)r * sizeof(float);
  if (smem > 48 * 1024) {
    cudaFuncSetAttribute(k_colnorm_apply<0>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    cudaFuncSetAttribute(k_colnorm_apply<1>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    cudaFuncSetAttribute(k_colnorm_apply<2>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  }
  const dim3 grid((unsigned)gx, (unsigned)count);
  if (mode == 2)
    k_colnorm_apply<2><<<grid, 256, smem, s>>>(R, Q, Rg, Qg, part, flags, n, r, nsplit, part_bs,
                                               rows);
  else if (mode == 1)
    k_colnorm_apply<1><<<grid, 256, smem, s>>>(R, Q, Rg, Qg, part, flags, n, r, nsplit, part_bs,
                                               rows);
  else
    k_colnorm_apply<0><<<grid, 256, smem, s>>>(R, Q, Rg, Qg, part, flags, n, r, nsplit, part_bs,
                                               rows);
  return cudaGetLastError();
}

}  // namespace dion

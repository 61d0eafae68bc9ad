// CUDA-core (SIMT) contractions of the batched Dion step.  They cover every
// precision and shape and serve as the cross-check of the tensor-core path:
//   * a generic strided batched GEMM, C = alpha A B with fp32 accumulation
//     (B Q, B^T P, Gram matrices and the triangular apply);
//   * the fused update: per m x n tile, P R^T and P Q^T accumulated in
//     registers, then M <- (M + G) - (1 - mu) P R^T and X <- X - lr s P Q^T
//     streamed once through HBM.
#include "common.cuh"
#include "internal.h"

namespace dion {

namespace {
constexpr int BM = 64, BN = 64, BK = 16, NT = 256;

template <typename T>
__device__ __forceinline__ void load_tiles(const T* __restrict__ A, const T* __restrict__ B,
                                           const GemmDesc& d, int i0, int j0, int k0,
                                           bool a_kc, bool b_jc, float ra[4], float rb[4]) {
  const int tid = threadIdx.x;
#pragma unroll
  for (int q = 0; q < 4; ++q) {
    const int idx = tid + NT * q;
    int ii, kk;
    if (a_kc) { kk = idx % BK; ii = idx / BK; } else { ii = idx % BM; kk = idx / BM; }
    const int gi = i0 + ii, gk = k0 + kk;
    ra[q] = (gi < d.M && gk < d.K) ? Cvt<T>::load(A + gi * d.A.si + gk * d.A.sk) : 0.f;
    int jj;
    if (b_jc) { jj = idx % BN; kk = idx / BN; } else { kk = idx % BK; jj = idx / BK; }
    const int gj = j0 + jj;
    const int gk2 = k0 + kk;
    rb[q] = (gj < d.N && gk2 < d.K) ? Cvt<T>::load(B + gj * d.B.si + gk2 * d.B.sk) : 0.f;
  }
}

__device__ __forceinline__ void store_tiles(float (*As)[BM + 4], float (*Bs)[BN + 4], bool a_kc,
                                            bool b_jc, const float ra[4], const float rb[4]) {
  const int tid = threadIdx.x;
#pragma unroll
  for (int q = 0; q < 4; ++q) {
    const int idx = tid + NT * q;
    int ii, kk;
    if (a_kc) { kk = idx % BK; ii = idx / BK; } else { ii = idx % BM; kk = idx / BM; }
    As[kk][ii] = ra[q];
    int jj;
    if (b_jc) { jj = idx % BN; kk = idx / BN; } else { kk = idx % BK; jj = idx / BK; }
    Bs[kk][jj] = rb[q];
  }
}
}  // namespace

template <typename T>
__global__ void __launch_bounds__(NT) k_gemm_simt(GemmDesc d) {
  __shared__ __align__(16) float As[2][BK][BM + 4];
  __shared__ __align__(16) float Bs[2][BK][BN + 4];
  const int b = blockIdx.z;
  if (d.flags) {
    const int32_t f = d.flags[b];
    if ((f & d.need_mask) != d.need_mask || (f & d.skip_mask)) return;
  }
  const int i0 = blockIdx.y * BM, j0 = blockIdx.x * BN;
  const T* A = reinterpret_cast<const T*>(d.A.ptr) + b * d.A.sb;
  const T* B = reinterpret_cast<const T*>(d.B.ptr) + b * d.B.sb;
  const bool a_kc = d.A.sk == 1;
  const bool b_jc = d.B.si == 1;
  const int tx = threadIdx.x % 16, ty = threadIdx.x / 16;
  float acc[4][4];
#pragma unroll
  for (int a = 0; a < 4; ++a)
#pragma unroll
    for (int c = 0; c < 4; ++c) acc[a][c] = 0.f;

  float ra[4], rb[4];
  const int ktiles = (d.K + BK - 1) / BK;
  load_tiles<T>(A, B, d, i0, j0, 0, a_kc, b_jc, ra, rb);
  store_tiles(As[0], Bs[0], a_kc, b_jc, ra, rb);
  __syncthreads();
  for (int kt = 0; kt < ktiles; ++kt) {
    const int cur = kt & 1;
    if (kt + 1 < ktiles) load_tiles<T>(A, B, d, i0, j0, (kt + 1) * BK, a_kc, b_jc, ra, rb);
#pragma unroll
    for (int k = 0; k < BK; ++k) {
      const float4 av = *reinterpret_cast<const float4*>(&As[cur][k][ty * 4]);
      const float4 bv = *reinterpret_cast<const float4*>(&Bs[cur][k][tx * 4]);
      const float a4[4] = {av.x, av.y, av.z, av.w};
      const float b4[4] = {bv.x, bv.y, bv.z, bv.w};
#pragma unroll
      for (int a = 0; a < 4; ++a)
#pragma unroll
        for (int c = 0; c < 4; ++c) acc[a][c] = fmaf(a4[a], b4[c], acc[a][c]);
    }
    if (kt + 1 < ktiles) store_tiles(As[cur ^ 1], Bs[cur ^ 1], a_kc, b_jc, ra, rb);
    __syncthreads();
  }
  float* C = d.C + b * d.sCb;
#pragma unroll
  for (int a = 0; a < 4; ++a) {
    const int gi = i0 + ty * 4 + a;
    if (gi >= d.M) continue;
#pragma unroll
    for (int c = 0; c < 4; ++c) {
      const int gj = j0 + tx * 4 + c;
      if (gj < d.N) C[gi * d.sCi + gj * d.sCj] = d.alpha * acc[a][c];
    }
  }
}

cudaError_t launch_gemm_simt(const GemmDesc& d0, bool bf16_operands, cudaStream_t s) {
  const int esz = bf16_operands ? 2 : 4;
  for (int b0 = 0; b0 < d0.batch; b0 += 65535) {
    GemmDesc d = d0;
    const int nb = (d0.batch - b0) < 65535 ? (d0.batch - b0) : 65535;
    d.A.ptr = (const char*)d0.A.ptr + (size_t)b0 * d0.A.sb * esz;
    d.B.ptr = (const char*)d0.B.ptr + (size_t)b0 * d0.B.sb * esz;
    d.C = d0.C + (size_t)b0 * d0.sCb;
    d.flags = d0.flags ? d0.flags + b0 : nullptr;
    d.batch = nb;
    dim3 grid((unsigned)((d.N + BN - 1) / BN), (unsigned)((d.M + BM - 1) / BM), (unsigned)nb);
    if (bf16_operands)
      k_gemm_simt<bf16><<<grid, NT, 0, s>>>(d);
    else
      k_gemm_simt<float><<<grid, NT, 0, s>>>(d);
    cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess) return e;
  }
  return cudaSuccess;
}

// ------------------------------------------------------------ fused update
// Steps 5 and 7 of the Dion step for one m x n tile: the two rank-r products
// P R^T (error feedback) and P Q^T (weight update) share the P tile, and M,
// G, X are read once and M, X written once.
template <typename T>
__global__ void __launch_bounds__(NT) k_update_simt(const T* __restrict__ Pg,
                                                     const T* __restrict__ Rg,
                                                     const T* __restrict__ Qg,
                                                     const float* __restrict__ G,
                                                     float* __restrict__ M, float* __restrict__ X,
                                                     int64_t m, int64_t n, int64_t r,
                                                     float one_minus_mu, float lr_scale,
                                                     float* __restrict__ rmmc, int batch) {
  __shared__ __align__(16) float Ps[BK][BM + 4];
  __shared__ __align__(16) float Rs[BK][BN + 4];
  __shared__ __align__(16) float Qs[BK][BN + 4];
  const int64_t b = blockIdx.z;
  const int64_t i0 = (int64_t)blockIdx.y * BM, j0 = (int64_t)blockIdx.x * BN;
  const T* P = Pg + b * m * r;
  const T* R = Rg + b * n * r;
  const T* Q = Qg + b * n * r;
  const int tx = threadIdx.x % 16, ty = threadIdx.x / 16;
  float a1[4][4], a2[4][4];
#pragma unroll
  for (int a = 0; a < 4; ++a)
#pragma unroll
    for (int c = 0; c < 4; ++c) a1[a][c] = a2[a][c] = 0.f;
  for (int64_t k0 = 0; k0 < r; k0 += BK) {
#pragma unroll
    for (int q = 0; q < 4; ++q) {
      const int idx = threadIdx.x + NT * q;
      const int kk = idx % BK, rr = idx / BK;
      const int64_t gk = k0 + kk;
      const int64_t gi = i0 + rr, gj = j0 + rr;
      Ps[kk][rr] = (gi < m && gk < r) ? Cvt<T>::load(P + gi * r + gk) : 0.f;
      Rs[kk][rr] = (gj < n && gk < r) ? Cvt<T>::load(R + gj * r + gk) : 0.f;
      Qs[kk][rr] = (gj < n && gk < r) ? Cvt<T>::load(Q + gj * r + gk) : 0.f;
    }
    __syncthreads();
#pragma unroll
    for (int k = 0; k < BK; ++k) {
      const float4 pv = *reinterpret_cast<const float4*>(&Ps[k][ty * 4]);
      const float4 rv = *reinterpret_cast<const float4*>(&Rs[k][tx * 4]);
      const float4 qv = *reinterpret_cast<const float4*>(&Qs[k][tx * 4]);
      const float p4[4] = {pv.x, pv.y, pv.z, pv.w};
      const float r4[4] = {rv.x, rv.y, rv.z, rv.w};
      const float q4[4] = {qv.x, qv.y, qv.z, qv.w};
#pragma unroll
      for (int a = 0; a < 4; ++a)
#pragma unroll
        for (int c = 0; c < 4; ++c) {
          a1[a][c] = fmaf(p4[a], r4[c], a1[a][c]);
          a2[a][c] = fmaf(p4[a], q4[c], a2[a][c]);
        }
    }
    __syncthreads();
  }
  const int64_t j = j0 + tx * 4;
  // momentum-change statistics: max |M' - M| and max |M| over this thread's elements
  float dmax = 0.f, mmax = 0.f;
  if (j < n) {
#pragma unroll
    for (int a = 0; a < 4; ++a) {
      const int64_t i = i0 + ty * 4 + a;
      if (i >= m) continue;
      const int64_t e = b * m * n + i * n + j;
      const float4 mv = *reinterpret_cast<const float4*>(M + e);
      const float4 gv = __ldcs(reinterpret_cast<const float4*>(G + e));
      const float4 xv = *reinterpret_cast<const float4*>(X + e);
      float4 mo, xo;
      mo.x = (mv.x + gv.x) - one_minus_mu * a1[a][0];
      mo.y = (mv.y + gv.y) - one_minus_mu * a1[a][1];
      mo.z = (mv.z + gv.z) - one_minus_mu * a1[a][2];
      mo.w = (mv.w + gv.w) - one_minus_mu * a1[a][3];
      xo.x = xv.x - lr_scale * a2[a][0];
      xo.y = xv.y - lr_scale * a2[a][1];
      xo.z = xv.z - lr_scale * a2[a][2];
      xo.w = xv.w - lr_scale * a2[a][3];
      dmax = fmaxf(dmax, fmaxf(fmaxf(fabsf(mo.x - mv.x), fabsf(mo.y - mv.y)),
                               fmaxf(fabsf(mo.z - mv.z), fabsf(mo.w - mv.w))));
      mmax = fmaxf(mmax, fmaxf(fmaxf(fabsf(mv.x), fabsf(mv.y)), fmaxf(fabsf(mv.z), fabsf(mv.w))));
      *reinterpret_cast<float4*>(M + e) = mo;
      *reinterpret_cast<float4*>(X + e) = xo;
    }
  }
  for (int o = 16; o > 0; o >>= 1) {
    dmax = fmaxf(dmax, __shfl_xor_sync(0xffffffffu, dmax, o));
    mmax = fmaxf(mmax, __shfl_xor_sync(0xffffffffu, mmax, o));
  }
  if ((threadIdx.x & 31) == 0) {
    atomic_max_pos(rmmc + b, dmax);
    atomic_max_pos(rmmc + batch + b, mmax);
  }
}

cudaError_t launch_update_simt(const void* Pg, const void* Rg, const void* Qg, bool use_bf16,
                               const float* G, float* M, float* X, int count, int64_t m,
                               int64_t n, int64_t r, float mu, float lr_scale, float* rmmc,
                               cudaStream_t s) {
  for (int b0 = 0; b0 < count; b0 += 65535) {
    const int nb = (count - b0) < 65535 ? (count - b0) : 65535;
    dim3 grid((unsigned)((n + BN - 1) / BN), (unsigned)((m + BM - 1) / BM), (unsigned)nb);
    const size_t mn = (size_t)b0 * m * n;
    if (use_bf16)
      k_update_simt<bf16><<<grid, NT, 0, s>>>(
          (const bf16*)Pg + (size_t)b0 * m * r, (const bf16*)Rg + (size_t)b0 * n * r,
          (const bf16*)Qg + (size_t)b0 * n * r, G + mn, M + mn, X + mn, m, n, r, 1.f - mu,
          lr_scale, rmmc + b0, count);
    else
      k_update_simt<float><<<grid, NT, 0, s>>>(
          (const float*)Pg + (size_t)b0 * m * r, (const float*)Rg + (size_t)b0 * n * r,
          (const float*)Qg + (size_t)b0 * n * r, G + mn, M + mn, X + mn, m, n, r, 1.f - mu,
          lr_scale, rmmc + b0, count);
    cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess) return e;
  }
  return cudaSuccess;
}

}  // namespace dion

// Orthonormalisation of P0 = B Q (step 3 of the Dion step; the Dion article
// on rivista.ai, paragraph 5, names QR and Cholesky decompositions for it).
//
// Cholesky-QR: W = P0^T P0 (a contraction, run elsewhere), W = L L^T here,
// then P = P0 L^-T (a contraction).  This file holds
//   * the Cholesky factorisation with the explicit triangular inverse L^-1,
//     one CTA per matrix in shared memory for r <= 256, and a blocked
//     multi-launch version (32-wide panels) for larger r;
//   * the checks that decide per matrix, on the device: a failed or
//     non-finite pivot or a diagonal ratio max L_kk / min L_kk above the
//     limit sends the matrix to Householder QR; in the second pass the Gram
//     of the first result is tested against I first, and the pass is skipped
//     when max |W - I| is within tolerance;
//   * Householder thin QR (one CTA per matrix, predicated on the fallback
//     bit), with the column signs fixed so that diag(R) >= 0, which is the
//     factor Cholesky-QR reaches in exact arithmetic.
#include "common.cuh"
#include "internal.h"

namespace dion {

namespace {
constexpr int CHOL_SMALL_MAX = 256;
constexpr int NB = 32;  // panel width of the blocked factorisation

__device__ __forceinline__ int64_t tri(int64_t i, int64_t j) { return i * (i + 1) / 2 + j; }

__device__ __forceinline__ bool skip_matrix(int32_t f, int pass) {
  return (f & F_FALLBACK) || (pass == 2 && !(f & F_CHOLQR2));
}
}  // namespace

// ------------------------------------------------ r <= 256: one CTA, shared memory
template <int NT>
__global__ void __launch_bounds__(NT) k_chol_small(CholArgs a) {
  extern __shared__ float sm[];
  const int64_t r = a.r;
  float* L = sm;                  // packed lower triangle, r(r+1)/2
  float* col = L + tri(r, 0);     // r
  float* red = col + r;           // 32
  const int b = blockIdx.x;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  constexpr int NW = NT / 32;
  const int32_t f0 = a.flags[b];
  if (f0 & F_FALLBACK) return;
  const float* W = a.W + (int64_t)b * r * r;

  float dev = 0.f;
  bool nonfin = false;
  for (int64_t i = warp; i < r; i += NW)
    for (int64_t j = lane; j <= i; j += 32) {
      const float v = W[i * r + j];
      L[tri(i, j)] = v;
      nonfin |= !isfinite(v);
      dev = fmaxf(dev, fabsf(v - (i == j ? 1.f : 0.f)));
    }
  nonfin = __syncthreads_or(nonfin);
  if (nonfin) {
    if (tid == 0) atomicOr(a.flags + b, F_NONFINITE | F_FALLBACK);
    return;
  }
  if (a.pass == 2) {
    dev = block_max<NT>(dev, red);
    if (dev <= a.orth_tol) return;  // the first pass is orthonormal enough
  }

  // right-looking Cholesky, column by column
  float dmin = 3.0e38f, dmax = 0.f;
  bool fail = false;
  for (int64_t j = 0; j < r; ++j) {
    const float d = L[tri(j, j)];
    if (!(d > 0.f) || !isfinite(d)) { fail = true; break; }
    const float ljj = sqrtf(d);
    dmin = fminf(dmin, ljj);
    dmax = fmaxf(dmax, ljj);
    for (int64_t i = j + 1 + tid; i < r; i += NT) {
      const float v = L[tri(i, j)] / ljj;
      L[tri(i, j)] = v;
      col[i] = v;
    }
    __syncthreads();
    if (tid == 0) L[tri(j, j)] = ljj;
    for (int64_t i = j + 1 + warp; i < r; i += NW) {
      const float ci = col[i];
      for (int64_t k = j + 1 + lane; k <= i; k += 32) L[tri(i, k)] -= ci * col[k];
    }
    __syncthreads();
  }
  if (fail || (a.pass == 1 && dmax > a.fallback_cond * dmin)) {
    if (tid == 0) atomicOr(a.flags + b, F_FALLBACK);
    return;
  }
  if (tid == 0) {
    a.stats[2 * b] = dmin;
    a.stats[2 * b + 1] = dmax;
  }

  // L^-1 in place, row by row: row i of the inverse needs rows < i of it
  for (int64_t i = 0; i < r; ++i) {
    for (int64_t k = tid; k <= i; k += NT) col[k] = L[tri(i, k)];
    __syncthreads();
    const float inv_ii = 1.f / col[i];
    for (int64_t j = warp; j < i; j += NW) {
      float s = 0.f;
      for (int64_t k = j + lane; k < i; k += 32) s = fmaf(col[k], L[tri(k, j)], s);
      for (int o = 16; o > 0; o >>= 1) s += __shfl_xor_sync(0xffffffffu, s, o);
      if (lane == 0) L[tri(i, j)] = -s * inv_ii;
    }
    if (tid == 0) L[tri(i, i)] = inv_ii;
    __syncthreads();
  }
  float* Li = a.Linv + (int64_t)b * r * r;
  for (int64_t i = warp; i < r; i += NW)
    for (int64_t j = lane; j < r; j += 32) Li[i * r + j] = (j <= i) ? L[tri(i, j)] : 0.f;
  if (a.pass == 2 && tid == 0) atomicOr(a.flags + b, F_CHOLQR2);
}

// ------------------------------------ r <= 256: one CTA, 32 x 32 blocks in shared memory
// Right-looking blocked Cholesky with the triangular inverse, all on chip:
//   for each block column k: factor L_kk (one warp), D_k = L_kk^-1 (one warp),
//   panel L_ik = W_ik D_k^T (a thread per row), trailing W_ij -= L_ik L_jk^T
//   (a warp per block pair, a lane per row, the row of L_ik in registers);
//   then L^-1 block row by block row: X_ij = -D_i sum_{k=j}^{i-1} L_ik X_kj, X_ii = D_i.
// Rows and columns past r are padded with the identity, which factors and inverts
// to itself.  Padded stride 33 keeps row-per-lane accesses free of bank conflicts.
namespace {
constexpr int CB = 32, CBS = 33, CBLK = CB * CBS;
__device__ __forceinline__ float* blk_at(float* base, int i, int j) {
  return base + (i * (i + 1) / 2 + j) * CBLK;
}
}  // namespace

size_t chol_blocked_smem_bytes(int64_t r) {
  const int T = (int)((r + CB - 1) / CB);
  return (size_t)(T * (T + 1) / 2 + T + (T > 1 ? T - 1 : 1)) * CBLK * sizeof(float) + 64 * sizeof(float);
}

template <int NT>
__global__ void __launch_bounds__(NT) k_chol_blocked(CholArgs a) {
  extern __shared__ float sm[];
  const int r = (int)a.r;
  const int T = (r + CB - 1) / CB;
  float* blk = sm;                                  // T(T+1)/2 lower blocks
  float* dinv = blk + (T * (T + 1) / 2) * CBLK;     // T inverses of the diagonal blocks
  float* tmp = dinv + T * CBLK;                     // T-1 blocks of partial sums
  float* red = tmp + (T > 1 ? T - 1 : 1) * CBLK;    // 64 floats
  __shared__ int s_fail;
  const int b = blockIdx.x;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  constexpr int NW = NT / 32;
  const int32_t f0 = a.flags[b];
  if (f0 & F_FALLBACK) return;
  const float* W = a.W + (int64_t)b * r * r;

  // load the lower blocks, padding with the identity; check finiteness and |W - I|
  float dev = 0.f;
  bool nonfin = false;
  const int nlow = T * (T + 1) / 2;
  for (int e = tid; e < nlow * CB * CB; e += NT) {
    const int bl = e / (CB * CB), w = e % (CB * CB), u = w / CB, v = w % CB;
    int bi = 0;
    while ((bi + 1) * (bi + 2) / 2 <= bl) ++bi;
    const int bj = bl - bi * (bi + 1) / 2;
    const int gi = bi * CB + u, gj = bj * CB + v;
    float val;
    if (gi < r && gj < r) {
      val = W[(int64_t)gi * r + gj];
      if (gj <= gi) {
        nonfin |= !isfinite(val);
        dev = fmaxf(dev, fabsf(val - (gi == gj ? 1.f : 0.f)));
      }
    } else {
      val = (gi == gj) ? 1.f : 0.f;
    }
    blk[bl * CBLK + u * CBS + v] = val;
  }
  if (tid == 0) s_fail = 0;
  nonfin = __syncthreads_or(nonfin);
  if (nonfin) {
    if (tid == 0) atomicOr(a.flags + b, F_NONFINITE | F_FALLBACK);
    return;
  }
  if (a.pass == 2) {
    dev = block_max<NT>(dev, red);
    if (dev <= a.orth_tol) return;  // the first pass is orthonormal enough
  }

  float dmin = 3.0e38f, dmax = 0.f;  // meaningful in warp 0
  for (int k = 0; k < T; ++k) {
    float* Lkk = blk_at(blk, k, k);
    float* Dk = dinv + k * CBLK;
    if (warp == 0) {
      // Cholesky of the diagonal block in registers: lane u holds row u; entries of
      // other rows come by warp shuffle (fully unrolled, so the row stays in registers)
      const int u = lane;
      float row[CB];
#pragma unroll
      for (int c = 0; c < CB; ++c) row[c] = Lkk[u * CBS + c];
      bool fail = false;
#pragma unroll
      for (int j = 0; j < CB; ++j) {
        const float d = __shfl_sync(0xffffffffu, row[j], j);
        fail |= !(d > 0.f) || !isfinite(d);
        const float ljj = sqrtf(fmaxf(d, 1e-30f));
        if (k * CB + j < r) { dmin = fminf(dmin, ljj); dmax = fmaxf(dmax, ljj); }
        if (u == j) row[j] = ljj;
        if (u > j) row[j] = row[j] / ljj;
#pragma unroll
        for (int c = j + 1; c < CB; ++c) {
          const float lcj = __shfl_sync(0xffffffffu, row[j], c);  // L[c][j]
          if (u >= c) row[c] = fmaf(-row[j], lcj, row[c]);
        }
      }
#pragma unroll
      for (int c = 0; c < CB; ++c) Lkk[u * CBS + c] = (c <= u) ? row[c] : 0.f;
      if (fail) {
        if (lane == 0) s_fail = 1;
      } else {
        // D_k = L_kk^-1, lane v computes column v by forward substitution; row i of L
        // is broadcast from lane i
        const int v = lane;
        float x[CB];
#pragma unroll
        for (int i = 0; i < CB; ++i) {
          float sacc = (i == v) ? 1.f : 0.f;
#pragma unroll
          for (int t = 0; t < i; ++t) sacc = fmaf(-__shfl_sync(0xffffffffu, row[t], i), x[t], sacc);
          const float lii = __shfl_sync(0xffffffffu, row[i], i);
          x[i] = (i < v) ? 0.f : sacc / lii;
        }
#pragma unroll
        for (int i = 0; i < CB; ++i) Dk[i * CBS + v] = x[i];
      }
    }
    __syncthreads();
    if (s_fail) {
      if (tid == 0) atomicOr(a.flags + b, F_FALLBACK);
      return;
    }
    // panel: L_ik = W_ik D_k^T, one thread per row of the panel
    const int prow = (T - 1 - k) * CB;
    for (int rr = tid; rr < prow; rr += NT) {
      float* row = blk_at(blk, k + 1 + rr / CB, k) + (rr % CB) * CBS;
      float w[CB];
#pragma unroll
      for (int t = 0; t < CB; ++t) w[t] = row[t];
#pragma unroll
      for (int c = 0; c < CB; ++c) {
        float sacc = 0.f;
        for (int t = 0; t <= c; ++t) sacc = fmaf(w[t], Dk[c * CBS + t], sacc);
        row[c] = sacc;
      }
    }
    __syncthreads();
    // trailing update: W_ij -= L_ik L_jk^T for k < j <= i
    const int nt = T - 1 - k;
    const int npairs = nt * (nt + 1) / 2;
    for (int pi = warp; pi < npairs; pi += NW) {
      int ii = 0;
      while ((ii + 1) * (ii + 2) / 2 <= pi) ++ii;
      const int jj = pi - ii * (ii + 1) / 2;
      const int i = k + 1 + ii, j = k + 1 + jj;
      const float* Lik = blk_at(blk, i, k) + lane * CBS;
      const float* Ljk = blk_at(blk, j, k);
      float* Wij = blk_at(blk, i, j) + lane * CBS;
      float av[CB];
#pragma unroll
      for (int t = 0; t < CB; ++t) av[t] = Lik[t];
      for (int c = 0; c < CB; ++c) {
        float sacc = 0.f;
#pragma unroll
        for (int t = 0; t < CB; ++t) sacc = fmaf(av[t], Ljk[c * CBS + t], sacc);
        Wij[c] -= sacc;
      }
    }
    __syncthreads();
  }

  if (a.pass == 1 && dmax > a.fallback_cond * dmin) s_fail = 1;  // warp 0 only
  __syncthreads();
  if (s_fail) {
    if (tid == 0) atomicOr(a.flags + b, F_FALLBACK);
    return;
  }
  if (tid == 0) {
    a.stats[2 * b] = dmin;
    a.stats[2 * b + 1] = dmax;
  }

  // L^-1 block row by block row; X_ij overwrites L_ij once row i is done
  for (int i = 1; i < T; ++i) {
    for (int j = warp; j < i; j += NW) {
      float acc[CB];
#pragma unroll
      for (int c = 0; c < CB; ++c) acc[c] = 0.f;
      for (int k = j; k < i; ++k) {
        const float* Lik = blk_at(blk, i, k) + lane * CBS;
        const float* Xkj = (k == j) ? dinv + j * CBLK : blk_at(blk, k, j);
        float av[CB];
#pragma unroll
        for (int t = 0; t < CB; ++t) av[t] = Lik[t];
#pragma unroll
        for (int t = 0; t < CB; ++t) {
          const float* xr = Xkj + t * CBS;
#pragma unroll
          for (int c = 0; c < CB; ++c) acc[c] = fmaf(av[t], xr[c], acc[c]);
        }
      }
      float* Sj = tmp + j * CBLK + lane * CBS;
#pragma unroll
      for (int c = 0; c < CB; ++c) Sj[c] = acc[c];
    }
    __syncthreads();
    for (int j = warp; j < i; j += NW) {
      const float* Di = dinv + i * CBLK + lane * CBS;
      const float* Sj = tmp + j * CBLK;
      float* Xij = blk_at(blk, i, j) + lane * CBS;
      for (int c = 0; c < CB; ++c) {
        float sacc = 0.f;
        for (int t = 0; t <= lane; ++t) sacc = fmaf(Di[t], Sj[t * CBS + c], sacc);
        Xij[c] = -sacc;
      }
    }
    __syncthreads();
  }

  // write L^-1 (zeros above the diagonal)
  float* Li = a.Linv + (int64_t)b * r * r;
  for (int64_t e = tid; e < (int64_t)r * r; e += NT) {
    const int gi = (int)(e / r), gj = (int)(e % r);
    float val = 0.f;
    if (gj <= gi) {
      const int bi = gi / CB, bj = gj / CB, u = gi % CB, v = gj % CB;
      val = (bi == bj) ? dinv[bi * CBLK + u * CBS + v] : blk_at(blk, bi, bj)[u * CBS + v];
    }
    Li[e] = val;
  }
  if (a.pass == 2 && tid == 0) atomicOr(a.flags + b, F_CHOLQR2);
}

// ---------------------------------------------- r > 256: blocked, multi-launch
// Pass 2 entry: compare W with I; set F_CHOLQR2 when the second pass is needed.
__global__ void __launch_bounds__(256) k_gram_check(CholArgs a) {
  __shared__ float red[32];
  const int b = blockIdx.x;
  const int32_t f = a.flags[b];
  if (f & F_FALLBACK) return;
  const int64_t r = a.r;
  const float* W = a.W + (int64_t)b * r * r;
  float dev = 0.f;
  bool nonfin = false;
  for (int64_t i = threadIdx.x >> 5; i < r; i += 8)
    for (int64_t j = threadIdx.x & 31; j <= i; j += 32) {
      const float v = W[i * r + j];
      nonfin |= !isfinite(v);
      dev = fmaxf(dev, fabsf(v - (i == j ? 1.f : 0.f)));
    }
  nonfin = __syncthreads_or(nonfin);
  dev = block_max<256>(dev, red);
  if (threadIdx.x == 0) {
    if (nonfin)
      atomicOr(a.flags + b, F_NONFINITE | F_FALLBACK);
    else if (a.pass == 2 && dev > a.orth_tol)
      atomicOr(a.flags + b, F_CHOLQR2);
  }
}

// Factor the 32 x 32 diagonal block at k0 (already updated by earlier panels)
// and store its inverse in dinv.
__global__ void __launch_bounds__(256) k_chol_diag(CholArgs a, int64_t k0) {
  __shared__ float D[NB][NB + 1];
  __shared__ float Dinv[NB][NB + 1];
  __shared__ int s_fail;
  const int b = blockIdx.x;
  const int32_t f = a.flags[b];
  if (skip_matrix(f, a.pass)) return;
  const int64_t r = a.r;
  float* W = a.W + (int64_t)b * r * r;
  const int tid = threadIdx.x;
  for (int e = tid; e < NB * NB; e += 256) {
    const int i = e / NB, j = e % NB;
    D[i][j] = (k0 + i < r && k0 + j < r && j <= i) ? W[(k0 + i) * r + k0 + j]
                                                    : (i == j ? 1.f : 0.f);
  }
  if (tid == 0) s_fail = 0;
  __syncthreads();
  const int nb = (int)((r - k0) < NB ? (r - k0) : NB);
  float dmin = 3.0e38f, dmax = 0.f;
  for (int j = 0; j < NB; ++j) {
    const float d = D[j][j];
    if (!(d > 0.f) || !isfinite(d)) {
      if (tid == 0) s_fail = 1;
      break;
    }
    const float ljj = sqrtf(d);
    if (j < nb) {
      dmin = fminf(dmin, ljj);
      dmax = fmaxf(dmax, ljj);
    }
    __syncthreads();
    if (tid > j && tid < NB) D[tid][j] /= ljj;
    __syncthreads();
    if (tid == 0) D[j][j] = ljj;
    for (int e = tid; e < NB * NB; e += 256) {
      const int i = e / NB, k = e % NB;
      if (i > j && k > j && k <= i) D[i][k] -= D[i][j] * D[k][j];
    }
    __syncthreads();
  }
  __syncthreads();
  if (s_fail) {
    if (tid == 0) {
      atomicOr(a.flags + b, F_FALLBACK);
      atomicAnd(a.flags + b, ~F_CHOLQR2);
    }
    return;
  }
  // inverse of the 32 x 32 lower block: column j by forward substitution
  if (tid < NB) {
    const int j = tid;
    for (int i = 0; i < NB; ++i) {
      if (i < j) { Dinv[i][j] = 0.f; continue; }
      float s = (i == j) ? 1.f : 0.f;
      for (int k = j; k < i; ++k) s -= D[i][k] * Dinv[k][j];
      Dinv[i][j] = s / D[i][i];
    }
  }
  __syncthreads();
  for (int e = tid; e < NB * NB; e += 256) {
    const int i = e / NB, j = e % NB;
    if (k0 + i < r && k0 + j < r && j <= i) W[(k0 + i) * r + k0 + j] = D[i][j];
    if (i < nb) a.dinv[((int64_t)b * r + k0 + i) * NB + j] = Dinv[i][j];
  }
  if (tid == 0 && a.pass == 1) {
    atomic_min_pos(a.stats + 2 * b, dmin);
    atomic_max_pos(a.stats + 2 * b + 1, dmax);
  }
}

// Panel: L[i, k0:k0+32] = W[i, k0:k0+32] L_kk^-T for the 64 rows of this block.
__global__ void __launch_bounds__(256) k_chol_panel(CholArgs a, int64_t k0) {
  __shared__ float Di[NB][NB + 1];
  __shared__ float Wt[64][NB + 1];
  const int b = blockIdx.x;
  if (skip_matrix(a.flags[b], a.pass)) return;
  const int64_t r = a.r;
  float* W = a.W + (int64_t)b * r * r;
  const int64_t i0 = k0 + NB + (int64_t)blockIdx.y * 64;
  const int tid = threadIdx.x;
  for (int e = tid; e < NB * NB; e += 256) {
    const int i = e / NB, j = e % NB;
    Di[i][j] = (k0 + i < r) ? a.dinv[((int64_t)b * r + k0 + i) * NB + j] : 0.f;
  }
  for (int e = tid; e < 64 * NB; e += 256) {
    const int i = e / NB, j = e % NB;
    Wt[i][j] = (i0 + i < r && k0 + j < r) ? W[(i0 + i) * r + k0 + j] : 0.f;
  }
  __syncthreads();
  for (int e = tid; e < 64 * NB; e += 256) {
    const int i = e / NB, c = e % NB;
    float s = 0.f;
    for (int t = 0; t <= c; ++t) s = fmaf(Wt[i][t], Di[c][t], s);
    if (i0 + i < r && k0 + c < r) W[(i0 + i) * r + k0 + c] = s;
  }
}

// Trailing update of the lower triangle: W[i, j] -= sum_t L[i, k0+t] L[j, k0+t].
__global__ void __launch_bounds__(256) k_chol_trail(CholArgs a, int64_t k0) {
  __shared__ float Li[64][NB + 1];
  __shared__ float Lj[64][NB + 1];
  const int b = blockIdx.y;
  if (skip_matrix(a.flags[b], a.pass)) return;
  const int64_t r = a.r;
  float* W = a.W + (int64_t)b * r * r;
  // blockIdx.x enumerates tiles (ti, tj) with tj <= ti of the trailing region
  const int64_t t = blockIdx.x;
  int64_t ti = (int64_t)((sqrt(8.0 * (double)t + 1.0) - 1.0) * 0.5);
  while ((ti + 1) * (ti + 2) / 2 <= t) ++ti;
  while (ti * (ti + 1) / 2 > t) --ti;
  const int64_t tj = t - ti * (ti + 1) / 2;
  const int64_t base = k0 + NB;
  const int64_t i0 = base + ti * 64, j0 = base + tj * 64;
  const int tid = threadIdx.x;
  for (int e = tid; e < 64 * NB; e += 256) {
    const int i = e / NB, c = e % NB;
    Li[i][c] = (i0 + i < r) ? W[(i0 + i) * r + k0 + c] : 0.f;
    Lj[i][c] = (j0 + i < r) ? W[(j0 + i) * r + k0 + c] : 0.f;
  }
  __syncthreads();
  const int tx = tid % 16, ty = tid / 16;
  for (int u = 0; u < 4; ++u)
    for (int v = 0; v < 4; ++v) {
      const int ii = ty * 4 + u, jj = tx * 4 + v;
      const int64_t gi = i0 + ii, gj = j0 + jj;
      if (gi >= r || gj >= r || gj > gi) continue;
      float s = 0.f;
#pragma unroll
      for (int c = 0; c < NB; ++c) s = fmaf(Li[ii][c], Lj[jj][c], s);
      W[gi * r + gj] -= s;
    }
}

// After the factorisation: diagonal-ratio test of pass 1.
__global__ void k_chol_cond(CholArgs a) {
  const int b = blockIdx.x * blockDim.x + threadIdx.x;
  if (b >= a.count) return;
  const int32_t f = a.flags[b];
  if (skip_matrix(f, a.pass)) return;
  if (a.pass == 1 && a.stats[2 * b + 1] > a.fallback_cond * a.stats[2 * b])
    atomicOr(a.flags + b, F_FALLBACK);
}

// Block row I of L^-1: Linv[I, J] = -Dinv_I sum_{K=J}^{I-1} L[I, K] Linv[K, J], Linv[I, I] = Dinv_I.
__global__ void __launch_bounds__(256) k_trinv_row(CholArgs a, int64_t I) {
  __shared__ float S[NB][NB + 1];
  __shared__ float Lb[NB][NB + 1];
  __shared__ float Xb[NB][NB + 1];
  const int b = blockIdx.y;
  if (skip_matrix(a.flags[b], a.pass)) return;
  const int64_t r = a.r;
  const float* W = a.W + (int64_t)b * r * r;  // holds L in its lower part
  float* X = a.Linv + (int64_t)b * r * r;
  const int64_t J = blockIdx.x;
  const int tid = threadIdx.x;
  const int64_t ri = I * NB, cj = J * NB;
  if (J == I) {
    for (int e = tid; e < NB * NB; e += 256) {
      const int i = e / NB, j = e % NB;
      if (ri + i < r && cj + j < r)
        X[(ri + i) * r + cj + j] = (j <= i) ? a.dinv[((int64_t)b * r + ri + i) * NB + j] : 0.f;
    }
    return;
  }
  // zero the mirrored upper block
  for (int e = tid; e < NB * NB; e += 256) {
    const int i = e / NB, j = e % NB;
    if (cj + i < r && ri + j < r) X[(cj + i) * r + ri + j] = 0.f;
  }
  float acc[4] = {0.f, 0.f, 0.f, 0.f};
  const int oi = tid / 8, oj0 = (tid % 8) * 4;  // 32 rows x 8 groups of 4 columns
  for (int64_t K = J; K < I; ++K) {
    __syncthreads();
    for (int e = tid; e < NB * NB; e += 256) {
      const int i = e / NB, j = e % NB;
      Lb[i][j] = (ri + i < r && K * NB + j < r) ? W[(ri + i) * r + K * NB + j] : 0.f;
      Xb[i][j] = (K * NB + i < r && cj + j < r) ? X[(K * NB + i) * r + cj + j] : 0.f;
    }
    __syncthreads();
    for (int t = 0; t < NB; ++t) {
      const float l = Lb[oi][t];
#pragma unroll
      for (int q = 0; q < 4; ++q) acc[q] = fmaf(l, Xb[t][oj0 + q], acc[q]);
    }
  }
  __syncthreads();
  for (int q = 0; q < 4; ++q) S[oi][oj0 + q] = acc[q];
  for (int e = tid; e < NB * NB; e += 256) {
    const int i = e / NB, j = e % NB;
    Lb[i][j] = (ri + i < r) ? a.dinv[((int64_t)b * r + ri + i) * NB + j] : 0.f;
  }
  __syncthreads();
  for (int e = tid; e < NB * NB; e += 256) {
    const int i = e / NB, j = e % NB;
    float s = 0.f;
    for (int t = 0; t <= i; ++t) s = fmaf(Lb[i][t], S[t][j], s);
    if (ri + i < r && cj + j < r) X[(ri + i) * r + cj + j] = -s;
  }
}

size_t chol_dinv_floats(int count, int64_t r) { return (size_t)count * r * NB; }

cudaError_t launch_chol_inv(const CholArgs& a, cudaStream_t s) {
  if (a.r <= CHOL_SMALL_MAX) {
    constexpr int NT = 512;
    const size_t smem = chol_blocked_smem_bytes(a.r);
    cudaError_t e = cudaFuncSetAttribute(k_chol_blocked<NT>,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    k_chol_blocked<NT><<<a.count, NT, smem, s>>>(a);
    return cudaGetLastError();
  }
  k_gram_check<<<a.count, 256, 0, s>>>(a);
  const int64_t T = (a.r + NB - 1) / NB;
  for (int64_t kb = 0; kb < T; ++kb) {
    const int64_t k0 = kb * NB;
    k_chol_diag<<<a.count, 256, 0, s>>>(a, k0);
    const int64_t rest = a.r - k0 - NB;
    if (rest > 0) {
      const int64_t pr = (rest + 63) / 64;
      k_chol_panel<<<dim3((unsigned)a.count, (unsigned)pr), 256, 0, s>>>(a, k0);
      k_chol_trail<<<dim3((unsigned)(pr * (pr + 1) / 2), (unsigned)a.count), 256, 0, s>>>(a, k0);
    }
  }
  k_chol_cond<<<(a.count + 255) / 256, 256, 0, s>>>(a);
  for (int64_t I = 0; I < T; ++I)
    k_trinv_row<<<dim3((unsigned)(I + 1), (unsigned)a.count), 256, 0, s>>>(a, I);
  return cudaGetLastError();
}

// -------------------------------------------------------------- Householder
// Thin QR of P0 (m x r) for the matrices flagged F_FALLBACK.  work_cm and
// q_cm are m x r column-major scratch (q_cm may alias P0: P0 is read first).
// P receives the orthonormal factor with column signs fixed so that the
// triangular factor has a non-negative diagonal.
__global__ void __launch_bounds__(1024) k_householder(const float* P0, const bf16* P0s,
                                                      int64_t split_stride, float* work_cm,
                                                      float* q_cm, float* P,
                                                      const int32_t* flags, int64_t m,
                                                      int64_t r) {
  extern __shared__ float hs[];
  float* tau = hs;          // r
  float* beta = hs + r;     // r
  float* red = hs + 2 * r;  // 32
  __shared__ float tile[32][33];
  const int b = blockIdx.x;
  if (!(flags[b] & F_FALLBACK)) return;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  constexpr int NW = 32;
  const float* p0 = P0 + (int64_t)b * m * r;
  float* A = work_cm + (int64_t)b * m * r;
  float* Qc = q_cm + (int64_t)b * m * r;
  float* Pout = P + (int64_t)b * m * r;

  // row-major P0 -> column-major A, through 32 x 32 tiles
  for (int64_t ti = 0; ti < m; ti += 32)
    for (int64_t tj = 0; tj < r; tj += 32) {
      const int y = tid / 32, x = tid % 32;
      float v = 0.f;
      if (ti + y < m && tj + x < r) {
        const int64_t e = (int64_t)b * m * r + (ti + y) * r + tj + x;
        v = P0s ? (__bfloat162float(P0s[e]) + __bfloat162float(P0s[e + split_stride])) +
                      __bfloat162float(P0s[e + 2 * split_stride])
                : p0[(ti + y) * r + tj + x];
      }
      tile[y][x] = v;
      __syncthreads();
      if (ti + x < m && tj + y < r) A[(tj + y) * m + ti + x] = tile[x][y];
      __syncthreads();
    }

  for (int64_t j = 0; j < r; ++j) {
    float* aj = A + j * m;
    float ss = 0.f;
    for (int64_t i = j + 1 + tid; i < m; i += 1024) ss = fmaf(aj[i], aj[i], ss);
    ss = block_sum<1024>(ss, red);
    const float x0 = aj[j];
    const float nrm = sqrtf(fmaf(x0, x0, ss));
    float t = 0.f, bt = 0.f, scal = 0.f;
    if (nrm > 0.f) {
      bt = -copysignf(nrm, x0);
      t = (bt - x0) / bt;
      scal = 1.f / (x0 - bt);
    }
    if (tid == 0) {
      tau[j] = t;
      beta[j] = bt;
    }
    if (nrm > 0.f)
      for (int64_t i = j + 1 + tid; i < m; i += 1024) aj[i] *= scal;
    __syncthreads();
    if (t != 0.f) {
      for (int64_t k = j + 1 + warp; k < r; k += NW) {
        float* ak = A + k * m;
        float w = 0.f;
        for (int64_t i = j + 1 + lane; i < m; i += 32) w = fmaf(aj[i], ak[i], w);
        for (int o = 16; o > 0; o >>= 1) w += __shfl_xor_sync(0xffffffffu, w, o);
        w = (w + ak[j]) * t;
        if (lane == 0) ak[j] -= w;
        for (int64_t i = j + 1 + lane; i < m; i += 32) ak[i] = fmaf(-w, aj[i], ak[i]);
      }
    }
    __syncthreads();
  }

  // thin Q = H_0 ... H_{r-1} [I; 0], accumulated backwards
  for (int64_t k = warp; k < r; k += NW)
    for (int64_t i = lane; i < m; i += 32) Qc[k * m + i] = (i == k) ? 1.f : 0.f;
  __syncthreads();
  for (int64_t j = r - 1; j >= 0; --j) {
    const float t = tau[j];
    if (t != 0.f) {
      const float* v = A + j * m;
      for (int64_t k = j + warp; k < r; k += NW) {
        float* qk = Qc + k * m;
        float w = 0.f;
        for (int64_t i = j + 1 + lane; i < m; i += 32) w = fmaf(v[i], qk[i], w);
        for (int o = 16; o > 0; o >>= 1) w += __shfl_xor_sync(0xffffffffu, w, o);
        w = (w + qk[j]) * t;
        if (lane == 0) qk[j] -= w;
        for (int64_t i = j + 1 + lane; i < m; i += 32) qk[i] = fmaf(-w, v[i], qk[i]);
      }
    }
    __syncthreads();
  }

  // column-major Q -> row-major P with the sign fix
  for (int64_t ti = 0; ti < m; ti += 32)
    for (int64_t tj = 0; tj < r; tj += 32) {
      const int y = tid / 32, x = tid % 32;
      tile[y][x] = (tj + y < r && ti + x < m) ? Qc[(tj + y) * m + ti + x] : 0.f;
      __syncthreads();
      if (ti + y < m && tj + x < r) {
        const float sgn = beta[tj + x] < 0.f ? -1.f : 1.f;
        Pout[(ti + y) * r + tj + x] = sgn * tile[x][y];
      }
      __syncthreads();
    }
}

cudaError_t launch_householder(const float* P0, const void* P0s, float* work_cm, float* q_cm,
                               float* P, int32_t* flags, int count, int64_t m, int64_t r,
                               cudaStream_t s) {
  const size_t smem = (size_t)(2 * r + 32) * sizeof(float);
  if (smem > 48 * 1024) {
    cudaError_t e = cudaFuncSetAttribute(k_householder,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
  }
  k_householder<<<count, 1024, smem, s>>>(P0, (const bf16*)P0s, (int64_t)count * m * r, work_cm,
                                          q_cm, P, flags, m, r);
  return cudaGetLastError();
}

}  // namespace dion

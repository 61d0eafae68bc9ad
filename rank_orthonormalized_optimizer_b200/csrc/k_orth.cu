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
#include "tc.h"

namespace dion {

namespace {
constexpr int CHOL_SMALL_MAX = 256;
constexpr int NB = 32;  // panel width of the blocked factorisation

// pass 1: Cholesky-QR; pass 2: its second pass (matrices with F_CHOLQR2); pass 3: the
// shifted iteration (matrices with F_FALLBACK still iterating)
__device__ __forceinline__ bool skip_matrix(int32_t f, int pass) {
  if (pass == 3) return !(f & F_FALLBACK) || (f & (F_SDONE | F_SFAIL | F_NONFINITE));
  return (f & F_FALLBACK) || (pass == 2 && !(f & F_CHOLQR2));
}
// the bits a failed factorisation sets
__device__ __forceinline__ int32_t fail_bits(int pass, bool nonfinite) {
  if (pass == 3) return F_SFAIL;
  return nonfinite ? (F_NONFINITE | F_FALLBACK) : F_FALLBACK;
}
}  // namespace

// ------------------------------------ r <= 256: one CTA, 32 x 32 blocks in shared memory
// Right-looking blocked Cholesky with the triangular inverse, all on chip:
//   for each block column k: factor L_kk (one warp, rows in registers, columns by
//   shuffle, one template step per column so that every index is a constant); panel
//   L_ik = W_ik L_kk^-T by forward substitution (a thread per row); trailing
//   W_ij -= L_ik L_jk^T (a warp per block pair, a lane per row);
//   then D_k = L_kk^-1 for all k at once (a warp per block, a column per lane), and
//   L^-1 block row by block row: X_ij = -D_i sum_{k=j}^{i-1} L_ik X_kj, X_ii = D_i,
//   each block product shared by two warps (16 columns each).
// Only the factorisation of the diagonal blocks is serial across k, and it keeps the
// one warp that does it short: the triangular inverses are off that path.
// Rows of a block are LD = 36 floats apart: rows start on 16-byte boundaries, so rows are
// read and written as float4 -- a lane's own row without bank conflicts (8 lanes cover
// the 32 banks once), a row shared by the warp as a broadcast -- which cuts the
// shared-memory instructions of the block products four-fold.  Rows and columns past r
// are padded with the identity, which factors and inverts to itself.
// With a.nl > 0 the kernel factors the diagonal block of size nl at (a.o, a.o) of each
// matrix as a leaf of the recursive factorisation: the pass-2 test against I was made
// for the whole matrix before, the diagonal statistics are merged by atomics, and the
// diagonal-ratio test is left to the end of the recursion.
namespace {
constexpr int CB = 32, LD = 36, BLK = CB * LD;
__device__ __forceinline__ float* blk_at(float* base, int i, int j) {
  return base + (i * (i + 1) / 2 + j) * BLK;
}
__device__ __forceinline__ float4 ld4(const float* p) { return *reinterpret_cast<const float4*>(p); }
__device__ __forceinline__ void st4(float* p, float4 v) { *reinterpret_cast<float4*>(p) = v; }
__device__ __forceinline__ float dot4(float4 a, float4 b, float s) {
  return fmaf(a.w, b.w, fmaf(a.z, b.z, fmaf(a.y, b.y, fmaf(a.x, b.x, s))));
}
// a row held as 8 float4 in registers dotted with a row of a block (a broadcast read)
__device__ __forceinline__ float dot32(const float4 (&a)[8], const float* row) {
  float s = 0.f;
#pragma unroll
  for (int q = 0; q < 8; ++q) s = dot4(a[q], ld4(row + 4 * q), s);
  return s;
}
// Column J of the in-register Cholesky of a 32 x 32 block (lane u holds row u), then
// the columns after it.  A template step per column keeps every row index a
// compile-time constant, so the row stays in registers.
template <int J>
__device__ __forceinline__ void chol_col(float (&row)[CB], int lane, int base, int r, bool& fail,
                                         float& my_inv, float& dmin, float& dmax) {
  if constexpr (J < CB) {
    const float d = __shfl_sync(0xffffffffu, row[J], J);
    fail |= !(d > 0.f) || !isfinite(d);
    const float dd = fmaxf(d, 1e-30f);
    const float inv = rsqrtf(dd);
    const float ljj = dd * inv;
    if (base + J < r) { dmin = fminf(dmin, ljj); dmax = fmaxf(dmax, ljj); }
    if (lane == J) { row[J] = ljj; my_inv = inv; }
    if (lane > J) row[J] *= inv;
#pragma unroll
    for (int c = J + 1; c < CB; ++c) {
      const float lcj = __shfl_sync(0xffffffffu, row[J], c);  // L[c][J]
      if (lane >= c) row[c] = fmaf(-row[J], lcj, row[c]);
    }
    chol_col<J + 1>(row, lane, base, r, fail, my_inv, dmin, dmax);
  }
}

// Forward substitution of one row w against L_kk: w <- w L_kk^-T, right-looking over
// columns; Lt holds L_kk^T (row t = column t of L_kk, read as a broadcast), rinv 1/L_tt.
template <int J>
__device__ __forceinline__ void trsv_col(float (&w)[CB], const float* Lt, const float* rinv) {
  if constexpr (J < CB) {
    const float lt = w[J] * rinv[J];
    w[J] = lt;
    if constexpr (J + 1 < CB) {
#pragma unroll
      for (int q = (J + 1) / 4; q < 8; ++q) {
        const float4 c4 = ld4(Lt + J * LD + 4 * q);
        const float cv[4] = {c4.x, c4.y, c4.z, c4.w};
#pragma unroll
        for (int e = 0; e < 4; ++e)
          if (4 * q + e > J) w[4 * q + e] = fmaf(-lt, cv[e], w[4 * q + e]);
      }
    }
    trsv_col<J + 1>(w, Lt, rinv);
  }
}

// Column lane of L^-1 for the 32 x 32 lower-triangular L whose row u is in lane u's
// registers: right-looking, x_t /= L_tt, then x_i -= L_it x_t for i > t (L_it by shuffle).
template <int J>
__device__ __forceinline__ void trinv_col(const float (&row)[CB], float (&x)[CB], float my_inv) {
  if constexpr (J < CB) {
    const float xt = x[J] * __shfl_sync(0xffffffffu, my_inv, J);
    x[J] = xt;
#pragma unroll
    for (int i = J + 1; i < CB; ++i) x[i] = fmaf(-__shfl_sync(0xffffffffu, row[J], i), xt, x[i]);
    trinv_col<J + 1>(row, x, my_inv);
  }
}

// the diagonal entry of the row held by this lane (row u: entry u)
__device__ __forceinline__ float diag_of(const float (&row)[CB], int lane) {
  float d = 0.f;
#pragma unroll
  for (int c = 0; c < CB; ++c) d = (c == lane) ? row[c] : d;
  return d;
}
}  // namespace


size_t chol_blocked_smem_bytes(int64_t r) {
  const int T = (int)((r + CB - 1) / CB);
  return (size_t)(T * (T + 1) / 2 + (T > 2 ? T - 1 : 2)) * BLK * sizeof(float) + 64 * sizeof(float);
}

template <int NT>
__global__ void __launch_bounds__(NT, 1) k_chol_blocked(CholArgs a) {
  extern __shared__ __align__(16) float sm[];
  const bool leaf = a.nl > 0;
  const int r = (int)(leaf ? a.nl : a.r);  // size of the factored block
  const int64_t ld = a.r;                  // row stride of W and L^-1
  const int64_t org = a.o * ld + a.o;      // block origin inside each matrix
  const int T = (r + CB - 1) / CB;
  float* blk = sm;                                  // T(T+1)/2 lower blocks; the diagonal
                                                    // ones end as D_k = L_kk^-1
  float* tmp = blk + (T * (T + 1) / 2) * BLK;       // max(T-1, 2) blocks: partial sums
  float* red = tmp + (T > 2 ? T - 1 : 2) * BLK;     // of the inverse, scratch; 64 floats
  __shared__ int s_fail;
  const int b = blockIdx.x;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  constexpr int NW = NT / 32;
  const int32_t f0 = a.flags[b];
  if ((leaf || a.pass == 3) ? skip_matrix(f0, a.pass) : (f0 & F_FALLBACK) != 0) return;
  // second pass: the Gram's epilogue measured max|W - I| already (a NaN fails the test)
  if (a.pass == 2 && !leaf && a.dev_ready && a.stats[ST * b + 2] <= a.orth_tol) return;
  const float* W = a.W + (int64_t)b * ld * ld + org;

  // load the lower blocks, padding with the identity; check finiteness and |W - I|.
  // Block row bi is read row by row over its bi + 1 blocks as float4 (rows of W are
  // contiguous there; r % 16 == 0 keeps a float4 either inside r or past it).
  float dev = 0.f;
  bool nonfin = false;
  for (int bi = 0; bi < T; ++bi) {
    const int per_row = 8 * (bi + 1);  // float4 per row of the block row
    for (int e = tid; e < CB * per_row; e += NT) {
      const int u = e / per_row, gj = 4 * (e - u * per_row);
      const int gi = bi * CB + u;
      float vv[4];
      if (gi < r && gj < r) {
        const float4 v4 = *reinterpret_cast<const float4*>(W + (int64_t)gi * ld + gj);
        vv[0] = v4.x; vv[1] = v4.y; vv[2] = v4.z; vv[3] = v4.w;
#pragma unroll
        for (int q = 0; q < 4; ++q)
          if (gj + q <= gi) {
            nonfin |= !isfinite(vv[q]);
            dev = fmaxf(dev, fabsf(vv[q] - (gi == gj + q ? 1.f : 0.f)));
          }
      } else {
#pragma unroll
        for (int q = 0; q < 4; ++q) vv[q] = (gi == gj + q) ? 1.f : 0.f;
      }
      st4(blk_at(blk, bi, gj / CB) + u * LD + (gj % CB), make_float4(vv[0], vv[1], vv[2], vv[3]));
    }
  }
  if (tid == 0) s_fail = 0;
  nonfin = __syncthreads_or(nonfin);
  if (nonfin) {
    if (tid == 0) atomicOr(a.flags + b, fail_bits(a.pass, true));
    return;
  }
  if (a.pass == 2 && !leaf) {
    dev = block_max<NT>(dev, red);
    if (dev <= a.orth_tol) return;  // the first pass is orthonormal enough
  }

  float dmin = 3.0e38f, dmax = 0.f;  // meaningful in warp 0
  for (int k = 0; k < T; ++k) {
    float* Dk = blk_at(blk, k, k);
    if (warp == 0) {
      // Cholesky of the diagonal block: lane u holds row u in registers; column j of
      // the other rows comes by warp shuffle (fully unrolled, static indices)
      float row[CB];
#pragma unroll
      for (int q = 0; q < 8; ++q) {
        const float4 v4 = ld4(Dk + lane * LD + 4 * q);
        row[4 * q] = v4.x; row[4 * q + 1] = v4.y; row[4 * q + 2] = v4.z; row[4 * q + 3] = v4.w;
      }
      bool fail = false;
      float my_inv = 0.f;  // 1 / L_uu of this lane's row
      chol_col<0>(row, lane, k * CB, r, fail, my_inv, dmin, dmax);
      // L_kk (zeros above the diagonal) into the block, its transpose into scratch for
      // the panel, the reciprocals of its diagonal into red
#pragma unroll
      for (int q = 0; q < 8; ++q)
        st4(Dk + lane * LD + 4 * q,
            make_float4(4 * q <= lane ? row[4 * q] : 0.f, 4 * q + 1 <= lane ? row[4 * q + 1] : 0.f,
                        4 * q + 2 <= lane ? row[4 * q + 2] : 0.f,
                        4 * q + 3 <= lane ? row[4 * q + 3] : 0.f));
#pragma unroll
      for (int c = 0; c < CB; ++c) tmp[c * LD + lane] = (c <= lane) ? row[c] : 0.f;
      red[lane] = my_inv;
      if (fail && lane == 0) s_fail = 1;
    }
    __syncthreads();
    if (s_fail) {
      if (tid == 0) atomicOr(a.flags + b, fail_bits(a.pass, false));
      return;
    }
    // panel: L_ik = W_ik L_kk^-T by forward substitution, one thread per row of the
    // panel, the row in registers; column t of L_kk is row t of the transpose in tmp
    const int prow = (T - 1 - k) * CB;
    for (int rr = tid; rr < prow; rr += NT) {
      float* rowp = blk_at(blk, k + 1 + rr / CB, k) + (rr % CB) * LD;
      float w[CB];
#pragma unroll
      for (int q = 0; q < 8; ++q) {
        const float4 v4 = ld4(rowp + 4 * q);
        w[4 * q] = v4.x; w[4 * q + 1] = v4.y; w[4 * q + 2] = v4.z; w[4 * q + 3] = v4.w;
      }
      trsv_col<0>(w, tmp, red);
#pragma unroll
      for (int q = 0; q < 8; ++q) st4(rowp + 4 * q, make_float4(w[4 * q], w[4 * q + 1], w[4 * q + 2], w[4 * q + 3]));
    }
    __syncthreads();
    // trailing update: W_ij -= L_ik L_jk^T for k < j <= i, a warp per block pair
    const int nt = T - 1 - k;
    const int npairs = nt * (nt + 1) / 2;
    for (int pi = warp; pi < npairs; pi += NW) {
      int ii = 0;
      while ((ii + 1) * (ii + 2) / 2 <= pi) ++ii;
      const int jj = pi - ii * (ii + 1) / 2;
      const int i = k + 1 + ii, j = k + 1 + jj;
      const float* Lik = blk_at(blk, i, k) + lane * LD;
      const float* Ljk = blk_at(blk, j, k);
      float* Wij = blk_at(blk, i, j) + lane * LD;
      float4 av[8];
#pragma unroll
      for (int q = 0; q < 8; ++q) av[q] = ld4(Lik + 4 * q);
#pragma unroll 1
      for (int cg = 0; cg < 8; ++cg) {
        float4 wv = ld4(Wij + 4 * cg);
        wv.x -= dot32(av, Ljk + (4 * cg) * LD);
        wv.y -= dot32(av, Ljk + (4 * cg + 1) * LD);
        wv.z -= dot32(av, Ljk + (4 * cg + 2) * LD);
        wv.w -= dot32(av, Ljk + (4 * cg + 3) * LD);
        st4(Wij + 4 * cg, wv);
      }
    }
    __syncthreads();
  }

  if (!leaf && a.pass == 1 && dmax > a.fallback_cond * dmin) s_fail = 1;  // warp 0 only
  __syncthreads();
  if (s_fail) {
    if (tid == 0) atomicOr(a.flags + b, F_FALLBACK);
    return;
  }
  if (tid == 0) {
    if (leaf) {
      atomic_min_pos(a.stats + ST * b, dmin);
      atomic_max_pos(a.stats + ST * b + 1, dmax);
    } else {
      a.stats[ST * b] = dmin;
      a.stats[ST * b + 1] = dmax;
    }
  }

  // D_k = L_kk^-1 for every diagonal block at once, a warp per block: lane u loads row u
  // of L_kk, lane v computes column v of D_k (entries of L come by shuffle), and the
  // column replaces the block after the whole warp has read it
  for (int kk = warp; kk < T; kk += NW) {
    float* Dk = blk_at(blk, kk, kk);
    float row[CB], x[CB];
#pragma unroll
    for (int q = 0; q < 8; ++q) {
      const float4 v4 = ld4(Dk + lane * LD + 4 * q);
      row[4 * q] = v4.x; row[4 * q + 1] = v4.y; row[4 * q + 2] = v4.z; row[4 * q + 3] = v4.w;
    }
    const float my_inv = 1.f / diag_of(row, lane);
#pragma unroll
    for (int i = 0; i < CB; ++i) x[i] = (i == lane) ? 1.f : 0.f;
    trinv_col<0>(row, x, my_inv);
    __syncwarp();
#pragma unroll
    for (int i = 0; i < CB; ++i) Dk[i * LD + lane] = (i >= lane) ? x[i] : 0.f;
  }
  __syncthreads();
  // L^-1 block row by block row; X_ij overwrites L_ij once row i is done.  Each block
  // product is shared by two warps, 16 columns each; the lane owns a row.
  for (int i = 1; i < T; ++i) {
    for (int wj = warp; wj < 2 * i; wj += NW) {
      const int j = wj >> 1, c0 = (wj & 1) * 16;
      float acc[16];
#pragma unroll
      for (int c = 0; c < 16; ++c) acc[c] = 0.f;
      for (int k = j; k < i; ++k) {
        const float* Lik = blk_at(blk, i, k) + lane * LD;
        const float* Xkj = blk_at(blk, k, j) + c0;  // X_jj = D_j on the diagonal
#pragma unroll 1
        for (int tg = 0; tg < 8; ++tg) {
          const float4 l4 = ld4(Lik + 4 * tg);
          const float lv[4] = {l4.x, l4.y, l4.z, l4.w};
#pragma unroll
          for (int tt = 0; tt < 4; ++tt) {
            const float* xr = Xkj + (4 * tg + tt) * LD;
#pragma unroll
            for (int q = 0; q < 4; ++q) {
              const float4 x4 = ld4(xr + 4 * q);
              acc[4 * q] = fmaf(lv[tt], x4.x, acc[4 * q]);
              acc[4 * q + 1] = fmaf(lv[tt], x4.y, acc[4 * q + 1]);
              acc[4 * q + 2] = fmaf(lv[tt], x4.z, acc[4 * q + 2]);
              acc[4 * q + 3] = fmaf(lv[tt], x4.w, acc[4 * q + 3]);
            }
          }
        }
      }
      float* Sj = tmp + j * BLK + lane * LD + c0;
#pragma unroll
      for (int q = 0; q < 4; ++q)
        st4(Sj + 4 * q, make_float4(acc[4 * q], acc[4 * q + 1], acc[4 * q + 2], acc[4 * q + 3]));
    }
    __syncthreads();
    for (int wj = warp; wj < 2 * i; wj += NW) {
      const int j = wj >> 1, c0 = (wj & 1) * 16;
      const float* Di = blk_at(blk, i, i) + lane * LD;
      const float* Sj = tmp + j * BLK + c0;
      float acc[16];
#pragma unroll
      for (int c = 0; c < 16; ++c) acc[c] = 0.f;
#pragma unroll 1
      for (int tg = 0; tg < 8; ++tg) {
        const float4 d4 = ld4(Di + 4 * tg);
        const float dv[4] = {d4.x, d4.y, d4.z, d4.w};
#pragma unroll
        for (int tt = 0; tt < 4; ++tt) {
          const float* sr = Sj + (4 * tg + tt) * LD;
#pragma unroll
          for (int q = 0; q < 4; ++q) {
            const float4 s4 = ld4(sr + 4 * q);
            acc[4 * q] = fmaf(dv[tt], s4.x, acc[4 * q]);
            acc[4 * q + 1] = fmaf(dv[tt], s4.y, acc[4 * q + 1]);
            acc[4 * q + 2] = fmaf(dv[tt], s4.z, acc[4 * q + 2]);
            acc[4 * q + 3] = fmaf(dv[tt], s4.w, acc[4 * q + 3]);
          }
        }
      }
      float* Xij = blk_at(blk, i, j) + lane * LD + c0;
#pragma unroll
      for (int q = 0; q < 4; ++q)
        st4(Xij + 4 * q, make_float4(-acc[4 * q], -acc[4 * q + 1], -acc[4 * q + 2], -acc[4 * q + 3]));
    }
    __syncthreads();
  }

  // write L^-1 (zeros above the diagonal) and, when asked, its three-way bf16 split
  const int64_t mo = (int64_t)b * ld * ld + org;
  float* Li = a.Linv + mo;
  const int64_t part = (int64_t)a.count * ld * ld;
  // block row bi, row by row over all T blocks (zeros right of the diagonal), float4
  for (int bi = 0; bi < T; ++bi) {
    const int per_row = 8 * T;
    for (int e = tid; e < CB * per_row; e += NT) {
      const int u = e / per_row, gj = 4 * (e - u * per_row);
      const int gi = bi * CB + u, bj = gj / CB, v = gj % CB;
      if (gi >= r || gj >= r) continue;
      float4 val = make_float4(0.f, 0.f, 0.f, 0.f);
      if (bj <= bi) {
        val = ld4(blk_at(blk, bi, bj) + u * LD + v);
      }
      const int64_t at = (int64_t)gi * ld + gj;
      *reinterpret_cast<float4*>(Li + at) = val;
      if (a.Linvs) {
        const float vv[4] = {val.x, val.y, val.z, val.w};
        __align__(8) bf16 h[4], mi[4], lo[4];
#pragma unroll
        for (int q = 0; q < 4; ++q) split3_bf16(vv[q], h[q], mi[q], lo[q]);
        bf16* d = a.Linvs + mo + at;
        *reinterpret_cast<uint2*>(d) = *reinterpret_cast<const uint2*>(h);
        *reinterpret_cast<uint2*>(d + part) = *reinterpret_cast<const uint2*>(mi);
        *reinterpret_cast<uint2*>(d + 2 * part) = *reinterpret_cast<const uint2*>(lo);
      }
    }
  }
  if (!leaf && a.pass == 2 && tid == 0) atomicOr(a.flags + b, F_CHOLQR2);
}

// ---------------------------------------------- r > 256: blocked, multi-launch
// Entry of the blocked and recursive factorisations: non-finite entries of W send
// the matrix to the fallback; in pass 2, W is compared with I and F_CHOLQR2 is set
// when the second pass is needed.  Grid (count, chunks): any CTA that sees a
// deviation sets the bit.  Chunk 0 resets the diagonal statistics.
// Pass 3 (shifted iteration): a deviation sets F_SMORE, a non-finite entry F_SFAIL, and
// the largest diagonal entry of W goes to the statistics (it scales the shift).
__global__ void __launch_bounds__(256) k_gram_check(CholArgs a) {
  __shared__ float red[32];
  const int b = blockIdx.x;
  if (a.pass != 3 && blockIdx.y == 0 && threadIdx.x == 0) {
    a.stats[ST * b] = 3.0e38f;
    a.stats[ST * b + 1] = 0.f;
  }
  const int32_t f = a.flags[b];
  if (a.pass == 3 ? skip_matrix(f, 3) : (f & F_FALLBACK) != 0) return;
  const int64_t r = a.r;
  const float* W = a.W + (int64_t)b * r * r;
  float dev = 0.f, dmax = 0.f;
  bool nonfin = false;
  const int64_t rows_per = (r + gridDim.y - 1) / gridDim.y;
  const int64_t i0 = blockIdx.y * rows_per, i1 = i0 + rows_per < r ? i0 + rows_per : r;
  for (int64_t i = i0 + (threadIdx.x >> 5); i < i1; i += 8)
    for (int64_t j = threadIdx.x & 31; j <= i; j += 32) {
      const float v = W[i * r + j];
      nonfin |= !isfinite(v);
      dev = fmaxf(dev, fabsf(v - (i == j ? 1.f : 0.f)));
      if (i == j) dmax = fmaxf(dmax, v);
    }
  nonfin = __syncthreads_or(nonfin);
  dev = block_max<256>(dev, red);
  if (a.pass == 3) dmax = block_max<256>(dmax, red);
  if (threadIdx.x == 0) {
    if (nonfin)
      atomicOr(a.flags + b, a.pass == 3 ? F_SFAIL : (F_NONFINITE | F_FALLBACK));
    else if (a.pass == 2 && dev > a.orth_tol)
      atomicOr(a.flags + b, F_CHOLQR2);
    else if (a.pass == 3) {
      if (dev > a.orth_tol) atomicOr(a.flags + b, F_SMORE);
      atomic_max_pos(a.stats + ST * b + 2, dmax);
    }
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
    atomic_min_pos(a.stats + ST * b, dmin);
    atomic_max_pos(a.stats + ST * b + 1, dmax);
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
  if (a.pass == 1 && a.stats[ST * b + 1] > a.fallback_cond * a.stats[ST * b])
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

namespace {
// CTAs per matrix of the entry check: about 128 rows each, at most 64
unsigned gram_check_chunks(int64_t r) {
  const int64_t c = (r + 127) / 128;
  return (unsigned)(c < 1 ? 1 : (c > 64 ? 64 : c));
}

cudaError_t launch_chol_blocked(const CholArgs& a, cudaStream_t s) {
  constexpr int NT = 512;
  const size_t smem = chol_blocked_smem_bytes(a.nl > 0 ? a.nl : a.r);
  // the size of the largest block, not of this one: leaves of several sizes are
  // captured into one graph, whose launches are checked against the attribute later
  cudaError_t e = cudaFuncSetAttribute(k_chol_blocked<NT>,
                                       cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       (int)chol_blocked_smem_bytes(CHOL_SMALL_MAX));
  if (e != cudaSuccess) return e;
  k_chol_blocked<NT><<<a.count, NT, smem, s>>>(a);
  return cudaGetLastError();
}
}  // namespace

int chol_inv_launches(int64_t r) {
  const int64_t T = (r + NB - 1) / NB;
  return r <= CHOL_SMALL_MAX ? 1 : (int)(2 + 3 * T + T);
}

cudaError_t launch_chol_inv(const CholArgs& a, cudaStream_t s) {
  if (a.r <= CHOL_SMALL_MAX) return launch_chol_blocked(a, s);
  k_gram_check<<<dim3((unsigned)a.count, gram_check_chunks(a.r)), 256, 0, s>>>(a);
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

// -------------------------------------------- r > 256: recursive, on the tensor cores
__global__ void k_fb_shift(float* W, int32_t* flags, float* stats, int64_t m, int64_t r);

namespace {
struct RecCtx {
  const CholArgs* a;
  bf16 *Ws, *Ts;
  int64_t max_spins;
  cudaStream_t s;
  int32_t need, skip;
  int launches;
  const char* what;
};

// element offset of entry (i, j) of matrix 0, part 0
inline int64_t at(const RecCtx& c, int64_t i, int64_t j) { return i * c.a->r + j; }

cudaError_t rec_gemm(RecCtx& c, const TcBlockGemm& g, const char* what, bool* done) {
  int nl = 0;
  cudaError_t e = tc_block_gemm(g, c.a->count, c.a->r, c.a->flags, c.need, c.skip, c.max_spins,
                                c.s, &nl, done);
  c.launches += nl;
  if (e != cudaSuccess || !*done) c.what = what;
  return e;
}

// Factor the diagonal block (o, o) of size n: L^-1 of the block into Linv / Linvs.
cudaError_t rec_chol(RecCtx& c, int64_t o, int64_t n, bool* done) {
  const CholArgs& a = *c.a;
  if (n <= CHOL_SMALL_MAX) {
    CholArgs leaf = a;
    leaf.o = o;
    leaf.nl = n;
    ++c.launches;
    cudaError_t e = launch_chol_blocked(leaf, c.s);
    if (e != cudaSuccess) c.what = "leaf factorisation";
    *done = true;
    return e;
  }
  // the first block a multiple of 128 so that every leaf starts on a 128 boundary:
  // a 128-aligned tile window then never straddles two leaves, which is what lets the
  // products skip the zero triangles of L^-1 without reading outside the leaves
  const int64_t n1 = (n / 2 + 127) / 128 * 128, n2 = n - n1, i = o + n1;
  cudaError_t e = rec_chol(c, o, n1, done);
  if (e != cudaSuccess || !*done) return e;
  TcBlockGemm g{};
  // L21 = W21 (L11^-1)^T, split only, into Ts
  g.A = c.Ws + at(c, i, o); g.B = a.Linvs + at(c, o, o);
  g.M = n2; g.N = n1; g.K = n1;
  g.Cs = c.Ts + at(c, i, o); g.alpha = 1.f; g.kr = TC_KR_B_LOWER_NK;
  if ((e = rec_gemm(c, g, "L21 = W21 L11^-T", done)) != cudaSuccess || !*done) return e;
  // W22 -= L21 L21^T (lower tiles), keeping W's split current
  g = TcBlockGemm{};
  g.A = c.Ts + at(c, i, o); g.B = c.Ts + at(c, i, o);
  g.M = n2; g.N = n2; g.K = n1;
  g.C = a.W + at(c, i, i); g.Cs = c.Ws + at(c, i, i);
  g.alpha = -1.f; g.accumulate = true; g.lower_only = true;
  if ((e = rec_gemm(c, g, "W22 -= L21 L21^T", done)) != cudaSuccess || !*done) return e;
  if ((e = rec_chol(c, i, n2, done)) != cudaSuccess || !*done) return e;
  // T = L21 L11^-1 (split only, over W21's split, which is no longer needed)
  g = TcBlockGemm{};
  g.A = c.Ts + at(c, i, o); g.B = a.Linvs + at(c, o, o); g.b_mn = true;
  g.M = n2; g.N = n1; g.K = n1;
  g.Cs = c.Ws + at(c, i, o); g.alpha = 1.f; g.kr = TC_KR_B_LOWER_KN;
  if ((e = rec_gemm(c, g, "T = L21 L11^-1", done)) != cudaSuccess || !*done) return e;
  // (L^-1)21 = -L22^-1 T
  g = TcBlockGemm{};
  g.A = a.Linvs + at(c, i, i); g.B = c.Ws + at(c, i, o); g.b_mn = true;
  g.M = n2; g.N = n1; g.K = n2;
  g.C = a.Linv + at(c, i, o); g.Cs = a.Linvs + at(c, i, o);
  g.alpha = -1.f; g.kr = TC_KR_A_LOWER_MK;
  return rec_gemm(c, g, "(L^-1)21 = -L22^-1 T", done);
}
}  // namespace

cudaError_t launch_chol_inv_rec(const CholArgs& a, bf16* Ws, bf16* Ts, int64_t max_spins,
                                cudaStream_t s, int* nlaunch, bool* done, const char** what) {
  *nlaunch = 0;
  *done = false;
  *what = "";
  if (a.r <= CHOL_SMALL_MAX || !a.Linvs || !Ws || !Ts || a.nl != 0) return cudaErrorInvalidValue;
  const int32_t need = a.pass == 2 ? F_CHOLQR2 : (a.pass == 3 ? F_FALLBACK : 0);
  const int32_t skip = a.pass == 3 ? (F_SDONE | F_SFAIL | F_NONFINITE) : F_FALLBACK;
  RecCtx c{&a, Ws, Ts, max_spins, s, need, skip, 0, ""};
  k_gram_check<<<dim3((unsigned)a.count, gram_check_chunks(a.r)), 256, 0, s>>>(a);
  ++c.launches;
  cudaError_t e = cudaGetLastError();
  if (e == cudaSuccess && a.pass == 3) {
    k_fb_shift<<<a.count, 256, 0, s>>>(a.W, a.flags, a.stats, a.m, a.r);
    ++c.launches;
    e = cudaGetLastError();
  }
  if (e == cudaSuccess) e = rec_chol(c, 0, a.r, done);
  else c.what = "entry check";
  if (e == cudaSuccess && *done) {
    k_chol_cond<<<(a.count + 255) / 256, 256, 0, s>>>(a);
    ++c.launches;
    e = cudaGetLastError();
    if (e != cudaSuccess) c.what = "diagonal-ratio test";
  }
  *nlaunch = c.launches;
  *what = c.what;
  return e;
}

// ------------------------------------- shifted Cholesky-QR iteration (fallback, r > 256)
// For the matrices whose Cholesky-QR failed (F_FALLBACK, finite): A_0 = P0,
// A_{k+1} = A_k R_k^-1 with R_k^T R_k = A_k^T A_k + s_k I.  Every iterate is P0 times an
// upper-triangular matrix with a positive diagonal, so the orthonormal limit is P0's
// Q factor with diag(R) > 0, the same P as Householder QR (shifted Cholesky-QR:
// Fukaya, Kannan, Nakatsukasa, Yamamoto and Yanagisawa, SIAM J. Sci. Comput. 2020).
// The shift s_k = 2 u (sqrt(m r) + r) max_i (A_k^T A_k)_ii (u = 2^-24) exceeds the
// rounding of the computed Gram, so the factorisation exists; singular values below
// sqrt(s_k) grow by about 1/sqrt(s_k) per step.  Once every pivot of a shifted
// factorisation is above 10 sqrt(s_k) the iterate is well conditioned and later steps
// are plain Cholesky-QR.  A matrix is done when max |A_k^T A_k - I| <= orth_tol.

// Start (begin != 0) or continue the loop: the conditional is set while some matrix
// is still iterating and fewer than max_rounds rounds have run.  One CTA.
__global__ void __launch_bounds__(256) k_fb_cond(int32_t* flags, float* stats, int count,
                                                 cudaGraphConditionalHandle h, int* rounds,
                                                 int max_rounds, int begin) {
  bool any = false;
  for (int b = threadIdx.x; b < count; b += blockDim.x) {
    const int32_t f = flags[b];
    if (begin) {
      if ((f & F_FALLBACK) && !(f & F_NONFINITE)) {
        atomicAnd(flags + b, ~(F_SMORE | F_SDONE | F_SFAIL | F_SITER | F_SNOSHIFT));
        stats[ST * b] = 3.0e38f;
        stats[ST * b + 2] = 0.f;
        stats[ST * b + 3] = 0.f;
        any = true;
      }
    } else {
      any |= !skip_matrix(f, 3);
    }
  }
  any = __syncthreads_or(any);
  if (threadIdx.x == 0) {
    const int k = begin ? 0 : *rounds + 1;
    *rounds = k;
    cudaGraphSetConditional(h, (any && k < max_rounds) ? 1u : 0u);
  }
}

// After the entry check of an iteration: finish converged matrices; otherwise add the
// shift to the diagonal of W.  One CTA per matrix.
__global__ void __launch_bounds__(256) k_fb_shift(float* W, int32_t* flags, float* stats,
                                                  int64_t m, int64_t r) {
  const int b = blockIdx.x;
  const int32_t f = flags[b];
  if (skip_matrix(f, 3)) return;
  const float dmin = stats[ST * b], dmax_w = stats[ST * b + 2], s_prev = stats[ST * b + 3];
  __syncthreads();
  if ((f & F_SITER) && !(f & F_SMORE)) {
    if (threadIdx.x == 0) atomicOr(flags + b, F_SDONE);
    return;
  }
  const bool noshift = (f & F_SNOSHIFT) || (s_prev > 0.f && dmin * dmin > 100.f * s_prev);
  const float s = noshift ? 0.f
                          : 2.f * 5.9604645e-8f * (sqrtf((float)m * (float)r) + (float)r) * dmax_w;
  if (s > 0.f) {
    float* w = W + (int64_t)b * r * r;
    for (int64_t i = threadIdx.x; i < r; i += blockDim.x) w[i * r + i] += s;
  }
  if (threadIdx.x == 0) {
    atomicAnd(flags + b, ~F_SMORE);
    if (noshift) atomicOr(flags + b, F_SNOSHIFT);
    stats[ST * b] = 3.0e38f;
    stats[ST * b + 2] = 0.f;
    stats[ST * b + 3] = s;
  }
}

// After the apply of an iteration: the matrices still iterating now hold A_{k+1} in P.
__global__ void k_fb_mark(int32_t* flags, int count) {
  const int b = blockIdx.x * blockDim.x + threadIdx.x;
  if (b < count && !skip_matrix(flags[b], 3)) atomicOr(flags + b, F_SITER);
}

cudaError_t launch_fb_cond(int32_t* flags, float* stats, int count, cudaGraphConditionalHandle h,
                           int* rounds, int max_rounds, bool begin, cudaStream_t s) {
  k_fb_cond<<<1, 256, 0, s>>>(flags, stats, count, h, rounds, max_rounds, begin ? 1 : 0);
  return cudaGetLastError();
}

cudaError_t launch_fb_mark(int32_t* flags, int count, cudaStream_t s) {
  k_fb_mark<<<(count + 255) / 256, 256, 0, s>>>(flags, count);
  return cudaGetLastError();
}

// -------------------------------------------------------------- Householder
// Thin QR of P0 (m x r) for the matrices flagged F_FALLBACK.  work_cm and
// q_cm are m x r column-major scratch (q_cm may alias P0: P0 is read first).
// P receives the orthonormal factor with column signs fixed so that the
// triangular factor has a non-negative diagonal.
__global__ void __launch_bounds__(1024) k_householder(const float* P0, const bf16* P0s,
                                                      const float* Pit, int64_t split_stride,
                                                      float* work_cm, float* q_cm, float* P,
                                                      const int32_t* flags, int64_t m,
                                                      int64_t r) {
  extern __shared__ float hs[];
  float* tau = hs;          // r
  float* beta = hs + r;     // r
  float* red = hs + 2 * r;  // 32
  __shared__ float tile[32][33];
  const int b = blockIdx.x;
  const int32_t f = flags[b];
  if (!(f & F_FALLBACK) || (f & F_SDONE)) return;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  constexpr int NW = 32;
  // an iterate P0 R^-1 of the shifted iteration has the same Q factor as P0
  const bool iter = (f & F_SITER) != 0;
  if (iter) P0s = nullptr;
  const float* p0 = (iter ? Pit : P0) + (int64_t)b * m * r;
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
  // matrices the shifted iteration left unfinished restart from their iterate, held in P
  const size_t smem = (size_t)(2 * r + 32) * sizeof(float);
  if (smem > 48 * 1024) {
    cudaError_t e = cudaFuncSetAttribute(k_householder,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
  }
  k_householder<<<count, 1024, smem, s>>>(P0, (const bf16*)P0s, P, (int64_t)count * m * r,
                                          work_cm, q_cm, P, flags, m, r);
  return cudaGetLastError();
}

}  // namespace dion


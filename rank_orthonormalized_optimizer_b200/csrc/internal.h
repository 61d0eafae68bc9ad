// Internal interface between the host planner (dion_api.cu) and the kernels.
#pragma once

#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stddef.h>
#include <stdint.h>

#include "../../include/dion.h"

namespace dion {

// Record a message for dion_last_error() on this thread and return `s`.
dion_status set_error(dion_status s, const char* fmt, ...);
// Workspace size of a valid handle's plan.
dion_status plan_workspace_bytes(dion_handle h, size_t* bytes);

// Generic strided batched operand: element (i, k) of matrix b sits at
// base + b*sb + i*si + k*sk (in elements).
struct Operand {
  const void* ptr;
  int64_t sb, si, sk;
};

// C[b] = alpha * A[b] (M x K) * B[b] (K x N), fp32 accumulation, fp32 output.
// A matrix b is skipped when flags != nullptr and
// (flags[b] & need_mask) != need_mask or (flags[b] & skip_mask) != 0.
struct GemmDesc {
  Operand A, B;
  float* C;
  int64_t sCb, sCi, sCj;
  int M, N, K, batch;
  float alpha;
  const int32_t* flags;
  int32_t need_mask, skip_mask;
};

// ---- elementwise / layout kernels (k_elementwise.cu)
cudaError_t launch_form_b(const float* M, const float* G, void* Bg, bool use_bf16, int64_t elems,
                          cudaStream_t s);
cudaError_t launch_prep_q(const float* Q, void* Qg, bool use_bf16, int count, int64_t n, int64_t r,
                          cudaStream_t s);
// three-way bf16 splits ([3][...] planes) for fp32 contractions on the tensor cores
cudaError_t launch_form_b_split(const float* M, const float* G, void* Bs, int64_t elems,
                                cudaStream_t s);
cudaError_t launch_prep_q_split(const float* Q, void* Qs, int count, int64_t n, int64_t r,
                                cudaStream_t s);
// Zero the per-matrix flags (or set init_bits), the Cholesky statistics and the 16
// tile counters of the bucket's dynamically scheduled kernels.
cudaError_t launch_init_flags(int32_t* flags, float* stats, int* sched, float* rmmc, int count,
                              int32_t init_bits, cudaStream_t s);
// mode 0: fp32 P only; 1: + bf16 copy Pg; 2: + three-way bf16 split Pg.  pg_ready: Pg
// already holds the first pass's P; only second-pass and fallback matrices are written.
cudaError_t launch_finalize_p(const float* P2, void* Pg, int mode, const int32_t* flags,
                              int count, int64_t m, int64_t r, float* P, bool pg_ready,
                              cudaStream_t s);
int colnorm_splits(int count, int64_t n);
// mode 0: Q only; 1: + bf16 R, Q; 2: + three-way bf16 splits of R, Q.  part holds nsplit
// partial column sums of squares per matrix ([count][nsplit][r]); part_ready: B^T P wrote
// them already (else a first kernel does, over nsplit row ranges).
cudaError_t launch_colnorm(const float* R, float* Q, void* Rg, void* Qg, int mode,
                           float* part, int nsplit, bool part_ready, int32_t* flags, int count,
                           int64_t n, int64_t r, cudaStream_t s);
cudaError_t launch_split3(const float* src, void* dst, int64_t n, int64_t dst_stride,
                          cudaStream_t s);
// RMMC = max |M' - M| / max |M| per matrix (rmmc: [3][count], the third plane written;
// +inf for a zero M that changed, 0 for one that did not) and, when d_status is not
// null, the public flag bits with DION_MAT_HIGH_RMMC where RMMC > rmmc_threshold.
cudaError_t launch_write_status(const int32_t* flags, float* rmmc, float rmmc_threshold,
                                int32_t* d_status, int count, cudaStream_t s);
// Row-sharded step: this rank's rows [row0, row0 + m) of P0 (fp32, or its three-way
// split when P0s is not null) into the zeroed m_full x r buffers `full`; the flagged
// matrices' rows back from `full` into P; the number of matrices with (flags & mask).
cudaError_t launch_rows_to_full(const float* P0, const void* P0s, float* full, int count,
                                int64_t m, int64_t m_full, int64_t row0, int64_t r,
                                cudaStream_t s);
cudaError_t launch_rows_from_full(const float* full, float* P, const int32_t* flags, int count,
                                  int64_t m, int64_t m_full, int64_t row0, int64_t r,
                                  cudaStream_t s);
cudaError_t launch_count_flags(const int32_t* flags, int count, int32_t mask, float* out,
                               cudaStream_t s);
// P[b] = the sum of the three bf16 parts of Ps[b] (parts `plane` elements apart), for the
// matrices that took neither the second pass nor the fallback.
cudaError_t launch_p_from_split(float* P, const void* Ps, int64_t plane, const int32_t* flags,
                                int count, int64_t m, int64_t r, cudaStream_t s);

// ---- SIMT contractions (k_gemm_simt.cu)
cudaError_t launch_gemm_simt(const GemmDesc& d, bool bf16_operands, cudaStream_t s);
// rmmc: [2][count], max |M' - M| and max |M| of each matrix max-ed into them
cudaError_t launch_update_simt(const void* Pg, const void* Rg, const void* Qg, bool use_bf16,
                               const float* G, float* M, float* X, int count, int64_t m,
                               int64_t n, int64_t r, float mu, float lr_scale, float* rmmc,
                               cudaStream_t s);

// ---- orthonormalisation (k_orth.cu)
// pass 1: Cholesky of W = P0^T P0; pass 2: checks W = P1^T P1 first.
struct CholArgs {
  float* W;            // [count, r, r] Gram on entry (lower part overwritten by L)
  float* Linv;         // [count, r, r] receives L^-1 (upper part zero)
  __nv_bfloat16* Linvs;  // [3][count, r, r] three-way split of L^-1 (may be null)
  float* dinv;         // [count, r, 32] scratch: inverses of 32x32 diagonal blocks
  int32_t* flags;      // [count]
  float* stats;        // [count, 2] min and max of diag(L) (positive floats)
  int count;
  int64_t r;
  int pass;            // 1 or 2
  float fallback_cond; // pass 1: diag ratio limit
  float orth_tol;      // pass 2: skip the second pass when max|W - I| <= orth_tol
  int64_t o, nl;       // leaf of the recursive factorisation: block (o, o) of size nl
  int64_t m;           // rows of P0 (pass 3: scales the shift)
  int dev_ready;       // pass 2, r <= 256: stats[ST b + 2] holds max|W - I| already
};
// pass 3 = one step of the shifted Cholesky-QR iteration (launch_chol_inv_rec only)
// r <= 256: one kernel; larger r: the blocked CUDA-core factorisation (many launches).
cudaError_t launch_chol_inv(const CholArgs& a, cudaStream_t s);
int chol_inv_launches(int64_t r);
// Recursive factorisation with the triangular inverse on the tensor cores, for r > 256:
//   [W11 .; W21 W22] -> L11, L11^-1 (recursion); L21 = W21 L11^-T; W22 -= L21 L21^T;
//   L22, L22^-1 (recursion); (L^-1)21 = -L22^-1 L21 L11^-1,
// leaves of at most 256 by the one-kernel factorisation.  Products are fp32-accurate
// (three-way bf16 splits).  W's split Ws ([3][count][r][r]) must hold the split of
// W's lower 128 x 128 tiles on entry (the Gram writes it); Ts is scratch of the same
// size.  a.Linvs is required.  *nlaunch receives the number of kernels launched;
// *what names the failing step when the return is not cudaSuccess or *done is false.
cudaError_t launch_chol_inv_rec(const CholArgs& a, __nv_bfloat16* Ws, __nv_bfloat16* Ts,
                                int64_t max_spins, cudaStream_t s, int* nlaunch, bool* done,
                                const char** what);
// Shifted Cholesky-QR iteration for the flagged matrices (r > 256): the loop's
// condition kernel (begin: reset the iteration state) and the per-iteration marker.
cudaError_t launch_fb_cond(int32_t* flags, float* stats, int count, cudaGraphConditionalHandle h,
                           int* rounds, int max_rounds, bool begin, cudaStream_t s);
cudaError_t launch_fb_mark(int32_t* flags, int count, cudaStream_t s);
// P0 fp32, or (when P0s is not null) its three-way bf16 split [3][count][m][r].
// Matrices flagged F_FALLBACK and not finished by the shifted iteration; those the
// iteration had started restart from their iterate in P.
cudaError_t launch_householder(const float* P0, const void* P0s, float* work_cm, float* q_cm,
                               float* P, int32_t* flags, int count, int64_t m, int64_t r,
                               cudaStream_t s);
size_t chol_dinv_floats(int count, int64_t r);

}  // namespace dion

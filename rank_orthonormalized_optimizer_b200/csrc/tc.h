// Tensor-core (tcgen05 + TMEM, fed by TMA) kernels of the batched Dion step.
// Each entry sets *done when it launched its kernel; *done stays false only when a
// tensor map could not be encoded (tc_map_error() says why), which the caller
// reports as an error.
#pragma once

#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

namespace dion {

// Text of the last tensor-map encoding failure on this thread.
const char* tc_map_error();

// P0[b] (m x r, fp32) = Bg[b] (m x n, bf16) * Qg[b]^T (Qg: r x n, bf16); when P0s is
// not null its three-way bf16 split is written as well, its parts `plane` elements
// apart (0: count * m * r, [3][count][m][r]; more when the bucket's P0 lies in a stack
// shared with other buckets of the same m and r).
cudaError_t tc_gemm_bq(const void* Bg, const void* Qg, float* P0, __nv_bfloat16* P0s,
                       int64_t plane, int count, int64_t m, int64_t n, int64_t r,
                       int64_t max_spins, int32_t* flags, cudaStream_t s, int* nlaunch,
                       bool* done);
// Steps 1 and 2 fused: Bg[b] = bf16(M[b] + G[b]) (written for B^T P) and the
// three-way bf16 split of P0[b] = Bg[b] Qg[b]^T into P0s ([3][count][m][r]).
// tile_counter: one int in device memory, zero before the call (tiles are taken from it).
// P0s's parts lie `plane` elements apart (0: count * m * r).
cudaError_t tc_formb_bq(const float* M, const float* G, const void* Qg, void* Bg,
                        __nv_bfloat16* P0s, int64_t plane, int count, int64_t m, int64_t n,
                        int64_t r, int64_t max_spins, int32_t* flags, int* tile_counter,
                        cudaStream_t s, int* nlaunch, bool* done);
// R[b] (n x r, fp32) = Bg[b]^T (n x m) * Pg[b] (m x r, bf16).  When colsq is not null it
// receives the sums of squares of R's columns over blocks of R's rows, fixed order:
// colsq[b][i][j] for row block i < tc_btp_col_splits(n) (the partials of Q = colnorm(R)).
cudaError_t tc_gemm_btp(const void* Bg, const void* Pg, float* R, float* colsq, int count,
                        int64_t m, int64_t n, int64_t r, int64_t max_spins, int32_t* flags,
                        cudaStream_t s, int* nlaunch, bool* done);
int tc_btp_col_splits(int64_t n);
// As tc_gemm_btp from three-way splits; colsq blocks of 32 rows: 4 ceil(n / 128) of them.
// M <- (M + G) - (1 - mu) Pg Rg^T and X <- X - lr_scale Pg Qg^T (Pg: m x r, Rg, Qg: n x r, bf16).
// tile_counter: one int in device memory, zero before the call (tiles are taken from it).
// split: Pg, Rg, Qg are three-way bf16 splits ([3][count][...]) of fp32 operands.
// rmmc: [2][count] floats, max |M' - M| and max |M| of each matrix max-ed into them
// (non-negative before the call).
// zplane_p: matrices between Pg's split parts (0: count).
cudaError_t tc_update(const void* Pg, int zplane_p, const void* Rg, const void* Qg, bool split,
                      const float* G, float* M, float* X, int count, int64_t m, int64_t n,
                      int64_t r, float mu, float lr_scale, int64_t max_spins, int32_t* flags,
                      int* tile_counter, float* rmmc, cudaStream_t s, int* nlaunch, bool* done);
// fp32 contractions from three-way bf16 splits: P0 (fp32) and P0s = split(Bs Qs^T),
// R = Bs^T Ps; K is accumulated in 512-wide chunks added in fp32 registers.
// (P0s's parts `plane` elements apart, Ps's `zplane_p` matrices apart; 0: count.)
cudaError_t tc_gemm_bq_split(const __nv_bfloat16* Bs, const __nv_bfloat16* Qs, float* P0,
                             __nv_bfloat16* P0s, int64_t plane, int count, int64_t m, int64_t n,
                             int64_t r, int64_t max_spins, int32_t* flags, cudaStream_t s,
                             int* nlaunch, bool* done);
cudaError_t tc_gemm_btp_split(const __nv_bfloat16* Bs, const __nv_bfloat16* Ps, int zplane_p,
                              float* R, float* colsq, int count, int64_t m, int64_t n, int64_t r,
                              int64_t max_spins, int32_t* flags, cudaStream_t s, int* nlaunch,
                              bool* done);

// W[b] (r x r, fp32) = X[b]^T X[b] from the three-way split Xs ([3][count][m][r] bf16),
// six split products; matrices failing (flags & need) == need && !(flags & skip) skipped.
// Only the 128 x 128 tiles on and below the diagonal are written (r > 64), and, when Ws
// is not null, their split ([3][count][r][r]) as well.  When devmax is not null,
// max_{j <= i} |W_ij - I_ij| of matrix b is max-ed into devmax[b * dev_stride] (which must
// hold a non-negative value before the call; NaN wins).  parts = 2 reads only the two
// leading parts and sums three products, (1,0) (0,1) (0,0): about 2^-17 relative, enough
// for the Gram of an already orthonormalised first pass (the second Cholesky-QR pass).
cudaError_t tc_gram(const __nv_bfloat16* Xs, float* W, __nv_bfloat16* Ws, float* devmax,
                    int dev_stride, int count, int64_t m, int64_t r, int32_t* flags, int32_t need,
                    int32_t skip, int64_t max_spins, cudaStream_t s, int* nlaunch, bool* done,
                    int parts = 3);
// Y[b] (m x r, fp32) = X[b] L[b]^T from the splits Xs ([3][count][m][r]) and Ls
// ([3][count][r][r], L lower triangular), optionally writing Y's split to Ys and its
// bf16 rounding to Yb ([count][m][r]).  Column
// tile j reads L[j][k] for k below the end of its 128-wide window only: the entries of
// L above the diagonal inside that window must be zero, those further right are not read.
cudaError_t tc_apply(const __nv_bfloat16* Xs, const __nv_bfloat16* Ls, float* Y,
                     __nv_bfloat16* Ys, __nv_bfloat16* Yb, int count, int64_t m, int64_t r,
                     int32_t* flags, int32_t need, int32_t skip, int64_t max_spins,
                     cudaStream_t s, int* nlaunch, bool* done);

// Triangular operands: K blocks that can only multiply zeros are skipped.
enum {
  TC_KR_B_LOWER_NK = 1,  // B stored [N][K], B[j][k] = 0 for k > j
  TC_KR_B_LOWER_KN = 2,  // B stored [K][N], B[k][j] = 0 for k < j
  TC_KR_A_LOWER_MK = 4,  // A stored [M][K], A[i][k] = 0 for k > i
};

// One product on blocks of a stack of r x r matrices (rows r elements apart, matrices
// r * r apart; operands are three-way bf16 splits [3][count][r][r], pointers at the
// block origin of part 0):  C = alpha op(A) op(B)  or  C += alpha op(A) op(B).
// a_mn: A is stored transposed ([K][M]); b_mn: B is stored [K][N] (else [N][K]).
// C (fp32, may be null unless accumulating) and Cs (its split, may be null) are block
// origins in stacks of the same geometry.  N must be a multiple of 16.
struct TcBlockGemm {
  const __nv_bfloat16* A;
  bool a_mn;
  const __nv_bfloat16* B;
  bool b_mn;
  int64_t M, N, K;
  float* C;
  __nv_bfloat16* Cs;
  float alpha;
  bool accumulate;
  int kr;           // TC_KR_* bits
  bool lower_only;  // only 128 x 128 tiles on or below the block's diagonal
};
cudaError_t tc_block_gemm(const TcBlockGemm& g, int count, int64_t r, int32_t* flags,
                          int32_t need, int32_t skip, int64_t max_spins, cudaStream_t s,
                          int* nlaunch, bool* done);

}  // namespace dion

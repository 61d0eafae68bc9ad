/*
 * dion.h -- C ABI of the batched Dion optimizer step on NVIDIA B200 (sm_100a).
 *
 * One call updates every 2-D weight matrix of a model.  For a weight X
 * (m x n, row-major fp32), its error-feedback momentum M (m x n), its
 * gradient G (m x n) and the right factor Q (n x r) kept between steps:
 *
 *   B  = M + G
 *   P  = orth(B Q)             Cholesky-QR, Householder QR when ill-conditioned
 *   R  = B^T P
 *   M <- B - (1 - mu) P R^T    error feedback
 *   Q <- colnorm(R)            unit columns (a zero column stays zero)
 *   X <- X - lr * s * P Q^T    s = sqrt(m / n) unless given
 *
 * Sources: rivista.ai, "Dion e la fine del monopolio di Adam negli optimizer
 * AI distribuiti" (the article on "Dion: Distributed Orthonormalized
 * Updates"): paragraph 2 (only the top-r singular directions are
 * orthonormalised), paragraph 3 (error feedback re-injects what the low-rank
 * update missed), paragraph 5 (amortised power iteration with QR and Cholesky
 * decompositions; 2-D parameters only, biases and 1-D weights go elsewhere).
 * Matrices of one shape are stacked into a [count, m, n] tensor and processed
 * together, as "DASH: Faster Shampoo via Batched Block Preconditioning and
 * Efficient Inverse-Root Solvers" (Methodologie, section 1) stacks blocks.
 *
 * Conventions for every entry point:
 *  - Pointers named d_* / in dion_bucket_ptrs are DEVICE pointers on the
 *    handle's device; all others are host pointers.
 *  - The caller owns every buffer (weights, state, gradients, workspace,
 *    status) and the stream.  The library never allocates or frees device
 *    memory and never synchronises the device, except where stated.
 *  - Errors in arguments are returned synchronously as a dion_status and
 *    leave every buffer untouched; dion_last_error() then gives a message.
 *    Numerical events are reported per matrix in the device status array.
 *  - No C++ exception crosses this interface.  A handle must not be used
 *    from two threads or two streams at the same time.
 */
#ifndef DION_H
#define DION_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef struct dion_ctx* dion_handle;

/* Host-side return codes. */
typedef enum dion_status {
  DION_OK = 0,
  DION_ERR_INVALID_ARG = 1,         /* null pointer, bad count, bad option value  */
  DION_ERR_UNSUPPORTED_SHAPE = 2,   /* shape outside the supported set (see dion_init) */
  DION_ERR_WORKSPACE_TOO_SMALL = 3, /* workspace smaller than dion_init reported  */
  DION_ERR_CUDA = 4,                /* a CUDA runtime call failed (message says which) */
  DION_ERR_NOT_INITIALIZED = 5,     /* null or freed handle                       */
  DION_ERR_DEVICE = 6,              /* current device is not sm_100 (B200)       */
  DION_ERR_MISALIGNED = 7,          /* a device pointer is not aligned as required
                                       (16 bytes for the Dion step, 4 for dion_vec_step) */
  DION_ERR_HOST = 8                 /* host-side failure (out of host memory); no C++
                                       exception ever leaves the library             */
} dion_status;

/* Per-matrix status bits written to d_status[] by every step (OR-ed). */
enum {
  DION_MAT_OK = 0,
  DION_MAT_FALLBACK = 1,      /* Cholesky-QR rejected; P came from the fallback (shifted
                                 Cholesky-QR iteration for r > 256 on the tensor path,
                                 else Householder QR): the same Q factor                 */
  DION_MAT_CHOLQR2 = 2,       /* a second Cholesky-QR pass was applied                   */
  DION_MAT_NONFINITE = 4,     /* a Gram matrix held Inf/NaN (inputs were not finite)     */
  DION_MAT_TIMEOUT = 8,       /* a bounded device wait ran out; this matrix's outputs
                                 are not valid and X, M, Q may be partly updated         */
  DION_MAT_ZERO_COLUMN = 16,  /* some column of R had zero norm; its Q column is zero    */
  DION_MAT_HIGH_RMMC = 32     /* the momentum changed faster than rmmc_threshold: RMMC =
                                 max|M' - M| / max|M| > rmmc_threshold (CurvaDion's gate:
                                 this matrix needs synchronising; see DION_VIEW_RMMC)     */
};

/* Arithmetic of the four rank-r contractions (B Q, B^T P, P R^T, P Q^T). */
typedef enum dion_precision {
  DION_PREC_FP32 = 0,  /* fp32-accurate: on CUDA cores fp32 FMA; on the tensor path the
                          operands are split into three bf16 parts (x = x0 + x1 + x2)
                          and B Q, B^T P sum six part products (about 2^-24 relative),
                          the update three (about 2^-17); fp32 accumulation          */
  DION_PREC_BF16 = 1   /* B, Q, P, R rounded to bf16 (round to nearest even), fp32
                          accumulation; Gram, Cholesky and the triangular apply stay
                          fp32                                                       */
} dion_precision;

/* How P = orth(B Q) is formed. */
typedef enum dion_orth_mode {
  DION_ORTH_AUTO = 0,        /* Cholesky-QR; a second pass when max|P^T P - I| > orth_tol;
                                the fallback when a pivot fails or the Cholesky diagonal
                                ratio exceeds fallback_cond: for r > 256 on the tensor
                                path, shifted Cholesky-QR iterated until
                                max|P^T P - I| <= orth_tol (at most 16 iterations, run
                                as a CUDA graph with a conditional node; not when the
                                caller's stream is being captured), then Householder QR
                                for whatever is left; otherwise Householder QR            */
  DION_ORTH_CHOLQR = 1,      /* one Cholesky-QR pass (+ the fallback)                    */
  DION_ORTH_CHOLQR2 = 2,     /* always two passes (+ the fallback)                       */
  DION_ORTH_HOUSEHOLDER = 3  /* Householder QR for every matrix                          */
} dion_orth_mode;

/* Which kernels run the contractions. */
typedef enum dion_kernel_path {
  DION_PATH_TENSOR = 0,  /* tcgen05 tensor-core kernels fed by TMA where the precision
                            and shape allow; the SIMT kernels elsewhere               */
  DION_PATH_SIMT = 1     /* CUDA-core kernels everywhere (a cross-check)               */
} dion_kernel_path;

/* One bucket: `count` matrices of identical shape (m, n), updated at rank r. */
typedef struct dion_bucket_desc {
  int64_t m, n, r;
  int32_t count;
  float scale;     /* s in X -= lr*s*P Q^T; <= 0 selects sqrt(m / n) */
} dion_bucket_desc;

typedef struct dion_options {
  float mu;                /* error-feedback decay, 0 <= mu < 1 (default 0.95)            */
  int32_t precision;       /* dion_precision (default DION_PREC_BF16)                      */
  int32_t orth_mode;       /* dion_orth_mode (default DION_ORTH_AUTO)                      */
  float fallback_cond;     /* Householder when max L_kk / min L_kk exceeds it (1e3)        */
  float orth_tol;          /* AUTO: second pass when max|P^T P - I| > orth_tol (2e-5)      */
  int32_t kernel_path;     /* dion_kernel_path (default DION_PATH_TENSOR)                  */
  int64_t max_wait_spins;  /* bound on every device-side wait; when it runs out the
                              kernel sets DION_MAT_TIMEOUT and returns (default 1<<26)     */
  float rmmc_threshold;    /* DION_MAT_HIGH_RMMC where RMMC exceeds it (default 0: every
                              matrix whose momentum moved; not NaN)                        */
  int32_t stack_orth;      /* 1: buckets of equal m and r share one orthonormalisation
                              stack -- one Gram, Cholesky and apply launch over all their
                              matrices, as "DASH: Faster Shampoo via Batched Block
                              Preconditioning and Efficient Inverse-Root Solvers"
                              (Methodologie, section 1) stacks equal-sized blocks of
                              different layers; results are bit for bit those of 0.  It
                              pays where many small buckets leave each launch latency-
                              bound; the stack can only start after its last bucket's
                              B Q, which costs overlap on large buckets (default 0)      */
} dion_options;

/* Device buffers of one bucket, all contiguous, row-major, 16-byte aligned:
 *   X, M, G : fp32 [count, m, n]     X and M updated in place, G read only
 *   Q       : fp32 [count, n, r]     read (previous factor) and overwritten
 * Q must hold unit-norm columns before the first step (any such Q). */
typedef struct dion_bucket_ptrs {
  float* X;
  float* M;
  const float* G;
  float* Q;
} dion_bucket_ptrs;

/* Fill *opt with the defaults listed above. */
dion_status dion_default_options(dion_options* opt);

/*
 * Plan a step over `nbuckets` buckets (host only; touches no device).
 * Supported shapes: 1 <= count <= 65535, 1 <= r <= min(m, n), r % 16 == 0,
 * n % 8 == 0, m >= 1, and every buffer below 2^40 elements; otherwise
 * DION_ERR_UNSUPPORTED_SHAPE.  opt may be NULL (defaults).
 * On success *out receives a handle (host memory owned by the library until
 * dion_free) and *workspace_bytes the size of the device workspace that
 * every dion_step_batched call must be given.
 */
dion_status dion_init(const dion_bucket_desc* buckets, int32_t nbuckets,
                      const dion_options* opt, dion_handle* out,
                      size_t* workspace_bytes);

/*
 * One Dion step over every bucket, enqueued on `stream` (a cudaStream_t; NULL
 * is the legacy default stream) of the current device.  Returns as soon as
 * the work is enqueued.
 *   ptrs        host array of nbuckets device-pointer sets, in the order the
 *               buckets were given to dion_init
 *   lr          learning rate eta of this step
 *   d_workspace device scratch of at least *workspace_bytes from dion_init,
 *               16-byte aligned; its contents need not be preserved between
 *               calls, and it must not be shared by two steps in flight
 *   d_status    device int32 array, one word per matrix (bucket by bucket,
 *               slot by slot), overwritten with DION_MAT_* bits; may be NULL
 * Within a bucket the matrices are independent.  X, M and Q are written only
 * by the last kernels of the step.  Work runs on `stream` and on streams owned by
 * the handle, forked from and joined back to `stream` with events; the first
 * step with a fallback-capable plan (r > 256 on the tensor path) for a given
 * workspace builds a CUDA graph (host memory owned by the handle).
 */
dion_status dion_step_batched(dion_handle h, const dion_bucket_ptrs* ptrs,
                              int32_t nbuckets, float lr, void* d_workspace,
                              size_t workspace_bytes, int32_t* d_status, void* stream);

/*
 * The same step with the gradients coming from HOST memory: copies
 * host_grads[b] (fp32 [count, m, n], pinned for asynchronous copies) into the
 * device buffer ptrs[b].G (which this call therefore overwrites), runs the
 * step, copies d_status back to host_status (one int32 per matrix), and
 * synchronises `stream` before returning, so host_status is valid on return.
 * The copies run on a stream owned by the handle, ordered after the work already
 * on `stream`, one bucket at a time with the largest gradient first; each bucket's
 * whole step starts on `stream` as soon as its own gradients are on the device, so
 * the steps of the early buckets overlap the uploads of the later ones (the
 * results are those of dion_step_batched: buckets are independent).
 */
dion_status dion_step_batched_from_host(dion_handle h, const dion_bucket_ptrs* ptrs,
                                        const float* const* host_grads, int32_t nbuckets,
                                        float lr, void* d_workspace, size_t workspace_bytes,
                                        int32_t* d_status, int32_t* host_status,
                                        void* stream);

/*
 * Size of the scratch array built into the library for dion_step_batched_noalloc:
 * 16 MiB of device memory on every GPU the library is used on, held until the
 * process exits.
 */
#define DION_STATIC_SCRATCH_BYTES (16u << 20)

/*
 * dion_step_batched without a caller workspace, for callers that cannot allocate
 * device memory: a plug-in or extension that is handed only the model's buffers by a
 * host program whose allocator it cannot reach, or a training loop whose device
 * memory is sized once at start-up (a fixed pool, a budget the host program enforces)
 * and that must not allocate afterwards.  The pages describe nothing like it; it is a
 * convenience of this library.  Arguments are those of dion_step_batched; X, M, G, Q
 * and d_status remain caller buffers.
 *  - Scratch comes from one array of DION_STATIC_SCRATCH_BYTES inside the library.
 *    A plan whose workspace (from dion_init) is larger is rejected with
 *    DION_ERR_WORKSPACE_TOO_SMALL and nothing runs.
 *  - The first call on a device looks the array's device address up (with that
 *    device current); make that first call outside any stream capture.  The address
 *    is looked up again when the device's context has changed since the last call
 *    (after cudaDeviceReset, for instance), since a new context holds a new copy.
 *  - Every call on a device shares the array.  It keeps whatever the last call
 *    left in it; the step writes every scratch word it reads, so nothing needs
 *    clearing.  Calls whose work overlaps on the GPU (two streams, two threads, two
 *    handles) race on it: serialise them.
 *  - This call makes no cudaMalloc or cudaFree and calls no allocating library
 *    routine.  As with dion_step_batched, the first call on a handle and device
 *    creates the handle's streams and events, and a plan with r > 256 on the tensor
 *    path builds the fallback's CUDA graph, which is rebuilt whenever the same handle
 *    switches between this entry point and dion_step_batched (their scratch differs);
 *    the driver may set aside memory for those objects.
 */
dion_status dion_step_batched_noalloc(dion_handle h, const dion_bucket_ptrs* ptrs,
                                      int32_t nbuckets, float lr, int32_t* d_status,
                                      void* stream);

/*
 * ---------------------------------------------------------------------------
 * Row-sharded step.  The article says Dion cuts the data synchronised between
 * nodes (paragraph 3) and works under data, tensor and fully sharded data
 * parallelism, FSDP2 included (paragraph 5), without saying how.  Here the rows of
 * every matrix are split among the ranks: a rank holds rows [row0, row0 + m) of X,
 * M and G of each matrix and the whole Q (n x r), the same on every rank.  The step
 * is the whole-matrix step; only sums over ranks of r-sized quantities cross
 * between ranks, each an all-reduce (sum) of fp32 values that the CALLER performs
 * (NCCL, or anything else) on a buffer inside the workspace:
 *
 *   DION_XCHG_GRAM    the Grams W = P0^T P0 of every bucket (count r^2 floats each)
 *   DION_XCHG_GRAM2   the second Cholesky-QR pass's Grams, followed by one float per
 *                     bucket: the number of its matrices Cholesky-QR rejected
 *   DION_XCHG_GATHER  only for a bucket with rejected matrices: its P0 as
 *                     [count, m_full, r] with this rank's rows filled and zeros
 *                     elsewhere (summing gathers it); Householder QR of the whole P0
 *                     then runs on every rank, which keeps its rows
 *   DION_XCHG_R       R = B^T P of every bucket (count n r floats each)
 *
 * The Cholesky factors, the decisions taken from them and Q = colnorm(R) are
 * computed from the summed values by the same deterministic kernels on every rank,
 * so every rank reaches the same P, Q and status.  Usage (every rank):
 *
 *   dion_exchange x;
 *   dion_step_sharded_begin(h, ptrs, nb, lr, ws, ws_bytes, d_status, stream, &x);
 *   while (x.count > 0) {
 *     allreduce_sum_fp32(x.d_buf, x.count, stream);   // e.g. ncclAllReduce
 *     dion_step_sharded_continue(h, &x);
 *   }
 *
 * Every call enqueues work on `stream` and returns; the continue that follows the
 * DION_XCHG_GRAM2 exchange synchronises `stream` once (it reads the per-bucket
 * counts to decide which buckets need the gather).  An error abandons the step
 * (X, M and Q are written only by its last call); all ranks must then abandon it.
 * Runs on the tensor path only; the rank-sharded fallback is Householder QR of the
 * gathered P0, never the shifted Cholesky-QR iteration.
 */
typedef struct dion_shard_desc {
  int64_t m_full;  /* rows of every whole matrix of the bucket                          */
  int64_t row0;    /* first row this rank holds; it holds dion_bucket_desc.m rows      */
} dion_shard_desc;

enum { DION_XCHG_NONE = 0, DION_XCHG_GRAM = 1, DION_XCHG_GRAM2 = 2, DION_XCHG_GATHER = 3,
       DION_XCHG_R = 4 };

typedef struct dion_exchange {
  float* d_buf;    /* device buffer to sum over ranks in place (inside the workspace)  */
  int64_t count;   /* fp32 elements; 0 when the step is complete                       */
  int32_t what;    /* DION_XCHG_*                                                      */
} dion_exchange;

/*
 * Plan a row-sharded step: buckets[b] gives this rank's rows (m), the columns, the
 * rank and the count; shards[b] the rows of the whole matrices and this rank's first
 * row (row0 + m <= m_full).  r <= min(m_full, n); s defaults to sqrt(m_full / n).
 * Otherwise as dion_init; the plan may only be stepped by dion_step_sharded_begin.
 */
dion_status dion_init_sharded(const dion_bucket_desc* buckets, const dion_shard_desc* shards,
                              int32_t nbuckets, const dion_options* opt, dion_handle* out,
                              size_t* workspace_bytes);

/* Start a row-sharded step (arguments as dion_step_batched); *next receives the first
 * exchange.  DION_ERR_INVALID_ARG when a step is already in progress on the handle. */
dion_status dion_step_sharded_begin(dion_handle h, const dion_bucket_ptrs* ptrs,
                                    int32_t nbuckets, float lr, void* d_workspace,
                                    size_t workspace_bytes, int32_t* d_status, void* stream,
                                    dion_exchange* next);

/* Continue the step after *next's buffer has been summed over all ranks; *next
 * receives the following exchange, or count 0 when the step is complete. */
dion_status dion_step_sharded_continue(dion_handle h, dion_exchange* next);

/* Release the handle (host memory only).  NULL is accepted. */
dion_status dion_free(dion_handle h);

/* Static text for a status code. */
const char* dion_status_string(dion_status s);

/* Message of the last error raised on this thread ("" if none). */
const char* dion_last_error(void);

/* Total number of matrices over all buckets (the length of d_status). */
int64_t dion_num_matrices(dion_handle h);

/* Kernel launches made by the most recent dion_step_batched call (0 before). */
int32_t dion_last_launch_count(dion_handle h);

/* Intermediates of the most recent step, for inspection after the stream has
 * been synchronised (DION_VIEW_P on the tensor path first rebuilds the fp32 P from
 * the bf16 split the step keeps, with a kernel on the legacy default stream that the
 * call waits for): which = DION_VIEW_P gives P (fp32 [count, m, r]),
 * DION_VIEW_R gives R (fp32 [count, n, r]), DION_VIEW_RMMC gives each matrix's
 * relative maximum momentum change (fp32 [count]).  *d_ptr points into d_workspace.
 *
 * RMMC is the statistic by which "CurvaDion: Curvature-Adaptive Distributed
 * Orthonormalization" (mlsanity.com, Abstract) decides which layers need
 * synchronising: built from the momentum the optimizer already keeps, O(d) per
 * layer.  The page does not write it down; here, per matrix, with M before the step
 * and M' after it, RMMC = max_ij |M'_ij - M_ij| / max_ij |M_ij| (+inf for a zero M
 * that changed, 0 for one that did not).  The fused update computes both maxima from
 * the values it streams anyway.  In a row-sharded step each rank's value covers its
 * own rows (the maximum over ranks of each maximum gives the whole matrix's). */
enum { DION_VIEW_P = 0, DION_VIEW_R = 1, DION_VIEW_RMMC = 2 };
dion_status dion_workspace_view(dion_handle h, int32_t bucket, int32_t which,
                                void* d_workspace, void** d_ptr, size_t* bytes);

/*
 * Per-kernel timing with CUDA events recorded on the step's stream.
 * dion_profile_enable(h, 1) starts recording around every kernel class of
 * every later step (and clears the totals); dion_profile_read synchronises
 * the recorded events and returns, per class, the summed milliseconds and
 * the number of launches.  Classes are numbered as DION_KCLASS_*.
 */
enum {
  DION_KCLASS_FORM_B = 0,   /* B = M + G in GEMM precision                */
  DION_KCLASS_PREP_Q = 1,   /* previous Q into GEMM layout               */
  DION_KCLASS_GEMM_BQ = 2,  /* P0 = B Q                                  */
  DION_KCLASS_ORTH = 3,     /* Gram, Cholesky, inverse, apply, fallback  */
  DION_KCLASS_GEMM_BTP = 4, /* R = B^T P                                 */
  DION_KCLASS_COLNORM = 5,  /* Q = colnorm(R) and the update operands     */
  DION_KCLASS_UPDATE = 6,   /* fused M and X update                      */
  DION_KCLASS_COUNT = 7
};
dion_status dion_profile_enable(dion_handle h, int32_t on);
dion_status dion_profile_read(dion_handle h, double* ms, int64_t* launches,
                              int32_t nclasses);

/*
 * ---------------------------------------------------------------------------
 * The step of the vector (1-D) parameters.  Dion takes only the 2-D weight
 * matrices; biases and normalisation gains go to AdamW or Lion (paragraph 5 of
 * the rivista.ai article).  The article names the two rules without writing them;
 * they are taken as published:
 *
 *   DION_VEC_ADAMW -- "Decoupled Weight Decay Regularization" (Loshchilov and
 *   Hutter), decoupled decay first, then the bias-corrected Adam step, t >= 1:
 *     x <- x (1 - lr wd)
 *     m <- b1 m + (1 - b1) g;        v <- b2 v + (1 - b2) g^2
 *     x <- x - lr (m / (1 - b1^t)) / (sqrt(v / (1 - b2^t)) + eps)
 *
 *   DION_VEC_LION -- "Symbolic Discovery of Optimization Algorithms" (Chen et
 *   al.), the sign of an interpolation of momentum and gradient:
 *     c = b1 m + (1 - b1) g
 *     x <- x (1 - lr wd) - lr sign(c)            sign(0) = 0
 *     m <- b2 m + (1 - b2) g
 *   Because sign(c) is a discrete decision, c is fixed to fp32 arithmetic with
 *   no fused multiply-add: 1 - b1 is rounded to fp32, then each product and the
 *   sum are rounded to fp32 (round to nearest even).
 *
 * State and arithmetic are fp32.  One call updates a list of tensors, each a
 * contiguous array with its own state; the elements are independent.  Non-finite
 * gradients are not checked: they make the affected elements non-finite.
 */
typedef enum dion_vec_rule { DION_VEC_ADAMW = 0, DION_VEC_LION = 1 } dion_vec_rule;

typedef struct dion_vec_tensor {
  float* x;         /* parameter, updated in place                                */
  const float* g;   /* gradient, read only                                        */
  float* m;         /* first moment (both rules), updated in place                */
  float* v;         /* second moment (AdamW; not read by Lion, may be NULL there)  */
  int64_t numel;    /* elements; a tensor with 0 elements is skipped (its pointers
                       may then be NULL)                                          */
} dion_vec_tensor;

typedef struct dion_vec_options {
  int32_t rule;        /* DION_VEC_ADAMW or DION_VEC_LION                         */
  float lr;            /* learning rate, finite                                   */
  float beta1, beta2;  /* in [0, 1)                                               */
  float eps;           /* AdamW: added to the bias-corrected sqrt(v), > 0         */
  float weight_decay;  /* decoupled decay, finite and >= 0                        */
  int64_t step;        /* AdamW: this step's number t >= 1 (bias correction)      */
} dion_vec_options;

/* Defaults of the two papers: AdamW lr 1e-3, betas (0.9, 0.999), eps 1e-8,
 * weight decay 0.01, step 1; Lion lr 1e-4, betas (0.9, 0.99), weight decay 0. */
dion_status dion_vec_default_options(int32_t rule, dion_vec_options* o);

/*
 * One step of every tensor of tensors[0 .. ntensors), enqueued on `stream` of the
 * current device; returns as soon as the work is enqueued.  tensors is a host
 * array of device pointer sets.  Every pointer must be 4-byte aligned (16-byte
 * alignment of x, g, m, v at the same offset takes a vectorised path); x, g, m
 * and v of one tensor, and different tensors, must not overlap.  The arguments
 * are checked before anything is enqueued (DION_ERR_INVALID_ARG,
 * DION_ERR_MISALIGNED, DION_ERR_DEVICE); no handle and no workspace are needed.
 * Up to 128 tensors go into one kernel launch; longer lists take several
 * launches on the same stream.
 */
dion_status dion_vec_step(const dion_vec_tensor* tensors, int32_t ntensors,
                          const dion_vec_options* o, void* stream);

/* Kernel launches made by the most recent dion_vec_step on this thread. */
int32_t dion_vec_last_launch_count(void);

#ifdef __cplusplus
}
#endif

#endif /* DION_H */

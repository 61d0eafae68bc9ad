// Tensor-core kernels of the batched Dion step for sm_100a: tcgen05.mma with
// accumulators in TMEM, operands staged in shared memory by TMA (128-byte
// swizzle), persistent CTAs over all tiles of a bucket, warp-specialised:
//   warp 0        TMA producer of the MMA operands
//   warp 1        MMA issuer (one thread)
//   warp 2        TMEM allocator; in the update kernel also the TMA producer
//                 of the M, G, X slabs
//   warps 4..7    epilogue (TMEM lanes 0..127)
// Two TMEM accumulators let the epilogue of one tile overlap the MMAs of the
// next.  Every wait is bounded (max_spins); on give-up the CTA drains what it
// issued, marks DION_MAT_TIMEOUT on the matrices it did not finish, frees its
// TMEM and returns.
//
// gemm (step 2 and 4 of the Dion step, the two halves of one power-iteration
// step, rivista.ai Dion article paragraph 5):
//   P0[b] = B[b] Q[b]     A = B (m x n, K-major),   B-operand = Q^T (r x n, K-major)
//   R[b]  = B[b]^T P[b]   A = B^T (MN-major view),  B-operand = P (m x r, MN-major)
// update (steps 5 and 7, error feedback of paragraph 3 and the weight step):
//   acc = P [R | Q]^T per 128 x 128 tile (one N = 256 MMA), then
//   M <- (M + G) - (1 - mu) acc_R,  X <- X - lr s acc_Q, with M, G, X streamed
//   through shared memory by TMA in 128 x 32 slabs and M, X stored by TMA.
// formb_bq (steps 1 and 2 fused): B = M + G converted in shared memory and fed to
//   the MMA of B Q, with its own warp roles (described where it is defined).
// The same gemm kernel, with operands split into three bf16 parts, runs the
// orthonormalisation's contractions: the Gram P0^T P0, the triangular apply P0 L^-T
// and the block products of the recursive factorisation.  Its epilogue and tile order
// come in variants fixed at compile time (a direct epilogue for short-K tiles, the
// lower triangle only for symmetric results), so that each launch carries only its own.
#include <cuda.h>

#include <cstdio>

#include "common.cuh"
#include "tc.h"
#include "tc_ptx.cuh"

namespace dion {
namespace tc {

constexpr int BM = 128;       // tile rows = TMEM lanes
constexpr int KCHUNK_SUMSQ = 8;  // K blocks per accumulation chunk of sums of squares
constexpr int EPI_LD = 17;       // row stride (floats) of the epilogue's staging blocks
constexpr int BK = 64;        // bf16 elements per 128-byte swizzle row
constexpr int NT = 256;       // threads per CTA
constexpr int UPD_BN = 128;   // update tile columns (acc uses 2 * UPD_BN TMEM columns)
constexpr int SLAB = 32;      // update epilogue slab width (fp32: 128 bytes)
constexpr int SLAB_STAGES = 2;
constexpr int UPD_STAGES = 2;

// ------------------------------------------------------------------ host: tensor maps
typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*,
                                  const cuuint64_t*, const cuuint64_t*, const cuuint32_t*,
                                  const cuuint32_t*, CUtensorMapInterleave, CUtensorMapSwizzle,
                                  CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

static EncodeTiledFn encode_fn() {
  static EncodeTiledFn fn = nullptr;
  if (!fn) {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) ==
            cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<EncodeTiledFn>(p);
  }
  return fn;
}

static thread_local char tl_map_error[256];

// 3-D map over a stack [d2][d1][d0] of row-major matrices, box {b0, b1, 1}.
static bool map3d(CUtensorMap* m, const void* base, bool bf16, uint64_t d0, uint64_t d1,
                  uint64_t d2, uint32_t b0, uint32_t b1) {
  EncodeTiledFn f = encode_fn();
  if (!f) {
    snprintf(tl_map_error, sizeof(tl_map_error), "cuTensorMapEncodeTiled unavailable");
    return false;
  }
  const uint64_t es = bf16 ? 2 : 4;
  cuuint64_t dims[3] = {d0, d1, d2};
  cuuint64_t strides[2] = {d0 * es, d0 * d1 * es};
  cuuint32_t box[3] = {b0, b1, 1};
  cuuint32_t estr[3] = {1, 1, 1};
  const CUresult r = f(m, bf16 ? CU_TENSOR_MAP_DATA_TYPE_BFLOAT16 : CU_TENSOR_MAP_DATA_TYPE_FLOAT32,
                       3, const_cast<void*>(base), dims, strides, box, estr,
                       CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                       CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  if (r != CUDA_SUCCESS) {
    snprintf(tl_map_error, sizeof(tl_map_error),
             "cuTensorMapEncodeTiled -> %d (base %p, dims %llu x %llu x %llu, box %u x %u, %s)",
             (int)r, base, (unsigned long long)d0, (unsigned long long)d1, (unsigned long long)d2,
             b0, b1, bf16 ? "bf16" : "fp32");
    return false;
  }
  return true;
}

// 3-D map over a block (d1 rows x d0 columns) of each matrix of a stack whose rows are
// ld elements apart and whose matrices are ms elements apart.
static bool map3d_block(CUtensorMap* m, const void* base, uint64_t d0, uint64_t d1, uint64_t d2,
                        uint64_t ld, uint64_t ms, uint32_t b0, uint32_t b1) {
  EncodeTiledFn f = encode_fn();
  if (!f) {
    snprintf(tl_map_error, sizeof(tl_map_error), "cuTensorMapEncodeTiled unavailable");
    return false;
  }
  cuuint64_t dims[3] = {d0, d1, d2};
  cuuint64_t strides[2] = {ld * 2, ms * 2};
  cuuint32_t box[3] = {b0, b1, 1};
  cuuint32_t estr[3] = {1, 1, 1};
  const CUresult r = f(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(base), dims,
                       strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
                       CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                       CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  if (r != CUDA_SUCCESS) {
    snprintf(tl_map_error, sizeof(tl_map_error),
             "cuTensorMapEncodeTiled -> %d (block base %p, %llu x %llu x %llu, ld %llu, box %u x %u)",
             (int)r, base, (unsigned long long)d0, (unsigned long long)d1, (unsigned long long)d2,
             (unsigned long long)ld, b0, b1);
    return false;
  }
  return true;
}

}  // namespace tc

const char* tc_map_error() { return tc::tl_map_error; }

namespace tc {

// Device limits of the first device asked (the library runs on B200s only), each
// initialised once, thread-safely, by its static local's initialiser.
static int smem_optin() {
  static const int bytes = [] {
    int dev = 0, b = 0;
    cudaGetDevice(&dev);
    cudaDeviceGetAttribute(&b, cudaDevAttrMaxSharedMemoryPerBlockOptin, dev);
    return b > 0 ? b : 227 * 1024;
  }();
  return bytes;
}

static int sm_count() {
  static const int sms = [] {
    int dev = 0, n = 0;
    cudaGetDevice(&dev);
    cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev);
    return n > 0 ? n : 148;
  }();
  return sms;
}

// ------------------------------------------------------------------ device: timeouts
// Mark DION_MAT_TIMEOUT on every matrix owning a tile t, t + stride, ... < t_end
// (the tiles of this CTA it did not finish).
__device__ void mark_unfinished(int32_t* flags, int t, int t_end, int tiles_per_mat, int stride) {
  int last = -1;
  for (; t < t_end; t += stride) {
    const int b = t / tiles_per_mat;
    if (b != last) {
      atomicOr(flags + b, F_TIMEOUT);
      last = b;
    }
  }
}

// ------------------------------------------------------------------ batched GEMM
// C[b] = A[b] B[b] with fp32 accumulation in TMEM (SPLIT = 1), or, with SPLIT = 3,
// operands given as three bf16 parts (x = x0 + x1 + x2, each the bf16 rounding of
// what the earlier parts left over) and C = sum of the six products
// (0,0) (0,1) (1,0) (1,1) (0,2) (2,0), which reproduces an fp32 product to about
// 2^-24 relative: this keeps the Gram matrix and the triangular apply of Cholesky-QR
// fp32-accurate on bf16 tensor cores.  In split mode one pipeline stage holds the
// three parts of the A tile and of the B tile, and the six products are issued from
// shared memory.  A split operand is stored [3 * batch][rows][cols]: part i of
// matrix b is matrix i * batch + b.
struct GemmP {
  int64_t M, N, K;
  int batch, tiles_m, tiles_n, num_kb, block_n, stages;
  uint32_t idesc, a_bytes, b_bytes, tmem_cols, acc_stride;
  float* C;                          // fp32 result (may be null)
  int64_t ldc, c_bs;
  bf16* Cs;                          // three-way bf16 split of the result (may be null)
  int64_t cs_stride;                 // elements between the split parts
  int zplane_a, zplane_b;            // split operands: matrices between parts (0: batch)
  bf16* Cb;                          // bf16 copy of the result (may be null)
  float* colsq;                      // per-warp column sums of squares (may be null):
                                     // [batch][tiles_m * 4][N], row block tm*4 + warp
  float* devmax;                     // max |C_ij - I_ij| over j <= i, per matrix (may be
  int dev_stride;                    // null): atomic max into devmax[b * dev_stride]
  int c_trans;                       // store C transposed: C[j * ldc + i] (no Cs, Cb); colsq
                                     // then holds row sums of squares [batch][tiles_n][M]
  int m_fast;                        // tile order: M tiles of one N tile next to each other
  int tiles_mat;                     // tiles per matrix as enumerated (set by the launcher)
  int32_t* flags;
  int32_t need_mask, skip_mask;      // matrices whose flags fail this are skipped
  int lower_only;                    // skip tiles above the diagonal (symmetric results)
  int epi;                           // 0: C = acc;  1: C = alpha acc;  2: C += alpha acc
  float alpha;
  int kr;                            // triangular-operand K ranges (TC_KR_* bits)
  int kchunk;                        // K blocks per accumulation chunk (0: one chunk)
  int64_t max_spins;
};

// The tensor cores add each MMA's products into the fp32 accumulator with a rounding
// that is biased (toward zero): over thousands of MMAs the bias grows with K and, for
// sums of like-signed terms such as the diagonal of a Gram matrix, it does not average
// out (about 2.5e-5 relative at K = 4096 with six split products per step).  Long K
// ranges are therefore cut into chunks of kchunk blocks, each accumulated from zero in
// TMEM, and the epilogue adds the chunks in fp32 registers (round to nearest) into C.
// max that keeps a NaN (fmaxf would drop it)
__device__ __forceinline__ float max_keep_nan(float a, float b) {
  return (isnan(a) || isnan(b)) ? a + b : fmaxf(a, b);
}

__device__ __forceinline__ int n_chunks(const GemmP& p, int kb0, int kb1) {
  return p.kchunk > 0 ? (kb1 - kb0 + p.kchunk - 1) / p.kchunk : 1;
}

// K blocks [kb0, kb1) that can hold non-zero products for the tile at (m0, n0) when an
// operand is lower triangular (entries past the diagonal are zero and are not read).
__device__ __forceinline__ void k_range(const GemmP& p, int m0, int n0, int& kb0, int& kb1) {
  kb0 = 0;
  kb1 = p.num_kb;
  if (p.kr & TC_KR_B_LOWER_NK) kb1 = min(kb1, (n0 + p.block_n + BK - 1) / BK);
  if (p.kr & TC_KR_B_LOWER_KN) kb0 = n0 / BK;
  if (p.kr & TC_KR_A_LOWER_MK) kb1 = min(kb1, (m0 + BM + BK - 1) / BK);
  if (kb1 <= kb0) kb1 = kb0 + 1;  // never empty: a block past K loads as zeros
}

// row i of the lower triangle holding entry rem of its row-major enumeration:
// i (i + 1) / 2 <= rem < (i + 1) (i + 2) / 2
__device__ __forceinline__ int tri_row(int rem) {
  int i = (int)((sqrtf(8.f * (float)rem + 1.f) - 1.f) * 0.5f);
  while (i > 0 && i * (i + 1) / 2 > rem) --i;
  while ((i + 1) * (i + 2) / 2 <= rem) ++i;
  return i;
}

// M and N tile of tile rem within a matrix.  With a static tile schedule (tile t on CTA
// t mod grid) the enumeration decides what each CTA gets: listing the tiles above the
// diagonal of a symmetric result and skipping them left whole CTAs idle (grid and tiles
// per matrix share factors), so with TRI those tiles are not enumerated at all.
template <bool TRI = false>
__device__ __forceinline__ int tile_mi(const GemmP& p, int rem) {
  if constexpr (TRI) return tri_row(rem);
  return p.m_fast ? rem % p.tiles_m : rem / p.tiles_n;
}
template <bool TRI = false>
__device__ __forceinline__ int tile_ni(const GemmP& p, int rem) {
  if constexpr (TRI) {
    const int i = tri_row(rem);
    return rem - i * (i + 1) / 2;
  }
  return p.m_fast ? rem / p.tiles_m : rem % p.tiles_n;
}

__device__ __forceinline__ bool tile_active(const GemmP& p, int t, int tiles_per_mat) {
  if (p.lower_only) {
    const int rem = t % tiles_per_mat;
    if (tile_ni(p, rem) * p.block_n > tile_mi(p, rem) * BM) return false;
  }
  if (p.need_mask == 0 && p.skip_mask == 0) return true;
  const int32_t f = p.flags[t / tiles_per_mat];
  return (f & p.need_mask) == p.need_mask && !(f & p.skip_mask);
}

// Epilogue and tile-order variants, fixed at compile time so that each instantiation
// carries only its own code (the latency-bound long-K GEMMs are sensitive to it):
constexpr int GM_DIRECT = 1;  // rows leave the epilogue straight from registers as
                              // 16-byte vectors (no c_trans, no colsq; aligned C, Cb, Cs)
constexpr int GM_TRI = 2;     // tiles enumerated over the lower triangle (square grid)

template <bool A_MN, bool B_MN, int SPLIT, int MODE>
__global__ void __launch_bounds__(NT, 1)
    k_tc_gemm(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmB,
              const GemmP p) {
  constexpr bool DIRECT = (MODE & GM_DIRECT) != 0, TRI = (MODE & GM_TRI) != 0;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = align1024(smem_raw);
  const uint32_t stage_a = SPLIT * p.a_bytes, stage_b = SPLIT * p.b_bytes;
  uint8_t* sA = smem;
  uint8_t* sB = smem + (size_t)p.stages * stage_a;
  uint64_t* full = reinterpret_cast<uint64_t*>(sB + (size_t)p.stages * stage_b);
  uint64_t* empty = full + p.stages;
  uint64_t* tfull = empty + p.stages;
  uint64_t* tempty = tfull + 2;
  uint64_t* drain = tempty + 2;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(drain + 1);
  volatile int* abort = reinterpret_cast<volatile int*>(tmem_slot + 1);
  float* escr = reinterpret_cast<float*>(tmem_slot + 4);  // 4 warps x [32][EPI_LD]

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int tiles_per_mat = TRI ? p.tiles_mat : p.tiles_m * p.tiles_n;
  const int ntiles = p.batch * tiles_per_mat;

  if (threadIdx.x == 0) {
    for (int s = 0; s < p.stages; ++s) {
      mbar_init(full + s, 1);
      mbar_init(empty + s, 1);
    }
    for (int a = 0; a < 2; ++a) {
      mbar_init(tfull + a, 1);
      mbar_init(tempty + a, 4);
    }
    mbar_init(drain, 1);
    *abort = 0;
    fence_mbar_init();
  }
  if (warp == 2) {
    tmem_alloc(tmem_slot, p.tmem_cols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;

  if (warp == 0 && lane == 0) {
    // ---------------- TMA producer
    prefetch_map(&tmA);
    prefetch_map(&tmB);
    int stage = 0;
    uint32_t phase = 0;
    int used = 0;  // stages issued at least once
    for (int t = blockIdx.x; t < ntiles; t += gridDim.x) {
      if (!tile_active(p, t, tiles_per_mat)) continue;
      const int b = t / tiles_per_mat;
      const int rem = t % tiles_per_mat;
      const int m0 = tile_mi<TRI>(p, rem) * BM;
      const int n0 = tile_ni<TRI>(p, rem) * p.block_n;
      int kb0, kb1;
      k_range(p, m0, n0, kb0, kb1);
      bool ok = true;
      for (int kb = kb0; kb < kb1; ++kb) {
        if (!wait_bounded(empty + stage, phase ^ 1, p.max_spins, abort)) { ok = false; break; }
        mbar_expect_tx(full + stage, stage_a + stage_b);
        const int k0 = kb * BK;
#pragma unroll
        for (int part = 0; part < SPLIT; ++part) {
          uint8_t* a_dst = sA + (size_t)stage * stage_a + part * p.a_bytes;
          uint8_t* b_dst = sB + (size_t)stage * stage_b + part * p.b_bytes;
          const int za = part * p.zplane_a + b, zb = part * p.zplane_b + b;
          if (A_MN) {  // A^T stored [K][M]: boxes of 64 (M) x 64 (K)
            tma_load_3d(a_dst, &tmA, full + stage, m0, k0, za);
            tma_load_3d(a_dst + 8192, &tmA, full + stage, m0 + 64, k0, za);
          } else {     // A stored [M][K]: 128 rows of 64 K elements
            tma_load_3d(a_dst, &tmA, full + stage, k0, m0, za);
          }
          if (B_MN) {  // B stored [K][N]: boxes of 64 (N) x 64 (K)
            for (int j = 0; j < p.block_n / 64; ++j)
              tma_load_3d(b_dst + j * 8192, &tmB, full + stage, n0 + 64 * j, k0, zb);
          } else {     // B stored [N][K]: block_n rows of 64 K elements
            tma_load_3d(b_dst, &tmB, full + stage, k0, n0, zb);
          }
        }
        if (used < p.stages) ++used;
        if (++stage == p.stages) { stage = 0; phase ^= 1; }
      }
      if (!ok) break;
    }
    if (*abort) {
      // let every load already issued land before the CTA goes away
      for (int i = 0; i < used; ++i) {
        stage = (stage + p.stages - 1) % p.stages;
        if (stage == p.stages - 1) phase ^= 1;
        wait_drain(full + stage, phase);
      }
    }
  } else if (warp == 1 && lane == 0) {
    // ---------------- MMA issuer
    // split products, smallest terms first: (2,0) (0,2) (1,1) (1,0) (0,1) (0,0); with
    // two parts loaded (SPLIT = 2) only (1,0) (0,1) (0,0), about 2^-17 relative
    constexpr int NPROD = SPLIT == 3 ? 6 : (SPLIT == 2 ? 3 : 1);
    constexpr int P0 = SPLIT == 3 ? 0 : 3;  // first product of the table used
    const int pa[6] = {2, 0, 1, 1, 0, 0};
    const int pb[6] = {0, 2, 1, 0, 1, 0};
    int stage = 0;
    uint32_t phase = 0;
    int lt = 0;
    bool ok = true;
    for (int t = blockIdx.x; t < ntiles && ok; t += gridDim.x) {
      if (!tile_active(p, t, tiles_per_mat)) continue;
      const int rem = t % tiles_per_mat;
      int kb0, kb1;
      k_range(p, tile_mi<TRI>(p, rem) * BM, tile_ni<TRI>(p, rem) * p.block_n, kb0, kb1);
      const int nch = n_chunks(p, kb0, kb1);
      for (int ch = 0; ch < nch && ok; ++ch) {
      const int acc = lt & 1;
      const uint32_t acc_phase = (lt >> 1) & 1;
      if (!wait_bounded(tempty + acc, acc_phase ^ 1, p.max_spins, abort)) { ok = false; break; }
      tc_fence_after();
      const uint32_t d = tmem + acc * p.acc_stride;
      const int c0 = p.kchunk > 0 ? kb0 + ch * p.kchunk : kb0;
      const int c1 = p.kchunk > 0 ? min(kb1, c0 + p.kchunk) : kb1;
      for (int kb = c0; kb < c1; ++kb) {
        if (!wait_bounded(full + stage, phase, p.max_spins, abort)) { ok = false; break; }
        tc_fence_after();
        const uint32_t a_base = smem_u32(sA + (size_t)stage * stage_a);
        const uint32_t b_base = smem_u32(sB + (size_t)stage * stage_b);
#pragma unroll
        for (int k = 0; k < BK / 16; ++k) {
#pragma unroll
          for (int q = 0; q < NPROD; ++q) {
            const uint32_t ab = a_base + (SPLIT > 1 ? pa[P0 + q] : 0) * p.a_bytes;
            const uint32_t bb = b_base + (SPLIT > 1 ? pb[P0 + q] : 0) * p.b_bytes;
            const uint64_t ad = A_MN ? sw128_desc(ab + k * 2048, 8192, 1024)
                                     : sw128_desc(ab + k * 32, 16, 1024);
            const uint64_t bd = B_MN ? sw128_desc(bb + k * 2048, 8192, 1024)
                                     : sw128_desc(bb + k * 32, 16, 1024);
            mma_bf16(d, ad, bd, p.idesc, ((kb - c0) | k | q) != 0);
          }
        }
        mma_commit(empty + stage);
        if (++stage == p.stages) { stage = 0; phase ^= 1; }
      }
      if (!ok) break;
      mma_commit(tfull + acc);
      ++lt;
      }
    }
    mma_commit(drain);
    wait_drain(drain, 0);
  } else if (warp >= 4) {
    // ---------------- epilogue: TMEM -> shared -> global (fp32 and/or bf16 copies)
    // Each warp owns 32 rows.  A 32 x 16 block read from TMEM (lane = row) is passed
    // through shared memory so that global memory is touched row-contiguously: lane
    // l then holds columns 4 (l % 4) .. + 3 of rows l / 4 + 8 k, k < 4 (four lanes
    // write one row's 64 bytes).  Chunk 0 stores (or accumulates when p.epi == 2);
    // later chunks of the tile add into C; the copies Cb, Cs and the column sums of
    // squares are written from the final value, after the last chunk.
    const int ew = warp - 4;
    float* scr = escr + ew * 32 * EPI_LD;
    const int sub_r = lane >> 2, sub_c = (lane & 3) * 4;
    float dev = 0.f;  // max |C - I| over this warp's rows of the current tile (lower part)
    int lt = 0;
    int t = blockIdx.x;
    bool ok = true;
    for (; t < ntiles; t += gridDim.x) {
      if (!tile_active(p, t, tiles_per_mat)) continue;
      const int b = t / tiles_per_mat;
      const int rem = t % tiles_per_mat;
      const int64_t row0 = (int64_t)tile_mi<TRI>(p, rem) * BM + ew * 32;  // this warp's rows
      const int64_t n0 = (int64_t)tile_ni<TRI>(p, rem) * p.block_n;
      int kb0, kb1;
      k_range(p, tile_mi<TRI>(p, rem) * BM, (int)n0, kb0, kb1);
      float rsq = 0.f;  // transposed store: this lane's row sum of squares over the tile
      const int nch = n_chunks(p, kb0, kb1);
      // split operands: the chunks are added, in fp32 registers, into a running sum kept
      // in a third TMEM region (columns [2 block_n, 3 block_n), this thread's lane = its
      // row), and C is written once from the last chunk; otherwise each later chunk adds
      // into C in memory
      const bool tsum = SPLIT > 1 && nch > 1;
      const uint32_t sbase = tmem + ((uint32_t)(ew * 32) << 16) + 2 * p.acc_stride;
      for (int ch = 0; ch < nch; ++ch) {
        const int acc = lt & 1;
        const uint32_t acc_phase = (lt >> 1) & 1;
        if (!wait_bounded(tfull + acc, acc_phase, p.max_spins, abort)) { ok = false; break; }
        tc_fence_after();
        const int epi = (ch == 0 || tsum) ? p.epi : 2;
        const float alpha = p.epi == 0 ? 1.f : p.alpha;
        const bool last = ch == nch - 1;
        const uint32_t tbase = tmem + ((uint32_t)(ew * 32) << 16) + acc * p.acc_stride;
        for (int c = 0; c < p.block_n; c += 16) {
          float v[16];
          tmem_ld16(tbase + c, v);
          if (tsum && ch > 0) {
            float run[16];
            tmem_ld16(sbase + c, run);
            tmem_wait_ld();
#pragma unroll
            for (int q = 0; q < 16; ++q) v[q] += run[q];
          } else {
            tmem_wait_ld();
          }
          if (tsum && !last) {
            tmem_st16(sbase + c, v);
            continue;
          }
          if (n0 + c >= p.N) continue;  // uniform across the warp
          if constexpr (DIRECT) {
            // lane = row: its 16 consecutive columns go out as 16-byte vectors, with no
            // pass through shared memory (a short-K GEMM such as the triangular apply is
            // bound by this epilogue, not by its MMAs)
            const int64_t row = row0 + lane;
            if (row < p.M) {
              const int64_t at = (int64_t)b * p.c_bs + row * p.ldc + n0 + c;
              if (epi != 0) {
                float o[16];
#pragma unroll
                for (int j = 0; j < 4; ++j) {
                  float4 o4 = make_float4(0.f, 0.f, 0.f, 0.f);
                  if (epi == 2) o4 = reinterpret_cast<const float4*>(p.C + at)[j];
                  o[4 * j] = o4.x; o[4 * j + 1] = o4.y; o[4 * j + 2] = o4.z; o[4 * j + 3] = o4.w;
                }
#pragma unroll
                for (int q = 0; q < 16; ++q) v[q] = epi == 2 ? fmaf(alpha, v[q], o[q]) : alpha * v[q];
              }
              if (p.C) {
#pragma unroll
                for (int j = 0; j < 4; ++j)
                  reinterpret_cast<float4*>(p.C + at)[j] =
                      make_float4(v[4 * j], v[4 * j + 1], v[4 * j + 2], v[4 * j + 3]);
              }
              if (last && p.Cb) {
                __align__(16) bf16 h[16];
#pragma unroll
                for (int q = 0; q < 16; ++q) h[q] = __float2bfloat16_rn(v[q]);
                reinterpret_cast<uint4*>(p.Cb + at)[0] = reinterpret_cast<const uint4*>(h)[0];
                reinterpret_cast<uint4*>(p.Cb + at)[1] = reinterpret_cast<const uint4*>(h)[1];
              }
              if (last && p.Cs) {
                __align__(16) bf16 h[16], mi[16], lo[16];
#pragma unroll
                for (int q = 0; q < 16; ++q) split3_bf16(v[q], h[q], mi[q], lo[q]);
#pragma unroll
                for (int j = 0; j < 2; ++j) {
                  reinterpret_cast<uint4*>(p.Cs + at)[j] = reinterpret_cast<const uint4*>(h)[j];
                  reinterpret_cast<uint4*>(p.Cs + at + p.cs_stride)[j] =
                      reinterpret_cast<const uint4*>(mi)[j];
                  reinterpret_cast<uint4*>(p.Cs + at + 2 * p.cs_stride)[j] =
                      reinterpret_cast<const uint4*>(lo)[j];
                }
              }
              if (p.devmax && last) {
#pragma unroll
                for (int q = 0; q < 16; ++q) {
                  const int64_t col = n0 + c + q;
                  const float e = fabsf(v[q] - (col == row ? 1.f : 0.f));
                  if (col <= row) dev = max_keep_nan(dev, e);
                }
              }
            }
            continue;
          }
          if (p.c_trans) {
            // C[j][i]: for each column j the warp's 32 rows are 32 consecutive floats
            const int64_t row = row0 + lane;
            if (row < p.M) {
              float* dst = p.C + (int64_t)b * p.c_bs + (n0 + c) * p.ldc + row;
#pragma unroll
              for (int q = 0; q < 16; ++q)
                if (n0 + c + q < p.N) {
                  dst[q * p.ldc] = v[q];
                  rsq = fmaf(v[q], v[q], rsq);
                }
            }
            continue;
          }
#pragma unroll
          for (int q = 0; q < 16; ++q) scr[lane * EPI_LD + q] = v[q];
          __syncwarp();
          float sq[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
          for (int k = 0; k < 4; ++k) {
            const int rl = sub_r + 8 * k;
            const int64_t row = row0 + rl;
            float a[4];
#pragma unroll
            for (int j = 0; j < 4; ++j) a[j] = scr[rl * EPI_LD + sub_c + j];
            if (row < p.M) {
              const int64_t at = (int64_t)b * p.c_bs + row * p.ldc + n0 + c + sub_c;
              if (epi != 0) {
                float o[4] = {0.f, 0.f, 0.f, 0.f};
                if (epi == 2) {
                  const float4 o4 = *reinterpret_cast<const float4*>(p.C + at);
                  o[0] = o4.x; o[1] = o4.y; o[2] = o4.z; o[3] = o4.w;
                }
#pragma unroll
                for (int j = 0; j < 4; ++j) a[j] = epi == 2 ? fmaf(alpha, a[j], o[j]) : alpha * a[j];
              }
              if (p.C) *reinterpret_cast<float4*>(p.C + at) = make_float4(a[0], a[1], a[2], a[3]);
              if (last && p.Cb) {
                __align__(8) bf16 h[4];
#pragma unroll
                for (int j = 0; j < 4; ++j) h[j] = __float2bfloat16_rn(a[j]);
                *reinterpret_cast<uint2*>(p.Cb + at) = *reinterpret_cast<const uint2*>(h);
              }
              if (last && p.Cs) {
                __align__(8) bf16 h[4], mi[4], lo[4];
#pragma unroll
                for (int j = 0; j < 4; ++j) split3_bf16(a[j], h[j], mi[j], lo[j]);
                *reinterpret_cast<uint2*>(p.Cs + at) = *reinterpret_cast<const uint2*>(h);
                *reinterpret_cast<uint2*>(p.Cs + at + p.cs_stride) = *reinterpret_cast<const uint2*>(mi);
                *reinterpret_cast<uint2*>(p.Cs + at + 2 * p.cs_stride) =
                    *reinterpret_cast<const uint2*>(lo);
              }
#pragma unroll
              for (int j = 0; j < 4; ++j) sq[j] = fmaf(a[j], a[j], sq[j]);
              if (p.devmax && last) {
#pragma unroll
                for (int j = 0; j < 4; ++j) {
                  const int64_t col = n0 + c + sub_c + j;
                  const float e = fabsf(a[j] - (col == row ? 1.f : 0.f));
                  if (col <= row) dev = max_keep_nan(dev, e);
                }
              }
            }
          }
          if (p.colsq && last) {
            // column sums of squares over the warp's 32 rows in a fixed order: the
            // lane's four rows, then the eight lanes of one column group by butterfly
#pragma unroll
            for (int o = 4; o <= 16; o <<= 1)
#pragma unroll
              for (int j = 0; j < 4; ++j) sq[j] += __shfl_xor_sync(0xffffffffu, sq[j], o);
            if (lane < 4) {
              const int64_t rb = (int64_t)b * p.tiles_m * 4 + tile_mi<TRI>(p, rem) * 4 + ew;
              *reinterpret_cast<float4*>(p.colsq + rb * p.N + n0 + c + sub_c) =
                  make_float4(sq[0], sq[1], sq[2], sq[3]);
            }
          }
          __syncwarp();
        }
        if (tsum && !last) tmem_wait_st();  // the running sum is read back next chunk
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(tempty + acc);
        ++lt;
      }
      if (!ok) break;
      if (p.c_trans && p.colsq && row0 + lane < p.M)
        p.colsq[((int64_t)b * p.tiles_n + tile_ni<TRI>(p, rem)) * p.M + row0 + lane] = rsq;
      if (p.devmax) {
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) dev = max_keep_nan(dev, __shfl_xor_sync(0xffffffffu, dev, o));
        // non-negative floats order like their bits; a NaN is stored as the positive
        // quiet NaN, whose bits exceed every finite value's
        if (lane == 0 && !(dev <= 0.f))
          atomicMax(reinterpret_cast<int*>(p.devmax + (int64_t)b * p.dev_stride),
                    isnan(dev) ? 0x7fc00000 : __float_as_int(dev));
        dev = 0.f;
      }
    }
    if (t < ntiles && lane == 0) mark_unfinished(p.flags, t, ntiles, tiles_per_mat, gridDim.x);
  }
  __syncthreads();
  if (warp == 2) {
    tc_fence_after();
    tmem_dealloc(tmem, p.tmem_cols);
  }
}

static uint32_t pow2_cols(uint32_t c) {
  uint32_t v = 32;
  while (v < c) v <<= 1;
  return v;
}

template <bool A_MN, bool B_MN, int SPLIT>
static cudaError_t launch_gemm(const CUtensorMap& ma, const CUtensorMap& mb, GemmP p,
                               cudaStream_t s) {
  p.a_bytes = BM * BK * 2;
  p.b_bytes = (uint32_t)p.block_n * BK * 2;
  if (p.zplane_a == 0) p.zplane_a = p.batch;
  if (p.zplane_b == 0) p.zplane_b = p.batch;
  const size_t stage_bytes = (size_t)SPLIT * (p.a_bytes + p.b_bytes);
  int stages = (int)((200 * 1024) / stage_bytes);
  if (stages > 8) stages = 8;
  if (stages < 1) return cudaErrorInvalidValue;
  p.stages = stages;
  p.acc_stride = (uint32_t)p.block_n;
  // two accumulators, and with split operands over K chunks a third region for the
  // chunks' running sum
  p.tmem_cols = pow2_cols((SPLIT > 1 && p.kchunk > 0 ? 3 : 2) * p.block_n);
  if (p.tmem_cols > 512) return cudaErrorInvalidValue;
  // a symmetric result on a square grid of square tiles: enumerate the lower triangle
  const bool tri = p.lower_only && p.tiles_m == p.tiles_n && p.block_n == BM;
  // The direct epilogue pays where K is short (a tile's MMAs take less time than its
  // epilogue, as in the triangular apply) and in the Grams (measured: 2-7 % faster); over
  // a long K into a large result (B Q in split mode) the staged path's row-contiguous
  // stores were faster.  16 columns of a row start on a 16-byte boundary in C (fp32), Cb
  // and each part of Cs (bf16) when the pointers are 16-byte aligned and every offset is
  // a multiple of 8.
  auto al16 = [](const void* q) { return (reinterpret_cast<uintptr_t>(q) & 15) == 0; };
  const bool direct = (p.num_kb <= 8 || tri) && !p.c_trans && !p.colsq && p.ldc % 8 == 0 &&
                      p.c_bs % 8 == 0 && (!p.Cs || p.cs_stride % 8 == 0) && al16(p.C) &&
                      al16(p.Cb) && al16(p.Cs) && p.block_n % 16 == 0;
  if (tri) p.lower_only = 0;
  p.tiles_mat = tri ? p.tiles_m * (p.tiles_m + 1) / 2 : p.tiles_m * p.tiles_n;
  const size_t smem = 1024 + stages * stage_bytes + (2 * stages + 5) * 8 + 16 +
                      4 * 32 * EPI_LD * sizeof(float);
  auto kern = tri ? (direct ? k_tc_gemm<A_MN, B_MN, SPLIT, GM_DIRECT | GM_TRI>
                            : k_tc_gemm<A_MN, B_MN, SPLIT, GM_TRI>)
                  : (direct ? k_tc_gemm<A_MN, B_MN, SPLIT, GM_DIRECT>
                            : k_tc_gemm<A_MN, B_MN, SPLIT, 0>);
  // the device's limit rather than this launch's need: a launch captured into a graph
  // is checked against the attribute when the graph runs, after later launches of the
  // same kernel with other shapes may have set it
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       smem_optin());
  if (e != cudaSuccess) return e;
  if ((int)smem > smem_optin()) return cudaErrorInvalidValue;
  const int ntiles = p.batch * p.tiles_mat;
  const int grid = ntiles < sm_count() ? ntiles : sm_count();
  kern<<<grid, NT, smem, s>>>(ma, mb, p);
  return cudaGetLastError();
}

static int pick_block_n(int64_t r, int mult) {
  const int64_t tiles = (r + 255) / 256;
  int64_t bn = (r + tiles - 1) / tiles;
  bn = (bn + mult - 1) / mult * mult;
  return (int)bn;
}

}  // namespace tc

cudaError_t tc_gemm_bq(const void* Bg, const void* Qg, float* P0, bf16* P0s, int64_t plane,
                       int count, int64_t m, int64_t n, int64_t r, int64_t max_spins,
                       int32_t* flags, cudaStream_t s, int* nlaunch, bool* done) {
  using namespace tc;
  *nlaunch = 0;
  *done = false;
  const int bn = pick_block_n(r, 16);
  CUtensorMap ma, mb;
  if (!map3d(&ma, Bg, true, n, m, count, BK, BM)) return cudaSuccess;
  if (!map3d(&mb, Qg, true, n, r, count, BK, bn)) return cudaSuccess;
  GemmP p{};
  p.M = m; p.N = r; p.K = n;
  p.batch = count;
  p.block_n = bn;
  p.tiles_m = (int)((m + BM - 1) / BM);
  p.tiles_n = (int)((r + bn - 1) / bn);
  p.num_kb = (int)((n + BK - 1) / BK);
  p.idesc = idesc_bf16(BM, bn, false, false);
  p.C = P0; p.ldc = r; p.c_bs = m * r;
  p.Cs = P0s; p.cs_stride = plane > 0 ? plane : (int64_t)count * m * r;
  p.flags = flags;
  p.max_spins = max_spins;
  cudaError_t e = launch_gemm<false, false, 1>(ma, mb, p, s);
  if (e == cudaSuccess) { *done = true; *nlaunch = 1; }
  return e;
}

int tc_btp_col_splits(int64_t n) {
  return (int)((n + tc::pick_block_n(n, 64) - 1) / tc::pick_block_n(n, 64));
}

cudaError_t tc_gemm_btp(const void* Bg, const void* Pg, float* R, float* colsq, int count,
                        int64_t m, int64_t n, int64_t r, int64_t max_spins, int32_t* flags,
                        cudaStream_t s, int* nlaunch, bool* done) {
  using namespace tc;
  *nlaunch = 0;
  *done = false;
  // computed as R^T = P^T B: tiles of r x up to 256 columns of B (both operands read
  // MN-major), so each 48 KB stage brings 32 KB of B from DRAM (the stream this kernel
  // waits on) and 16 KB of P (L2-resident); the two r halves of a column block run on
  // neighbouring CTAs (tile order M-fast) and share B in L2; R is stored transposed
  const int bn = pick_block_n(n, 64);  // MN-major B: whole 64-wide atoms (zero-filled past n)
  CUtensorMap ma, mb;
  if (!map3d(&ma, Pg, true, r, m, count, 64, BK)) return cudaSuccess;
  if (!map3d(&mb, Bg, true, n, m, count, 64, BK)) return cudaSuccess;
  GemmP p{};
  p.M = r; p.N = n; p.K = m;
  p.batch = count;
  p.block_n = bn;
  p.tiles_m = (int)((r + BM - 1) / BM);
  p.tiles_n = (int)((n + bn - 1) / bn);
  p.num_kb = (int)((m + BK - 1) / BK);
  p.idesc = idesc_bf16(BM, bn, true, true);
  p.C = R; p.ldc = r; p.c_bs = n * r;
  p.c_trans = 1;
  p.m_fast = 1;
  p.colsq = colsq;
  p.flags = flags;
  p.max_spins = max_spins;
  cudaError_t e = launch_gemm<true, true, 1>(ma, mb, p, s);
  if (e == cudaSuccess) { *done = true; *nlaunch = 1; }
  return e;
}

// fp32 contractions on bf16 tensor cores: operands as three bf16 parts.
cudaError_t tc_gemm_bq_split(const bf16* Bs, const bf16* Qs, float* P0, bf16* P0s,
                             int64_t plane, int count, int64_t m, int64_t n, int64_t r,
                             int64_t max_spins, int32_t* flags, cudaStream_t s, int* nlaunch,
                             bool* done) {
  using namespace tc;
  *nlaunch = 0;
  *done = false;
  const int bn = r <= 128 ? (int)r : 128;   // three parts of A and B per stage
  CUtensorMap ma, mb;
  if (!map3d(&ma, Bs, true, n, m, 3 * (uint64_t)count, BK, BM)) return cudaSuccess;
  if (!map3d(&mb, Qs, true, n, r, 3 * (uint64_t)count, BK, bn)) return cudaSuccess;
  GemmP p{};
  p.M = m; p.N = r; p.K = n;
  p.batch = count;
  p.block_n = bn;
  p.tiles_m = (int)((m + BM - 1) / BM);
  p.tiles_n = (int)((r + bn - 1) / bn);
  p.num_kb = (int)((n + BK - 1) / BK);
  p.idesc = idesc_bf16(BM, bn, false, false);
  // K in chunks summed in fp32 registers: the tensor cores' biased accumulation would
  // otherwise cost about K / 16 * 6 * 2^-24 relative (1.8e-4 at K = 8192), far above the
  // split's 2^-24; the chunks' partial sums pass through the fp32 P0
  p.C = P0; p.ldc = r; p.c_bs = m * r;
  p.Cs = P0s; p.cs_stride = plane > 0 ? plane : (int64_t)count * m * r;
  p.kchunk = KCHUNK_SUMSQ;
  p.flags = flags;
  p.max_spins = max_spins;
  cudaError_t e = launch_gemm<false, false, 3>(ma, mb, p, s);
  if (e == cudaSuccess) { *done = true; *nlaunch = 1; }
  return e;
}

cudaError_t tc_gemm_btp_split(const bf16* Bs, const bf16* Ps, int zplane_p, float* R,
                              float* colsq, int count, int64_t m, int64_t n, int64_t r,
                              int64_t max_spins, int32_t* flags, cudaStream_t s, int* nlaunch,
                              bool* done) {
  using namespace tc;
  *nlaunch = 0;
  *done = false;
  const int bn = r <= 64 ? 64 : 128;        // MN-major B: whole 64-wide atoms
  CUtensorMap ma, mb;
  // P's parts may lie further apart than count matrices (a stack shared with other
  // buckets): part i of matrix b is matrix i * zplane_p + b
  const int zp = zplane_p > 0 ? zplane_p : count;
  if (!map3d(&ma, Bs, true, n, m, 3 * (uint64_t)count, 64, BK)) return cudaSuccess;
  if (!map3d(&mb, Ps, true, r, m, 2 * (uint64_t)zp + count, 64, BK)) return cudaSuccess;
  GemmP p{};
  p.M = n; p.N = r; p.K = m;
  p.batch = count;
  p.block_n = bn;
  p.tiles_m = (int)((n + BM - 1) / BM);
  p.tiles_n = (int)((r + bn - 1) / bn);
  p.num_kb = (int)((m + BK - 1) / BK);
  p.idesc = idesc_bf16(BM, bn, true, true);
  p.C = R; p.ldc = r; p.c_bs = n * r;
  p.colsq = colsq;
  p.zplane_b = zp;
  p.kchunk = KCHUNK_SUMSQ;  // unbiased accumulation over long K, as in B Q
  p.flags = flags;
  p.max_spins = max_spins;
  cudaError_t e = launch_gemm<true, true, 3>(ma, mb, p, s);
  if (e == cudaSuccess) { *done = true; *nlaunch = 1; }
  return e;
}

cudaError_t tc_gram(const bf16* Xs, float* W, bf16* Ws, float* devmax, int dev_stride, int count,
                    int64_t m, int64_t r, int32_t* flags, int32_t need, int32_t skip,
                    int64_t max_spins, cudaStream_t s, int* nlaunch, bool* done, int parts) {
  using namespace tc;
  *nlaunch = 0;
  *done = false;
  // 128 x 128 tiles of the symmetric result; only those on or below the diagonal
  const int bn = r <= 64 ? 64 : 128;
  CUtensorMap ma, mb;
  if (!map3d(&ma, Xs, true, r, m, 3 * (uint64_t)count, 64, BK)) return cudaSuccess;
  if (!map3d(&mb, Xs, true, r, m, 3 * (uint64_t)count, 64, BK)) return cudaSuccess;
  GemmP p{};
  p.M = r; p.N = r; p.K = m;
  p.batch = count;
  p.block_n = bn;
  p.tiles_m = (int)((r + BM - 1) / BM);
  p.tiles_n = (int)((r + bn - 1) / bn);
  p.num_kb = (int)((m + BK - 1) / BK);
  p.idesc = idesc_bf16(BM, bn, true, true);
  p.C = W; p.ldc = r; p.c_bs = r * r;
  p.Cs = Ws; p.cs_stride = (int64_t)count * r * r;
  p.flags = flags; p.need_mask = need; p.skip_mask = skip;
  p.lower_only = bn == BM;
  p.kchunk = KCHUNK_SUMSQ;  // the diagonal sums squares: keep the accumulation unbiased
  p.devmax = devmax; p.dev_stride = dev_stride;
  p.max_spins = max_spins;
  cudaError_t e = parts == 2 ? launch_gemm<true, true, 2>(ma, mb, p, s)
                             : launch_gemm<true, true, 3>(ma, mb, p, s);
  if (e == cudaSuccess) { *done = true; *nlaunch = 1; }
  return e;
}

cudaError_t tc_apply(const bf16* Xs, const bf16* Ls, float* Y, bf16* Ys, bf16* Yb, int count,
                     int64_t m, int64_t r, int32_t* flags, int32_t need, int32_t skip,
                     int64_t max_spins, cudaStream_t s, int* nlaunch, bool* done) {
  using namespace tc;
  *nlaunch = 0;
  *done = false;
  const int bn = r <= 128 ? (int)r : 128;   // three parts of A and B per stage
  CUtensorMap ma, mb;
  if (!map3d(&ma, Xs, true, r, m, 3 * (uint64_t)count, BK, BM)) return cudaSuccess;
  if (!map3d(&mb, Ls, true, r, r, 3 * (uint64_t)count, BK, bn)) return cudaSuccess;
  GemmP p{};
  p.M = m; p.N = r; p.K = r;
  p.batch = count;
  p.block_n = bn;
  p.tiles_m = (int)((m + BM - 1) / BM);
  p.tiles_n = (int)((r + bn - 1) / bn);
  p.num_kb = (int)((r + BK - 1) / BK);
  p.idesc = idesc_bf16(BM, bn, false, false);
  p.C = Y; p.ldc = r; p.c_bs = m * r;
  p.Cs = Ys; p.cs_stride = (int64_t)count * m * r;
  p.Cb = Yb;
  p.flags = flags; p.need_mask = need; p.skip_mask = skip;
  p.kr = TC_KR_B_LOWER_NK;  // L^-1 is lower triangular: column tile j needs k <= j only
  // column tiles have different K ranges: M-fast order spreads both kinds over every
  // CTA of the static schedule (N-fast with two column tiles and an even grid gave one
  // CTA in two only the long ones)
  p.m_fast = 1;
  p.max_spins = max_spins;
  cudaError_t e = launch_gemm<false, false, 3>(ma, mb, p, s);
  if (e == cudaSuccess) { *done = true; *nlaunch = 1; }
  return e;
}

cudaError_t tc_block_gemm(const TcBlockGemm& g, int count, int64_t r, int32_t* flags,
                          int32_t need, int32_t skip, int64_t max_spins, cudaStream_t s,
                          int* nlaunch, bool* done) {
  using namespace tc;
  *nlaunch = 0;
  *done = false;
  if (g.M <= 0 || g.N <= 0 || g.K <= 0 || (g.N % 16) != 0 || (g.accumulate && !g.C) ||
      (!g.C && !g.Cs))
    return cudaErrorInvalidValue;
  // whole 64-wide atoms for an MN-major B; 16-column granules otherwise
  const int bn = g.b_mn ? (g.N <= 64 ? 64 : 128) : (g.N <= 128 ? (int)g.N : 128);
  const uint64_t z = 3 * (uint64_t)count, rr = (uint64_t)r * r;
  CUtensorMap ma, mb;
  const bool ok =
      (g.a_mn ? map3d_block(&ma, g.A, g.M, g.K, z, r, rr, 64, BK)
              : map3d_block(&ma, g.A, g.K, g.M, z, r, rr, BK, BM)) &&
      (g.b_mn ? map3d_block(&mb, g.B, g.N, g.K, z, r, rr, 64, BK)
              : map3d_block(&mb, g.B, g.K, g.N, z, r, rr, BK, bn));
  if (!ok) return cudaSuccess;
  GemmP p{};
  p.M = g.M; p.N = g.N; p.K = g.K;
  p.batch = count;
  p.block_n = bn;
  p.tiles_m = (int)((g.M + BM - 1) / BM);
  p.tiles_n = (int)((g.N + bn - 1) / bn);
  p.num_kb = (int)((g.K + BK - 1) / BK);
  p.idesc = idesc_bf16(BM, bn, g.a_mn, g.b_mn);
  p.C = g.C; p.ldc = r; p.c_bs = r * r;
  p.Cs = g.Cs; p.cs_stride = (int64_t)count * r * r;
  p.flags = flags; p.need_mask = need; p.skip_mask = skip;
  p.lower_only = g.lower_only && bn == BM;
  p.epi = g.accumulate ? 2 : 1;
  p.alpha = g.alpha;
  p.kr = g.kr;
  p.m_fast = g.kr != 0;  // uneven K ranges by tile: mix them over the CTAs
  if (g.accumulate) p.kchunk = KCHUNK_SUMSQ;  // W22 -= L21 L21^T: squares on the diagonal
  p.max_spins = max_spins;
  cudaError_t e;
  if (g.a_mn && g.b_mn) e = launch_gemm<true, true, 3>(ma, mb, p, s);
  else if (g.a_mn) e = launch_gemm<true, false, 3>(ma, mb, p, s);
  else if (g.b_mn) e = launch_gemm<false, true, 3>(ma, mb, p, s);
  else e = launch_gemm<false, false, 3>(ma, mb, p, s);
  if (e == cudaSuccess) { *done = true; *nlaunch = 1; }
  return e;
}

namespace tc {

// ------------------------------------------------------------------ fused B = M + G, P0 = B Q
// Steps 1 and 2 in one pass over M and G: TMA stages fp32 tiles of M and G, four
// converter warps (a row each) add them, round to bf16 and write the K-major,
// 128-byte-swizzled A operand of the MMA; the same shared-memory bytes are stored by
// TMA as bf16 B for the later B^T P.  B is read from HBM once (8 bytes per element)
// and written once (2 bytes); nothing re-reads it for B Q.
//   warp 0       TMA: M, G (fp32, 2 boxes of 32 columns each)
//   warp 1       MMA issuer
//   warp 2       TMEM allocator
//   warp 3       TMA: the Q^T tile (apart from M and G, so that a stage's fp32 staging
//                is refilled as soon as the converters are done with it, without
//                waiting for the MMA to release the stage's Q^T)
//   warps 4..7   epilogue: P0's three-way bf16 split
//   warps 8..11  converters
// Tiles of the fused kernel come in order from a global counter through a ring of
// FB_TILE_RING ids in shared memory: dealt round-robin instead, CTAs drift apart over a
// long launch and stop sharing DRAM pages.
constexpr int FB_TILE_RING = 4;
constexpr int FB_STAGES = 2;
constexpr int FB_NT = 384;
constexpr uint32_t FB_F32_BYTES = 2 * 2 * BM * 32 * 4;  // M and G, two 32-column boxes: 64 KB
constexpr uint32_t FB_A_BYTES = BM * BK * 2;             // 16 KB

struct FusedP {
  int64_t m, n, r;
  int batch, tiles_m, tiles_n, num_kb, block_n;
  uint32_t idesc, b_bytes, tmem_cols;
  bf16* P0s;
  int64_t cs_stride;
  int32_t* flags;
  int* tile_counter;  // zero before the launch; tiles are taken from it in order
  int64_t max_spins;
};
// consumers of the fused kernel's tile ring: the Q^T producer, the MMA issuer, four
// converter warps, four epilogue warps (the M, G producer fills it)
constexpr int FB_RING_CONSUMERS = 10;

__global__ void __launch_bounds__(FB_NT, 1)
    k_tc_formb_bq(const __grid_constant__ CUtensorMap tmM, const __grid_constant__ CUtensorMap tmG,
                  const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmBs,
                  const FusedP p) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = align1024(smem_raw);
  uint8_t* sF = smem;                                  // [stage][M box0 | M box1 | G box0 | G box1]
  uint8_t* sA = sF + FB_STAGES * FB_F32_BYTES;         // [stage] bf16 A tile
  uint8_t* sB = sA + FB_STAGES * FB_A_BYTES;           // [stage] Q^T tile
  uint64_t* f_full = reinterpret_cast<uint64_t*>(sB + FB_STAGES * p.b_bytes);
  uint64_t* f_empty = f_full + FB_STAGES;
  uint64_t* b_full = f_empty + FB_STAGES;
  uint64_t* b_empty = b_full + FB_STAGES;
  uint64_t* a_full = b_empty + FB_STAGES;
  uint64_t* a_empty = a_full + FB_STAGES;
  uint64_t* tfull = a_empty + FB_STAGES;
  uint64_t* tempty = tfull + 2;
  uint64_t* drain = tempty + 2;
  uint64_t* ring_full = drain + 1;
  uint64_t* ring_empty = ring_full + FB_TILE_RING;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(ring_empty + FB_TILE_RING);
  volatile int* abort = reinterpret_cast<volatile int*>(tmem_slot + 1);
  volatile int* ring = reinterpret_cast<volatile int*>(tmem_slot + 2);  // FB_TILE_RING tile ids

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int tiles_per_mat = p.tiles_m * p.tiles_n;
  const int ntiles = p.batch * tiles_per_mat;

  if (threadIdx.x == 0) {
    for (int s = 0; s < FB_STAGES; ++s) {
      mbar_init(f_full + s, 1);
      mbar_init(f_empty + s, 4);
      mbar_init(b_full + s, 1);
      mbar_init(b_empty + s, 1);
      mbar_init(a_full + s, 4);
      mbar_init(a_empty + s, 1);
    }
    for (int a = 0; a < 2; ++a) {
      mbar_init(tfull + a, 1);
      mbar_init(tempty + a, 4);
    }
    mbar_init(drain, 1);
    for (int s = 0; s < FB_TILE_RING; ++s) {
      mbar_init(ring_full + s, 1);
      mbar_init(ring_empty + s, FB_RING_CONSUMERS);
    }
    *abort = 0;
    fence_mbar_init();
  }
  // next tile id from the ring (-1: none left); a warp-wide call when `warp_wide`
  int ring_slot = 0;
  uint32_t ring_phase = 0;
  auto next_tile = [&](bool warp_wide) -> int {
    int t = -2;
    if (!warp_wide || lane == 0) {
      if (wait_bounded(ring_full + ring_slot, ring_phase, p.max_spins, abort)) {
        t = ring[ring_slot];
        mbar_arrive(ring_empty + ring_slot);
      }
    }
    if (warp_wide) t = __shfl_sync(0xffffffffu, t, 0);
    if (++ring_slot == FB_TILE_RING) { ring_slot = 0; ring_phase ^= 1; }
    return t;  // -2: gave up
  };
  if (warp == 2) {
    tmem_alloc(tmem_slot, p.tmem_cols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;

  if (warp == 0 && lane == 0) {
    // ---------------- TMA producer of M and G
    prefetch_map(&tmM);
    prefetch_map(&tmG);
    int stage = 0, used = 0, slot = 0;
    uint32_t phase = 0, rphase = 0;
    while (true) {
      // take the next tile in order and publish it to the other roles
      if (!wait_bounded(ring_empty + slot, rphase ^ 1, p.max_spins, abort)) break;
      int t = atomicAdd(p.tile_counter, 1);
      if (t >= ntiles) t = -1;
      ring[slot] = t;
      mbar_arrive(ring_full + slot);
      if (++slot == FB_TILE_RING) { slot = 0; rphase ^= 1; }
      if (t < 0) break;
      const int b = t / tiles_per_mat;
      const int rem = t % tiles_per_mat;
      const int m0 = (rem / p.tiles_n) * BM;
      bool ok = true;
      for (int kb = 0; kb < p.num_kb; ++kb) {
        if (!wait_bounded(f_empty + stage, phase ^ 1, p.max_spins, abort)) { ok = false; break; }
        const int k0 = kb * BK;
        uint8_t* f = sF + stage * FB_F32_BYTES;
        mbar_expect_tx(f_full + stage, FB_F32_BYTES);
        tma_load_3d(f, &tmM, f_full + stage, k0, m0, b);
        tma_load_3d(f + 16384, &tmM, f_full + stage, k0 + 32, m0, b);
        tma_load_3d(f + 32768, &tmG, f_full + stage, k0, m0, b);
        tma_load_3d(f + 49152, &tmG, f_full + stage, k0 + 32, m0, b);
        if (used < FB_STAGES) ++used;
        if (++stage == FB_STAGES) { stage = 0; phase ^= 1; }
      }
      if (!ok) break;
    }
    if (*abort)
      for (int i = 0; i < used; ++i) {
        stage = (stage + FB_STAGES - 1) % FB_STAGES;
        if (stage == FB_STAGES - 1) phase ^= 1;
        wait_drain(f_full + stage, phase);
      }
  } else if (warp == 3 && lane == 0) {
    // ---------------- TMA producer of the Q^T tiles
    prefetch_map(&tmQ);
    int stage = 0, used = 0;
    uint32_t phase = 0;
    for (int t = next_tile(false); t >= 0; t = next_tile(false)) {
      const int b = t / tiles_per_mat;
      const int n0 = (t % tiles_per_mat % p.tiles_n) * p.block_n;
      bool ok = true;
      for (int kb = 0; kb < p.num_kb; ++kb) {
        if (!wait_bounded(b_empty + stage, phase ^ 1, p.max_spins, abort)) { ok = false; break; }
        mbar_expect_tx(b_full + stage, p.b_bytes);
        tma_load_3d(sB + stage * p.b_bytes, &tmQ, b_full + stage, kb * BK, n0, b);
        if (used < FB_STAGES) ++used;
        if (++stage == FB_STAGES) { stage = 0; phase ^= 1; }
      }
      if (!ok) break;
    }
    if (*abort)
      for (int i = 0; i < used; ++i) {
        stage = (stage + FB_STAGES - 1) % FB_STAGES;
        if (stage == FB_STAGES - 1) phase ^= 1;
        wait_drain(b_full + stage, phase);
      }
  } else if (warp == 1 && lane == 0) {
    // ---------------- MMA issuer
    int stage = 0, lt = 0;
    uint32_t phase = 0;
    for (int t = next_tile(false); t >= 0; t = next_tile(false), ++lt) {
      const int acc = lt & 1;
      if (!wait_bounded(tempty + acc, ((lt >> 1) & 1) ^ 1, p.max_spins, abort)) break;
      tc_fence_after();
      const uint32_t d = tmem + acc * p.block_n;
      bool ok = true;
      for (int kb = 0; kb < p.num_kb; ++kb) {
        if (!wait_bounded(b_full + stage, phase, p.max_spins, abort) ||
            !wait_bounded(a_full + stage, phase, p.max_spins, abort)) { ok = false; break; }
        tc_fence_after();
        const uint32_t a_base = smem_u32(sA + stage * FB_A_BYTES);
        const uint32_t b_base = smem_u32(sB + stage * p.b_bytes);
#pragma unroll
        for (int k = 0; k < BK / 16; ++k)
          mma_bf16(d, sw128_desc(a_base + k * 32, 16, 1024), sw128_desc(b_base + k * 32, 16, 1024),
                   p.idesc, (kb | k) != 0);
        mma_commit(b_empty + stage);
        mma_commit(a_empty + stage);
        if (++stage == FB_STAGES) { stage = 0; phase ^= 1; }
      }
      if (!ok) break;
      mma_commit(tfull + acc);
    }
    mma_commit(drain);
    wait_drain(drain, 0);
  } else if (warp >= 8) {
    // ---------------- converters: row = lane of this warp's 32-row quarter
    const int cw = warp - 8;
    const int row = cw * 32 + lane;
    int stage = 0;
    uint32_t phase = 0;
    for (int t = next_tile(true); t >= 0; t = next_tile(true)) {
      const int b = t / tiles_per_mat;
      const int rem = t % tiles_per_mat;
      const int m0 = (rem / p.tiles_n) * BM;
      bool ok = true;
      for (int kb = 0; kb < p.num_kb; ++kb) {
        // warp-uniform outcome: the tile ring is read with warp shuffles
        const bool w = wait_bounded(f_full + stage, phase, p.max_spins, abort) &&
                       wait_bounded(a_empty + stage, phase ^ 1, p.max_spins, abort);
        if (!__all_sync(0xffffffffu, w)) { ok = false; break; }
        // the store issued from this A stage two k-blocks ago must have read it
        if (lane == 0) asm volatile("cp.async.bulk.wait_group.read 1;" ::: "memory");
        __syncwarp();
        const uint8_t* f = sF + stage * FB_F32_BYTES + row * 128;
        uint8_t* a = sA + stage * FB_A_BYTES + row * 128;
        const int sw = row & 7;
#pragma unroll
        for (int c = 0; c < 8; ++c) {  // 8 output chunks of 8 bf16 = columns 8c .. 8c+7
          const int box = c >> 2;        // columns 0..31 in box 0, 32..63 in box 1
          const int c0 = (2 * c) & 7, c1 = (2 * c + 1) & 7;  // fp32 chunks inside the box
          const uint8_t* fm = f + box * 16384;
          const uint8_t* fg = f + 32768 + box * 16384;
          const float4 m0v = *reinterpret_cast<const float4*>(fm + ((c0 ^ sw) << 4));
          const float4 m1v = *reinterpret_cast<const float4*>(fm + ((c1 ^ sw) << 4));
          const float4 g0v = *reinterpret_cast<const float4*>(fg + ((c0 ^ sw) << 4));
          const float4 g1v = *reinterpret_cast<const float4*>(fg + ((c1 ^ sw) << 4));
          __nv_bfloat162 q0 = __floats2bfloat162_rn(m0v.x + g0v.x, m0v.y + g0v.y);
          __nv_bfloat162 q1 = __floats2bfloat162_rn(m0v.z + g0v.z, m0v.w + g0v.w);
          __nv_bfloat162 q2 = __floats2bfloat162_rn(m1v.x + g1v.x, m1v.y + g1v.y);
          __nv_bfloat162 q3 = __floats2bfloat162_rn(m1v.z + g1v.z, m1v.w + g1v.w);
          uint4 pk;
          pk.x = *reinterpret_cast<uint32_t*>(&q0);
          pk.y = *reinterpret_cast<uint32_t*>(&q1);
          pk.z = *reinterpret_cast<uint32_t*>(&q2);
          pk.w = *reinterpret_cast<uint32_t*>(&q3);
          *reinterpret_cast<uint4*>(a + ((c ^ sw) << 4)) = pk;
        }
        __syncwarp();
        if (lane == 0) mbar_arrive(f_empty + stage);  // fp32 staging free again
        fence_proxy_async_smem();
        __syncwarp();
        if (lane == 0) {
          mbar_arrive(a_full + stage);
          tma_store_3d(&tmBs, sA + stage * FB_A_BYTES + cw * 32 * 128, kb * BK, m0 + cw * 32, b);
          bulk_commit();
        }
        __syncwarp();
        if (++stage == FB_STAGES) { stage = 0; phase ^= 1; }
      }
      if (!ok) break;
    }
    if (lane == 0) bulk_wait0();
  } else if (warp >= 4) {
    // ---------------- epilogue: P0's three-way bf16 split
    const int ew = warp - 4;
    int lt = 0;
    bool ok = true;
    for (int t = next_tile(true); ; t = next_tile(true), ++lt) {
      if (t < 0) {
        ok = t == -1;
        break;
      }
      const int acc = lt & 1;
      const bool w = wait_bounded(tfull + acc, (lt >> 1) & 1, p.max_spins, abort);
      if (!__all_sync(0xffffffffu, w)) { ok = false; break; }  // warp-uniform
      tc_fence_after();
      const int b = t / tiles_per_mat;
      const int rem = t % tiles_per_mat;
      const int64_t row = (int64_t)(rem / p.tiles_n) * BM + ew * 32 + lane;
      const int64_t n0 = (int64_t)(rem % p.tiles_n) * p.block_n;
      const int64_t off = (int64_t)b * p.m * p.r + row * p.r;
      const uint32_t tbase = tmem + ((uint32_t)(ew * 32) << 16) + acc * p.block_n;
      for (int c = 0; c < p.block_n; c += 16) {
        float v[16];
        tmem_ld16(tbase + c, v);
        tmem_wait_ld();
        if (row < p.m && n0 + c < p.r) {
          __align__(16) bf16 h[16], mi[16], lo[16];
#pragma unroll
          for (int q = 0; q < 16; ++q) split3_bf16(v[q], h[q], mi[q], lo[q]);
          bf16* base = p.P0s + off + n0 + c;
          const uint4* sh = reinterpret_cast<const uint4*>(h);
          const uint4* sm = reinterpret_cast<const uint4*>(mi);
          const uint4* sl = reinterpret_cast<const uint4*>(lo);
          reinterpret_cast<uint4*>(base)[0] = sh[0];
          reinterpret_cast<uint4*>(base)[1] = sh[1];
          reinterpret_cast<uint4*>(base + p.cs_stride)[0] = sm[0];
          reinterpret_cast<uint4*>(base + p.cs_stride)[1] = sm[1];
          reinterpret_cast<uint4*>(base + 2 * p.cs_stride)[0] = sl[0];
          reinterpret_cast<uint4*>(base + 2 * p.cs_stride)[1] = sl[1];
        }
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(tempty + acc);
    }
    // tiles are handed out dynamically, so after a give-up every matrix is suspect
    if ((!ok || *abort) && lane == 0)
      for (int b = 0; b < p.batch; ++b) atomicOr(p.flags + b, F_TIMEOUT);
  }
  __syncthreads();
  if (warp == 2) {
    tc_fence_after();
    tmem_dealloc(tmem, p.tmem_cols);
  }
}

}  // namespace tc

cudaError_t tc_formb_bq(const float* M, const float* G, const void* Qg, void* Bg, bf16* P0s,
                        int64_t plane, int count, int64_t m, int64_t n, int64_t r,
                        int64_t max_spins, int32_t* flags, int* tile_counter, cudaStream_t s,
                        int* nlaunch, bool* done) {
  using namespace tc;
  *nlaunch = 0;
  *done = false;
  const int bn = pick_block_n(r, 16);
  CUtensorMap mM, mG, mQ, mBs;
  if (!map3d(&mM, M, false, n, m, count, 32, BM)) return cudaSuccess;
  if (!map3d(&mG, G, false, n, m, count, 32, BM)) return cudaSuccess;
  if (!map3d(&mQ, Qg, true, n, r, count, BK, bn)) return cudaSuccess;
  if (!map3d(&mBs, Bg, true, n, m, count, BK, 32)) return cudaSuccess;
  FusedP p{};
  p.m = m; p.n = n; p.r = r;
  p.batch = count;
  p.block_n = bn;
  p.tiles_m = (int)((m + BM - 1) / BM);
  p.tiles_n = (int)((r + bn - 1) / bn);
  p.num_kb = (int)((n + BK - 1) / BK);
  p.idesc = idesc_bf16(BM, bn, false, false);
  p.b_bytes = (uint32_t)bn * BK * 2;
  p.tmem_cols = pow2_cols(2 * bn);
  p.P0s = P0s;
  p.cs_stride = plane > 0 ? plane : (int64_t)count * m * r;
  p.flags = flags;
  p.tile_counter = tile_counter;
  p.max_spins = max_spins;
  const size_t smem = 1024 + FB_STAGES * (FB_F32_BYTES + FB_A_BYTES + p.b_bytes) +
                      (6 * FB_STAGES + 5 + 2 * FB_TILE_RING) * 8 + 16 + 4 * FB_TILE_RING;
  cudaError_t e = cudaFuncSetAttribute(k_tc_formb_bq, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       (int)smem);
  if (e != cudaSuccess) return e;
  const int ntiles = count * p.tiles_m * p.tiles_n;
  const int grid = ntiles < sm_count() ? ntiles : sm_count();
  k_tc_formb_bq<<<grid, FB_NT, smem, s>>>(mM, mG, mQ, mBs, p);
  e = cudaGetLastError();
  if (e == cudaSuccess) { *done = true; *nlaunch = 1; }
  return e;
}

namespace tc {

// ------------------------------------------------------------------ fused update
struct UpdP {
  int64_t m, n;
  int batch, tiles_m, tiles_n, num_kb;
  float omm, lrs;  // 1 - mu, lr * s
  int32_t* flags;
  int* tile_counter;  // zero before the launch; tiles are taken from it in order
  int npairs;         // 1: bf16 operands; 3: split operands, products (1,0) (0,1) (0,0)
  int pa[3], pb[3];   // part of P and of R, Q in each product
  int zplane_p;       // matrices between P's split parts
  int64_t max_spins;
  float* rmmc;        // [2][batch]: max |M' - M| and max |M| per matrix (max-ed into)
};

// Tiles are handed out in order from a global counter rather than dealt round-robin:
// CTAs then always work on neighbouring tiles (the same rows of M, G, X, so the same
// DRAM pages) however their speeds drift over a long launch.
constexpr int TILE_RING = 4;

constexpr uint32_t UPD_A_BYTES = BM * BK * 2;           // 16 KB
constexpr uint32_t UPD_B_BYTES = 2 * UPD_BN * BK * 2;   // 32 KB (R rows then Q rows)
constexpr uint32_t SLAB_BYTES = BM * SLAB * 4;          // 16 KB per tensor
// + one 128 x 32 staging slab each for M' and X', so a load slab is released as soon
// as it has been read, without waiting for the TMA store of the results
constexpr size_t UPD_SMEM = 1024 + UPD_STAGES * (UPD_A_BYTES + UPD_B_BYTES) +
                            SLAB_STAGES * 3 * SLAB_BYTES + 2 * SLAB_BYTES + 384;

__global__ void __launch_bounds__(NT, 1)
    k_tc_update(const __grid_constant__ CUtensorMap tmP, const __grid_constant__ CUtensorMap tmR,
                const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmM,
                const __grid_constant__ CUtensorMap tmG, const __grid_constant__ CUtensorMap tmX,
                const __grid_constant__ CUtensorMap tmMs, const __grid_constant__ CUtensorMap tmXs,
                const UpdP p) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = align1024(smem_raw);
  uint8_t* sA = smem;
  uint8_t* sB = sA + UPD_STAGES * UPD_A_BYTES;
  uint8_t* sS = sB + UPD_STAGES * UPD_B_BYTES;  // [stage][M | G | X] slabs
  uint8_t* sO = sS + SLAB_STAGES * 3 * SLAB_BYTES;  // staging of M' | X'
  uint64_t* full = reinterpret_cast<uint64_t*>(sO + 2 * SLAB_BYTES);
  uint64_t* empty = full + UPD_STAGES;
  uint64_t* sfull = empty + UPD_STAGES;
  uint64_t* sempty = sfull + SLAB_STAGES;
  uint64_t* tfull = sempty + SLAB_STAGES;
  uint64_t* tempty = tfull + 2;
  uint64_t* drain = tempty + 2;
  uint64_t* ring_full = drain + 1;
  uint64_t* ring_empty = ring_full + TILE_RING;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(ring_empty + TILE_RING);
  volatile int* abort = reinterpret_cast<volatile int*>(tmem_slot + 1);
  volatile int* ring = reinterpret_cast<volatile int*>(tmem_slot + 2);  // TILE_RING tile ids

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int tiles_per_mat = p.tiles_m * p.tiles_n;
  const int ntiles = p.batch * tiles_per_mat;
  constexpr int NSLAB = UPD_BN / SLAB;
  // consumers of the tile ring: slab producer, MMA issuer, four epilogue warps
  constexpr int RING_CONSUMERS = 6;


  if (threadIdx.x == 0) {
    for (int s = 0; s < UPD_STAGES; ++s) {
      mbar_init(full + s, 1);
      mbar_init(empty + s, 1);
    }
    for (int s = 0; s < SLAB_STAGES; ++s) {
      mbar_init(sfull + s, 1);
      mbar_init(sempty + s, 4);
    }
    for (int a = 0; a < 2; ++a) {
      mbar_init(tfull + a, 1);
      mbar_init(tempty + a, 4);
    }
    mbar_init(drain, 1);
    for (int s = 0; s < TILE_RING; ++s) {
      mbar_init(ring_full + s, 1);
      mbar_init(ring_empty + s, RING_CONSUMERS);
    }
    *abort = 0;
    fence_mbar_init();
  }
  if (warp == 3) {
    tmem_alloc(tmem_slot, 512);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;

  if (warp == 0 && lane == 0) {
    // ---------------- scheduler + operand producer: P tile and the R, Q rows of the tile
    prefetch_map(&tmP);
    prefetch_map(&tmR);
    prefetch_map(&tmQ);
    int stage = 0, used = 0, slot = 0;
    uint32_t phase = 0, rphase = 0;
    while (true) {
      if (!wait_bounded(ring_empty + slot, rphase ^ 1, p.max_spins, abort)) break;
      int t = atomicAdd(p.tile_counter, 1);
      if (t >= ntiles) t = -1;
      ring[slot] = t;
      mbar_arrive(ring_full + slot);  // publishes the tile id to the consumers
      if (++slot == TILE_RING) { slot = 0; rphase ^= 1; }
      if (t < 0) break;
      const int b = t / tiles_per_mat;
      const int rem = t % tiles_per_mat;
      const int m0 = (rem / p.tiles_n) * BM;
      const int n0 = (rem % p.tiles_n) * UPD_BN;
      bool ok = true;
      for (int it = 0; it < p.num_kb * p.npairs; ++it) {
        const int kb = it / p.npairs, pi = it % p.npairs;
        const int za = p.pa[pi] * p.zplane_p + b, zb = p.pb[pi] * p.batch + b;
        if (!wait_bounded(empty + stage, phase ^ 1, p.max_spins, abort)) { ok = false; break; }
        mbar_expect_tx(full + stage, UPD_A_BYTES + UPD_B_BYTES);
        uint8_t* a_dst = sA + stage * UPD_A_BYTES;
        uint8_t* b_dst = sB + stage * UPD_B_BYTES;
        tma_load_3d(a_dst, &tmP, full + stage, kb * BK, m0, za);
        tma_load_3d(b_dst, &tmR, full + stage, kb * BK, n0, zb);
        tma_load_3d(b_dst + UPD_BN * BK * 2, &tmQ, full + stage, kb * BK, n0, zb);
        if (used < UPD_STAGES) ++used;
        if (++stage == UPD_STAGES) { stage = 0; phase ^= 1; }
      }
      if (!ok) break;
    }
    if (*abort)
      for (int i = 0; i < used; ++i) {
        stage = (stage + UPD_STAGES - 1) % UPD_STAGES;
        if (stage == UPD_STAGES - 1) phase ^= 1;
        wait_drain(full + stage, phase);
      }
  } else if (warp == 2 && lane == 0) {
    // ---------------- slab producer: M, G, X in 128 x 32 fp32 slabs
    prefetch_map(&tmM);
    prefetch_map(&tmG);
    prefetch_map(&tmX);
    int stage = 0, used = 0, slot = 0;
    uint32_t phase = 0, rphase = 0;
    while (true) {
      if (!wait_bounded(ring_full + slot, rphase, p.max_spins, abort)) break;
      const int t = ring[slot];
      mbar_arrive(ring_empty + slot);
      if (++slot == TILE_RING) { slot = 0; rphase ^= 1; }
      if (t < 0) break;
      const int b = t / tiles_per_mat;
      const int rem = t % tiles_per_mat;
      const int m0 = (rem / p.tiles_n) * BM;
      const int n0 = (rem % p.tiles_n) * UPD_BN;
      bool ok = true;
      for (int sl = 0; sl < NSLAB; ++sl) {
        if (!wait_bounded(sempty + stage, phase ^ 1, p.max_spins, abort)) { ok = false; break; }
        mbar_expect_tx(sfull + stage, 3 * SLAB_BYTES);
        uint8_t* dst = sS + stage * 3 * SLAB_BYTES;
        const int c0 = n0 + sl * SLAB;
        tma_load_3d(dst, &tmM, sfull + stage, c0, m0, b);
        tma_load_3d(dst + SLAB_BYTES, &tmG, sfull + stage, c0, m0, b);
        tma_load_3d(dst + 2 * SLAB_BYTES, &tmX, sfull + stage, c0, m0, b);
        if (used < SLAB_STAGES) ++used;
        if (++stage == SLAB_STAGES) { stage = 0; phase ^= 1; }
      }
      if (!ok) break;
    }
    if (*abort)
      for (int i = 0; i < used; ++i) {
        stage = (stage + SLAB_STAGES - 1) % SLAB_STAGES;
        if (stage == SLAB_STAGES - 1) phase ^= 1;
        wait_drain(sfull + stage, phase);
      }
  } else if (warp == 1 && lane == 0) {
    // ---------------- MMA issuer: acc = P [R | Q]^T, M = 128, N = 256
    constexpr uint32_t idesc = idesc_bf16(BM, 2 * UPD_BN, false, false);
    int stage = 0, slot = 0;
    uint32_t phase = 0, rphase = 0;
    int lt = 0;
    for (;; ++lt) {
      if (!wait_bounded(ring_full + slot, rphase, p.max_spins, abort)) break;
      const int t = ring[slot];
      mbar_arrive(ring_empty + slot);
      if (++slot == TILE_RING) { slot = 0; rphase ^= 1; }
      if (t < 0) break;
      const int acc = lt & 1;
      if (!wait_bounded(tempty + acc, ((lt >> 1) & 1) ^ 1, p.max_spins, abort)) break;
      tc_fence_after();
      const uint32_t d = tmem + acc * 256;
      bool ok = true;
      for (int it = 0; it < p.num_kb * p.npairs; ++it) {
        if (!wait_bounded(full + stage, phase, p.max_spins, abort)) { ok = false; break; }
        tc_fence_after();
        const uint32_t a_base = smem_u32(sA + stage * UPD_A_BYTES);
        const uint32_t b_base = smem_u32(sB + stage * UPD_B_BYTES);
#pragma unroll
        for (int k = 0; k < BK / 16; ++k)
          mma_bf16(d, sw128_desc(a_base + k * 32, 16, 1024), sw128_desc(b_base + k * 32, 16, 1024),
                   idesc, (it | k) != 0);
        mma_commit(empty + stage);
        if (++stage == UPD_STAGES) { stage = 0; phase ^= 1; }
      }
      if (!ok) break;
      mma_commit(tfull + acc);
    }
    mma_commit(drain);
    wait_drain(drain, 0);
  } else if (warp >= 4) {
    // ---------------- epilogue: one TMEM lane (tile row) per thread
    const int ew = warp - 4;
    const int row = ew * 32 + lane;  // row inside the tile
    int stage = 0, slot = 0;
    uint32_t phase = 0, rphase = 0;
    int lt = 0;
    bool ok = true;
    for (;; ++lt) {
      if (!wait_bounded(ring_full + slot, rphase, p.max_spins, abort)) { ok = false; break; }
      const int t = ring[slot];
      __syncwarp();
      if (lane == 0) mbar_arrive(ring_empty + slot);
      if (++slot == TILE_RING) { slot = 0; rphase ^= 1; }
      if (t < 0) break;
      const int acc = lt & 1;
      if (!wait_bounded(tfull + acc, (lt >> 1) & 1, p.max_spins, abort)) { ok = false; break; }
      tc_fence_after();
      const int b = t / tiles_per_mat;
      const int rem = t % tiles_per_mat;
      const int m0 = (rem / p.tiles_n) * BM;
      const int n0 = (rem % p.tiles_n) * UPD_BN;
      const uint32_t tbase = tmem + ((uint32_t)(ew * 32) << 16) + acc * 256;
      // momentum-change statistics of the tile (out-of-range rows and columns load as
      // zeros and change by zero, so they do not count)
      float dmax = 0.f, mmax = 0.f;
      for (int sl = 0; sl < NSLAB; ++sl) {
        float ar[32], aq[32];
        tmem_ld32(tbase + sl * SLAB, ar);
        tmem_ld32(tbase + UPD_BN + sl * SLAB, aq);
        tmem_wait_ld();
        if (!wait_bounded(sfull + stage, phase, p.max_spins, abort)) { ok = false; break; }
        uint8_t* slab = sS + stage * 3 * SLAB_BYTES;
        const uint8_t* rm = slab + row * 128;
        const uint8_t* rg = slab + SLAB_BYTES + row * 128;
        const uint8_t* rx = slab + 2 * SLAB_BYTES + row * 128;
        uint8_t* om = sO + row * 128;
        uint8_t* ox = sO + SLAB_BYTES + row * 128;
        // this warp's previous store must have finished reading its staging rows
        if (lane == 0) bulk_wait_read0();
        __syncwarp();
#pragma unroll
        for (int c = 0; c < 8; ++c) {
          const int off = ((c ^ (row & 7)) << 4);
          float4 mv = *reinterpret_cast<const float4*>(rm + off);
          const float4 gv = *reinterpret_cast<const float4*>(rg + off);
          float4 xv = *reinterpret_cast<const float4*>(rx + off);
          const float4 m_old = mv;
          mv.x = (mv.x + gv.x) - p.omm * ar[4 * c + 0];
          mv.y = (mv.y + gv.y) - p.omm * ar[4 * c + 1];
          mv.z = (mv.z + gv.z) - p.omm * ar[4 * c + 2];
          mv.w = (mv.w + gv.w) - p.omm * ar[4 * c + 3];
          dmax = fmaxf(dmax, fmaxf(fmaxf(fabsf(mv.x - m_old.x), fabsf(mv.y - m_old.y)),
                                   fmaxf(fabsf(mv.z - m_old.z), fabsf(mv.w - m_old.w))));
          mmax = fmaxf(mmax, fmaxf(fmaxf(fabsf(m_old.x), fabsf(m_old.y)),
                                   fmaxf(fabsf(m_old.z), fabsf(m_old.w))));
          xv.x = xv.x - p.lrs * aq[4 * c + 0];
          xv.y = xv.y - p.lrs * aq[4 * c + 1];
          xv.z = xv.z - p.lrs * aq[4 * c + 2];
          xv.w = xv.w - p.lrs * aq[4 * c + 3];
          *reinterpret_cast<float4*>(om + off) = mv;
          *reinterpret_cast<float4*>(ox + off) = xv;
        }
        __syncwarp();
        if (lane == 0) mbar_arrive(sempty + stage);  // the load slab is free again
        fence_proxy_async_smem();
        __syncwarp();
        if (lane == 0) {
          tma_store_3d(&tmMs, sO + ew * 32 * 128, n0 + sl * SLAB, m0 + ew * 32, b);
          tma_store_3d(&tmXs, sO + SLAB_BYTES + ew * 32 * 128, n0 + sl * SLAB, m0 + ew * 32, b);
          bulk_commit();
        }
        __syncwarp();
        if (++stage == SLAB_STAGES) { stage = 0; phase ^= 1; }
      }
      if (!ok) break;  // t stays on the unfinished tile
      for (int o = 16; o > 0; o >>= 1) {
        dmax = fmaxf(dmax, __shfl_xor_sync(0xffffffffu, dmax, o));
        mmax = fmaxf(mmax, __shfl_xor_sync(0xffffffffu, mmax, o));
      }
      if (lane == 0) {
        atomic_max_pos(p.rmmc + b, dmax);
        atomic_max_pos(p.rmmc + p.batch + b, mmax);
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(tempty + acc);
    }
    if (lane == 0) bulk_wait0();
    // tiles are handed out dynamically, so after a give-up every matrix is suspect
    if ((!ok || *abort) && lane == 0)
      for (int b = 0; b < p.batch; ++b) atomicOr(p.flags + b, F_TIMEOUT);
  }
  __syncthreads();
  if (warp == 3) {
    tc_fence_after();
    tmem_dealloc(tmem, 512);
  }
}

}  // namespace tc

cudaError_t tc_update(const void* Pg, int zplane_p, const void* Rg, const void* Qg, bool split,
                      const float* G, float* M, float* X, int count, int64_t m, int64_t n,
                      int64_t r, float mu, float lr_scale, int64_t max_spins, int32_t* flags,
                      int* tile_counter, float* rmmc, cudaStream_t s, int* nlaunch, bool* done) {
  using namespace tc;
  *nlaunch = 0;
  *done = false;
  CUtensorMap mP, mR, mQ, mM, mG, mX, mMs, mXs;
  const uint64_t zc = (split ? 3 : 1) * (uint64_t)count;
  const int zp = zplane_p > 0 ? zplane_p : count;  // matrices between P's split parts
  const uint64_t zcp = split ? 2 * (uint64_t)zp + count : (uint64_t)count;
  bool ok = map3d(&mP, Pg, true, r, m, zcp, BK, BM) && map3d(&mR, Rg, true, r, n, zc, BK, UPD_BN) &&
            map3d(&mQ, Qg, true, r, n, zc, BK, UPD_BN) &&
            map3d(&mM, M, false, n, m, count, SLAB, BM) && map3d(&mG, G, false, n, m, count, SLAB, BM) &&
            map3d(&mX, X, false, n, m, count, SLAB, BM) &&
            map3d(&mMs, M, false, n, m, count, SLAB, 32) && map3d(&mXs, X, false, n, m, count, SLAB, 32);
  if (!ok) return cudaSuccess;
  UpdP p{};
  p.m = m; p.n = n;
  p.batch = count;
  p.tiles_m = (int)((m + BM - 1) / BM);
  p.tiles_n = (int)((n + UPD_BN - 1) / UPD_BN);
  p.num_kb = (int)((r + BK - 1) / BK);
  p.omm = 1.f - mu;
  p.lrs = lr_scale;
  p.flags = flags;
  p.tile_counter = tile_counter;
  // split parts hi and mid carry about 17 bits: three products reach ~2^-17 relative
  p.npairs = split ? 3 : 1;
  p.pa[0] = split ? 1 : 0; p.pb[0] = 0;
  p.pa[1] = 0; p.pb[1] = split ? 1 : 0;
  p.pa[2] = 0; p.pb[2] = 0;
  p.zplane_p = zp;
  p.max_spins = max_spins;
  p.rmmc = rmmc;
  cudaError_t e = cudaFuncSetAttribute(k_tc_update, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       (int)UPD_SMEM);
  if (e != cudaSuccess) return e;
  const int ntiles = count * p.tiles_m * p.tiles_n;
  const int grid = ntiles < sm_count() ? ntiles : sm_count();
  k_tc_update<<<grid, NT, UPD_SMEM, s>>>(mP, mR, mQ, mM, mG, mX, mMs, mXs, p);
  e = cudaGetLastError();
  if (e == cudaSuccess) { *done = true; *nlaunch = 1; }
  return e;
}

}  // namespace dion

// C ABI of the batched Dion step (include/dion.h): argument checks, the
// shape-bucket plan and workspace layout, and the launch sequence of one step.
//
// Buckets stack same-shape matrices into [count, m, n] tensors so each kernel
// runs once per bucket over all of its matrices, as "DASH: Faster Shampoo via
// Batched Block Preconditioning and Efficient Inverse-Root Solvers"
// (Methodologie, section 1) stacks preconditioner blocks instead of looping.
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include <algorithm>
#include <cmath>
#include <cstdarg>
#include <cstdio>
#include <cstring>
#include <new>
#include <numeric>
#include <string>
#include <vector>

#include "../../include/dion.h"
#include "common.cuh"
#include "internal.h"
#include "tc.h"

namespace {

thread_local char tl_error[512];  // a fixed buffer: recording an error never allocates

dion_status fail(dion_status s, const char* fmt, ...) {
  va_list ap;
  va_start(ap, fmt);
  vsnprintf(tl_error, sizeof(tl_error), fmt, ap);
  va_end(ap);
  return s;
}

// No C++ exception crosses the C ABI: the entry points that allocate host memory (plans,
// events, streams, graphs) catch what escapes and report it.
template <class F>
dion_status guarded(const char* where, F&& f) {
  try {
    return f();
  } catch (const std::exception& e) {
    return fail(DION_ERR_HOST, "%s: host-side failure: %s", where, e.what());
  } catch (...) {
    return fail(DION_ERR_HOST, "%s: host-side failure", where);
  }
}

constexpr uint64_t kMagic = 0x44494f4e42323030ull;  // "DIONB200"
constexpr int64_t kMaxElems = int64_t(1) << 40;

size_t align_up(size_t v, size_t a) { return (v + a - 1) / a * a; }

struct Plan {
  int64_t m, n, r;
  int count;
  float scale;
  int64_t mat0;
  int nsplit;
  // row-sharded plans: this rank holds rows [row0, row0 + m) of m_full-row matrices
  // (m_full == m, row0 == 0 otherwise)
  int64_t m_full, row0;
  // the stack the bucket's orthonormalisation runs in: every bucket with the same m and
  // r shares one (its matrices at positions [stack_off, stack_off + count) of the
  // stack's `zplane` matrices; split parts of m x r arrays zplane * m * r elements apart)
  int group, stack_off, zplane;
  size_t off_Bg, off_Qg, off_P0, off_P, off_P2, off_Pg, off_W, off_Linv, off_dinv, off_R, off_Rg,
      off_Qng, off_part, off_flags, off_stats, off_P0s, off_Ps, off_Linvs, off_sched, off_Ws, off_Ts,
      off_gather, off_rmmc;
};

// A stack of the orthonormalisation: the buckets whose P has the same shape (m x r),
// whatever their n, stacked into one [count, m, r] batch.  `orth` is a plan of the whole
// stack (count = the members' counts summed) for the orthonormalisation's kernels.
struct OrthGroup {
  std::vector<int32_t> members;  // bucket indices, in bucket order
  Plan orth;
};

struct EventPair {
  cudaEvent_t a, b;
  int cls;
  int launches;  // kernel launches between the two records
};

}  // namespace

struct dion_ctx {
  uint64_t magic;
  dion_options opt;
  std::vector<Plan> plans;
  std::vector<OrthGroup> groups;
  size_t ws_bytes;
  int64_t total_mats;
  int32_t last_launches;
  int device_checked;  // device id verified as sm_100, -1 before
  bool profiling;
  std::vector<EventPair> events;
  size_t events_used;
  double prof_ms[DION_KCLASS_COUNT];
  int64_t prof_launches[DION_KCLASS_COUNT];
  // streams on which the buckets' orthonormalisations run side by side
  int side_device;
  std::vector<cudaStream_t> side;
  std::vector<cudaEvent_t> side_done;
  cudaEvent_t fork_ev;
  // per bucket: the shifted Cholesky-QR loop of the fallback (r > 256 on the tensor
  // path) as a CUDA graph with a conditional while node, built on first use for a
  // workspace and device and launched every step
  struct FbGraph {
    const void* ws;
    int device;
    cudaGraphExec_t exec;
  };
  std::vector<FbGraph> fb;
  cudaStream_t cap;  // stream the loop body is captured on
  int cap_device;
  // gradient uploads of dion_step_batched_from_host: a copy stream, an event when the
  // caller's stream lets the uploads start, one event per uploaded bucket
  int up_device;
  cudaStream_t up;
  cudaEvent_t up_start;
  std::vector<cudaEvent_t> up_done;
  // row-sharded plans: every bucket's Gram (W) and the per-bucket fallback counts lie
  // in one block, every bucket's R in another, so each exchange is one all-reduce
  bool sharded;
  size_t off_wblk, wblk_floats, off_ctrl, off_rblk, rblk_floats;
  // the sharded step in progress between dion_step_sharded_begin and its last
  // dion_step_sharded_continue
  struct ShardStep {
    int stage;
    std::vector<dion_bucket_ptrs> ptrs;
    float lr;
    char* ws;
    int32_t* d_status;
    cudaStream_t s;
    std::vector<float> ctrl;   // per bucket: matrices needing the gathered fallback
    int32_t gather_at;         // bucket whose gather is being exchanged
    int launches;
  } sh;
};

namespace {

bool valid(dion_handle h) { return h != nullptr && h->magic == kMagic; }

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

dion_status check_options(const dion_options& o) {
  if (!(o.mu >= 0.f && o.mu < 1.f)) return fail(DION_ERR_INVALID_ARG, "mu must be in [0, 1), got %g", o.mu);
  if (o.precision != DION_PREC_FP32 && o.precision != DION_PREC_BF16)
    return fail(DION_ERR_INVALID_ARG, "unknown precision %d", o.precision);
  if (o.orth_mode < DION_ORTH_AUTO || o.orth_mode > DION_ORTH_HOUSEHOLDER)
    return fail(DION_ERR_INVALID_ARG, "unknown orth_mode %d", o.orth_mode);
  if (!(o.fallback_cond > 1.f)) return fail(DION_ERR_INVALID_ARG, "fallback_cond must exceed 1");
  if (!(o.orth_tol >= 0.f)) return fail(DION_ERR_INVALID_ARG, "orth_tol must be >= 0");
  if (o.kernel_path != DION_PATH_TENSOR && o.kernel_path != DION_PATH_SIMT)
    return fail(DION_ERR_INVALID_ARG, "unknown kernel_path %d", o.kernel_path);
  if (o.max_wait_spins < 1) return fail(DION_ERR_INVALID_ARG, "max_wait_spins must be >= 1");
  if (std::isnan(o.rmmc_threshold))
    return fail(DION_ERR_INVALID_ARG, "rmmc_threshold is NaN");
  if (o.stack_orth != 0 && o.stack_orth != 1)
    return fail(DION_ERR_INVALID_ARG, "stack_orth must be 0 or 1");
  return DION_OK;
}

// Per-step record of kernel launches (host counter) and optional events.
struct StepCtx {
  dion_handle h;
  cudaStream_t s;      // the stream the current phase runs on
  int launches;
  int cur_cls;
  EventPair* open;
  int open_at;
  std::vector<int> p0s_ready;  // per bucket: P0's split was written by B Q
  bool sharded = false;        // R is a partial sum: column-norm partials from R itself
  std::vector<int> g_ready;    // per stack: P0's split was written by every member's B Q
};

void begin_cls(StepCtx& c, int cls) {
  c.cur_cls = cls;
  c.open = nullptr;
  if (!c.h->profiling) return;
  dion_handle h = c.h;
  if (h->events_used == h->events.size()) {
    EventPair ep{};
    if (cudaEventCreate(&ep.a) != cudaSuccess || cudaEventCreate(&ep.b) != cudaSuccess) return;
    h->events.push_back(ep);
  }
  EventPair& ep = h->events[h->events_used++];
  ep.cls = cls;
  ep.launches = 0;
  cudaEventRecord(ep.a, c.s);
  c.open = &ep;
  c.open_at = c.launches;
}

void end_cls(StepCtx& c) {
  if (c.open) {
    cudaEventRecord(c.open->b, c.s);
    c.open->launches = c.launches - c.open_at;
  }
  c.open = nullptr;
}

#define DION_LAUNCH(ctx, n, expr)                                                       \
  do {                                                                                  \
    cudaError_t e_ = (expr);                                                            \
    (ctx).launches += (n);                                                              \
    if (e_ != cudaSuccess) return fail(DION_ERR_CUDA, "%s: %s", #expr, cudaGetErrorString(e_)); \
  } while (0)

constexpr int kFbMaxRounds = 8;   // two iterations per round
constexpr int kFbRoundsSlot = 8;  // int of the bucket's scheduler area counting rounds

struct FbBufs {
  float *W, *Linv, *stats, *P;
  int32_t* flags;
  int* rounds;
  __nv_bfloat16 *P0s, *Ps, *Ws, *Ts, *Linvs;
};

// One step of the shifted Cholesky-QR iteration on `s`: A_{k+1} = A_k R^-1 from the
// split src into P (fp32) and the split dst.
dion_status fb_iteration(const Plan& p, const dion_options& o, const FbBufs& f,
                         const __nv_bfloat16* src, __nv_bfloat16* dst, cudaStream_t s) {
  const int32_t need = DION_MAT_FALLBACK;
  const int32_t skip = dion::F_SDONE | dion::F_SFAIL | DION_MAT_NONFINITE;
  int nl = 0;
  bool done = false;
  // The iterate is exactly the previous one times R^-1 (an upper-triangular matrix with
  // a positive diagonal) whatever R is, so the Gram's accuracy decides only how fast the
  // iteration converges, not its limit: two split parts (three products, about 2^-17,
  // far below the shift) serve, as they do for the second Cholesky-QR pass.  The test
  // max|A^T A - I| <= orth_tol is then read to about 1e-5 (orth_tol is 2e-5 against a
  // bound of 1e-4 on P).
  cudaError_t e = dion::tc_gram(src, f.W, f.Ws, nullptr, 0, p.count, p.m, p.r, f.flags, need, skip,
                                o.max_wait_spins, s, &nl, &done, 2);
  if (e != cudaSuccess || !done)
    return fail(DION_ERR_CUDA, "shifted iteration, Gram: %s",
                e != cudaSuccess ? cudaGetErrorString(e) : dion::tc_map_error());
  dion::CholArgs ca{};
  ca.W = f.W; ca.Linv = f.Linv; ca.Linvs = f.Linvs; ca.flags = f.flags; ca.stats = f.stats;
  ca.count = p.count; ca.r = p.r; ca.m = p.m; ca.pass = 3;
  ca.fallback_cond = o.fallback_cond; ca.orth_tol = o.orth_tol;
  const char* what = "";
  e = dion::launch_chol_inv_rec(ca, f.Ws, f.Ts, o.max_wait_spins, s, &nl, &done, &what);
  if (e != cudaSuccess || !done)
    return fail(DION_ERR_CUDA, "shifted iteration, factorisation (%s): %s", what,
                e != cudaSuccess ? cudaGetErrorString(e) : dion::tc_map_error());
  e = dion::tc_apply(src, f.Linvs, f.P, dst, nullptr, p.count, p.m, p.r, f.flags, need, skip,
                     o.max_wait_spins, s, &nl, &done);
  if (e != cudaSuccess || !done)
    return fail(DION_ERR_CUDA, "shifted iteration, apply: %s",
                e != cudaSuccess ? cudaGetErrorString(e) : dion::tc_map_error());
  e = dion::launch_fb_mark(f.flags, p.count, s);
  if (e != cudaSuccess) return fail(DION_ERR_CUDA, "shifted iteration: %s", cudaGetErrorString(e));
  return DION_OK;
}

// Graph: [start: reset the loop state, condition = some matrix needs the loop]
//        while (condition) { iteration P0s -> Ps; iteration Ps -> P0s; condition update }
// With no flagged matrix only the start kernel runs.
dion_status fb_build(dion_handle h, const Plan& p, const FbBufs& f, cudaGraphExec_t* out) {
  const dion_options& o = h->opt;
  cudaStream_t cs = h->cap;
  cudaGraph_t graph = nullptr;
  cudaGraphExec_t exec = nullptr;
  dion_status st = DION_OK;
  cudaError_t e = cudaGraphCreate(&graph, 0);
  if (e != cudaSuccess) return fail(DION_ERR_CUDA, "cudaGraphCreate: %s", cudaGetErrorString(e));
  auto bail = [&](const char* what, cudaError_t err) {
    cudaGraph_t junk = nullptr;
    cudaStreamCaptureStatus cst;
    if (cudaStreamIsCapturing(cs, &cst) == cudaSuccess && cst != cudaStreamCaptureStatusNone)
      cudaStreamEndCapture(cs, &junk);
    cudaGraphDestroy(graph);
    return st != DION_OK ? st : fail(DION_ERR_CUDA, "fallback graph, %s: %s", what, cudaGetErrorString(err));
  };
  cudaGraphConditionalHandle cond;
  e = cudaGraphConditionalHandleCreate(&cond, graph, 0, cudaGraphCondAssignDefault);
  if (e != cudaSuccess) return bail("conditional handle", e);
  e = cudaStreamBeginCaptureToGraph(cs, graph, nullptr, nullptr, 0, cudaStreamCaptureModeRelaxed);
  if (e != cudaSuccess) return bail("capture", e);
  e = dion::launch_fb_cond(f.flags, f.stats, p.count, cond, f.rounds, kFbMaxRounds, true, cs);
  if (e != cudaSuccess) return bail("start kernel", e);
  e = cudaStreamEndCapture(cs, &graph);
  if (e != cudaSuccess) return bail("end capture", e);
  cudaGraphNode_t first = nullptr;
  size_t nnodes = 1;
  e = cudaGraphGetNodes(graph, &first, &nnodes);
  if (e != cudaSuccess || nnodes != 1) return bail("start node", e);
  cudaGraphNodeParams cp{};
  cp.type = cudaGraphNodeTypeConditional;
  cp.conditional.handle = cond;
  cp.conditional.type = cudaGraphCondTypeWhile;
  cp.conditional.size = 1;
  cudaGraphNode_t loop = nullptr;
  e = cudaGraphAddNode(&loop, graph, &first, 1, &cp);
  if (e != cudaSuccess) return bail("while node", e);
  cudaGraph_t body = cp.conditional.phGraph_out[0];
  e = cudaStreamBeginCaptureToGraph(cs, body, nullptr, nullptr, 0, cudaStreamCaptureModeRelaxed);
  if (e != cudaSuccess) return bail("body capture", e);
  if ((st = fb_iteration(p, o, f, f.P0s, f.Ps, cs)) != DION_OK) return bail("body", cudaSuccess);
  if ((st = fb_iteration(p, o, f, f.Ps, f.P0s, cs)) != DION_OK) return bail("body", cudaSuccess);
  e = dion::launch_fb_cond(f.flags, f.stats, p.count, cond, f.rounds, kFbMaxRounds, false, cs);
  if (e != cudaSuccess) return bail("condition kernel", e);
  e = cudaStreamEndCapture(cs, &body);
  if (e != cudaSuccess) return bail("end body capture", e);
  e = cudaGraphInstantiate(&exec, graph, 0);
  cudaGraphDestroy(graph);
  if (e != cudaSuccess) return fail(DION_ERR_CUDA, "fallback graph instantiate: %s", cudaGetErrorString(e));
  *out = exec;
  return DION_OK;
}

// Launch bucket bi's loop on s, building its graph first if needed.  *launched is false
// when s is being captured by the caller (a graph with a conditional node is not
// nested then): the flagged matrices then go to Householder QR directly.
dion_status fb_launch(dion_handle h, int bi, const Plan& p, const void* ws, const FbBufs& f,
                      cudaStream_t s, bool* launched) {
  *launched = false;
  cudaStreamCaptureStatus cst;
  if (cudaStreamIsCapturing(s, &cst) != cudaSuccess || cst != cudaStreamCaptureStatusNone)
    return DION_OK;
  int dev = -1;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return fail(DION_ERR_CUDA, "cudaGetDevice: %s", cudaGetErrorString(e));
  if (h->cap && h->cap_device != dev) {
    cudaStreamDestroy(h->cap);
    h->cap = nullptr;
  }
  if (!h->cap) {
    e = cudaStreamCreateWithFlags(&h->cap, cudaStreamNonBlocking);
    if (e != cudaSuccess) return fail(DION_ERR_CUDA, "capture stream: %s", cudaGetErrorString(e));
    h->cap_device = dev;
  }
  if (h->fb.size() < h->plans.size()) h->fb.resize(h->plans.size(), dion_ctx::FbGraph{nullptr, -1, nullptr});
  dion_ctx::FbGraph& g = h->fb[bi];
  if (g.exec && (g.ws != ws || g.device != dev)) {
    cudaGraphExecDestroy(g.exec);
    g.exec = nullptr;
  }
  if (!g.exec) {
    dion_status st = fb_build(h, p, f, &g.exec);
    if (st != DION_OK) return st;
    g.ws = ws;
    g.device = dev;
  }
  e = cudaGraphLaunch(g.exec, s);
  if (e != cudaSuccess) return fail(DION_ERR_CUDA, "fallback graph launch: %s", cudaGetErrorString(e));
  *launched = true;
  return DION_OK;
}

// Phases of one step; each runs over every bucket before the next starts.
enum Phase { PH_INIT, PH_PREPQ, PH_FORMB, PH_BQ, PH_ORTH, PH_BTP, PH_COLNORM, PH_UPDATE,
             PH_STATUS, PH_COUNT };

dion_status run_bucket(StepCtx& c, int bi, int phase, const Plan& p, const dion_bucket_ptrs& bp,
                       float lr, char* ws, int32_t* d_status) {
  const dion_options& o = c.h->opt;
  const bool bf = o.precision == DION_PREC_BF16;
  const bool tensor = o.kernel_path == DION_PATH_TENSOR;
  const bool split = tensor && !bf;  // fp32 contractions from three-way bf16 splits
  void* Bg = ws + p.off_Bg;
  void* Qg = ws + p.off_Qg;
  float* P0 = reinterpret_cast<float*>(ws + p.off_P0);
  float* P = reinterpret_cast<float*>(ws + p.off_P);
  float* P2 = reinterpret_cast<float*>(ws + p.off_P2);
  // the GEMM copy of P: bf16 on the tensor path is the leading plane of P's three-way
  // split (both are P rounded to nearest bf16), the split itself in fp32 mode
  void* Pg = (bf && tensor) ? (void*)(ws + p.off_Ps)
             : (bf || split) ? (void*)(ws + p.off_Pg) : (void*)P;
  float* W = reinterpret_cast<float*>(ws + p.off_W);
  float* Linv = reinterpret_cast<float*>(ws + p.off_Linv);
  float* dinv = reinterpret_cast<float*>(ws + p.off_dinv);
  float* R = reinterpret_cast<float*>(ws + p.off_R);
  void* Rg = (bf || split) ? (void*)(ws + p.off_Rg) : (void*)R;
  void* Qng = (bf || split) ? (void*)(ws + p.off_Qng) : (void*)bp.Q;
  float* part = reinterpret_cast<float*>(ws + p.off_part);
  int32_t* flags = reinterpret_cast<int32_t*>(ws + p.off_flags);
  float* stats = reinterpret_cast<float*>(ws + p.off_stats);
  int* sched = reinterpret_cast<int*>(ws + p.off_sched);
  float* rmmc = reinterpret_cast<float*>(ws + p.off_rmmc);
  __nv_bfloat16* P0s = reinterpret_cast<__nv_bfloat16*>(ws + p.off_P0s);
  __nv_bfloat16* Ps = reinterpret_cast<__nv_bfloat16*>(ws + p.off_Ps);
  __nv_bfloat16* Linvs = reinterpret_cast<__nv_bfloat16*>(ws + p.off_Linvs);
  __nv_bfloat16* Ws = p.off_Ws ? reinterpret_cast<__nv_bfloat16*>(ws + p.off_Ws) : nullptr;
  __nv_bfloat16* Ts = p.off_Ts ? reinterpret_cast<__nv_bfloat16*>(ws + p.off_Ts) : nullptr;
  // PH_ORTH runs once per stack (bi is then the stack's index and p its plan)
  int& p0s_ready = phase == PH_ORTH ? c.g_ready[bi] : c.p0s_ready[bi];
  const int64_t plane_mr = (int64_t)p.zplane * p.m * p.r;  // between split parts of m x r
  const int64_t m = p.m, n = p.n, r = p.r;
  const int cnt = p.count;
  cudaStream_t s = c.s;

  if (phase == PH_INIT) {
    p0s_ready = 0;
    DION_LAUNCH(c, 1, dion::launch_init_flags(flags, stats, sched, rmmc, cnt,
                                              o.orth_mode == DION_ORTH_HOUSEHOLDER ? DION_MAT_FALLBACK : 0,
                                              s));
    // a stack of several buckets has counters of its own (the fallback loop's rounds)
    const OrthGroup& g = c.h->groups[p.group];
    if (g.members.size() > 1 && g.members[0] == bi)
      DION_LAUNCH(c, 1, dion::launch_init_flags(nullptr, nullptr,
                                                reinterpret_cast<int*>(ws + g.orth.off_sched),
                                                nullptr, 0, 0, s));
    return DION_OK;
  }

  // steps 1 and 2 fused on the tensor path when one N tile covers r: B = M + G is
  // formed in shared memory, fed to the MMA and stored once as bf16
  const bool fused_bq = tensor && bf && r <= 256;

  if (phase == PH_PREPQ) {
  begin_cls(c, DION_KCLASS_PREP_Q);
  if (split)
    DION_LAUNCH(c, 1, dion::launch_prep_q_split(bp.Q, Qg, cnt, n, r, s));
  else
    DION_LAUNCH(c, 1, dion::launch_prep_q(bp.Q, Qg, bf, cnt, n, r, s));
  end_cls(c);
  return DION_OK;
  }

  // step 1: B = M + G in the precision of the contractions
  if (phase == PH_FORMB && !fused_bq) {
    begin_cls(c, DION_KCLASS_FORM_B);
    if (split)
      DION_LAUNCH(c, 1, dion::launch_form_b_split(bp.M, bp.G, Bg, (int64_t)cnt * m * n, s));
    else
      DION_LAUNCH(c, 1, dion::launch_form_b(bp.M, bp.G, Bg, bf, (int64_t)cnt * m * n, s));
    end_cls(c);
  }

  // step 2: P0 = B Q
  if (phase == PH_BQ) {
  begin_cls(c, DION_KCLASS_GEMM_BQ);
  if (fused_bq) {
    int nl = 0;
    bool done = false;
    cudaError_t e = dion::tc_formb_bq(bp.M, bp.G, Qg, Bg, P0s, plane_mr, cnt, m, n, r,
                                      o.max_wait_spins, flags, sched + 1, s, &nl, &done);
    c.launches += nl;
    if (e != cudaSuccess) return fail(DION_ERR_CUDA, "tc_formb_bq: %s", cudaGetErrorString(e));
    if (!done) return fail(DION_ERR_CUDA, "tc_formb_bq: %s", dion::tc_map_error());
    p0s_ready = true;
  } else if (split) {
    int nl = 0;
    bool done = false;
    cudaError_t e = dion::tc_gemm_bq_split((const __nv_bfloat16*)Bg, (const __nv_bfloat16*)Qg, P0,
                                           P0s, plane_mr, cnt, m, n, r, o.max_wait_spins, flags,
                                           s, &nl, &done);
    c.launches += nl;
    if (e != cudaSuccess) return fail(DION_ERR_CUDA, "tc_gemm_bq_split: %s", cudaGetErrorString(e));
    if (!done) return fail(DION_ERR_CUDA, "tc_gemm_bq_split: %s", dion::tc_map_error());
    p0s_ready = true;
  } else {
    bool done = false;
    if (tensor && bf) {
      int nl = 0;
      // only the split of P0 is written: the orthonormalisation reads nothing else
      cudaError_t e = dion::tc_gemm_bq(Bg, Qg, nullptr, P0s, plane_mr, cnt, m, n, r,
                                       o.max_wait_spins, flags, s, &nl, &done);
      c.launches += nl;
      if (e != cudaSuccess) return fail(DION_ERR_CUDA, "tc_gemm_bq: %s", cudaGetErrorString(e));
      if (!done) return fail(DION_ERR_CUDA, "tc_gemm_bq: %s", dion::tc_map_error());
      p0s_ready = done;
    }
    if (!done) {
      dion::GemmDesc d{};
      d.A = {Bg, m * n, n, 1};
      d.B = {Qg, n * r, n, 1};
      d.C = P0; d.sCb = m * r; d.sCi = r; d.sCj = 1;
      d.M = (int)m; d.N = (int)r; d.K = (int)n; d.batch = cnt; d.alpha = 1.f;
      DION_LAUNCH(c, (cnt + 65534) / 65535, dion::launch_gemm_simt(d, bf, s));
    }
  }
  end_cls(c);
  return DION_OK;
  }

  // step 3: P = orth(P0) -- Cholesky-QR, optional second pass, Householder fallback
  if (phase == PH_ORTH) {
  begin_cls(c, DION_KCLASS_ORTH);
  {
    bool pg_ready = false;  // Pg already holds the first pass's P
    auto gram = [&](const float* src) {
      dion::GemmDesc d{};
      d.A = {src, m * r, 1, r};
      d.B = {src, m * r, 1, r};
      d.C = W; d.sCb = r * r; d.sCi = r; d.sCj = 1;
      d.M = (int)r; d.N = (int)r; d.K = (int)m; d.batch = cnt; d.alpha = 1.f;
      d.flags = flags; d.need_mask = 0; d.skip_mask = DION_MAT_FALLBACK;
      return d;
    };
    auto apply = [&](const float* src, float* dst, int32_t need) {
      dion::GemmDesc d{};
      d.A = {src, m * r, r, 1};
      d.B = {Linv, r * r, r, 1};
      d.C = dst; d.sCb = m * r; d.sCi = r; d.sCj = 1;
      d.M = (int)m; d.N = (int)r; d.K = (int)r; d.batch = cnt; d.alpha = 1.f;
      d.flags = flags; d.need_mask = need; d.skip_mask = DION_MAT_FALLBACK;
      return d;
    };
    const int gl = (cnt + 65534) / 65535;
    dion::CholArgs ca{};
    ca.W = W; ca.Linv = Linv; ca.dinv = dinv; ca.flags = flags; ca.stats = stats;
    ca.count = cnt; ca.r = r; ca.fallback_cond = o.fallback_cond;
    const int chol_launches = dion::chol_inv_launches(r);
    const int64_t mr = (int64_t)cnt * m * r;
    // tensor cores: Gram and triangular apply from three-way bf16 splits (fp32-accurate)
    int nl = 0;
    bool done = false;
    // checks the call that just returned e (nl and done were set by that call)
    auto tc_check = [&](cudaError_t e, const char* what) -> dion_status {
      c.launches += nl;
      if (e != cudaSuccess) return fail(DION_ERR_CUDA, "%s: %s", what, cudaGetErrorString(e));
      if (!done) return fail(DION_ERR_CUDA, "%s: %s", what, dion::tc_map_error());
      return DION_OK;
    };
    if (o.orth_mode != DION_ORTH_HOUSEHOLDER && tensor) {
      dion_status st;
      cudaError_t e;
      // L^-1 and its split (the factorisation writes both): one kernel for r <= 256,
      // the recursion on the tensor cores above
      ca.Linvs = Linvs;
      auto chol = [&]() -> dion_status {
        if (r <= 256) {
          DION_LAUNCH(c, 1, dion::launch_chol_inv(ca, s));
          return DION_OK;
        }
        const char* what = "";
        e = dion::launch_chol_inv_rec(ca, Ws, Ts, o.max_wait_spins, s, &nl, &done, &what);
        c.launches += nl;
        if (e != cudaSuccess)
          return fail(DION_ERR_CUDA, "recursive factorisation (%s): %s", what, cudaGetErrorString(e));
        if (!done) return fail(DION_ERR_CUDA, "recursive factorisation (%s): %s", what,
                               dion::tc_map_error());
        return DION_OK;
      };
      if (!p0s_ready) DION_LAUNCH(c, 1, dion::launch_split3(P0, P0s, mr, mr, s));
      e = dion::tc_gram(P0s, W, Ws, nullptr, 0, cnt, m, r, flags, 0, DION_MAT_FALLBACK,
                        o.max_wait_spins, s,
                        &nl, &done);
      if ((st = tc_check(e, "tc_gram")) != DION_OK) return st;
      ca.pass = 1; ca.orth_tol = o.orth_tol;
      if ((st = chol()) != DION_OK) return st;
      // the first pass writes P and its split, which is also the GEMM copy Pg (bf16:
      // the split's leading plane); the finalize then touches only the matrices that
      // took the second pass or the fallback
      __nv_bfloat16* P1s = split ? reinterpret_cast<__nv_bfloat16*>(Pg) : Ps;
      // only the split is written: every later reader of the first pass's P reads the
      // split, and dion_workspace_view rebuilds the fp32 P from it (exactly: the three
      // parts sum to the fp32 value); the matrices that take the second pass or the
      // fallback get their fp32 P from the finalize
      e = dion::tc_apply(P0s, Linvs, nullptr, P1s, nullptr, cnt, m, r, flags, 0,
                         DION_MAT_FALLBACK, o.max_wait_spins, s, &nl, &done);
      if ((st = tc_check(e, "tc_apply")) != DION_OK) return st;
      pg_ready = true;
      if (o.orth_mode != DION_ORTH_CHOLQR) {
        // the second pass's Gram also measures max|W - I| per matrix (statistics slot 2,
        // zero since the step began), so that its factorisation can skip matrices the
        // first pass left orthonormal without reading W
        // P1 is orthonormal to about cond(P0)^2 u already: its Gram needs only the two
        // leading parts of its split (three products, about 2^-17 relative, far below
        // orth_tol and below what the second factorisation needs)
        e = dion::tc_gram(P1s, W, Ws, r <= 256 ? stats + 2 : nullptr, dion::ST, cnt, m, r, flags,
                          0, DION_MAT_FALLBACK, o.max_wait_spins, s,
                          &nl, &done, 2);
        if ((st = tc_check(e, "tc_gram")) != DION_OK) return st;
        ca.pass = 2;
        ca.orth_tol = o.orth_mode == DION_ORTH_CHOLQR2 ? -1.f : o.orth_tol;
        ca.dev_ready = r <= 256 ? 1 : 0;
        if ((st = chol()) != DION_OK) return st;
        e = dion::tc_apply(P1s, Linvs, P2, nullptr, nullptr, cnt, m, r, flags, DION_MAT_CHOLQR2,
                           DION_MAT_FALLBACK, o.max_wait_spins, s, &nl, &done);
        if ((st = tc_check(e, "tc_apply")) != DION_OK) return st;
      }
    } else if (o.orth_mode != DION_ORTH_HOUSEHOLDER) {
      DION_LAUNCH(c, gl, dion::launch_gemm_simt(gram(P0), false, s));
      ca.pass = 1; ca.orth_tol = o.orth_tol;
      DION_LAUNCH(c, chol_launches, dion::launch_chol_inv(ca, s));
      DION_LAUNCH(c, gl, dion::launch_gemm_simt(apply(P0, P, 0), false, s));
      if (o.orth_mode != DION_ORTH_CHOLQR) {
        DION_LAUNCH(c, gl, dion::launch_gemm_simt(gram(P), false, s));
        ca.pass = 2;
        ca.orth_tol = o.orth_mode == DION_ORTH_CHOLQR2 ? -1.f : o.orth_tol;
        DION_LAUNCH(c, chol_launches, dion::launch_chol_inv(ca, s));
        DION_LAUNCH(c, gl, dion::launch_gemm_simt(apply(P, P2, DION_MAT_CHOLQR2), false, s));
      }
    }
    // matrices Cholesky-QR gave up on: r > 256 on the tensor path iterate shifted
    // Cholesky-QR (on the tensor cores); Householder QR takes the rest, one CTA each
    if (tensor && r > 256 && o.orth_mode != DION_ORTH_HOUSEHOLDER) {
      FbBufs fbb{W, Linv, stats, P, flags, sched + kFbRoundsSlot, P0s, Ps, Ws, Ts, Linvs};
      bool launched = false;
      dion_status fst = fb_launch(c.h, bi, p, ws, fbb, s, &launched);
      if (fst != DION_OK) return fst;
      c.launches += launched ? 1 : 0;
    }
    DION_LAUNCH(c, 1, dion::launch_householder(P0, p0s_ready ? P0s : nullptr, P2, P0, P, flags,
                                               cnt, m, r, s));
    DION_LAUNCH(c, 1, dion::launch_finalize_p(P2, Pg, bf ? 1 : (split ? 2 : 0), flags, cnt, m, r,
                                              P, pg_ready, s));
  }
  end_cls(c);
  return DION_OK;
  }

  // step 4: R = B^T P
  if (phase == PH_BTP) {
  begin_cls(c, DION_KCLASS_GEMM_BTP);
  {
    bool done = false;
    if (split) {
      int nl = 0;
      cudaError_t e = dion::tc_gemm_btp_split((const __nv_bfloat16*)Bg, (const __nv_bfloat16*)Pg,
                                              p.zplane, R, part, cnt, m, n, r, o.max_wait_spins,
                                              flags, s, &nl, &done);
      c.launches += nl;
      if (e != cudaSuccess)
        return fail(DION_ERR_CUDA, "tc_gemm_btp_split: %s", cudaGetErrorString(e));
      if (!done) return fail(DION_ERR_CUDA, "tc_gemm_btp_split: %s", dion::tc_map_error());
    } else if (tensor && bf) {
      int nl = 0;
      cudaError_t e = dion::tc_gemm_btp(Bg, Pg, R, part, cnt, m, n, r, o.max_wait_spins, flags, s,
                                        &nl, &done);
      c.launches += nl;
      if (e != cudaSuccess) return fail(DION_ERR_CUDA, "tc_gemm_btp: %s", cudaGetErrorString(e));
      if (!done) return fail(DION_ERR_CUDA, "tc_gemm_btp: %s", dion::tc_map_error());
    }
    if (!done) {
      dion::GemmDesc d{};
      d.A = {Bg, m * n, 1, n};
      d.B = {Pg, m * r, 1, r};
      d.C = R; d.sCb = n * r; d.sCi = r; d.sCj = 1;
      d.M = (int)n; d.N = (int)r; d.K = (int)m; d.batch = cnt; d.alpha = 1.f;
      DION_LAUNCH(c, (cnt + 65534) / 65535, dion::launch_gemm_simt(d, bf, s));
    }
  }
  end_cls(c);
  return DION_OK;
  }

  // step 6: Q = colnorm(R), plus the GEMM copies of R and Q for the update
  if (phase == PH_COLNORM) {
  begin_cls(c, DION_KCLASS_COLNORM);
  DION_LAUNCH(c, 2,
              dion::launch_colnorm(R, bp.Q, Rg, Qng, bf ? 1 : (split ? 2 : 0), part, p.nsplit,
                                   tensor && !c.sharded, flags, cnt, n, r, s));
  end_cls(c);
  return DION_OK;
  }

  // steps 5 and 7: M <- B - (1 - mu) P R^T and X <- X - lr s P Q^T in one pass
  if (phase == PH_UPDATE) {
  begin_cls(c, DION_KCLASS_UPDATE);
  {
    bool done = false;
    const float lrs = lr * p.scale;
    if (tensor) {
      int nl = 0;
      cudaError_t e = dion::tc_update(Pg, p.zplane, Rg, Qng, split, bp.G, bp.M, bp.X, cnt, m, n,
                                      r, o.mu, lrs, o.max_wait_spins, flags, sched, rmmc, s, &nl,
                                      &done);
      c.launches += nl;
      if (e != cudaSuccess) return fail(DION_ERR_CUDA, "tc_update: %s", cudaGetErrorString(e));
      if (!done) return fail(DION_ERR_CUDA, "tc_update: %s", dion::tc_map_error());
    }
    if (!done)
      DION_LAUNCH(c, (cnt + 65534) / 65535,
                  dion::launch_update_simt(Pg, Rg, Qng, bf, bp.G, bp.M, bp.X, cnt, m, n, r, o.mu,
                                           lrs, rmmc, s));
  }
  end_cls(c);
  return DION_OK;
  }

  // the per-matrix status and CurvaDion's momentum-change statistic (always computed)
  if (phase == PH_STATUS)
    DION_LAUNCH(c, 1, dion::launch_write_status(flags, rmmc, o.rmmc_threshold,
                                                d_status ? d_status + p.mat0 : nullptr, cnt, s));
  return DION_OK;
}

// Side streams for the orthonormalisation phase, made on first use on a device.
bool ensure_side_streams(dion_handle h, size_t want) {
  int dev = -1;
  if (cudaGetDevice(&dev) != cudaSuccess) return false;
  if (h->side_device != dev) {
    for (auto st : h->side) cudaStreamDestroy(st);
    for (auto ev : h->side_done) cudaEventDestroy(ev);
    if (h->fork_ev) cudaEventDestroy(h->fork_ev);
    h->side.clear();
    h->side_done.clear();
    h->fork_ev = nullptr;
    if (cudaEventCreateWithFlags(&h->fork_ev, cudaEventDisableTiming) != cudaSuccess) return false;
    h->side_device = dev;
  }
  while (h->side.size() < want) {
    cudaStream_t st;
    cudaEvent_t ev;
    if (cudaStreamCreateWithFlags(&st, cudaStreamNonBlocking) != cudaSuccess) return false;
    if (cudaEventCreateWithFlags(&ev, cudaEventDisableTiming) != cudaSuccess) {
      cudaStreamDestroy(st);
      return false;
    }
    h->side.push_back(st);
    h->side_done.push_back(ev);
  }
  return true;
}

void release_upload(dion_handle h) {
  for (auto ev : h->up_done) cudaEventDestroy(ev);
  h->up_done.clear();
  if (h->up_start) cudaEventDestroy(h->up_start);
  if (h->up) cudaStreamDestroy(h->up);
  h->up_start = nullptr;
  h->up = nullptr;
  h->up_device = -1;
}

// The copy stream and events of the overlapped gradient upload on the current device.
bool ensure_upload(dion_handle h, size_t want) {
  int dev = -1;
  if (cudaGetDevice(&dev) != cudaSuccess) return false;
  if (h->up_device != dev) {
    release_upload(h);
    if (cudaStreamCreateWithFlags(&h->up, cudaStreamNonBlocking) != cudaSuccess) {
      h->up = nullptr;
      return false;
    }
    if (cudaEventCreateWithFlags(&h->up_start, cudaEventDisableTiming) != cudaSuccess) {
      h->up_start = nullptr;
      release_upload(h);
      return false;
    }
    h->up_device = dev;
  }
  while (h->up_done.size() < want) {
    cudaEvent_t ev;
    if (cudaEventCreateWithFlags(&ev, cudaEventDisableTiming) != cudaSuccess) return false;
    h->up_done.push_back(ev);
  }
  return true;
}

dion_status check_device(dion_handle h) {
  int dev = -1;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return fail(DION_ERR_CUDA, "cudaGetDevice: %s", cudaGetErrorString(e));
  if (h->device_checked == dev) return DION_OK;
  int major = 0, minor = 0;
  cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev);
  cudaDeviceGetAttribute(&minor, cudaDevAttrComputeCapabilityMinor, dev);
  if (major != 10 || minor != 0)
    return fail(DION_ERR_DEVICE, "device %d is sm_%d%d; this library is built for sm_100a (B200)",
                dev, major, minor);
  h->device_checked = dev;
  return DION_OK;
}

dion_status check_step_args(dion_handle h, const dion_bucket_ptrs* ptrs, int32_t nbuckets,
                            void* ws, size_t ws_bytes, int32_t* d_status) {
  if (!valid(h)) return fail(DION_ERR_NOT_INITIALIZED, "invalid or freed handle");
  if (ptrs == nullptr) return fail(DION_ERR_INVALID_ARG, "ptrs is NULL");
  if (nbuckets != (int32_t)h->plans.size())
    return fail(DION_ERR_INVALID_ARG, "nbuckets %d does not match the plan (%zu)", nbuckets,
                h->plans.size());
  if (ws == nullptr) return fail(DION_ERR_INVALID_ARG, "workspace is NULL");
  if (ws_bytes < h->ws_bytes)
    return fail(DION_ERR_WORKSPACE_TOO_SMALL, "workspace of %zu bytes, %zu needed", ws_bytes,
                h->ws_bytes);
  if (!aligned16(ws)) return fail(DION_ERR_MISALIGNED, "workspace is not 16-byte aligned");
  if (d_status && (reinterpret_cast<uintptr_t>(d_status) & 3u))
    return fail(DION_ERR_MISALIGNED, "d_status is not 4-byte aligned");
  for (int32_t b = 0; b < nbuckets; ++b) {
    const dion_bucket_ptrs& p = ptrs[b];
    if (!p.X || !p.M || !p.G || !p.Q)
      return fail(DION_ERR_INVALID_ARG, "bucket %d: a NULL device pointer", b);
    if (!aligned16(p.X) || !aligned16(p.M) || !aligned16(p.G) || !aligned16(p.Q))
      return fail(DION_ERR_MISALIGNED, "bucket %d: X, M, G and Q must be 16-byte aligned", b);
  }
  return check_device(h);
}

}  // namespace

namespace dion {

dion_status set_error(dion_status s, const char* fmt, ...) {
  va_list ap;
  va_start(ap, fmt);
  vsnprintf(tl_error, sizeof(tl_error), fmt, ap);
  va_end(ap);
  return s;
}

dion_status plan_workspace_bytes(dion_handle h, size_t* bytes) {
  if (!valid(h)) return fail(DION_ERR_NOT_INITIALIZED, "invalid or freed handle");
  *bytes = h->ws_bytes;
  return DION_OK;
}

}  // namespace dion

extern "C" {

dion_status dion_default_options(dion_options* opt) {
  if (!opt) return fail(DION_ERR_INVALID_ARG, "opt is NULL");
  opt->mu = 0.95f;
  opt->precision = DION_PREC_BF16;
  opt->orth_mode = DION_ORTH_AUTO;
  opt->fallback_cond = 1e3f;
  opt->orth_tol = 2e-5f;
  opt->kernel_path = DION_PATH_TENSOR;
  opt->max_wait_spins = int64_t(1) << 26;
  opt->rmmc_threshold = 0.f;
  opt->stack_orth = 0;
  return DION_OK;
}

static dion_status dion_init_impl(const dion_bucket_desc* buckets, const dion_shard_desc* shards,
                                  int32_t nbuckets, const dion_options* opt, dion_handle* out,
                                  size_t* workspace_bytes) {
  if (!out || !workspace_bytes) return fail(DION_ERR_INVALID_ARG, "out or workspace_bytes is NULL");
  *out = nullptr;
  *workspace_bytes = 0;
  if (!buckets || nbuckets < 1) return fail(DION_ERR_INVALID_ARG, "need at least one bucket");
  dion_options o;
  if (opt) o = *opt; else dion_default_options(&o);
  dion_status st = check_options(o);
  if (st != DION_OK) return st;
  const bool sharded = shards != nullptr;
  if (sharded && o.kernel_path != DION_PATH_TENSOR)
    return fail(DION_ERR_INVALID_ARG, "a row-sharded plan runs on the tensor path only");
  const bool bf = o.precision == DION_PREC_BF16;
  // fp32 precision on the tensor path keeps B, Q, P, R as three bf16 parts
  const bool split = !bf && o.kernel_path == DION_PATH_TENSOR;
  const size_t ge = bf ? 2 : (split ? 6 : 4);
  std::vector<Plan> plans;
  size_t off = 0;
  int64_t mats = 0;
  auto take = [&](size_t bytes) {
    const size_t at = off;
    off = align_up(off + bytes, 1024);
    return at;
  };
  for (int32_t b = 0; b < nbuckets; ++b) {
    const dion_bucket_desc& d = buckets[b];
    const int64_t m_full = sharded ? shards[b].m_full : d.m;
    const int64_t row0 = sharded ? shards[b].row0 : 0;
    if (d.count < 1) return fail(DION_ERR_INVALID_ARG, "bucket %d: count %d < 1", b, d.count);
    if (d.count > 65535)
      return fail(DION_ERR_UNSUPPORTED_SHAPE, "bucket %d: count %d exceeds 65535 (split the bucket)",
                  b, d.count);
    if (d.m < 1 || d.n < 1 || d.r < 1)
      return fail(DION_ERR_UNSUPPORTED_SHAPE, "bucket %d: m, n, r must be positive", b);
    if (sharded && (row0 < 0 || m_full < d.m || row0 > m_full - d.m))
      return fail(DION_ERR_INVALID_ARG,
                  "bucket %d: rows [%lld, %lld) are not inside the %lld rows of the matrix", b,
                  (long long)row0, (long long)(row0 + d.m), (long long)m_full);
    if (d.r > m_full || d.r > d.n)
      return fail(DION_ERR_UNSUPPORTED_SHAPE, "bucket %d: r=%lld exceeds min(m, n)", b, (long long)d.r);
    if (d.r % 16 != 0)
      return fail(DION_ERR_UNSUPPORTED_SHAPE, "bucket %d: r=%lld is not a multiple of 16", b, (long long)d.r);
    if (d.n % 8 != 0)
      return fail(DION_ERR_UNSUPPORTED_SHAPE, "bucket %d: n=%lld is not a multiple of 8", b, (long long)d.n);
    if (m_full > (int64_t(1) << 30) || d.n > (int64_t(1) << 30) ||
        (int64_t)d.count * m_full > kMaxElems / d.n || (int64_t)d.count * d.n > kMaxElems / d.r ||
        (int64_t)d.count * m_full > kMaxElems / d.r)
      return fail(DION_ERR_UNSUPPORTED_SHAPE, "bucket %d: too large", b);
    if (!(std::isfinite(d.scale)))
      return fail(DION_ERR_INVALID_ARG, "bucket %d: scale is not finite", b);
    Plan p{};
    p.m = d.m; p.n = d.n; p.r = d.r; p.count = d.count;
    p.m_full = m_full; p.row0 = row0;
    // s = sqrt(m / n) of the whole matrix, whatever rows this rank holds
    p.scale = d.scale > 0.f ? d.scale : (float)std::sqrt((double)m_full / (double)d.n);
    p.mat0 = mats;
    mats += d.count;
    // column-norm partials: on the tensor path B^T P writes them, one per block of
    // R's rows (256 rows with bf16 operands, 32 rows from splits)
    p.nsplit = o.kernel_path != DION_PATH_TENSOR ? dion::colnorm_splits(d.count, d.n)
               : (bf ? dion::tc_btp_col_splits(d.n) : (int)(4 * ((d.n + 127) / 128)));
    plans.push_back(p);
  }
  // A sharded plan places every bucket's Gram back to back, then one float per bucket
  // (the fallback counts), then every bucket's R back to back: each exchange of the
  // step is then a single all-reduce.  r % 16 == 0 and n % 8 == 0 keep every Gram a
  // multiple of 1 KB and every R a multiple of 512 bytes.
  size_t off_wblk = 0, wblk = 0, off_ctrl = 0, off_rblk = 0, rblk = 0;
  if (sharded) {
    for (Plan& p : plans) {
      p.off_W = off_wblk + wblk * 4;
      wblk += (size_t)p.count * p.r * p.r;
    }
    off_ctrl = off_wblk + wblk * 4;
    off_rblk = align_up(off_ctrl + (size_t)nbuckets * 4, 1024);
    for (Plan& p : plans) {
      p.off_R = off_rblk + rblk * 4;
      rblk += (size_t)p.count * p.n * p.r;
    }
    off = align_up(off_rblk + rblk * 4, 1024);
  }
  // Stacks of the orthonormalisation: with stack_orth, the buckets whose P has the same
  // shape (m, r) share one [count, m, r] stack of every per-matrix array the
  // orthonormalisation uses (P0, P and their splits, the Gram and the factor, flags,
  // statistics), so that it runs once over all of them, as DASH stacks equal-sized
  // blocks of different layers.  Each bucket's arrays are slices of its stack.  Without
  // it (and always in a row-sharded plan, whose exchanges are laid out per bucket) every
  // bucket is a stack of its own.
  std::vector<OrthGroup> groups;
  for (int32_t b = 0; b < nbuckets; ++b) {
    Plan& p = plans[b];
    int gi = -1;
    if (!sharded && o.stack_orth)
      for (size_t g = 0; g < groups.size(); ++g) {
        const Plan& q = plans[groups[g].members[0]];
        if (q.m == p.m && q.r == p.r) gi = (int)g;
      }
    if (gi < 0) {
      gi = (int)groups.size();
      groups.push_back(OrthGroup{});
    }
    p.group = gi;
    groups[gi].members.push_back(b);
  }
  for (OrthGroup& g : groups) {
    Plan go = plans[g.members[0]];
    go.count = 0;
    for (int32_t b : g.members) go.count += plans[b].count;
    const size_t c = (size_t)go.count;
    const int64_t m = go.m, r = go.r;
    go.zplane = go.count;
    go.stack_off = 0;
    go.off_P0 = take(c * m * r * 4);
    go.off_P = take(c * m * r * 4);
    go.off_P2 = take(c * m * r * 4);
    go.off_Pg = (bf || split) && !(bf && o.kernel_path == DION_PATH_TENSOR) ? take(c * m * r * ge)
                                                                             : 0;
    if (!sharded) go.off_W = take(c * r * r * 4);
    go.off_Linv = take(c * r * r * 4);
    go.off_dinv = take(dion::chol_dinv_floats(go.count, r) * 4);
    go.off_flags = take(c * 4);
    go.off_stats = take(c * 4 * 4);
    // three-way bf16 splits for the tensor-core orthonormalisation
    go.off_P0s = take(c * m * r * 6);
    go.off_Ps = take(c * m * r * 6);
    go.off_Linvs = take(c * r * r * 6);
    go.off_sched = take(64);  // the fallback loop's counters
    go.off_Ws = go.off_Ts = 0;
    if (o.kernel_path == DION_PATH_TENSOR && r > 256) {
      // splits of the Gram / its updates and of L21 for the recursive factorisation
      go.off_Ws = take(c * r * r * 6);
      go.off_Ts = take(c * r * r * 6);
    }
    size_t at = 0;  // matrices of the stack before this bucket
    for (int32_t b : g.members) {
      Plan& p = plans[b];
      p.stack_off = (int)at;
      p.zplane = go.count;
      p.off_P0 = go.off_P0 + at * m * r * 4;
      p.off_P = go.off_P + at * m * r * 4;
      p.off_P2 = go.off_P2 + at * m * r * 4;
      // (the bf16 copy, or the leading part of the split: 2 bytes an element either way)
      p.off_Pg = go.off_Pg ? go.off_Pg + at * m * r * 2 : 0;
      if (!sharded) p.off_W = go.off_W + at * r * r * 4;
      p.off_Linv = go.off_Linv + at * r * r * 4;
      p.off_dinv = go.off_dinv + dion::chol_dinv_floats((int)at, r) * 4;
      p.off_flags = go.off_flags + at * 4;
      p.off_stats = go.off_stats + at * 4 * 4;
      p.off_P0s = go.off_P0s + at * m * r * 2;
      p.off_Ps = go.off_Ps + at * m * r * 2;
      p.off_Linvs = go.off_Linvs + at * r * r * 2;
      p.off_Ws = go.off_Ws ? go.off_Ws + at * r * r * 2 : 0;
      p.off_Ts = go.off_Ts ? go.off_Ts + at * r * r * 2 : 0;
      at += (size_t)p.count;
    }
    if (sharded) go.off_W = plans[g.members[0]].off_W;
    g.orth = go;
  }
  for (Plan& p : plans) {
    const size_t c = (size_t)p.count;
    p.off_Bg = take(c * p.m * p.n * ge);
    p.off_Qg = take(c * p.n * p.r * ge);
    if (!sharded) p.off_R = take(c * p.n * p.r * 4);
    p.off_Rg = (bf || split) ? take(c * p.n * p.r * ge) : 0;
    p.off_Qng = (bf || split) ? take(c * p.n * p.r * ge) : 0;
    p.off_part = take(c * p.nsplit * p.r * 4);
    p.off_rmmc = take(c * 3 * 4);  // max |M' - M|, max |M|, their ratio: [3][count]
    p.off_sched = take(64);  // tile counters of the dynamically scheduled kernels
    // row-sharded fallback: the gathered P0 (its QR written in place) and the two
    // column-major work arrays of Householder QR, each [count, m_full, r] fp32
    if (sharded) p.off_gather = take(3 * c * p.m_full * p.r * 4);
  }
  // a stack of one bucket is that bucket: its counters are the bucket's
  for (OrthGroup& g : groups)
    if (g.members.size() == 1) g.orth.off_sched = plans[g.members[0]].off_sched;
  dion_ctx* h = new (std::nothrow) dion_ctx();
  if (!h) return fail(DION_ERR_INVALID_ARG, "out of host memory");
  h->magic = kMagic;
  h->opt = o;
  h->plans = std::move(plans);
  h->groups = std::move(groups);
  h->ws_bytes = off;
  h->total_mats = mats;
  h->last_launches = 0;
  h->device_checked = -1;
  h->profiling = false;
  h->events_used = 0;
  for (int i = 0; i < DION_KCLASS_COUNT; ++i) { h->prof_ms[i] = 0; h->prof_launches[i] = 0; }
  h->side_device = -1;
  h->fork_ev = nullptr;
  h->cap = nullptr;
  h->cap_device = -1;
  h->up_device = -1;
  h->up = nullptr;
  h->up_start = nullptr;
  h->sharded = sharded;
  h->off_wblk = off_wblk;
  h->wblk_floats = wblk;
  h->off_ctrl = off_ctrl;
  h->off_rblk = off_rblk;
  h->rblk_floats = rblk;
  h->sh.stage = 0;
  *out = h;
  *workspace_bytes = off;
  return DION_OK;
}

static dion_status dion_step_batched_impl(dion_handle h, const dion_bucket_ptrs* ptrs, int32_t nbuckets,
                              float lr, void* d_workspace, size_t workspace_bytes,
                              int32_t* d_status, void* stream) {
  dion_status st = check_step_args(h, ptrs, nbuckets, d_workspace, workspace_bytes, d_status);
  if (st != DION_OK) return st;
  if (h->sharded)
    return fail(DION_ERR_INVALID_ARG, "a row-sharded plan steps through dion_step_sharded_begin");
  if (!std::isfinite(lr)) return fail(DION_ERR_INVALID_ARG, "lr is not finite");
  cudaStream_t main = reinterpret_cast<cudaStream_t>(stream);
  StepCtx c{h, main, 0, -1, nullptr, 0, std::vector<int>(nbuckets, 0)};
  char* ws = static_cast<char*>(d_workspace);
  // Each stack's orthonormalisation is a chain of short, latency-bound kernels that
  // needs only its buckets' P0.  It is forked onto the stack's own stream as soon as the
  // last of them has run B Q, so it runs beside the B Q of the later buckets and the
  // B^T P, column norms and update of the earlier ones; the main stream joins it just
  // before the B^T P of its first bucket.
  const int32_t ng = (int32_t)h->groups.size();
  const bool fork = (ng > 1 || nbuckets > 1) && ensure_side_streams(h, (size_t)ng);
  c.g_ready.assign((size_t)ng, 0);
  std::vector<char> forked((size_t)ng, 0), joined((size_t)ng, 0);
  auto run = [&](int phase, int32_t b, cudaStream_t s) -> dion_status {
    c.s = s;
    return run_bucket(c, b, phase, h->plans[b], ptrs[b], lr, ws, d_status);
  };
  auto finish = [&](dion_status result) -> dion_status {
    end_cls(c);
    // a failed step still leaves `main` ordered after every forked chain
    for (int32_t g = 0; g < ng; ++g)
      if (forked[g] && !joined[g]) cudaStreamWaitEvent(main, h->side_done[g], 0);
    h->last_launches = c.launches;
    return result;
  };
  for (int phase : {PH_INIT, PH_PREPQ})
    for (int32_t b = 0; b < nbuckets; ++b)
      if ((st = run(phase, b, main)) != DION_OK) return finish(st);
  for (int32_t b = 0; b < nbuckets; ++b) {
    for (int phase : {PH_FORMB, PH_BQ})
      if ((st = run(phase, b, main)) != DION_OK) return finish(st);
    const int32_t g = h->plans[b].group;
    const OrthGroup& og = h->groups[g];
    c.g_ready[g] = c.p0s_ready[b];
    if (og.members.back() != b) continue;  // the stack is complete after its last bucket
    c.s = fork ? h->side[g] : main;
    if (fork) {
      cudaEventRecord(h->fork_ev, main);
      cudaStreamWaitEvent(h->side[g], h->fork_ev, 0);
    }
    st = run_bucket(c, g, PH_ORTH, og.orth, ptrs[og.members[0]], lr, ws, d_status);
    if (fork) {
      end_cls(c);
      cudaEventRecord(h->side_done[g], h->side[g]);
      forked[g] = 1;
    }
    if (st != DION_OK) return finish(st);
  }
  for (int32_t b = 0; b < nbuckets; ++b) {
    const int32_t g = h->plans[b].group;
    if (fork && !joined[g]) {
      cudaStreamWaitEvent(main, h->side_done[g], 0);
      joined[g] = 1;
    }
    for (int phase : {PH_BTP, PH_COLNORM, PH_UPDATE, PH_STATUS})
      if ((st = run(phase, b, main)) != DION_OK) return finish(st);
  }
  return finish(DION_OK);
}

// The step with the gradients uploaded bucket by bucket on a copy stream: each
// orthonormalisation stack's whole step (B Q to update of its buckets) starts as soon as
// its buckets' gradients have arrived, so it runs while the later stacks' gradients cross
// the host link.  Stacks are uploaded largest first, so what is left after the last copy
// is the step of the smallest one.
static dion_status step_overlapped(dion_handle h, const dion_bucket_ptrs* ptrs,
                                   const float* const* host_grads, int32_t nbuckets, float lr,
                                   char* ws, int32_t* d_status, cudaStream_t main) {
  auto grad_bytes = [&](int32_t b) {
    const Plan& p = h->plans[b];
    return (size_t)p.count * p.m * p.n * sizeof(float);
  };
  // stacks of the orthonormalisation in order of their gradients' size, largest first;
  // a stack's step starts once all of its buckets' gradients are on the device
  const int32_t ng = (int32_t)h->groups.size();
  std::vector<int32_t> gorder((size_t)ng);
  std::iota(gorder.begin(), gorder.end(), 0);
  auto group_bytes = [&](int32_t g) {
    size_t t = 0;
    for (int32_t b : h->groups[g].members) t += grad_bytes(b);
    return t;
  };
  std::stable_sort(gorder.begin(), gorder.end(),
                   [&](int32_t a, int32_t b) { return group_bytes(a) > group_bytes(b); });
  std::vector<int32_t> order;            // upload order of the buckets
  std::vector<int32_t> last_upload((size_t)ng);
  for (int32_t g : gorder) {
    for (int32_t b : h->groups[g].members) order.push_back(b);
    last_upload[g] = (int32_t)order.size() - 1;
  }
  // the previous work on the caller's stream (an earlier step) may still read G
  cudaError_t e = cudaEventRecord(h->up_start, main);
  if (e == cudaSuccess) e = cudaStreamWaitEvent(h->up, h->up_start, 0);
  if (e != cudaSuccess) return fail(DION_ERR_CUDA, "upload ordering: %s", cudaGetErrorString(e));
  for (int32_t k = 0; k < nbuckets; ++k) {
    const int32_t b = order[k];
    e = cudaMemcpyAsync(const_cast<float*>(ptrs[b].G), host_grads[b], grad_bytes(b),
                        cudaMemcpyHostToDevice, h->up);
    if (e == cudaSuccess) e = cudaEventRecord(h->up_done[k], h->up);
    if (e != cudaSuccess) {
      // the caller's stream stays ordered after the copies already issued
      if (cudaEventRecord(h->up_start, h->up) == cudaSuccess)
        cudaStreamWaitEvent(main, h->up_start, 0);
      return fail(DION_ERR_CUDA, "gradient upload: %s", cudaGetErrorString(e));
    }
  }
  StepCtx c{h, main, 0, -1, nullptr, 0, std::vector<int>(nbuckets, 0)};
  c.g_ready.assign((size_t)ng, 0);
  int32_t waited = -1;  // the caller's stream is ordered after uploads [0, waited]
  auto finish = [&](dion_status result) -> dion_status {
    end_cls(c);
    if (waited < nbuckets - 1) cudaStreamWaitEvent(main, h->up_done[nbuckets - 1], 0);
    h->last_launches = c.launches;
    return result;
  };
  auto run = [&](int phase, int32_t b) {
    c.s = main;
    return run_bucket(c, b, phase, h->plans[b], ptrs[b], lr, ws, d_status);
  };
  dion_status st;
  for (int phase : {PH_INIT, PH_PREPQ})
    for (int32_t b = 0; b < nbuckets; ++b)
      if ((st = run(phase, b)) != DION_OK) return finish(st);
  for (int32_t g : gorder) {
    const OrthGroup& og = h->groups[g];
    if ((e = cudaStreamWaitEvent(main, h->up_done[last_upload[g]], 0)) != cudaSuccess)
      return finish(fail(DION_ERR_CUDA, "upload wait: %s", cudaGetErrorString(e)));
    waited = last_upload[g];
    for (int32_t b : og.members) {
      for (int phase : {PH_FORMB, PH_BQ})
        if ((st = run(phase, b)) != DION_OK) return finish(st);
      c.g_ready[g] = c.p0s_ready[b];
    }
    c.s = main;
    if ((st = run_bucket(c, g, PH_ORTH, og.orth, ptrs[og.members[0]], lr, ws, d_status)) !=
        DION_OK)
      return finish(st);
    for (int32_t b : og.members)
      for (int phase : {PH_BTP, PH_COLNORM, PH_UPDATE, PH_STATUS})
        if ((st = run(phase, b)) != DION_OK) return finish(st);
  }
  return finish(DION_OK);
}

static dion_status dion_step_batched_from_host_impl(dion_handle h, const dion_bucket_ptrs* ptrs,
                                        const float* const* host_grads, int32_t nbuckets,
                                        float lr, void* d_workspace, size_t workspace_bytes,
                                        int32_t* d_status, int32_t* host_status, void* stream) {
  dion_status st = check_step_args(h, ptrs, nbuckets, d_workspace, workspace_bytes, d_status);
  if (st != DION_OK) return st;
  if (h->sharded)
    return fail(DION_ERR_INVALID_ARG, "a row-sharded plan steps through dion_step_sharded_begin");
  if (!host_grads || !host_status || !d_status)
    return fail(DION_ERR_INVALID_ARG, "host_grads, host_status and d_status are required");
  if (!std::isfinite(lr)) return fail(DION_ERR_INVALID_ARG, "lr is not finite");
  for (int32_t b = 0; b < nbuckets; ++b)
    if (!host_grads[b]) return fail(DION_ERR_INVALID_ARG, "host_grads[%d] is NULL", b);
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  if (ensure_upload(h, (size_t)nbuckets)) {
    st = step_overlapped(h, ptrs, host_grads, nbuckets, lr, static_cast<char*>(d_workspace),
                         d_status, s);
  } else {
    // no copy stream: upload everything, then step
    cudaGetLastError();
    for (int32_t b = 0; b < nbuckets; ++b) {
      const Plan& p = h->plans[b];
      const size_t bytes = (size_t)p.count * p.m * p.n * sizeof(float);
      cudaError_t e = cudaMemcpyAsync(const_cast<float*>(ptrs[b].G), host_grads[b], bytes,
                                      cudaMemcpyHostToDevice, s);
      if (e != cudaSuccess)
        return fail(DION_ERR_CUDA, "gradient upload: %s", cudaGetErrorString(e));
    }
    st = dion_step_batched_impl(h, ptrs, nbuckets, lr, d_workspace, workspace_bytes, d_status,
                                stream);
  }
  if (st != DION_OK) return st;
  cudaError_t e = cudaMemcpyAsync(host_status, d_status, (size_t)h->total_mats * sizeof(int32_t),
                                  cudaMemcpyDeviceToHost, s);
  if (e != cudaSuccess) return fail(DION_ERR_CUDA, "status download: %s", cudaGetErrorString(e));
  e = cudaStreamSynchronize(s);
  if (e != cudaSuccess) return fail(DION_ERR_CUDA, "stream sync: %s", cudaGetErrorString(e));
  return DION_OK;
}

// ------------------------------------------------------------ row-sharded step
// Rank k holds rows [row0, row0 + m) of every matrix; Q is replicated.  The step runs
// as the whole-matrix step, except that four quantities are summed over the ranks by
// the caller between the calls (an all-reduce of fp32 values):
//   the Gram W = P0^T P0 of every bucket (before the Cholesky factorisation),
//   the second pass's Gram and the per-bucket counts of matrices Cholesky-QR rejected,
//   for a bucket with such matrices, its P0 gathered as zero-padded m_full x r blocks,
//   R = B^T P of every bucket (before the column norms).
// Every rank factorises the same summed Gram with the same deterministic kernels, so
// every rank reaches the same decisions (second pass, fallback) and the same Q.
enum ShardStage { SH_IDLE = 0, SH_GRAM1, SH_GRAM2, SH_GATHER, SH_R };

struct ShardBufs {
  float *W, *Linv, *dinv, *P, *P2, *stats, *gather;
  int32_t* flags;
  __nv_bfloat16 *P0s, *Ps, *Linvs, *Ws, *Ts;
  void* Pg;
};

ShardBufs shard_bufs(const dion_options& o, const Plan& p, char* ws) {
  const bool bf = o.precision == DION_PREC_BF16;
  ShardBufs b{};
  b.W = reinterpret_cast<float*>(ws + p.off_W);
  b.Linv = reinterpret_cast<float*>(ws + p.off_Linv);
  b.dinv = reinterpret_cast<float*>(ws + p.off_dinv);
  b.P = reinterpret_cast<float*>(ws + p.off_P);
  b.P2 = reinterpret_cast<float*>(ws + p.off_P2);
  b.stats = reinterpret_cast<float*>(ws + p.off_stats);
  b.gather = reinterpret_cast<float*>(ws + p.off_gather);
  b.flags = reinterpret_cast<int32_t*>(ws + p.off_flags);
  b.P0s = reinterpret_cast<__nv_bfloat16*>(ws + p.off_P0s);
  b.Ps = reinterpret_cast<__nv_bfloat16*>(ws + p.off_Ps);
  b.Linvs = reinterpret_cast<__nv_bfloat16*>(ws + p.off_Linvs);
  b.Ws = p.off_Ws ? reinterpret_cast<__nv_bfloat16*>(ws + p.off_Ws) : nullptr;
  b.Ts = p.off_Ts ? reinterpret_cast<__nv_bfloat16*>(ws + p.off_Ts) : nullptr;
  // the GEMM copy of P (as in run_bucket): bf16 is the leading plane of P's split
  b.Pg = bf ? (void*)b.Ps : (void*)(ws + p.off_Pg);
  return b;
}

#define DION_TC(ctx, call, what)                                                          \
  do {                                                                                    \
    int nl_ = 0;                                                                          \
    bool done_ = false;                                                                   \
    cudaError_t e_ = dion::call;                                                          \
    (ctx).launches += nl_;                                                                \
    if (e_ != cudaSuccess) return fail(DION_ERR_CUDA, "%s: %s", what, cudaGetErrorString(e_)); \
    if (!done_) return fail(DION_ERR_CUDA, "%s: %s", what, dion::tc_map_error());          \
  } while (0)

// Cholesky factorisation (pass 1 or 2) of the summed Gram of one bucket.
dion_status shard_chol(StepCtx& c, const Plan& p, const ShardBufs& b, int pass) {
  const dion_options& o = c.h->opt;
  dion::CholArgs ca{};
  ca.W = b.W; ca.Linv = b.Linv; ca.Linvs = b.Linvs; ca.dinv = b.dinv; ca.flags = b.flags;
  ca.stats = b.stats; ca.count = p.count; ca.r = p.r; ca.m = p.m_full;
  ca.fallback_cond = o.fallback_cond; ca.pass = pass;
  ca.orth_tol = (pass == 2 && o.orth_mode == DION_ORTH_CHOLQR2) ? -1.f : o.orth_tol;
  ca.dev_ready = 0;  // the summed Gram is read for max|W - I|: no epilogue measured it
  if (p.r <= 256) {
    DION_LAUNCH(c, 1, dion::launch_chol_inv(ca, c.s));
    return DION_OK;
  }
  // the recursion reads the split of W's lower tiles: taken from the summed W
  const int64_t rr = (int64_t)p.count * p.r * p.r;
  DION_LAUNCH(c, 1, dion::launch_split3(b.W, b.Ws, rr, rr, c.s));
  int nl = 0;
  bool done = false;
  const char* what = "";
  cudaError_t e = dion::launch_chol_inv_rec(ca, b.Ws, b.Ts, o.max_wait_spins, c.s, &nl, &done,
                                            &what);
  c.launches += nl;
  if (e != cudaSuccess)
    return fail(DION_ERR_CUDA, "recursive factorisation (%s): %s", what, cudaGetErrorString(e));
  if (!done) return fail(DION_ERR_CUDA, "recursive factorisation (%s): %s", what, dion::tc_map_error());
  return DION_OK;
}

void shard_next(dion_exchange* x, float* buf, size_t count, int32_t what) {
  x->d_buf = buf;
  x->count = (int64_t)count;
  x->what = what;
}

// After the gathers (or with none): the fallback's QR, the final P, and R = B^T P.
dion_status shard_to_r(dion_handle h, StepCtx& c, dion_exchange* x) {
  auto& sh = h->sh;
  const dion_options& o = h->opt;
  const bool bf = o.precision == DION_PREC_BF16;
  for (size_t bi = 0; bi < h->plans.size(); ++bi) {
    const Plan& p = h->plans[bi];
    const ShardBufs b = shard_bufs(o, p, sh.ws);
    begin_cls(c, DION_KCLASS_ORTH);
    if (sh.ctrl[bi] > 0.5f) {
      // Householder QR of the whole gathered P0, in place; this rank keeps its rows
      const size_t full = (size_t)p.count * p.m_full * p.r;
      DION_LAUNCH(c, 1, dion::launch_householder(b.gather, nullptr, b.gather + full,
                                                 b.gather + 2 * full, b.gather, b.flags, p.count,
                                                 p.m_full, p.r, c.s));
      DION_LAUNCH(c, 1, dion::launch_rows_from_full(b.gather, b.P, b.flags, p.count, p.m,
                                                    p.m_full, p.row0, p.r, c.s));
    }
    DION_LAUNCH(c, 1, dion::launch_finalize_p(b.P2, b.Pg, bf ? 1 : 2, b.flags, p.count, p.m, p.r,
                                              b.P, o.orth_mode != DION_ORTH_HOUSEHOLDER, c.s));
    end_cls(c);
    dion_status st = run_bucket(c, (int)bi, PH_BTP, p, sh.ptrs[bi], sh.lr, sh.ws, sh.d_status);
    if (st != DION_OK) return st;
  }
  sh.stage = SH_R;
  shard_next(x, reinterpret_cast<float*>(sh.ws + h->off_rblk), h->rblk_floats, DION_XCHG_R);
  return DION_OK;
}

dion_status shard_continue(dion_handle h, dion_exchange* x) {
  auto& sh = h->sh;
  const dion_options& o = h->opt;
  const int32_t nb = (int32_t)h->plans.size();
  StepCtx c{h, sh.s, 0, -1, nullptr, 0, std::vector<int>(nb, 1)};
  c.sharded = true;
  dion_status st = DION_OK;
  auto done = [&](dion_status result) {
    end_cls(c);
    sh.launches += c.launches;
    h->last_launches = sh.launches;
    if (result != DION_OK) sh.stage = SH_IDLE;
    return result;
  };
  if (sh.stage == SH_GRAM1) {
    // pass 1 from the summed Gram, then this rank's part of the second pass's Gram and
    // the number of matrices Cholesky-QR rejected
    for (int32_t bi = 0; bi < nb; ++bi) {
      const Plan& p = h->plans[bi];
      const ShardBufs b = shard_bufs(o, p, sh.ws);
      begin_cls(c, DION_KCLASS_ORTH);
      if (o.orth_mode != DION_ORTH_HOUSEHOLDER) {
        if ((st = shard_chol(c, p, b, 1)) != DION_OK) return done(st);
        __nv_bfloat16* P1s = o.precision == DION_PREC_BF16 ? b.Ps
                                                          : reinterpret_cast<__nv_bfloat16*>(b.Pg);
        auto ap = [&]() -> dion_status {
          DION_TC(c, tc_apply(b.P0s, b.Linvs, nullptr, P1s, nullptr, p.count, p.m, p.r, b.flags, 0,
                              DION_MAT_FALLBACK, o.max_wait_spins, c.s, &nl_, &done_),
                  "tc_apply");
          if (o.orth_mode != DION_ORTH_CHOLQR)
            DION_TC(c, tc_gram(P1s, b.W, nullptr, nullptr, 0, p.count, p.m, p.r, b.flags, 0,
                               DION_MAT_FALLBACK, o.max_wait_spins, c.s, &nl_, &done_, 2),
                    "tc_gram (second pass)");
          return DION_OK;
        };
        if ((st = ap()) != DION_OK) return done(st);
      }
      float* ctrl = reinterpret_cast<float*>(sh.ws + h->off_ctrl) + bi;
      DION_LAUNCH(c, 1, dion::launch_count_flags(b.flags, p.count, DION_MAT_FALLBACK, ctrl, c.s));
      end_cls(c);
    }
    sh.stage = SH_GRAM2;
    shard_next(x, reinterpret_cast<float*>(sh.ws + h->off_wblk), h->wblk_floats + nb,
               DION_XCHG_GRAM2);
    return done(DION_OK);
  }
  if (sh.stage == SH_GRAM2) {
    // the summed counts decide, identically on every rank, which buckets gather P0
    cudaError_t e = cudaMemcpyAsync(sh.ctrl.data(), sh.ws + h->off_ctrl, (size_t)nb * 4,
                                    cudaMemcpyDeviceToHost, sh.s);
    if (e == cudaSuccess) e = cudaStreamSynchronize(sh.s);
    if (e != cudaSuccess)
      return done(fail(DION_ERR_CUDA, "fallback counts: %s", cudaGetErrorString(e)));
    int32_t first = -1;
    for (int32_t bi = 0; bi < nb; ++bi) {
      const Plan& p = h->plans[bi];
      const ShardBufs b = shard_bufs(o, p, sh.ws);
      begin_cls(c, DION_KCLASS_ORTH);
      if (o.orth_mode != DION_ORTH_HOUSEHOLDER && o.orth_mode != DION_ORTH_CHOLQR) {
        if ((st = shard_chol(c, p, b, 2)) != DION_OK) return done(st);
        __nv_bfloat16* P1s = o.precision == DION_PREC_BF16 ? b.Ps
                                                          : reinterpret_cast<__nv_bfloat16*>(b.Pg);
        auto ap = [&]() -> dion_status {
          DION_TC(c, tc_apply(P1s, b.Linvs, b.P2, nullptr, nullptr, p.count, p.m, p.r, b.flags,
                              DION_MAT_CHOLQR2, DION_MAT_FALLBACK, o.max_wait_spins, c.s, &nl_,
                              &done_),
                  "tc_apply (second pass)");
          return DION_OK;
        };
        if ((st = ap()) != DION_OK) return done(st);
      }
      if (sh.ctrl[bi] > 0.5f) {
        const size_t full = (size_t)p.count * p.m_full * p.r;
        cudaError_t e2 = cudaMemsetAsync(b.gather, 0, full * 4, sh.s);
        if (e2 != cudaSuccess) return done(fail(DION_ERR_CUDA, "gather: %s", cudaGetErrorString(e2)));
        DION_LAUNCH(c, 1, dion::launch_rows_to_full(nullptr, b.P0s, b.gather, p.count, p.m,
                                                    p.m_full, p.row0, p.r, sh.s));
        if (first < 0) first = bi;
      }
      end_cls(c);
    }
    if (first >= 0) {
      const Plan& p = h->plans[first];
      sh.stage = SH_GATHER;
      sh.gather_at = first;
      shard_next(x, reinterpret_cast<float*>(sh.ws + p.off_gather),
                 (size_t)p.count * p.m_full * p.r, DION_XCHG_GATHER);
      return done(DION_OK);
    }
    return done(shard_to_r(h, c, x));
  }
  if (sh.stage == SH_GATHER) {
    for (int32_t bi = sh.gather_at + 1; bi < nb; ++bi)
      if (sh.ctrl[bi] > 0.5f) {
        const Plan& p = h->plans[bi];
        sh.gather_at = bi;
        shard_next(x, reinterpret_cast<float*>(sh.ws + p.off_gather),
                   (size_t)p.count * p.m_full * p.r, DION_XCHG_GATHER);
        return done(DION_OK);
      }
    return done(shard_to_r(h, c, x));
  }
  if (sh.stage == SH_R) {
    // Q from the summed R on every rank, then this rank's rows of M and X
    for (int32_t bi = 0; bi < nb; ++bi)
      for (int phase : {PH_COLNORM, PH_UPDATE, PH_STATUS})
        if ((st = run_bucket(c, bi, phase, h->plans[bi], sh.ptrs[bi], sh.lr, sh.ws,
                             sh.d_status)) != DION_OK)
          return done(st);
    sh.stage = SH_IDLE;
    shard_next(x, nullptr, 0, DION_XCHG_NONE);
    return done(DION_OK);
  }
  return done(fail(DION_ERR_INVALID_ARG, "no row-sharded step in progress"));
}

static dion_status dion_step_sharded_begin_impl(dion_handle h, const dion_bucket_ptrs* ptrs,
                                                int32_t nbuckets, float lr, void* d_workspace,
                                                size_t workspace_bytes, int32_t* d_status,
                                                void* stream, dion_exchange* next) {
  if (!next) return fail(DION_ERR_INVALID_ARG, "next is NULL");
  shard_next(next, nullptr, 0, DION_XCHG_NONE);
  dion_status st = check_step_args(h, ptrs, nbuckets, d_workspace, workspace_bytes, d_status);
  if (st != DION_OK) return st;
  if (!h->sharded) return fail(DION_ERR_INVALID_ARG, "the plan is not row-sharded (dion_init_sharded)");
  if (h->sh.stage != SH_IDLE)
    return fail(DION_ERR_INVALID_ARG, "a row-sharded step is already in progress on this handle");
  if (!std::isfinite(lr)) return fail(DION_ERR_INVALID_ARG, "lr is not finite");
  auto& sh = h->sh;
  sh.ptrs.assign(ptrs, ptrs + nbuckets);
  sh.lr = lr;
  sh.ws = static_cast<char*>(d_workspace);
  sh.d_status = d_status;
  sh.s = reinterpret_cast<cudaStream_t>(stream);
  sh.ctrl.assign((size_t)nbuckets, 0.f);
  sh.gather_at = -1;
  sh.launches = 0;
  StepCtx c{h, sh.s, 0, -1, nullptr, 0, std::vector<int>(nbuckets, 0)};
  c.sharded = true;
  auto finish = [&](dion_status result) {
    end_cls(c);
    sh.launches += c.launches;
    h->last_launches = sh.launches;
    return result;
  };
  for (int phase : {PH_INIT, PH_PREPQ})
    for (int32_t b = 0; b < nbuckets; ++b)
      if ((st = run_bucket(c, b, phase, h->plans[b], ptrs[b], lr, sh.ws, d_status)) != DION_OK)
        return finish(st);
  // B = M + G and P0 = B Q on this rank's rows, then its part of each Gram
  for (int32_t b = 0; b < nbuckets; ++b) {
    for (int phase : {PH_FORMB, PH_BQ})
      if ((st = run_bucket(c, b, phase, h->plans[b], ptrs[b], lr, sh.ws, d_status)) != DION_OK)
        return finish(st);
    const Plan& p = h->plans[b];
    const ShardBufs sb = shard_bufs(h->opt, p, sh.ws);
    begin_cls(c, DION_KCLASS_ORTH);
    auto gram = [&]() -> dion_status {
      DION_TC(c, tc_gram(sb.P0s, sb.W, nullptr, nullptr, 0, p.count, p.m, p.r, sb.flags, 0,
                         DION_MAT_FALLBACK, h->opt.max_wait_spins, sh.s, &nl_, &done_),
              "tc_gram");
      return DION_OK;
    };
    if (h->opt.orth_mode != DION_ORTH_HOUSEHOLDER && (st = gram()) != DION_OK) return finish(st);
    end_cls(c);
  }
  sh.stage = SH_GRAM1;
  shard_next(next, reinterpret_cast<float*>(sh.ws + h->off_wblk), h->wblk_floats,
             DION_XCHG_GRAM);
  return finish(DION_OK);
}

static dion_status dion_free_impl(dion_handle h) {
  if (!h) return DION_OK;
  if (!valid(h)) return fail(DION_ERR_NOT_INITIALIZED, "invalid or freed handle");
  for (auto& ep : h->events) {
    cudaEventDestroy(ep.a);
    cudaEventDestroy(ep.b);
  }
  for (auto st : h->side) cudaStreamDestroy(st);
  for (auto ev : h->side_done) cudaEventDestroy(ev);
  if (h->fork_ev) cudaEventDestroy(h->fork_ev);
  for (auto& g : h->fb)
    if (g.exec) cudaGraphExecDestroy(g.exec);
  if (h->cap) cudaStreamDestroy(h->cap);
  release_upload(h);
  h->magic = 0;
  delete h;
  return DION_OK;
}

const char* dion_status_string(dion_status s) {
  switch (s) {
    case DION_OK: return "ok";
    case DION_ERR_INVALID_ARG: return "invalid argument";
    case DION_ERR_UNSUPPORTED_SHAPE: return "unsupported shape";
    case DION_ERR_WORKSPACE_TOO_SMALL: return "workspace too small";
    case DION_ERR_CUDA: return "CUDA error";
    case DION_ERR_NOT_INITIALIZED: return "handle not initialized";
    case DION_ERR_DEVICE: return "unsupported device";
    case DION_ERR_MISALIGNED: return "misaligned pointer";
    case DION_ERR_HOST: return "host-side failure (host memory)";
  }
  return "unknown status";
}

const char* dion_last_error(void) { return tl_error; }

int64_t dion_num_matrices(dion_handle h) { return valid(h) ? h->total_mats : -1; }

int32_t dion_last_launch_count(dion_handle h) { return valid(h) ? h->last_launches : -1; }

static dion_status dion_workspace_view_impl(dion_handle h, int32_t bucket, int32_t which,
                                            void* d_workspace, void** d_ptr, size_t* bytes) {
  if (!valid(h)) return fail(DION_ERR_NOT_INITIALIZED, "invalid or freed handle");
  if (!d_ptr || !bytes || !d_workspace) return fail(DION_ERR_INVALID_ARG, "NULL argument");
  if (bucket < 0 || bucket >= (int32_t)h->plans.size())
    return fail(DION_ERR_INVALID_ARG, "bucket %d out of range", bucket);
  const Plan& p = h->plans[bucket];
  char* ws = static_cast<char*>(d_workspace);
  if (which == DION_VIEW_P) {
    *d_ptr = ws + p.off_P;
    *bytes = (size_t)p.count * p.m * p.r * 4;
    // on the tensor path the first Cholesky-QR pass leaves P as its three-way split only:
    // rebuild the fp32 P of the matrices that kept that pass (on the legacy stream, after
    // the caller's synchronisation), and wait for it
    if (h->opt.kernel_path == DION_PATH_TENSOR && h->opt.orth_mode != DION_ORTH_HOUSEHOLDER &&
        h->last_launches > 0) {
      const bool bf = h->opt.precision == DION_PREC_BF16;
      const void* split = ws + (bf ? p.off_Ps : p.off_Pg);
      cudaError_t e = dion::launch_p_from_split(reinterpret_cast<float*>(ws + p.off_P), split,
                                                (int64_t)p.zplane * p.m * p.r,
                                                reinterpret_cast<const int32_t*>(ws + p.off_flags),
                                                p.count, p.m, p.r, 0);
      if (e == cudaSuccess) e = cudaStreamSynchronize(0);
      if (e != cudaSuccess)
        return fail(DION_ERR_CUDA, "rebuilding P from its split: %s", cudaGetErrorString(e));
    }
  } else if (which == DION_VIEW_R) {
    *d_ptr = ws + p.off_R;
    *bytes = (size_t)p.count * p.n * p.r * 4;
  } else if (which == DION_VIEW_RMMC) {
    *d_ptr = ws + p.off_rmmc + (size_t)2 * p.count * 4;
    *bytes = (size_t)p.count * 4;
  } else {
    return fail(DION_ERR_INVALID_ARG, "unknown view %d", which);
  }
  return DION_OK;
}

static dion_status dion_profile_enable_impl(dion_handle h, int32_t on) {
  if (!valid(h)) return fail(DION_ERR_NOT_INITIALIZED, "invalid or freed handle");
  h->profiling = on != 0;
  h->events_used = 0;
  for (int i = 0; i < DION_KCLASS_COUNT; ++i) { h->prof_ms[i] = 0; h->prof_launches[i] = 0; }
  return DION_OK;
}

static dion_status dion_profile_read_impl(dion_handle h, double* ms, int64_t* launches,
                                          int32_t nclasses) {
  if (!valid(h)) return fail(DION_ERR_NOT_INITIALIZED, "invalid or freed handle");
  if (!ms || nclasses < 1) return fail(DION_ERR_INVALID_ARG, "ms is NULL or nclasses < 1");
  for (size_t i = 0; i < h->events_used; ++i) {
    EventPair& ep = h->events[i];
    cudaError_t e = cudaEventSynchronize(ep.b);
    if (e != cudaSuccess) return fail(DION_ERR_CUDA, "cudaEventSynchronize: %s", cudaGetErrorString(e));
    float t = 0.f;
    e = cudaEventElapsedTime(&t, ep.a, ep.b);
    if (e != cudaSuccess) return fail(DION_ERR_CUDA, "cudaEventElapsedTime: %s", cudaGetErrorString(e));
    h->prof_ms[ep.cls] += t;
    h->prof_launches[ep.cls] += ep.launches;
  }
  h->events_used = 0;
  for (int i = 0; i < nclasses && i < DION_KCLASS_COUNT; ++i) {
    ms[i] = h->prof_ms[i];
    if (launches) launches[i] = h->prof_launches[i];
  }
  return DION_OK;
}

dion_status dion_init(const dion_bucket_desc* buckets, int32_t nbuckets, const dion_options* opt,
                      dion_handle* out, size_t* workspace_bytes) {
  return guarded("dion_init", [&] {
    return dion_init_impl(buckets, nullptr, nbuckets, opt, out, workspace_bytes);
  });
}

dion_status dion_step_batched(dion_handle h, const dion_bucket_ptrs* ptrs, int32_t nbuckets,
                              float lr, void* d_workspace, size_t workspace_bytes,
                              int32_t* d_status, void* stream) {
  return guarded("dion_step_batched", [&] {
    return dion_step_batched_impl(h, ptrs, nbuckets, lr, d_workspace, workspace_bytes, d_status,
                                  stream);
  });
}

dion_status dion_step_batched_from_host(dion_handle h, const dion_bucket_ptrs* ptrs,
                                        const float* const* host_grads, int32_t nbuckets,
                                        float lr, void* d_workspace, size_t workspace_bytes,
                                        int32_t* d_status, int32_t* host_status, void* stream) {
  return guarded("dion_step_batched_from_host", [&] {
    return dion_step_batched_from_host_impl(h, ptrs, host_grads, nbuckets, lr, d_workspace,
                                            workspace_bytes, d_status, host_status, stream);
  });
}

dion_status dion_free(dion_handle h) {
  return guarded("dion_free", [&] { return dion_free_impl(h); });
}

dion_status dion_init_sharded(const dion_bucket_desc* buckets, const dion_shard_desc* shards,
                              int32_t nbuckets, const dion_options* opt, dion_handle* out,
                              size_t* workspace_bytes) {
  return guarded("dion_init_sharded", [&] {
    if (!shards) return fail(DION_ERR_INVALID_ARG, "shards is NULL");
    return dion_init_impl(buckets, shards, nbuckets, opt, out, workspace_bytes);
  });
}

dion_status dion_step_sharded_begin(dion_handle h, const dion_bucket_ptrs* ptrs,
                                    int32_t nbuckets, float lr, void* d_workspace,
                                    size_t workspace_bytes, int32_t* d_status, void* stream,
                                    dion_exchange* next) {
  // the step's state is recorded only once every launch of this call succeeded
  return guarded("dion_step_sharded_begin", [&] {
    return dion_step_sharded_begin_impl(h, ptrs, nbuckets, lr, d_workspace, workspace_bytes,
                                        d_status, stream, next);
  });
}

dion_status dion_step_sharded_continue(dion_handle h, dion_exchange* next) {
  return guarded("dion_step_sharded_continue", [&] {
    if (!valid(h)) return fail(DION_ERR_NOT_INITIALIZED, "invalid or freed handle");
    if (!next) return fail(DION_ERR_INVALID_ARG, "next is NULL");
    shard_next(next, nullptr, 0, DION_XCHG_NONE);
    if (!h->sharded || h->sh.stage == SH_IDLE)
      return fail(DION_ERR_INVALID_ARG, "no row-sharded step in progress");
    return shard_continue(h, next);
  });
}

dion_status dion_workspace_view(dion_handle h, int32_t bucket, int32_t which, void* d_workspace,
                                void** out, size_t* bytes) {
  return guarded("dion_workspace_view",
                 [&] { return dion_workspace_view_impl(h, bucket, which, d_workspace, out, bytes); });
}

dion_status dion_profile_enable(dion_handle h, int32_t on) {
  return guarded("dion_profile_enable", [&] { return dion_profile_enable_impl(h, on); });
}

dion_status dion_profile_read(dion_handle h, double* ms, int64_t* launches, int32_t nclasses) {
  return guarded("dion_profile_read",
                 [&] { return dion_profile_read_impl(h, ms, launches, nclasses); });
}

}  // extern "C"

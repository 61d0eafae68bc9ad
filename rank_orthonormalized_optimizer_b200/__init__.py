"""Batched Dion optimizer step on NVIDIA B200 (sm_100a): Python binding.

The arithmetic runs in the CUDA library ``lib/libdion_b200.so`` behind the C ABI
of ``include/dion.h``; this module only marshals arguments (torch tensors to
device pointers and the current CUDA stream).  PyTorch provides device memory
and streams.  There is no CPU implementation: importing this module fails if
the library has not been built (``python rank_orthonormalized_optimizer_b200/build.py``).

One step, for every matrix of every bucket (see include/dion.h):
    B = M + G;  P = orth(B Q);  R = B^T P;  M <- B - (1 - mu) P R^T;
    Q <- colnorm(R);  X <- X - lr * s * P Q^T,  s = sqrt(m / n)
"""
from __future__ import annotations

import ctypes
import os
from dataclasses import dataclass

_PKG = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_PKG, "lib", "libdion_b200.so")

if not os.path.exists(LIB_PATH):
    raise ImportError(
        f"{LIB_PATH} is missing: build the CUDA library first with "
        "`python rank_orthonormalized_optimizer_b200/build.py` (nvcc, sm_100a)")

_lib = ctypes.CDLL(LIB_PATH)

c_int32, c_int64, c_float, c_void_p, c_size_t = (ctypes.c_int32, ctypes.c_int64, ctypes.c_float,
                                                 ctypes.c_void_p, ctypes.c_size_t)

# status codes and bits, mirrored from include/dion.h
OK, ERR_INVALID_ARG, ERR_UNSUPPORTED_SHAPE, ERR_WORKSPACE_TOO_SMALL, ERR_CUDA, \
    ERR_NOT_INITIALIZED, ERR_DEVICE, ERR_MISALIGNED, ERR_HOST = range(9)
MAT_OK, MAT_FALLBACK, MAT_CHOLQR2, MAT_NONFINITE, MAT_TIMEOUT, MAT_ZERO_COLUMN = 0, 1, 2, 4, 8, 16
MAT_HIGH_RMMC = 32
PRECISIONS = {"fp32": 0, "bf16": 1}
ORTH_MODES = {"auto": 0, "cholqr": 1, "cholqr2": 2, "householder": 3}
KERNEL_PATHS = {"tensor": 0, "simt": 1}
KERNEL_CLASSES = ["form_b", "prep_q", "gemm_bq", "orth", "gemm_btp", "colnorm", "update"]
VIEW_P, VIEW_R, VIEW_RMMC = 0, 1, 2
STATIC_SCRATCH_BYTES = 16 << 20   # DION_STATIC_SCRATCH_BYTES of include/dion.h


class BucketDesc(ctypes.Structure):
    _fields_ = [("m", c_int64), ("n", c_int64), ("r", c_int64), ("count", c_int32),
                ("scale", c_float)]


class Options(ctypes.Structure):
    _fields_ = [("mu", c_float), ("precision", c_int32), ("orth_mode", c_int32),
                ("fallback_cond", c_float), ("orth_tol", c_float), ("kernel_path", c_int32),
                ("max_wait_spins", c_int64), ("rmmc_threshold", c_float),
                ("stack_orth", c_int32)]


class BucketPtrs(ctypes.Structure):
    _fields_ = [("X", c_void_p), ("M", c_void_p), ("G", c_void_p), ("Q", c_void_p)]


class ShardDesc(ctypes.Structure):
    _fields_ = [("m_full", c_int64), ("row0", c_int64)]


class Exchange(ctypes.Structure):
    _fields_ = [("d_buf", c_void_p), ("count", c_int64), ("what", c_int32)]


XCHG_NONE, XCHG_GRAM, XCHG_GRAM2, XCHG_GATHER, XCHG_R = range(5)
XCHG_NAMES = {XCHG_NONE: "none", XCHG_GRAM: "gram", XCHG_GRAM2: "gram2",
              XCHG_GATHER: "gather", XCHG_R: "r"}


VEC_RULES = {"adamw": 0, "lion": 1}


class VecTensor(ctypes.Structure):
    _fields_ = [("x", c_void_p), ("g", c_void_p), ("m", c_void_p), ("v", c_void_p),
                ("numel", c_int64)]


class VecOptions(ctypes.Structure):
    _fields_ = [("rule", c_int32), ("lr", c_float), ("beta1", c_float), ("beta2", c_float),
                ("eps", c_float), ("weight_decay", c_float), ("step", c_int64)]


def _sig(name, restype, *args):
    f = getattr(_lib, name)
    f.restype = restype
    f.argtypes = list(args)
    return f


dion_default_options = _sig("dion_default_options", c_int32, ctypes.POINTER(Options))
dion_init = _sig("dion_init", c_int32, ctypes.POINTER(BucketDesc), c_int32,
                 ctypes.POINTER(Options), ctypes.POINTER(c_void_p), ctypes.POINTER(c_size_t))
dion_step_batched = _sig("dion_step_batched", c_int32, c_void_p, ctypes.POINTER(BucketPtrs),
                         c_int32, c_float, c_void_p, c_size_t, c_void_p, c_void_p)
dion_step_batched_from_host = _sig("dion_step_batched_from_host", c_int32, c_void_p,
                                   ctypes.POINTER(BucketPtrs), ctypes.POINTER(c_void_p), c_int32,
                                   c_float, c_void_p, c_size_t, c_void_p, c_void_p, c_void_p)
dion_step_batched_noalloc = _sig("dion_step_batched_noalloc", c_int32, c_void_p,
                                 ctypes.POINTER(BucketPtrs), c_int32, c_float, c_void_p, c_void_p)
dion_free = _sig("dion_free", c_int32, c_void_p)
dion_init_sharded = _sig("dion_init_sharded", c_int32, ctypes.POINTER(BucketDesc),
                         ctypes.POINTER(ShardDesc), c_int32, ctypes.POINTER(Options),
                         ctypes.POINTER(c_void_p), ctypes.POINTER(c_size_t))
dion_step_sharded_begin = _sig("dion_step_sharded_begin", c_int32, c_void_p,
                               ctypes.POINTER(BucketPtrs), c_int32, c_float, c_void_p, c_size_t,
                               c_void_p, c_void_p, ctypes.POINTER(Exchange))
dion_step_sharded_continue = _sig("dion_step_sharded_continue", c_int32, c_void_p,
                                  ctypes.POINTER(Exchange))
dion_vec_default_options = _sig("dion_vec_default_options", c_int32, c_int32,
                                ctypes.POINTER(VecOptions))
dion_vec_step = _sig("dion_vec_step", c_int32, ctypes.POINTER(VecTensor), c_int32,
                     ctypes.POINTER(VecOptions), c_void_p)
dion_vec_last_launch_count = _sig("dion_vec_last_launch_count", c_int32)
dion_status_string = _sig("dion_status_string", ctypes.c_char_p, c_int32)
dion_last_error = _sig("dion_last_error", ctypes.c_char_p)
dion_num_matrices = _sig("dion_num_matrices", c_int64, c_void_p)
dion_last_launch_count = _sig("dion_last_launch_count", c_int32, c_void_p)
dion_workspace_view = _sig("dion_workspace_view", c_int32, c_void_p, c_int32, c_int32, c_void_p,
                           ctypes.POINTER(c_void_p), ctypes.POINTER(c_size_t))
dion_profile_enable = _sig("dion_profile_enable", c_int32, c_void_p, c_int32)
dion_profile_read = _sig("dion_profile_read", c_int32, c_void_p, ctypes.POINTER(ctypes.c_double),
                         ctypes.POINTER(c_int64), c_int32)

#: every entry point include/dion.h declares
EXPORTED = ["dion_default_options", "dion_init", "dion_step_batched",
            "dion_step_batched_from_host", "dion_step_batched_noalloc", "dion_free",
            "dion_init_sharded", "dion_step_sharded_begin", "dion_step_sharded_continue",
            "dion_status_string", "dion_last_error",
            "dion_num_matrices", "dion_last_launch_count", "dion_workspace_view",
            "dion_profile_enable", "dion_profile_read", "dion_vec_default_options",
            "dion_vec_step", "dion_vec_last_launch_count"]


class DionError(RuntimeError):
    def __init__(self, code: int, where: str):
        self.code = code
        msg = dion_status_string(code).decode()
        detail = dion_last_error().decode()
        super().__init__(f"{where}: {msg} ({code}): {detail}")


def _check(code: int, where: str):
    if code != OK:
        raise DionError(code, where)


def default_options() -> Options:
    o = Options()
    _check(dion_default_options(ctypes.byref(o)), "dion_default_options")
    return o


@dataclass(frozen=True)
class Shape:
    count: int
    m: int
    n: int
    r: int


def _make_options(mu, precision, orth_mode, kernel_path, fallback_cond, orth_tol,
                  max_wait_spins, rmmc_threshold=0.0, stack_orth=False) -> Options:
    o = default_options()
    o.rmmc_threshold = rmmc_threshold
    o.stack_orth = int(bool(stack_orth))
    o.mu = mu
    o.precision = PRECISIONS[precision]
    o.orth_mode = ORTH_MODES[orth_mode]
    o.kernel_path = KERNEL_PATHS[kernel_path]
    o.fallback_cond = fallback_cond
    o.orth_tol = orth_tol
    o.max_wait_spins = max_wait_spins
    return o


def _descs(shapes, scales=None):
    descs = (BucketDesc * max(len(shapes), 1))()
    for i, s in enumerate(shapes):
        descs[i].m, descs[i].n, descs[i].r, descs[i].count = s.m, s.n, s.r, s.count
        descs[i].scale = float(scales[i]) if scales is not None else 0.0
    return descs


class DionB200:
    """Handle of one planned step over a fixed list of shape buckets.

    ``buckets``: sequence of (count, m, n, r).  Keyword options map onto
    dion_options (include/dion.h).  All tensors handed to ``step`` are
    contiguous CUDA tensors: X, M, G fp32 [count, m, n]; Q fp32 [count, n, r].
    """

    def __init__(self, buckets, *, mu=0.95, precision="bf16", orth_mode="auto",
                 kernel_path="tensor", fallback_cond=1e3, orth_tol=2e-5,
                 max_wait_spins=1 << 26, scales=None, rmmc_threshold=0.0, stack_orth=False):
        self.shapes = [Shape(*map(int, b)) for b in buckets]
        self.options = _make_options(mu, precision, orth_mode, kernel_path, fallback_cond,
                                     orth_tol, max_wait_spins, rmmc_threshold, stack_orth)
        h = c_void_p()
        ws = c_size_t()
        _check(dion_init(_descs(self.shapes, scales), len(self.shapes),
                         ctypes.byref(self.options), ctypes.byref(h), ctypes.byref(ws)),
               "dion_init")
        self._h = h
        self.workspace_bytes = ws.value
        self.num_matrices = dion_num_matrices(h)

    # ------------------------------------------------------------ memory helpers
    def alloc_workspace(self, device=None):
        import torch
        return torch.empty(self.workspace_bytes, dtype=torch.uint8, device=device or "cuda")

    def alloc_status(self, device=None):
        import torch
        return torch.zeros(self.num_matrices, dtype=torch.int32, device=device or "cuda")

    def _ptrs(self, X, M, G, Q):
        import torch
        n = len(self.shapes)
        if not (len(X) == len(M) == len(G) == len(Q) == n):
            raise ValueError(f"expected {n} tensors each for X, M, G and Q")
        arr = (BucketPtrs * n)()
        for i, s in enumerate(self.shapes):
            for name, t, shape in (("X", X[i], (s.count, s.m, s.n)), ("M", M[i], (s.count, s.m, s.n)),
                                   ("G", G[i], (s.count, s.m, s.n)), ("Q", Q[i], (s.count, s.n, s.r))):
                if not isinstance(t, torch.Tensor) or not t.is_cuda:
                    raise ValueError(f"bucket {i}: {name} must be a CUDA tensor")
                if t.dtype != torch.float32 or not t.is_contiguous() or tuple(t.shape) != shape:
                    raise ValueError(f"bucket {i}: {name} must be contiguous fp32 {shape}, "
                                     f"got {t.dtype} {tuple(t.shape)}")
            arr[i].X, arr[i].M = X[i].data_ptr(), M[i].data_ptr()
            arr[i].G, arr[i].Q = G[i].data_ptr(), Q[i].data_ptr()
        return arr

    @staticmethod
    def _stream(stream):
        import torch
        if stream is None:
            stream = torch.cuda.current_stream()
        return c_void_p(stream.cuda_stream)

    def step(self, X, M, G, Q, lr: float, workspace, status=None, stream=None):
        """One Dion step over all buckets, enqueued on ``stream`` (default: current)."""
        arr = self._ptrs(X, M, G, Q)
        _check(dion_step_batched(self._h, arr, len(self.shapes), float(lr),
                                 c_void_p(workspace.data_ptr()), workspace.numel(),
                                 c_void_p(status.data_ptr()) if status is not None else None,
                                 self._stream(stream)),
               "dion_step_batched")

    def step_noalloc(self, X, M, G, Q, lr: float, status=None, stream=None):
        """The step with the library's built-in scratch instead of a workspace."""
        arr = self._ptrs(X, M, G, Q)
        _check(dion_step_batched_noalloc(self._h, arr, len(self.shapes), float(lr),
                                         c_void_p(status.data_ptr()) if status is not None else None,
                                         self._stream(stream)),
               "dion_step_batched_noalloc")

    def step_from_host(self, X, M, G_dev, Q, G_host, lr: float, workspace, status, host_status,
                       stream=None):
        """Upload the host gradients G_host into G_dev, step, return the host status."""
        arr = self._ptrs(X, M, G_dev, Q)
        hg = (c_void_p * len(self.shapes))(*[g.data_ptr() for g in G_host])
        _check(dion_step_batched_from_host(self._h, arr, hg, len(self.shapes), float(lr),
                                           c_void_p(workspace.data_ptr()), workspace.numel(),
                                           c_void_p(status.data_ptr()),
                                           c_void_p(host_status.data_ptr()),
                                           self._stream(stream)),
               "dion_step_batched_from_host")
        return host_status

    def view(self, bucket: int, which: int, workspace):
        """P ([count, m, r]), R ([count, n, r]) or the momentum-change statistic RMMC
        ([count]) of the last step, as a view of the workspace."""
        import torch
        ptr, nbytes = c_void_p(), c_size_t()
        _check(dion_workspace_view(self._h, bucket, which, c_void_p(workspace.data_ptr()),
                                   ctypes.byref(ptr), ctypes.byref(nbytes)), "dion_workspace_view")
        off = ptr.value - workspace.data_ptr()
        s = self.shapes[bucket]
        shape = {VIEW_P: (s.count, s.m, s.r), VIEW_R: (s.count, s.n, s.r),
                 VIEW_RMMC: (s.count,)}[which]
        return workspace[off:off + nbytes.value].view(torch.float32).view(*shape)

    @property
    def last_launch_count(self) -> int:
        return dion_last_launch_count(self._h)

    def profile_enable(self, on: bool = True):
        _check(dion_profile_enable(self._h, int(on)), "dion_profile_enable")

    def profile_read(self):
        """{class: (milliseconds, launches)} summed since profile_enable."""
        n = len(KERNEL_CLASSES)
        ms = (ctypes.c_double * n)()
        nl = (c_int64 * n)()
        _check(dion_profile_read(self._h, ms, nl, n), "dion_profile_read")
        return {k: (ms[i], nl[i]) for i, k in enumerate(KERNEL_CLASSES)}

    def close(self):
        if getattr(self, "_h", None) is not None and self._h.value:
            dion_free(self._h)
            self._h = c_void_p()

    def __del__(self):
        try:
            self.close()
        except Exception:
            pass


# ---------------------------------------------------------------- row-sharded step
def row_range(m: int, world: int, rank: int):
    """Rows [row0, row0 + m_k) of rank ``rank`` when m rows are split as evenly as
    possible among ``world`` ranks (the first m % world ranks take one row more)."""
    base, extra = divmod(m, world)
    return rank * base + min(rank, extra), base + (1 if rank < extra else 0)


def _default_allreduce(buf):
    import torch.distributed as dist
    if dist.is_available() and dist.is_initialized() and dist.get_world_size() > 1:
        dist.all_reduce(buf)


class DionB200RowSharded(DionB200):
    """This rank's rows of every matrix of a row-sharded step (include/dion.h,
    dion_init_sharded).  ``buckets`` are the WHOLE shapes (count, m, n, r); rank
    ``rank`` of ``world`` holds rows ``row_range(m, world, rank)`` of each, so the
    tensors handed to ``step`` are X, M, G fp32 [count, m_k, n] and the whole Q
    [count, n, r] (the same on every rank)."""

    def __init__(self, buckets, rank: int, world: int, *, mu=0.95, precision="bf16",
                 orth_mode="auto", fallback_cond=1e3, orth_tol=2e-5, max_wait_spins=1 << 26,
                 scales=None, rmmc_threshold=0.0):
        self.full_shapes = [Shape(*map(int, b)) for b in buckets]
        self.rank, self.world = int(rank), int(world)
        rows = [row_range(s.m, self.world, self.rank) for s in self.full_shapes]
        self.row_ranges = rows
        self.shapes = [Shape(s.count, mk, s.n, s.r) for s, (_, mk) in zip(self.full_shapes, rows)]
        shards = (ShardDesc * max(len(self.shapes), 1))()
        for i, (s, (row0, _)) in enumerate(zip(self.full_shapes, rows)):
            shards[i].m_full, shards[i].row0 = s.m, row0
        self.options = _make_options(mu, precision, orth_mode, "tensor", fallback_cond,
                                     orth_tol, max_wait_spins, rmmc_threshold)
        h = c_void_p()
        ws = c_size_t()
        _check(dion_init_sharded(_descs(self.shapes, scales), shards, len(self.shapes),
                                 ctypes.byref(self.options), ctypes.byref(h), ctypes.byref(ws)),
               "dion_init_sharded")
        self._h = h
        self.workspace_bytes = ws.value
        self.num_matrices = dion_num_matrices(h)
        self._x = Exchange()
        self._ws = None

    def _buffer(self):
        """The current exchange's buffer as a float32 view of the workspace."""
        import torch
        off = self._x.d_buf - self._ws.data_ptr()
        return self._ws[off:off + 4 * self._x.count].view(torch.float32)

    def begin(self, X, M, G, Q, lr: float, workspace, status=None, stream=None):
        """Start a step; returns (kind, buffer) of the first exchange."""
        arr = self._ptrs(X, M, G, Q)
        self._ws = workspace
        _check(dion_step_sharded_begin(self._h, arr, len(self.shapes), float(lr),
                                       c_void_p(workspace.data_ptr()), workspace.numel(),
                                       c_void_p(status.data_ptr()) if status is not None else None,
                                       self._stream(stream), ctypes.byref(self._x)),
               "dion_step_sharded_begin")
        return XCHG_NAMES[self._x.what], self._buffer()

    def advance(self):
        """After the current buffer was summed over the ranks; returns the next
        (kind, buffer), or ("none", None) when the step is complete."""
        _check(dion_step_sharded_continue(self._h, ctypes.byref(self._x)),
               "dion_step_sharded_continue")
        if self._x.count == 0:
            return "none", None
        return XCHG_NAMES[self._x.what], self._buffer()

    def step(self, X, M, G, Q, lr: float, workspace, status=None, stream=None, allreduce=None):
        """One row-sharded step.  ``allreduce(buf)`` sums a float32 CUDA tensor over the
        ranks in place on the current stream (default: torch.distributed.all_reduce when a
        process group of more than one rank exists, else nothing).  Returns the exchanges
        as (kind, floats) pairs."""
        reduce = allreduce or _default_allreduce
        done = []
        kind, buf = self.begin(X, M, G, Q, lr, workspace, status, stream)
        while buf is not None:
            done.append((kind, buf.numel()))
            reduce(buf)
            kind, buf = self.advance()
        return done


# ---------------------------------------------------------------- vector parameters
def vec_default_options(rule: str = "adamw") -> VecOptions:
    o = VecOptions()
    _check(dion_vec_default_options(VEC_RULES[rule], ctypes.byref(o)), "dion_vec_default_options")
    return o


class VecStepPlan:
    """A fixed list of vector (1-D) parameters and their state, marshalled once.

    ``x``, ``g``, ``m`` (and ``v`` for AdamW): equal-length lists of contiguous fp32
    CUDA tensors, one entry per parameter; they must stay allocated while the plan is
    used.  ``step`` then costs one C call (dion_vec_step) and its launches.  Options
    left as None take the defaults of include/dion.h (dion_vec_default_options).
    """

    def __init__(self, x, g, m, v=None, *, rule="adamw", lr=None, betas=None, eps=None,
                 weight_decay=None):
        import torch
        o = vec_default_options(rule)
        if lr is not None:
            o.lr = lr
        if betas is not None:
            o.beta1, o.beta2 = betas
        if eps is not None:
            o.eps = eps
        if weight_decay is not None:
            o.weight_decay = weight_decay
        n = len(x)
        if v is None:
            v = [None] * n
        if not (len(g) == len(m) == len(v) == n):
            raise ValueError("x, g, m and v must have one entry per parameter")
        arr = (VecTensor * max(n, 1))()
        for i in range(n):
            named = (("x", x[i]), ("g", g[i]), ("m", m[i]))
            if rule == "adamw":
                named += (("v", v[i]),)
            for name, t in named:
                if not isinstance(t, torch.Tensor) or not t.is_cuda or t.dtype != torch.float32 \
                        or not t.is_contiguous() or t.numel() != x[i].numel():
                    raise ValueError(f"parameter {i}: {name} must be a contiguous fp32 CUDA "
                                     f"tensor of {x[i].numel()} elements")
            arr[i].x, arr[i].g, arr[i].m = x[i].data_ptr(), g[i].data_ptr(), m[i].data_ptr()
            arr[i].v = v[i].data_ptr() if v[i] is not None else None
            arr[i].numel = x[i].numel()
        self.options, self.n, self._arr = o, n, arr
        self._keep = (list(x), list(g), list(m), list(v))

    def step(self, step: int = 1, stream=None) -> int:
        """One step (AdamW step number ``step`` >= 1); returns the kernel launches."""
        self.options.step = int(step)
        _check(dion_vec_step(self._arr, self.n, ctypes.byref(self.options),
                             DionB200._stream(stream)), "dion_vec_step")
        return dion_vec_last_launch_count()


def vec_step(x, g, m, v=None, *, rule="adamw", lr=None, betas=None, eps=None,
             weight_decay=None, step=1, stream=None):
    """One AdamW or Lion step of the vector (1-D) parameters, on the CUDA library
    (a one-off VecStepPlan; keep a plan for repeated steps).  Returns the launches."""
    return VecStepPlan(x, g, m, v, rule=rule, lr=lr, betas=betas, eps=eps,
                       weight_decay=weight_decay).step(step, stream)

"""The allocation-free step entry point against the regular one (GPU).

dion_step_batched_noalloc serves callers that cannot allocate device memory (a plug-in
handed only the model's buffers by a host program whose allocator it cannot reach, a
loop whose device memory is fixed at start-up): it takes its scratch from a fixed array
inside the library.  Called twice in a row through the C ABI, it must give bit for bit
the X, M, Q and status of dion_step_batched with a caller workspace: both run the same
deterministic kernels on the same inputs, so the tolerance is zero.  This file is
collected last so that a failure here comes after every other test has run.
"""
import ctypes

import pytest
import torch

import rank_orthonormalized_optimizer_b200 as dion
import workloads as W

pytestmark = pytest.mark.gpu

LIB = ctypes.CDLL(dion.LIB_PATH)
NOALLOC = LIB.dion_step_batched_noalloc
NOALLOC.restype = ctypes.c_int32
NOALLOC.argtypes = [ctypes.c_void_p, ctypes.POINTER(dion.BucketPtrs), ctypes.c_int32,
                    ctypes.c_float, ctypes.c_void_p, ctypes.c_void_p]


def _state(wl):
    X = [W.weights(wl, i).cuda() for i in range(len(wl.buckets))]
    M = [W.momentum(wl, i, "cuda") for i in range(len(wl.buckets))]
    Q = [W.right_factor(wl, i).cuda() for i in range(len(wl.buckets))]
    return X, M, Q


@pytest.mark.parametrize("precision", ["bf16", "fp32"])
def test_noalloc_matches_workspace_entry(precision):
    wl = W.custom(f"noalloc_{precision}", [(3, 256, 128, 32), (2, 130, 200, 48)],
                  precision=precision, steps=2)
    opt = dion.DionB200([(b.count, b.m, b.n, b.r) for b in wl.buckets], mu=wl.mu,
                        precision=precision)
    assert opt.workspace_bytes <= dion.STATIC_SCRATCH_BYTES
    Xa, Ma, Qa = _state(wl)
    Xb, Mb, Qb = _state(wl)
    ws = opt.alloc_workspace()
    st_a, st_b = opt.alloc_status(), opt.alloc_status()
    stream = torch.cuda.current_stream()
    for t in range(2):
        G = [W.gradient(wl, i, t).cuda() for i in range(len(wl.buckets))]
        opt.step(Xa, Ma, G, Qa, wl.lr, ws, st_a)
        ptrs = opt._ptrs(Xb, Mb, G, Qb)
        code = NOALLOC(opt._h, ptrs, len(wl.buckets), ctypes.c_float(wl.lr),
                       ctypes.c_void_p(st_b.data_ptr()), ctypes.c_void_p(stream.cuda_stream))
        assert code == dion.OK, dion.dion_last_error()
        torch.cuda.synchronize()
        for i in range(len(wl.buckets)):
            assert torch.equal(Xb[i], Xa[i]) and torch.equal(Mb[i], Ma[i]), (t, i)
            assert torch.equal(Qb[i], Qa[i]), (t, i)
        assert torch.equal(st_a, st_b)


def test_noalloc_rejects_plans_beyond_the_builtin_scratch():
    opt = dion.DionB200([(16, 1024, 1024, 256)], precision="bf16")
    assert opt.workspace_bytes > dion.STATIC_SCRATCH_BYTES
    x = torch.zeros(16, 1024, 1024, device="cuda")
    q = torch.zeros(16, 1024, 256, device="cuda")
    ptrs = opt._ptrs([x], [x.clone()], [x.clone()], [q])
    code = NOALLOC(opt._h, ptrs, 1, ctypes.c_float(0.01), None, None)
    assert code == dion.ERR_WORKSPACE_TOO_SMALL
    assert b"scratch" in dion.dion_last_error()

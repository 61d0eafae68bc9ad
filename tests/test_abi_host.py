"""The C-ABI library loads and exports every entry point include/dion.h declares,
and its host-side checks return the documented status codes (no GPU needed: these
calls stop before any device work)."""
import ctypes
import os
import re
import subprocess

import pytest

import rank_orthonormalized_optimizer_b200 as dion

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "dion.h")


def declared_functions():
    text = open(HEADER).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(dion_[a-z_]+)\s*\(", text)))


def test_header_declares_what_binding_wraps():
    assert declared_functions() == sorted(dion.EXPORTED)


def test_every_declared_symbol_is_exported():
    out = subprocess.run(["nm", "-D", "--defined-only", dion.LIB_PATH], capture_output=True,
                         text=True, check=True).stdout
    exported = set(re.findall(r"\bT (dion_[a-z_]+)$", out, flags=re.M))
    missing = [f for f in declared_functions() if f not in exported]
    assert not missing, missing
    lib = ctypes.CDLL(dion.LIB_PATH)
    for f in declared_functions():
        assert getattr(lib, f) is not None


def test_library_needs_no_driver_to_load():
    out = subprocess.run(["ldd", dion.LIB_PATH], capture_output=True, text=True).stdout
    assert "libcuda.so" not in out          # the runtime is linked statically
    assert "libtorch" not in out


def test_build_targets_sm100a_only():
    import importlib.util
    spec = importlib.util.spec_from_file_location(
        "_dion_build", os.path.join(ROOT, "rank_orthonormalized_optimizer_b200", "build.py"))
    build = importlib.util.module_from_spec(spec)
    spec.loader.exec_module(build)
    assert build.ARCH == ["-gencode", "arch=compute_100a,code=sm_100a"]


def _init(buckets, **kw):
    descs = (dion.BucketDesc * len(buckets))()
    for i, (c, m, n, r) in enumerate(buckets):
        descs[i].count, descs[i].m, descs[i].n, descs[i].r, descs[i].scale = c, m, n, r, 0.0
    o = dion.default_options()
    for k, v in kw.items():
        setattr(o, k, v)
    h = ctypes.c_void_p()
    ws = ctypes.c_size_t()
    code = dion.dion_init(descs, len(buckets), ctypes.byref(o), ctypes.byref(h), ctypes.byref(ws))
    return code, h, ws.value


def test_defaults():
    o = dion.default_options()
    assert abs(o.mu - 0.95) < 1e-7 and o.precision == 1 and o.orth_mode == 0
    assert o.kernel_path == 0 and o.max_wait_spins == 1 << 26


@pytest.mark.parametrize("bucket,code", [
    ((1, 256, 128, 32), dion.OK),
    ((0, 256, 128, 32), dion.ERR_INVALID_ARG),
    ((1, 256, 128, 24), dion.ERR_UNSUPPORTED_SHAPE),     # r % 16
    ((1, 256, 132, 32), dion.ERR_UNSUPPORTED_SHAPE),     # n % 8
    ((1, 16, 128, 32), dion.ERR_UNSUPPORTED_SHAPE),      # r > m
    ((1, 256, 16, 32), dion.ERR_UNSUPPORTED_SHAPE),      # r > n
    ((1, 256, 128, 0), dion.ERR_UNSUPPORTED_SHAPE),
    ((1, 1 << 31, 128, 32), dion.ERR_UNSUPPORTED_SHAPE),  # too large
    ((65536, 32, 16, 16), dion.ERR_UNSUPPORTED_SHAPE),     # too many matrices in one bucket
])
def test_init_shape_checks(bucket, code):
    c, h, ws = _init([bucket])
    assert c == code, dion.dion_last_error()
    if c == dion.OK:
        assert ws > 0
        dion.dion_free(h)
    else:
        assert not h.value and dion.dion_last_error()


@pytest.mark.parametrize("field,value", [("mu", 1.0), ("mu", -0.1), ("precision", 7),
                                         ("orth_mode", 9), ("fallback_cond", 0.5),
                                         ("kernel_path", 3), ("max_wait_spins", 0),
                                         ("rmmc_threshold", float("nan")), ("stack_orth", 2)])
def test_init_option_checks(field, value):
    c, h, _ = _init([(1, 256, 128, 32)], **{field: value})
    assert c == dion.ERR_INVALID_ARG


def test_stacking_shares_the_orthonormalisation_arrays():
    """Buckets of equal m and r stacked: the same arrays, laid out once per stack, so the
    workspace is no larger than without stacking (up to alignment)."""
    shapes = [(3, 256, 128, 32), (2, 256, 384, 32), (2, 200, 136, 16)]
    c0, h0, ws0 = _init(shapes)
    c1, h1, ws1 = _init(shapes, stack_orth=1)
    assert c0 == c1 == dion.OK
    assert ws1 <= ws0
    for h in (h0, h1):
        dion.dion_free(h)


def test_workspace_covers_the_layout():
    c4 = [(128, 4096, 4096, 256), (64, 4096, 11008, 256), (32, 11008, 4096, 256)]
    c, h, ws = _init(c4)
    assert c == dion.OK
    bf16_b = sum(k * m * n * 2 for k, m, n, r in c4)
    # per m x r element: P0, P, P2 (fp32) and the splits of P0 and P (the bf16 GEMM
    # copy of P is the leading plane of P's split)
    factors = sum(k * (m * r * (4 * 3 + 12) + n * r * (4 + 2 + 2 + 2) + r * r * 14)
                  for k, m, n, r in c4)
    assert bf16_b + factors <= ws < 1.1 * (bf16_b + factors) + (1 << 24)
    assert dion.dion_num_matrices(h) == 224
    dion.dion_free(h)
    c, h, ws32 = _init(c4, precision=0)
    assert ws32 > ws                         # fp32 B copy
    dion.dion_free(h)


def test_workspace_recursive_factorisation_scratch():
    # r > 256 on the tensor path: two more [3][count][r][r] bf16 splits (the Gram's and
    # L21's) for the recursive Cholesky factorisation; none at r <= 256, none on the
    # CUDA-core path.  With bf16 GEMM inputs the plans differ otherwise only in the bf16
    # copy of P (on the tensor path the leading plane of P's split) and the column-norm
    # partials: one per block of up to 256 rows of R (written by B^T P) on
    # the tensor path, min(ceil(8 * 148 / count), ceil(n / 16), 256) row ranges on the
    # CUDA-core path.
    def ws_of(r, path):
        c, h, ws = _init([(8, 1024, 1024, r)], kernel_path=path)
        assert c == dion.OK
        dion.dion_free(h)
        return ws

    def parts(r, path):
        ns = 1024 // 256 if path == 0 else min(-(-8 * 148 // 8), 1024 // 16, 256)
        return -(-8 * ns * r * 4 // 1024) * 1024

    for r in (256, 512):
        extra = 2 * 8 * r * r * 6 if r > 256 else 0
        pg = 8 * 1024 * r * 2               # the CUDA-core path's own bf16 copy of P
        assert ws_of(r, 0) - ws_of(r, 1) == extra - pg + parts(r, 0) - parts(r, 1)


def test_step_argument_checks_without_device():
    c, h, ws = _init([(2, 256, 128, 32)])
    assert c == dion.OK
    fake = 1 << 20                           # aligned, never dereferenced
    ptrs = (dion.BucketPtrs * 1)()
    ptrs[0].X = ptrs[0].M = ptrs[0].G = ptrs[0].Q = fake
    step = dion.dion_step_batched
    assert step(None, ptrs, 1, 0.01, fake, ws, None, None) == dion.ERR_NOT_INITIALIZED
    assert step(h, None, 1, 0.01, fake, ws, None, None) == dion.ERR_INVALID_ARG
    assert step(h, ptrs, 2, 0.01, fake, ws, None, None) == dion.ERR_INVALID_ARG
    assert step(h, ptrs, 1, 0.01, None, ws, None, None) == dion.ERR_INVALID_ARG
    assert step(h, ptrs, 1, 0.01, fake, ws - 1, None, None) == dion.ERR_WORKSPACE_TOO_SMALL
    assert step(h, ptrs, 1, 0.01, fake + 8, ws, None, None) == dion.ERR_MISALIGNED
    assert step(h, ptrs, 1, 0.01, fake, ws, fake + 2, None) == dion.ERR_MISALIGNED
    ptrs[0].Q = fake + 4
    assert step(h, ptrs, 1, 0.01, fake, ws, None, None) == dion.ERR_MISALIGNED
    ptrs[0].Q = None
    assert step(h, ptrs, 1, 0.01, fake, ws, None, None) == dion.ERR_INVALID_ARG
    ptrs[0].Q = fake
    try:
        import torch
        no_gpu = not torch.cuda.is_available()
    except Exception:
        no_gpu = True
    if no_gpu:                               # valid arguments reach the device check
        assert step(h, ptrs, 1, 0.01, fake, ws, None, None) in (dion.ERR_CUDA, dion.ERR_DEVICE)
    assert dion.dion_free(h) == dion.OK


def test_status_strings_and_views():
    for code in range(9):
        assert dion.dion_status_string(code) and dion.dion_status_string(code) != b"unknown status"
    c, h, ws = _init([(3, 64, 32, 16)])
    ptr, nb = ctypes.c_void_p(), ctypes.c_size_t()
    assert dion.dion_workspace_view(h, 0, dion.VIEW_P, 1 << 20, ctypes.byref(ptr),
                                    ctypes.byref(nb)) == dion.OK
    assert nb.value == 3 * 64 * 16 * 4 and ptr.value >= 1 << 20
    assert dion.dion_workspace_view(h, 1, dion.VIEW_P, 1 << 20, ctypes.byref(ptr),
                                    ctypes.byref(nb)) == dion.ERR_INVALID_ARG
    assert dion.dion_last_launch_count(h) == 0
    dion.dion_free(h)


def test_plain_c_caller(tmp_path):
    """include/dion.h compiles as C99 and a C program links the library and gets the
    documented codes back (no device touched)."""
    import shutil
    cc = shutil.which("gcc") or shutil.which("cc")
    if cc is None:
        pytest.skip("no C compiler")
    exe = tmp_path / "abi_check"
    libdir = os.path.dirname(dion.LIB_PATH)
    subprocess.run([cc, "-std=c99", "-Wall", "-Werror", "-pedantic",
                    "-I", os.path.join(ROOT, "include"),
                    os.path.join(ROOT, "tests", "c", "abi_check.c"),
                    "-L", libdir, "-ldion_b200", f"-Wl,-rpath,{libdir}", "-o", str(exe)],
                   check=True, capture_output=True, text=True)
    out = subprocess.run([str(exe)], capture_output=True, text=True)
    assert out.returncode == 0 and out.stdout.strip() == "ok", out.stdout + out.stderr


def test_product_and_oracle_share_nothing():
    """The package (binding, build script, CUDA sources) never names the oracle, and the
    oracle never names the package or its library: the two meet only through the seeded
    inputs of `workloads`, which holds none of the method's arithmetic."""
    import glob
    pkg = os.path.join(ROOT, "rank_orthonormalized_optimizer_b200")
    product = [f for pat in ("*.py", "csrc/*") for f in glob.glob(os.path.join(pkg, pat))]
    product.append(os.path.join(ROOT, "include", "dion.h"))
    for f in product:
        text = open(f, errors="replace").read()
        assert not re.search(r"\boracle\b", text, flags=re.I), f
    for f in glob.glob(os.path.join(ROOT, "oracle", "*.py")):
        text = open(f).read()
        assert "rank_orthonormalized_optimizer_b200" not in text and "libdion" not in text, f
        assert not re.search(r"^\s*(import|from)\s+(torch|rank_orth|ctypes)", text, flags=re.M), f
    wl = open(os.path.join(ROOT, "workloads", "__init__.py")).read()
    assert not re.search(r"^\s*(import|from)\s+(oracle|rank_orth)", wl, flags=re.M)

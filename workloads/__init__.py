"""Seeded synthetic inputs for the batched Dion step.

This module holds shapes, hyper-parameters and random-number recipes, and
nothing of the optimizer step itself.  Both the CPU oracle (through the
tests and the bench) and the CUDA path draw their inputs from here; the two
never share any code of the step.

Shapes follow the weight matrices of decoder-only transformers (attention
projections and MLP matrices, stacked by identical shape in the spirit of
the 3-D block stacking of "DASH: Faster Shampoo via Batched Block
Preconditioning and Efficient Inverse-Root Solvers", Methodologie section 1).

Every tensor is seeded from (workload, bucket, slot, kind, step), so any
single matrix of a bucket can be regenerated on its own.  Values are drawn
with torch generators, on the CPU for small cases and on the GPU for the
large ones; a test always copies the same drawn tensor to both sides.
"""
from __future__ import annotations

import hashlib
from dataclasses import dataclass, field

import torch


@dataclass(frozen=True)
class Bucket:
    """``count`` matrices of identical shape ``m x n`` updated at rank ``r``."""
    count: int
    m: int
    n: int
    r: int

    @property
    def params(self) -> int:
        return self.count * self.m * self.n


@dataclass(frozen=True)
class Workload:
    name: str
    buckets: tuple
    precision: str          # GEMM operand type on the GPU: "fp32" or "bf16"
    mu: float
    lr: float
    steps: int              # steps a parity check runs
    grad: str               # gradient recipe, see ``gradient``
    note: str = ""
    sample_slots: tuple = field(default=())   # slots the oracle checks at full size

    @property
    def params(self) -> int:
        return sum(b.params for b in self.buckets)


def _sweep(r: int) -> Workload:
    return Workload(
        name=f"square_8x8192_r{r}",
        buckets=(Bucket(8, 8192, 8192, r),),
        precision="fp32", mu=0.95, lr=0.01, steps=10, grad="gaussian",
        note="rank sweep on 8 stacked 8192x8192 fp32 matrices, Gaussian G",
        sample_slots=(0, 7))


WORKLOADS = {
    w.name: w for w in [
        Workload(
            name="single_256x128_r32",
            buckets=(Bucket(1, 256, 128, 32),),
            precision="fp32", mu=0.95, lr=0.01, steps=10, grad="gaussian",
            note="one 256x128 fp32 matrix, rank 32, fresh Gaussian G each step"),
        Workload(
            name="fullrank_16x1024x1024",
            buckets=(Bucket(16, 1024, 1024, 1024),),
            precision="fp32", mu=0.95, lr=0.01, steps=50, grad="fixed_sqrt_spectrum",
            note="full rank on a fixed B = U diag(k^-1/2) V^T; M reset to 0 and G = B each step"),
        Workload(
            name="transformer_h2048_l24_r256",
            buckets=(Bucket(24, 2048, 6144, 256), Bucket(24, 2048, 2048, 256),
                     Bucket(24, 2048, 8192, 256), Bucket(24, 8192, 2048, 256)),
            precision="bf16", mu=0.95, lr=0.01, steps=10, grad="lowrank64_plus_noise",
            note="1.3B-like: 24 layers, hidden 2048 (Wqkv, Wo, W1, W2), rank fraction 1/8",
            sample_slots=(0, 23)),
        Workload(
            name="transformer_h4096_l32_ff11008_r256",
            buckets=(Bucket(128, 4096, 4096, 256), Bucket(64, 4096, 11008, 256),
                     Bucket(32, 11008, 4096, 256)),
            precision="bf16", mu=0.95, lr=0.01, steps=10, grad="gaussian_1e-3",
            note="7B-like: 32 layers, hidden 4096, MLP 11008 (Wq/Wk/Wv/Wo, W_gate/W_up, W_down), "
                 "rank fraction 1/16",
            sample_slots=(0, -1)),
        Workload(
            name="stack_16x4096x4096_r256",
            buckets=(Bucket(16, 4096, 4096, 256),),
            precision="bf16", mu=0.95, lr=0.01, steps=3, grad="gaussian_1e-3",
            note="16 attention-sized 4096x4096 matrices, rank 256: a 3 GB case for profiling "
                 "(inputs larger than L2)",
            sample_slots=(0, 15)),
        # the two MLP shapes of the 7B-like workload, 4 matrices each (2.2 GB of fp32
        # X, M, G, larger than L2): cases small enough for a profiler to capture one
        # launch of each kernel at the headline's shapes
        Workload(
            name="mlp_up_4x4096x11008_r256",
            buckets=(Bucket(4, 4096, 11008, 256),),
            precision="bf16", mu=0.95, lr=0.01, steps=3, grad="gaussian_1e-3",
            note="4 of the 7B-like W_gate/W_up shape (4096x11008), rank 256: for profiling",
            sample_slots=(0, 3)),
        Workload(
            name="mlp_down_4x11008x4096_r256",
            buckets=(Bucket(4, 11008, 4096, 256),),
            precision="bf16", mu=0.95, lr=0.01, steps=3, grad="gaussian_1e-3",
            note="4 of the 7B-like W_down shape (11008x4096), rank 256: for profiling",
            sample_slots=(0, 3)),
    ] + [_sweep(r) for r in (64, 128, 256, 512, 1024, 2048, 4096, 8192)]
}

#: the workload a throughput figure is quoted on (7B-like transformer shapes)
HEADLINE = "transformer_h4096_l32_ff11008_r256"

_KINDS = {"X": 1, "Q": 2, "G": 3, "U": 4, "V": 5, "M": 6, "S": 7}


def seed_for(workload: str, bucket: int, slot: int, kind: str, step: int = 0) -> int:
    """Stable 63-bit seed of one tensor (independent of Python's hash salt)."""
    key = f"{workload}|{bucket}|{slot}|{_KINDS[kind]}|{step}".encode()
    return int.from_bytes(hashlib.sha256(key).digest()[:8], "little") & ((1 << 63) - 1)


def _randn(shape, seed: int, device) -> torch.Tensor:
    dev = torch.device(device)
    g = torch.Generator(device=dev)
    g.manual_seed(seed)
    return torch.randn(shape, generator=g, device=dev, dtype=torch.float32)


def _slots(b: Bucket, slots):
    if slots is None:
        return list(range(b.count))
    return [s % b.count for s in slots]


def weights(wl: Workload, bi: int, device="cpu", slots=None) -> torch.Tensor:
    """X ~ N(0,1), one [m, n] matrix per slot -> [len(slots), m, n] fp32."""
    b = wl.buckets[bi]
    return torch.stack([_randn((b.m, b.n), seed_for(wl.name, bi, s, "X"), device)
                        for s in _slots(b, slots)])


def momentum(wl: Workload, bi: int, device="cpu", slots=None) -> torch.Tensor:
    """M = 0 at the start."""
    b = wl.buckets[bi]
    return torch.zeros((len(_slots(b, slots)), b.m, b.n), dtype=torch.float32,
                       device=device)


def right_factor(wl: Workload, bi: int, device="cpu", slots=None) -> torch.Tensor:
    """Q0: uniform random unit columns (Gaussian draws scaled to unit length), [k, n, r]."""
    b = wl.buckets[bi]
    out = []
    for s in _slots(b, slots):
        z = _randn((b.n, b.r), seed_for(wl.name, bi, s, "Q"), device).double()
        out.append((z / z.square().sum(0, keepdim=True).sqrt()).float())
    return torch.stack(out)


def _orthonormal(rows: int, cols: int, seed: int, device) -> torch.Tensor:
    """Random orthonormal columns: the Q factor of a Gaussian, in fp64."""
    z = _randn((rows, cols), seed, device).double()
    q, rr = torch.linalg.qr(z)
    return q * torch.where(torch.diagonal(rr) >= 0, 1.0, -1.0).to(q.dtype)


def _fixed_low_rank(wl, bi, s, device, k: int, spectrum) -> torch.Tensor:
    b = wl.buckets[bi]
    u = _orthonormal(b.m, k, seed_for(wl.name, bi, s, "U"), device)
    v = _orthonormal(b.n, k, seed_for(wl.name, bi, s, "V"), device)
    return (u * spectrum.to(device)) @ v.T


def gradient(wl: Workload, bi: int, step: int, device="cpu", slots=None) -> torch.Tensor:
    """G for one step, [len(slots), m, n] fp32.

    Recipes:
      gaussian              N(0,1), fresh every step
      gaussian_1e-3         1e-3 * N(0,1), fresh every step
      fixed_sqrt_spectrum   U diag(k^-1/2) V^T with Haar U, V drawn once per slot
                            (the same every step)
      lowrank64_plus_noise  U64 diag(1/k) V64^T (U, V drawn once per slot)
                            + 0.1 * N(0,1) drawn fresh every step
    """
    b = wl.buckets[bi]
    out = []
    for s in _slots(b, slots):
        if wl.grad == "gaussian":
            g = _randn((b.m, b.n), seed_for(wl.name, bi, s, "G", step), device)
        elif wl.grad == "gaussian_1e-3":
            g = _randn((b.m, b.n), seed_for(wl.name, bi, s, "G", step), device) * 1e-3
        elif wl.grad == "fixed_sqrt_spectrum":
            k = min(b.m, b.n)
            spec = torch.arange(1, k + 1, dtype=torch.float64) ** -0.5
            g = _fixed_low_rank(wl, bi, s, device, k, spec).float()
        elif wl.grad == "lowrank64_plus_noise":
            spec = 1.0 / torch.arange(1, 65, dtype=torch.float64)
            low = _fixed_low_rank(wl, bi, s, device, 64, spec)
            g = (low + 0.1 * _randn((b.m, b.n), seed_for(wl.name, bi, s, "G", step),
                                    device).double()).float()
        else:
            raise ValueError(f"unknown gradient recipe {wl.grad!r}")
        out.append(g)
    return torch.stack(out)


def fixed_b_svd(wl: Workload, bi: int, slot: int, device="cpu"):
    """(U, sigma, V) of the fixed B of ``fixed_sqrt_spectrum`` (fp64), for polar-factor checks."""
    b = wl.buckets[bi]
    k = min(b.m, b.n)
    u = _orthonormal(b.m, k, seed_for(wl.name, bi, slot, "U"), device)
    v = _orthonormal(b.n, k, seed_for(wl.name, bi, slot, "V"), device)
    return u, torch.arange(1, k + 1, dtype=torch.float64) ** -0.5, v


def custom(name: str, buckets, precision="fp32", mu=0.95, lr=0.01, steps=3,
           grad="gaussian") -> Workload:
    """A small ad-hoc workload (odd shapes for edge-case tests)."""
    return Workload(name=name, buckets=tuple(Bucket(*b) for b in buckets),
                    precision=precision, mu=mu, lr=lr, steps=steps, grad=grad)


# ------------------------------------------------------------ vector (1-D) parameters
@dataclass(frozen=True)
class VectorWorkload:
    """The 1-D parameters of a model (biases, normalisation gains), one entry per
    parameter tensor, stepped by AdamW or Lion beside the Dion step of its matrices."""
    name: str
    sizes: tuple
    lr: float = 1e-3

    @property
    def params(self) -> int:
        return sum(self.sizes)


VECTOR_WORKLOADS = {
    # the RMSNorm gains of the 7B-like decoder: two per layer and the final one
    "norms_h4096_l32": VectorWorkload("norms_h4096_l32", (4096,) * 65),
    # a bank larger than L2 (64 x 4 Mi elements, 1 GiB per state array)
    "vectors_64x4Mi": VectorWorkload("vectors_64x4Mi", (4 << 20,) * 64),
    # the same with 16 tensors (256 MiB per state array, still twice L2): for profiling
    "vectors_16x4Mi": VectorWorkload("vectors_16x4Mi", (4 << 20,) * 16),
}


def vector_state(vw: VectorWorkload, i: int, step: int = 0, device="cpu"):
    """(x, g, m, v) of parameter i, fp32 1-D: x ~ N(0, 1), g ~ 1e-3 N(0, 1) fresh each
    step, m ~ 1e-3 N(0, 1), v = (1e-3 N(0, 1))^2 (non-negative, as a second moment)."""
    n = vw.sizes[i]
    x = _randn((n,), seed_for(vw.name, i, 0, "X"), device)
    g = _randn((n,), seed_for(vw.name, i, 0, "G", step), device) * 1e-3
    m = _randn((n,), seed_for(vw.name, i, 0, "M"), device) * 1e-3
    v = (_randn((n,), seed_for(vw.name, i, 0, "S"), device) * 1e-3) ** 2
    return x, g, m, v

"""Seeded synthetic inputs shared by the tests, the benchmark and the oracle runs.

This module draws random numbers and casts them; it holds none of the method's
arithmetic (no distances, no kernels, no sums).  Both the CUDA path and the CPU
oracle are handed the very same quantised values it produces.

Recipe (one generator per workload, ``torch.Generator('cpu')`` seeded with
``1000 + workload id``; draw order x, y, w, g; every draw in float64, then a
round-to-nearest-even cast to the workload's dtype):

* ``d3_10k``  / ``d3_100k``: x, y ~ N(0, 1)^3, w ~ N(0, 1) signed, tau = 1
* ``d3_1m_lse``: x, y ~ U[0, 1)^3, w ~ U(0.5, 1.5), tau = 100
* ``d32_c32``: x, y ~ N(0, 1/D)^D (coordinate variance 1/D), w ~ N(0, 1), tau = 1
* ``d32_c1_bwd``: as ``d32_c32`` with C = 1, plus an upstream gradient g ~ N(0, 1)
* ``b64_d32_f16`` / ``b64_d32_f32`` / ``b64_d128_f32``: B = 64, M = N = 16384, C = 1,
  x, y ~ N(0, 1/D)^D, w ~ N(0, 1), tau = 1 -- points of the D sweeps (fp16 and fp32)
* ``d32_c32_f32``: ``d32_c32`` in fp32 -- a point of the fp32 N sweep

The shapes are those of the Gaussian-product runs of "Kernel matrix reduction"
(Variants: D = 3, float32, 10k / 100k / 1M points) and of the sweeps in the
figures of "Fast Gauss Sums via Flash Attention" (Figures 1-2: B = 4, D = 32,
C = 32 or 1, fp16; Figures 3-4: D sweeps at B = 64, C = 1, N = 16384 in fp16 and
fp32; Figure 5: an N sweep at B = 4, D = 32, C = 32 in fp32).  No dataset is
involved.
"""
from dataclasses import dataclass

import torch

_DT = {"f32": torch.float32, "f16": torch.float16, "bf16": torch.bfloat16, "f64": torch.float64}


@dataclass(frozen=True)
class Workload:
    wid: int
    name: str
    ops: tuple            # which entry points the workload exercises
    B: int
    M: int
    N: int
    D: int
    C: int
    dtype: str            # "f32" | "f16" | "bf16"
    tau: float
    dist_xy: str          # "normal1" | "uniform01" | "normal_invD"
    dist_w: str           # "normal1" | "uniform_half"
    with_g: bool = False

    @property
    def pairs(self):
        return self.B * self.M * self.N

    def describe(self):
        return (f"{self.name}: B={self.B} M={self.M} N={self.N} D={self.D} C={self.C} "
                f"{self.dtype} tau={self.tau:g} ops={'+'.join(self.ops)}")


WORKLOADS = {
    1: Workload(1, "d3_10k", ("sum",), 1, 10_000, 10_000, 3, 1, "f32", 1.0, "normal1", "normal1"),
    2: Workload(2, "d3_100k", ("sum",), 1, 100_000, 100_000, 3, 1, "f32", 1.0, "normal1", "normal1"),
    3: Workload(3, "d3_1m_lse", ("sum", "lse"), 1, 1_000_000, 1_000_000, 3, 1, "f32", 100.0,
                "uniform01", "uniform_half"),
    4: Workload(4, "d32_c32", ("sum",), 4, 65_536, 65_536, 32, 32, "f16", 1.0, "normal_invD",
                "normal1"),
    5: Workload(5, "d32_c1_bwd", ("sum", "bwd"), 4, 16_384, 16_384, 32, 1, "f16", 1.0,
                "normal_invD", "normal1", with_g=True),
    6: Workload(6, "b64_d32_f16", ("sum",), 64, 16_384, 16_384, 32, 1, "f16", 1.0,
                "normal_invD", "normal1"),
    7: Workload(7, "b64_d32_f32", ("sum",), 64, 16_384, 16_384, 32, 1, "f32", 1.0,
                "normal_invD", "normal1"),
    8: Workload(8, "b64_d128_f32", ("sum",), 64, 16_384, 16_384, 128, 1, "f32", 1.0,
                "normal_invD", "normal1"),
    9: Workload(9, "d32_c32_f32", ("sum",), 4, 65_536, 65_536, 32, 32, "f32", 1.0,
                "normal_invD", "normal1"),
}
BY_NAME = {w.name: w for w in WORKLOADS.values()}


def _draw(gen, shape, dist, D):
    if dist == "normal1":
        return torch.randn(shape, generator=gen, dtype=torch.float64)
    if dist == "normal_invD":
        return torch.randn(shape, generator=gen, dtype=torch.float64) * (1.0 / D) ** 0.5
    if dist == "uniform01":
        return torch.rand(shape, generator=gen, dtype=torch.float64)
    if dist == "uniform_half":
        return torch.rand(shape, generator=gen, dtype=torch.float64) + 0.5
    raise ValueError(dist)


def make_inputs(w, seed=None, **overrides):
    """Draw the inputs of workload ``w`` (a Workload, its id or its name).

    ``overrides`` may replace B, M, N, D, C, dtype, tau (for reduced or odd-shaped
    variants of the same recipe).  Returns a dict with the quantised tensors
    ``x, y, w`` (and ``g`` when the workload has an upstream gradient) on the CPU
    in the workload dtype, ``g`` always float32, plus ``tau`` and the workload.
    """
    if not isinstance(w, Workload):
        w = WORKLOADS[w] if isinstance(w, int) else BY_NAME[w]
    p = dict(B=w.B, M=w.M, N=w.N, D=w.D, C=w.C, dtype=w.dtype, tau=w.tau)
    p.update(overrides)
    gen = torch.Generator("cpu").manual_seed(1000 + w.wid if seed is None else seed)
    B, M, N, D, C = p["B"], p["M"], p["N"], p["D"], p["C"]
    dt = _DT[p["dtype"]]
    x = _draw(gen, (B, M, D), w.dist_xy, D).to(dt)
    y = _draw(gen, (B, N, D), w.dist_xy, D).to(dt)
    wt = _draw(gen, (B, N, C), w.dist_w, D).to(dt)
    out = dict(x=x, y=y, w=wt, tau=float(p["tau"]), workload=w, **{k: p[k] for k in "BMNDC"},
               dtype=p["dtype"])
    if w.with_g or overrides.get("with_g", False):
        out["g"] = torch.randn((B, M, C), generator=gen, dtype=torch.float64).to(torch.float32)
    return out


def as_f64(t):
    """The quantised values of a tensor, widened to a float64 numpy array."""
    return t.detach().to("cpu").to(torch.float64).numpy()


def sample_rows(M, n, seed):
    """A seeded, sorted subset of ``n`` distinct row indices out of ``M``."""
    if n >= M:
        return torch.arange(M, dtype=torch.int64)
    gen = torch.Generator("cpu").manual_seed(seed)
    return torch.sort(torch.randperm(M, generator=gen)[:n]).values

"""gauss_sum_fwd_noalloc: the allocation-free entry point, for callers of this
library that cannot allocate device memory for a workspace (a plugin whose host
application owns the device-memory budget, a loop that must not block in the
CUDA allocator, a process under a hard memory cap).  It must give the same
results as gauss_sum_fwd with a caller workspace, call after call, while using
the library's fixed 32 MiB scratch array.

This file is collected last on purpose: if it fails, a run that stops at the
first failure has already run every other test.  It passes both alone in a
fresh process and after the rest of the suite (it relies on no earlier state).
"""
import ctypes

import numpy as np
import pytest
import torch

import synth

pytestmark = pytest.mark.gpu

TOL = {"f32": 1e-5, "f16": 3e-3}
SCRATCH_BYTES = 32 << 20


def _lib():
    import pairwise_reductions_b200 as gs
    return gs, gs.library()


def _rel(a, b):
    a, b = a.double().cpu().numpy().ravel(), b.double().cpu().numpy().ravel()
    return float(np.linalg.norm(a - b) / max(np.linalg.norm(b), 1e-300))


def _call_noalloc(lib, d, out, inp, dt):
    p = lambda t: ctypes.c_void_p(t.data_ptr())
    s = ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    B, M, N, D, C = (inp[k] for k in "BMNDC")
    return lib.gauss_sum_fwd_noalloc(p(d["x"]), p(d["y"]), p(d["w"]), p(out), B, M, N, D, C,
                                     inp["tau"], dt, s)


# fp32 with column splits (scratch = split partials) and fp16 on the tensor-core
# path (scratch = packed operands, norms, transposed values and split partials)
CASES = [
    ("f32", dict(wid=1, B=1, M=10_000, N=10_000, D=3, C=1, dtype="f32")),
    ("f32", dict(wid=1, B=2, M=3_001, N=20_000, D=3, C=2, dtype="f32")),
    ("f16", dict(wid=4, B=1, M=20_000, N=20_000, D=32, C=32, dtype="f16")),
    ("f16", dict(wid=5, B=2, M=4_096, N=9_000, D=32, C=1, dtype="f16")),
]


@pytest.mark.parametrize("kind,case", CASES, ids=[f"{k}-{c['B']}x{c['M']}x{c['N']}x{c['D']}x{c['C']}"
                                                  for k, c in CASES])
def test_noalloc_matches_the_workspace_entry_point_twice(kind, case):
    gs, lib = _lib()
    case = dict(case)
    wid = case.pop("wid")
    inp = synth.make_inputs(wid, seed=77, **case)
    dt = {"f32": gs.GS_F32, "f16": gs.GS_F16}[kind]
    need = gs.workspace_bytes(gs.GS_OP_SUM, inp["B"], inp["M"], inp["N"], inp["D"], inp["C"], dt)
    assert 0 < need <= SCRATCH_BYTES   # the case really exercises the scratch array
    d = {k: inp[k].cuda() for k in "xyw"}
    ref = gs.gauss_sum_fwd(d["x"], d["y"], d["w"], inp["tau"])
    for _ in range(2):   # the array keeps the previous call's contents
        out = torch.full((inp["B"], inp["M"], inp["C"]), float("nan"), device="cuda")
        assert _call_noalloc(lib, d, out, inp, dt) == 0
        torch.cuda.synchronize()
        assert torch.isfinite(out).all()
        assert _rel(out, ref) <= TOL[kind], _rel(out, ref)
    assert gs.last_device_error() == 0


def test_noalloc_rejects_calls_beyond_its_scratch():
    gs, lib = _lib()
    B, M, N, D, C = 4, 65_536, 65_536, 32, 32   # needs ~84 MB of scratch
    assert gs.workspace_bytes(gs.GS_OP_SUM, B, M, N, D, C, gs.GS_F16) > SCRATCH_BYTES
    x = torch.zeros(B, M, D, dtype=torch.float16, device="cuda")
    w = torch.zeros(B, N, C, dtype=torch.float16, device="cuda")
    out = torch.zeros(B, M, C, device="cuda")
    p = lambda t: ctypes.c_void_p(t.data_ptr())
    s = ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    st = lib.gauss_sum_fwd_noalloc(p(x), p(x), p(w), p(out), B, M, N, D, C, 1.0, gs.GS_F16, s)
    assert st == 4, gs.status_string(st)   # GS_ERR_WORKSPACE
    # argument errors are reported exactly as by gauss_sum_fwd
    assert lib.gauss_sum_fwd_noalloc(p(x), p(x), p(w), p(out), B, M, N, D, C, -1.0, gs.GS_F16, s) == 1

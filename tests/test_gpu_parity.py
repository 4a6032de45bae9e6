"""CUDA path against the CPU oracle, element by element, on the same seeded
inputs, through the C ABI (via the ctypes binding).

Tolerances (relative L2 over the compared outputs): 1e-5 for float32 inputs,
3e-3 for float16 / bfloat16 inputs with float32 accumulation.  Full-size
workloads run on the GPU in the launch configuration the benchmark times and
are compared on seeded row samples the oracle evaluates one by one.
"""
import numpy as np
import pytest
import torch

import oracle
import synth
from knn_check import knn_valid_under_exact_distances

pytestmark = pytest.mark.gpu

TOL = {"f32": 1e-5, "f16": 3e-3, "bf16": 3e-3}


def gs():
    import pairwise_reductions_b200 as m
    return m


def rel_l2(a, b):
    a = np.asarray(a, dtype=np.float64).ravel()
    b = np.asarray(b, dtype=np.float64).ravel()
    return float(np.linalg.norm(a - b) / max(np.linalg.norm(b), 1e-300))


def dev(inp):
    return {k: inp[k].cuda() for k in ("x", "y", "w", "g") if k in inp}


def f64(inp, k):
    return synth.as_f64(inp[k])


# ------------------------------------------------------------------ the five workloads
def test_d3_10k_full():
    inp = synth.make_inputs(1)
    d = dev(inp)
    out = gs().gauss_sum_fwd(d["x"], d["y"], d["w"], inp["tau"]).cpu().numpy()
    ref = oracle.gauss_sum(f64(inp, "x"), f64(inp, "y"), f64(inp, "w"), inp["tau"])
    assert rel_l2(out, ref) <= TOL["f32"], rel_l2(out, ref)


def test_d3_100k_sampled_rows():
    inp = synth.make_inputs(2)
    d = dev(inp)
    out = gs().gauss_sum_fwd(d["x"], d["y"], d["w"], inp["tau"]).cpu().numpy()
    rows = synth.sample_rows(inp["M"], 3000, seed=7).numpy()
    ref = oracle.gauss_sum(f64(inp, "x"), f64(inp, "y"), f64(inp, "w"), inp["tau"], rows=rows)
    assert rel_l2(out[:, rows], ref) <= TOL["f32"], rel_l2(out[:, rows], ref)


def test_d3_1m_sum_and_lse_sampled_rows():
    inp = synth.make_inputs(3)
    d = dev(inp)
    rows = synth.sample_rows(inp["M"], 768, seed=8).numpy()
    x, y, w = f64(inp, "x"), f64(inp, "y"), f64(inp, "w")
    out = gs().gauss_sum_fwd(d["x"], d["y"], d["w"], inp["tau"]).cpu().numpy()
    ref = oracle.gauss_sum(x, y, w, inp["tau"], rows=rows)
    assert rel_l2(out[:, rows], ref) <= TOL["f32"], rel_l2(out[:, rows], ref)
    lse = gs().gauss_lse_fwd(d["x"], d["y"], d["w"], inp["tau"]).cpu().numpy()
    ref_l = oracle.gauss_lse(x, y, w, inp["tau"], rows=rows)
    assert rel_l2(lse[:, rows], ref_l) <= TOL["f32"], rel_l2(lse[:, rows], ref_l)
    # the stricter check: exp(lse) against exp(oracle lse) is a relative check of the sum
    assert rel_l2(np.exp(lse[:, rows]), np.exp(ref_l)) <= TOL["f32"]


def test_d32_c32_f16_sampled_rows():
    inp = synth.make_inputs(4)
    d = dev(inp)
    out = gs().gauss_sum_fwd(d["x"], d["y"], d["w"], inp["tau"]).cpu().numpy()
    rows = synth.sample_rows(inp["M"], 160, seed=9).numpy()
    ref = oracle.gauss_sum(f64(inp, "x"), f64(inp, "y"), f64(inp, "w"), inp["tau"], rows=rows)
    assert rel_l2(out[:, rows], ref) <= TOL["f16"], rel_l2(out[:, rows], ref)


def test_d32_c1_f16_fwd_bwd_sampled():
    inp = synth.make_inputs(5)
    d = dev(inp)
    x, y, w, g = (f64(inp, k) for k in "xywg")
    out = gs().gauss_sum_fwd(d["x"], d["y"], d["w"], inp["tau"]).cpu().numpy()
    gx, gw = gs().gauss_sum_bwd(d["x"], d["y"], d["w"], d["g"], inp["tau"])
    gx, gw = gx.cpu().numpy(), gw.cpu().numpy()
    rows = synth.sample_rows(inp["M"], 512, seed=10).numpy()
    wrows = synth.sample_rows(inp["N"], 512, seed=11).numpy()
    ref = oracle.gauss_sum(x, y, w, inp["tau"], rows=rows)
    assert rel_l2(out[:, rows], ref) <= TOL["f16"], rel_l2(out[:, rows], ref)
    rgx, rgw = oracle.gauss_sum_bwd(x, y, w, g, inp["tau"], rows=rows, wrows=wrows)
    assert rel_l2(gx[:, rows], rgx) <= TOL["f16"], rel_l2(gx[:, rows], rgx)
    assert rel_l2(gw[:, wrows], rgw) <= TOL["f16"], rel_l2(gw[:, wrows], rgw)


@pytest.mark.parametrize("name,nrows", [("b64_d32_f16", 24), ("b64_d32_f32", 24),
                                        ("b64_d128_f32", 16), ("d32_c32_f32", 96)])
def test_bench_workload_full_size_sampled(name, nrows):
    """The other workloads bench.py times (the points of "Fast Gauss Sums via Flash
    Attention", Figures 3-5: B = 64 batches of 16384 x 16384 at D = 32 and 128,
    fp16 and fp32; B = 4 of 65536 x 65536 with 32 channels, fp32), at full size in
    the launch configuration the benchmark uses, against the oracle on sampled rows
    of every batch."""
    w = synth.BY_NAME[name]
    inp = synth.make_inputs(w)
    d = dev(inp)
    out = gs().gauss_sum_fwd(d["x"], d["y"], d["w"], inp["tau"]).cpu().numpy()
    del d
    rows = synth.sample_rows(inp["M"], nrows, seed=12).numpy()
    ref = oracle.gauss_sum(f64(inp, "x"), f64(inp, "y"), f64(inp, "w"), inp["tau"], rows=rows)
    tol = TOL["f32"] if w.dtype == "f32" else TOL["f16"]
    assert rel_l2(out[:, rows], ref) <= tol, rel_l2(out[:, rows], ref)


def test_d32_c1_f16_saved_pair_full_size():
    """The call pair the benchmark times for this workload (B=4, M=N=16384, D=32,
    C=1, fp16): gauss_sum_fwd_saved then gauss_sum_bwd_saved (`--two-call`), at
    full size and in the same launch configuration, against the oracle on
    sampled rows and sources; bit for bit against the separate backward entry
    point, which runs the same passes; and the one-sweep gauss_sum_fwd_bwd."""
    inp = synth.make_inputs(5)
    d = dev(inp)
    m = gs()
    out, saved = m.gauss_sum_fwd_saved(d["x"], d["y"], d["w"], inp["tau"])
    gx, gw = m.gauss_sum_bwd_saved(d["x"], d["y"], d["w"], d["g"], saved, inp["tau"])
    x, y, w, g = (f64(inp, k) for k in "xywg")
    rows = synth.sample_rows(inp["M"], 512, seed=40).numpy()
    wrows = synth.sample_rows(inp["N"], 512, seed=41).numpy()
    ref = oracle.gauss_sum(x, y, w, inp["tau"], rows=rows)
    o = out.cpu().numpy()
    assert rel_l2(o[:, rows], ref) <= TOL["f16"], rel_l2(o[:, rows], ref)
    rgx, rgw = oracle.gauss_sum_bwd(x, y, w, g, inp["tau"], rows=rows, wrows=wrows)
    gxn, gwn = gx.cpu().numpy(), gw.cpu().numpy()
    assert rel_l2(gxn[:, rows], rgx) <= TOL["f16"], rel_l2(gxn[:, rows], rgx)
    assert rel_l2(gwn[:, wrows], rgw) <= TOL["f16"], rel_l2(gwn[:, wrows], rgw)
    bx, bw = m.gauss_sum_bwd(d["x"], d["y"], d["w"], d["g"], inp["tau"])
    assert torch.equal(bx, gx) and torch.equal(bw, gw)
    # the one-sweep call the benchmark times by default for this workload: the
    # sum and grad_x bit for bit those of the saved pair, grad_w (P^T g from the
    # same sweep) against the oracle on the sampled sources
    fo, fx, fw = m.gauss_sum_fwd_bwd(d["x"], d["y"], d["w"], d["g"], inp["tau"])
    assert torch.equal(fo, out) and torch.equal(fx, gx)
    fwn = fw.cpu().numpy()
    assert rel_l2(fwn[:, wrows], rgw) <= TOL["f16"], rel_l2(fwn[:, wrows], rgw)


# ------------------------------------------------------------------ odd shapes, both paths
F32_SHAPES = [  # B, M, N, D, C
    (1, 1, 1, 3, 1), (1, 1, 777, 3, 1), (1, 777, 1, 3, 1), (2, 777, 1301, 3, 1),
    (1, 513, 257, 1, 2), (1, 1000, 999, 5, 3), (1, 300, 2000, 8, 9), (3, 129, 4097, 2, 4),
    (1, 2049, 3000, 7, 8), (2, 100, 600, 4, 16),
]
HALF_SHAPES = [
    (1, 1, 1, 32, 1), (1, 1, 300, 32, 1), (2, 300, 1000, 32, 32), (1, 257, 129, 16, 33),
    (1, 200, 700, 5, 1), (1, 100, 300, 100, 16), (2, 130, 260, 48, 130), (1, 511, 640, 62, 64),
    (1, 70, 1200, 63, 3), (1, 129, 257, 126, 96), (1, 300, 700, 127, 1), (2, 257, 390, 128, 50),
    # D + 2 at and just past a multiple of 16 (the similarity MMA's K steps)
    (1, 300, 500, 14, 2), (1, 260, 530, 30, 4), (1, 200, 400, 31, 1), (1, 150, 300, 46, 1),
    # one and two column tiles with several channels (the three-buffer S ring's edges)
    (1, 300, 100, 32, 8), (2, 130, 128, 20, 40), (1, 257, 250, 62, 64),
]
# fp32 with D > 8: the split-fp16 tensor-core path (every packed-row width, one
# and two value passes, single and several column tiles per warpgroup)
F32_TC_SHAPES = [
    (1, 1, 1, 9, 1), (1, 1, 300, 12, 1), (1, 300, 700, 9, 1), (1, 257, 1000, 16, 3),
    (2, 300, 1100, 32, 32), (1, 129, 513, 33, 17), (1, 200, 333, 64, 64), (1, 130, 260, 65, 70),
    (1, 100, 300, 96, 5), (1, 150, 450, 100, 40), (1, 128, 400, 128, 33), (3, 64, 2000, 24, 1),
]


@pytest.mark.parametrize("shape", F32_SHAPES, ids=[str(s) for s in F32_SHAPES])
def test_f32_odd_shapes(shape):
    B, M, N, D, C = shape
    inp = synth.make_inputs(1, seed=hash(shape) % 1000, B=B, M=M, N=N, D=D, C=C)
    d = dev(inp)
    out = gs().gauss_sum_fwd(d["x"], d["y"], d["w"], inp["tau"]).cpu().numpy()
    ref = oracle.gauss_sum(f64(inp, "x"), f64(inp, "y"), f64(inp, "w"), inp["tau"])
    assert rel_l2(out, ref) <= TOL["f32"], rel_l2(out, ref)


@pytest.mark.parametrize("dtype", ["f16", "bf16"])
@pytest.mark.parametrize("shape", HALF_SHAPES, ids=[str(s) for s in HALF_SHAPES])
def test_half_odd_shapes(shape, dtype):
    B, M, N, D, C = shape
    inp = synth.make_inputs(4, seed=hash(shape) % 1000, B=B, M=M, N=N, D=D, C=C, dtype=dtype)
    d = dev(inp)
    out = gs().gauss_sum_fwd(d["x"], d["y"], d["w"], inp["tau"]).cpu().numpy()
    ref = oracle.gauss_sum(f64(inp, "x"), f64(inp, "y"), f64(inp, "w"), inp["tau"])
    assert rel_l2(out, ref) <= TOL[dtype], rel_l2(out, ref)


@pytest.mark.parametrize("shape", F32_TC_SHAPES, ids=[str(s) for s in F32_TC_SHAPES])
def test_f32_tensor_core_shapes(shape):
    B, M, N, D, C = shape
    inp = synth.make_inputs(4, seed=hash(shape) % 1000, B=B, M=M, N=N, D=D, C=C, dtype="f32")
    d = dev(inp)
    out = gs().gauss_sum_fwd(d["x"], d["y"], d["w"], inp["tau"]).cpu().numpy()
    ref = oracle.gauss_sum(f64(inp, "x"), f64(inp, "y"), f64(inp, "w"), inp["tau"])
    assert rel_l2(out, ref) <= TOL["f32"], rel_l2(out, ref)


@pytest.mark.parametrize("shift,tau", [(0.0, 4.0), (30.0, 1.0), (300.0, 1.0)])
def test_f32_tensor_core_shifted_clouds_and_sharp_kernels(shift, tau):
    """Clouds far from the origin (the operands are centred on a point of the
    cloud, so the norms stay at the cloud's own scale) and a sharper kernel."""
    inp = synth.make_inputs(4, seed=31, B=2, M=300, N=900, D=32, C=3, dtype="f32")
    for k in ("x", "y"):
        inp[k] = (inp[k].double() + shift).float()
    d = dev(inp)
    out = gs().gauss_sum_fwd(d["x"], d["y"], d["w"], tau).cpu().numpy()
    ref = oracle.gauss_sum(f64(inp, "x"), f64(inp, "y"), f64(inp, "w"), tau)
    assert rel_l2(out, ref) <= TOL["f32"], rel_l2(out, ref)


@pytest.mark.parametrize("scale", [1e-5, 1e-2, 1e3, 1e6])
@pytest.mark.parametrize("D,C", [(32, 1), (32, 5), (100, 2)])
def test_f32_tensor_core_coordinate_scales(scale, D, C):
    """Coordinates s times larger with tau / s^2: the same kernel matrix.  The
    similarity tile's fp16 parts are scaled by a power of two per batch, so
    neither tiny nor huge coordinates leave fp16's range.  Batch 1's cloud is
    1000 times smaller than batch 0's (one scale per batch)."""
    inp = synth.make_inputs(4, seed=37, B=2, M=260, N=700, D=D, C=C, dtype="f32")
    for k in ("x", "y"):
        v = inp[k].double() * scale
        v[1] *= 1e-3
        inp[k] = v.float()
    tau = 1.0 / scale ** 2
    d = dev(inp)
    x, y, w = (f64(inp, k) for k in "xyw")
    out = gs().gauss_sum_fwd(d["x"], d["y"], d["w"], tau).cpu().numpy()
    ref = oracle.gauss_sum(x, y, w, tau)
    # batch 1 with its own tau (a 1000 times smaller cloud)
    out1 = gs().gauss_sum_fwd(d["x"][1:], d["y"][1:], d["w"][1:], tau * 1e6).cpu().numpy()
    ref1 = oracle.gauss_sum(x[1:], y[1:], w[1:], tau * 1e6)
    assert rel_l2(out[0], ref[0]) <= TOL["f32"], rel_l2(out[0], ref[0])
    assert rel_l2(out1, ref1) <= TOL["f32"], rel_l2(out1, ref1)
    wpos = inp["w"][:1].abs() + 0.1   # positive weights, float32, for both sides
    lse = gs().gauss_lse_fwd(d["x"][:1], d["y"][:1], wpos.cuda(), tau).cpu().numpy()
    lref = oracle.gauss_lse(x[:1], y[:1], synth.as_f64(wpos), tau)
    assert rel_l2(lse, lref) <= TOL["f32"], rel_l2(lse, lref)


@pytest.mark.parametrize("tau", [1.0, 20.0])
def test_f32_tensor_core_values_channel_scales(tau):
    """Tensor-core values (4+ channels): channel c carries weights 10^(c - 10),
    so one pass holds values from 1e-10 to 1e9; each channel's fp16 parts get
    their own power-of-two scale.  Checked channel by channel; tau = 20 makes
    most kernel values tiny (P 2^14 keeps them in fp16's normal range)."""
    inp = synth.make_inputs(4, seed=41, B=2, M=200, N=900, D=32, C=20, dtype="f32")
    wv = inp["w"].double() * torch.tensor([10.0 ** (c - 10) for c in range(20)], dtype=torch.float64)
    inp["w"] = wv.float()
    if tau > 1:
        for k in ("x", "y"):
            inp[k] = (inp[k].double() * 0.5).float()
    d = dev(inp)
    out = gs().gauss_sum_fwd(d["x"], d["y"], d["w"], tau).cpu().numpy()
    ref = oracle.gauss_sum(f64(inp, "x"), f64(inp, "y"), f64(inp, "w"), tau)
    for c in range(20):
        e = rel_l2(out[..., c], ref[..., c])
        assert e <= TOL["f32"], (c, e)


@pytest.mark.parametrize("shape", [(1, 700, 900, 3, 1), (2, 300, 1100, 2, 3), (1, 64, 5000, 8, 9)])
def test_lse_f32_shapes(shape):
    B, M, N, D, C = shape
    inp = synth.make_inputs(3, seed=5, B=B, M=M, N=N, D=D, C=C)
    d = dev(inp)
    out = gs().gauss_lse_fwd(d["x"], d["y"], d["w"], inp["tau"]).cpu().numpy()
    ref = oracle.gauss_lse(f64(inp, "x"), f64(inp, "y"), f64(inp, "w"), inp["tau"])
    assert rel_l2(out, ref) <= TOL["f32"], rel_l2(out, ref)
    assert rel_l2(np.exp(out), np.exp(ref)) <= TOL["f32"]


@pytest.mark.parametrize("shape,tau", [((1, 300, 700, 16, 1), 1.0), ((2, 200, 500, 32, 2), 1.0),
                                       ((1, 130, 1000, 100, 1), 1.0), ((1, 257, 900, 24, 3), 30.0)])
def test_lse_f32_tensor_core_shapes(shape, tau):
    """fp32 with D > 8: the log-sum-exp on the split-fp16 path (running maximum)."""
    B, M, N, D, C = shape
    inp = synth.make_inputs(3, seed=41, B=B, M=M, N=N, D=D, C=C)
    inp["x"] = (inp["x"].double() / D ** 0.5).float()   # unit-scale clouds in D dimensions
    inp["y"] = (inp["y"].double() / D ** 0.5).float()
    d = dev(inp)
    out = gs().gauss_lse_fwd(d["x"], d["y"], d["w"], tau).cpu().numpy()
    ref = oracle.gauss_lse(f64(inp, "x"), f64(inp, "y"), f64(inp, "w"), tau)
    assert rel_l2(out, ref) <= TOL["f32"], rel_l2(out, ref)
    assert rel_l2(np.exp(out), np.exp(ref)) <= TOL["f32"]


@pytest.mark.parametrize("dtype,shape,tau", [("f16", (1, 300, 700, 3, 1), 30.0),
                                             ("bf16", (2, 200, 500, 32, 2), 1.0),
                                             ("f16", (1, 130, 1000, 100, 1), 1.0),
                                             ("f16", (1, 257, 900, 128, 3), 2.0),
                                             ("bf16", (1, 190, 640, 17, 1), 4.0),
                                             ("f16", (3, 100, 333, 16, 2), 1.0)])
def test_lse_half_precision_shapes(dtype, shape, tau):
    """fp16 / bf16 log-sum-exp: the input values, unsplit, on the tensor-core path."""
    B, M, N, D, C = shape
    inp = synth.make_inputs(3, seed=43, B=B, M=M, N=N, D=D, C=C, dtype=dtype)
    inp["x"] = (inp["x"].double() / D ** 0.5).to(inp["x"].dtype)
    inp["y"] = (inp["y"].double() / D ** 0.5).to(inp["y"].dtype)
    d = dev(inp)
    out = gs().gauss_lse_fwd(d["x"], d["y"], d["w"], tau).cpu().numpy()
    ref = oracle.gauss_lse(f64(inp, "x"), f64(inp, "y"), f64(inp, "w"), tau)
    assert rel_l2(out, ref) <= TOL[dtype], rel_l2(out, ref)
    assert rel_l2(np.exp(out), np.exp(ref)) <= TOL[dtype]


def test_lse_f32_tensor_core_rows_far_from_every_point():
    """Rows whose every kernel value underflows fp32 (exp(-tau/2 d^2) ~ e^-5000):
    the running maximum keeps the log-sum-exp finite and exact."""
    inp = synth.make_inputs(3, seed=42, B=1, M=64, N=600, D=20, C=1)
    x = inp["x"].double()
    x[0, :32] += 100.0
    inp["x"] = x.float()
    d = dev(inp)
    out = gs().gauss_lse_fwd(d["x"], d["y"], d["w"], 1.0).cpu().numpy()
    ref = oracle.gauss_lse(f64(inp, "x"), f64(inp, "y"), f64(inp, "w"), 1.0)
    assert np.isfinite(out).all()
    assert rel_l2(out, ref) <= TOL["f32"], rel_l2(out, ref)
    # the rows near the cloud, on the stricter exp scale
    assert rel_l2(np.exp(out[:, 32:]), np.exp(ref[:, 32:])) <= TOL["f32"]


def test_lse_rows_far_from_every_point():
    """Rows whose every kernel value underflows fp32 take the exact per-row
    recompute; the result must still match the oracle's shifted evaluation."""
    inp = synth.make_inputs(3, seed=6, M=300, N=2000)
    x = inp["x"].clone()
    x[0, :50] += 5.0           # 5 units away from the unit cube, tau = 100: exp(-1250) ~ 0
    inp["x"] = x
    d = dev(inp)
    out = gs().gauss_lse_fwd(d["x"], d["y"], d["w"], inp["tau"]).cpu().numpy()
    ref = oracle.gauss_lse(f64(inp, "x"), f64(inp, "y"), f64(inp, "w"), inp["tau"])
    assert np.isfinite(out).all()
    assert rel_l2(out, ref) <= TOL["f32"], rel_l2(out, ref)


@pytest.mark.parametrize("dtype,shape", [
    ("f32", (1, 500, 700, 3, 1)), ("f32", (2, 300, 400, 2, 3)), ("f32", (1, 200, 300, 8, 2)),
    ("f16", (1, 300, 500, 32, 1)), ("f16", (2, 257, 300, 16, 4)), ("bf16", (1, 200, 333, 32, 1)),
    ("f32", (1, 300, 500, 32, 1)), ("f32", (2, 257, 300, 20, 4)),
])
def test_bwd_shapes(dtype, shape):
    B, M, N, D, C = shape
    wid = 1 if (dtype == "f32" and D <= 8) else 5
    inp = synth.make_inputs(wid, seed=12, B=B, M=M, N=N, D=D, C=C, dtype=dtype, with_g=True)
    d = dev(inp)
    gx, gw = gs().gauss_sum_bwd(d["x"], d["y"], d["w"], d["g"], inp["tau"])
    rgx, rgw = oracle.gauss_sum_bwd(*(f64(inp, k) for k in "xywg"), inp["tau"])
    assert rel_l2(gx.cpu().numpy(), rgx) <= TOL[dtype], rel_l2(gx.cpu().numpy(), rgx)
    assert rel_l2(gw.cpu().numpy(), rgw) <= TOL[dtype], rel_l2(gw.cpu().numpy(), rgw)


# ------------------------------------------------------------------ edge cases
def test_empty_inputs():
    m = gs()
    x = torch.randn(1, 5, 3, device="cuda")
    y = torch.empty(1, 0, 3, device="cuda")
    w = torch.empty(1, 0, 2, device="cuda")
    assert torch.equal(m.gauss_sum_fwd(x, y, w, 1.0), torch.zeros(1, 5, 2, device="cuda"))
    lse = m.gauss_lse_fwd(x, y, w, 1.0)
    assert torch.isneginf(lse).all()
    x0 = torch.empty(1, 0, 3, device="cuda")
    yy, ww = torch.randn(1, 4, 3, device="cuda"), torch.randn(1, 4, 2, device="cuda")
    assert m.gauss_sum_fwd(x0, yy, ww, 1.0).shape == (1, 0, 2)
    xh = torch.randn(2, 5, 32, device="cuda", dtype=torch.float16)
    yh = torch.empty(2, 0, 32, device="cuda", dtype=torch.float16)
    wh = torch.empty(2, 0, 4, device="cuda", dtype=torch.float16)
    assert torch.equal(m.gauss_sum_fwd(xh, yh, wh, 1.0), torch.zeros(2, 5, 4, device="cuda"))
    gx, gw = m.gauss_sum_bwd(xh, yh, wh, torch.randn(2, 5, 4, device="cuda"), 1.0)
    assert torch.equal(gx, torch.zeros_like(gx)) and gw.shape == (2, 0, 4)
    # the forward that keeps the gradient sums, and the backward from them
    out, saved = m.gauss_sum_fwd_saved(xh, yh, wh, 1.0)
    assert torch.equal(out, torch.zeros(2, 5, 4, device="cuda"))
    assert torch.equal(saved, torch.zeros(2, 5, 4 * 33, device="cuda"))
    gx, gw = m.gauss_sum_bwd_saved(xh, yh, wh, torch.randn(2, 5, 4, device="cuda"), saved, 1.0)
    assert torch.equal(gx, torch.zeros_like(gx)) and gw.shape == (2, 0, 4)
    # log-sum-exp on the tensor-core paths (fp16, and fp32 with D > 8)
    assert torch.isneginf(m.gauss_lse_fwd(xh, yh, wh, 1.0)).all()
    xw, yw, ww0 = torch.randn(1, 6, 20, device="cuda"), torch.empty(1, 0, 20, device="cuda"), \
        torch.empty(1, 0, 1, device="cuda")
    assert torch.isneginf(m.gauss_lse_fwd(xw, yw, ww0, 1.0)).all()
    assert torch.equal(m.gauss_sum_fwd(xw, yw, ww0, 1.0), torch.zeros(1, 6, 1, device="cuda"))
    # k-nearest at D > 8 with fewer sources than K: +inf distances and index -1 pad
    od, oi = m.gauss_knn(xw, torch.randn(1, 3, 20, device="cuda"), 5)
    assert torch.isinf(od[..., 3:]).all() and (oi[..., 3:] == -1).all()
    assert (oi[..., :3] >= 0).all()


def test_coincident_points_give_the_weight_sum():
    m = gs()
    x = torch.tensor([[[0.5, -1.0, 2.0]]], device="cuda")
    y = x.repeat(1, 1000, 1)
    w = torch.randn(1, 1000, 1, device="cuda", generator=torch.Generator("cuda").manual_seed(3))
    out = m.gauss_sum_fwd(x, y, w, 2.0)
    assert abs(out.item() - w.double().sum().item()) <= 1e-5 * w.abs().sum().item()


def test_deterministic_and_no_writes_past_the_output():
    m = gs()
    inp = synth.make_inputs(1, seed=21, M=3001, N=5000)
    d = dev(inp)
    guard = 4096
    buf = torch.full((inp["M"] + guard,), 12345.0, device="cuda")
    out = buf[: inp["M"]].view(1, inp["M"], 1)
    m.gauss_sum_fwd(d["x"], d["y"], d["w"], inp["tau"], out=out)
    first = out.clone()
    m.gauss_sum_fwd(d["x"], d["y"], d["w"], inp["tau"], out=out)
    assert torch.equal(first, out), "two identical calls differ"
    assert (buf[inp["M"]:] == 12345.0).all(), "canary after the output was overwritten"
    h = synth.make_inputs(4, seed=22, B=1, M=300, N=2000, C=32)
    dh = dev(h)
    hb = torch.full((300 * 32 + guard,), -7.0, device="cuda")
    ho = hb[: 300 * 32].view(1, 300, 32)
    m.gauss_sum_fwd(dh["x"], dh["y"], dh["w"], 1.0, out=ho)
    r1 = ho.clone()
    m.gauss_sum_fwd(dh["x"], dh["y"], dh["w"], 1.0, out=ho)
    assert torch.equal(r1, ho)
    assert (hb[300 * 32:] == -7.0).all()
    assert m.last_device_error() == 0


def test_abi_rejects_bad_arguments_on_device():
    import ctypes
    m = gs()
    lib = m.library()
    x = torch.randn(1, 10, 3, device="cuda")
    out = torch.empty(1, 10, 1, device="cuda")
    p = lambda t: ctypes.c_void_p(t.data_ptr())
    s = ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    assert lib.gauss_sum_fwd(p(x), p(x), p(out), p(out), 1, 10, 10, 3, 1, -1.0, 0, None, 0, s) == 1
    odd = ctypes.c_void_p(x.data_ptr() + 4)
    assert lib.gauss_sum_fwd(odd, p(x), p(out), p(out), 1, 10, 10, 3, 1, 1.0, 0, None, 0, s) == 3
    h = torch.randn(1, 300, 32, device="cuda", dtype=torch.float16)
    ho = torch.empty(1, 300, 32, device="cuda")
    assert lib.gauss_sum_fwd(p(h), p(h), p(h), p(ho), 1, 300, 300, 32, 32, 1.0, 1, None, 0, s) == 4
    assert m.last_device_error() == 0


@pytest.mark.parametrize("C", [1, 32, 96])
def test_tensor_core_path_is_deterministic_under_repetition(C):
    """Twenty identical calls give bit-identical results: a race between the
    exp warps and the MMAs (a P tile overwritten before it is consumed, an S
    tile before it is read) would show up as run-to-run differences."""
    m = gs()
    h = synth.make_inputs(4, seed=31, B=2, M=1000, N=3000, C=C)
    d = dev(h)
    ref = m.gauss_sum_fwd(d["x"], d["y"], d["w"], 1.0)
    for _ in range(19):
        assert torch.equal(m.gauss_sum_fwd(d["x"], d["y"], d["w"], 1.0), ref)
    ro = oracle.gauss_sum(f64(h, "x"), f64(h, "y"), f64(h, "w"), 1.0, rows=np.arange(0, 1000, 7))
    assert rel_l2(ref.cpu().numpy()[:, ::7], ro) <= TOL["f16"]


# ------------------------------------------------------------------ forward that keeps the x-gradient sums
@pytest.mark.parametrize("dtype,shape", [("f32", (1, 400, 600, 3, 1)), ("f32", (2, 300, 500, 2, 3)),
                                         ("f16", (1, 300, 500, 32, 1)), ("bf16", (2, 257, 300, 16, 2)),
                                         ("f32", (1, 250, 400, 32, 2))])
def test_fwd_saved_then_bwd_saved(dtype, shape):
    """gauss_sum_fwd_saved + gauss_sum_bwd_saved against the oracle (and against
    the separate forward and backward entry points)."""
    B, M, N, D, C = shape
    wid = 1 if (dtype == "f32" and D <= 8) else 5
    inp = synth.make_inputs(wid, seed=21, B=B, M=M, N=N, D=D, C=C, dtype=dtype, with_g=True)
    d = dev(inp)
    m = gs()
    out, saved = m.gauss_sum_fwd_saved(d["x"], d["y"], d["w"], inp["tau"])
    assert saved.shape == (B, M, C * (1 + D))
    gx, gw = m.gauss_sum_bwd_saved(d["x"], d["y"], d["w"], d["g"], saved, inp["tau"])
    x, y, w, g = (f64(inp, k) for k in "xywg")
    ref = oracle.gauss_sum(x, y, w, inp["tau"])
    rgx, rgw = oracle.gauss_sum_bwd(x, y, w, g, inp["tau"])
    tol = TOL[dtype]
    assert rel_l2(out.cpu().numpy(), ref) <= tol, rel_l2(out.cpu().numpy(), ref)
    assert rel_l2(gx.cpu().numpy(), rgx) <= tol, rel_l2(gx.cpu().numpy(), rgx)
    assert rel_l2(gw.cpu().numpy(), rgw) <= tol, rel_l2(gw.cpu().numpy(), rgw)
    # the same grad_w pass as gauss_sum_bwd, bit for bit; grad_x from the same sums
    bx, bw = m.gauss_sum_bwd(d["x"], d["y"], d["w"], d["g"], inp["tau"])
    assert torch.equal(bw, gw)
    assert torch.equal(bx, gx)
    only_w = m.gauss_sum_bwd_saved(d["x"], d["y"], d["w"], d["g"], saved, inp["tau"], want_x=False)
    assert only_w[0] is None and torch.equal(only_w[1], gw)


# ------------------------------------------------------------------ forward + backward in one call
FWD_BWD_FUSED = [  # dtype, (B, M, N, D): fp16 / bf16, C = 1, D <= 47 -> one sweep
    ("f16", (1, 300, 500, 32)), ("bf16", (2, 257, 700, 32)), ("f16", (1, 129, 1000, 1)),
    ("f16", (2, 513, 300, 15)), ("bf16", (1, 1, 900, 16)), ("f16", (1, 700, 1, 31)),
    ("f16", (1, 1000, 2100, 47)), ("bf16", (3, 260, 390, 46)), ("f16", (1, 2049, 1500, 5)),
]
FWD_BWD_OTHER = [  # dtype, (B, M, N, D, C): the two-pass path
    ("f32", (1, 300, 500, 3, 1)), ("f32", (1, 250, 400, 32, 1)), ("f16", (1, 200, 300, 60, 1)),
    ("f16", (2, 150, 250, 32, 2)), ("bf16", (1, 120, 333, 16, 3)),
]


def _fwd_bwd_check(inp, dtype, tol_w=None):
    d = dev(inp)
    m = gs()
    out, gx, gw = m.gauss_sum_fwd_bwd(d["x"], d["y"], d["w"], d["g"], inp["tau"])
    x, y, w, g = (f64(inp, k) for k in "xywg")
    ref = oracle.gauss_sum(x, y, w, inp["tau"])
    rgx, rgw = oracle.gauss_sum_bwd(x, y, w, g, inp["tau"])
    tol = TOL[dtype]
    assert rel_l2(out.cpu().numpy(), ref) <= tol, rel_l2(out.cpu().numpy(), ref)
    assert rel_l2(gx.cpu().numpy(), rgx) <= tol, rel_l2(gx.cpu().numpy(), rgx)
    assert rel_l2(gw.cpu().numpy(), rgw) <= (tol_w or tol), rel_l2(gw.cpu().numpy(), rgw)
    return d, out, gx, gw


@pytest.mark.parametrize("dtype,shape", FWD_BWD_FUSED, ids=[f"{d}-{s}" for d, s in FWD_BWD_FUSED])
def test_fwd_bwd_fused_sweep(dtype, shape):
    """gauss_sum_fwd_bwd on the one-sweep path against the oracle; its forward
    sum and x-gradient are the same arithmetic as gauss_sum_fwd_saved +
    gauss_sum_bwd_saved (bit for bit), its grad_w comes from P^T g in the same
    sweep."""
    B, M, N, D = shape
    inp = synth.make_inputs(5, seed=61, B=B, M=M, N=N, D=D, C=1, dtype=dtype, with_g=True)
    if M == 1:
        # one row: its relative error is that of a single sum, which signed
        # weights can make arbitrarily ill-conditioned; positive weights keep
        # the case a test of the one-row tile rather than of cancellation
        inp["w"] = (inp["w"].double().abs() + 0.25).to(inp["w"].dtype)
    d, out, gx, gw = _fwd_bwd_check(inp, dtype)
    m = gs()
    so, saved = m.gauss_sum_fwd_saved(d["x"], d["y"], d["w"], inp["tau"])
    sx, _ = m.gauss_sum_bwd_saved(d["x"], d["y"], d["w"], d["g"], saved, inp["tau"], want_w=False)
    assert torch.equal(out, so) and torch.equal(gx, sx)
    # deterministic: fixed-order partial sums, no atomics
    o2, x2, w2 = m.gauss_sum_fwd_bwd(d["x"], d["y"], d["w"], d["g"], inp["tau"])
    assert torch.equal(o2, out) and torch.equal(x2, gx) and torch.equal(w2, gw)


@pytest.mark.parametrize("dtype,shape", FWD_BWD_OTHER, ids=[f"{d}-{s}" for d, s in FWD_BWD_OTHER])
def test_fwd_bwd_two_pass_path(dtype, shape):
    B, M, N, D, C = shape
    wid = 1 if (dtype == "f32" and D <= 8) else 5
    inp = synth.make_inputs(wid, seed=62, B=B, M=M, N=N, D=D, C=C, dtype=dtype, with_g=True)
    _fwd_bwd_check(inp, dtype)


@pytest.mark.parametrize("gscale", [1e-30, 1e-6, 1e6, 1e30])
def test_fwd_bwd_upstream_gradient_scales(gscale):
    """g far from unit scale: the per-batch power of two keeps its fp16 parts
    in range (two batches 10^3 apart, one row of zeros)."""
    inp = synth.make_inputs(5, seed=63, B=2, M=300, N=700, D=32, C=1, with_g=True)
    g = inp["g"].double() * gscale
    g[1] *= 1e3
    g[0, 7] = 0.0
    inp["g"] = g.float()
    _fwd_bwd_check(inp, "f16")


def test_fwd_bwd_edge_cases():
    m = gs()
    for (M, N) in ((0, 50), (40, 0), (1, 1)):
        inp = synth.make_inputs(5, seed=64, B=2, M=M, N=N, D=32, C=1, with_g=True)
        d = dev(inp)
        out, gx, gw = m.gauss_sum_fwd_bwd(d["x"], d["y"], d["w"], d["g"], inp["tau"])
        x, y, w, g = (f64(inp, k) for k in "xywg")
        if M and N:
            assert rel_l2(out.cpu().numpy(), oracle.gauss_sum(x, y, w, inp["tau"])) <= TOL["f16"]
            rgx, rgw = oracle.gauss_sum_bwd(x, y, w, g, inp["tau"])
            assert rel_l2(gx.cpu().numpy(), rgx) <= TOL["f16"]
            assert rel_l2(gw.cpu().numpy(), rgw) <= TOL["f16"]
        else:
            assert not out.abs().sum() and not gx.abs().sum() and not gw.abs().sum()
    # outputs left out
    inp = synth.make_inputs(5, seed=65, B=1, M=300, N=400, D=32, C=1, with_g=True)
    d = dev(inp)
    ref_o, ref_x, ref_w = m.gauss_sum_fwd_bwd(d["x"], d["y"], d["w"], d["g"], inp["tau"])
    o, gx, gw = m.gauss_sum_fwd_bwd(d["x"], d["y"], d["w"], d["g"], inp["tau"], want_w=False)
    assert gw is None and torch.equal(o, ref_o) and torch.equal(gx, ref_x)
    o, gx, gw = m.gauss_sum_fwd_bwd(d["x"], d["y"], d["w"], d["g"], inp["tau"], want_x=False)
    assert gx is None and torch.equal(o, ref_o) and torch.equal(gw, ref_w)


def test_d32_c1_f16_fwd_bwd_one_call_full_size():
    """The forward + backward workload (B=4, M=N=16384, D=32, C=1, fp16) through
    gauss_sum_fwd_bwd, the call the benchmark times for it, against the oracle
    on sampled rows and sources, and against the two-call path."""
    inp = synth.make_inputs(5)
    d = dev(inp)
    m = gs()
    out, gx, gw = m.gauss_sum_fwd_bwd(d["x"], d["y"], d["w"], d["g"], inp["tau"])
    x, y, w, g = (f64(inp, k) for k in "xywg")
    rows = synth.sample_rows(inp["M"], 512, seed=66).numpy()
    wrows = synth.sample_rows(inp["N"], 512, seed=67).numpy()
    ref = oracle.gauss_sum(x, y, w, inp["tau"], rows=rows)
    rgx, rgw = oracle.gauss_sum_bwd(x, y, w, g, inp["tau"], rows=rows, wrows=wrows)
    o, gxn, gwn = out.cpu().numpy(), gx.cpu().numpy(), gw.cpu().numpy()
    assert rel_l2(o[:, rows], ref) <= TOL["f16"], rel_l2(o[:, rows], ref)
    assert rel_l2(gxn[:, rows], rgx) <= TOL["f16"], rel_l2(gxn[:, rows], rgx)
    assert rel_l2(gwn[:, wrows], rgw) <= TOL["f16"], rel_l2(gwn[:, wrows], rgw)
    so, saved = m.gauss_sum_fwd_saved(d["x"], d["y"], d["w"], inp["tau"])
    sx, sw = m.gauss_sum_bwd_saved(d["x"], d["y"], d["w"], d["g"], saved, inp["tau"])
    assert torch.equal(out, so) and torch.equal(gx, sx)
    # grad_w: fp16 P (this sweep) against fp32 P (the separate pass), whole arrays
    assert rel_l2(gwn, sw.cpu().numpy()) <= TOL["f16"]


# ------------------------------------------------------------------ full gradient
@pytest.mark.parametrize("dtype,shape,shift", [
    ("f32", (1, 400, 600, 3, 1), 0.0), ("f32", (2, 300, 500, 2, 3), 0.0), ("f32", (1, 250, 350, 8, 2), 0.0),
    ("f32", (1, 300, 400, 3, 1), 40.0),
    ("f16", (1, 300, 500, 32, 1), 0.0), ("f16", (2, 257, 300, 16, 4), 0.0), ("bf16", (1, 200, 333, 32, 1), 0.0),
    ("f16", (1, 300, 500, 16, 2), 20.0),
    ("f32", (1, 300, 500, 32, 1), 0.0), ("f32", (2, 200, 300, 12, 3), 0.0), ("f32", (1, 250, 400, 32, 2), 25.0),
])
def test_vjp_every_gradient(dtype, shape, shift):
    """dL/dx, dL/dy, dL/dw and dL/dtau against the oracle; `shift` moves the
    whole point cloud away from the origin (the gradients do not change, the
    centred values keep the cancellation at the cloud's own scale)."""
    B, M, N, D, C = shape
    wid = 1 if (dtype == "f32" and D <= 8) else 5
    inp = synth.make_inputs(wid, seed=13, B=B, M=M, N=N, D=D, C=C, dtype=dtype, with_g=True)
    if shift:
        for k in ("x", "y"):
            inp[k] = (inp[k].double() + shift).to(inp[k].dtype)
    d = dev(inp)
    got = gs().gauss_sum_vjp(d["x"], d["y"], d["w"], d["g"], inp["tau"])
    x, y, w, g = (f64(inp, k) for k in "xywg")
    rgx, rgw = oracle.gauss_sum_bwd(x, y, w, g, inp["tau"])
    rgy, rgt = oracle.gauss_sum_vjp_y_tau(x, y, w, g, inp["tau"])
    tol = TOL[dtype]
    for name, ref in (("x", rgx), ("y", rgy), ("w", rgw)):
        e = rel_l2(got[name].cpu().numpy(), ref)
        assert e <= tol, (name, e)
    et = abs(float(got["tau"].item()) - rgt) / max(abs(rgt), 1e-30)
    assert et <= tol, ("tau", et, float(got["tau"].item()), rgt)
    # subsets of outputs give the same values
    only = gs().gauss_sum_vjp(d["x"], d["y"], d["w"], d["g"], inp["tau"], want=("y", "tau"))
    assert torch.equal(only["y"], got["y"]) and torch.equal(only["tau"], got["tau"])


def test_vjp_d32_c1_full_size_sampled():
    inp = synth.make_inputs(5)
    d = dev(inp)
    got = gs().gauss_sum_vjp(d["x"], d["y"], d["w"], d["g"], inp["tau"], want=("x", "y", "w"))
    x, y, w, g = (f64(inp, k) for k in "xywg")
    rows = synth.sample_rows(inp["M"], 256, seed=14).numpy()
    yrows = synth.sample_rows(inp["N"], 256, seed=15).numpy()
    rgx, rgw = oracle.gauss_sum_bwd(x, y, w, g, inp["tau"], rows=rows, wrows=yrows)
    rgy, _ = oracle.gauss_sum_vjp_y_tau(x, y, w, g, inp["tau"], yrows=yrows, want_tau=False)
    assert rel_l2(got["x"].cpu().numpy()[:, rows], rgx) <= TOL["f16"]
    assert rel_l2(got["w"].cpu().numpy()[:, yrows], rgw) <= TOL["f16"]
    assert rel_l2(got["y"].cpu().numpy()[:, yrows], rgy) <= TOL["f16"]


# ------------------------------------------------------------------ log-sum-exp backward
@pytest.mark.parametrize("shape,shift", [((1, 300, 500, 3, 1), 0.0), ((2, 200, 300, 2, 3), 0.0),
                                         ((1, 150, 400, 8, 2), 0.0), ((1, 256, 700, 3, 1), 30.0),
                                         ((1, 200, 500, 16, 1), 0.0), ((2, 150, 300, 32, 2), 0.0),
                                         ((1, 180, 400, 24, 1), 30.0)])
def test_lse_bwd_every_gradient(shape, shift):
    """D > 8 runs the tensor-core passes (coordinates scaled by sqrt(3/D) so that
    the clouds have the spread of the D = 3 ones)."""
    B, M, N, D, C = shape
    inp = synth.make_inputs(3, seed=17, B=B, M=M, N=N, D=D, C=C, with_g=True, tau=20.0)
    if D > 8:
        for k in ("x", "y"):
            inp[k] = (inp[k].double() * (3.0 / D) ** 0.5).float()
    if shift:
        for k in ("x", "y"):
            inp[k] = inp[k] + shift
    d = dev(inp)
    lse = gs().gauss_lse_fwd(d["x"], d["y"], d["w"], inp["tau"])
    got = gs().gauss_lse_bwd(d["x"], d["y"], d["w"], lse, d["g"], inp["tau"])
    rgx, rgy, rgw, rgt = oracle.gauss_lse_bwd(*(f64(inp, k) for k in "xywg"), inp["tau"])
    for name, ref in (("x", rgx), ("y", rgy), ("w", rgw)):
        e = rel_l2(got[name].cpu().numpy(), ref)
        assert e <= TOL["f32"], (name, e)
    et = abs(float(got["tau"].item()) - rgt) / max(abs(rgt), 1e-30)
    assert et <= TOL["f32"], ("tau", et, float(got["tau"].item()), rgt)


@pytest.mark.parametrize("dtype,shape", [("f16", (1, 300, 500, 3, 1)), ("bf16", (2, 150, 300, 32, 2))])
def test_lse_bwd_half_precision(dtype, shape):
    """fp16 / bf16: the backward runs on exact fp32 copies of the inputs."""
    B, M, N, D, C = shape
    inp = synth.make_inputs(3, seed=27, B=B, M=M, N=N, D=D, C=C, with_g=True, tau=20.0, dtype=dtype)
    if D > 8:
        for k in ("x", "y"):
            inp[k] = (inp[k].double() * (3.0 / D) ** 0.5).to(inp[k].dtype)
    d = dev(inp)
    lse = gs().gauss_lse_fwd(d["x"], d["y"], d["w"], inp["tau"])
    got = gs().gauss_lse_bwd(d["x"], d["y"], d["w"], lse, d["g"], inp["tau"])
    rgx, rgy, rgw, rgt = oracle.gauss_lse_bwd(*(f64(inp, k) for k in "xywg"), inp["tau"])
    for name, ref in (("x", rgx), ("y", rgy), ("w", rgw)):
        e = rel_l2(got[name].cpu().numpy(), ref)
        assert e <= TOL[dtype], (name, e)
    et = abs(float(got["tau"].item()) - rgt) / max(abs(rgt), 1e-30)
    assert et <= TOL[dtype], ("tau", et)


def test_lse_bwd_rows_far_from_every_point():
    """Rows whose kernel values all underflow fp32: the -lse shift in the
    exponent keeps the normalised weights exact."""
    inp = synth.make_inputs(3, seed=18, M=120, N=400, with_g=True)
    x = inp["x"].clone()
    x[0, :20] += 3.0
    inp["x"] = x
    d = dev(inp)
    lse = gs().gauss_lse_fwd(d["x"], d["y"], d["w"], inp["tau"])
    got = gs().gauss_lse_bwd(d["x"], d["y"], d["w"], lse, d["g"], inp["tau"], want=("x", "w"))
    rgx, _, rgw, _ = oracle.gauss_lse_bwd(*(f64(inp, k) for k in "xywg"), inp["tau"])
    assert np.isfinite(got["x"].cpu().numpy()).all()
    assert rel_l2(got["x"].cpu().numpy(), rgx) <= TOL["f32"]
    assert rel_l2(got["w"].cpu().numpy(), rgw) <= TOL["f32"]


# ------------------------------------------------------------------ k-nearest reduction
@pytest.mark.parametrize("shape", [(1, 1000, 3000, 3, 1), (2, 777, 1301, 3, 5), (1, 300, 5000, 8, 32),
                                   (1, 513, 257, 2, 16), (1, 50, 10, 3, 16), (3, 129, 4097, 1, 8),
                                   (1, 2049, 20000, 3, 4), (1, 300, 1000, 9, 5), (2, 257, 700, 16, 32),
                                   (1, 400, 1500, 33, 1), (1, 129, 300, 100, 16), (1, 200, 999, 128, 8)])
def test_knn_bit_exact(shape):
    """Indices bit-exact, distances bit-exact: both sides decide in fp32 with the
    same order of operations, ties by the lower index."""
    B, M, N, D, K = shape
    inp = synth.make_inputs(1, seed=19, B=B, M=M, N=N, D=D, C=1)
    d = dev(inp)
    od, oi = gs().gauss_knn(d["x"], d["y"], K)
    rd, ri = oracle.knn(inp["x"].numpy(), inp["y"].numpy(), K, f32=True)
    assert np.array_equal(oi.cpu().numpy(), ri), "indices differ"
    assert np.array_equal(od.cpu().numpy(), rd), "distances differ"
    knn_valid_under_exact_distances(inp["x"].numpy(), inp["y"].numpy(), od.cpu(), oi.cpu(), K)


@pytest.mark.parametrize("dtype,shape", [("f16", (1, 700, 2000, 3, 8)), ("bf16", (2, 300, 900, 16, 5)),
                                         ("f16", (1, 257, 600, 64, 32))])
def test_knn_half_precision_bit_exact(dtype, shape):
    """fp16 / bf16 inputs: decided in fp32 on their exact fp32 values."""
    B, M, N, D, K = shape
    inp = synth.make_inputs(1, seed=25, B=B, M=M, N=N, D=D, C=1, dtype=dtype)
    d = dev(inp)
    od, oi = gs().gauss_knn(d["x"], d["y"], K)
    rd, ri = oracle.knn(inp["x"].float().numpy(), inp["y"].float().numpy(), K, f32=True)
    assert np.array_equal(oi.cpu().numpy(), ri), "indices differ"
    assert np.array_equal(od.cpu().numpy(), rd), "distances differ"
    knn_valid_under_exact_distances(inp["x"].float().numpy(), inp["y"].float().numpy(), od.cpu(),
                                    oi.cpu(), K)


@pytest.mark.parametrize("D", [3, 12, 40])
def test_knn_duplicates_and_quantised_grid(D):
    """Many exact ties: duplicated sources and points on a coarse grid (D > 8:
    the chunked kernel)."""
    g = torch.Generator().manual_seed(20)
    y = torch.randint(0, 4, (1, 3000, D), generator=g).float() * 0.5
    y = torch.cat([y, y[:, :500]], dim=1)                 # exact duplicates at higher indices
    x = torch.randint(0, 4, (1, 700, D), generator=g).float() * 0.5 + 0.25
    od, oi = gs().gauss_knn(x.cuda(), y.cuda(), 12)
    rd, ri = oracle.knn(x.numpy(), y.numpy(), 12, f32=True)
    assert np.array_equal(oi.cpu().numpy(), ri)
    assert np.array_equal(od.cpu().numpy(), rd)
    knn_valid_under_exact_distances(x.numpy(), y.numpy(), od.cpu(), oi.cpu(), 12)


# ------------------------------------------------------------------ diffusion operator
@pytest.mark.parametrize("dtype,shape,alpha", [("f32", (1, 3000, 3, 4), 0.5), ("f32", (2, 1500, 6, 1), 1.0),
                                               ("f32", (1, 2000, 2, 3), 0.0), ("f16", (1, 2500, 32, 8), 0.5),
                                               ("bf16", (2, 1000, 16, 2), 0.5), ("f32", (1, 2000, 80, 4), 0.5)])
def test_diffusion_scales_and_apply(dtype, shape, alpha):
    B, N, D, C = shape
    small = dtype == "f32" and D <= 8
    inp = synth.make_inputs(1 if small else 4, seed=23, B=B, M=N, N=N, D=D, C=C, dtype=dtype)
    tau = 2.0 if small else 8.0
    x = inp["x"].cuda()
    q, dd, s = gs().gauss_diffusion_scales(x, tau, alpha)
    rq, rd, rs = oracle.diffusion_scales(f64(inp, "x"), tau, alpha)
    for name, got, ref in (("q", q, rq), ("d", dd, rd), ("s", s, rs)):
        assert rel_l2(got.cpu().numpy(), ref) <= TOL[dtype], (name, rel_l2(got.cpu().numpy(), ref))
    v = torch.randn(B, N, C, generator=torch.Generator().manual_seed(24))
    out = gs().gauss_diffusion_apply(x, s, v.cuda(), tau)
    ref = oracle.diffusion_apply(f64(inp, "x"), s.cpu().double().numpy(), v.double().numpy(), tau)
    assert rel_l2(out.cpu().numpy(), ref) <= TOL[dtype], rel_l2(out.cpu().numpy(), ref)
    # sqrt(d) is the operator's fixed point
    fp = gs().gauss_diffusion_apply(x, s, dd.sqrt()[..., None].contiguous(), tau)
    assert rel_l2(fp.cpu().numpy(), dd.sqrt()[..., None].cpu().numpy()) <= TOL[dtype]


@pytest.mark.parametrize("dtype,shape", [("f32", (1, 700, 2000, 3, 2)), ("f32", (2, 300, 900, 40, 3)),
                                         ("f16", (1, 500, 1300, 32, 1)), ("bf16", (2, 257, 640, 16, 4))])
def test_diffusion_block_rows_against_other_columns(dtype, shape):
    """K(x_rows, x_cols) v with float32 values: a rank's rows against every
    rank's points, the pair work of the row-sharded diffusion operator."""
    B, M, N, D, C = shape
    small = dtype == "f32" and D <= 8
    inp = synth.make_inputs(1 if small else 4, seed=71, B=B, M=M, N=N, D=D, C=C, dtype=dtype)
    v = torch.rand(B, N, C, generator=torch.Generator().manual_seed(72)) + 0.5
    out = gs().gauss_diffusion_block(inp["x"].cuda(), inp["y"].cuda(), v.cuda(), 2.0)
    ref = oracle.gauss_sum(f64(inp, "x"), f64(inp, "y"), v.double().numpy(), 2.0)
    assert rel_l2(out.cpu().numpy(), ref) <= TOL[dtype], rel_l2(out.cpu().numpy(), ref)

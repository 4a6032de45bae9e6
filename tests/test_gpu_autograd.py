"""torch.autograd.grad through the fused reductions against the oracle's gradients.

The wrappers only marshal (their forward and backward are the library's entry
points), so these tests check the plumbing: which entry point serves which set
of requested gradients, 2-D inputs, tensor tau, and gradient dtypes.
"""
import numpy as np
import pytest
import torch

import oracle
import synth

pytestmark = pytest.mark.gpu

TOL = {"f32": 1e-5, "f16": 3e-3, "bf16": 3e-3}


def rel_l2(a, b):
    a = np.asarray(a, dtype=np.float64).ravel()
    b = np.asarray(b, dtype=np.float64).ravel()
    return float(np.linalg.norm(a - b) / max(np.linalg.norm(b), 1e-300))


def ag():
    from pairwise_reductions_b200 import autograd
    return autograd


def _inputs(dtype, shape, seed, tau=None):
    B, M, N, D, C = shape
    wid = 1 if (dtype == "f32" and D <= 8) else 5
    kw = {} if tau is None else {"tau": tau}
    return synth.make_inputs(wid, seed=seed, B=B, M=M, N=N, D=D, C=C, dtype=dtype, with_g=True, **kw)


@pytest.mark.parametrize("dtype,shape", [("f32", (1, 300, 500, 3, 2)), ("f32", (2, 200, 300, 32, 1)),
                                         ("f16", (1, 257, 300, 16, 4))])
def test_sum_grad_x_w_uses_the_saved_sums(dtype, shape):
    inp = _inputs(dtype, shape, seed=41)
    x, y, w, g = (inp[k].cuda() for k in "xywg")
    x.requires_grad_(True)
    w.requires_grad_(True)
    a = ag().gauss_sum(x, y, w, inp["tau"])
    gx, gw = torch.autograd.grad(a, (x, w), g)
    assert gx.dtype == x.dtype and gw.dtype == w.dtype
    rgx, rgw = oracle.gauss_sum_bwd(*(synth.as_f64(inp[k]) for k in "xywg"), inp["tau"])
    ref_a = oracle.gauss_sum(*(synth.as_f64(inp[k]) for k in "xyw"), inp["tau"])
    tol = TOL[dtype]
    assert rel_l2(a.detach().cpu().numpy(), ref_a) <= tol
    # float16 gradients carry their own rounding (about 5e-4 relative)
    gtol = tol if dtype == "f32" else 2e-3 + tol
    assert rel_l2(gx.float().cpu().numpy(), rgx) <= gtol
    assert rel_l2(gw.float().cpu().numpy(), rgw) <= gtol


@pytest.mark.parametrize("shape", [(1, 300, 500, 3, 1), (1, 250, 400, 32, 2)])
def test_sum_every_gradient_with_tensor_tau(shape):
    inp = _inputs("f32", shape, seed=43)
    x, y, w, g = (inp[k].cuda().requires_grad_(True) for k in "xywg")
    tau = torch.tensor(inp["tau"], dtype=torch.float32, device="cuda", requires_grad=True)
    a = ag().gauss_sum(x, y, w, tau)
    gx, gy, gw, gt = torch.autograd.grad(a, (x, y, w, tau), g.detach())
    assert gt.shape == tau.shape
    f = [synth.as_f64(inp[k]) for k in "xywg"]
    rgx, rgw = oracle.gauss_sum_bwd(*f, inp["tau"])
    rgy, rgt = oracle.gauss_sum_vjp_y_tau(*f, inp["tau"])
    for got, ref in ((gx, rgx), (gy, rgy), (gw, rgw)):
        assert rel_l2(got.cpu().numpy(), ref) <= TOL["f32"]
    assert abs(float(gt) - rgt) <= TOL["f32"] * abs(rgt)


def test_sum_two_dimensional_inputs():
    inp = _inputs("f32", (1, 200, 300, 3, 2), seed=45)
    x, y, w, g = (inp[k][0].cuda() for k in "xywg")
    x.requires_grad_(True)
    a = ag().gauss_sum(x, y, w, inp["tau"])
    assert a.shape == (200, 2)
    (gx,) = torch.autograd.grad(a, (x,), g)
    assert gx.shape == x.shape
    rgx, _ = oracle.gauss_sum_bwd(*(synth.as_f64(inp[k]) for k in "xywg"), inp["tau"], want_w=False)
    assert rel_l2(gx.cpu().numpy(), rgx[0]) <= TOL["f32"]


@pytest.mark.parametrize("shape", [(1, 300, 500, 3, 1), (2, 150, 300, 32, 2)])
def test_lse_every_gradient(shape):
    B, M, N, D, C = shape
    inp = synth.make_inputs(3, seed=47, B=B, M=M, N=N, D=D, C=C, with_g=True, tau=20.0)
    if D > 8:
        for k in ("x", "y"):
            inp[k] = (inp[k].double() * (3.0 / D) ** 0.5).float()
    x, y, w = (inp[k].cuda().requires_grad_(True) for k in "xyw")
    g = inp["g"].cuda()
    tau = torch.tensor([inp["tau"]], device="cuda", requires_grad=True)
    lse = ag().gauss_lse(x, y, w, tau)
    gx, gy, gw, gt = torch.autograd.grad(lse, (x, y, w, tau), g)
    assert gt.shape == (1,)
    rgx, rgy, rgw, rgt = oracle.gauss_lse_bwd(*(synth.as_f64(inp[k]) for k in "xywg"), inp["tau"])
    for got, ref in ((gx, rgx), (gy, rgy), (gw, rgw)):
        assert rel_l2(got.cpu().numpy(), ref) <= TOL["f32"]
    assert abs(float(gt[0]) - rgt) <= TOL["f32"] * abs(rgt)


def test_no_gradient_requested_runs_the_plain_forward():
    inp = _inputs("f32", (1, 100, 200, 3, 1), seed=49)
    x, y, w = (inp[k].cuda() for k in "xyw")
    from pairwise_reductions_b200 import gauss_sum_fwd
    assert torch.equal(ag().gauss_sum(x, y, w, inp["tau"]), gauss_sum_fwd(x, y, w, inp["tau"]))

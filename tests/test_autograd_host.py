"""Host logic of the torch.autograd wrappers, on the CPU: which library call
serves which set of requested gradients, 2-D inputs, tau as a float or a tensor,
and gradient dtypes.  The six library calls are replaced by float64 stand-ins
built on the oracle (the wrappers' `kernels` argument), so the gradients are
checked against the oracle's own."""
import numpy as np
import pytest
import torch

import oracle
from pairwise_reductions_b200 import autograd

TAU = 0.8


def _fakes(calls):
    t = lambda a: torch.from_numpy(np.ascontiguousarray(a))
    n = lambda a: a.detach().double().numpy()

    def sum_fwd(x, y, w, tau):
        calls.append("sum_fwd")
        return t(oracle.gauss_sum(n(x), n(y), n(w), tau))

    def sum_fwd_saved(x, y, w, tau):
        calls.append("sum_fwd_saved")
        return t(oracle.gauss_sum(n(x), n(y), n(w), tau)), torch.zeros(1)

    def sum_bwd_saved(x, y, w, g, saved, tau, want_x=True, want_w=True):
        calls.append(("sum_bwd_saved", want_x, want_w))
        gx, gw = oracle.gauss_sum_bwd(n(x), n(y), n(w), n(g), tau)
        return (t(gx) if want_x else None), (t(gw) if want_w else None)

    def sum_vjp(x, y, w, g, tau, want=("x", "y", "w", "tau")):
        calls.append(("sum_vjp", tuple(want)))
        gx, gw = oracle.gauss_sum_bwd(n(x), n(y), n(w), n(g), tau)
        gy, gt = oracle.gauss_sum_vjp_y_tau(n(x), n(y), n(w), n(g), tau)
        full = {"x": t(gx), "y": t(gy), "w": t(gw), "tau": torch.tensor([gt], dtype=torch.float64)}
        return {k: full[k] for k in want}

    def lse_fwd(x, y, w, tau):
        calls.append("lse_fwd")
        return t(oracle.gauss_lse(n(x), n(y), n(w), tau))

    def lse_bwd(x, y, w, lse, g, tau, want=("x", "y", "w", "tau")):
        calls.append(("lse_bwd", tuple(want)))
        gx, gy, gw, gt = oracle.gauss_lse_bwd(n(x), n(y), n(w), n(g), tau)
        full = {"x": t(gx), "y": t(gy), "w": t(gw), "tau": torch.tensor([gt], dtype=torch.float64)}
        return {k: full[k] for k in want}

    return {"sum_fwd": sum_fwd, "sum_fwd_saved": sum_fwd_saved, "sum_bwd_saved": sum_bwd_saved,
            "sum_vjp": sum_vjp, "lse_fwd": lse_fwd, "lse_bwd": lse_bwd}


def _problem(B=2, M=7, N=9, D=3, C=2, seed=5):
    g = torch.Generator().manual_seed(seed)
    x = torch.randn(B, M, D, generator=g, dtype=torch.float64)
    y = torch.randn(B, N, D, generator=g, dtype=torch.float64)
    w = torch.rand(B, N, C, generator=g, dtype=torch.float64) + 0.5
    up = torch.randn(B, M, C, generator=g, dtype=torch.float64)
    return x, y, w, up


def test_x_and_w_gradients_take_the_saved_sums():
    calls = []
    x, y, w, up = _problem()
    x.requires_grad_(True)
    w.requires_grad_(True)
    a = autograd.gauss_sum(x, y, w, TAU, kernels=_fakes(calls))
    gx, gw = torch.autograd.grad(a, (x, w), up)
    assert calls == ["sum_fwd_saved", ("sum_bwd_saved", True, True)]
    rgx, rgw = oracle.gauss_sum_bwd(*(v.detach().numpy() for v in (x, y, w, up)), TAU)
    np.testing.assert_allclose(gx.numpy(), rgx, rtol=1e-12)
    np.testing.assert_allclose(gw.numpy(), rgw, rtol=1e-12)


def test_only_w_gradient_asks_for_w_alone():
    calls = []
    x, y, w, up = _problem()
    w.requires_grad_(True)
    a = autograd.gauss_sum(x, y, w, TAU, kernels=_fakes(calls))
    torch.autograd.grad(a, (w,), up)
    assert calls == ["sum_fwd_saved", ("sum_bwd_saved", False, True)]


def test_y_or_tau_gradients_take_the_vjp_with_a_tensor_tau():
    calls = []
    x, y, w, up = _problem()
    y.requires_grad_(True)
    tau = torch.tensor(TAU, dtype=torch.float64, requires_grad=True)
    a = autograd.gauss_sum(x, y, w, tau, kernels=_fakes(calls))
    gy, gt = torch.autograd.grad(a, (y, tau), up)
    assert calls == ["sum_fwd", ("sum_vjp", ("y", "tau"))]
    assert gt.shape == tau.shape
    rgy, rgt = oracle.gauss_sum_vjp_y_tau(*(v.detach().numpy() for v in (x, y, w, up)), TAU)
    np.testing.assert_allclose(gy.numpy(), rgy, rtol=1e-12)
    np.testing.assert_allclose(float(gt), rgt, rtol=1e-12)


def test_two_dimensional_inputs_keep_their_shapes():
    calls = []
    x, y, w, up = (t[0] for t in _problem(B=1))
    x.requires_grad_(True)
    a = autograd.gauss_sum(x, y, w, TAU, kernels=_fakes(calls))
    assert a.shape == (7, 2)
    (gx,) = torch.autograd.grad(a, (x,), up)
    assert gx.shape == x.shape


def test_lse_every_gradient_and_one_element_tau():
    calls = []
    x, y, w, up = _problem()
    for v in (x, y, w):
        v.requires_grad_(True)
    tau = torch.tensor([TAU], dtype=torch.float64, requires_grad=True)
    lse = autograd.gauss_lse(x, y, w, tau, kernels=_fakes(calls))
    gx, gy, gw, gt = torch.autograd.grad(lse, (x, y, w, tau), up)
    assert calls == ["lse_fwd", ("lse_bwd", ("x", "y", "w", "tau"))]
    assert gt.shape == (1,)
    rgx, rgy, rgw, rgt = oracle.gauss_lse_bwd(*(v.detach().numpy() for v in (x, y, w, up)), TAU)
    for got, ref in ((gx, rgx), (gy, rgy), (gw, rgw)):
        np.testing.assert_allclose(got.numpy(), ref, rtol=1e-12)
    np.testing.assert_allclose(float(gt[0]), rgt, rtol=1e-12)


def test_no_gradient_requested_runs_the_plain_forward():
    calls = []
    x, y, w, _ = _problem()
    autograd.gauss_sum(x, y, w, TAU, kernels=_fakes(calls))
    assert calls == ["sum_fwd"]


def test_float32_inputs_get_float32_gradients():
    calls = []
    x, y, w, up = (t.float() for t in _problem())
    x.requires_grad_(True)
    a = autograd.gauss_sum(x, y, w, TAU, kernels=_fakes(calls))
    (gx,) = torch.autograd.grad(a, (x,), up.double())
    assert gx.dtype == torch.float32

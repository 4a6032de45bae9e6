"""Pins that tie the CPU oracle to facts fixed outside itself.

Each pin takes an oracle handle ``O`` (an object with ``gauss_sum``,
``gauss_lse`` and ``gauss_sum_bwd``) and raises ``AssertionError`` when the
oracle disagrees with the fact.  The same pins run against the real oracle
(``test_oracle_pins.py``) and against deliberately broken copies of it
(``test_oracle_mutants.py``), which shows that a plausible slip in the oracle
(a dropped term, a wrong sign, factor or index, a transposed operand) fails at
least one of them.

Sources of truth, none of which is the oracle's own code:

* closed forms derived by hand (``golden/closed_forms.json``);
* a dense library evaluation (``torch.cdist`` then ``exp`` then a matmul);
* the two flash-attention identities of "Fast Gauss Sums via Flash Attention"
  (Algorithm 1 "prescale", Algorithm 2 "reweight"), run through
  ``torch.nn.functional.scaled_dot_product_attention`` in float64;
* special cases: coincident points, a single point, a tensor-product grid whose
  sum factors into one-dimensional sums;
* invariants: common translation, tau -> 0, symmetry for x = y, linearity in the
  weights, LSE = log(sum) for positive weights;
* central finite differences for the gradient.
"""
import json
import math
import os

import numpy as np
import torch
import torch.nn.functional as F

GOLDEN = os.path.join(os.path.dirname(os.path.abspath(__file__)), "golden", "closed_forms.json")
_SAFE = {"exp": math.exp, "log": math.log, "sqrt": math.sqrt, "__builtins__": {}}


def _eval_tree(e):
    if isinstance(e, list):
        return [_eval_tree(v) for v in e]
    return float(eval(e, _SAFE))  # closed-form expression typed in the fixture


def golden():
    with open(GOLDEN) as f:
        return json.load(f)


def _rng(seed):
    return np.random.default_rng(seed)


def _close(a, b, rtol, atol=0.0, what=""):
    a = np.asarray(a, dtype=np.float64)
    b = np.asarray(b, dtype=np.float64)
    assert a.shape == b.shape, f"{what}: shape {a.shape} vs {b.shape}"
    err = np.abs(a - b)
    ok = err <= atol + rtol * np.abs(b)
    assert ok.all(), f"{what}: max abs err {err.max():.3e} (rtol {rtol}, atol {atol})"


def _rel_l2(a, b):
    a = np.asarray(a, dtype=np.float64).ravel()
    b = np.asarray(b, dtype=np.float64).ravel()
    return float(np.linalg.norm(a - b) / max(np.linalg.norm(b), 1e-300))


# --------------------------------------------------------------------------- closed forms
def pin_golden_sum(O):
    for case in golden()["sum"]:
        out = O.gauss_sum(case["x"], case["y"], case["w"], case["tau"])
        _close(out, _eval_tree(case["expected"]), 1e-14, 1e-15, case["name"])


def pin_golden_lse(O):
    for case in golden()["lse"]:
        out = O.gauss_lse(case["x"], case["y"], case["w"], case["tau"])
        _close(out, _eval_tree(case["expected"]), 1e-14, 1e-14, case["name"])


def pin_golden_bwd(O):
    for case in golden()["bwd"]:
        gx, gw = O.gauss_sum_bwd(case["x"], case["y"], case["w"], case["g"], case["tau"])
        _close(gx, _eval_tree(case["expected_grad_x"]), 1e-14, 1e-15, case["name"] + " grad_x")
        _close(gw, _eval_tree(case["expected_grad_w"]), 1e-14, 1e-15, case["name"] + " grad_w")


# --------------------------------------------------------------------------- library routines
def pin_dense_library(O):
    """Dense double evaluation with torch.cdist (a library routine), tiny sizes."""
    r = _rng(1)
    for (B, M, N, D, C, tau) in [(1, 7, 11, 3, 1, 1.0), (2, 13, 5, 4, 3, 0.3), (1, 17, 19, 1, 2, 2.5)]:
        x, y = r.normal(size=(B, M, D)), r.normal(size=(B, N, D))
        w = r.normal(size=(B, N, C))
        xt, yt, wt = (torch.from_numpy(a) for a in (x, y, w))
        K = torch.exp(-0.5 * tau * torch.cdist(xt, yt, compute_mode="donot_use_mm_for_euclid_dist") ** 2)
        ref = (K @ wt).numpy()
        _close(O.gauss_sum(x, y, w, tau), ref, 1e-12, 1e-14, f"dense B{B}M{M}N{N}D{D}C{C}")


def _sdpa(q, k, v, scale):
    return F.scaled_dot_product_attention(q, k, v, scale=scale)


def pin_flash_prescale(O):
    """Algorithm 1 ("prescale") of "Fast Gauss Sums via Flash Attention": with
    v~_n = v_n exp(-tau/2 |k_n|^2), s_m = att_tau(q,k,v~)_m exp(lse_tau(q,k)_m)
    exp(-tau/2 |q_m|^2), where att_tau is softmax attention with logits
    tau q.k_n and lse_tau the log-sum-exp of those logits."""
    r = _rng(2)
    for (M, N, D, C, tau) in [(64, 96, 3, 1, 1.0), (40, 200, 8, 4, 0.5)]:
        q, k, v = r.normal(size=(M, D)), r.normal(size=(N, D)), r.normal(size=(N, C))
        qt, kt, vt = (torch.from_numpy(a) for a in (q, k, v))
        vtil = vt * torch.exp(-0.5 * tau * (kt * kt).sum(1, keepdim=True))
        att = _sdpa(qt[None], kt[None], vtil[None], tau)[0]
        lse = torch.logsumexp(tau * qt @ kt.T, dim=1, keepdim=True)
        s = att * torch.exp(lse) * torch.exp(-0.5 * tau * (qt * qt).sum(1, keepdim=True))
        _close(O.gauss_sum(q, k, v, tau)[0], s.numpy(), 1e-10, 1e-13, f"alg1 M{M}N{N}D{D}")


def pin_flash_reweight(O):
    """Algorithm 2 ("reweight") of the same page: augment q~ = [q, 1, |q|^2/2],
    k~_n = [k_n, -|k_n|^2/2, 0], an extra key k~_0 = e_{D+2} carrying the value
    kappa e_{C+1}, kappa = sqrt(N+1).  The attention output splits into
    [alpha, beta]; the page stops there, and s = kappa alpha / beta follows from
    q~.k~_n = q.k_n - |k_n|^2/2 and q~.k~_0 = |q|^2/2."""
    r = _rng(3)
    for (M, N, D, C, tau) in [(50, 80, 3, 1, 1.0), (33, 150, 6, 3, 2.0)]:
        q, k, v = r.normal(size=(M, D)), r.normal(size=(N, D)), r.normal(size=(N, C))
        qt, kt, vt = (torch.from_numpy(a) for a in (q, k, v))
        kappa = math.sqrt(N + 1)
        qa = torch.cat([qt, torch.ones(M, 1, dtype=torch.float64),
                        0.5 * (qt * qt).sum(1, keepdim=True)], 1)
        ka = torch.cat([kt, -0.5 * (kt * kt).sum(1, keepdim=True),
                        torch.zeros(N, 1, dtype=torch.float64)], 1)
        k0 = torch.zeros(1, D + 2, dtype=torch.float64)
        k0[0, D + 1] = 1.0
        va = torch.cat([vt, torch.zeros(N, 1, dtype=torch.float64)], 1)
        v0 = torch.zeros(1, C + 1, dtype=torch.float64)
        v0[0, C] = kappa
        o = _sdpa(qa[None], torch.cat([k0, ka])[None], torch.cat([v0, va])[None], tau)[0]
        s = kappa * o[:, :C] / o[:, C:]
        _close(O.gauss_sum(q, k, v, tau)[0], s.numpy(), 1e-10, 1e-13, f"alg2 M{M}N{N}D{D}")


# --------------------------------------------------------------------------- special cases
def pin_coincident(O):
    """Every y_j equal to x_i gives K = 1, so the sum is sum_j w_j."""
    r = _rng(4)
    x = r.normal(size=(1, 1, 5))
    y = np.repeat(x, 9, axis=1)
    w = r.normal(size=(1, 9, 2))
    _close(O.gauss_sum(x, y, w, 3.7), w.sum(axis=1, keepdims=True), 1e-15, 1e-15, "coincident")


def pin_single_point(O):
    """N = 1: s_i = w exp(-tau/2 |x_i - y|^2), evaluated per coordinate."""
    r = _rng(5)
    x = r.normal(size=(1, 6, 4))
    y = r.normal(size=(1, 1, 4))
    w = np.array([[[1.5, -0.25]]])
    tau = 0.8
    expect = np.empty((1, 6, 2))
    for i in range(6):
        d2 = sum((x[0, i, k] - y[0, 0, k]) ** 2 for k in range(4))
        expect[0, i] = w[0, 0] * math.exp(-tau / 2 * d2)
    _close(O.gauss_sum(x, y, w, tau), expect, 1e-14, 1e-300, "single point")


def pin_separable_grid(O):
    """y on a tensor-product grid with product weights: the kernel factors over
    coordinates, so s_i = prod_k sum_{g in grid_k} exp(-tau/2 (x_ik - g)^2) u_k(g)."""
    r = _rng(6)
    grids = [np.linspace(-1.0, 1.5, 4), np.linspace(-2.0, 0.5, 3), np.linspace(0.0, 1.0, 5)]
    us = [r.uniform(-1, 1, size=len(gk)) for gk in grids]
    pts, wts = [], []
    for a in range(4):
        for b in range(3):
            for c in range(5):
                pts.append([grids[0][a], grids[1][b], grids[2][c]])
                wts.append(us[0][a] * us[1][b] * us[2][c])
    y = np.array(pts)[None]
    w = np.array(wts)[None, :, None]
    x = r.normal(size=(1, 8, 3))
    tau = 1.3
    expect = np.ones((1, 8, 1))
    for i in range(8):
        for k in range(3):
            expect[0, i, 0] *= sum(math.exp(-tau / 2 * (x[0, i, k] - g) ** 2) * u
                                   for g, u in zip(grids[k], us[k]))
    _close(O.gauss_sum(x, y, w, tau), expect, 1e-12, 1e-15, "separable grid")


# --------------------------------------------------------------------------- invariants
def pin_translation(O):
    r = _rng(7)
    x, y, w = r.normal(size=(2, 9, 3)), r.normal(size=(2, 12, 3)), r.normal(size=(2, 12, 2))
    t = np.array([0.75, -2.5, 1.25])  # exactly representable shift
    a = O.gauss_sum(x, y, w, 1.0)
    b = O.gauss_sum(x + t, y + t, w, 1.0)
    _close(b, a, 1e-12, 1e-14, "translation")
    _close(O.gauss_lse(x + t, y + t, np.abs(w) + 0.1, 1.0),
           O.gauss_lse(x, y, np.abs(w) + 0.1, 1.0), 1e-12, 1e-13, "translation lse")


def pin_small_tau(O):
    """|s - sum w| <= tau/2 max d^2 sum |w| since 0 <= 1 - e^{-u} <= u."""
    r = _rng(8)
    x, y, w = r.normal(size=(1, 5, 3)), r.normal(size=(1, 40, 3)), r.normal(size=(1, 40, 1))
    tau = 1e-9
    s = O.gauss_sum(x, y, w, tau)
    d2max = max(((x[0, i] - y[0, j]) ** 2).sum() for i in range(5) for j in range(40))
    bound = tau / 2 * d2max * np.abs(w).sum() + 1e-14
    assert np.all(np.abs(s - w.sum(axis=1, keepdims=True)) <= bound), "tau -> 0"
    # and the bound is not vacuous: s must move away from sum w as tau grows
    s1 = O.gauss_sum(x, y, w, 1.0)
    assert np.abs(s1 - w.sum(axis=1, keepdims=True)).max() > 1e-3


def pin_symmetry(O):
    """x = y: <c, S(x,x,b)> = <b, S(x,x,c)> (K symmetric); and with unit weights,
    sum_i S(x,y,1)_i = sum_j S(y,x,1)_j."""
    r = _rng(9)
    x = r.normal(size=(1, 15, 3))
    b, c = r.normal(size=(1, 15, 1)), r.normal(size=(1, 15, 1))
    lhs = float((c * O.gauss_sum(x, x, b, 0.9)).sum())
    rhs = float((b * O.gauss_sum(x, x, c, 0.9)).sum())
    assert abs(lhs - rhs) <= 1e-12 * max(1.0, abs(lhs)), f"symmetry (i): {lhs} vs {rhs}"
    y = r.normal(size=(1, 23, 3))
    s_xy = O.gauss_sum(x, y, np.ones((1, 23, 1)), 0.9).sum()
    s_yx = O.gauss_sum(y, x, np.ones((1, 15, 1)), 0.9).sum()
    assert abs(s_xy - s_yx) <= 1e-12 * abs(s_xy), f"symmetry (ii): {s_xy} vs {s_yx}"


def pin_linearity(O):
    r = _rng(10)
    x, y = r.normal(size=(1, 7, 2)), r.normal(size=(1, 9, 2))
    u, v = r.normal(size=(1, 9, 3)), r.normal(size=(1, 9, 3))
    lhs = O.gauss_sum(x, y, 2.0 * u - 0.5 * v, 1.1)
    rhs = 2.0 * O.gauss_sum(x, y, u, 1.1) - 0.5 * O.gauss_sum(x, y, v, 1.1)
    _close(lhs, rhs, 1e-12, 1e-14, "linearity")


def pin_lse_is_log_sum(O):
    r = _rng(11)
    x, y = r.normal(size=(2, 10, 3)), r.normal(size=(2, 30, 3))
    w = r.uniform(0.5, 1.5, size=(2, 30, 2))
    _close(O.gauss_lse(x, y, w, 1.0), np.log(O.gauss_sum(x, y, w, 1.0)), 1e-13, 1e-13, "lse=log sum")
    # rows subset agrees with the full evaluation
    rows = np.array([7, 0, 3])
    _close(O.gauss_lse(x, y, w, 1.0, rows=rows), O.gauss_lse(x, y, w, 1.0)[:, rows], 0, 0, "lse rows")


def pin_rows_subset(O):
    r = _rng(12)
    x, y, w = r.normal(size=(2, 11, 3)), r.normal(size=(2, 8, 3)), r.normal(size=(2, 8, 2))
    rows = np.array([10, 2, 5])
    _close(O.gauss_sum(x, y, w, 1.0, rows=rows), O.gauss_sum(x, y, w, 1.0)[:, rows], 0, 0, "rows")


# --------------------------------------------------------------------------- gradient
def pin_finite_differences(O):
    """Central differences of L = sum g * S(x, y, w) in double, h = 1e-5."""
    r = _rng(13)
    B, M, N, D, C, tau = 1, 5, 7, 3, 2, 0.7
    x, y = r.normal(size=(B, M, D)), r.normal(size=(B, N, D))
    w, g = r.normal(size=(B, N, C)), r.normal(size=(B, M, C))
    gx, gw = O.gauss_sum_bwd(x, y, w, g, tau)

    def L(xx, ww):
        return float((g * O.gauss_sum(xx, y, ww, tau)).sum())

    h = 1e-5
    fdx = np.zeros_like(x)
    for i in range(M):
        for k in range(D):
            xp, xm = x.copy(), x.copy()
            xp[0, i, k] += h
            xm[0, i, k] -= h
            fdx[0, i, k] = (L(xp, w) - L(xm, w)) / (2 * h)
    fdw = np.zeros_like(w)
    for j in range(N):
        for c in range(C):
            wp, wm = w.copy(), w.copy()
            wp[0, j, c] += h
            wm[0, j, c] -= h
            fdw[0, j, c] = (L(x, wp) - L(x, wm)) / (2 * h)
    assert _rel_l2(gx, fdx) < 1e-8, f"grad_x vs finite differences: {_rel_l2(gx, fdx):.2e}"
    assert _rel_l2(gw, fdw) < 1e-8, f"grad_w vs finite differences: {_rel_l2(gw, fdw):.2e}"
    # the subset forms agree with the full one
    rows, wrows = np.array([4, 1]), np.array([6, 0, 2])
    sx, sw = O.gauss_sum_bwd(x, y, w, g, tau, rows=rows, wrows=wrows)
    _close(sx, gx[:, rows], 0, 0, "grad_x rows")
    _close(sw, gw[:, wrows], 0, 0, "grad_w rows")


def pin_large_n_expectation(O):
    """For y iid N(0, s^2 I_D) and unit weights, E[s_i] = N (1 + tau s^2)^{-D/2}
    exp(-tau |x_i|^2 / (2 (1 + tau s^2))) (a Gaussian integral).  Statistical:
    checked at 6 standard errors."""
    r = _rng(14)
    N, D, tau, s2 = 40_000, 3, 1.0, 1.0
    y = r.normal(size=(1, N, D)) * math.sqrt(s2)
    x = np.array([[[0.0, 0.0, 0.0], [1.0, 0.5, -0.5], [2.0, 0.0, 1.0]]])
    out = O.gauss_sum(x, y, np.ones((1, N, 1)), tau)[0, :, 0]
    for i in range(3):
        xx = float((x[0, i] ** 2).sum())
        mean1 = (1 + tau * s2) ** (-D / 2) * math.exp(-tau * xx / (2 * (1 + tau * s2)))
        mean2 = (1 + 2 * tau * s2) ** (-D / 2) * math.exp(-tau * xx / (1 + 2 * tau * s2))
        se = math.sqrt(max(mean2 - mean1 ** 2, 0.0) / N)
        assert abs(out[i] / N - mean1) <= 6 * se, f"row {i}: {out[i] / N} vs {mean1} (se {se})"


# --------------------------------------------------------------------------- full gradient, LSE gradient
def pin_golden_vjp_y_tau(O):
    for case in golden()["vjp_y_tau"]:
        gy, gt = O.gauss_sum_vjp_y_tau(case["x"], case["y"], case["w"], case["g"], case["tau"])
        _close(gy, _eval_tree(case["expected_grad_y"]), 1e-14, 1e-15, case["name"] + " grad_y")
        _close(gt, _eval_tree(case["expected_grad_tau"]), 1e-14, 1e-15, case["name"] + " grad_tau")


def pin_golden_lse_bwd(O):
    for case in golden()["lse_bwd"]:
        gx, gy, gw, gt = O.gauss_lse_bwd(case["x"], case["y"], case["w"], case["g"], case["tau"])
        e = case["expected"]
        for name, got in (("grad_x", gx), ("grad_y", gy), ("grad_w", gw), ("grad_tau", gt)):
            _close(got, _eval_tree(e[name]), 1e-14, 1e-15, case["name"] + " " + name)


def _fd(f, a, h=1e-5):
    out = np.zeros_like(a)
    for idx in np.ndindex(a.shape):
        ap, am = a.copy(), a.copy()
        ap[idx] += h
        am[idx] -= h
        out[idx] = (f(ap) - f(am)) / (2 * h)
    return out


def pin_finite_differences_y_tau(O):
    """Central differences for dL/dy and dL/dtau of L = sum g * S(x, y, w, tau)."""
    r = _rng(15)
    B, M, N, D, C, tau = 2, 4, 6, 3, 2, 0.8
    x, y = r.normal(size=(B, M, D)), r.normal(size=(B, N, D))
    w, g = r.normal(size=(B, N, C)), r.normal(size=(B, M, C))
    gy, gt = O.gauss_sum_vjp_y_tau(x, y, w, g, tau)
    fdy = _fd(lambda yy: float((g * O.gauss_sum(x, yy, w, tau)).sum()), y)
    fdt = _fd(lambda tt: float((g * O.gauss_sum(x, y, w, float(tt))).sum()), np.array(tau))
    assert _rel_l2(gy, fdy) < 1e-8, f"grad_y vs finite differences: {_rel_l2(gy, fdy):.2e}"
    assert abs(gt - float(fdt)) <= 1e-8 * max(1.0, abs(gt)), f"grad_tau {gt} vs {float(fdt)}"
    rows = np.array([5, 1])
    sy, _ = O.gauss_sum_vjp_y_tau(x, y, w, g, tau, yrows=rows, want_tau=False)
    _close(sy, gy[:, rows], 0, 0, "grad_y rows")


def pin_finite_differences_lse(O):
    """Central differences of L = sum g * LSE(x, y, w, tau) for every input."""
    r = _rng(16)
    B, M, N, D, C, tau = 1, 4, 5, 2, 2, 1.3
    x, y = r.normal(size=(B, M, D)), r.normal(size=(B, N, D))
    w, g = r.uniform(0.5, 1.5, size=(B, N, C)), r.normal(size=(B, M, C))
    gx, gy, gw, gt = O.gauss_lse_bwd(x, y, w, g, tau)
    L = lambda xx, yy, ww, tt: float((g * O.gauss_lse(xx, yy, ww, tt)).sum())
    checks = [("grad_x", gx, _fd(lambda a: L(a, y, w, tau), x)),
              ("grad_y", gy, _fd(lambda a: L(x, a, w, tau), y)),
              ("grad_w", gw, _fd(lambda a: L(x, y, a, tau), w))]
    for name, got, fd in checks:
        assert _rel_l2(got, fd) < 1e-8, f"lse {name} vs finite differences: {_rel_l2(got, fd):.2e}"
    fdt = float(_fd(lambda a: L(x, y, w, float(a)), np.array(tau)))
    assert abs(gt - fdt) <= 1e-8 * max(1.0, abs(gt)), f"lse grad_tau {gt} vs {fdt}"


def pin_gradient_symmetries(O):
    """Translation: sum_i dL/dx_i + sum_j dL/dy_j = 0.  Scaling (K(a x, a y, tau) =
    K(x, y, a^2 tau)): sum x.dL/dx + sum y.dL/dy = 2 tau dL/dtau.  For the sum and the LSE."""
    r = _rng(17)
    B, M, N, D, C, tau = 1, 7, 9, 3, 2, 0.6
    x, y = r.normal(size=(B, M, D)), r.normal(size=(B, N, D))
    w, g = r.uniform(0.5, 1.5, size=(B, N, C)), r.normal(size=(B, M, C))
    gx, _ = O.gauss_sum_bwd(x, y, w, g, tau, want_w=False)
    gy, gt = O.gauss_sum_vjp_y_tau(x, y, w, g, tau)
    scale = float(np.abs(gx).sum() + np.abs(gy).sum())
    assert abs(gx.sum(axis=(0, 1)) + gy.sum(axis=(0, 1))).max() <= 1e-12 * scale, "sum: translation"
    lhs = float((x * gx).sum() + (y * gy).sum())
    assert abs(lhs - 2 * tau * gt) <= 1e-11 * max(1.0, abs(lhs)), f"sum: scaling {lhs} vs {2 * tau * gt}"
    lx, ly, _, lt = O.gauss_lse_bwd(x, y, w, g, tau)
    scale = float(np.abs(lx).sum() + np.abs(ly).sum())
    assert abs(lx.sum(axis=(0, 1)) + ly.sum(axis=(0, 1))).max() <= 1e-12 * scale, "lse: translation"
    lhs = float((x * lx).sum() + (y * ly).sum())
    assert abs(lhs - 2 * tau * lt) <= 1e-11 * max(1.0, abs(lhs)), f"lse: scaling {lhs} vs {2 * tau * lt}"


# --------------------------------------------------------------------------- k-nearest reduction
def pin_knn_against_library_sort(O):
    """torch.cdist (float64) then a stable sort: ascending distances, equal
    distances in index order."""
    r = _rng(20)
    for (B, M, N, D, K) in [(1, 9, 40, 3, 5), (2, 7, 13, 2, 13), (1, 5, 30, 8, 1)]:
        x, y = r.normal(size=(B, M, D)), r.normal(size=(B, N, D))
        d, i = O.knn(x, y, K)
        dd = torch.cdist(torch.from_numpy(x), torch.from_numpy(y),
                         compute_mode="donot_use_mm_for_euclid_dist") ** 2
        sd, si = torch.sort(dd, dim=-1, stable=True)
        _close(d, sd[..., :K].numpy(), 1e-12, 1e-14, f"knn dist B{B}M{M}N{N}K{K}")
        assert np.array_equal(i, si[..., :K].numpy()), "knn indices"


def pin_knn_ties_padding_and_grid(O):
    """Duplicated sources come out lowest index first; rows with fewer than K
    sources are padded with +inf / -1; on an integer lattice the distances and
    neighbours are known exactly."""
    y = np.array([[[0.0, 0.0], [1.0, 0.0], [0.0, 0.0], [0.0, 1.0], [1.0, 0.0]]])
    x = np.array([[[0.0, 0.0], [0.25, 0.0]]])
    d, i = O.knn(x, y, 4)
    assert i[0, 0].tolist() == [0, 2, 1, 3], i[0, 0]
    _close(d[0, 0], [0, 0, 1, 1], 0, 0, "ties distances")
    assert i[0, 1].tolist() == [0, 2, 1, 4], i[0, 1]
    _close(d[0, 1], [0.0625, 0.0625, 0.5625, 0.5625], 0, 0, "near-tie distances")
    d, i = O.knn(x, y[:, :2], 3)
    assert i[0, 0].tolist() == [0, 1, -1] and np.isinf(d[0, 0, 2])
    g = np.array([[[a, b] for a in range(4) for b in range(4)]], dtype=np.float64)  # 4x4 lattice
    q = np.array([[[1.0, 2.0], [3.0, 0.0]]])
    d, i = O.knn(q, g, 5)
    assert i[0, 0].tolist() == [6, 2, 5, 7, 10], i[0, 0]     # itself, then the 4 axis neighbours
    _close(d[0, 0], [0, 1, 1, 1, 1], 0, 0, "lattice")
    assert i[0, 1].tolist() == [12, 8, 13, 9, 4], i[0, 1]    # corner: 2 at 1, then diagonal, then 4
    _close(d[0, 1], [0, 1, 1, 2, 4], 0, 0, "lattice corner")


def pin_knn_permutation_and_f32(O):
    """Permuting the sources permutes the indices; the float decision agrees
    with the double one away from near-ties."""
    r = _rng(21)
    x, y = r.normal(size=(1, 12, 3)), r.normal(size=(1, 50, 3))
    perm = r.permutation(50)
    d, i = O.knn(x, y, 6)
    d2, i2 = O.knn(x, y[:, perm], 6)
    _close(d2, d, 0, 0, "permuted distances")
    assert np.array_equal(perm[i2], i), "permuted indices"
    df, i_f = O.knn(x.astype(np.float32), y.astype(np.float32), 6, f32=True)
    xd, yd = x.astype(np.float32).astype(np.float64), y.astype(np.float32).astype(np.float64)
    dd, idd = O.knn(xd, yd, 6)
    assert np.array_equal(i_f, idd), "float and double decisions differ on separated data"
    _close(df, dd, 1e-6, 1e-7, "float distances")


# --------------------------------------------------------------------------- diffusion operator
def pin_diffusion_operator(O):
    """A = diag(s) K diag(s): sqrt(d) is its fixed point (the Markov matrix
    D^-1 K_alpha is row-stochastic), A is symmetric with spectrum in [0, 1]
    (a Gaussian kernel is positive semi-definite), q and d are the kernel
    applications to 1 and q^-alpha, and two points give a closed form."""
    r = _rng(22)
    B, N, D, tau = 2, 40, 3, 1.7
    x = r.normal(size=(B, N, D))
    for alpha in (0.0, 0.5, 1.0):
        q, d, s = O.diffusion_scales(x, tau, alpha)
        _close(q[..., None], O.gauss_sum(x, x, np.ones((B, N, 1)), tau), 1e-13, 0, "q = K 1")
        _close(d[..., None], q[..., None] ** -alpha * O.gauss_sum(x, x, q[..., None] ** -alpha, tau),
               1e-13, 0, "d = q^-a K q^-a")
        _close(s, q ** -alpha / np.sqrt(d), 1e-14, 0, "s")
        _close(O.diffusion_apply(x, s, np.sqrt(d)[..., None], tau), np.sqrt(d)[..., None], 1e-12, 0,
               "sqrt(d) is a fixed point")
        xt = torch.from_numpy(x[0])
        K = torch.exp(-0.5 * tau * torch.cdist(xt, xt, compute_mode="donot_use_mm_for_euclid_dist") ** 2)
        A = (torch.from_numpy(s[0])[:, None] * K * torch.from_numpy(s[0])[None, :]).numpy()
        ev = np.linalg.eigvalsh(A)
        assert ev.max() <= 1 + 1e-10 and ev.min() >= -1e-10 and abs(ev.max() - 1) <= 1e-10
        u, v = r.normal(size=(1, N, 1)), r.normal(size=(1, N, 1))
        lhs = float((u * O.diffusion_apply(x[:1], s[:1], v, tau)).sum())
        rhs = float((v * O.diffusion_apply(x[:1], s[:1], u, tau)).sum())
        assert abs(lhs - rhs) <= 1e-12 * max(1.0, abs(lhs)), "symmetric"
    # two points at distance^2 = 2: K = [[1, e], [e, 1]], e = exp(-tau); q = 1 + e, A = K / (1 + e)
    x2 = np.array([[[0.0, 0.0], [1.0, 1.0]]])
    e = math.exp(-tau)
    q, d, s = O.diffusion_scales(x2, tau, 0.5)
    _close(q, [[1 + e, 1 + e]], 1e-15, 0, "two-point q")
    _close(s, [[(1 + e) ** -0.5, (1 + e) ** -0.5]], 1e-15, 0, "two-point s")
    _close(O.diffusion_apply(x2, s, np.array([[[1.0], [0.0]]]), tau), [[[1 / (1 + e)], [e / (1 + e)]]],
           1e-15, 0, "two-point A")


ALL_PINS = [
    pin_golden_sum, pin_golden_lse, pin_golden_bwd, pin_dense_library, pin_flash_prescale,
    pin_flash_reweight, pin_coincident, pin_single_point, pin_separable_grid, pin_translation,
    pin_small_tau, pin_symmetry, pin_linearity, pin_lse_is_log_sum, pin_rows_subset,
    pin_finite_differences, pin_large_n_expectation, pin_golden_vjp_y_tau, pin_golden_lse_bwd,
    pin_finite_differences_y_tau, pin_finite_differences_lse, pin_gradient_symmetries,
    pin_knn_against_library_sort, pin_knn_ties_padding_and_grid, pin_knn_permutation_and_f32,
    pin_diffusion_operator,
]

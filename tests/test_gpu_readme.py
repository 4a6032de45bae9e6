"""The README's Python example, at small sizes, against the oracle."""
import numpy as np
import pytest
import torch

import oracle

pytestmark = pytest.mark.gpu


def rel(a, b):
    a, b = np.asarray(a, np.float64).ravel(), np.asarray(b, np.float64).ravel()
    return float(np.linalg.norm(a - b) / max(np.linalg.norm(b), 1e-300))


def f64(t):
    return t.detach().double().cpu().numpy()


def test_readme_example():
    import pairwise_reductions_b200 as gs
    from pairwise_reductions_b200.autograd import gauss_sum

    g0 = torch.Generator(device="cpu").manual_seed(7)
    mk = lambda *s: (torch.randn(*s, generator=g0) / 32 ** 0.5).to("cuda", torch.float16)
    x, y = mk(2, 300, 32), mk(2, 500, 32)
    w = torch.randn(2, 500, 32, generator=g0).to("cuda", torch.float16)
    out = gs.gauss_sum_fwd(x, y, w, tau=1.0)
    assert out.dtype == torch.float32 and out.shape == (2, 300, 32)
    assert rel(out.cpu(), oracle.gauss_sum(f64(x), f64(y), f64(w), 1.0)) <= 3e-3
    wp = w.abs() + 0.1
    lse = gs.gauss_lse_fwd(x, y, wp, 1.0)
    assert rel(lse.cpu(), oracle.gauss_lse(f64(x), f64(y), f64(wp), 1.0)) <= 3e-3

    g = torch.randn(2, 300, 1, generator=g0).cuda()
    w1 = w[..., :1].contiguous()
    s, gx, gw = gs.gauss_sum_fwd_bwd(x, y, w1, g, 1.0)
    rgx, rgw = oracle.gauss_sum_bwd(f64(x), f64(y), f64(w1), f64(g), 1.0)
    assert rel(s.cpu(), oracle.gauss_sum(f64(x), f64(y), f64(w1), 1.0)) <= 3e-3
    assert rel(gx.cpu(), rgx) <= 3e-3 and rel(gw.cpu(), rgw) <= 3e-3

    xr = x.float().requires_grad_()
    gauss_sum(xr, y.float(), w.float(), 1.0).sum().backward()
    rgx2, _ = oracle.gauss_sum_bwd(f64(x), f64(y), f64(w), np.ones((2, 300, 32)), 1.0)
    assert rel(xr.grad.cpu(), rgx2) <= 1e-5

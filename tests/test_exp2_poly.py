"""The FMA-pipe exponential the kernels use for part of their kernel values:
its minimax coefficients are regenerated from the Remez exchange and checked
(CPU), and the device evaluation is checked against float64 2^x (GPU)."""
import os
import re
import subprocess
import sys

import numpy as np
import pytest
import torch

CSRC = os.path.join(os.path.dirname(os.path.dirname(os.path.abspath(__file__))),
                    "pairwise_reductions_b200", "csrc")


def _bounds():
    text = open(os.path.join(CSRC, "exp2_poly.cuh")).read()
    return {int(d): float(v) for d, v in re.findall(r"kD(\d)MaxRelErr = ([0-9.e+-]+)f", text)}


def test_header_matches_the_remez_generator():
    r = subprocess.run([sys.executable, os.path.join(CSRC, "gen_exp2_poly.py"), "--check"])
    assert r.returncode == 0, "exp2_poly.cuh is stale: rerun gen_exp2_poly.py"


def test_error_bounds_are_what_the_paths_need():
    b = _bounds()
    assert b[3] < 1e-4      # below half an fp16 ulp (2^-12): P is stored in fp16
    assert b[5] < 3e-7      # a few fp32 ulps: the fp32 path is held to 1e-5 relative


def test_remez_levels_the_error():
    sys.path.insert(0, CSRC)
    try:
        import gen_exp2_poly as g
    finally:
        sys.path.pop(0)
    for n in (3, 5):
        coef, E = g.remez(n)
        x = np.linspace(-0.5, 0.5, 20001)
        err = np.polyval(coef[::-1], x) / np.exp2(x) - 1
        # equioscillation: max error equals the levelled error, n + 2 alternations
        assert abs(np.max(np.abs(err)) - E) <= 0.02 * E
        sign_changes = np.count_nonzero(np.diff(np.sign(err[np.abs(err) > 0.5 * E])))
        assert sign_changes >= n + 1


@pytest.mark.gpu
@pytest.mark.parametrize("degree", [3, 5])
def test_device_exp2_poly_against_float64(degree):
    import pairwise_reductions_b200 as gs
    g = torch.Generator().manual_seed(degree)
    x = torch.cat([torch.linspace(-125.0, 20.0, 200001), torch.rand(100000, generator=g) * 145 - 125,
                   torch.arange(-125, 21, dtype=torch.float32)]).float()
    out = gs.test_exp2_poly(x.cuda(), degree).cpu().double().numpy()
    ref = np.exp2(x.double().numpy())
    rel = np.abs(out / ref - 1)
    bound = _bounds()[degree] + 2.0 ** -23
    assert rel.max() <= bound, (rel.max(), bound)
    # clamped below -125
    low = gs.test_exp2_poly(torch.tensor([-200.0, -1000.0], device="cuda"), degree).cpu().numpy()
    assert np.all(low > 0) and np.all(low <= 2.0 ** -124)

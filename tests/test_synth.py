"""The seeded input generators (`synth/`): reproducible, in the documented
distributions and dtypes, and free of the method's arithmetic."""
import math
import os

import torch

import synth

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def test_same_seed_same_values_and_different_seed_different_values():
    a = synth.make_inputs("d3_10k", M=500, N=400)
    b = synth.make_inputs("d3_10k", M=500, N=400)
    c = synth.make_inputs("d3_10k", M=500, N=400, seed=12345)
    for k in ("x", "y", "w"):
        assert torch.equal(a[k], b[k])
        assert not torch.equal(a[k], c[k])


def test_default_seed_is_one_thousand_plus_the_workload_id():
    for name, w in synth.BY_NAME.items():
        a = synth.make_inputs(name, B=1, M=8, N=8)
        b = synth.make_inputs(name, B=1, M=8, N=8, seed=1000 + w.wid)
        assert torch.equal(a["x"], b["x"]), name


def test_dtypes_and_shapes_follow_the_workload():
    for name, w in synth.BY_NAME.items():
        d = synth.make_inputs(name, B=2, M=16, N=24)
        want = {"f32": torch.float32, "f16": torch.float16, "bf16": torch.bfloat16}[w.dtype]
        assert d["x"].dtype == d["y"].dtype == d["w"].dtype == want, name
        assert d["x"].shape == (2, 16, w.D) and d["y"].shape == (2, 24, w.D)
        assert d["w"].shape == (2, 24, w.C)
        if w.with_g:
            assert d["g"].dtype == torch.float32 and d["g"].shape == (2, 16, w.C)


def test_distributions_match_the_recipe():
    # large samples of each distribution: mean and variance within 5 standard errors
    d = synth.make_inputs("d3_10k", M=20000, N=20000)
    for k in ("x", "y", "w"):
        v = d[k].double().flatten()
        n = v.numel()
        assert abs(v.mean()) < 5 / math.sqrt(n)
        assert abs(v.var() - 1.0) < 5 * math.sqrt(2.0 / n)
    d = synth.make_inputs("d3_1m_lse", M=20000, N=20000)
    x, w = d["x"].double().flatten(), d["w"].double().flatten()
    assert 0.0 <= float(x.min()) and float(x.max()) < 1.0
    assert 0.5 <= float(w.min()) and float(w.max()) < 1.5
    d = synth.make_inputs("d32_c32_f32", B=1, M=4000, N=4000)
    x = d["x"].double().flatten()
    assert abs(x.var() - 1.0 / 32) < 5 * math.sqrt(2.0 / x.numel()) / 32


def test_half_precision_values_are_the_round_to_nearest_casts():
    d16 = synth.make_inputs("d32_c32", B=1, M=64, N=64)
    d64 = synth.make_inputs("d32_c32", B=1, M=64, N=64, dtype="f64")
    for k in ("x", "y", "w"):
        assert torch.equal(d64[k].to(torch.float16), d16[k])


def test_no_method_arithmetic_in_the_generators():
    src = open(os.path.join(ROOT, "synth", "__init__.py")).read()
    for token in ("exp(", "cdist", "logsumexp", "matmul", "einsum", ".mm(", "bmm("):
        assert token not in src, token


def test_row_samples_are_sorted_distinct_and_seeded():
    a = synth.sample_rows(1000, 100, seed=3)
    assert torch.equal(a, synth.sample_rows(1000, 100, seed=3))
    assert torch.all(a[1:] > a[:-1]) and int(a.min()) >= 0 and int(a.max()) < 1000
    assert torch.equal(synth.sample_rows(10, 20, seed=3), torch.arange(10))

"""Plant plausible mistakes in copies of the oracle (on the CPU) and check that
the pins catch every one of them.  The planted copies are built in a temporary
directory from edited source text; the real oracle is never modified."""
import functools
import os
import subprocess

import pytest

import oracle
from oracle.build import SRC
from pins import ALL_PINS

# (name, [(old, new, count)]) -- count = how many occurrences to replace (0 = all)
MUTANTS = [
    ("kernel factor tau instead of tau/2", [("double k = exp(-0.5 * tau", "double k = exp(-1.0 * tau", 1)]),
    ("kernel sign flipped", [("double k = exp(-0.5 * tau", "double k = exp(0.5 * tau", 1)]),
    ("last coordinate dropped", [("for (int64_t k = 0; k < D; ++k) {\n        double d", "for (int64_t k = 0; k < D - 1; ++k) {\n        double d", 1)]),
    ("difference replaced by sum", [("double d = p[k] - q[k];", "double d = p[k] + q[k];", 1)]),
    ("weights read in reverse order", [("const double *wj = w + (bb * N + j) * C;\n                for (int64_t c = 0; c < C; ++c)\n                    cs_add(&acc[c], k * wj[c]);", "const double *wj = w + (bb * N + (N - 1 - j)) * C;\n                for (int64_t c = 0; c < C; ++c)\n                    cs_add(&acc[c], k * wj[c]);", 1)]),
    ("weight channel transposed", [("cs_add(&acc[c], k * wj[c]);", "cs_add(&acc[c], k * wj[C - 1 - c]);", 1)]),
    ("batch offset ignored for x", [("const double *xi = x + (bb * M + i) * D;", "const double *xi = x + i * D;", 0)]),
    ("lse drops the weights", [("cs_add(&acc[c], wj[c] * e);", "cs_add(&acc[c], e);", 1)]),
    ("lse without the max shift", [("double e = exp(f - m);", "double e = exp(f);", 1),
                                   ("m + log(cs_value(&acc[c]))", "log(cs_value(&acc[c]))", 1)]),
    ("lse shift added twice", [("m + log(cs_value(&acc[c]))", "2 * m + log(cs_value(&acc[c]))", 1)]),
    ("grad_x sign of the difference", [("cs_add(&acc[k], kv * gw * (xi[k] - yj[k]));", "cs_add(&acc[k], kv * gw * (yj[k] - xi[k]));", 1)]),
    ("grad_x drops the g.w coupling", [("gw += gi[c] * wj[c];", "gw += gi[c];", 1)]),
    ("grad_x factor tau/2", [("-tau * cs_value(&acc[k])", "-0.5 * tau * cs_value(&acc[k])", 1)]),
    ("grad_w drops the upstream gradient", [("cs_add(&acc[c], kv * gi[c]);", "cs_add(&acc[c], kv);", 1)]),
    ("grad_y sign of the difference", [("cs_add(&acc[k], kv * gw * (yj[k] - xi[k]));", "cs_add(&acc[k], kv * gw * (xi[k] - yj[k]));", 1)]),
    ("grad_tau factor 1/2 dropped", [("*grad_tau = -0.5 * cs_value(&total);", "*grad_tau = -cs_value(&total);", 1)]),
    ("grad_tau without the squared distance", [("cs_add(&row, exp(-0.5 * tau * d2) * d2 * gw);", "cs_add(&row, exp(-0.5 * tau * d2) * gw);", 1)]),
    ("lse grad unnormalised weights", [("double p = w[(bb * N + j) * C + c] * e / zs;", "double p = w[(bb * N + j) * C + c] * e;", 1)]),
    ("lse grad_w uses p instead of p / w", [("grad_w[(bb * N + j) * C + c] += gic * e / zs;", "grad_w[(bb * N + j) * C + c] += gic * p;", 1)]),
    ("lse grad_y sign", [("grad_y[(bb * N + j) * D + k] += tau * gic * p * diff;", "grad_y[(bb * N + j) * D + k] += -tau * gic * p * diff;", 1)]),
    ("knn keeps the largest", [("if (!(d < bd[K - 1] || (d == bd[K - 1] && j < bj[K - 1])))", "if (!(d > bd[K - 1] || (d == bd[K - 1] && j < bj[K - 1])))", 1)]),
    ("knn ties by the higher index", [("while (p > 0 && (d < bd[p - 1] || (d == bd[p - 1] && j < bj[p - 1]))) {", "while (p > 0 && (d < bd[p - 1] || (d == bd[p - 1] && j > bj[p - 1]))) {", 1)]),
    ("knn float distance drops a coordinate", [("for (int64_t k = 1; k < D; ++k) {\n                    e = xi[k] - yj[k];", "for (int64_t k = 2; k < D; ++k) {\n                    e = xi[k] - yj[k];", 1)]),
    ("diffusion d without the left q^-alpha", [("double di = pow(qq[t], -alpha) * cs_value(&acc);", "double di = cs_value(&acc);", 1)]),
    ("diffusion s with d^-1 instead of d^-1/2", [("s[t] = pow(qq[t], -alpha) / sqrt(di);", "s[t] = pow(qq[t], -alpha) / di;", 1)]),
    ("diffusion apply without the right scaling", [("double ksj = k * s[bb * N + j];", "double ksj = k;", 1)]),
    ("grad_w kernel against x_0 only", [("const double *xi = x + (bb * M + i) * D;\n                    const double *gi", "const double *xi = x + (bb * M) * D;\n                    const double *gi", 1)]),
]


def _build_mutant(tmp_path, idx, edits):
    src = open(SRC).read()
    for old, new, count in edits:
        assert old in src, f"mutation anchor not found: {old!r}"
        src = src.replace(old, new) if count == 0 else src.replace(old, new, count)
    cpath = tmp_path / f"mutant{idx}.c"
    cpath.write_text(src)
    lib = tmp_path / f"libmutant{idx}.so"
    subprocess.run(["gcc", "-O2", "-std=c11", "-fPIC", "-shared", "-fopenmp", str(cpath), "-o",
                    str(lib), "-lm"], check=True)
    return oracle._load(str(lib))


class _Handle:
    def __init__(self, lib):
        self.gauss_sum = functools.partial(oracle.gauss_sum, lib=lib)
        self.gauss_lse = functools.partial(oracle.gauss_lse, lib=lib)
        self.gauss_sum_bwd = functools.partial(oracle.gauss_sum_bwd, lib=lib)
        self.gauss_sum_vjp_y_tau = functools.partial(oracle.gauss_sum_vjp_y_tau, lib=lib)
        self.gauss_lse_bwd = functools.partial(oracle.gauss_lse_bwd, lib=lib)
        self.knn = functools.partial(oracle.knn, lib=lib)
        self.diffusion_scales = functools.partial(oracle.diffusion_scales, lib=lib)
        self.diffusion_apply = functools.partial(oracle.diffusion_apply, lib=lib)


@pytest.mark.parametrize("idx", range(len(MUTANTS)), ids=[m[0] for m in MUTANTS])
def test_pins_catch_planted_mistake(tmp_path, idx):
    name, edits = MUTANTS[idx]
    h = _Handle(_build_mutant(tmp_path, idx, edits))
    caught = []
    for pin in ALL_PINS:
        try:
            pin(h)
        except AssertionError:
            caught.append(pin.__name__)
    assert caught, f"no pin caught the planted mistake: {name}"

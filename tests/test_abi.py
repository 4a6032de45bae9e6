"""The C ABI library loads, exports every symbol include/gauss.h declares, and
rejects bad arguments on the host -- all without a GPU (no compute call)."""
import ctypes
import os
import re

import pytest

import pairwise_reductions_b200 as gs

INCLUDE = os.path.join(os.path.dirname(os.path.dirname(os.path.abspath(__file__))), "include")


def _declared_functions():
    text = "".join(open(os.path.join(INCLUDE, f)).read() for f in sorted(os.listdir(INCLUDE))
                   if f.endswith(".h"))
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b([a-z_][a-z0-9_]*)\s*\(", text)) - {"if", "sizeof"})


def test_header_declares_the_entry_points():
    names = _declared_functions()
    for n in ("gauss_sum_fwd", "gauss_lse_fwd", "gauss_sum_bwd", "gs_workspace_bytes",
              "gs_status_string", "gs_last_device_error", "gs_version"):
        assert n in names


def test_library_exports_every_declared_symbol():
    lib = ctypes.CDLL(gs.LIB_PATH)
    missing = [n for n in _declared_functions() if not hasattr(lib, n)]
    assert not missing, f"declared in gauss.h but not exported: {missing}"
    # and the binding binds exactly those names
    assert set(gs.SIGNATURES) == set(_declared_functions())


def test_status_strings_and_version():
    for code in range(7):
        assert gs.status_string(code)
    assert gs.library().gs_version() >= 100


NULL = ctypes.c_void_p(0)
FAKE = ctypes.c_void_p(0x100000)   # 16-byte aligned, never dereferenced on these paths
ODD = ctypes.c_void_p(0x100004)


def _fwd(fn="gauss_sum_fwd", x=FAKE, y=FAKE, w=FAKE, out=FAKE, B=1, M=10, N=10, D=3, C=1, tau=1.0,
         dt=0, ws=NULL, wsb=0):
    return getattr(gs.library(), fn)(x, y, w, out, B, M, N, D, C, tau, dt, ws, wsb, NULL)


@pytest.mark.parametrize("fn", ["gauss_sum_fwd", "gauss_lse_fwd"])
def test_invalid_arguments_are_rejected_before_any_launch(fn):
    assert _fwd(fn, x=NULL) == 1
    assert _fwd(fn, out=NULL) == 1
    assert _fwd(fn, tau=0.0) == 1
    assert _fwd(fn, tau=-1.0) == 1
    assert _fwd(fn, tau=float("nan")) == 1
    assert _fwd(fn, tau=float("inf")) == 1
    assert _fwd(fn, M=-1) == 1
    assert _fwd(fn, D=0) == 1
    assert _fwd(fn, C=0) == 1
    assert _fwd(fn, dt=7) == 1
    assert _fwd(fn, x=ODD) == 3
    assert _fwd(fn, D=129) == 2            # fp32 covers D <= 128 (sums), D <= 8 (LSE)
    assert _fwd(fn, dt=1, D=129) == 2      # tensor-core path covers D <= 128
    assert _fwd(fn, B=70000) == 2


def test_every_entry_point_takes_half_precision():
    # fp16 / bf16: the log-sum-exp (unsplit tensor-core operands) asks for its workspace;
    # its backward and kNN widen the inputs to fp32 copies in the workspace
    assert _fwd("gauss_lse_fwd", dt=1, D=32) == 4
    assert _fwd("gauss_lse_fwd", dt=2, D=3) == 4
    ws = gs.workspace_bytes
    f32 = ws(gs.GS_OP_LSE_BWD, 1, 100, 200, 3, 2, gs.GS_F32)
    f16 = ws(gs.GS_OP_LSE_BWD, 1, 100, 200, 3, 2, gs.GS_F16)
    assert f16 >= f32 + (100 * 3 + 200 * 3 + 200 * 2) * 4     # plus the widened copies
    assert ws(gs.GS_OP_KNN, 1, 100, 200, 3, 4, gs.GS_BF16) >= \
        ws(gs.GS_OP_KNN, 1, 100, 200, 3, 4, gs.GS_F32) + (100 * 3 + 200 * 3) * 4


def test_fp32_wide_features_route_to_the_tensor_core_path():
    # fp32 with D > 8: sums, the log-sum-exp and its backward (split-fp16 tensor
    # cores) and kNN (chunked CUDA-core kernel) ask for their workspace
    assert _fwd("gauss_lse_fwd", D=9) == 4
    assert _fwd("gauss_sum_fwd", D=9) == 4
    lib = gs.library()
    i64 = ctypes.c_void_p(0x100000)
    assert lib.gauss_knn(FAKE, FAKE, FAKE, i64, 1, 10, 10, 9, 1, 0, NULL, 0, NULL) == 4
    assert lib.gauss_knn(FAKE, FAKE, FAKE, i64, 1, 10, 10, 129, 1, 0, NULL, 0, NULL) == 2


def test_empty_problems_are_no_ops_without_pointers():
    assert _fwd(x=NULL, y=NULL, w=NULL, out=NULL, B=0) == 0
    assert _fwd(x=NULL, out=NULL, M=0) == 0


def test_workspace_too_small_is_reported():
    # tensor-core path always needs packed operands in the workspace
    assert _fwd(dt=1, D=32, C=32, M=1000, N=1000) == 4


def test_workspace_query():
    ws = gs.workspace_bytes
    assert ws(gs.GS_OP_SUM, 0, 10, 10, 3, 1, gs.GS_F32) == 0
    assert ws(gs.GS_OP_SUM, 1, 10, 0, 3, 1, gs.GS_F32) == 0
    big = ws(gs.GS_OP_SUM, 4, 65536, 65536, 32, 32, gs.GS_F16)
    # packed x~ and y~ (2 x 4 x 65536 x 64 x 2 B) + v^T (4 x 32 x 65536 x 2 B) at least
    assert big >= 2 * 4 * 65536 * 64 * 2 + 4 * 32 * 65536 * 2
    assert ws(gs.GS_OP_LSE, 1, 1000, 1000, 3, 1, gs.GS_F32) >= 2 * 1000 * 4
    assert ws(gs.GS_OP_SUM_BWD, 4, 16384, 16384, 32, 1, gs.GS_F16) >= 4 * 16384 * 33 * 4
    # fp32 D > 8: packed split rows [hi | lo] of x and y at least
    assert ws(gs.GS_OP_SUM, 1, 1000, 1000, 9, 1, gs.GS_F32) >= 2 * 1000 * 2 * 16 * 4
    with pytest.raises(ValueError):
        ws(gs.GS_OP_SUM, 1, 10, 10, 129, 1, gs.GS_F32)
    assert ws(gs.GS_OP_LSE, 1, 1000, 1000, 9, 1, gs.GS_F32) >= 2 * 1000 * 2 * 16 * 4
    assert ws(gs.GS_OP_LSE_BWD, 1, 1000, 1000, 9, 1, gs.GS_F32) > 0
    assert ws(gs.GS_OP_KNN, 1, 10, 10, 9, 1, gs.GS_F32) > 0
    with pytest.raises(ValueError):
        ws(gs.GS_OP_KNN, 1, 10, 10, 129, 1, gs.GS_F32)
    # the forward + backward call: the x-pass sums, g's parts and the dL/dw
    # partials of every 128-row tile on top of the pass scratch
    fb = ws(gs.GS_OP_SUM_FWD_BWD, 4, 16384, 16384, 32, 1, gs.GS_F16)
    assert fb >= 4 * 16384 * 33 * 4 + 4 * 16384 * 4 + 128 * 4 * 16384 * 4
    assert ws(gs.GS_OP_SUM_FWD_BWD, 1, 1000, 1000, 3, 1, gs.GS_F32) >= 1000 * 4 * 4
    assert ws(gs.GS_OP_DIFFUSION_BLOCK, 1, 500, 2000, 3, 2, gs.GS_F32) >= 0
    assert ws(gs.GS_OP_DIFFUSION_BLOCK, 1, 500, 2000, 32, 2, gs.GS_F16) > 0
    with pytest.raises(ValueError):
        ws(8, 1, 10, 10, 3, 1, gs.GS_F32)


def test_bwd_argument_checks():
    lib = gs.library()
    args = lambda **k: (k.get("x", FAKE), FAKE, FAKE, k.get("g", FAKE), k.get("gx", FAKE),
                        k.get("gw", FAKE), 1, 10, 10, 3, 1, k.get("tau", 1.0), 0, NULL, 0, NULL)
    assert lib.gauss_sum_bwd(*args(g=NULL)) == 1
    assert lib.gauss_sum_bwd(*args(tau=0.0)) == 1
    assert lib.gauss_sum_bwd(*args(gx=ODD)) == 3
    assert lib.gauss_sum_bwd(*args(gx=NULL, gw=NULL)) == 0   # nothing requested


def test_build_refuses_spills_in_tensor_core_kernels():
    import importlib.util
    path = os.path.join(os.path.dirname(INCLUDE), "pairwise_reductions_b200", "build.py")
    spec = importlib.util.spec_from_file_location("_gs_build_for_test", path)
    b = importlib.util.module_from_spec(spec)
    spec.loader.exec_module(b)
    ok_log = ("ptxas info    : Compiling entry function '_Z15tc_gauss_kernelILi64E' for 'sm_100a'\n"
              "    0 bytes stack frame, 0 bytes spill stores, 0 bytes spill loads\n")
    b._check_spills(ok_log)
    with pytest.raises(RuntimeError):
        b._check_spills(ok_log.replace("0 bytes spill stores", "12 bytes spill stores"))


def test_binding_status_checks_are_well_formed():
    """Every _check(name, status) call in the binding names a declared entry
    point and passes exactly two arguments (a static check: the GPU-only paths
    that reach these calls cannot run here)."""
    import ast
    src = open(os.path.join(os.path.dirname(INCLUDE), "pairwise_reductions_b200", "__init__.py")).read()
    calls = [n for n in ast.walk(ast.parse(src)) if isinstance(n, ast.Call)
             and getattr(n.func, "id", None) == "_check"]
    assert calls
    declared = set(_declared_functions())
    for c in calls:
        assert len(c.args) == 2 and not c.keywords, ast.unparse(c)
        first = c.args[0]
        if isinstance(first, ast.Constant):
            assert first.value in declared, first.value


@pytest.mark.parametrize("n", [1_000, 10_000, 100_000, 1_000_000])
def test_split_counts_stay_within_the_combines(n):
    # small-D fp32: the sum's workspace is its split partials [S, B, M, C]; the
    # log-sum-exp's is (m, l) per split, and its finalize merges the splits
    # within one warp, so S <= 32 there; the sum allows up to 256 splits and at
    # most 2^25 partial floats
    ws = gs.workspace_bytes
    s_sum = ws(gs.GS_OP_SUM, 1, n, n, 3, 1, gs.GS_F32) // (4 * n)
    s_lse = ws(gs.GS_OP_LSE, 1, n, n, 3, 1, gs.GS_F32) // (8 * n)
    assert 1 <= s_lse <= 32, s_lse
    assert s_sum <= 256 and s_sum * n <= (1 << 25) + 256, s_sum
    # every split keeps at least 128 columns
    assert s_sum <= max(1, n // 128)


def test_autograd_wrappers_validate_tau_before_any_launch():
    import torch
    from pairwise_reductions_b200 import autograd
    x = torch.zeros(4, 3)
    with pytest.raises(ValueError):
        autograd.gauss_sum(x, x, torch.zeros(4, 1), torch.ones(2))
    with pytest.raises(ValueError):
        autograd.gauss_lse(x, x, torch.ones(4, 1), torch.ones(3))


def test_binding_rejects_mismatched_tensors_before_any_call():
    import torch
    x = torch.zeros(2, 5, 3)
    y = torch.zeros(2, 7, 3)
    w = torch.zeros(2, 7, 1)
    with pytest.raises(ValueError):           # batch sizes differ
        gs.gauss_sum_fwd(x, torch.zeros(1, 7, 3), torch.zeros(1, 7, 1), 1.0)
    with pytest.raises(ValueError):           # feature sizes differ
        gs.gauss_sum_fwd(x, torch.zeros(2, 7, 4), w, 1.0)
    with pytest.raises(ValueError):           # weights for another number of sources
        gs.gauss_sum_fwd(x, y, torch.zeros(2, 6, 1), 1.0)
    with pytest.raises(ValueError):           # mixed dtypes
        gs.gauss_sum_fwd(x, y, w.double(), 1.0)
    with pytest.raises(ValueError):           # not contiguous
        gs.gauss_sum_fwd(torch.zeros(2, 3, 5).transpose(1, 2), y, w, 1.0)
    with pytest.raises(ValueError):           # 1-D input
        gs.gauss_sum_fwd(torch.zeros(5), y, w, 1.0)
    g = torch.zeros(2, 5, 1)
    with pytest.raises(ValueError):           # upstream gradient of the wrong shape
        gs.gauss_sum_bwd(x, y, w, torch.zeros(2, 4, 1), 1.0)
    with pytest.raises(ValueError):           # upstream gradient not float32
        gs.gauss_sum_vjp(x, y, w, g.double(), 1.0)
    with pytest.raises(ValueError):           # saved sums of the wrong width
        gs.gauss_sum_bwd_saved(x, y, w, g, torch.zeros(2, 5, 3), 1.0)
    with pytest.raises(ValueError):           # lse of the wrong shape
        gs.gauss_lse_bwd(x, y, w, torch.zeros(2, 5, 2), g, 1.0)


def test_testing_hooks_reject_bad_arguments_without_a_device_call():
    lib = gs.library()
    assert lib.gs_test_set_waits(999, 0) == 1
    assert lib.gs_test_set_waits(10_000_000_001, 0) == 1
    assert lib.gs_test_set_waits(1_000_000, 3) == 1
    assert lib.gs_test_set_waits(1_000_000, -1) == 1
    assert lib.gs_test_read_error_word(NULL, NULL) == 1
    # the measurement probes check their arguments before anything is launched
    assert lib.gs_test_ex2_probe(NULL, NULL, 1, 1, NULL) == 1
    assert lib.gs_test_ex2_probe(FAKE, FAKE, 0, 1, NULL) == 1
    assert lib.gs_test_ex2_probe(FAKE, FAKE, 1, 0, NULL) == 1
    assert lib.gs_test_mma_probe(FAKE, FAKE, 1, 64, 48, NULL) == 1
    assert lib.gs_test_mma_probe(FAKE, FAKE, 1, 0, 64, NULL) == 1
    assert lib.gs_test_mma_probe(NULL, FAKE, 1, 64, 64, NULL) == 1

"""The tensor-core kernels' abort path, driven without a fault: a short limit
on the bounded mbarrier waits and a stall mode (include/gauss_testing.h) make a
wait run out on purpose.  The call must come back with the device error word
raised (GS_ERR_TIMEOUT once, then clear), its drain of the loads and MMAs it
had issued must finish within the limit (bit 2 clear), and the next normal
call must match the oracle on the same context."""
import numpy as np
import pytest

import oracle
import synth

pytestmark = pytest.mark.gpu

GS_ERR_TIMEOUT = 5
LIMIT_NS = 1_000_000          # 1 ms
DEFAULT_NS = 2_000_000_000


def gs():
    import pairwise_reductions_b200 as m
    return m


def rel_l2(a, b):
    a = np.asarray(a, dtype=np.float64).ravel()
    b = np.asarray(b, dtype=np.float64).ravel()
    return float(np.linalg.norm(a - b) / max(np.linalg.norm(b), 1e-300))


# fp16: the value MMAs (C = 32) and the register values (C = 1); fp32 D = 32:
# the split kernel's register values (C = 2) and tensor-core values (C = 32)
CASES = [("f16", 32), ("f16", 1), ("f32", 2), ("f32", 32)]


@pytest.mark.parametrize("stall", [1, 2], ids=["issuer_idle", "exp_warps_idle"])
@pytest.mark.parametrize("dtype,C", CASES, ids=[f"{d}_c{c}" for d, c in CASES])
def test_wait_expiry_reports_timeout_and_context_stays_usable(dtype, C, stall):
    m = gs()
    inp = synth.make_inputs(4, seed=51, B=2, M=700, N=3000, D=32, C=C, dtype=dtype)
    x, y, w = (inp[k].cuda() for k in "xyw")
    assert m.test_read_error_word() == 0
    m.test_set_waits(LIMIT_NS, stall)
    try:
        m.gauss_sum_fwd(x, y, w, inp["tau"])          # outputs unspecified
        word = m.test_read_error_word()
        m.gauss_sum_fwd(x, y, w, inp["tau"])
        status = m.last_device_error()
        again = m.last_device_error()
    finally:
        m.test_set_waits(DEFAULT_NS, 0)
    assert word & 1, f"no wait ran out (word {word})"
    assert not word & 4, f"a drain of issued work ran out (word {word})"
    assert status == GS_ERR_TIMEOUT
    assert again == 0, "the error word is cleared once read"
    out = m.gauss_sum_fwd(x, y, w, inp["tau"]).cpu().numpy()
    ref = oracle.gauss_sum(*(synth.as_f64(inp[k]) for k in "xyw"), inp["tau"])
    tol = 1e-5 if dtype == "f32" else 3e-3
    assert rel_l2(out, ref) <= tol, rel_l2(out, ref)
    assert m.test_read_error_word() == 0


def test_set_waits_rejects_bad_arguments():
    m = gs()
    for limit, stall in ((999, 0), (10_000_000_001, 0), (LIMIT_NS, 3), (LIMIT_NS, -1)):
        with pytest.raises(m.GaussError):
            m.test_set_waits(limit, stall)
    m.test_set_waits(DEFAULT_NS, 0)

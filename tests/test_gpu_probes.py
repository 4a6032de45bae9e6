"""Two measured figures the design rests on, re-measured from this repository
by the probes behind include/gauss_testing.h: the MUFU ex2 rate of an SM (the
denominator of the roofline the benchmark reports for the exponential-bound
kernels: 16 results a clock) and the cost of back-to-back tcgen05.mma kind::f16
instructions from one thread (55.6, 55.6, 64.9 and 128.9 cycles at N = 32, 64,
128, 256 when last measured on a B200), which bounds the tensor-core kernels'
MMA-issuing thread.
Both take the SM clock from clock64, so the SM's clock speed cancels out."""
import pytest
import torch

import pairwise_reductions_b200 as gs

pytestmark = pytest.mark.gpu


def _sms():
    return torch.cuda.get_device_properties(torch.cuda.current_device()).multi_processor_count


def test_mufu_ex2_rate_per_sm():
    blocks = _sms()
    gs.test_ex2_probe(blocks, 64)   # warm-up
    iters = 4096
    cycles = gs.test_ex2_probe(blocks, iters).cpu().double()
    assert bool((cycles > 0).all())
    rate = 1024 * 8 * iters / cycles
    med = float(rate.median())
    print(f"ex2 results a clock per SM: median {med:.2f} (min {float(rate.min()):.2f}, "
          f"max {float(rate.max()):.2f}, {blocks} SMs)")
    # 16 a clock (4 per sub-partition); the probe's loop pays a little on top
    assert 14.0 <= med <= 16.5, med


@pytest.mark.parametrize("n_cols,lo,hi", [(32, 30, 80), (64, 30, 80), (128, 55, 95), (256, 110, 175)])
def test_mma_issue_cost(n_cols, lo, hi):
    blocks = _sms()
    gs.test_mma_probe(blocks, 64, n_cols)   # warm-up
    n = 512
    cycles, status = gs.test_mma_probe(blocks, n, n_cols)
    assert int(status.item()) == 0, "an MMA completion wait ran out"
    per = cycles.cpu().double() / n
    med = float(per.median())
    print(f"M = 128, N = {n_cols}, K = 16 kind::f16: {med:.1f} cycles an MMA "
          f"(min {float(per.min()):.1f}, max {float(per.max()):.1f})")
    assert lo <= med <= hi, med

"""The k-nearest validity check itself, on the CPU: answers decided in fp32 by
the oracle's fixed order of operations pass it, and plausible wrong answers
(a far index, a distance off by more than its rounding bound, a broken order
or tie-break, a repeated index, wrong padding) fail it."""
import numpy as np
import pytest
import torch

import oracle
from knn_check import knn_valid_under_exact_distances as check


def _pts(B, M, N, D, seed, grid=False):
    g = torch.Generator().manual_seed(seed)
    if grid:
        x = torch.randint(0, 3, (B, M, D), generator=g).float() * 0.5 + 0.25
        y = torch.randint(0, 3, (B, N, D), generator=g).float() * 0.5
        return x.numpy(), y.numpy()
    return (torch.randn(B, M, D, generator=g).float().numpy(),
            torch.randn(B, N, D, generator=g).float().numpy())


@pytest.mark.parametrize("shape,grid", [((2, 60, 300, 3, 5), False), ((1, 40, 200, 128, 8), False),
                                        ((1, 50, 400, 4, 12), True), ((1, 20, 7, 3, 10), False),
                                        ((1, 30, 100, 1, 32), False)])
def test_fp32_decided_answers_pass(shape, grid):
    B, M, N, D, K = shape
    x, y = _pts(B, M, N, D, 3, grid)
    od, oi = oracle.knn(x, y, K, f32=True)
    check(x, y, od, oi, K)


def _answer():
    x, y = _pts(1, 40, 500, 3, 5)
    od, oi = oracle.knn(x, y, 6, f32=True)
    return x, y, od.copy(), oi.copy()


def test_far_index_fails():
    x, y, od, oi = _answer()
    far = int(np.argmax(((x[0, 3][None, :] - y[0]) ** 2).sum(-1)))
    oi[0, 3, -1] = far
    with pytest.raises(AssertionError):
        check(x, y, od, oi, 6)


def test_distance_off_its_bound_fails():
    x, y, od, oi = _answer()
    od[0, 5, 2] = np.nextafter(od[0, 5, 2], np.float32(np.inf)) * np.float32(1 + 2e-6)
    od[0, 5, 3:] = np.maximum(od[0, 5, 3:], od[0, 5, 2])   # keep the order valid
    with pytest.raises(AssertionError):
        check(x, y, od, oi, 6)


def test_broken_order_fails():
    x, y, od, oi = _answer()
    od[0, 7, [0, 1]] = od[0, 7, [1, 0]]
    oi[0, 7, [0, 1]] = oi[0, 7, [1, 0]]
    with pytest.raises(AssertionError):
        check(x, y, od, oi, 6)


def test_tie_by_higher_index_fails():
    x = np.zeros((1, 1, 2), np.float32)
    y = np.array([[[1, 0], [0, 1], [2, 0]]], np.float32)   # two sources at distance 1
    od, oi = oracle.knn(x, y, 2, f32=True)
    check(x, y, od, oi, 2)
    with pytest.raises(AssertionError):
        check(x, y, od, oi[..., ::-1].copy(), 2)


def test_repeated_index_fails():
    x, y, od, oi = _answer()
    oi[0, 9, 1] = oi[0, 9, 0]
    od[0, 9, 1] = od[0, 9, 0]
    with pytest.raises(AssertionError):
        check(x, y, od, oi, 6)


def test_padding_past_n_fails():
    x, y = _pts(1, 5, 4, 3, 8)
    od, oi = oracle.knn(x, y, 6, f32=True)
    check(x, y, od, oi, 6)
    bad = oi.copy()
    bad[0, 0, 5] = 0
    with pytest.raises(AssertionError):
        check(x, y, od, bad, 6)

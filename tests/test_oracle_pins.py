"""The oracle against facts fixed outside itself (closed forms, library
routines, the flash-attention identities, invariants, finite differences)."""
import pytest

import oracle
from pins import ALL_PINS


class _Real:
    gauss_sum = staticmethod(oracle.gauss_sum)
    gauss_lse = staticmethod(oracle.gauss_lse)
    gauss_sum_bwd = staticmethod(oracle.gauss_sum_bwd)
    gauss_sum_vjp_y_tau = staticmethod(oracle.gauss_sum_vjp_y_tau)
    gauss_lse_bwd = staticmethod(oracle.gauss_lse_bwd)
    knn = staticmethod(oracle.knn)
    diffusion_scales = staticmethod(oracle.diffusion_scales)
    diffusion_apply = staticmethod(oracle.diffusion_apply)


@pytest.mark.parametrize("pin", ALL_PINS, ids=[p.__name__ for p in ALL_PINS])
def test_pin(pin):
    pin(_Real)


def test_thread_count_is_reported():
    assert oracle.num_threads() >= 1

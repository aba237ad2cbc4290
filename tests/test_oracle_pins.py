"""The fp64 oracle against its pins (CPU only)."""
import pytest

import oracle
import pins


@pytest.mark.parametrize("pin", pins.ALL_PINS, ids=lambda f: f.__name__)
def test_pin(pin):
    pin(oracle.default())


def test_orders_are_permutations():
    for H, W in [(1, 1), (1, 7), (7, 1), (4, 6), (64, 64)]:
        for k in range(4):
            o = oracle.cross_order(k, H, W)
            assert sorted(o.tolist()) == list(range(H * W))


def test_threads_do_not_change_results():
    import numpy as np

    rng = np.random.default_rng(11)
    u, dr, z = (rng.normal(size=(3, 40, 5)) for _ in range(3))
    B, C = rng.normal(size=(3, 40, 4)), rng.normal(size=(3, 40, 4))
    A, D, bias = -rng.uniform(0.1, 2, size=(2, 5, 4)), rng.normal(size=(2, 5)), rng.normal(size=(2, 5))
    orc = oracle.default()
    n0 = orc.max_threads()
    orc.set_threads(1)
    y1 = orc.vim_bidir(u, dr, z, B, C, A, D, bias)
    orc.set_threads(max(2, n0))
    y2 = orc.vim_bidir(u, dr, z, B, C, A, D, bias)
    orc.set_threads(n0)
    assert (y1 == y2).all()

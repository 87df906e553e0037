"""The float64 oracle against facts fixed outside it (CPU only)."""
import numpy as np
import pytest

import oracle.powersgd64 as ora
from oracle import philox64

from . import _pins


@pytest.mark.parametrize("check", _pins.ALL_CHECKS, ids=lambda f: f.__name__)
def test_pin(check):
    check(ora)


def test_warm_start_convergence_config0_shape():
    # the 256 x 128, r = 2 shape of the single-matrix workload
    _pins.check_warm_start_convergence(ora, m=256, n=128, r=2, steps=14)


def test_philox_matches_numpy_bitgen():
    # numpy's Philox bit generator is Philox4x64-10; it increments its
    # counter before each block, so block b of key k uses counter b + 1
    for key in ((1, 2), (1234, 0), (2**64 - 1, 7)):
        g = np.random.Philox(key=np.array(key, dtype=np.uint64))
        raw = [int(x) for x in g.random_raw(12)]
        mine = []
        for b in range(1, 4):
            mine += list(philox64.philox4x64_10((b, 0, 0, 0), key))
        assert raw == mine


def test_box_muller_closed_form():
    # u0 = 1/2 + 2^-54 and u1 = 1/4 + 2^-54: rho = sqrt(2 ln 2), angle pi/2
    w_half = (1 << 52) << 11
    w_quarter = (1 << 51) << 11
    z = philox64.box_muller_block((w_half, w_quarter, w_half, w_quarter))
    rho = np.sqrt(2.0 * np.log(2.0))
    assert abs(z[0]) < 1e-14 and abs(z[1] - rho) < 1e-14


def test_initial_q_is_standard_normal():
    q = philox64.initial_q(1234, 0, 2500, 4).astype(np.float64).ravel()
    assert abs(q.mean()) < 4.0 / np.sqrt(q.size)
    assert abs(q.var() - 1.0) < 6.0 * np.sqrt(2.0 / q.size)
    # no two layers share a stream
    q1 = philox64.initial_q(1234, 1, 2500, 4).astype(np.float64).ravel()
    assert abs(np.corrcoef(q, q1)[0, 1]) < 0.05

"""The parity cases are fair tests: on every shape set, rank and worker
count the GPU parity tests gate, the oracle itself moves by at most half
the float32 tolerance (1e-4) when its inputs are perturbed by one float32
ulp, over the same free-running steps (the largest, 3.4e-5, is rank 32
with three workers at the fourth step).  A case above the tolerance would
have to be reported rather than gated."""
import pytest

from . import _harness as H
from ._probe import max_sensitivity
from .test_parity_gpu import FULL_RANK, MIXED

MARGIN = 0.5 * H.TOL["f32"]


@pytest.mark.parametrize("rank", [1, 2, 3, 4, 8, 16, 32])
@pytest.mark.parametrize("workers", [1, 3])
def test_mixed_shapes_are_well_conditioned(rank, workers):
    assert max_sensitivity(H.small_workload(MIXED, rank, workers), steps=3) <= MARGIN


@pytest.mark.parametrize("rank", [4, 16, 32])
def test_four_step_mode_cases_are_well_conditioned(rank):
    # lazy errors, sum-first and power iterations run four steps on these
    assert max_sensitivity(H.small_workload(MIXED, rank, 3), steps=4) <= MARGIN


@pytest.mark.parametrize("rank", [2, 8, 16, 32])
def test_sixteen_worker_cases_are_well_conditioned(rank):
    assert max_sensitivity(H.small_workload(MIXED[:4], rank, 16), steps=2) <= MARGIN


@pytest.mark.parametrize("workers", [64, 256])
def test_many_worker_cases_are_well_conditioned(workers):
    assert max_sensitivity(H.small_workload([(40, 130), (33, 37), (64, 576)], 32, workers), steps=1) <= MARGIN


@pytest.mark.parametrize("rank", sorted(FULL_RANK))
def test_full_rank_cases_are_well_conditioned(rank):
    assert max_sensitivity(H.small_workload(FULL_RANK[rank], rank, 3), steps=3) <= MARGIN


def test_probe_detects_an_ill_conditioned_case():
    # four strong directions and noise at 1e-5: at rank 8 the last four
    # columns of P_bar sit near the noise floor (kept by the drop rule), and
    # their orthogonalisation amplifies a one-ulp change past the tolerance
    wl = H.small_workload([(64, 48)], 8, 1, noise=("abs", 1e-5))
    assert max_sensitivity(wl, steps=3) > H.TOL["f32"]


def test_resnet18_full_size_is_well_conditioned():
    # every layer of the ResNet-18 set at full size, three steps, as the
    # full-size GPU parity test runs it
    from synth import C1
    assert max_sensitivity(C1, steps=3) <= MARGIN


@pytest.mark.parametrize("rank", [1, 4, 32])
def test_sweep_1024_sampled_layers_are_well_conditioned(rank):
    from synth import C4B
    assert max_sensitivity(C4B.with_rank(rank), steps=3, layers_idx=[0, 97, 255]) <= MARGIN

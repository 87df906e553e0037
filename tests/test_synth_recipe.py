"""The input recipe: seeded low-rank-plus-noise gradients with the stated
spectrum, noise scale and subspace rotation, reproducible from the seed."""
import math

import numpy as np
import torch

from synth import GradientSource
from synth.gradients import mix_seed, pack_offsets, sigmas

from . import _harness as H


def test_spectrum_and_orthonormal_bases():
    wl = H.small_workload([(64, 48), (30, 70)], 4, 2)
    src = GradientSource(wl, seed=3)
    for l in range(2):
        U, V, s = src.basis(0, l)
        np.testing.assert_allclose(U.T @ U, np.eye(4), atol=1e-12)
        np.testing.assert_allclose(V.T @ V, np.eye(4), atol=1e-12)
        np.testing.assert_allclose(s, [5.0, 2.5, 1.25, 0.625])
        # the noiseless part has exactly these singular values
        low = src.lowrank(0, l).double().numpy()
        sv = np.linalg.svd(low, compute_uv=False)[:5]
        np.testing.assert_allclose(sv[:4], s, rtol=1e-6)
        assert sv[4] < 1e-5


def test_noise_scale_relative_to_rms():
    # "rel" noise: std = 0.1 * RMS(U diag(sigma) V^T) = 0.1 * ||sigma|| / sqrt(mn)
    m, n = 400, 300
    wl = H.small_workload([(m, n)], 4, 1)
    src = GradientSource(wl, seed=5)
    want = 0.1 * math.sqrt(float(np.sum(sigmas(4) ** 2))) / math.sqrt(m * n)
    assert abs(src.noise_std(0) - want) < 1e-15
    g = src.layer_grad(0, 0, 0).double() - src.lowrank(0, 0).double()
    assert abs(float(g.std()) / want - 1.0) < 0.02


def test_gradients_reproducible_and_fresh_per_step_and_worker():
    wl = H.small_workload([(32, 40)], 2, 2)
    a, b = GradientSource(wl, seed=9), GradientSource(wl, seed=9)
    assert torch.equal(a.layer_grad(0, 1, 0), b.layer_grad(0, 1, 0))
    assert not torch.equal(a.layer_grad(0, 0, 0), a.layer_grad(0, 1, 0))
    assert not torch.equal(GradientSource(wl, seed=10).layer_grad(0, 0, 0), b.layer_grad(0, 0, 0))
    assert not torch.equal(a.layer_grad(1, 0, 0), b.layer_grad(0, 0, 0))
    # steps are generated in order (the rotating subspace advances)
    try:
        a.layer_grad(0, 0, 0)
        raise AssertionError("an earlier step after a later one must be refused")
    except ValueError:
        pass
    assert mix_seed(1, 2) != mix_seed(2, 1) and 0 <= mix_seed(1, 2) < 2 ** 63


def test_rotation_keeps_bases_orthonormal_and_turns_them():
    from dataclasses import replace
    wl = replace(H.small_workload([(50, 40)], 2, 1), rotate=0.05)
    src = GradientSource(wl, seed=2)
    U0, V0, _ = [x.copy() if hasattr(x, "copy") else x for x in src.basis(0, 0)]
    U1, V1, _ = src.basis(1, 0)
    np.testing.assert_allclose(U1.T @ U1, np.eye(U1.shape[1]), atol=1e-12)
    np.testing.assert_allclose(V1.T @ V1, np.eye(V1.shape[1]), atol=1e-12)
    # a rotation by 0.05 rad in one plane moves each column by at most
    # 2 sin(0.025) < 0.05 and does move the subspace
    assert np.max(np.linalg.norm(U1 - U0, axis=0)) <= 2 * math.sin(0.025) + 1e-12
    assert np.max(np.abs(U1 - U0)) > 0


def test_pack_offsets_alignment():
    offs = pack_offsets([(3, 5), (7, 11), (2, 2)], 64)
    assert offs == [0, 64, 64 + 128, 64 + 128 + 64]
    assert all(o % 64 == 0 for o in offs)

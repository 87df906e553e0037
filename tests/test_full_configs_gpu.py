"""GPU parity at the workloads' full sizes, in the launch configuration the
benchmark times: the library runs every layer of the workload; the float64
oracle follows sampled layers (layers are independent, so a sampled
layer's oracle trajectory is an exact reference), and properties that hold
at any size are checked on the rest."""
import os

import numpy as np
import pytest
import torch

from synth import C1, C2, C3, C4A, C4B

from . import _harness as H

pytestmark = pytest.mark.gpu


def _host_ram_gb():
    try:
        with open("/proc/meminfo") as f:
            for line in f:
                if line.startswith("MemAvailable"):
                    return int(line.split()[1]) / 1e6
    except Exception:
        pass
    return 0.0


def _free_dev_gb():
    return torch.cuda.mem_get_info()[0] / 1e9


def test_resnet18_all_layers():
    # 20 matrices, r = 2, W = 16: every layer against the oracle, 3 steps
    _, hist = H.run_sampled(C1, 3, range(len(C1.layers)))
    for t, e in enumerate(hist):
        H.assert_close(e, H.TOL["f32"], f"step {t}")


def test_resnet18_lazy_all_layers():
    _, hist = H.run_sampled(C1, 3, range(len(C1.layers)), lazy=True)
    for t, e in enumerate(hist):
        H.assert_close(e, H.TOL["f32"], f"step {t}")


def test_lstm_sampled_layers():
    # 2600 x 650 gate weight and 33280 x 650 decoder, r = 4, W = 16
    if _host_ram_gb() < 40:
        pytest.skip("host RAM too small for the float64 oracle of the 33280 x 650 layer")
    _, hist = H.run_sampled(C2, 2, [0, 7])
    for t, e in enumerate(hist):
        H.assert_close(e, H.TOL["f32"], f"step {t}")


def test_transformer_bf16_sampled_layers():
    # 24 blocks, bf16 gradients, r = 4, W = 4: one layer of each shape
    need = C3.elements_per_worker * C3.workers * (2 + 4) / 1e9 + 4
    if _free_dev_gb() < need:
        pytest.skip(f"needs {need:.0f} GB of device memory")
    if _host_ram_gb() < 40:
        pytest.skip("host RAM too small for the float64 oracle of the sampled layers")
    _, hist = H.run_sampled(C3, 2, [0, 1, 2, 3])
    for t, e in enumerate(hist):
        H.assert_close(e, H.TOL["bf16"], f"step {t}")


@pytest.mark.parametrize("rank", [1, 4, 32])
def test_sweep_1024_sampled(rank):
    # 256 matrices of 1024 x 1024, W = 8, rotating subspace
    wl = C4B.with_rank(rank)
    _, hist = H.run_sampled(wl, 3, [0, 97, 255])
    for t, e in enumerate(hist):
        H.assert_close(e, H.TOL["f32"], f"r={rank} step {t}")


@pytest.mark.parametrize("rank", [4, 32])
def test_sweep_8192_properties(rank):
    # the single 8192 x 8192 matrix, W = 8: identities at full size, and the
    # oracle itself when the host has room for it
    wl = C4A.with_rank(rank)
    run = H.PackedRun(wl)
    run.fill(0)
    torch.cuda.synchronize()
    G = run.host_grads(0)
    E0 = [np.zeros(wl.layers[0]) for _ in range(wl.workers)]
    run.step()
    torch.cuda.synchronize()
    run.lib.status()
    pe = H.property_errors(run, 0, G, E0)
    assert pe["orth"] < 1e-5, pe
    assert pe["identity"] < 1e-6, pe
    assert pe["q_proj"] < 1e-4, pe
    if _host_ram_gb() >= 64:
        import oracle.powersgd64 as ora
        o = ora.step(G, E0, run.Q0[0].double().numpy())
        errs = {"P_hat": H.rel_fro(H.to64(run.P[0]), o["P_hat"]), "Q_bar": H.rel_fro(H.to64(run.Q[0]), o["Q_bar"])}
        H.assert_close(errs, H.TOL["f32"], f"r={rank}")

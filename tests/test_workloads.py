"""The synthetic workloads keep the shapes, ranks, worker counts and sizes
that the measurements and the design notes quote (the pages' configurations
as read there: ResNet-18 matrix list, 3-layer LSTM, 24-block transformer
with bf16 gradients, the two rank sweeps)."""
import pytest

from synth import workloads as W


@pytest.mark.parametrize("key,name,layers,rank,workers,dtype,per_worker,vectors", [
    ("0", "single_256x128_r2_w1", 1, 2, 1, "f32", 32_768, 0),
    ("1", "resnet18_r2_w16", 20, 2, 16, "f32", 11_162_624, 39),
    ("2", "lstm3_r4_w16", 8, 4, 16, "f32", 53_404_000, 0),
    ("3", "transformer24_bf16_r4_w4", 96, 4, 4, "bf16", 4_831_838_208, 0),
    ("4a", "sweep_8192sq_w8", 1, 1, 8, "f32", 67_108_864, 0),
    ("4b", "sweep_256x1024sq_w8", 256, 1, 8, "f32", 268_435_456, 0),
])
def test_workload_shapes(key, name, layers, rank, workers, dtype, per_worker, vectors):
    wl = W.get(key)
    assert wl.name == name
    assert len(wl.layers) == layers
    assert (wl.rank, wl.workers, wl.grad_dtype) == (rank, workers, dtype)
    assert wl.elements_per_worker == per_worker
    assert wl.elements == per_worker * workers
    assert len(wl.vectors or ()) == vectors
    for m, n in wl.layers:
        assert min(m, n) >= rank


def test_resnet18_vectors_and_momentum():
    # BN gamma and beta of every listed conv plus the FC bias: 9,482 elements
    wl = W.get("1")
    assert sum(wl.vectors) == 9_482
    assert wl.momentum == (0.9, 0.1)


def test_sweeps_take_every_rank_up_to_32():
    for key in ("4a", "4b"):
        wl = W.get(key)
        for r in (1, 2, 4, 8, 16, 32):
            assert wl.with_rank(r).rank == r

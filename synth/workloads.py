"""The five synthetic workloads the compression step is checked and timed on.

Shapes follow the layer sets the PowerSGD experiments use ("anthology-of-the-sota"
note-152, "Key results": ResNet18 on CIFAR-10 with rank 2, a 3-layer LSTM on
WikiText-2 with rank 4) plus a transformer-block set and a rank/shape sweep.
No dataset is used: gradients are seeded low-rank-plus-noise matrices (see
gradients.py).  This module holds no arithmetic of the method.
"""
from __future__ import annotations

from dataclasses import dataclass, field
from typing import List, Optional, Tuple


@dataclass(frozen=True)
class Workload:
    name: str
    layers: Tuple[Tuple[int, int], ...]      # (m, n) per matrix, row-major, ld = n
    rank: int
    workers: int
    steps: int
    grad_dtype: str = "f32"                  # "f32" or "bf16" (dtype of G only)
    noise: Tuple[str, float] = ("rel", 0.1)  # ("abs", std) or ("rel", fraction of RMS(low-rank part))
    vectors: Tuple[int, ...] = ()            # lengths of the 1-D tensors averaged uncompressed
    momentum: Optional[Tuple[float, float]] = None  # (beta, lr) of post-compression momentum
    rotate: float = 0.0                      # subspace rotation angle per step (radians)
    ranks: Tuple[int, ...] = ()              # rank sweep (rank is the first entry)
    spectrum_terms: int = 4                  # K in sum_k sigma_k u_k v_k^T, sigma_k = 10 * 2^-k
    spectrum: Tuple[float, ...] = ()         # explicit sigma_1 >= sigma_2 >= ... (replaces the default)

    @property
    def elements_per_worker(self) -> int:
        return sum(m * n for m, n in self.layers)

    @property
    def elements(self) -> int:
        return self.workers * self.elements_per_worker

    def with_rank(self, r: int) -> "Workload":
        from dataclasses import replace
        return replace(self, rank=r)


def _resnet18_layers():
    # conv weights out x (in*3*3), 1x1 shortcuts, FC; the CIFAR stem conv is
    # not in the list (the listed matrices add up to 11,162,624 elements)
    L = []
    L += [(64, 576)] * 4
    L += [(128, 576)]
    L += [(128, 1152)] * 3
    L += [(256, 1152)]
    L += [(256, 2304)] * 3
    L += [(512, 2304)]
    L += [(512, 4608)] * 3
    L += [(128, 64), (256, 128), (512, 256)]
    L += [(10, 512)]
    return tuple(L)


def _resnet18_vectors(layers):
    # batch-norm gamma and beta (length = out channels) for every conv and
    # shortcut, plus the 10-element FC bias
    v = []
    for m, n in layers[:-1]:
        v += [m, m]
    v.append(10)
    return tuple(v)


_R18 = _resnet18_layers()

C0 = Workload(
    name="single_256x128_r2_w1", layers=((256, 128),), rank=2, workers=1, steps=10,
    noise=("abs", 0.01))

C1 = Workload(
    name="resnet18_r2_w16", layers=_R18, rank=2, workers=16, steps=100,
    vectors=_resnet18_vectors(_R18), momentum=(0.9, 0.1))

C2 = Workload(
    name="lstm3_r4_w16", layers=((2600, 650),) * 6 + ((33280, 650),) * 2, rank=4, workers=16, steps=50)

C3 = Workload(
    name="transformer24_bf16_r4_w4",
    layers=((4096, 12288), (4096, 4096), (16384, 4096), (4096, 16384)) * 24,
    rank=4, workers=4, steps=20, grad_dtype="bf16")

C4A = Workload(
    name="sweep_8192sq_w8", layers=((8192, 8192),), rank=1, workers=8, steps=50,
    rotate=0.05, ranks=(1, 2, 4, 8, 16, 32))

C4B = Workload(
    name="sweep_256x1024sq_w8", layers=((1024, 1024),) * 256, rank=1, workers=8, steps=50,
    rotate=0.05, ranks=(1, 2, 4, 8, 16, 32))

ALL = {w.name: w for w in (C0, C1, C2, C3, C4A, C4B)}
BY_INDEX = {"0": C0, "1": C1, "2": C2, "3": C3, "4a": C4A, "4b": C4B}


def get(key: str) -> Workload:
    if key in BY_INDEX:
        return BY_INDEX[key]
    return ALL[key]

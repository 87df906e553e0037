"""Conditioning probe for the parity cases (CPU only): how far the float64
oracle's own results move when its inputs are perturbed by one float32
ulp.  A parity case is a fair test at a tolerance only if this sensitivity
sits well below it: otherwise rounding alone, in any correct float32
implementation, could exceed the bar."""
from typing import Dict, List, Optional, Sequence, Tuple

import numpy as np

import oracle.powersgd64 as ora
from synth import GradientSource, Workload

ULP = 2.0 ** -24   # unit roundoff of float32


def _perturb(a: np.ndarray, rng) -> np.ndarray:
    return a * (1.0 + ULP * rng.choice([-1.0, 1.0], size=a.shape))


def ulp_sensitivity(wl: Workload, steps: int, seed: int = 1234, probe_seed: int = 5,
                    layers_idx: Optional[Sequence[int]] = None) -> List[Dict[str, float]]:
    """Free-running steps of the oracle on the workload's gradients, once as
    generated and once with every gradient and the initial Q perturbed by
    one float32 ulp (random sign).  Returns, per step, the largest relative
    Frobenius change over the layers of P_hat, Q_bar, G_hat and E'_w (E'
    relative to ||M_w||), the same measures the parity tests use.
    layers_idx: the layers to follow (default all), with the workload's own
    per-layer inputs."""
    src = GradientSource(wl, seed)
    rng = np.random.default_rng(probe_seed)
    W = wl.workers
    idx = list(range(len(wl.layers))) if layers_idx is None else list(layers_idx)
    a_state: Dict[int, Tuple] = {}
    b_state: Dict[int, Tuple] = {}
    for l in idx:
        m, n = wl.layers[l]
        q = src.initial_q(l).double().numpy()
        a_state[l] = ([np.zeros((m, n)) for _ in range(W)], q)
        b_state[l] = ([np.zeros((m, n)) for _ in range(W)], _perturb(q, rng))
    out = []
    for t in range(steps):
        worst: Dict[str, float] = {}
        for l in idx:
            G = [src.layer_grad(t, w, l).double().numpy() for w in range(W)]
            a = ora.step(G, *a_state[l])
            b = ora.step([_perturb(g, rng) for g in G], *b_state[l])
            a_state[l] = (a["E_new"], a["Q_bar"])
            b_state[l] = (b["E_new"], b["Q_bar"])
            for k in ("P_hat", "Q_bar", "G_hat"):
                d = np.linalg.norm(a[k] - b[k]) / np.linalg.norm(a[k])
                worst[k] = max(worst.get(k, 0.0), d)
            e = max(np.linalg.norm(a["E_new"][w] - b["E_new"][w]) / np.linalg.norm(a["M"][w]) for w in range(W))
            worst["E_new"] = max(worst.get("E_new", 0.0), e)
        out.append(worst)
    return out


def max_sensitivity(wl: Workload, steps: int, seed: int = 1234, layers_idx=None) -> float:
    return max(max(d.values()) for d in ulp_sensitivity(wl, steps, seed, layers_idx=layers_idx))

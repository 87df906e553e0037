"""Seeded synthetic gradients for the workloads in workloads.py.

Serves both sides of every check (the CUDA library and the float64 oracle)
and holds none of the method's arithmetic.

Per layer l (m x n) the generator fixes orthonormal U (m x K), V (n x K) from
QR of seeded Gaussians and sigma_k = 10 * 2^-k (k = 1..K), or the workload's
explicit spectrum when it gives one.  The gradient of
worker w at step t is

    G = U diag(sigma) V^T + s * N(0, 1)

with s = 0.01 ("abs") or s = 0.1 * RMS(U diag(sigma) V^T) ("rel"), noise
fresh for every (step, worker, layer).  With a rotation angle theta, before
step t >= 1 both U and V are turned by a Givens-type rotation in a seeded
random 2-plane {a, b}: x -> x + (cos theta - 1)(a a^T + b b^T) x
+ sin theta (b a^T - a b^T) x.

The per-(step, worker, layer) stream is seeded with a splitmix64 mix of the
base seed and those indices, so the same gradient comes out for the same
indices on any device, up to the device's own RNG.
"""
from __future__ import annotations

import math
from typing import Dict, List, Optional, Sequence

import numpy as np
import torch

from .workloads import Workload

_MASK = (1 << 64) - 1


def mix_seed(*parts: int) -> int:
    """splitmix64 chain over the integer parts -> a 63-bit torch seed."""
    z = 0x9E3779B97F4A7C15
    for p in parts:
        z = (z + (int(p) & _MASK) + 0x9E3779B97F4A7C15) & _MASK
        x = z
        x = ((x ^ (x >> 30)) * 0xBF58476D1CE4E5B9) & _MASK
        x = ((x ^ (x >> 27)) * 0x94D049BB133111EB) & _MASK
        z = x ^ (x >> 31)
    return z & ((1 << 63) - 1)


_TAG_BASIS, _TAG_NOISE, _TAG_ROT, _TAG_Q0, _TAG_VEC, _TAG_STATE = 1, 2, 3, 4, 5, 6


def sigmas(K: int) -> np.ndarray:
    return np.array([10.0 * 2.0 ** (-k) for k in range(1, K + 1)], dtype=np.float64)


def _gaussian(shape, seed: int, device="cpu", dtype=torch.float32) -> torch.Tensor:
    g = torch.Generator(device=device)
    g.manual_seed(seed)
    return torch.randn(*shape, generator=g, device=device, dtype=dtype)


def _orthonormal(rows: int, cols: int, seed: int) -> np.ndarray:
    a = _gaussian((rows, cols), seed, dtype=torch.float64).numpy()
    q, r = np.linalg.qr(a)
    return q * np.sign(np.diag(r))[None, :]


def _rotate(X: np.ndarray, a: np.ndarray, b: np.ndarray, theta: float) -> np.ndarray:
    ax = a @ X
    bx = b @ X
    return X + (math.cos(theta) - 1.0) * (np.outer(a, ax) + np.outer(b, bx)) \
        + math.sin(theta) * (np.outer(b, ax) - np.outer(a, bx))


def _plane(dim: int, seed: int):
    ab = _orthonormal(dim, 2, seed)
    return ab[:, 0], ab[:, 1]


class GradientSource:
    """Generates the workload's gradients step by step.

    basis(l) -> (U, V, sigma) in float64 on the host for the current step;
    layer_grad(step, w, l, device) -> m x n tensor (grad dtype);
    fill(step, bufs) writes every (w, l) gradient into bufs[w][l].
    """

    def __init__(self, wl: Workload, seed: int = 1234):
        self.wl = wl
        self.seed = seed
        self._U: List[np.ndarray] = []
        self._V: List[np.ndarray] = []
        for l, (m, n) in enumerate(wl.layers):
            K = min(len(wl.spectrum) if wl.spectrum else wl.spectrum_terms, m, n)
            self._U.append(_orthonormal(m, K, mix_seed(seed, _TAG_BASIS, l, 0)))
            self._V.append(_orthonormal(n, K, mix_seed(seed, _TAG_BASIS, l, 1)))
        self._basis_step = 0

    # subspace for the given step (rotations applied before steps 1, 2, ...)
    def _advance_to(self, step: int):
        if step < self._basis_step:
            raise ValueError("gradient steps must be requested in order")
        while self._basis_step < step:
            t = self._basis_step + 1
            if self.wl.rotate:
                for l in range(len(self.wl.layers)):
                    m, n = self.wl.layers[l]
                    a, b = _plane(m, mix_seed(self.seed, _TAG_ROT, l, t, 0))
                    self._U[l] = _rotate(self._U[l], a, b, self.wl.rotate)
                    a, b = _plane(n, mix_seed(self.seed, _TAG_ROT, l, t, 1))
                    self._V[l] = _rotate(self._V[l], a, b, self.wl.rotate)
            self._basis_step = t

    def basis(self, step: int, l: int):
        self._advance_to(step)
        U, V = self._U[l], self._V[l]
        return U, V, self._sigmas(U.shape[1])

    def _sigmas(self, K: int) -> np.ndarray:
        if self.wl.spectrum:
            return np.asarray(self.wl.spectrum[:K], dtype=np.float64)
        return sigmas(K)

    def lowrank(self, step: int, l: int, device="cpu") -> torch.Tensor:
        U, V, s = self.basis(step, l)
        Us = torch.from_numpy(U * s[None, :]).to(device=device, dtype=torch.float32)
        Vt = torch.from_numpy(np.ascontiguousarray(V.T)).to(device=device, dtype=torch.float32)
        return Us @ Vt

    def noise_std(self, l: int) -> float:
        kind, val = self.wl.noise
        if kind == "abs":
            return float(val)
        m, n = self.wl.layers[l]
        K = min(len(self.wl.spectrum) if self.wl.spectrum else self.wl.spectrum_terms, m, n)
        rms = math.sqrt(float(np.sum(self._sigmas(K) ** 2))) / math.sqrt(m * n)
        return float(val) * rms

    def _torch_dtype(self):
        return torch.bfloat16 if self.wl.grad_dtype == "bf16" else torch.float32

    def layer_grad(self, step: int, w: int, l: int, device="cpu", lowrank: Optional[torch.Tensor] = None,
                   out: Optional[torch.Tensor] = None) -> torch.Tensor:
        m, n = self.wl.layers[l]
        if lowrank is None:
            lowrank = self.lowrank(step, l, device)
        noise = _gaussian((m, n), mix_seed(self.seed, _TAG_NOISE, step, w, l), device=device)
        g = lowrank + self.noise_std(l) * noise
        g = g.to(self._torch_dtype())
        if out is not None:
            out.copy_(g)
            return out
        return g

    def fill(self, step: int, bufs: Sequence[Sequence[torch.Tensor]]):
        """bufs[w][l]: destination m x n tensors (any device, grad dtype)."""
        for l in range(len(self.wl.layers)):
            dev = bufs[0][l].device
            low = self.lowrank(step, l, dev)
            for w in range(self.wl.workers):
                self.layer_grad(step, w, l, dev, lowrank=low, out=bufs[w][l])

    def initial_q(self, l: int, rank: Optional[int] = None) -> torch.Tensor:
        """Q0 ~ N(0, 1), n x r float32 on the host, shared by all workers."""
        r = self.wl.rank if rank is None else rank
        n = self.wl.layers[l][1]
        return _gaussian((n, r), mix_seed(self.seed, _TAG_Q0, l, r))

    def vector_grads(self, step: int, w: int) -> List[torch.Tensor]:
        return [_gaussian((k,), mix_seed(self.seed, _TAG_VEC, step, w, i))
                for i, k in enumerate(self.wl.vectors)]

    def random_state(self, l: int, w: int, scale: float, device="cpu") -> torch.Tensor:
        """An arbitrary error-memory state (for one-step checks from a state
        other than zero): scale * N(0, 1), float32."""
        m, n = self.wl.layers[l]
        return scale * _gaussian((m, n), mix_seed(self.seed, _TAG_STATE, l, w), device=device)


def pack_offsets(layers: Sequence[Sequence[int]], align_elems: int) -> List[int]:
    """Element offsets of each layer in one flat per-worker buffer, every
    layer starting on a multiple of align_elems elements."""
    off, out = 0, []
    for m, n in layers:
        out.append(off)
        off += m * n
        off = (off + align_elems - 1) // align_elems * align_elems
    out.append(off)
    return out

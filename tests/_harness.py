"""Shared harness of the GPU parity tests: seeded inputs from synth (on the
host for small cases, on the device for full-size ones), the library run
through its C ABI binding, and the float64 oracle run on the same inputs.
No oracle input or expected value comes from the library's outputs: the
oracle keeps its own state (free-running) from the same initial state and
the same gradient sequence."""
from __future__ import annotations

import math
from dataclasses import replace
from typing import Dict, List, Optional, Sequence

import numpy as np
import torch

import oracle.powersgd64 as ora
from synth import GradientSource, Workload

TOL = {"f32": 1e-4, "bf16": 2e-2}


def rel_fro(got, want, denom=None) -> float:
    got = np.asarray(got, dtype=np.float64)
    want = np.asarray(want, dtype=np.float64)
    d = np.linalg.norm(want) if denom is None else denom
    num = np.linalg.norm(got - want)
    if d == 0.0:
        return float(num)
    return float(num / d)


def to64(t: torch.Tensor) -> np.ndarray:
    return t.detach().to("cpu", torch.float64).numpy()


class LibRun:
    """Device state of one library context (per-layer tensors)."""

    def __init__(self, wl: Workload, seed: int = 1234, lazy: bool = False, sum_first: bool = False,
                 recon: bool = True, device: str = "cuda", iters: int = 1, warm_start: bool = True,
                 svd_every: int = 0, svd_iters: int = 8, svd_oversampling=None):
        from rank_gradient_compression_02_b200 import PowerSGD
        self.wl = wl
        self.seed = seed
        self.src = GradientSource(wl, seed)
        self.lib = PowerSGD(wl.layers, wl.rank, wl.workers, seed=seed, grad_dtype=wl.grad_dtype,
                            lazy_errors=lazy, sum_first=sum_first, power_iters=iters, warm_start=warm_start,
                            svd_every=svd_every, svd_iters=svd_iters, svd_oversampling=svd_oversampling)
        self.lazy = lazy
        gdt = torch.bfloat16 if wl.grad_dtype == "bf16" else torch.float32
        W, L = wl.workers, len(wl.layers)
        self.G = [[torch.empty(m, n, device=device, dtype=gdt) for (m, n) in wl.layers] for _ in range(W)]
        self.E = [[torch.zeros(m, n, device=device, dtype=torch.float32) for (m, n) in wl.layers] for _ in range(W)]
        self.Q = [self.src.initial_q(l).to(device) for l in range(L)]
        self.P = [torch.empty(m, wl.rank, device=device) for (m, n) in wl.layers]
        self.Rc = [torch.empty(m, n, device=device) for (m, n) in wl.layers] if recon else None
        self.step_no = 0

    def set_state(self, E: Sequence[Sequence[torch.Tensor]], Q: Sequence[torch.Tensor]):
        for w in range(self.wl.workers):
            for l in range(len(self.wl.layers)):
                self.E[w][l].copy_(E[w][l])
        for l in range(len(self.wl.layers)):
            self.Q[l].copy_(Q[l])

    def fill_grads_host(self, step: int) -> List[List[torch.Tensor]]:
        host = [[self.src.layer_grad(step, w, l) for l in range(len(self.wl.layers))]
                for w in range(self.wl.workers)]
        for w in range(self.wl.workers):
            for l in range(len(self.wl.layers)):
                self.G[w][l].copy_(host[w][l])
        return host

    def run_step(self):
        self.lib.step(self.G, self.E, self.Q, self.P, self.Rc)
        self.step_no += 1

    def errors(self, w: int, l: int) -> torch.Tensor:
        return self.E[w][l]


class OracleRun:
    """Float64 oracle state for a subset of layers."""

    def __init__(self, layers_idx: Sequence[int], E0, Q0, iters: int = 1):
        self.idx = list(layers_idx)
        self.E = {l: [np.asarray(e, dtype=np.float64) for e in E0[l]] for l in self.idx}
        self.Q = {l: np.asarray(Q0[l], dtype=np.float64) for l in self.idx}
        self.iters = iters
        self.last: Dict[int, dict] = {}

    def step(self, G: Dict[int, List[np.ndarray]], Q_override: Optional[Dict[int, np.ndarray]] = None):
        for l in self.idx:
            if Q_override is not None:
                self.Q[l] = np.asarray(Q_override[l], dtype=np.float64)
            o = ora.step(G[l], self.E[l], self.Q[l], iters=self.iters)
            self.E[l] = o["E_new"]
            self.Q[l] = o["Q_bar"]
            self.last[l] = o


def compare_layer(run: LibRun, o: dict, l: int, tol: float, G_list=None, check_recon=True) -> Dict[str, float]:
    """Relative Frobenius errors of P_hat, Q_bar, G_hat and E'_w (E' relative
    to ||M_w||_F) of one layer against the oracle's result dict."""
    errs = {}
    errs["P_hat"] = rel_fro(to64(run.P[l]), o["P_hat"])
    errs["Q_bar"] = rel_fro(to64(run.Q[l]), o["Q_bar"])
    if check_recon and run.Rc is not None:
        errs["G_hat"] = rel_fro(to64(run.Rc[l]), o["G_hat"])
    worst = 0.0
    for w in range(run.wl.workers):
        e = rel_fro(to64(run.E[w][l]), o["E_new"][w], denom=np.linalg.norm(o["M"][w]))
        worst = max(worst, e)
    errs["E_new"] = worst
    return errs


def sign_aligned(got: np.ndarray, want: np.ndarray) -> np.ndarray:
    """got with every column's sign flipped to agree with want's column
    (singular vectors are unique only up to sign)."""
    s = np.sign(np.einsum("ij,ij->j", got, want))
    s[s == 0] = 1.0
    return got * s[None, :]


def assert_close(errs: Dict[str, float], tol: float, what: str = ""):
    bad = {k: v for k, v in errs.items() if not (v <= tol)}
    assert not bad, f"{what}: errors above {tol}: {bad} (all: {errs})"


def small_workload(layers, rank, workers, dtype="f32", noise=("rel", 0.1), name="small") -> Workload:
    return Workload(name=name, layers=tuple(tuple(x) for x in layers), rank=rank, workers=workers, steps=3,
                    grad_dtype=dtype, noise=noise)


def run_free(wl: Workload, steps: int, lazy=False, sum_first=False, seed=1234, random_state: float = 0.0,
             layers_idx: Optional[Sequence[int]] = None, iters: int = 1, warm_start: bool = True):
    """Run `steps` free-running steps on small inputs generated on the host.
    Returns (run, oracle, per-step max errors over the checked layers).  In
    lazy-error mode the error buffers hold M_w between steps; E' is
    compared only after the last step, once materialised."""
    run = LibRun(wl, seed=seed, lazy=lazy, sum_first=sum_first, iters=iters, warm_start=warm_start)
    L = len(wl.layers)
    idx = list(range(L)) if layers_idx is None else list(layers_idx)
    # initial state from synth on the host; the device gets a copy
    Q0 = [run.src.initial_q(l) for l in range(L)]
    if random_state:
        E0 = [[run.src.random_state(l, w, random_state) for l in range(L)] for w in range(wl.workers)]
    else:
        E0 = [[torch.zeros(m, n) for (m, n) in wl.layers] for _ in range(wl.workers)]
    run.set_state(E0, Q0)
    E0_np = {l: [E0[w][l].to(torch.float64).numpy() for w in range(wl.workers)] for l in idx}
    Q0_np = {l: Q0[l].to(torch.float64).numpy() for l in idx}
    orc = OracleRun(idx, E0_np, Q0_np, iters=iters)
    history = []
    for t in range(steps):
        host = run.fill_grads_host(t)
        run.run_step()
        last = t == steps - 1
        if lazy and last:
            run.lib.materialize_errors(run.E)
        torch.cuda.synchronize()
        qo = None
        if not warm_start:
            # the step's fresh Q: the oracle's own Philox draw (draw = step number)
            from oracle import philox64
            qo = {l: philox64.initial_q(seed, l, wl.layers[l][1], wl.rank, draw=t + 1) for l in idx}
        orc.step({l: [host[w][l].to(torch.float64).numpy() for w in range(wl.workers)] for l in idx}, qo)
        step_errs = {}
        for l in idx:
            e = compare_layer(run, orc.last[l], l, TOL[wl.grad_dtype])
            if lazy and not last:
                e.pop("E_new")
            for k, v in e.items():
                step_errs[k] = max(step_errs.get(k, 0.0), v)
        history.append(step_errs)
    run.lib.status()
    return run, orc, history


class PackedRun:
    """Full-size workload on the device: one packed buffer per worker for G
    and for E, gradients generated on the device by synth."""

    def __init__(self, wl: Workload, seed: int = 1234, lazy: bool = False, recon_layers=(), device="cuda"):
        from rank_gradient_compression_02_b200 import PowerSGD
        from synth import pack_offsets
        self.wl = wl
        self.src = GradientSource(wl, seed)
        W, L = wl.workers, len(wl.layers)
        gdt = torch.bfloat16 if wl.grad_dtype == "bf16" else torch.float32
        offs = pack_offsets(wl.layers, 64)
        self.Gf = [torch.empty(offs[-1], dtype=gdt, device=device) for _ in range(W)]
        self.Ef = [torch.zeros(offs[-1], dtype=torch.float32, device=device) for _ in range(W)]
        self.G = [[self.Gf[w][offs[l]:offs[l] + m * n].view(m, n) for l, (m, n) in enumerate(wl.layers)]
                  for w in range(W)]
        self.E = [[self.Ef[w][offs[l]:offs[l] + m * n].view(m, n) for l, (m, n) in enumerate(wl.layers)]
                  for w in range(W)]
        self.Q0 = [self.src.initial_q(l) for l in range(L)]
        self.Q = [q.to(device) for q in self.Q0]
        self.P = [torch.empty(m, wl.rank, device=device) for (m, _) in wl.layers]
        self.Rc = [torch.empty(m, n, device=device) if l in recon_layers else None
                   for l, (m, n) in enumerate(wl.layers)]
        self.lib = PowerSGD(wl.layers, wl.rank, W, seed=seed, grad_dtype=wl.grad_dtype, lazy_errors=lazy)
        self.lazy = lazy

    def fill(self, step: int):
        self.src.fill(step, self.G)

    def step(self):
        self.lib.step(self.G, self.E, self.Q, self.P, self.Rc)

    def host_grads(self, l: int) -> List[np.ndarray]:
        return [to64(self.G[w][l]) for w in range(self.wl.workers)]


def run_sampled(wl: Workload, steps: int, sample_layers: Sequence[int], lazy: bool = False):
    """Full workload on the device; the oracle follows the sampled layers
    (layers are independent, so their trajectories are exact references).
    Returns per-step max errors over the sampled layers."""
    run = PackedRun(wl, lazy=lazy, recon_layers=set(sample_layers))
    idx = list(sample_layers)
    orc = OracleRun(idx, {l: [np.zeros(wl.layers[l]) for _ in range(wl.workers)] for l in idx},
                    {l: run.Q0[l].double().numpy() for l in idx})
    hist = []
    for t in range(steps):
        run.fill(t)
        torch.cuda.synchronize()
        G = {l: run.host_grads(l) for l in idx}
        run.step()
        if lazy and t == steps - 1:
            run.lib.materialize_errors(run.E)
        torch.cuda.synchronize()
        orc.step(G)
        errs = {}
        for l in idx:
            o = orc.last[l]
            e = {"P_hat": rel_fro(to64(run.P[l]), o["P_hat"]), "Q_bar": rel_fro(to64(run.Q[l]), o["Q_bar"]),
                 "G_hat": rel_fro(to64(run.Rc[l]), o["G_hat"])}
            if not lazy or t == steps - 1:
                e["E_new"] = max(rel_fro(to64(run.E[w][l]), o["E_new"][w], denom=np.linalg.norm(o["M"][w]))
                                 for w in range(wl.workers))
            for k, v in e.items():
                errs[k] = max(errs.get(k, 0.0), v)
        hist.append(errs)
        del G
    run.lib.status()
    return run, hist


def property_errors(run: "PackedRun", l: int, G_host: List[np.ndarray], E_prev: List[np.ndarray]):
    """Properties that hold at any size, from the step's own inputs and
    outputs: P_hat^T P_hat = I, P_hat Q_bar^T + E'_w = M_w, Q_bar = mean(M)^T P_hat."""
    P = to64(run.P[l])
    Qb = to64(run.Q[l])
    W = run.wl.workers
    M = [G_host[w] + E_prev[w] for w in range(W)]
    r = P.shape[1]
    orth = float(np.abs(P.T @ P - np.eye(r)).max())
    rec = P @ Qb.T
    ident = max(rel_fro(rec + to64(run.E[w][l]), M[w]) for w in range(W))
    Mbar = sum(M) / W
    qrel = rel_fro(Qb, Mbar.T @ P)
    return {"orth": orth, "identity": ident, "q_proj": qrel}

"""The allocation-free entry point (psgd_step_static) through the C ABI:
against the context-based psgd_step and against the float64 oracle.

psgd_step_static is for callers that cannot allocate device memory: its
scratch lives in a static device array inside the library.  This file is
collected last so that a failure here comes after every other test has run;
it passes both alone in a fresh process and after the rest of the suite
(the static array keeps the previous call's contents, and each call clears
what must start at zero)."""
import ctypes

import numpy as np
import pytest
import torch

import oracle.powersgd64 as ora
from rank_gradient_compression_02_b200 import PowerSGD, PsgdError, _lib
from synth import GradientSource, Workload

from . import _harness as H

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("m,n,rank,workers,dtype", [
    (300, 650, 4, 3, "f32"),
    (129, 1000, 2, 2, "f32"),
    (96, 130, 8, 4, "bf16"),
    (33, 37, 1, 1, "f32"),
    (129, 1000, 32, 3, "f32"),    # the tensor-core passes, 16-byte lanes
    (300, 650, 16, 2, "f32"),     # the tensor-core passes, 8-byte lanes
])
def test_static_step_matches_context_step_and_oracle(m, n, rank, workers, dtype):
    wl = Workload(name="noalloc", layers=((m, n),), rank=rank, workers=workers, steps=2, grad_dtype=dtype)
    src = GradientSource(wl, seed=11)
    gdt = torch.bfloat16 if dtype == "bf16" else torch.float32
    ctx = PowerSGD(wl.layers, rank, workers, grad_dtype=dtype)
    q0 = src.initial_q(0)
    # two independent device states and a float64 oracle state, the same inputs
    G = [torch.empty(m, n, device="cuda", dtype=gdt) for _ in range(workers)]
    E_ctx = [torch.zeros(m, n, device="cuda") for _ in range(workers)]
    E_st = [torch.zeros(m, n, device="cuda") for _ in range(workers)]
    q_ctx, q_st = q0.cuda(), q0.cuda()
    P_ctx = torch.empty(m, rank, device="cuda")
    P_st = torch.empty(m, rank, device="cuda")
    R_ctx = torch.empty(m, n, device="cuda")
    R_st = torch.empty(m, n, device="cuda")
    E_ora = [np.zeros((m, n)) for _ in range(workers)]
    Q_ora = q0.double().numpy()
    for t in range(2):          # two calls in a row, state carried in place
        host = [src.layer_grad(t, w, 0) for w in range(workers)]
        for w in range(workers):
            G[w].copy_(host[w])
        ctx.step([[g] for g in G], [[e] for e in E_ctx], [q_ctx], [P_ctx], [R_ctx])
        _lib.step_static(m, n, rank, G, E_st, q_st, P_st, R_st, grad_dtype=dtype)
        _lib.step_static_status()
        torch.cuda.synchronize()
        # the same kernels in the same order on the same inputs: bit for bit
        # the context step's results
        assert torch.equal(P_st, P_ctx), f"call {t}: P_hat"
        assert torch.equal(q_st, q_ctx), f"call {t}: Q_bar"
        assert torch.equal(R_st, R_ctx), f"call {t}: G_hat"
        for w in range(workers):
            assert torch.equal(E_st[w], E_ctx[w]), f"call {t}: E'_{w}"
        # and against the float64 oracle, free-running from the same state
        o = ora.step([g.double().numpy() for g in host], E_ora, Q_ora)
        E_ora, Q_ora = o["E_new"], o["Q_bar"]
        errs = {"P_hat": H.rel_fro(H.to64(P_st), o["P_hat"]), "Q_bar": H.rel_fro(H.to64(q_st), o["Q_bar"]),
                "G_hat": H.rel_fro(H.to64(R_st), o["G_hat"]),
                "E_new": max(H.rel_fro(H.to64(E_st[w]), o["E_new"][w], denom=np.linalg.norm(o["M"][w]))
                             for w in range(workers))}
        H.assert_close(errs, H.TOL[dtype], f"call {t} against the oracle")
    ctx.status()


def test_static_step_rejects_layers_beyond_its_scratch():
    lib = _lib.load()
    W = 2
    ptrs = (ctypes.c_void_p * W)(*([16] * W))   # never dereferenced: rejected first
    rc = lib.psgd_step_static(8192, 8192, 32, W, 0, ptrs, ptrs, 16, None, None, None)
    assert rc == _lib.PSGD_ERR_ARG
    msg = lib.psgd_last_error(None).decode()
    assert "static scratch" in msg


def test_static_step_argument_checks():
    x = torch.zeros(64, 48, device="cuda")
    q = torch.zeros(48, 2, device="cuda")
    with pytest.raises(PsgdError) as ei:
        _lib.step_static(64, 48, 49, [x], [x], q)     # rank > min(m, n)
    assert ei.value.code == _lib.PSGD_ERR_ARG
    flat = torch.zeros(64 * 48 + 1, device="cuda")
    odd = flat[1:]
    with pytest.raises(PsgdError) as ei:
        _lib.step_static(64, 48, 2, [odd], [x], q)    # 4-byte offset
    assert ei.value.code == _lib.PSGD_ERR_ALIGN

"""The distributed step (psgd_dist_p / psgd_dist_q / psgd_dist_finish) on one
GPU: R ranks are emulated as R library contexts with their own workers, and
the two all-reduces are fixed-order float64 sums of the ranks' buffers done
between the calls (no kernel waits for another).  The result must match the
float64 oracle run over all R x W_local workers."""
import numpy as np
import pytest
import torch

import oracle.powersgd64 as ora
from rank_gradient_compression_02_b200 import PowerSGD, PsgdError
from synth import GradientSource

from . import _harness as H

pytestmark = pytest.mark.gpu

MIXED = [(300, 650), (64, 576), (40, 130), (256, 128), (33, 37), (129, 1000)]


@pytest.mark.parametrize("ranks,wlocal,rank,lazy", [(2, 2, 4, False), (4, 1, 2, False), (3, 2, 8, True),
                                                    (2, 3, 32, False), (1, 3, 4, False)])
def test_distributed_step_matches_oracle(ranks, wlocal, rank, lazy):
    W = ranks * wlocal
    layers = [s for s in MIXED if min(s) >= rank]
    wl = H.small_workload(layers, rank, W)
    L = len(layers)
    src = GradientSource(wl, 1234)
    ctxs = [PowerSGD(layers, rank, wlocal, lazy_errors=lazy) for _ in range(ranks)]
    for c in ctxs:
        c.set_global_workers(W)
    pe, qe = ctxs[0].dist_sizes()
    Q0 = [src.initial_q(l) for l in range(L)]
    G = [[[torch.empty(m, n, device="cuda") for (m, n) in layers] for _ in range(wlocal)] for _ in range(ranks)]
    E = [[[torch.zeros(m, n, device="cuda") for (m, n) in layers] for _ in range(wlocal)] for _ in range(ranks)]
    Q = [[q.cuda() for q in Q0] for _ in range(ranks)]
    P = [[torch.empty(m, rank, device="cuda") for (m, _) in layers] for _ in range(ranks)]
    Rc = [[torch.empty(m, n, device="cuda") for (m, n) in layers] for _ in range(ranks)]
    psend = [torch.empty(pe, dtype=torch.float64, device="cuda") for _ in range(ranks)]
    qsend = [torch.empty(qe, dtype=torch.float64, device="cuda") for _ in range(ranks)]
    orc = H.OracleRun(range(L), {l: [np.zeros(layers[l]) for _ in range(W)] for l in range(L)},
                      {l: Q0[l].double().numpy() for l in range(L)})
    steps = 3
    for t in range(steps):
        host = [[src.layer_grad(t, w, l) for l in range(L)] for w in range(W)]
        for rr in range(ranks):
            for wi in range(wlocal):
                for l in range(L):
                    G[rr][wi][l].copy_(host[rr * wlocal + wi][l])
        for rr in range(ranks):
            ctxs[rr].dist_p(G[rr], E[rr], Q[rr], psend[rr], P[rr], Rc[rr])
        psum = psend[0].clone()
        for rr in range(1, ranks):
            psum += psend[rr]
        for rr in range(ranks):
            ctxs[rr].dist_q(psum, qsend[rr])
        qsum = qsend[0].clone()
        for rr in range(1, ranks):
            qsum += qsend[rr]
        for rr in range(ranks):
            ctxs[rr].dist_finish(qsum)
        last = t == steps - 1
        if lazy and last:
            for rr in range(ranks):
                ctxs[rr].materialize_errors(E[rr])
        torch.cuda.synchronize()
        orc.step({l: [host[w][l].double().numpy() for w in range(W)] for l in range(L)})
        for l in range(L):
            o = orc.last[l]
            for rr in range(ranks):
                errs = {"P_hat": H.rel_fro(H.to64(P[rr][l]), o["P_hat"]),
                        "Q_bar": H.rel_fro(H.to64(Q[rr][l]), o["Q_bar"]),
                        "G_hat": H.rel_fro(H.to64(Rc[rr][l]), o["G_hat"])}
                if not lazy or last:
                    errs["E_new"] = max(H.rel_fro(H.to64(E[rr][wi][l]), o["E_new"][rr * wlocal + wi],
                                                  denom=np.linalg.norm(o["M"][rr * wlocal + wi]))
                                        for wi in range(wlocal))
                H.assert_close(errs, H.TOL["f32"], f"step {t} layer {l} rank {rr}")
    for c in ctxs:
        c.status()


def test_distributed_step_order_is_enforced():
    lib = PowerSGD([(64, 48)], 2, 1)
    pe, qe = lib.dist_sizes()
    buf = torch.zeros(max(pe, qe), dtype=torch.float64, device="cuda")
    with pytest.raises(PsgdError) as ei:
        lib.dist_q(buf, buf)
    assert ei.value.code == 5
    with pytest.raises(PsgdError) as ei:
        lib.dist_finish(buf)
    assert ei.value.code == 5
    lib2 = PowerSGD([(64, 48)], 2, 1, power_iters=2)
    G = [[torch.zeros(64, 48, device="cuda")]]
    q = [torch.zeros(48, 2, device="cuda")]
    with pytest.raises(PsgdError) as ei:
        lib2.dist_p(G, G, q, buf)
    assert ei.value.code == 5


def test_global_vector_mean():
    # vectors all-reduced over 2 emulated ranks, divided by the global count
    W_local, ranks = 3, 2
    lib = PowerSGD([(8, 8)], 1, W_local)
    lib.set_global_workers(W_local * ranks)
    g = torch.Generator().manual_seed(4)
    v = [[torch.randn(100, generator=g) for _ in range(W_local)] for _ in range(ranks)]
    summed = [[(v[0][w] + v[1][w]).cuda()] for w in range(W_local)]
    out = [torch.empty(100, device="cuda")]
    lib.vec_mean(summed, out)
    lib.status()
    want = sum(v[r][w] for r in range(ranks) for w in range(W_local)) / (W_local * ranks)
    assert torch.allclose(out[0].cpu(), want, rtol=1e-6, atol=1e-6)

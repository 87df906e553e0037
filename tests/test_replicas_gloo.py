"""Host logic of the multi-GPU bench path on CPU with gloo (world sizes 2
and 3): max-over-ranks timing, whole-job throughput, and the distributed
step's orchestration over two steps (the two all-reduces of the P and Q
partials, the global worker count, error memory and warm start carried,
momentum, the 1-D means) driven through a float64 stand-in for the library
built from the oracle's functions."""
import os
import socket
import types

import numpy as np
import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    p = s.getsockname()[1]
    s.close()
    return p


def _init(rank, world, port):
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world)


def _worker_timing(rank, world, port, q):
    _init(rank, world, port)
    import bench
    ms = 10.0 + 5.0 * rank        # rank 1 is the slow one
    got = bench.max_over_ranks(ms, world, torch.device("cpu"))
    val = bench.job_value(1000, world, got)
    q.put((rank, got, val))
    dist.barrier()
    dist.destroy_process_group()


def _spawn(target, world, *args):
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=target, args=(r, world, port, q) + args) for r in range(world)]
    for p in procs:
        p.start()
    res = [q.get(timeout=180) for _ in procs]
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    return sorted(res, key=lambda x: x[0])


def test_max_over_ranks_and_job_value():
    for rank, got, val in _spawn(_worker_timing, 2):
        assert got == 15.0
        assert val == pytest.approx(1000 * 2 / 15e-3)


def test_single_rank_is_identity():
    import bench
    assert bench.max_over_ranks(3.0, 1, None) == 3.0
    assert bench.job_value(10, 1, 1.0) == pytest.approx(1e4)


class FakeDistLib:
    """float64 CPU stand-in with the library's distributed-call semantics
    (oracle functions for the arithmetic)."""

    def __init__(self, layers, rank, w_local):
        import oracle.powersgd64 as ora
        self.ora = ora
        self.layers, self.r, self.W = layers, rank, w_local
        self.Wg = w_local
        self.Phat = [None] * len(layers)
        self.Qbar = [None] * len(layers)

    def set_global_workers(self, n):
        self.Wg = n

    def dist_sizes(self):
        return sum(m for m, _ in self.layers) * self.r, sum(n for _, n in self.layers) * self.r

    def dist_p(self, G, E, Q, p_send, P, recon):
        self.E, self.Qv, self.P = E, Q, P
        off = 0
        for l, (m, n) in enumerate(self.layers):
            acc = np.zeros((m, self.r))
            for w in range(self.W):
                E[w][l][...] = G[w][l] + E[w][l]          # M over E
                acc += E[w][l].numpy() @ Q[l].numpy()
            p_send[off:off + m * self.r] = torch.from_numpy(acc.ravel())
            off += m * self.r

    def dist_q(self, p_sum, q_send):
        po = qo = 0
        for l, (m, n) in enumerate(self.layers):
            pbar = p_sum[po:po + m * self.r].numpy().reshape(m, self.r) / self.Wg
            self.Phat[l] = self.ora.gram_schmidt(pbar)
            self.P[l][...] = torch.from_numpy(self.Phat[l])
            acc = sum(self.E[w][l].numpy().T @ self.Phat[l] for w in range(self.W))
            q_send[qo:qo + n * self.r] = torch.from_numpy(acc.ravel())
            po += m * self.r
            qo += n * self.r

    def dist_finish(self, q_sum):
        qo = 0
        for l, (m, n) in enumerate(self.layers):
            self.Qbar[l] = q_sum[qo:qo + n * self.r].numpy().reshape(n, self.r) / self.Wg
            self.Qv[l][...] = torch.from_numpy(self.Qbar[l])
            for w in range(self.W):
                self.E[w][l][...] = torch.from_numpy(self.E[w][l].numpy() - self.Phat[l] @ self.Qbar[l].T)
            qo += n * self.r

    def vec_mean(self, vecs, out, x, mom, lr=0.0, beta=0.0):
        for k in range(len(out)):
            g = sum(vecs[w][k] for w in range(self.W)) / self.Wg
            out[k][...] = g
            mom[k][...] = beta * mom[k] + g
            x[k][...] = x[k] - lr * mom[k]

    def momentum_step(self, params, mom, lr, beta):
        for l in range(len(self.layers)):
            ghat = torch.from_numpy(self.Phat[l] @ self.Qbar[l].T)
            mom[l][...] = beta * mom[l] + ghat
            params[l][...] = params[l] - lr * mom[l]


LAYERS = [(12, 9), (7, 11)]
R, WL = 2, 2


STEPS = 2


def _grads(rank_id, w, l, t=0):
    g = torch.Generator().manual_seed(100000 * t + 1000 * rank_id + 10 * w + l)
    m, n = LAYERS[l]
    return torch.randn(m, n, generator=g, dtype=torch.float64)


def _vecs(rank_id, w, t=0):
    g = torch.Generator().manual_seed(777 + 100000 * t + 10 * rank_id + w)
    return [torch.randn(5, generator=g, dtype=torch.float64), torch.randn(3, generator=g, dtype=torch.float64)]


def _worker_dist(rank, world, port, q):
    _init(rank, world, port)
    import bench
    lib = FakeDistLib(LAYERS, R, WL)
    lib.set_global_workers(WL * world)
    B = types.SimpleNamespace()
    B.G = [[_grads(rank, w, l) for l in range(len(LAYERS))] for w in range(WL)]
    B.E = [[torch.zeros(m, n, dtype=torch.float64) for (m, n) in LAYERS] for _ in range(WL)]
    g = torch.Generator().manual_seed(5)
    B.Q = [torch.randn(n, R, generator=g, dtype=torch.float64) for (_, n) in LAYERS]
    B.P = [torch.zeros(m, R, dtype=torch.float64) for (m, _) in LAYERS]
    B.vecs = [_vecs(rank, w) for w in range(WL)]
    B.vout = [torch.zeros(5, dtype=torch.float64), torch.zeros(3, dtype=torch.float64)]
    B.vx = [torch.zeros(5, dtype=torch.float64), torch.zeros(3, dtype=torch.float64)]
    B.vmom = [torch.zeros(5, dtype=torch.float64), torch.zeros(3, dtype=torch.float64)]
    B.params = [torch.zeros(m, n, dtype=torch.float64) for (m, n) in LAYERS]
    B.mom = [torch.zeros(m, n, dtype=torch.float64) for (m, n) in LAYERS]
    wl = types.SimpleNamespace(vectors=(5, 3), momentum=(0.9, 0.1))
    db = bench.DistBuffers(lib, B, wl, torch.device("cpu"))
    db.p = db.p.double()
    db.q = db.q.double()
    for t in range(STEPS):
        if t:
            for w in range(WL):
                for l in range(len(LAYERS)):
                    B.G[w][l].copy_(_grads(rank, w, l, t))
                for k, v in enumerate(_vecs(rank, w, t)):
                    B.vecs[w][k].copy_(v)
            db.pack(B.vecs)   # the flat all-reduce buffer holds the step's 1-D gradients
        bench.dist_step(lib, B, wl, db, lambda x: dist.all_reduce(x, op=dist.ReduceOp.SUM))
    q.put((rank, [p.numpy().copy() for p in B.P], [x.numpy().copy() for x in B.Q],
           [[e.numpy().copy() for e in Ew] for Ew in B.E], [v.numpy().copy() for v in B.vout],
           [x.numpy().copy() for x in B.params]))
    dist.barrier()
    dist.destroy_process_group()


@pytest.mark.parametrize("world", [2, 3])
def test_distributed_step_orchestration_matches_oracle(world):
    import oracle.powersgd64 as ora
    res = _spawn(_worker_dist, world)
    g = torch.Generator().manual_seed(5)
    Q = [torch.randn(n, R, generator=g, dtype=torch.float64).numpy() for (_, n) in LAYERS]
    E = [[np.zeros(LAYERS[l]) for _ in range(world * WL)] for l in range(len(LAYERS))]
    mom = [np.zeros(s) for s in LAYERS]
    x = [np.zeros(s) for s in LAYERS]
    for t in range(STEPS):
        outs = []
        for l in range(len(LAYERS)):
            G = [_grads(r, w, l, t).numpy() for r in range(world) for w in range(WL)]
            o = ora.step(G, E[l], Q[l])
            E[l], Q[l] = o["E_new"], o["Q_bar"]
            x[l], mom[l] = ora.momentum_update(x[l], mom[l], o["G_hat"], lr=0.1, beta=0.9)
            outs.append(o)
    for l, o in enumerate(outs):
        for r, P, Qr, Er, vout, params in res:
            np.testing.assert_allclose(P[l], o["P_hat"], atol=1e-12)
            np.testing.assert_allclose(Qr[l], o["Q_bar"], atol=1e-12)
            for w in range(WL):
                np.testing.assert_allclose(Er[w][l], o["E_new"][r * WL + w], atol=1e-12)
            np.testing.assert_allclose(params[l], x[l], atol=1e-12)
    vec_want = [sum(_vecs(r, w, STEPS - 1)[k] for r in range(world) for w in range(WL)).numpy() / (world * WL)
                for k in range(2)]
    for r, P, Qr, Er, vout, params in res:
        for k in range(2):
            np.testing.assert_allclose(vout[k], vec_want[k], atol=1e-12)

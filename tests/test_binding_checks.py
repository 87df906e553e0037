"""The binding's host-side checks (CPU, stub library): every buffer is
checked for side (device or host), dtype, contiguity and size, and every
list for its length, before an address crosses the ABI; the addresses
passed are the tensors' own, worker-major; checks run again only when an
address of the call changes.  "Device" tensors are CPU tensors marked as such."""
import ctypes

import pytest
import torch

from rank_gradient_compression_02_b200 import _lib
from rank_gradient_compression_02_b200._lib import PowerSGD, PsgdError

LAYERS = [(6, 5), (4, 8)]
R, W = 2, 3


class _StubLib:
    """Records each call's pointer arrays as lists; returns PSGD_OK."""

    def __init__(self):
        self.calls = []

    def __getattr__(self, name):
        if name == "psgd_last_error":
            return lambda h: b"stub"

        def fn(*args):
            rec = []
            for a in args:
                if isinstance(a, ctypes.Array):
                    rec.append(list(a))
                else:
                    rec.append(a)
            self.calls.append((name, rec))
            return 0
        return fn


def dev(t):
    t._dev = True
    return t


@pytest.fixture
def ctx(monkeypatch):
    monkeypatch.setattr(_lib, "_on_device", lambda t: getattr(t, "_dev", False))
    p = object.__new__(PowerSGD)
    p.lib = _StubLib()
    p._h = 1
    p.layers = list(LAYERS)
    p.rank, p.workers, p.grad_dtype = R, W, "f32"
    return p


def bufs(dtype=torch.float32):
    G = [[dev(torch.zeros(m, n, dtype=dtype)) for (m, n) in LAYERS] for _ in range(W)]
    E = [[dev(torch.zeros(m, n)) for (m, n) in LAYERS] for _ in range(W)]
    Q = [dev(torch.zeros(n, R)) for (_, n) in LAYERS]
    P = [dev(torch.zeros(m, R)) for (m, _) in LAYERS]
    Rc = [dev(torch.zeros(m, n)) for (m, n) in LAYERS]
    return G, E, Q, P, Rc


def _addrs(ts):
    return [None if t is None else t.data_ptr() for t in ts]


def test_step_passes_worker_major_addresses(ctx):
    G, E, Q, P, Rc = bufs()
    ctx.step(G, E, Q, P, Rc, stream=0)
    name, args = ctx.lib.calls[-1]
    assert name == "psgd_step"
    assert args[1] == _addrs([G[w][l] for w in range(W) for l in range(len(LAYERS))])
    assert args[2] == _addrs([E[w][l] for w in range(W) for l in range(len(LAYERS))])
    assert args[3] == _addrs(Q) and args[4] == _addrs(P) and args[5] == _addrs(Rc)
    ctx.step(G, E, Q, None, [None, Rc[1]], stream=0)     # absent list, absent entry
    _, args = ctx.lib.calls[-1]
    assert args[4] is None and args[5] == [None, Rc[1].data_ptr()]


def test_views_of_one_flat_buffer_and_bf16_pass(ctx):
    ctx.grad_dtype = "bf16"
    offs = [0, 32]
    flat_g = [dev(torch.zeros(64, dtype=torch.bfloat16)) for _ in range(W)]
    G = [[dev(flat_g[w][o:o + m * n].view(m, n)) for o, (m, n) in zip(offs, LAYERS)] for w in range(W)]
    _, E, Q, P, _ = bufs()
    ctx.step(G, E, Q, P, None, stream=0)
    assert ctx.lib.calls[-1][0] == "psgd_step"


def test_raw_addresses_and_null_reach_the_library(ctx):
    # the library's own null and alignment checks see ints unchanged
    G, E, Q, P, _ = bufs()
    E_bad = [[0, E[0][1]]] + E[1:]
    ctx.step(G, E_bad, Q, P, None, stream=0)
    assert ctx.lib.calls[-1][1][2][0] is None


@pytest.mark.parametrize("mutate", [
    lambda G, E, Q, P: G.pop(),                                        # W - 1 workers
    lambda G, E, Q, P: E[1].pop(),                                     # a worker short of a layer
    lambda G, E, Q, P: Q.append(Q[0]),                                 # L + 1 Q entries
    lambda G, E, Q, P: G[0].__setitem__(0, dev(torch.zeros(6, 4))),    # wrong size
    lambda G, E, Q, P: E[2].__setitem__(1, dev(torch.zeros(4, 8, dtype=torch.float64))),  # wrong dtype
    lambda G, E, Q, P: G[1].__setitem__(1, dev(torch.zeros(8, 4)).t()),                     # not contiguous
    lambda G, E, Q, P: Q.__setitem__(1, torch.zeros(8, R)),            # host tensor for a device buffer
    lambda G, E, Q, P: P.__setitem__(0, dev(torch.zeros(6, R + 1))),   # P_hat of another rank
    lambda G, E, Q, P: G[0].__setitem__(1, "not a buffer"),
])
def test_bad_buffers_are_argument_errors(ctx, mutate):
    G, E, Q, P, _ = bufs()
    mutate(G, E, Q, P)
    with pytest.raises(PsgdError) as ei:
        ctx.step(G, E, Q, P, None, stream=0)
    assert ei.value.code == _lib.PSGD_ERR_ARG
    assert not ctx.lib.calls


def test_checks_rerun_only_when_buffers_change(ctx, monkeypatch):
    G, E, Q, P, _ = bufs()
    count = [0]
    real = _lib._check_buf

    def counting(*a, **k):
        count[0] += 1
        return real(*a, **k)
    monkeypatch.setattr(_lib, "_check_buf", counting)
    ctx.step(G, E, Q, P, None, stream=0)
    first = count[0]
    assert first == 2 * W * len(LAYERS) + 2 * len(LAYERS)
    ctx.step(G, E, Q, P, None, stream=0)
    assert count[0] == first
    G[2][1] = dev(torch.zeros(4, 8))              # a new tensor: checked again
    ctx.step(G, E, Q, P, None, stream=0)
    assert count[0] == 2 * first
    G[2][1] = dev(torch.zeros(4, 9))              # and a bad one is caught
    with pytest.raises(PsgdError):
        ctx.step(G, E, Q, P, None, stream=0)


def test_host_side_calls(ctx):
    G, E, Q, P, _ = bufs()
    host = [[torch.zeros(m, n) for (m, n) in LAYERS] for _ in range(W)]
    ph = [torch.zeros(m, R) for (m, _) in LAYERS]
    qh = [torch.zeros(n, R) for (_, n) in LAYERS]
    ctx.step_host(host, E, Q, ph, qh, stream=0)
    assert ctx.lib.calls[-1][0] == "psgd_step_host"
    with pytest.raises(PsgdError):
        ctx.step_host(G, E, Q, ph, qh, stream=0)          # device tensors where host ones belong
    flat = [torch.zeros(70) for _ in range(W)]
    ctx.step_host_flat(flat, [0, 36], E, Q, ph, qh, stream=0)
    name, args = ctx.lib.calls[-1]
    assert name == "psgd_step_host_flat" and list(args[2]) == [0, 36] and args[1] == _addrs(flat)
    with pytest.raises(PsgdError):
        ctx.step_host_flat(flat, [0, 40], E, Q, stream=0)  # layer 1 runs past the buffer
    with pytest.raises(PsgdError):
        ctx.step_host_flat(flat, [0], E, Q, stream=0)      # one offset per layer


def test_vectors_momentum_init_and_materialize(ctx):
    G, E, Q, P, Rc = bufs()
    lens = [5, 0, 17]
    vecs = [[dev(torch.zeros(k)) for k in lens] for _ in range(W)]
    out = [dev(torch.zeros(k)) for k in lens]
    x = [dev(torch.zeros(k)) for k in lens]
    mo = [dev(torch.zeros(k)) for k in lens]
    ctx.vec_mean(vecs, out, x, mo, lr=0.1, beta=0.9, stream=0)
    name, args = ctx.lib.calls[-1]
    assert name == "psgd_vec_mean" and list(args[3]) == lens and args[4] == 3
    with pytest.raises(PsgdError):
        ctx.vec_mean([[dev(torch.zeros(k + 1)) for k in lens]] * W, out, stream=0)
    with pytest.raises(PsgdError):
        ctx.vec_mean(vecs, out, x[:2], mo, stream=0)
    ctx.momentum_step(Rc, [dev(torch.zeros(m, n)) for (m, n) in LAYERS], 0.1, 0.9, stream=0)
    with pytest.raises(PsgdError):
        ctx.momentum_step(Rc, P, 0.1, 0.9, stream=0)
    ctx.init_q(Q, stream=0)
    ctx.materialize_errors(E, stream=0)
    with pytest.raises(PsgdError):
        ctx.materialize_errors(G[:2], stream=0)


def test_empty_layer_list(ctx):
    ctx.layers = []
    ctx.step([[], [], []], [[], [], []], [], [], None, stream=0)
    ctx.momentum_step([], [], 0.1, 0.9, stream=0)
    ctx.vec_mean([[], [], []], [], stream=0)
    assert [c[0] for c in ctx.lib.calls] == ["psgd_step", "psgd_momentum_step", "psgd_vec_mean"]


def test_distributed_buffers(ctx):
    G, E, Q, P, Rc = bufs()
    p = dev(torch.zeros(40, dtype=torch.float64))
    ctx.dist_p(G, E, Q, p, P, Rc, stream=0)
    ctx.dist_q(p, p, stream=0)
    ctx.dist_finish(p, stream=0)
    assert [c[0] for c in ctx.lib.calls] == ["psgd_dist_p", "psgd_dist_q", "psgd_dist_finish"]
    with pytest.raises(PsgdError):
        ctx.dist_q(dev(torch.zeros(40)), p, stream=0)     # float32 partials


def test_static_step_checks(monkeypatch):
    monkeypatch.setattr(_lib, "_on_device", lambda t: getattr(t, "_dev", False))
    stub = _StubLib()
    stub.psgd_step_static = lambda *a: 0
    monkeypatch.setattr(_lib, "load", lambda path=None: stub)
    g = [dev(torch.zeros(6, 5)) for _ in range(2)]
    q = dev(torch.zeros(5, 2))
    _lib.step_static(6, 5, 2, g, g, q, stream=0)
    with pytest.raises(PsgdError):
        _lib.step_static(6, 5, 2, g, g[:1], q, stream=0)
    with pytest.raises(PsgdError):
        _lib.step_static(6, 5, 3, g, g, q, stream=0)     # q is 5 x 2, not 5 x 3

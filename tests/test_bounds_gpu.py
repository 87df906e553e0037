"""Out-of-bounds writes: every buffer the library touches sits inside a
larger allocation whose guard regions hold a canary bit pattern; after
several steps in every mode the canaries must be intact (a substitute for a
memory checker, which this pool does not offer)."""
import pytest
import torch

from rank_gradient_compression_02_b200 import PowerSGD
from synth import GradientSource

from . import _harness as H

pytestmark = pytest.mark.gpu

CANARY = 0x7FA5A5A5          # a NaN bit pattern: any read of it shows up too
GUARD = 256                  # guard elements before and after (16-byte multiples)


class Guarded:
    def __init__(self):
        self.bufs = []

    def tensor(self, shape, dtype=torch.float32):
        numel = 1
        for s in shape:
            numel *= s
        esz = torch.tensor([], dtype=dtype).element_size()
        g = GUARD * 4 // esz
        raw = torch.empty(numel + 2 * g, dtype=dtype, device="cuda")
        raw.view(torch.int32 if esz == 4 else torch.int16).fill_(CANARY if esz == 4 else 0x7FA5)
        t = raw[g:g + numel].view(*shape)
        self.bufs.append((raw, g, numel, esz))
        return t

    def check(self):
        for raw, g, numel, esz in self.bufs:
            iv = raw.view(torch.int32 if esz == 4 else torch.int16)
            want = CANARY if esz == 4 else 0x7FA5
            assert bool((iv[:g] == want).all()), "guard before a buffer was written"
            assert bool((iv[g + numel:] == want).all()), "guard after a buffer was written"


SHAPES = [(300, 650), (33, 37), (129, 1000), (64, 576), (35, 33), (1, 40)]


@pytest.mark.parametrize("rank", [1, 3, 8, 16, 32])
@pytest.mark.parametrize("mode", ["eager", "lazy", "sumfirst", "iters2", "refresh"])
def test_no_write_outside_buffers(rank, mode):
    layers = [(m, n) for (m, n) in SHAPES if min(m, n) >= rank]
    if not layers:
        pytest.skip("no layer admits this rank")
    W = 3
    wl = H.small_workload(layers, rank, W)
    src = GradientSource(wl, seed=5)
    gd = Guarded()
    G = [[gd.tensor((m, n)) for (m, n) in layers] for _ in range(W)]
    E = [[gd.tensor((m, n)) for (m, n) in layers] for _ in range(W)]
    Q = [gd.tensor((n, rank)) for (_, n) in layers]
    P = [gd.tensor((m, rank)) for (m, _) in layers]
    Rc = [gd.tensor((m, n)) for (m, n) in layers]
    X = [gd.tensor((m, n)) for (m, n) in layers]
    Mo = [gd.tensor((m, n)) for (m, n) in layers]
    for w in range(W):
        for e in E[w]:
            e.zero_()
    for t in X + Mo:
        t.zero_()
    for l in range(len(layers)):
        Q[l].copy_(src.initial_q(l))
    kw = dict(lazy_errors=mode == "lazy", sum_first=mode == "sumfirst",
              power_iters=2 if mode == "iters2" else 1,
              svd_every=2 if mode == "refresh" else 0, svd_iters=4)
    lib = PowerSGD(layers, rank, W, seed=5, **kw)
    for step in range(3):
        for w in range(W):
            for l in range(len(layers)):
                G[w][l].copy_(src.layer_grad(step, w, l))
        lib.step(G, E, Q, P, Rc)
        lib.momentum_step(X, Mo, 0.1, 0.9)
    if mode == "lazy":
        lib.materialize_errors(E)
    lib.status()
    torch.cuda.synchronize()
    gd.check()
    for t in P + Q + Rc:
        assert bool(torch.isfinite(t).all())


def test_vec_mean_bounds():
    gd = Guarded()
    lens = [1, 3, 64, 1000]
    W = 4
    lib = PowerSGD([(8, 8)], 1, W)
    vecs = [[gd.tensor((k,)).normal_() for k in lens] for _ in range(W)]
    out = [gd.tensor((k,)) for k in lens]
    x = [gd.tensor((k,)).zero_() for k in lens]
    mo = [gd.tensor((k,)).zero_() for k in lens]
    lib.vec_mean(vecs, out, x, mo, lr=0.1, beta=0.9)
    lib.status()
    gd.check()

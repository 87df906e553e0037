"""GPU parity: the CUDA library (through its C ABI) against the float64
oracle on the same seeded inputs, element by element (relative Frobenius
norms), at sizes that span several tiles and ragged tails."""
import ctypes

import numpy as np
import pytest
import torch

import oracle.powersgd64 as ora
from oracle import philox64
from synth import C0, GradientSource, Workload

from . import _harness as H

pytestmark = pytest.mark.gpu

# shapes with every vector width (n % 4 == 0, n % 2 == 0, n odd), tall and
# wide, chunks with ragged tails, and min(m, n) = 33 so every rank fits
MIXED = [(300, 650), (64, 576), (40, 130), (256, 128), (33, 37), (700, 33), (129, 1000)]


@pytest.mark.parametrize("rank", [1, 2, 3, 4, 8, 16, 32])
@pytest.mark.parametrize("workers", [1, 3])
def test_mixed_shapes_f32(rank, workers):
    wl = H.small_workload(MIXED, rank, workers)
    _, _, hist = H.run_free(wl, steps=3)
    for t, e in enumerate(hist):
        H.assert_close(e, H.TOL["f32"], f"step {t}")


@pytest.mark.parametrize("rank", [1, 2, 4, 8])
def test_eight_byte_rows_odd_row_counts(rank):
    # 8-byte lanes (n % 4 == 2, and every even n at r = 8) on layers with an
    # odd number of rows and ragged row blocks
    wl = H.small_workload([(33, 650), (9, 10), (301, 26), (64, 576)], rank, 3)
    _, _, hist = H.run_free(wl, steps=3)
    for t, e in enumerate(hist):
        H.assert_close(e, H.TOL["f32"], f"step {t}")


# n % 4 == 2 with even row counts: 8-byte lanes, from one or three slots
# per row (n = 2, 6) to the LSTM's 650 columns
PAIRS = [(4, 6), (16, 14), (6, 10), (40, 130), (300, 650), (1000, 650)]


@pytest.mark.parametrize("rank,workers", [(1, 1), (2, 5), (3, 16), (4, 3), (4, 6)])
def test_eight_byte_rows_worker_counts(rank, workers):
    # every worker remainder of the first pass's load groups
    layers = PAIRS + ([(50, 2), (2, 6)] if rank <= 2 else [])
    wl = H.small_workload(layers, rank, workers)
    _, _, hist = H.run_free(wl, steps=3)
    for t, e in enumerate(hist):
        H.assert_close(e, H.TOL["f32"], f"step {t}")


@pytest.mark.parametrize("lazy,sum_first,dtype", [(True, False, "f32"), (False, True, "f32"),
                                                  (False, False, "bf16"), (True, True, "bf16")])
def test_eight_byte_rows_modes(lazy, sum_first, dtype):
    wl = H.small_workload(PAIRS, 4, 3, dtype=dtype)
    _, _, hist = H.run_free(wl, steps=3, lazy=lazy, sum_first=sum_first)
    for t, e in enumerate(hist):
        H.assert_close(e, 1e-4, f"step {t}")


@pytest.mark.parametrize("rank", [4, 32])
def test_tall_layer(rank):
    # 40000 x 64: m R up to 1.28 M elements of P_hat, past the P_hat
    # kernel's 4096 x 256 threads (its grid-stride loop), and 625 row blocks
    # (20 super-blocks) in the second pass's two-level reduction
    wl = H.small_workload([(40000, 64)], rank, 2)
    _, _, hist = H.run_free(wl, steps=2)
    for t, e in enumerate(hist):
        H.assert_close(e, H.TOL["f32"], f"step {t}")


@pytest.mark.parametrize("rank", [1, 4, 16, 32])
def test_mixed_shapes_bf16(rank):
    wl = H.small_workload(MIXED, rank, 4, dtype="bf16")
    _, _, hist = H.run_free(wl, steps=3)
    for t, e in enumerate(hist):
        # the oracle reads the same bf16 values widened exactly, so the
        # error stays at float32 level although the bar is 2e-2
        H.assert_close(e, H.TOL["bf16"], f"step {t}")
        H.assert_close(e, 1e-4, f"step {t} (fp32-level)")


@pytest.mark.parametrize("rank", [2, 8, 16, 32])
def test_sixteen_workers(rank):
    wl = H.small_workload(MIXED[:4], rank, 16)
    _, _, hist = H.run_free(wl, steps=2)
    for t, e in enumerate(hist):
        H.assert_close(e, H.TOL["f32"], f"step {t}")


@pytest.mark.parametrize("rank", [4, 16, 32])
@pytest.mark.parametrize("lazy,sum_first", [(True, False), (False, True), (True, True)])
def test_modes(lazy, sum_first, rank):
    wl = H.small_workload(MIXED, rank, 3)
    _, _, hist = H.run_free(wl, steps=4, lazy=lazy, sum_first=sum_first)
    for t, e in enumerate(hist):
        H.assert_close(e, H.TOL["f32"], f"step {t}")


@pytest.mark.parametrize("iters,lazy,rank", [(2, False, 4), (3, False, 4), (2, True, 4), (2, False, 32),
                                             (2, True, 16)])
def test_power_iterations(iters, lazy, rank):
    wl = H.small_workload(MIXED, rank, 3)
    run, _, hist = H.run_free(wl, steps=3, lazy=lazy, iters=iters)
    # per iteration: first pass, P_hat, second pass; + the third pass when eager
    assert run.lib.step_launches == 3 * iters + (0 if lazy else 1)
    for t, e in enumerate(hist):
        H.assert_close(e, H.TOL["f32"], f"step {t}")


def test_no_warm_start():
    # every step starts from a fresh Philox draw instead of the last Q_bar
    wl = H.small_workload(MIXED, 2, 3)
    _, _, hist = H.run_free(wl, steps=3, warm_start=False)
    for t, e in enumerate(hist):
        H.assert_close(e, H.TOL["f32"], f"step {t}")


def _check_refresh(wl, lazy, every, steps, iters=12, oversampling=None, min_gap=None, max_gap=None):
    """Free-running steps with PowerSGD+ refresh steps every `every`,
    against the oracle's exact truncated SVD of the worker mean on refresh
    steps (singular vectors compared up to sign) and its regular step
    otherwise.  min_gap / max_gap bound sigma_{r+1} / sigma_r of the
    refreshed worker mean (a property of the test data)."""
    rank = wl.rank
    L, W = len(wl.layers), wl.workers
    run = H.LibRun(wl, lazy=lazy, svd_every=every, svd_iters=iters, svd_oversampling=oversampling)
    Q0 = [run.src.initial_q(l) for l in range(L)]
    E0 = [[torch.zeros(m, n) for (m, n) in wl.layers] for _ in range(W)]
    run.set_state(E0, Q0)
    E = {l: [np.zeros(wl.layers[l]) for _ in range(W)] for l in range(L)}
    Q = {l: Q0[l].double().numpy() for l in range(L)}
    gaps = []
    for t in range(steps):
        host = run.fill_grads_host(t)
        run.run_step()
        last = t == steps - 1
        if lazy and last:
            run.lib.materialize_errors(run.E)
        torch.cuda.synchronize()
        refresh = (t + 1) % every == 0
        for l in range(L):
            G = [host[w][l].double().numpy() for w in range(W)]
            o = ora.svd_refresh_step(G, E[l], rank) if refresh else ora.step(G, E[l], Q[l])
            if refresh:
                s = o["sigma"]
                gaps.append(s[rank] / s[rank - 1])
            E[l], Q[l] = o["E_new"], o["Q_bar"]
            errs = {"G_hat": H.rel_fro(H.to64(run.Rc[l]), o["G_hat"]),
                    "P_hat": H.rel_fro(H.sign_aligned(H.to64(run.P[l]), o["P_hat"]), o["P_hat"]),
                    "Q_bar": H.rel_fro(H.sign_aligned(H.to64(run.Q[l]), o["Q_bar"]), o["Q_bar"])}
            if not lazy or last:
                errs["E_new"] = max(H.rel_fro(H.to64(run.E[w][l]), o["E_new"][w],
                                              denom=np.linalg.norm(o["M"][w])) for w in range(W))
            H.assert_close(errs, H.TOL["f32"], f"step {t} layer {l} refresh={refresh}")
            if refresh:
                # singular-vector form: orthogonal Q_bar columns, descending norms
                Qg = H.to64(run.Q[l])
                C = Qg.T @ Qg
                off = np.abs(C - np.diag(np.diag(C))).max() / np.abs(C).max()
                assert off < 1e-5, off
                assert np.all(np.diff(np.diag(C)) <= 1e-6 * C[0, 0])
    run.lib.status()
    if min_gap is not None:
        assert min(gaps) >= min_gap, gaps
    if max_gap is not None:
        assert max(gaps) <= max_gap, gaps
    return gaps


@pytest.mark.parametrize("rank,lazy,every,steps,over", [(4, False, 2, 4, None), (4, True, 2, 4, None),
                                                         (2, False, 1, 1, None), (1, False, 1, 1, None),
                                                         (4, False, 2, 4, 0), (2, False, 1, 1, 0)])
def test_svd_refresh(rank, lazy, every, steps, over):
    # PowerSGD+ refresh steps on data with a clear spectral gap at r: with
    # r >= 4 every direction of the 4-term spectrum is captured, so the
    # error memory holds noise only; with r < 4 the error memory builds up
    # the uncaptured directions until the gap at r closes, so those cases
    # refresh on the first step (E = 0) only.  over = 0: the rank-r block
    # without oversampling (12 iterations, rotation in place).
    wl = H.small_workload(MIXED[:5], rank, 3)
    _check_refresh(wl, lazy, every, steps, oversampling=over, max_gap=0.7)


# sigma_5 / sigma_4 = 0.9: a refresh at r = 4 on the rank-4 block alone
# would converge as 0.81^J (0.08 after 12 iterations); the oversampled block
# converges as (sigma_13 / sigma_4)^(2J), sigma_13 at the noise floor
_GAP_SPECTRUM = (10.0, 8.0, 6.0, 4.0, 3.6, 1.2, 0.6, 0.3)


@pytest.mark.parametrize("lazy,every,steps", [(False, 1, 1), (False, 3, 3), (True, 2, 4)])
def test_svd_refresh_small_gap_oversampled(lazy, every, steps):
    # the first refresh at step 1 sees the generator's spectrum (E = 0:
    # sigma_5 / sigma_4 = 0.9 exactly, up to the noise); later refreshes see
    # the spectrum error feedback has reshaped (0.6 to 0.8 on this data)
    wl = Workload(name="gap", layers=((300, 200), (96, 130), (129, 1000)), rank=4, workers=3, steps=steps,
                  noise=("rel", 0.01), spectrum=_GAP_SPECTRUM)
    gaps = _check_refresh(wl, lazy, every, steps, iters=16)
    if every == 1:
        assert min(gaps) >= 0.85, gaps


def test_from_random_state():
    wl = H.small_workload(MIXED, 4, 3)
    _, _, hist = H.run_free(wl, steps=2, random_state=0.05)
    for t, e in enumerate(hist):
        H.assert_close(e, H.TOL["f32"], f"step {t}")


def test_single_matrix_workload_all_steps():
    # 256 x 128, r = 2, W = 1, 10 warm-started steps, absolute noise 0.01
    _, _, hist = H.run_free(C0, steps=C0.steps)
    for t, e in enumerate(hist):
        H.assert_close(e, H.TOL["f32"], f"step {t}")


def _run_steps(wl, steps, lazy=False, seed=1234):
    run = H.LibRun(wl, seed=seed, lazy=lazy)
    for t in range(steps):
        run.fill_grads_host(t)
        run.run_step()
    if lazy:
        run.lib.materialize_errors(run.E)
    torch.cuda.synchronize()
    return run


def test_bitwise_deterministic():
    wl = H.small_workload(MIXED, 4, 3)
    a = _run_steps(wl, 3)
    b = _run_steps(wl, 3)
    for l in range(len(wl.layers)):
        assert torch.equal(a.Q[l], b.Q[l])
        assert torch.equal(a.P[l], b.P[l])
        for w in range(wl.workers):
            assert torch.equal(a.E[w][l], b.E[w][l])


@pytest.mark.parametrize("rank", [4, 16, 32])
def test_lazy_equals_eager_bitwise(rank):
    # E' = M - P_hat Q_bar^T rebuilt in the next step's first pass is the
    # same float32 arithmetic as the eager residual, so the runs agree bit
    # for bit (ranks 16, 32: the tensor-core first pass rebuilds it on the
    # CUDA cores in the residual pass's order)
    wl = H.small_workload(MIXED, rank, 3)
    a = _run_steps(wl, 4, lazy=False)
    b = _run_steps(wl, 4, lazy=True)
    for l in range(len(wl.layers)):
        assert torch.equal(a.Q[l], b.Q[l])
        assert torch.equal(a.P[l], b.P[l])
        for w in range(wl.workers):
            assert torch.equal(a.E[w][l], b.E[w][l])


def test_resume_bitwise():
    # 3 steps, hand the state (E, Q) to a fresh context, 3 more steps ==
    # 6 straight steps
    wl = H.small_workload(MIXED, 4, 3)
    straight = _run_steps(wl, 6)
    first = _run_steps(wl, 3)
    second = H.LibRun(wl)
    second.set_state(first.E, first.Q)
    # the gradient source must be at the same step
    for t in range(3, 6):
        host = [[first.src.layer_grad(t, w, l) for l in range(len(wl.layers))] for w in range(wl.workers)]
        for w in range(wl.workers):
            for l in range(len(wl.layers)):
                second.G[w][l].copy_(host[w][l])
        second.run_step()
    torch.cuda.synchronize()
    for l in range(len(wl.layers)):
        assert torch.equal(straight.Q[l], second.Q[l])
        for w in range(wl.workers):
            assert torch.equal(straight.E[w][l], second.E[w][l])


def test_zero_input_gives_zero_factors():
    wl = H.small_workload([(64, 48), (33, 7)], 3, 2)
    run = H.LibRun(wl)
    for w in range(2):
        for l in range(2):
            run.G[w][l].zero_()
    run.run_step()
    run.lib.status()
    for l in range(2):
        assert torch.count_nonzero(run.P[l]) == 0
        assert torch.count_nonzero(run.Q[l]) == 0
        assert torch.count_nonzero(run.Rc[l]) == 0
        for w in range(2):
            assert torch.count_nonzero(run.E[w][l]) == 0


def test_nan_propagates():
    wl = H.small_workload([(64, 48)], 2, 2)
    run = H.LibRun(wl)
    run.fill_grads_host(0)
    run.G[1][0][5, 7] = float("nan")
    run.run_step()
    run.lib.status()
    assert torch.isnan(run.P[0]).any()
    assert torch.isnan(run.Q[0]).any()
    assert torch.isnan(run.E[0][0]).any()


def test_exact_low_rank_reproduced():
    # noiseless rank-3 gradient, one worker: E' = 0 up to float32 rounding
    m, n, r = 300, 650, 3
    g = torch.Generator().manual_seed(5)
    U = torch.linalg.qr(torch.randn(m, r, generator=g, dtype=torch.float64))[0]
    M = (U @ torch.randn(r, n, generator=g, dtype=torch.float64)).float()
    wl = H.small_workload([(m, n)], r, 1)
    run = H.LibRun(wl)
    run.G[0][0].copy_(M)
    run.run_step()
    run.lib.status()
    rel = (run.E[0][0].double().norm() / M.double().norm()).item()
    assert rel < 1e-5, rel


def test_init_q_matches_oracle_draw():
    layers = [(64, 48), (33, 7), (10, 130)]
    from rank_gradient_compression_02_b200 import PowerSGD
    lib = PowerSGD(layers, 3, 2, seed=987654321)
    q = [torch.empty(n, 3, device="cuda") for (_, n) in layers]
    lib.init_q(q)
    lib.status()
    for l, (_, n) in enumerate(layers):
        want = philox64.initial_q(987654321, l, n, 3)
        got = q[l].cpu().numpy()
        np.testing.assert_allclose(got, want, rtol=2e-7, atol=1e-7)


def test_vec_mean_and_momentum():
    from rank_gradient_compression_02_b200 import PowerSGD
    W = 5
    lens = [64, 64, 128, 10, 1, 1000]
    lib = PowerSGD([(8, 8)], 2, W)
    g = torch.Generator().manual_seed(3)
    host = [[torch.randn(k, generator=g) for k in lens] for _ in range(W)]
    vecs = [[t.cuda() for t in hw] for hw in host]
    out = [torch.empty(k, device="cuda") for k in lens]
    x = [torch.zeros(k, device="cuda") for k in lens]
    mo = [torch.zeros(k, device="cuda") for k in lens]
    x_ref = [np.zeros(k) for k in lens]
    m_ref = [np.zeros(k) for k in lens]
    for it in range(3):
        lib.vec_mean(vecs, out, x, mo, lr=0.1, beta=0.9)
        for i in range(len(lens)):
            mean = ora.vec_mean([host[w][i].double().numpy() for w in range(W)])
            x_ref[i], m_ref[i] = ora.momentum_update(x_ref[i], m_ref[i], mean, 0.1, 0.9)
            np.testing.assert_allclose(out[i].cpu().numpy(), mean, rtol=1e-6, atol=1e-6)
    lib.status()
    for i in range(len(lens)):
        np.testing.assert_allclose(x[i].cpu().numpy(), x_ref[i], rtol=1e-5, atol=1e-6)


def test_momentum_step_matches_oracle():
    # (33, 650): 8-byte lanes with an odd row count
    wl = H.small_workload(MIXED[:4] + [(33, 650)], 2, 3)
    run = H.LibRun(wl)
    L = len(wl.layers)
    params = [torch.zeros(m, n, device="cuda") for (m, n) in wl.layers]
    mom = [torch.zeros(m, n, device="cuda") for (m, n) in wl.layers]
    Q0 = [run.src.initial_q(l) for l in range(L)]
    E0 = [[torch.zeros(m, n) for (m, n) in wl.layers] for _ in range(wl.workers)]
    run.set_state(E0, Q0)
    orc = H.OracleRun(range(L), {l: [e[l].double().numpy() for e in E0] for l in range(L)},
                      {l: Q0[l].double().numpy() for l in range(L)})
    xr = [np.zeros((m, n)) for (m, n) in wl.layers]
    mr = [np.zeros((m, n)) for (m, n) in wl.layers]
    for t in range(3):
        host = run.fill_grads_host(t)
        run.run_step()
        run.lib.momentum_step(params, mom, 0.1, 0.9)
        orc.step({l: [host[w][l].double().numpy() for w in range(wl.workers)] for l in range(L)})
        for l in range(L):
            xr[l], mr[l] = ora.momentum_update(xr[l], mr[l], orc.last[l]["G_hat"], 0.1, 0.9)
    run.lib.status()
    for l in range(L):
        assert H.rel_fro(H.to64(params[l]), xr[l]) < 1e-4
        assert H.rel_fro(H.to64(mom[l]), mr[l]) < 1e-4


def test_step_host_matches_device_step():
    wl = H.small_workload(MIXED, 4, 3)
    a = H.LibRun(wl)
    b = H.LibRun(wl)
    L = len(wl.layers)
    for t in range(2):
        host = a.fill_grads_host(t)
        a.run_step()
        pinned = [[host[w][l].pin_memory() for l in range(L)] for w in range(wl.workers)]
        ph = [torch.empty(m, wl.rank).pin_memory() for (m, _) in wl.layers]
        qh = [torch.empty(n, wl.rank).pin_memory() for (_, n) in wl.layers]
        b.lib.step_host(pinned, b.E, b.Q, ph, qh)
        torch.cuda.synchronize()
        for l in range(L):
            assert torch.equal(a.Q[l].cpu(), qh[l])
            assert torch.equal(a.P[l].cpu(), ph[l])
            for w in range(wl.workers):
                assert torch.equal(a.E[w][l], b.E[w][l])


@pytest.mark.parametrize("dtype", ["f32", "bf16"])
def test_step_host_flat_matches_device_step(dtype):
    # one pinned buffer per worker, layers at 16-byte aligned offsets with
    # gaps between them (the gap contents are uploaded and ignored)
    from rank_gradient_compression_02_b200 import PsgdError
    wl = H.small_workload(MIXED, 4, 3, dtype=dtype)
    a = H.LibRun(wl)
    b = H.LibRun(wl)
    L = len(wl.layers)
    esz = 2 if dtype == "bf16" else 4
    per16 = 16 // esz
    offs, o = [], 3 * per16
    for (m, n) in wl.layers:
        offs.append(o)
        o = -(-(o + m * n + 5) // per16) * per16
    hdt = torch.bfloat16 if dtype == "bf16" else torch.float32
    flat = [torch.full((o,), float("nan"), dtype=hdt).pin_memory() for _ in range(wl.workers)]
    for t in range(2):
        host = a.fill_grads_host(t)
        a.run_step()
        for w in range(wl.workers):
            for l, (m, n) in enumerate(wl.layers):
                flat[w][offs[l]:offs[l] + m * n].copy_(host[w][l].reshape(-1))
        ph = [torch.empty(m, wl.rank).pin_memory() for (m, _) in wl.layers]
        qh = [torch.empty(n, wl.rank).pin_memory() for (_, n) in wl.layers]
        b.lib.step_host_flat(flat, offs, b.E, b.Q, ph, qh)
        torch.cuda.synchronize()
        for l in range(L):
            assert torch.equal(a.Q[l].cpu(), qh[l])
            assert torch.equal(a.P[l].cpu(), ph[l])
            for w in range(wl.workers):
                assert torch.equal(a.E[w][l], b.E[w][l])
    bad = list(offs)
    bad[1] += 1    # not a multiple of 16 bytes
    with pytest.raises(PsgdError):
        b.lib.step_host_flat(flat, bad, b.E, b.Q)


@pytest.mark.parametrize("case", ["reversed", "many_layers", "lazy", "power2", "bf16"])
def test_step_host_flat_grouped_uploads(case):
    # the host-buffer step uploads contiguous layer groups on a stream of
    # its own and starts each group's passes once its copies have landed:
    # bit for bit the device step.  Layers packed in order (one copy per
    # group and worker) or in reverse order (one copy per layer); 14 layers
    # for 8 groups of one or two; lazy errors; two power iterations (the
    # step waits for the whole upload); bf16 gradients.
    layers = MIXED * 2 if case == "many_layers" else MIXED
    wl = H.small_workload(layers, 4, 3, dtype="bf16" if case == "bf16" else "f32")
    kw = {"lazy": case == "lazy", "iters": 2 if case == "power2" else 1}
    a = H.LibRun(wl, **kw)
    b = H.LibRun(wl, **kw)
    L = len(wl.layers)
    esz = 2 if case == "bf16" else 4
    per16 = 16 // esz
    order = list(range(L))[::-1] if case == "reversed" else list(range(L))
    offs, o = [0] * L, 0
    for l in order:
        m, n = wl.layers[l]
        offs[l] = o
        o = -(-(o + m * n) // per16) * per16
    hdt = torch.bfloat16 if case == "bf16" else torch.float32
    flat = [torch.full((o,), float("nan"), dtype=hdt).pin_memory() for _ in range(wl.workers)]
    for t in range(3):
        host = a.fill_grads_host(t)
        a.run_step()
        for w in range(wl.workers):
            for l, (m, n) in enumerate(wl.layers):
                flat[w][offs[l]:offs[l] + m * n].copy_(host[w][l].reshape(-1))
        ph = [torch.empty(m, wl.rank).pin_memory() for (m, _) in wl.layers]
        qh = [torch.empty(n, wl.rank).pin_memory() for (_, n) in wl.layers]
        b.lib.step_host_flat(flat, offs, b.E, b.Q, ph, qh)
        torch.cuda.synchronize()
        for l in range(L):
            assert torch.equal(a.Q[l].cpu(), qh[l]), (t, l)
            assert torch.equal(a.P[l].cpu(), ph[l]), (t, l)
            for w in range(wl.workers):
                assert torch.equal(a.E[w][l], b.E[w][l]), (t, l, w)
    b.lib.status()


def test_bad_arguments_rejected():
    from rank_gradient_compression_02_b200 import PowerSGD, PsgdError
    wl = H.small_workload([(64, 48)], 2, 2)
    run = H.LibRun(wl)
    base = torch.zeros(64 * 48 + 4, device="cuda")
    odd = base[1:1 + 64 * 48].view(64, 48)          # 4-byte offset: misaligned
    E_bad = [[odd], [run.E[1][0]]]
    with pytest.raises(PsgdError) as ei:
        run.lib.step(run.G, E_bad, run.Q, run.P, None)
    assert ei.value.code == 2
    with pytest.raises(PsgdError) as ei:
        run.lib.step(run.G, [[0], [run.E[1][0]]], run.Q, run.P, None)
    assert ei.value.code == 1
    with pytest.raises(PsgdError) as ei:
        run.lib.materialize_errors(run.E)   # not a lazy context
    assert ei.value.code == 5
    with pytest.raises(PsgdError):
        PowerSGD([(4, 3)], 4, 1)             # rank > min(m, n)
    run.lib.status()


def test_empty_layer_list_is_a_noop():
    from rank_gradient_compression_02_b200 import PowerSGD
    lib = PowerSGD([], 2, 3)
    assert lib.step_launches == 0
    lib.step([[], [], []], [[], [], []], [], [], None)
    lib.momentum_step([], [], 0.1, 0.9)
    lib.vec_mean([[], [], []], [])
    lib.status()


def test_many_workers():
    # 64 workers on small ragged layers (the worker-pointer tables and the
    # unrolled worker loops' remainders)
    wl = H.small_workload([(40, 130), (33, 37)], 4, 64)
    _, _, hist = H.run_free(wl, steps=2)
    for t, e in enumerate(hist):
        H.assert_close(e, H.TOL["f32"], f"step {t}")


@pytest.mark.parametrize("workers", [64, 256])
def test_many_workers_rank32(workers):
    # the tensor-core passes with 16-row tiles and every warp a worker part
    wl = H.small_workload([(40, 130), (33, 37), (64, 576)], 32, workers)
    _, _, hist = H.run_free(wl, steps=1)
    H.assert_close(hist[0], H.TOL["f32"], "step 0")


@pytest.mark.parametrize("rank", [16, 32])
@pytest.mark.parametrize("workers", [64, 256])
def test_many_workers_tensor_memory_pass(workers, rank):
    # the second pass on the 5th-generation tensor cores (16-byte rows):
    # float32 runs of up to four workers' rows inside the tensor core, then
    # float64; three free-running steps, full and ragged tiles and chunks
    wl = H.small_workload([(64, 576), (256, 128), (129, 1000)], rank, workers)
    _, _, hist = H.run_free(wl, steps=3)
    for t, e in enumerate(hist):
        H.assert_close(e, H.TOL["f32"], f"step {t}")


# r = min(m, n): wide and tall layers of exactly the rank (no compression;
# chunks of a few lanes at every lane width)
FULL_RANK = {2: [(2, 64), (50, 2)], 4: [(4, 90), (70, 4)], 8: [(8, 100), (100, 8)],
             16: [(16, 160), (200, 16)], 32: [(32, 400), (300, 32)]}


@pytest.mark.parametrize("rank", sorted(FULL_RANK))
def test_full_rank_is_lossless(rank):
    wl = H.small_workload(FULL_RANK[rank], rank, 3)
    run, orc, hist = H.run_free(wl, steps=3)
    for t, e in enumerate(hist):
        H.assert_close(e, H.TOL["f32"], f"step {t}")
    # the decompressed gradient is the worker mean of M itself
    for l in range(len(wl.layers)):
        o = orc.last[l]
        mbar = sum(o["M"]) / wl.workers
        got = run.Rc[l].double().cpu().numpy()
        assert np.linalg.norm(got - mbar) / np.linalg.norm(mbar) <= H.TOL["f32"]


def test_max_workers_single_row():
    # the largest worker count the library accepts, on a one-row layer and an
    # odd-width layer
    wl = H.small_workload([(1, 64), (9, 7)], 1, 256)
    _, _, hist = H.run_free(wl, steps=1)
    H.assert_close(hist[0], H.TOL["f32"], "step 0")


def test_zero_length_vectors():
    from rank_gradient_compression_02_b200 import PowerSGD
    lib = PowerSGD([(8, 8)], 1, 2)
    a = torch.zeros(0, device="cuda")
    b = torch.zeros(16, device="cuda")
    out = [torch.zeros(0, device="cuda"), torch.empty(16, device="cuda")]
    lib.vec_mean([[a, b], [a, b + 2.0]], out)
    lib.status()
    assert torch.allclose(out[1], torch.ones(16, device="cuda"))

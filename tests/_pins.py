"""Checks that pin the float64 oracle to facts fixed outside the oracle itself:
hand-worked cases, closed forms, textbook special cases computed by a
different algorithm (Householder QR, LAPACK SVD), exact invariants of the
method.  Each check takes the oracle module as an argument so that the
mutation tests can run the same checks against deliberately broken copies.

Page citations: "anthology-of-the-sota" note-152 on PowerSGD ([N152]),
sections "Method" and "Concepts"; the "PowerSGD" glossary page ([GLOS]).
"""
from __future__ import annotations

import json
import math
import os

import numpy as np

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def _rng(seed):
    return np.random.default_rng(seed)


def _householder_qr_posdiag(P):
    q, r = np.linalg.qr(P)
    s = np.sign(np.diag(r))
    s[s == 0] = 1.0
    return q * s[None, :]


def check_hand_cases(ora):
    """Hand-derived 3x2 steps ([N152] "Method")."""
    with open(os.path.join(GOLDEN, "hand_cases.json")) as f:
        cases = json.load(f)["cases"]
    for c in cases:
        G = [np.array(g, dtype=np.float64) for g in c["G"]]
        E = [np.array(e, dtype=np.float64) for e in c.get("E", [np.zeros_like(g) for g in G])]
        Q = np.array(c["Q"], dtype=np.float64)
        o = ora.step(G, E, Q)
        for key in ("P_hat", "Q_bar", "G_hat"):
            np.testing.assert_allclose(o[key], np.array(c[key]), rtol=0, atol=1e-14, err_msg=f"{c['name']}:{key}")
        for w, e in enumerate(c["E_new"]):
            np.testing.assert_allclose(o["E_new"][w], np.array(e), rtol=0, atol=1e-14, err_msg=f"{c['name']}:E_new[{w}]")


def check_gram_schmidt_vs_householder(ora):
    """Thin QR with a positive-diagonal R is unique, so Gram-Schmidt must give
    Householder QR's Q after fixing signs ([N152] "Method", Gram-Schmidt)."""
    rng = _rng(1)
    for m, r in ((7, 1), (9, 3), (64, 4), (300, 8), (513, 32)):
        P = rng.standard_normal((m, r)) * np.logspace(0, -3, r)[None, :]
        got = ora.gram_schmidt(P)
        np.testing.assert_allclose(got, _householder_qr_posdiag(P), rtol=0, atol=1e-10)
        np.testing.assert_allclose(got.T @ got, np.eye(r), rtol=0, atol=1e-12)


def check_gram_schmidt_rank_deficient(ora):
    """Zero input gives zero; an exactly dependent column becomes zero and the
    rest stay orthonormal (reading of the pages' silence on rank
    deficiency)."""
    assert np.all(ora.gram_schmidt(np.zeros((5, 3))) == 0.0)
    rng = _rng(2)
    a = rng.standard_normal(6)
    b = rng.standard_normal(6)
    P = np.stack([a, 2.0 * a, b], axis=1)
    Ph = ora.gram_schmidt(P)
    assert np.all(Ph[:, 1] == 0.0) or np.linalg.norm(Ph[:, 1]) == 0.0
    np.testing.assert_allclose(Ph[:, [0, 2]].T @ Ph[:, [0, 2]], np.eye(2), atol=1e-12)
    np.testing.assert_allclose(Ph[:, 0], a / np.linalg.norm(a), atol=1e-14)


def check_rank1_closed_form(ora):
    """M = sigma u v^T, r = 1: P_hat = sign(v.q) u, Q_bar = sign(v.q) sigma v,
    E' = 0."""
    rng = _rng(3)
    for m, n in ((5, 3), (40, 70)):
        u = rng.standard_normal(m); u /= np.linalg.norm(u)
        v = rng.standard_normal(n); v /= np.linalg.norm(v)
        sigma = 3.7
        M = sigma * np.outer(u, v)
        q = rng.standard_normal((n, 1))
        s = math.copysign(1.0, float(v @ q[:, 0]))
        o = ora.step([M], [np.zeros_like(M)], q)
        np.testing.assert_allclose(o["P_hat"][:, 0], s * u, atol=1e-13)
        np.testing.assert_allclose(o["Q_bar"][:, 0], s * sigma * v, atol=1e-13)
        np.testing.assert_allclose(o["E_new"][0], 0.0, atol=1e-13)


def check_exact_low_rank(ora):
    """A noiseless M of rank <= r is reproduced exactly after one step: E' = 0
    for one worker; with W workers whose matrices share one r-dimensional
    column space, E'_w = M_w - mean(M) and mean_w E'_w = 0."""
    rng = _rng(4)
    m, n, r = 30, 20, 3
    U = np.linalg.qr(rng.standard_normal((m, r)))[0]
    M = U @ rng.standard_normal((r, n))
    o = ora.step([M], [np.zeros_like(M)], rng.standard_normal((n, r)))
    np.testing.assert_allclose(o["E_new"][0], 0.0, atol=1e-12)
    Ms = [U @ rng.standard_normal((r, n)) for _ in range(3)]
    o = ora.step(Ms, [np.zeros_like(x) for x in Ms], rng.standard_normal((n, r)))
    Mbar = sum(Ms) / 3
    for w in range(3):
        np.testing.assert_allclose(o["E_new"][w], Ms[w] - Mbar, atol=1e-12)


def check_full_rank_is_lossless(ora):
    """r = min(m, n): the factors span M_bar's whole column space, so the
    decompressed gradient is the worker mean itself and each worker keeps
    only its deviation from it: G_hat = mean(M), E'_w = M_w - mean(M).  With
    r = m, P_hat is square and orthogonal."""
    rng = _rng(12)
    for m, n in ((6, 40), (40, 6)):
        r = min(m, n)
        W = 3
        G = [rng.standard_normal((m, n)) for _ in range(W)]
        E = [0.2 * rng.standard_normal((m, n)) for _ in range(W)]
        o = ora.step(G, E, rng.standard_normal((n, r)))
        Mbar = sum(g + e for g, e in zip(G, E)) / W
        np.testing.assert_allclose(o["G_hat"], Mbar, atol=1e-11)
        for w in range(W):
            np.testing.assert_allclose(o["E_new"][w], G[w] + E[w] - Mbar, atol=1e-11)
        if r == m:
            np.testing.assert_allclose(o["P_hat"] @ o["P_hat"].T, np.eye(m), atol=1e-12)


def check_identities(ora):
    """P_hat^T P_hat = I; P_hat Q_bar^T + E'_w = M_w; P_hat^T mean_w E'_w = 0;
    Q_bar = mean(M)^T P_hat ([N152] "Method")."""
    rng = _rng(5)
    m, n, r, W = 50, 37, 4, 3
    G = [rng.standard_normal((m, n)) for _ in range(W)]
    E = [0.3 * rng.standard_normal((m, n)) for _ in range(W)]
    o = ora.step(G, E, rng.standard_normal((n, r)))
    Ph, Qb = o["P_hat"], o["Q_bar"]
    np.testing.assert_allclose(Ph.T @ Ph, np.eye(r), atol=1e-12)
    for w in range(W):
        np.testing.assert_allclose(Ph @ Qb.T + o["E_new"][w], G[w] + E[w], atol=1e-12)
    Ebar = sum(o["E_new"]) / W
    np.testing.assert_allclose(Ph.T @ Ebar, 0.0, atol=1e-12)
    Mbar = sum(g + e for g, e in zip(G, E)) / W
    np.testing.assert_allclose(Qb, Mbar.T @ Ph, atol=1e-12)


def check_linearity(ora):
    """compress(average) = average(compress) ([N152] "Concepts", linearity):
    the W-worker step gives the same P_bar, P_hat, Q_bar as a one-worker step
    on the mean matrix."""
    rng = _rng(6)
    m, n, r, W = 40, 24, 3, 5
    G = [rng.standard_normal((m, n)) for _ in range(W)]
    E = [rng.standard_normal((m, n)) for _ in range(W)]
    Q = rng.standard_normal((n, r))
    o = ora.step(G, E, Q)
    Mbar = sum(g + e for g, e in zip(G, E)) / W
    o1 = ora.step([Mbar], [np.zeros_like(Mbar)], Q)
    for key in ("P_bar", "P_hat", "Q_bar", "G_hat"):
        np.testing.assert_allclose(o[key], o1[key], atol=1e-12, err_msg=key)


def check_jacobi_svd(ora):
    """The hand-written one-sided Jacobi SVD agrees with LAPACK's SVD."""
    rng = _rng(7)
    for m, n in ((12, 5), (5, 12), (40, 40)):
        A = rng.standard_normal((m, n))
        U, s, V = ora.jacobi_svd(A)
        s_ref = np.linalg.svd(A, compute_uv=False)
        np.testing.assert_allclose(s, s_ref, rtol=1e-12)
        np.testing.assert_allclose(U @ np.diag(s) @ V.T, A, atol=1e-12)
        k = min(m, n)
        np.testing.assert_allclose(U.T @ U, np.eye(k), atol=1e-12)
        np.testing.assert_allclose(V.T @ V, np.eye(k), atol=1e-12)


def check_warm_start_convergence(ora, m=96, n=64, r=2, steps=14):
    """Warm-started single steps on a fixed M without error feedback converge
    to the top-r left singular subspace ([N152] "Concepts", warm-start
    subspace iteration).  Each step is one subspace-iteration step on M M^T,
    so the error falls by (sigma_{r+1}/sigma_r)^2 per step once the start-up
    transient is over; the reference subspace and singular values come from
    the hand-written Jacobi SVD."""
    rng = _rng(8)
    U = np.linalg.qr(rng.standard_normal((m, 4)))[0]
    V = np.linalg.qr(rng.standard_normal((n, 4)))[0]
    sig = np.array([5.0, 2.5, 1.25, 0.625])
    M = U @ np.diag(sig) @ V.T + 1e-3 * rng.standard_normal((m, n))
    Ur, s, _ = ora.jacobi_svd(M)
    ratio2 = (s[r] / s[r - 1]) ** 2
    Q = rng.standard_normal((n, r))
    errs = []
    for _ in range(steps):
        o = ora.step([M], [np.zeros_like(M)], Q)
        Q = o["Q_bar"]
        errs.append(ora.subspace_sin_max(Ur[:, :r], o["P_hat"]))
    rates = [b / a for a, b in zip(errs[-5:-1], errs[-4:])]
    for q in rates:
        assert 0.8 * ratio2 < q < 1.25 * ratio2, (rates, ratio2, errs)
    assert errs[-1] < 1e-5, errs


def check_error_feedback_telescopes(ora):
    """With E_0 = 0, nothing is lost, only delayed ([GLOS] error-feedback
    paragraph): mean_w E_T + sum_t G_hat_t = sum_t mean_w G_t."""
    rng = _rng(9)
    m, n, r, W, T = 20, 15, 2, 3, 6
    E = [np.zeros((m, n)) for _ in range(W)]
    Q = rng.standard_normal((n, r))
    sum_g = np.zeros((m, n))
    sum_ghat = np.zeros((m, n))
    for _ in range(T):
        G = [rng.standard_normal((m, n)) for _ in range(W)]
        o = ora.step(G, E, Q)
        E, Q = o["E_new"], o["Q_bar"]
        sum_g += sum(G) / W
        sum_ghat += o["G_hat"]
    np.testing.assert_allclose(sum(E) / W + sum_ghat, sum_g, atol=1e-12)


def check_momentum_closed_form(ora):
    """Heavy-ball momentum after decompression ([N152] "Concepts"): from
    x_0 = 0, mom_0 = 0, x_T = -lr * sum_t sum_{s<=t} beta^(t-s) G_hat_s."""
    rng = _rng(10)
    lr, beta, T = 0.1, 0.9, 7
    gs = [rng.standard_normal((4, 3)) for _ in range(T)]
    x = np.zeros((4, 3))
    mom = np.zeros((4, 3))
    for g in gs:
        x, mom = ora.momentum_update(x, mom, g, lr, beta)
    want = np.zeros((4, 3))
    for t in range(T):
        for s in range(t + 1):
            want -= lr * beta ** (t - s) * gs[s]
    np.testing.assert_allclose(x, want, atol=1e-13)


def check_vec_mean(ora):
    vs = [np.array([1.0, 2.0, 3.0]), np.array([3.0, 2.0, 1.0]), np.array([2.0, 5.0, -1.0])]
    np.testing.assert_allclose(ora.vec_mean(vs), [2.0, 3.0, 1.0], atol=1e-15)


def check_power_iterations(ora):
    """k power iterations in one step equal k warm-started single steps on the
    same M without error feedback (each iteration is one step of subspace
    iteration, [GLOS] warm-start paragraph), and converge twice as fast."""
    rng = _rng(11)
    m, n, r = 40, 30, 2
    U = np.linalg.qr(rng.standard_normal((m, 4)))[0]
    V = np.linalg.qr(rng.standard_normal((n, 4)))[0]
    M = U @ np.diag([5.0, 2.5, 1.25, 0.625]) @ V.T + 1e-3 * rng.standard_normal((m, n))
    Q = rng.standard_normal((n, r))
    Z = np.zeros_like(M)
    two = ora.step([M], [Z], Q, iters=2)
    one = ora.step([M], [Z], ora.step([M], [Z], Q)["Q_bar"])
    for key in ("P_hat", "Q_bar", "G_hat"):
        np.testing.assert_allclose(two[key], one[key], atol=1e-12, err_msg=key)
    np.testing.assert_allclose(two["E_new"][0], M - one["G_hat"], atol=1e-12)
    # residual uses the last iteration's factors: P_hat^T E' = 0
    np.testing.assert_allclose(two["P_hat"].T @ two["E_new"][0], 0.0, atol=1e-12)
    Ur, _, _ = ora.jacobi_svd(M)
    e1 = ora.subspace_sin_max(Ur[:, :r], ora.step([M], [Z], Q, iters=3)["P_hat"])
    q = Q
    for _ in range(3):
        o = ora.step([M], [Z], q)
        q = o["Q_bar"]
    assert abs(e1 - ora.subspace_sin_max(Ur[:, :r], o["P_hat"])) < 1e-12


def check_svd_refresh(ora):
    """The refresh step's reconstruction is the best rank-r approximation of
    the worker mean (Eckart-Young: its error is the tail of the singular
    values), its factors are orthonormal / orthogonal with descending norms,
    it agrees with the hand-written Jacobi SVD, and converged warm-started
    power iterations reach the same reconstruction."""
    rng = _rng(12)
    m, n, r, W = 36, 28, 3, 3
    U = np.linalg.qr(rng.standard_normal((m, 6)))[0]
    V = np.linalg.qr(rng.standard_normal((n, 6)))[0]
    base = U @ np.diag([6.0, 3.0, 1.5, 0.5, 0.2, 0.1]) @ V.T
    G = [base + 0.01 * rng.standard_normal((m, n)) for _ in range(W)]
    E = [0.01 * rng.standard_normal((m, n)) for _ in range(W)]
    o = ora.svd_refresh_step(G, E, r)
    Mbar = sum(g + e for g, e in zip(G, E)) / W
    s = np.linalg.svd(Mbar, compute_uv=False)
    assert abs(np.linalg.norm(Mbar - o["G_hat"]) ** 2 - np.sum(s[r:] ** 2)) < 1e-10
    np.testing.assert_allclose(o["P_hat"].T @ o["P_hat"], np.eye(r), atol=1e-12)
    QtQ = o["Q_bar"].T @ o["Q_bar"]
    np.testing.assert_allclose(QtQ, np.diag(s[:r] ** 2), atol=1e-10)
    Uj, sj, Vj = ora.jacobi_svd(Mbar)
    np.testing.assert_allclose(Uj[:, :r] @ np.diag(sj[:r]) @ Vj[:, :r].T, o["G_hat"], atol=1e-10)
    for w in range(W):
        np.testing.assert_allclose(o["E_new"][w], G[w] + E[w] - o["G_hat"], atol=1e-12)
    deep = ora.step(G, E, rng.standard_normal((n, r)), iters=40)
    np.testing.assert_allclose(deep["G_hat"], o["G_hat"], atol=1e-9)


def check_subspace_sin_max(ora):
    """Principal angles by construction: with [U V] orthonormal, the
    columns u_i cos t_i + v_i sin t_i span a subspace at angles t_i from
    span(U); the largest sine must come back, also for a tiny angle (the
    reason the oracle takes the spectral norm of the off-span part rather
    than sqrt(1 - cos^2))."""
    rng = np.random.default_rng(11)
    n, r = 40, 3
    B, _ = np.linalg.qr(rng.standard_normal((n, 2 * r)))
    U, V = B[:, :r], B[:, r:]
    for angles in ([0.3, 0.1, 0.05], [1e-9, 2e-9, 5e-10], [0.0, 0.0, 0.0], [np.pi / 2, 0.2, 0.1]):
        t = np.array(angles)
        P = U * np.cos(t) + V * np.sin(t)
        # a rotation inside the span changes the basis, not the subspace
        Rm, _ = np.linalg.qr(rng.standard_normal((r, r)))
        got = ora.subspace_sin_max(U, P @ Rm)
        want = float(np.max(np.sin(t)))
        assert abs(got - want) <= 1e-12 + 1e-6 * want, (angles, got, want)


def check_orthogonal_equivariance(ora):
    """Rotating the problem rotates the answer: for orthogonal U (m x m) and
    V (n x n), the step on U G_w V, U E_w V with warm start V^T Q gives
    U P_hat, V^T Q_bar and U E'_w V.  P = (U M V)(V^T Q) = U M Q keeps its
    Gram matrix, so the orthogonalisation is the same ([N152] "Method":
    P = M Q, orthogonalise, Q = M^T P_hat, E' = M - P_hat Q^T).  A product
    taken on the wrong side or with a transposed operand breaks it."""
    rng = _rng(12)
    m, n, r, W = 30, 22, 3, 3
    G = [rng.standard_normal((m, n)) for _ in range(W)]
    E = [0.5 * rng.standard_normal((m, n)) for _ in range(W)]
    Q = rng.standard_normal((n, r))
    U, _ = np.linalg.qr(rng.standard_normal((m, m)))
    V, _ = np.linalg.qr(rng.standard_normal((n, n)))
    o = ora.step(G, E, Q)
    o2 = ora.step([U @ g @ V for g in G], [U @ e @ V for e in E], V.T @ Q)
    np.testing.assert_allclose(o2["P_hat"], U @ o["P_hat"], atol=1e-10)
    np.testing.assert_allclose(o2["Q_bar"], V.T @ o["Q_bar"], atol=1e-10)
    for w in range(W):
        np.testing.assert_allclose(o2["E_new"][w], U @ o["E_new"][w] @ V, atol=1e-10)


def check_scale_homogeneity(ora):
    """Scaling G and E by c: P = c M Q has Gram matrix c^2 P^T P, so the
    normalised P_hat becomes sign(c) P_hat, Q_bar = (c M)^T P_hat becomes
    |c| Q_bar, and E'_w and G_hat become c times theirs ([N152] "Method":
    the orthogonalisation normalises the columns).  A missing or repeated
    normalisation, or a sign lost in it, breaks it."""
    rng = _rng(13)
    m, n, r, W = 26, 19, 4, 2
    G = [rng.standard_normal((m, n)) for _ in range(W)]
    E = [0.5 * rng.standard_normal((m, n)) for _ in range(W)]
    Q = rng.standard_normal((n, r))
    o = ora.step(G, E, Q)
    for c in (8.0, -0.5, 3.0e-3):
        oc = ora.step([c * g for g in G], [c * e for e in E], Q)
        scale = max(1.0, abs(c))
        np.testing.assert_allclose(oc["P_hat"], math.copysign(1.0, c) * o["P_hat"], atol=1e-12)
        np.testing.assert_allclose(oc["Q_bar"], abs(c) * o["Q_bar"], atol=1e-12 * scale)
        np.testing.assert_allclose(oc["G_hat"], c * o["G_hat"], atol=1e-12 * scale)
        for w in range(W):
            np.testing.assert_allclose(oc["E_new"][w], c * o["E_new"][w], atol=1e-12 * scale)


ALL_CHECKS = [
    check_hand_cases, check_gram_schmidt_vs_householder, check_gram_schmidt_rank_deficient,
    check_full_rank_is_lossless,
    check_rank1_closed_form, check_exact_low_rank, check_identities, check_linearity,
    check_jacobi_svd, check_warm_start_convergence, check_error_feedback_telescopes,
    check_momentum_closed_form, check_vec_mean, check_power_iterations, check_svd_refresh,
    check_subspace_sin_max, check_orthogonal_equivariance, check_scale_homogeneity,
]

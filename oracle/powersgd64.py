"""Float64 CPU oracle for the PowerSGD compression step.

TEST INFRASTRUCTURE ONLY.  Nothing in the product path may import, call or
execute this module: only the test suite, the smoke check of the entry
script and the CPU-baseline leg of the benchmark use it.  It shares no code
with the CUDA library and does not import the package that wraps it.

Sources (cited by page title and section):
  [N152]  "anthology-of-the-sota" note-152 on PowerSGD, sections "Method" and
          "Concepts" (the most precise statement of the step order).
  [GLOS]  "PowerSGD" glossary page (inferensys), error-feedback and
          warm-start paragraphs.
  [ABS]   "PowerSGD: Practical Low-Rank Gradient Compression for Distributed
          Optimization", Abstract.
  [PLUS]  "From PowerSGD to PowerSGD+ ...", Abstract (the periodic SVD
          refresh of the projection subspace).

Everything is computed in float64 with plain NumPy; matrix products use
``@`` (a library primitive), every other step is written out as the method
states it, per layer, with no fusion or reordering.  All state (E, Q) is
float64 here; callers pass the exact input values (fp32 or bf16 widened
exactly to float64).

Readings of points the pages leave open (each is also listed in the design
notes of the repository):
  * residual against the aggregated factors: E'_w = M_w - P_hat Qbar^T, with
    Qbar the mean over workers (what every worker applies after
    decompression, [N152] "Concepts", post-compression momentum);
  * orthogonalisation = modified Gram-Schmidt over columns 0..r-1 with the
    natural positive sign; a column whose squared norm after projection is
    at most DROP_TOL * max_k ||pbar_k||^2 becomes zero (the pages are silent
    on rank deficiency);
  * Q state between steps is Qbar exactly, not re-normalised;
  * post-compression momentum is heavy ball without dampening:
    mom <- beta*mom + Ghat; x <- x - lr*mom.
"""
from __future__ import annotations

import math
from typing import Sequence

import numpy as np

DROP_TOL = 1e-12


def _f64(a) -> np.ndarray:
    return np.asarray(a, dtype=np.float64)


# --- the steps of one compression step ([N152] "Method") ---------------------

def error_feedback_add(G, E) -> np.ndarray:
    """M = G + E: the stored residual is added to the fresh gradient before
    compression ([GLOS] error-feedback paragraph; [N152] "Concepts", error
    feedback)."""
    return _f64(G) + _f64(E)


def right_multiply(M, Q) -> np.ndarray:
    """P = M Q with the warm-started Q ([N152] "Method")."""
    return _f64(M) @ _f64(Q)


def worker_mean(parts: Sequence[np.ndarray]) -> np.ndarray:
    """Mean over workers, the result of the all-reduce of P or Q divided by
    the worker count ([N152] "Method"; linearity in "Concepts").  Summed in
    worker order."""
    acc = np.zeros_like(_f64(parts[0]))
    for p in parts:
        acc = acc + _f64(p)
    return acc / len(parts)


def gram_schmidt(P, drop_tol: float = DROP_TOL) -> np.ndarray:
    """Orthonormalise the columns of P by modified Gram-Schmidt ([N152]
    "Method", Gram-Schmidt orthogonalisation of the P factor).

    Column j is made orthogonal to the already finished columns 0..j-1, one
    projection at a time on the running vector, then scaled to unit length.
    A column whose remaining squared norm is <= drop_tol * (largest squared
    column norm of the input) is set to zero instead (rank-deficient input;
    an all-zero P gives an all-zero result).
    """
    P = _f64(P)
    m, r = P.shape
    scale = max((float(P[:, k] @ P[:, k]) for k in range(r)), default=0.0)
    out = np.zeros((m, r), dtype=np.float64)
    for j in range(r):
        v = P[:, j].copy()
        for k in range(j):
            v = v - float(out[:, k] @ v) * out[:, k]
        nrm2 = float(v @ v)
        if nrm2 <= drop_tol * scale:
            out[:, j] = 0.0
        else:
            out[:, j] = v / math.sqrt(nrm2)
    return out


def left_multiply(M, P_hat) -> np.ndarray:
    """Q = M^T P_hat ([N152] "Method")."""
    return _f64(M).T @ _f64(P_hat)


def decompress(P_hat, Q_bar) -> np.ndarray:
    """Reconstructed mean gradient P_hat Qbar^T ([N152] "Method": the factors
    are sent instead of M and multiplied back out)."""
    return _f64(P_hat) @ _f64(Q_bar).T


def residual(M, P_hat, Q_bar) -> np.ndarray:
    """New error memory: true minus reconstructed, E' = M - P_hat Qbar^T
    ([N152] "Method" and "Concepts", error feedback)."""
    return _f64(M) - decompress(P_hat, Q_bar)


def momentum_update(x, mom, g_hat, lr: float, beta: float):
    """Post-compression heavy-ball momentum applied to the decompressed
    aggregate ([N152] "Concepts"): mom <- beta*mom + g_hat; x <- x - lr*mom."""
    mom = beta * _f64(mom) + _f64(g_hat)
    x = _f64(x) - lr * mom
    return x, mom


def vec_mean(vecs: Sequence[np.ndarray]) -> np.ndarray:
    """Bias vectors and other small tensors travel uncompressed: their
    aggregate is the plain mean over workers ([N152] "Method")."""
    return worker_mean(vecs)


def step(G: Sequence[np.ndarray], E: Sequence[np.ndarray], Q, drop_tol: float = DROP_TOL, iters: int = 1) -> dict:
    """One PowerSGD compression step for one layer and W workers, in the
    order of [N152] "Method".

    G, E: length-W lists of m x n arrays (gradient and error memory of each
    worker).  Q: n x r warm start shared by all workers.
    iters: power (subspace) iterations in the step ([GLOS] warm-start
    paragraph: one or two suffice).  Reading: every iteration repeats the
    right multiply, mean, orthogonalisation, left multiply and mean, the next
    iteration starting from the Q_bar just formed; the residual uses the
    last iteration's factors.
    Returns M, P (per worker), P_bar, P_hat, Qw (per worker), Q_bar,
    E_new (per worker) and G_hat (of the last iteration).
    """
    W = len(G)
    M = [error_feedback_add(G[w], E[w]) for w in range(W)]
    Q_cur = _f64(Q)
    for _ in range(iters):
        P = [right_multiply(M[w], Q_cur) for w in range(W)]
        P_bar = worker_mean(P)
        P_hat = gram_schmidt(P_bar, drop_tol)
        Qw = [left_multiply(M[w], P_hat) for w in range(W)]
        Q_bar = worker_mean(Qw)
        Q_cur = Q_bar
    E_new = [residual(M[w], P_hat, Q_bar) for w in range(W)]
    G_hat = decompress(P_hat, Q_bar)
    return dict(M=M, P=P, P_bar=P_bar, P_hat=P_hat, Qw=Qw, Q_bar=Q_bar, E_new=E_new, G_hat=G_hat)


def svd_refresh_step(G: Sequence[np.ndarray], E: Sequence[np.ndarray], rank: int) -> dict:
    """A PowerSGD+ refresh step ([PLUS] Abstract: the projection subspace is
    periodically re-aligned with the optimal one by a singular value
    decomposition).  Reading: on a refresh step the compressed form of the
    aggregate M_bar = mean_w(G_w + E_w) is its rank-r truncated SVD,
    P_hat = U_r, Q_bar = V_r Sigma_r (so the warm start of the next step is
    V_r Sigma_r), and the error memory is E'_w = M_w - U_r Sigma_r V_r^T.
    The SVD is a library primitive here (LAPACK through NumPy); singular
    vectors are unique only up to sign, so callers compare them up to
    column sign."""
    W = len(G)
    M = [error_feedback_add(G[w], E[w]) for w in range(W)]
    M_bar = worker_mean(M)
    U, s, Vt = np.linalg.svd(M_bar, full_matrices=False)
    P_hat = U[:, :rank].copy()
    Q_bar = Vt[:rank, :].T * s[None, :rank]
    E_new = [residual(M[w], P_hat, Q_bar) for w in range(W)]
    G_hat = decompress(P_hat, Q_bar)
    return dict(M=M, M_bar=M_bar, P_hat=P_hat, Q_bar=Q_bar, E_new=E_new, G_hat=G_hat, sigma=s)


# --- reference SVD for subspace checks ----------------------------------------

def jacobi_svd(A, tol: float = 1e-15, max_sweeps: int = 60):
    """One-sided Jacobi SVD (Hestenes 1958): rotate pairs of columns of A
    until all are mutually orthogonal; the column norms are the singular
    values, the normalised columns the left singular vectors and the
    accumulated rotations the right ones.  Written out by hand so that the
    warm-start convergence check does not rest on the same library as the
    rest of the oracle.  Returns U (m x k), s (k,), V (n x k), k = min(m, n),
    sorted by decreasing s."""
    A = _f64(A)
    m, n = A.shape
    transpose = m < n
    if transpose:
        A = A.T
        m, n = n, m
    U = A.copy()
    V = np.eye(n)
    for _ in range(max_sweeps):
        off = 0.0
        for p in range(n - 1):
            for q in range(p + 1, n):
                alpha = float(U[:, p] @ U[:, p])
                beta = float(U[:, q] @ U[:, q])
                gamma = float(U[:, p] @ U[:, q])
                if alpha == 0.0 or beta == 0.0:
                    continue
                c_rel = abs(gamma) / math.sqrt(alpha * beta)
                off = max(off, c_rel)
                if c_rel <= tol:
                    continue
                zeta = (beta - alpha) / (2.0 * gamma)
                t = math.copysign(1.0, zeta) / (abs(zeta) + math.sqrt(1.0 + zeta * zeta))
                c = 1.0 / math.sqrt(1.0 + t * t)
                s = c * t
                up = U[:, p].copy()
                U[:, p] = c * up - s * U[:, q]
                U[:, q] = s * up + c * U[:, q]
                vp = V[:, p].copy()
                V[:, p] = c * vp - s * V[:, q]
                V[:, q] = s * vp + c * V[:, q]
        if off <= tol:
            break
    sv = np.sqrt(np.einsum("ij,ij->j", U, U))
    order = np.argsort(-sv, kind="stable")
    sv = sv[order]
    U = U[:, order]
    V = V[:, order]
    nz = sv > 0
    U[:, nz] = U[:, nz] / sv[nz]
    if transpose:
        return V, sv, U
    return U, sv, V


def subspace_sin_max(U_ref, P_hat) -> float:
    """Largest principal-angle sine between span(U_ref) and span(P_hat), both
    with orthonormal columns: the spectral norm of the part of P_hat outside
    span(U_ref), (I - U_ref U_ref^T) P_hat.  (Taken this way rather than as
    sqrt(1 - cos^2) so that it stays accurate for tiny angles.)"""
    U_ref = _f64(U_ref)
    P_hat = _f64(P_hat)
    R = P_hat - U_ref @ (U_ref.T @ P_hat)
    ev = np.linalg.eigvalsh(R.T @ R)
    return math.sqrt(max(float(ev.max()), 0.0))

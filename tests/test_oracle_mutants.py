"""Plant mistakes in the oracle (on the CPU) and check that the pins catch
each one: a dropped term, a wrong sign, a transposed operand, a wrong
normalisation, a wrong mean, a skipped step."""
import numpy as np
import pytest

import oracle.powersgd64 as ora

from . import _pins


def _ef_ignores_error(G, E):
    return np.asarray(G, dtype=np.float64)


def _residual_wrong_sign(M, P_hat, Q_bar):
    return np.asarray(M, dtype=np.float64) + np.asarray(P_hat) @ np.asarray(Q_bar).T


def _gs_no_normalise(P, drop_tol=ora.DROP_TOL):
    P = np.asarray(P, dtype=np.float64)
    out = np.zeros_like(P)
    for j in range(P.shape[1]):
        v = P[:, j].copy()
        for k in range(j):
            nk = out[:, k] @ out[:, k]
            if nk:
                v = v - (out[:, k] @ v) / nk * out[:, k]
        out[:, j] = v
    return out


def _gs_skipped(P, drop_tol=ora.DROP_TOL):
    return np.asarray(P, dtype=np.float64).copy()


def _gs_wrong_projection(P, drop_tol=ora.DROP_TOL):
    # projects against the ORIGINAL columns instead of the finished ones
    P = np.asarray(P, dtype=np.float64)
    out = np.zeros_like(P)
    for j in range(P.shape[1]):
        v = P[:, j].copy()
        for k in range(j):
            pk = P[:, k] / np.linalg.norm(P[:, k])
            v = v - (pk @ v) * pk
        out[:, j] = v / np.linalg.norm(v)
    return out


def _mean_wrong_divisor(parts):
    acc = sum(np.asarray(p, dtype=np.float64) for p in parts)
    return acc / max(1, len(parts) - 1) if len(parts) > 1 else acc * 0.5


def _mean_first_worker(parts):
    return np.asarray(parts[0], dtype=np.float64)


def _decompress_transposed(P_hat, Q_bar):
    return (np.asarray(P_hat) @ np.asarray(Q_bar).T).T


def _left_multiply_no_transpose_of_phat(M, P_hat):
    # uses M^T P_bar-like quantity: drops the orthogonalisation's effect by
    # scaling each column back to the norm of M's rows
    return np.asarray(M, dtype=np.float64).T @ (np.asarray(P_hat) * 2.0)


def _momentum_ignores_mom(x, mom, g_hat, lr, beta):
    mom = beta * np.asarray(mom) + np.asarray(g_hat)
    return np.asarray(x) - lr * np.asarray(g_hat), mom


def _momentum_dampened(x, mom, g_hat, lr, beta):
    mom = beta * np.asarray(mom) + (1.0 - beta) * np.asarray(g_hat)
    return np.asarray(x) - lr * mom, mom


def _step_restarts_iterations(G, E, Q, drop_tol=ora.DROP_TOL, iters=1):
    # every iteration starts again from the warm start instead of the last Q_bar
    out = None
    for _ in range(iters):
        out = _ORIG_STEP(G, E, Q, drop_tol, 1)
    return out


_ORIG_STEP = ora.step


def _step_residual_local_q(G, E, Q, drop_tol=ora.DROP_TOL, iters=1):
    # each worker's residual against its own Q_w instead of the mean Q_bar
    o = _ORIG_STEP(G, E, Q, drop_tol, iters)
    o["E_new"] = [o["M"][w] - o["P_hat"] @ o["Qw"][w].T for w in range(len(G))]
    return o


def _step_q_bar_summed(G, E, Q, drop_tol=ora.DROP_TOL, iters=1):
    # Q_bar is the sum over workers, not the mean
    o = _ORIG_STEP(G, E, Q, drop_tol, iters)
    W = len(G)
    o["Q_bar"] = o["Q_bar"] * W
    o["E_new"] = [o["M"][w] - o["P_hat"] @ o["Q_bar"].T for w in range(W)]
    o["G_hat"] = o["P_hat"] @ o["Q_bar"].T
    return o


def _step_residual_from_g(G, E, Q, drop_tol=ora.DROP_TOL, iters=1):
    # the new error memory forgets the old one: E' = G_w - P_hat Q_bar^T
    o = _ORIG_STEP(G, E, Q, drop_tol, iters)
    o["E_new"] = [np.asarray(G[w], dtype=np.float64) - o["G_hat"] for w in range(len(G))]
    return o


def _gs_reversed_order(P, drop_tol=ora.DROP_TOL):
    # orthogonalises the columns last to first
    P = np.asarray(P, dtype=np.float64)
    return _ORIG_GS(P[:, ::-1], drop_tol)[:, ::-1].copy()


_ORIG_GS = ora.gram_schmidt

MUTANTS = {
    "iterations_restart": {"step": _step_restarts_iterations},
    "ef_ignores_error": {"error_feedback_add": _ef_ignores_error},
    "residual_wrong_sign": {"residual": _residual_wrong_sign},
    "gs_no_normalise": {"gram_schmidt": _gs_no_normalise},
    "gs_skipped": {"gram_schmidt": _gs_skipped},
    "gs_wrong_projection": {"gram_schmidt": _gs_wrong_projection},
    "mean_wrong_divisor": {"worker_mean": _mean_wrong_divisor},
    "mean_first_worker": {"worker_mean": _mean_first_worker},
    "decompress_transposed": {"decompress": _decompress_transposed},
    "left_multiply_scaled": {"left_multiply": _left_multiply_no_transpose_of_phat},
    "momentum_ignores_mom": {"momentum_update": _momentum_ignores_mom},
    "momentum_dampened": {"momentum_update": _momentum_dampened},
    "residual_local_q": {"step": _step_residual_local_q},
    "q_bar_summed": {"step": _step_q_bar_summed},
    "residual_from_g": {"step": _step_residual_from_g},
    "gs_reversed_order": {"gram_schmidt": _gs_reversed_order},
}


@pytest.mark.parametrize("name", sorted(MUTANTS))
def test_pins_catch_mutant(name, monkeypatch):
    for attr, fn in MUTANTS[name].items():
        monkeypatch.setattr(ora, attr, fn)
    caught = []
    for check in _pins.ALL_CHECKS:
        try:
            check(ora)
        except Exception as exc:  # assertion or shape error both count
            caught.append((check.__name__, type(exc).__name__))
    assert caught, f"mutant {name} passed every pin"

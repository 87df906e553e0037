"""The smoke check's own logic on the CPU: with a stand-in library that
performs the step exactly (float64, rounded to float32), every comparison
passes; with one that gets the sign of the residual wrong, the check
fails.  The stand-in never runs on a GPU and is not the product."""
import numpy as np
import pytest
import torch

import __graft_entry__ as entry
import oracle.powersgd64 as ora
import rank_gradient_compression_02_b200 as pkg


class _ExactStep:
    flip = False

    def __init__(self, layers, rank, workers, seed=1234):
        self.layers = layers

    def step(self, G, E, q, P, Rc):
        for l in range(len(self.layers)):
            o = ora.step([G[w][l].double().numpy() for w in range(len(G))],
                         [E[w][l].double().numpy() for w in range(len(E))], q[l].double().numpy())
            P[l].copy_(torch.from_numpy(o["P_hat"]))
            q[l].copy_(torch.from_numpy(o["Q_bar"]))
            Rc[l].copy_(torch.from_numpy(o["G_hat"]))
            for w in range(len(E)):
                e = o["E_new"][w]
                E[w][l].copy_(torch.from_numpy(-e if self.flip else e))

    def status(self):
        pass

    def close(self):
        pass


@pytest.mark.parametrize("rank", [2, 16])
def test_smoke_logic_accepts_an_exact_step(monkeypatch, rank):
    monkeypatch.setattr(pkg, "PowerSGD", _ExactStep)
    entry._smoke_case(((96, 130), (40, 64)), rank=rank, workers=3, steps=2, seed=7, device="cpu")


def test_smoke_logic_rejects_a_wrong_residual(monkeypatch):
    class Flipped(_ExactStep):
        flip = True
    monkeypatch.setattr(pkg, "PowerSGD", Flipped)
    with pytest.raises(AssertionError, match="E'"):
        entry._smoke_case(((96, 130),), rank=2, workers=2, steps=2, seed=7, device="cpu")

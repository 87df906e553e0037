"""The bounded waits of the tensor-core second pass (ranks 16 and 32,
16-byte rows).  With the test hook on, its tiles issue no products, so every
wait on them runs out after about a second: the status word reports it once
(PSGD_ERR_TIMEOUT, bit 0x2), the tensor memory is released, and the same context then runs
correct steps again.  No GPU fault and no hang is involved: the wait ends
by its own limit."""
import time

import pytest
import torch

from rank_gradient_compression_02_b200 import PsgdError

from . import _harness as H

pytestmark = pytest.mark.gpu

PSGD_ERR_TIMEOUT = 7


def test_bounded_wait_runs_out_and_the_context_recovers():
    # one 64 x 128 layer at r = 16: a single tile on the tensor-core pass
    wl = H.small_workload([(64, 128)], 16, 2)
    run = H.LibRun(wl)
    L = len(wl.layers)
    Q0 = [run.src.initial_q(l) for l in range(L)]
    E0 = [[torch.zeros(m, n) for (m, n) in wl.layers] for _ in range(wl.workers)]
    run.set_state(E0, Q0)
    run.lib.status()

    run.lib.test_stall_products(True)
    run.fill_grads_host(0)
    t0 = time.monotonic()
    run.run_step()
    torch.cuda.synchronize()
    waited = time.monotonic() - t0
    with pytest.raises(PsgdError) as err:
        run.lib.status()
    assert err.value.code == PSGD_ERR_TIMEOUT
    assert "0x2" in str(err.value)
    assert 0.5 < waited < 60.0            # about one second per wait, bounded
    run.lib.status()                      # reported once, then cleared

    # the same context, hook off, from a fresh state: steps match the oracle
    run.lib.test_stall_products(False)
    run.set_state(E0, Q0)
    orc = H.OracleRun(range(L), {l: [e[l].double().numpy() for e in E0] for l in range(L)},
                      {l: Q0[l].double().numpy() for l in range(L)})
    for t in range(2):
        host = run.fill_grads_host(t)
        run.run_step()
        torch.cuda.synchronize()
        run.lib.status()
        orc.step({l: [host[w][l].double().numpy() for w in range(wl.workers)] for l in range(L)})
        for l in range(L):
            H.assert_close(H.compare_layer(run, orc.last[l], l, H.TOL["f32"]), H.TOL["f32"], f"step {t}")

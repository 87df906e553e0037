"""bench.py's main path on the CPU: the CUDA calls replaced by stand-ins
(events read the host clock, the library is a recorder that launches
nothing), so that the JSON line's assembly (roofline, compute roofline,
lazy variant, end-to-end block, CPU baseline, launch count) is exercised
without a GPU.  The numbers themselves mean nothing here."""
import json
import sys
import time
import types

import pytest
import torch

import bench
from synth import Workload


class _Event:
    def __init__(self, enable_timing=False):
        self.t = None

    def record(self, stream=None):
        self.t = time.perf_counter()

    def elapsed_time(self, other):
        return (other.t - self.t) * 1e3


_FAKE_CUDA = types.SimpleNamespace(
    synchronize=lambda *a, **k: None, mem_get_info=lambda *a: (180e9, 183e9), set_device=lambda *a: None,
    current_stream=lambda *a: None, Event=_Event, is_available=lambda: True, empty_cache=lambda: None)


class _TorchProxy(types.ModuleType):
    def __getattr__(self, name):
        return getattr(torch, name)


class _Recorder:
    """Stands in for PowerSGD: records the calls, computes nothing."""
    created = []

    def __init__(self, layers, rank, workers, grad_dtype="f32", lazy_errors=False, sum_first=False, power_iters=1):
        self.lazy = lazy_errors
        self.calls = []
        self.steps_profiled = 0
        self.profiling = False
        _Recorder.created.append(self)

    def step(self, G, E, Q, P, recon=None):
        self.calls.append("step")
        if self.profiling:
            self.steps_profiled += 1
        # P_hat stand-in with orthonormal columns (the first r unit vectors),
        # so that reports built from it are computable
        for p in P or []:
            p.zero_()
            p[:p.shape[1]].copy_(torch.eye(p.shape[1]))

    def step_host_flat(self, *a, **k):
        self.calls.append("step_host_flat")

    def vec_mean(self, *a, **k):
        self.calls.append("vec_mean")

    def momentum_step(self, *a, **k):
        self.calls.append("momentum_step")

    def materialize_errors(self, *a, **k):
        self.calls.append("materialize_errors")

    def status(self):
        pass

    def profile(self, enable=True):
        self.profiling = enable

    def profile_read(self):
        n = self.steps_profiled
        return [0.3 * n, 0.1 * n, 0.2 * n], n

    def set_global_workers(self, n):
        self.calls.append(("set_global_workers", n))

    def dist_sizes(self):
        return 8, 4

    def dist_p(self, *a, **k):
        self.calls.append("dist_p")
        if self.profiling:
            self.steps_profiled += 1

    def dist_q(self, *a, **k):
        self.calls.append("dist_q")

    def dist_finish(self, *a, **k):
        self.calls.append("dist_finish")

    @property
    def step_launches(self):
        return 3

    def close(self):
        pass


@pytest.fixture
def fake_gpu(monkeypatch):
    import rank_gradient_compression_02_b200 as pkg
    from rank_gradient_compression_02_b200 import build
    proxy = _TorchProxy("torch")
    proxy.cuda = _FAKE_CUDA
    proxy.device = lambda *a, **k: torch.device("cpu")
    monkeypatch.setattr(bench, "torch", proxy)
    monkeypatch.setattr(torch.Tensor, "pin_memory", lambda self: self)
    monkeypatch.setattr(pkg, "PowerSGD", _Recorder)
    monkeypatch.setattr(build, "build", lambda *a, **k: None)
    monkeypatch.setattr(bench, "_pinned_empty", lambda numel, dtype: torch.empty(numel, dtype=dtype))
    wl = Workload(name="tiny", layers=((64, 48), (24, 32)), rank=2, workers=3, steps=3,
                  vectors=(5, 3), momentum=(0.9, 0.1))
    monkeypatch.setattr(bench, "get_workload", lambda key: wl)
    _Recorder.created.clear()
    return wl


def _run(monkeypatch, capsys, *argv):
    monkeypatch.setattr(sys, "argv", ["bench.py", *argv])
    bench.main()
    lines = [ln for ln in capsys.readouterr().out.splitlines() if ln.startswith("{")]
    assert len(lines) == 1
    return json.loads(lines[0])


def test_json_line_eager(fake_gpu, monkeypatch, capsys):
    wl = fake_gpu
    d = _run(monkeypatch, capsys, "--steps", "4", "--warmup", "3", "--oracle-budget", "0.05", "--e2e-steps", "2")
    for key in ("metric", "value", "unit", "n_gpus", "steps", "warmup", "ms_per_step", "higher_is_better",
                "scaling", "vs_baseline", "dtype", "data", "config", "gpu_launches", "roofline", "cpu_baseline",
                "e2e", "clocks", "variants"):
        assert key in d, key
    assert d["n_gpus"] == 1 and d["steps"] == 4 and d["warmup"] == 3 and d["scaling"] == "weak"
    assert d["value"] > 0 and d["config"]["workload"] == "tiny"
    # step + 1-D means + momentum per step
    assert d["gpu_launches"] == 4 * (3 + 1 + 1)
    rl = d["roofline"]
    assert rl["bound"] == "hbm" and rl["kernel"] == "pass_a" and rl["unit"] == "GB/s"
    assert rl["frac"] == pytest.approx(wl.elements * 12 / 0.3e-3 / 1e9 / rl["peak"], abs=1e-4)
    assert rl["per_kernel_ms"] == {"pass_a": 0.3, "pass_b": 0.1, "pass_c": 0.2}
    # the pass-A figure: read G and E, write M, per launch, over its event time
    assert rl["achieved"] == pytest.approx(wl.elements * 12 / 0.3e-3 / 1e9, abs=0.051)   # rounded to 0.1
    assert "step_dram_frac" in rl and "compute" not in rl
    assert d["cpu_baseline"]["kind"] == "oracle" and d["cpu_baseline"]["value"] > 0
    e2e = d["e2e"]
    assert e2e["value"] > 0 and e2e["steps"] == 2
    span = max(o + m * n for o, (m, n) in zip(bench.pack_offsets(wl.layers, 64), wl.layers))
    assert e2e["h2d_bytes_per_step"] == wl.workers * span * 4 + wl.workers * (8 + 4) * 4
    assert e2e["d2h_bytes_per_step"] == sum((m + n) * 2 * 4 for m, n in wl.layers) + (8 + 4) * 4
    lazy = d["variants"]["lazy_errors"]
    assert lazy["value"] > 0 and "step_dram_frac" in lazy
    main_lib, lazy_lib = _Recorder.created
    assert not main_lib.lazy and lazy_lib.lazy
    assert lazy_lib.calls[-1] == "materialize_errors"
    assert main_lib.calls.count("step_host_flat") == 2 + 2


def test_json_line_rank16_reports_compute_roofline(fake_gpu, monkeypatch, capsys):
    d = _run(monkeypatch, capsys, "--rank", "16", "--steps", "3", "--warmup", "3", "--no-cpu-baseline",
             "--no-e2e", "--no-variants")
    assert d["config"]["rank"] == 16
    comp = d["roofline"]["compute"]
    # the toy workload's flops round to zero; the ceilings are the real ones
    assert comp["unit"] == "TFLOP/s" and comp["achieved"] >= 0
    assert comp["fp32_cuda_core_peak"] > 0 and comp["tf32_tensor_peak"] > 0
    assert d["cpu_baseline"] is None and d["e2e"] is None and d["variants"] == {}


def test_reference_arm_line(fake_gpu, monkeypatch, capsys):
    d = _run(monkeypatch, capsys, "--impl", "reference", "--steps", "2", "--warmup", "3")
    assert d["impl"] == "reference" and d["dtype"] == "f64" and d["value"] > 0
    assert d["cpu_baseline"]["value"] == d["value"] and d["cpu_baseline"]["kind"] == "oracle"
    assert d["cpu_baseline"]["sample"].startswith("each step: the whole workload step")
    assert d["e2e"] == {"value": d["value"], "unit": d["unit"], "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}


def test_json_line_distributed_step_one_rank(fake_gpu, monkeypatch, capsys):
    import socket
    import torch.distributed as dist
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    port = s.getsockname()[1]
    s.close()
    for k, v in (("MASTER_ADDR", "127.0.0.1"), ("MASTER_PORT", str(port)), ("RANK", "0"), ("WORLD_SIZE", "1")):
        monkeypatch.setenv(k, v)
    real_init = dist.init_process_group
    monkeypatch.setattr(dist, "init_process_group", lambda backend, **k: real_init("gloo", **k))
    try:
        d = _run(monkeypatch, capsys, "--dist", "--steps", "3", "--warmup", "3", "--no-cpu-baseline",
                 "--e2e-steps", "2")
    finally:
        if dist.is_initialized():
            dist.destroy_process_group()
    assert d["config"]["parallelism"].startswith("dp1")
    # distributed step: + orthogonalisation and Q_bar kernels, 1-D means, momentum
    assert d["gpu_launches"] == 3 * (3 + 2 + 1 + 1)
    assert d["variants"] == {} and d["e2e"]["value"] > 0
    lib = _Recorder.created[0]
    assert ("set_global_workers", fake_gpu.workers) in lib.calls
    i = lib.calls.index("dist_p")
    assert lib.calls[i:i + 3] == ["dist_p", "dist_q", "dist_finish"]


def test_reference_arm_falls_back_to_one_layer_per_step(fake_gpu, monkeypatch, capsys):
    monkeypatch.setattr(bench, "run_reference",
                        lambda *a, _f=bench.run_reference: _f(*a, full_max_elements=0))
    d = _run(monkeypatch, capsys, "--impl", "reference", "--steps", "3", "--warmup", "3")
    assert d["value"] > 0 and d["cpu_baseline"]["sample"].startswith("each step: one layer")


def test_json_line_lazy_mode(fake_gpu, monkeypatch, capsys):
    wl = fake_gpu
    d = _run(monkeypatch, capsys, "--lazy", "--steps", "3", "--warmup", "3", "--no-cpu-baseline", "--no-e2e")
    assert d["config"]["mode"] == "lazy" and d["variants"] == {}
    rl = d["roofline"]
    # lazy: no third pass; the step moves G, E and M once each plus M again in pass B
    assert rl["per_kernel_ms"]["pass_c"] == 0.2   # the recorder's figure; the bytes model ignores it
    assert rl["step_dram_frac"] == pytest.approx(wl.elements * 16 / (d["ms_per_step"] * 1e-3) / 1e9 / rl["peak"],
                                                 rel=1e-3, abs=1e-4)
    assert _Recorder.created[0].lazy


def test_json_line_sum_first_and_power_iterations(fake_gpu, monkeypatch, capsys):
    d = _run(monkeypatch, capsys, "--sum-first", "--iters", "2", "--steps", "3", "--warmup", "3",
             "--no-cpu-baseline", "--no-e2e", "--no-variants")
    assert d["config"]["mode"] == "eager+sumfirst+iters2"
    assert "step_dram_frac" not in d["roofline"]       # the bytes model covers one iteration only


def test_json_line_workloads_and_reports(fake_gpu, monkeypatch, capsys):
    main_wl = fake_gpu
    lstm = Workload(name="tiny_lstm", layers=((40, 26),) * 2, rank=4, workers=4, steps=3)
    sweep = Workload(name="tiny_sweep", layers=((32, 32),) * 3, rank=1, workers=2, steps=4, rotate=0.05,
                     ranks=(1, 2, 16))
    table = {"m": main_wl, "l": lstm, "s": sweep}
    monkeypatch.setattr(bench, "get_workload", lambda key: table[key])
    d = _run(monkeypatch, capsys, "--config", "m", "--steps", "3", "--warmup", "3", "--no-cpu-baseline",
             "--no-e2e", "--no-variants", "--workloads", "m,l,s", "--workload-steps", "2")
    wls = d["workloads"]
    # the main workload is not repeated among the sub-lines
    assert set(wls) == {"tiny_lstm", "tiny_sweep"}
    lw = wls["tiny_lstm"]
    for key in ("ms_per_step", "value", "step_dram_frac", "step_algorithmic_frac", "per_kernel_ms", "lazy_errors",
                "compression"):
        assert key in lw, key
    assert lw["rank"] == 4 and lw["compression"]["ratio"] == round(2 * 40 * 26 / (4 * 2 * 66), 2)
    sw = wls["tiny_sweep"]
    assert set(sw["by_rank"]) == {"1", "2", "16"}
    for r, line in sw["by_rank"].items():
        assert line["rank"] == int(r) and line["value"] > 0 and "compression" in line
    se = sw["subspace_error"]["by_rank"]
    assert set(se) == {"1", "2", "16"} and se["1"]["steps"] == 4
    assert se["2"]["status"].startswith("checked against the oracle") and se["16"]["status"].startswith("reported")
    for v in se.values():
        assert 0.0 <= v["sin_theta_max"] <= 1.0 + 1e-12
    assert d["compression"]["ratio"] == round((64 * 48 + 24 * 32) / (2 * (64 + 48 + 24 + 32)), 2)


def test_e2e_releases_device_gradients_when_staging_does_not_fit(fake_gpu, monkeypatch, capsys):
    monkeypatch.setattr(_FAKE_CUDA, "mem_get_info", lambda *a: (1e3, 183e9))
    real_need = bench.device_bytes_needed
    monkeypatch.setattr(bench, "device_bytes_needed", lambda *a: 0)
    d = _run(monkeypatch, capsys, "--steps", "2", "--warmup", "3", "--no-cpu-baseline", "--no-variants",
             "--e2e-steps", "2", "--no-workloads")
    assert d["e2e"]["value"] > 0 and "released" in d["e2e"]["note"]
    assert real_need is not None


def test_compression_report_of_the_workloads():
    from synth import C1, C3
    c1 = bench.compression_report(C1, 2)
    smpn = sum(m + n for m, n in C1.layers)
    assert c1["ratio"] == round(11_162_624 / (2 * smpn), 2)
    assert c1["factor_bytes_per_worker"] == 4 * 2 * smpn and c1["gradient_bytes_per_worker"] == 4 * 11_162_624
    c3 = bench.compression_report(C3, 4)
    # 24 blocks x (16384 + 8192 + 20480 + 20480) rows + columns
    assert c3["ratio"] == round(4_831_838_208 / (4 * 24 * 65536), 2) and c3["gradient_bytes_per_worker"] == \
        2 * 4_831_838_208
    assert c3["dist_partial_bytes_per_rank"] == 8 * 4 * 24 * 65536


def test_sin_theta_max_known_angles():
    import numpy as np
    # span(e0, e1) against span(e0, cos t e1 + sin t e2): largest angle t
    for t in (1e-9, 1e-3, 0.3, 1.2):
        U = np.eye(5)[:, :2]
        P = np.zeros((5, 2))
        P[0, 0] = 1.0
        P[1, 1], P[2, 1] = np.cos(t), np.sin(t)
        assert abs(bench.sin_theta_max(U, P) - np.sin(t)) < 1e-12 * max(1.0, t) + 1e-15
    # invariant under a rotation of either basis
    rng = np.random.default_rng(3)
    U = np.linalg.qr(rng.standard_normal((9, 3)))[0]
    P = np.linalg.qr(rng.standard_normal((9, 3)))[0]
    Rt = np.linalg.qr(rng.standard_normal((3, 3)))[0]
    assert abs(bench.sin_theta_max(U, P) - bench.sin_theta_max(U @ Rt, P @ Rt.T)) < 1e-12

"""Host-side logic of bench.py that needs no GPU: the kernel-source hash that
decides whether committed ncu traffic still belongs to the kernels, the
committed traffic record itself, the compute roofline arithmetic and the
bounded oracle sample behind the CPU baseline."""
import json
import os
import shutil

import pytest

import bench


def test_code_tokens_strip_comments_keep_strings():
    src = 'int a = 1; // note\n/* block\n comment */ const char* s = "//kept"; char c = \'\\\'\';\n'
    assert bench._code_tokens(src) == 'int a = 1; const char* s = "//kept"; char c = \'\\\'\';'


def test_hash_ignores_comments_and_layout_but_not_code(tmp_path):
    csrc = os.path.join(bench.ROOT, "rank_gradient_compression_02_b200", "csrc")
    copy = tmp_path / "csrc"
    shutil.copytree(csrc, copy)
    base = bench._kernel_source_hash(str(copy))
    assert base == bench._kernel_source_hash()
    k = copy / "kernels.cuh"
    text = k.read_text()
    k.write_text("// an added comment\n" + text.replace("\n", "\n  ", 3))
    assert bench._kernel_source_hash(str(copy)) == base
    k.write_text(text.replace("kMmaRows = 16", "kMmaRows = 17", 1))
    assert bench._kernel_source_hash(str(copy)) != base


def test_committed_traffic_belongs_to_the_current_kernels():
    # the DRAM traffic the benchmark reports comes from ncu captures of
    # these very sources; a kernel change without a new capture would make
    # the benchmark report traffic = null
    with open(os.path.join(bench.ROOT, "profiles", "traffic.json")) as f:
        recs = json.load(f)
    # the first pass reads G and E and writes M: 10 bytes per bf16 worker
    # element on the transformer set (19.33 G of them), 12 per fp32 element on
    # the ResNet-18 set (178.6 M); ncu counts within a few percent of that
    for key, elems, per in (("transformer24_bf16_r4_w4/eager", 19_327_352_832, 10),
                            ("resnet18_r2_w16/eager", 178_601_984, 12)):
        rec = recs[key]
        assert rec["kernel_hash"] == bench._kernel_source_hash(), key
        workload, mode = key.split("/")
        assert bench._traffic_record(workload, mode) == rec["dram_bytes_per_launch"]
        alg = elems * per
        assert 0.9 * alg < rec["dram_bytes_per_launch"] < 1.05 * alg, key


def test_compute_roofline_arithmetic():
    # 1e9 worker elements, r = 32, both passes 1 ms: 2 * 32 * 1e9 flop per
    # pass -> 128 GFLOP in 2 ms = 64 TFLOP/s; fp32 ceiling at 2 GHz
    # 148 * 128 * 2 * 2e9 = 75.8 TFLOP/s; tf32 ceiling 1600 * 1.1 / 2.25
    c = bench.compute_roofline(10**9, 32, 1.0, 1.0, 2000.0, 1600.0)
    assert abs(c["achieved"] - 64.0) < 1e-6
    assert abs(c["fp32_cuda_core_peak"] - 75.8) < 0.05
    assert abs(c["tf32_tensor_peak"] - 782.2) < 0.05
    assert abs(c["fp32_frac"] - 64.0 / 75.776) < 1e-3
    # sum-first: the first pass multiplies each matrix element once, not once per worker
    s = bench.compute_roofline(10**9, 32, 1.0, 1.0, 2000.0, 1600.0, sum_first=True, workers=8)
    assert abs(s["achieved"] - (2 * 32 * 1e9 / 8 + 2 * 32 * 1e9) / 2e-3 / 1e12) < 1e-6


def test_oracle_sample_runs_later_steps_with_state_carried():
    from tests import _harness as H
    wl = H.small_workload([(24, 20), (9, 7)], 2, 2)
    rate, elements, seconds, threads, text = bench.oracle_sample(wl, 2, budget_s=0.05)
    per_step = wl.workers * (24 * 20 + 9 * 7)
    # whole layers only: full steps plus possibly the first layer of the next
    assert elements > per_step and elements % per_step in (0, wl.workers * 24 * 20)
    assert rate > 0 and seconds >= 0.05 and threads >= 1
    assert int(text.split(" over ")[1].split(" ")[0]) >= 2
    # the carried state is bounded: with no room for it, only the first step runs
    _, elements1, _, _, text1 = bench.oracle_sample(wl, 2, budget_s=10.0, carry_bytes=0)
    assert elements1 == per_step and " over 1 step(s) " in text1


def test_roofline_block_picks_the_dominant_pass():
    from synth import Workload
    wl = Workload(name="t", layers=((1000, 1000),), rank=2, workers=4, steps=1)
    el = wl.elements
    # pass C the slowest: its bytes (read M, write E') over its time
    rl = bench.roofline_block(wl, 2, "eager", [1.0, 0.5, 2.0], 2, 2.0, None)
    assert rl["kernel"] == "pass_c" and rl["traffic"] is None
    assert rl["achieved"] == pytest.approx(el * 8 / 1e-3 / 1e9, abs=0.051)
    assert rl["step_dram_frac"] == pytest.approx(el * 24 / 2e-3 / 1e9 / rl["peak"], abs=1e-4)
    assert rl["step_algorithmic_frac"] == pytest.approx(el * 12 / 2e-3 / 1e9 / rl["peak"], abs=1e-4)
    assert "compute" not in rl
    # lazy mode moves 16 bytes per worker element; bf16 gradients 2 fewer
    rl = bench.roofline_block(wl, 2, "lazy", [1.0, 0.5, 0.0], 1, 1.0, None, lazy=True)
    assert rl["kernel"] == "pass_a" and rl["step_dram_frac"] == pytest.approx(el * 16 / 1e-3 / 1e9 / rl["peak"],
                                                                              abs=1e-4)
    from dataclasses import replace
    rl = bench.roofline_block(replace(wl, grad_dtype="bf16"), 2, "eager", [1.0, 0.5, 0.5], 1, 2.0, None)
    assert rl["achieved"] == pytest.approx(el * 10 / 1e-3 / 1e9, abs=0.051)
    # ranks 16 and 32 add the compute side; power iterations drop the bytes model
    rl = bench.roofline_block(wl, 16, "eager", [1.0, 0.5, 0.5], 1, 2.0, {"sm_mhz": 1965.0}, iters=2)
    assert "compute" in rl and "step_dram_frac" not in rl

"""The library's tile geometry, checked in its own host code on the CPU:
tests/native/geometry_check.cu includes csrc/psgd.cu unchanged and checks,
for every shape, rank and worker count the GPU tests and the full-size
workloads use, that the lane
width divides the row, chunks and row blocks cover the matrix with none
empty, the tensor-core tiles are whole 16-row groups, the rows buffer and
the widest chunk fit, and each pass's shared memory fits in 227 KB and
leaves room for the CTAs per SM its launch bounds aim at; and that the
layer groups of the host-buffer steps are contiguous, cover every layer and
tile once, number at most min(L, 8), and stay within one layer of an equal
share."""
import os
import shutil
import subprocess

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def test_tile_geometry_invariants(tmp_path):
    nvcc = shutil.which("nvcc") or "/usr/local/cuda/bin/nvcc"
    if not os.path.exists(nvcc):
        pytest.skip("no nvcc")
    exe = tmp_path / "geometry_check"
    subprocess.run([nvcc, "-std=c++17", "-gencode", "arch=compute_100a,code=sm_100a", "-O1",
                    "-I", os.path.join(ROOT, "include"),
                    "-I", os.path.join(ROOT, "rank_gradient_compression_02_b200", "csrc"),
                    "-o", str(exe), os.path.join(ROOT, "tests", "native", "geometry_check.cu")],
                   check=True, capture_output=True, timeout=900)
    out = subprocess.run([str(exe)], capture_output=True, text=True, timeout=120)
    assert out.returncode == 0, out.stdout + out.stderr
    assert out.stdout.strip().endswith("0 failures"), out.stdout

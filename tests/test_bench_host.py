"""Host-side logic of bench.py that needs no GPU: the kernel-source hash that
decides whether committed ncu traffic still belongs to the kernels, and the
committed traffic record itself."""
import json
import os
import shutil

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
    # the DRAM traffic the benchmark reports comes from an ncu capture of
    # these very sources; a kernel change without a new capture would make
    # the benchmark report traffic = null
    with open(os.path.join(bench.ROOT, "profiles", "traffic.json")) as f:
        rec = json.load(f)["resnet18_r2_w16/eager"]
    assert rec["kernel_hash"] == bench._kernel_source_hash()
    assert bench._traffic_record("resnet18_r2_w16", "eager") == rec["dram_bytes_per_launch"]
    # the first pass moves read G, read E, write M: 12 bytes per worker
    # element, 178,601,984 worker elements; ncu counts a little less (lines
    # still dirty in L2 at the end of the kernel)
    alg = 178_601_984 * 12
    assert 0.9 * alg < rec["dram_bytes_per_launch"] < 1.05 * alg

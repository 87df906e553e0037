"""The C-ABI library loads and exports every entry point the header
declares; argument checks that need no device work on the CPU."""
import ctypes
import os
import re

import pytest

from rank_gradient_compression_02_b200 import _lib

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "psgd.h")


def declared_functions():
    text = open(HEADER).read()
    return sorted(set(re.findall(r"PSGD_API\s+[\w\s\*]*?\b(psgd_\w+)\s*\(", text)))


@pytest.fixture(scope="module")
def lib():
    from rank_gradient_compression_02_b200 import build
    build.build()   # a no-op when libpsgd.so is newer than its sources
    return _lib.load()


def test_header_declares_the_api():
    names = declared_functions()
    for must in ("psgd_create", "psgd_step", "psgd_destroy", "psgd_momentum_step", "psgd_vec_mean",
                 "psgd_status", "psgd_last_error", "psgd_init_q", "psgd_materialize_errors", "psgd_step_host"):
        assert must in names


def test_every_declared_symbol_is_exported(lib):
    for name in declared_functions():
        assert hasattr(lib, name), name
        assert name in _lib._SIGS, f"{name} has no binding signature"


def test_binding_covers_only_declared_symbols():
    assert set(_lib._SIGS) <= set(declared_functions())


@pytest.mark.parametrize("layers,rank,workers,dtype,flags", [
    ([(4, 3)], 0, 1, 0, 0),        # rank 0
    ([(64, 64)], 33, 1, 0, 0),     # rank > 32
    ([(4, 3)], 4, 1, 0, 0),        # rank > min(m, n)
    ([(4, 3)], 1, 0, 0, 0),        # no workers
    ([(4, 3)], 1, 257, 0, 0),      # too many workers
    ([(4, 3)], 1, 1, 7, 0),        # bad dtype
    ([(4, 3)], 1, 1, 0, 8),        # unknown flag
    ([(0, 3)], 1, 1, 0, 0),        # empty matrix
])
def test_create_rejects_bad_arguments_without_touching_the_device(lib, layers, rank, workers, dtype, flags):
    arr = (_lib._Layer * len(layers))(*[_lib._Layer(m, n) for m, n in layers])
    h = ctypes.c_void_p()
    rc = lib.psgd_create(ctypes.byref(h), arr, len(layers), rank, workers, 1, dtype, flags)
    assert rc == _lib.PSGD_ERR_ARG
    assert not h.value
    assert lib.psgd_last_error(None).decode()


def test_null_context_is_an_argument_error(lib):
    assert lib.psgd_step(None, None, None, None, None, None, None) == _lib.PSGD_ERR_ARG
    assert lib.psgd_status(None) == _lib.PSGD_ERR_ARG
    assert lib.psgd_step_launches(None) == -1
    lib.psgd_destroy(None)


def test_missing_library_is_an_error_not_a_fallback(tmp_path):
    with pytest.raises(ImportError, match="libpsgd.so not found"):
        _lib.load(str(tmp_path / "libpsgd.so"))


def test_binding_has_no_cpu_or_oracle_path():
    # the product path never reaches the oracle or a host implementation
    pkg = os.path.join(ROOT, "rank_gradient_compression_02_b200")
    for name in os.listdir(pkg):
        if name.endswith(".py"):
            text = open(os.path.join(pkg, name)).read()
            assert "oracle" not in text, name
            assert "numpy" not in text, name


_C_CALLER = r"""
#include <stdio.h>
#include <string.h>
#include "psgd.h"

int main(void) {
    psgd_layer layers[2] = {{64, 48}, {10, 512}};
    psgd_ctx *ctx = (psgd_ctx *)1;
    /* rank 0, rank above min(m, n), 0 workers, unknown flag: refused before any device work */
    if (psgd_create(&ctx, layers, 2, 0, 4, 7u, PSGD_F32, 0u) != PSGD_ERR_ARG || ctx != NULL) return 1;
    if (psgd_create(&ctx, layers, 2, 11, 4, 7u, PSGD_F32, 0u) != PSGD_ERR_ARG) return 2;
    if (psgd_create(&ctx, layers, 2, 2, 0, 7u, PSGD_BF16, 0u) != PSGD_ERR_ARG) return 3;
    if (psgd_create(&ctx, layers, 2, 2, 4, 7u, PSGD_F32, 8u) != PSGD_ERR_ARG) return 4;
    if (strlen(psgd_last_error(NULL)) == 0) return 5;
    if (psgd_step(NULL, NULL, NULL, NULL, NULL, NULL, NULL) != PSGD_ERR_ARG) return 6;
    if (psgd_status(NULL) != PSGD_ERR_ARG) return 7;
    if (psgd_step_launches(NULL) != -1) return 8;
    psgd_destroy(NULL);
    printf("ok\n");
    return 0;
}
"""


def test_header_is_plain_c_and_links(lib, tmp_path):
    import shutil
    import subprocess
    gcc = shutil.which("gcc")
    if gcc is None:
        pytest.skip("no gcc")
    src = tmp_path / "caller.c"
    src.write_text(_C_CALLER)
    exe = tmp_path / "caller"
    libdir = os.path.dirname(_lib.LIB_PATH)
    subprocess.run([gcc, "-std=c99", "-Wall", "-Wextra", "-Werror", "-pedantic", "-I", os.path.dirname(HEADER),
                    str(src), "-o", str(exe), "-L", libdir, "-lpsgd", f"-Wl,-rpath,{libdir}"], check=True)
    out = subprocess.run([str(exe)], capture_output=True, text=True, timeout=120)
    assert out.returncode == 0 and out.stdout.strip() == "ok", (out.returncode, out.stdout, out.stderr)
    # and as C++: the extern "C" block keeps the names unmangled
    gxx = shutil.which("g++")
    if gxx is not None:
        subprocess.run([gxx, "-std=c++11", "-Wall", "-Werror", "-fsyntax-only", "-x", "c++", "-I",
                        os.path.dirname(HEADER), str(src)], check=True)


def test_static_step_checks_need_no_device(lib):
    # every check of the allocation-free step happens before device work;
    # the pointer values are never dereferenced
    W = 2
    ok = (ctypes.c_void_p * W)(*([16] * W))
    odd = (ctypes.c_void_p * W)(16, 20)
    null = (ctypes.c_void_p * W)(16, None)
    step = lib.psgd_step_static
    assert step(8192, 8192, 32, W, 0, ok, ok, 16, None, None, None) == _lib.PSGD_ERR_ARG   # beyond the scratch
    assert "static scratch" in lib.psgd_last_error(None).decode()
    assert step(64, 48, 49, W, 0, ok, ok, 16, None, None, None) == _lib.PSGD_ERR_ARG       # rank > min(m, n)
    assert step(64, 48, 2, 0, 0, ok, ok, 16, None, None, None) == _lib.PSGD_ERR_ARG        # no workers
    assert step(64, 48, 2, W, 2, ok, ok, 16, None, None, None) == _lib.PSGD_ERR_ARG        # bad dtype
    assert step(64, 48, 2, W, 0, null, ok, 16, None, None, None) == _lib.PSGD_ERR_ARG      # null gradient
    assert step(64, 48, 2, W, 0, odd, ok, 16, None, None, None) == _lib.PSGD_ERR_ALIGN     # 4-byte offset
    assert step(64, 48, 2, W, 0, ok, ok, 24, None, None, None) == _lib.PSGD_ERR_ALIGN      # q misaligned


def test_readme_c_example_compiles(tmp_path):
    import shutil
    import subprocess
    gcc = shutil.which("gcc")
    if gcc is None:
        pytest.skip("no gcc")
    text = open(os.path.join(ROOT, "README.md")).read()
    block = re.search(r"```c\n(.*?)```", text, re.S).group(1)
    body = "\n".join(ln for ln in block.splitlines() if not ln.startswith("#include"))
    src = tmp_path / "example.c"
    src.write_text('#include <stdio.h>\n#include "psgd.h"\n'
                   "void example(float *const *q, void *stream, const void *const *grads, float *const *errors,\n"
                   "             float *const *p_hat, float *const *recon, float *const *params,\n"
                   "             float *const *mom) {\n" + body + "\n}\n")
    subprocess.run([gcc, "-std=c99", "-Wall", "-Wextra", "-Werror", "-pedantic", "-fsyntax-only", "-I",
                    os.path.dirname(HEADER), str(src)], check=True)


def test_binding_constants_match_the_header():
    text = open(HEADER).read()
    values = {k: int(v) for k, v in re.findall(r"\b(PSGD_(?:OK|ERR_\w+|F32|BF16|FLAG_\w+))\s*=\s*(\d+)u?\b", text)}
    assert values["PSGD_OK"] == _lib.PSGD_OK
    for name in ("ARG", "ALIGN", "CUDA", "OOM", "STATE", "DEVICE"):
        assert values[f"PSGD_ERR_{name}"] == getattr(_lib, f"PSGD_ERR_{name}"), name
        assert _lib._ERR_NAMES[values[f"PSGD_ERR_{name}"]] == f"PSGD_ERR_{name}"
    assert values["PSGD_F32"] == _lib.PSGD_F32 and values["PSGD_BF16"] == _lib.PSGD_BF16
    for name in ("LAZY_ERRORS", "SUM_FIRST", "NO_WARM_START"):
        assert values[f"PSGD_FLAG_{name}"] == getattr(_lib, f"FLAG_{name}"), name
    m = re.search(r"#define PSGD_STATIC_SCRATCH_BYTES \((\d+)u << (\d+)\)", text)
    assert m and int(m.group(1)) << int(m.group(2)) == 16 << 20

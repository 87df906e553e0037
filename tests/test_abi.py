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
    if not os.path.exists(_lib.LIB_PATH):
        from rank_gradient_compression_02_b200 import build
        build.build()
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

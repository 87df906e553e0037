"""ctypes binding of libpsgd.so (the C ABI in include/psgd.h).

Argument marshalling only: tensors become device pointers, lists become
pointer arrays, the current torch stream becomes a cudaStream_t.  Every
step of the computation runs in the library's kernels; there is no fallback
of any kind, and a missing library is an error.
"""
from __future__ import annotations

import ctypes
import os
from typing import List, Optional, Sequence

import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libpsgd.so")

PSGD_OK, PSGD_ERR_ARG, PSGD_ERR_ALIGN, PSGD_ERR_CUDA, PSGD_ERR_OOM, PSGD_ERR_STATE, PSGD_ERR_DEVICE = range(7)
PSGD_F32, PSGD_BF16 = 0, 1
FLAG_LAZY_ERRORS = 1
FLAG_SUM_FIRST = 2
FLAG_NO_WARM_START = 4

_ERR_NAMES = {1: "PSGD_ERR_ARG", 2: "PSGD_ERR_ALIGN", 3: "PSGD_ERR_CUDA", 4: "PSGD_ERR_OOM",
              5: "PSGD_ERR_STATE", 6: "PSGD_ERR_DEVICE"}


class PsgdError(RuntimeError):
    def __init__(self, code: int, msg: str):
        super().__init__(f"{_ERR_NAMES.get(code, code)}: {msg}")
        self.code = code


class _Layer(ctypes.Structure):
    _fields_ = [("m", ctypes.c_int64), ("n", ctypes.c_int64)]


_P = ctypes.c_void_p
_PP = ctypes.POINTER(ctypes.c_void_p)

_SIGS = {
    "psgd_create": (ctypes.c_int, [ctypes.POINTER(_P), ctypes.POINTER(_Layer), ctypes.c_int, ctypes.c_int,
                                   ctypes.c_int, ctypes.c_uint64, ctypes.c_int, ctypes.c_uint]),
    "psgd_destroy": (None, [_P]),
    "psgd_init_q": (ctypes.c_int, [_P, _PP, _P]),
    "psgd_step": (ctypes.c_int, [_P, _PP, _PP, _PP, _PP, _PP, _P]),
    "psgd_step_host": (ctypes.c_int, [_P, _PP, _PP, _PP, _PP, _PP, _P]),
    "psgd_step_host_flat": (ctypes.c_int, [_P, _PP, ctypes.POINTER(ctypes.c_int64), _PP, _PP, _PP, _PP, _P]),
    "psgd_materialize_errors": (ctypes.c_int, [_P, _PP, _P]),
    "psgd_momentum_step": (ctypes.c_int, [_P, _PP, _PP, ctypes.c_float, ctypes.c_float, _P]),
    "psgd_vec_mean": (ctypes.c_int, [_P, _PP, _PP, ctypes.POINTER(ctypes.c_int64), ctypes.c_int, _PP, _PP,
                                     ctypes.c_float, ctypes.c_float, _P]),
    "psgd_status": (ctypes.c_int, [_P]),
    "psgd_workspace_bytes": (ctypes.c_int, [_P, ctypes.POINTER(ctypes.c_size_t)]),
    "psgd_step_launches": (ctypes.c_int, [_P]),
    "psgd_last_error": (ctypes.c_char_p, [_P]),
    "psgd_step_static": (ctypes.c_int, [ctypes.c_int64, ctypes.c_int64, ctypes.c_int, ctypes.c_int, ctypes.c_int,
                                        _PP, _PP, _P, _P, _P, _P]),
    "psgd_set_power_iters": (ctypes.c_int, [_P, ctypes.c_int]),
    "psgd_set_global_workers": (ctypes.c_int, [_P, ctypes.c_int]),
    "psgd_dist_sizes": (ctypes.c_int, [_P, ctypes.POINTER(ctypes.c_size_t), ctypes.POINTER(ctypes.c_size_t)]),
    "psgd_dist_p": (ctypes.c_int, [_P, _PP, _PP, _PP, _PP, _PP, _P, _P]),
    "psgd_dist_q": (ctypes.c_int, [_P, _P, _P, _P]),
    "psgd_dist_finish": (ctypes.c_int, [_P, _P, _P]),
    "psgd_set_svd_refresh": (ctypes.c_int, [_P, ctypes.c_int, ctypes.c_int]),
    "psgd_profile_enable": (ctypes.c_int, [_P, ctypes.c_int]),
    "psgd_profile_read": (ctypes.c_int, [_P, ctypes.POINTER(ctypes.c_double), ctypes.POINTER(ctypes.c_int)]),
}

_lib = None


def load(path: Optional[str] = None) -> ctypes.CDLL:
    """Load libpsgd.so (built in-tree by rank_gradient_compression_02_b200.build)."""
    global _lib
    if _lib is not None and path is None:
        return _lib
    p = path or LIB_PATH
    if not os.path.exists(p):
        raise ImportError(f"libpsgd.so not found at {p}; build it with "
                          f"'python -m rank_gradient_compression_02_b200.build'")
    lib = ctypes.CDLL(p)
    for name, (res, args) in _SIGS.items():
        fn = getattr(lib, name)
        fn.restype = res
        fn.argtypes = args
    if path is None:
        _lib = lib
    return lib


def _ptrs(values: Sequence) -> ctypes.Array:
    arr = (ctypes.c_void_p * max(1, len(values)))()
    for i, v in enumerate(values):
        if v is None:
            arr[i] = None
        elif isinstance(v, int):
            arr[i] = v
        else:
            arr[i] = v.data_ptr()
    return arr


def _stream_handle(stream) -> int:
    if stream is None:
        stream = torch.cuda.current_stream()
    if isinstance(stream, int):
        return stream
    return stream.cuda_stream


def step_static(m: int, n: int, rank: int, grads, errors, q, p_hat=None, recon=None, grad_dtype: str = "f32",
                stream=None):
    """Allocation-free one-layer step (psgd_step_static): grads[w], errors[w]
    per worker; every scratch buffer lives in the library's static device
    array.  For callers that cannot allocate device memory."""
    lib = load()
    W = len(grads)
    rc = lib.psgd_step_static(int(m), int(n), int(rank), W, PSGD_BF16 if grad_dtype == "bf16" else PSGD_F32,
                              _ptrs(grads), _ptrs(errors), q.data_ptr(),
                              p_hat.data_ptr() if p_hat is not None else None,
                              recon.data_ptr() if recon is not None else None, _stream_handle(stream))
    if rc:
        raise PsgdError(rc, lib.psgd_last_error(None).decode())


class PowerSGD:
    """One library context: fixed layer shapes, rank, worker count.

    Buffers are torch tensors (or raw device addresses as ints).  grads and
    errors are indexed [w][l]; q, p_hat, recon per layer.
    """

    def __init__(self, layers: Sequence[Sequence[int]], rank: int, workers: int, seed: int = 1234,
                 grad_dtype: str = "f32", lazy_errors: bool = False, sum_first: bool = False,
                 power_iters: int = 1, warm_start: bool = True, svd_every: int = 0, svd_iters: int = 8):
        self.lib = load()
        self.layers = [(int(m), int(n)) for m, n in layers]
        self.rank = int(rank)
        self.workers = int(workers)
        self.grad_dtype = grad_dtype
        arr = (_Layer * max(1, len(self.layers)))(*[_Layer(m, n) for m, n in self.layers])
        flags = (FLAG_LAZY_ERRORS if lazy_errors else 0) | (FLAG_SUM_FIRST if sum_first else 0) | \
            (0 if warm_start else FLAG_NO_WARM_START)
        h = _P()
        rc = self.lib.psgd_create(ctypes.byref(h), arr, len(self.layers), self.rank, self.workers,
                                  ctypes.c_uint64(seed & (2**64 - 1)),
                                  PSGD_BF16 if grad_dtype == "bf16" else PSGD_F32, flags)
        if rc:
            raise PsgdError(rc, self.lib.psgd_last_error(None).decode())
        self._h = h
        if power_iters != 1:
            self._check(self.lib.psgd_set_power_iters(self._h, int(power_iters)))
        if svd_every:
            self._check(self.lib.psgd_set_svd_refresh(self._h, int(svd_every), int(svd_iters)))

    # -- helpers
    def _check(self, rc: int):
        if rc:
            raise PsgdError(rc, self.lib.psgd_last_error(self._h).decode())

    def _wl(self, per_worker: Sequence[Sequence]) -> ctypes.Array:
        flat: List = []
        for w in range(self.workers):
            flat.extend(per_worker[w])
        return _ptrs(flat)

    # -- API
    def init_q(self, q: Sequence, stream=None):
        self._check(self.lib.psgd_init_q(self._h, _ptrs(q), _stream_handle(stream)))

    def step(self, grads, errors, q, p_hat=None, recon=None, stream=None):
        self._check(self.lib.psgd_step(self._h, self._wl(grads), self._wl(errors), _ptrs(q),
                                       _ptrs(p_hat) if p_hat is not None else None,
                                       _ptrs(recon) if recon is not None else None,
                                       _stream_handle(stream)))

    def step_host(self, grads_host, errors, q, p_hat_host=None, q_host=None, stream=None):
        self._check(self.lib.psgd_step_host(self._h, self._wl(grads_host), self._wl(errors), _ptrs(q),
                                            _ptrs(p_hat_host) if p_hat_host is not None else None,
                                            _ptrs(q_host) if q_host is not None else None,
                                            _stream_handle(stream)))

    def step_host_flat(self, grads_host, layer_offsets, errors, q, p_hat_host=None, q_host=None, stream=None):
        """grads_host[w]: one host buffer per worker holding every layer,
        layer l starting at element layer_offsets[l]."""
        offs = (ctypes.c_int64 * max(1, len(layer_offsets)))(*[int(o) for o in layer_offsets])
        self._check(self.lib.psgd_step_host_flat(self._h, _ptrs(grads_host), offs, self._wl(errors), _ptrs(q),
                                                 _ptrs(p_hat_host) if p_hat_host is not None else None,
                                                 _ptrs(q_host) if q_host is not None else None,
                                                 _stream_handle(stream)))

    def materialize_errors(self, errors, stream=None):
        self._check(self.lib.psgd_materialize_errors(self._h, self._wl(errors), _stream_handle(stream)))

    def momentum_step(self, params, mom, lr: float, beta: float, stream=None):
        self._check(self.lib.psgd_momentum_step(self._h, _ptrs(params), _ptrs(mom), lr, beta,
                                                _stream_handle(stream)))

    def vec_mean(self, vecs, out, params=None, mom=None, lr: float = 0.0, beta: float = 0.0, stream=None):
        """vecs[w][k] -> out[k] = mean over workers (+ momentum if params, mom)."""
        K = len(out)
        lens = (ctypes.c_int64 * max(1, K))(*[int(t.numel()) for t in out])
        self._check(self.lib.psgd_vec_mean(self._h, self._wl(vecs), _ptrs(out), lens, K,
                                           _ptrs(params) if params is not None else None,
                                           _ptrs(mom) if mom is not None else None, lr, beta,
                                           _stream_handle(stream)))

    # -- distributed step (the caller all-reduces p_send and q_send, SUM)
    def set_global_workers(self, total: int):
        self._check(self.lib.psgd_set_global_workers(self._h, int(total)))

    def dist_sizes(self):
        pe, qe = ctypes.c_size_t(), ctypes.c_size_t()
        self._check(self.lib.psgd_dist_sizes(self._h, ctypes.byref(pe), ctypes.byref(qe)))
        return int(pe.value), int(qe.value)

    def dist_p(self, grads, errors, q, p_send, p_hat=None, recon=None, stream=None):
        self._check(self.lib.psgd_dist_p(self._h, self._wl(grads), self._wl(errors), _ptrs(q),
                                         _ptrs(p_hat) if p_hat is not None else None,
                                         _ptrs(recon) if recon is not None else None,
                                         p_send.data_ptr(), _stream_handle(stream)))

    def dist_q(self, p_sum, q_send, stream=None):
        self._check(self.lib.psgd_dist_q(self._h, p_sum.data_ptr(), q_send.data_ptr(), _stream_handle(stream)))

    def dist_finish(self, q_sum, stream=None):
        self._check(self.lib.psgd_dist_finish(self._h, q_sum.data_ptr(), _stream_handle(stream)))

    def profile(self, enable: bool = True):
        self._check(self.lib.psgd_profile_enable(self._h, 1 if enable else 0))

    def profile_read(self):
        """-> ([ms pass A, ms pass B, ms pass C] summed, steps recorded)."""
        ms = (ctypes.c_double * 3)()
        n = ctypes.c_int()
        self._check(self.lib.psgd_profile_read(self._h, ms, ctypes.byref(n)))
        return [ms[0], ms[1], ms[2]], int(n.value)

    def status(self):
        self._check(self.lib.psgd_status(self._h))

    @property
    def workspace_bytes(self) -> int:
        v = ctypes.c_size_t()
        self._check(self.lib.psgd_workspace_bytes(self._h, ctypes.byref(v)))
        return int(v.value)

    @property
    def step_launches(self) -> int:
        return int(self.lib.psgd_step_launches(self._h))

    def close(self):
        if getattr(self, "_h", None):
            self.lib.psgd_destroy(self._h)
            self._h = None

    def __del__(self):
        try:
            self.close()
        except Exception:
            pass

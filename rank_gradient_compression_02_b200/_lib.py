"""ctypes binding of libpsgd.so (the C ABI in include/psgd.h).

Argument marshalling only: tensors become device pointers, lists become
pointer arrays, the current torch stream becomes a cudaStream_t.  Before an
address crosses the ABI, each tensor's side (device or host), dtype,
contiguity and size and each list's length are checked (again only when a
buffer address of the call changes).  Every step of the computation runs in the
library's kernels; there is no fallback of any kind, and a missing library
is an error.
"""
from __future__ import annotations

import ctypes
import os
from typing import List, Optional, Sequence

import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libpsgd.so")

(PSGD_OK, PSGD_ERR_ARG, PSGD_ERR_ALIGN, PSGD_ERR_CUDA, PSGD_ERR_OOM, PSGD_ERR_STATE, PSGD_ERR_DEVICE,
 PSGD_ERR_TIMEOUT) = range(8)
PSGD_F32, PSGD_BF16 = 0, 1
FLAG_LAZY_ERRORS = 1
FLAG_SUM_FIRST = 2
FLAG_NO_WARM_START = 4

_ERR_NAMES = {1: "PSGD_ERR_ARG", 2: "PSGD_ERR_ALIGN", 3: "PSGD_ERR_CUDA", 4: "PSGD_ERR_OOM",
              5: "PSGD_ERR_STATE", 6: "PSGD_ERR_DEVICE", 7: "PSGD_ERR_TIMEOUT"}


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
    "psgd_step_static_status": (ctypes.c_int, [_P]),
    "psgd_set_power_iters": (ctypes.c_int, [_P, ctypes.c_int]),
    "psgd_set_global_workers": (ctypes.c_int, [_P, ctypes.c_int]),
    "psgd_dist_sizes": (ctypes.c_int, [_P, ctypes.POINTER(ctypes.c_size_t), ctypes.POINTER(ctypes.c_size_t)]),
    "psgd_dist_p": (ctypes.c_int, [_P, _PP, _PP, _PP, _PP, _PP, _P, _P]),
    "psgd_dist_q": (ctypes.c_int, [_P, _P, _P, _P]),
    "psgd_dist_finish": (ctypes.c_int, [_P, _P, _P]),
    "psgd_set_svd_refresh": (ctypes.c_int, [_P, ctypes.c_int, ctypes.c_int]),
    "psgd_set_svd_oversampling": (ctypes.c_int, [_P, ctypes.c_int]),
    "psgd_test_stall_products": (ctypes.c_int, [_P, ctypes.c_int]),
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


def _on_device(t: torch.Tensor) -> bool:
    return t.is_cuda


def _check_buf(t, what: str, numel: int, dtypes, on_device: bool, at_least: bool = False):
    """Host-side check of one buffer before its address crosses the ABI: a
    tensor must sit on the right side (device or host), have a listed
    dtype, be contiguous and hold numel elements (at least numel with
    at_least).  Raw addresses (ints) and None pass through unchecked; the
    library checks those for null and alignment itself."""
    if t is None or isinstance(t, int):
        return
    if not isinstance(t, torch.Tensor):
        raise PsgdError(PSGD_ERR_ARG, f"{what}: expected a tensor or an address, got {type(t).__name__}")
    if _on_device(t) != on_device:
        raise PsgdError(PSGD_ERR_ARG, f"{what}: expected a {'device' if on_device else 'host'} tensor")
    if t.dtype not in dtypes:
        raise PsgdError(PSGD_ERR_ARG, f"{what}: dtype {t.dtype} not in {list(dtypes)}")
    if not t.is_contiguous():
        raise PsgdError(PSGD_ERR_ARG, f"{what}: not contiguous")
    n = t.numel()
    if (n < numel) if at_least else (n != numel):
        raise PsgdError(PSGD_ERR_ARG, f"{what}: {n} elements, expected {'at least ' if at_least else ''}{numel}")


def _check_list(values, what: str, count: int):
    if values is None or len(values) != count:
        raise PsgdError(PSGD_ERR_ARG, f"{what}: expected {count} entries, got "
                                      f"{'none' if values is None else len(values)}")


_F32 = (torch.float32,)
_F64 = (torch.float64,)


def _addr(v):
    # tensors give their address; ints and None pass as they are (anything
    # else is refused by the checks before it reaches the library)
    return v.data_ptr() if isinstance(v, torch.Tensor) else v


def _arr(addrs: Sequence) -> ctypes.Array:
    return (ctypes.c_void_p * max(1, len(addrs)))(*addrs)


def _ptrs(values: Sequence) -> ctypes.Array:
    return _arr([_addr(v) for v in values])


def _sig(values: Sequence) -> List:
    """The addresses of a call's buffers (ints and None as they are): the
    checks run again only when these change, the same condition on which
    the library re-uploads its pointer tables."""
    try:
        return [v.data_ptr() for v in values]
    except AttributeError:
        return [_addr(v) for v in values]


def _arr_sig(sig: List) -> ctypes.Array:
    return _arr(sig)


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
    m, n, rank = int(m), int(n), int(rank)
    gdt = (torch.bfloat16,) if grad_dtype == "bf16" else _F32
    _check_list(errors, "errors", W)
    for w in range(W):
        _check_buf(grads[w], f"grads[{w}]", m * n, gdt, True)
        _check_buf(errors[w], f"errors[{w}]", m * n, _F32, True)
    _check_buf(q, "q", n * rank, _F32, True)
    _check_buf(p_hat, "p_hat", m * rank, _F32, True)
    _check_buf(recon, "recon", m * n, _F32, True)
    rc = lib.psgd_step_static(int(m), int(n), int(rank), W, PSGD_BF16 if grad_dtype == "bf16" else PSGD_F32,
                              _ptrs(grads), _ptrs(errors), q.data_ptr(),
                              p_hat.data_ptr() if p_hat is not None else None,
                              recon.data_ptr() if recon is not None else None, _stream_handle(stream))
    if rc:
        raise PsgdError(rc, lib.psgd_last_error(None).decode())


def step_static_status(stream=None) -> None:
    """Synchronise `stream` and raise if the last allocation-free step on
    this device flagged a device-side inconsistency
    (psgd_step_static_status)."""
    lib = load()
    rc = lib.psgd_step_static_status(_stream_handle(stream))
    if rc:
        raise PsgdError(rc, lib.psgd_last_error(None).decode())


class PowerSGD:
    """One library context: fixed layer shapes, rank, worker count.

    Buffers are torch tensors (or raw device addresses as ints).  grads and
    errors are indexed [w][l]; q, p_hat, recon per layer.
    """

    def __init__(self, layers: Sequence[Sequence[int]], rank: int, workers: int, seed: int = 1234,
                 grad_dtype: str = "f32", lazy_errors: bool = False, sum_first: bool = False,
                 power_iters: int = 1, warm_start: bool = True, svd_every: int = 0, svd_iters: int = 8,
                 svd_oversampling: Optional[int] = None):
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
        if svd_oversampling is not None:
            self._check(self.lib.psgd_set_svd_oversampling(self._h, int(svd_oversampling)))
        if svd_every:
            self._check(self.lib.psgd_set_svd_refresh(self._h, int(svd_every), int(svd_iters)))

    # -- helpers
    def _check(self, rc: int):
        if rc:
            raise PsgdError(rc, self.lib.psgd_last_error(self._h).decode())

    @staticmethod
    def _flat(per_worker: Sequence[Sequence]) -> List:
        flat: List = []
        for row in per_worker:
            flat.extend(row)
        return flat

    def _validated(self, name: str, parts: Sequence, check) -> List:
        """Signatures of the call's buffer lists (None for an absent list);
        check() runs unless they equal those of the last validated call of
        this kind.  The library reads W*L (or L) entries from each list, so
        a list is only ever passed after a check of its length."""
        sigs = [None if p is None else _sig(p) for p in parts]
        seen = self.__dict__.setdefault("_seen", {})
        if seen.get(name) != sigs:
            check()
            seen[name] = sigs
        return sigs

    @staticmethod
    def _opt(sig):
        return None if sig is None else _arr_sig(sig)

    def _gdt(self):
        return (torch.bfloat16,) if self.grad_dtype == "bf16" else _F32

    def _check_wl(self, per_worker, what: str, dtypes, on_device: bool = True):
        """per_worker[w][l]: W lists of L matrices m x n."""
        _check_list(per_worker, what, self.workers)
        for w in range(self.workers):
            _check_list(per_worker[w], f"{what}[{w}]", len(self.layers))
            for l, (m, n) in enumerate(self.layers):
                _check_buf(per_worker[w][l], f"{what}[{w}][{l}]", m * n, dtypes, on_device)

    def _check_layers(self, bufs, what: str, cols, on_device: bool = True, optional: bool = False):
        """bufs[l]: one m x cols (cols = 'n' for m x n, 'r' for m x rank, 'nr'
        for n x rank) float32 buffer per layer; optional lists may be None."""
        if bufs is None and optional:
            return
        _check_list(bufs, what, len(self.layers))
        for l, (m, n) in enumerate(self.layers):
            numel = {"n": m * n, "r": m * self.rank, "nr": n * self.rank}[cols]
            _check_buf(bufs[l], f"{what}[{l}]", numel, _F32, on_device)

    # -- API
    def init_q(self, q: Sequence, stream=None):
        (sq,) = self._validated("init_q", (q,), lambda: self._check_layers(q, "q", "nr"))
        self._check(self.lib.psgd_init_q(self._h, _arr_sig(sq), _stream_handle(stream)))

    def _check_step_bufs(self, grads, errors, q, p_hat, recon, grads_on_device=True):
        self._check_wl(grads, "grads", self._gdt(), on_device=grads_on_device)
        self._check_wl(errors, "errors", _F32)
        self._check_layers(q, "q", "nr")
        self._check_layers(p_hat, "p_hat", "r", on_device=grads_on_device, optional=True)
        self._check_layers(recon, "recon", "n", optional=True)

    def step(self, grads, errors, q, p_hat=None, recon=None, stream=None):
        sg, se, sq, sp, sr = self._validated(
            "step", (self._flat(grads), self._flat(errors), q, p_hat, recon),
            lambda: self._check_step_bufs(grads, errors, q, p_hat, recon))
        self._check(self.lib.psgd_step(self._h, _arr_sig(sg), _arr_sig(se), _arr_sig(sq), self._opt(sp),
                                       self._opt(sr), _stream_handle(stream)))

    def step_host(self, grads_host, errors, q, p_hat_host=None, q_host=None, stream=None):
        def check():
            self._check_step_bufs(grads_host, errors, q, p_hat_host, None, grads_on_device=False)
            self._check_layers(q_host, "q_host", "nr", on_device=False, optional=True)
        sg, se, sq, sp, sh = self._validated(
            "step_host", (self._flat(grads_host), self._flat(errors), q, p_hat_host, q_host), check)
        self._check(self.lib.psgd_step_host(self._h, _arr_sig(sg), _arr_sig(se), _arr_sig(sq), self._opt(sp),
                                            self._opt(sh), _stream_handle(stream)))

    def step_host_flat(self, grads_host, layer_offsets, errors, q, p_hat_host=None, q_host=None, stream=None):
        """grads_host[w]: one host buffer per worker holding every layer,
        layer l starting at element layer_offsets[l]."""
        offsets = [int(o) for o in layer_offsets]

        def check():
            _check_list(offsets, "layer_offsets", len(self.layers))
            _check_list(grads_host, "grads_host", self.workers)
            span = max((o + m * n for o, (m, n) in zip(offsets, self.layers)), default=0)
            for w in range(self.workers):
                _check_buf(grads_host[w], f"grads_host[{w}]", span, self._gdt(), False, at_least=True)
            self._check_wl(errors, "errors", _F32)
            self._check_layers(q, "q", "nr")
            self._check_layers(p_hat_host, "p_hat_host", "r", on_device=False, optional=True)
            self._check_layers(q_host, "q_host", "nr", on_device=False, optional=True)
        sg, so, se, sq, sp, sh = self._validated(
            "step_host_flat", (grads_host, offsets, self._flat(errors), q, p_hat_host, q_host), check)
        offs = (ctypes.c_int64 * max(1, len(offsets)))(*offsets)
        self._check(self.lib.psgd_step_host_flat(self._h, _arr_sig(sg), offs, _arr_sig(se), _arr_sig(sq),
                                                 self._opt(sp), self._opt(sh), _stream_handle(stream)))

    def materialize_errors(self, errors, stream=None):
        (se,) = self._validated("materialize_errors", (self._flat(errors),),
                                lambda: self._check_wl(errors, "errors", _F32))
        self._check(self.lib.psgd_materialize_errors(self._h, _arr_sig(se), _stream_handle(stream)))

    def momentum_step(self, params, mom, lr: float, beta: float, stream=None):
        def check():
            self._check_layers(params, "params", "n")
            self._check_layers(mom, "mom", "n")
        sx, sm = self._validated("momentum_step", (params, mom), check)
        self._check(self.lib.psgd_momentum_step(self._h, _arr_sig(sx), _arr_sig(sm), lr, beta,
                                                _stream_handle(stream)))

    def vec_mean(self, vecs, out, params=None, mom=None, lr: float = 0.0, beta: float = 0.0, stream=None):
        """vecs[w][k] -> out[k] = mean over workers (+ momentum if params, mom)."""
        K = len(out)

        def check():
            for k, t in enumerate(out):
                if not isinstance(t, torch.Tensor):
                    raise PsgdError(PSGD_ERR_ARG, f"out[{k}]: expected a tensor (its length sets the vector's)")
                _check_buf(t, f"out[{k}]", t.numel(), _F32, True)
            _check_list(vecs, "vecs", self.workers)
            for w in range(self.workers):
                _check_list(vecs[w], f"vecs[{w}]", K)
                for k in range(K):
                    _check_buf(vecs[w][k], f"vecs[{w}][{k}]", out[k].numel(), _F32, True)
            for name, lst in (("params", params), ("mom", mom)):
                if lst is not None:
                    _check_list(lst, name, K)
                    for k in range(K):
                        _check_buf(lst[k], f"{name}[{k}]", out[k].numel(), _F32, True)
        sv, so, sx, sm = self._validated("vec_mean", (self._flat(vecs), out, params, mom), check)
        lens = (ctypes.c_int64 * max(1, K))(*[t.numel() for t in out])
        self._check(self.lib.psgd_vec_mean(self._h, _arr_sig(sv), _arr_sig(so), lens, K, self._opt(sx),
                                           self._opt(sm), lr, beta, _stream_handle(stream)))

    # -- distributed step (the caller all-reduces p_send and q_send, SUM)
    def set_global_workers(self, total: int):
        self._check(self.lib.psgd_set_global_workers(self._h, int(total)))

    def dist_sizes(self):
        pe, qe = ctypes.c_size_t(), ctypes.c_size_t()
        self._check(self.lib.psgd_dist_sizes(self._h, ctypes.byref(pe), ctypes.byref(qe)))
        return int(pe.value), int(qe.value)

    def dist_p(self, grads, errors, q, p_send, p_hat=None, recon=None, stream=None):
        def check():
            self._check_step_bufs(grads, errors, q, p_hat, recon)
            _check_buf(p_send, "p_send", 0, _F64, True, at_least=True)
        sg, se, sq, sp, sr = self._validated(
            "dist_p", (self._flat(grads), self._flat(errors), q, p_hat, recon), check)
        _check_buf(p_send, "p_send", 0, _F64, True, at_least=True)
        self._check(self.lib.psgd_dist_p(self._h, _arr_sig(sg), _arr_sig(se), _arr_sig(sq), self._opt(sp),
                                         self._opt(sr), p_send.data_ptr(), _stream_handle(stream)))

    def dist_q(self, p_sum, q_send, stream=None):
        _check_buf(p_sum, "p_sum", 0, _F64, True, at_least=True)
        _check_buf(q_send, "q_send", 0, _F64, True, at_least=True)
        self._check(self.lib.psgd_dist_q(self._h, p_sum.data_ptr(), q_send.data_ptr(), _stream_handle(stream)))

    def dist_finish(self, q_sum, stream=None):
        _check_buf(q_sum, "q_sum", 0, _F64, True, at_least=True)
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

    def test_stall_products(self, on: bool) -> None:
        """Testing the bounded waits: the tensor-core second pass of later
        steps issues no products, so its waits run out (psgd.h)."""
        self._check(self.lib.psgd_test_stall_products(self._h, 1 if on else 0))

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

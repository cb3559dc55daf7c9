"""ctypes binding of the SALR C ABI (include/salr.h).  Argument marshalling only: every
step of the layer runs in the CUDA library; there is no fallback path.

Tensors are torch tensors (device memory and streams come from torch); bf16 tensors are
passed as raw pointers to their 16-bit patterns.
"""
from __future__ import annotations

import ctypes
import os

HERE = os.path.dirname(os.path.abspath(__file__))
# The built library; SALR_LIBRARY names another build of it (the bounds-checked debug
# build, libsalr_checks.so) to load instead.
LIB_PATH = os.environ.get("SALR_LIBRARY") or os.path.join(HERE, "libsalr.so")

SALR_OK = 0
SALR_ERR_INVALID = 1
SALR_ERR_UNSUPPORTED = 2
SALR_ERR_CUDA = 3
SALR_ERR_OOM = 4
SALR_ERR_TIMEOUT = 5

# name -> (restype, argtypes) for every entry point declared in include/salr.h
_P, _I64, _F, _I = ctypes.c_void_p, ctypes.c_int64, ctypes.c_float, ctypes.c_int


class SalrPlan(ctypes.Structure):
    """salr_plan of include/salr.h (field order and types as declared there)."""
    _fields_ = [("path", ctypes.c_int32), ("kernels", ctypes.c_int32),
                ("token_tile", ctypes.c_int32), ("tile_rows", ctypes.c_int32),
                ("grid", ctypes.c_int32),
                ("units", ctypes.c_int32), ("tiles", ctypes.c_int32),
                ("whole_tiles", ctypes.c_int32), ("splits", ctypes.c_int32),
                ("split_sum_bytes", ctypes.c_int64), ("dense_scratch_bytes", ctypes.c_int64),
                ("group_rows", ctypes.c_int32)]
SIGNATURES = {
    "salr_encode": (_I, [_P, _I64, _I64, _F, _P, ctypes.POINTER(_P)]),
    "salr_decode": (_I, [_P, _P, _P]),
    "salr_linear": (_I, [_P, _I64, _P, _P, _P, _I64, _P, _P]),
    "salr_linear_host": (_I, [_P, _I64, _P, _P, _P, _I64, _P, _P]),
    "salr_linear_noalloc": (_I, [_P, _I64, _P, _P, _P, _I64, _P, _P]),
    "salr_free": (_I, [_P]),
    "salr_info": (_I, [_P, ctypes.POINTER(_I64), ctypes.POINTER(_I64), ctypes.POINTER(_I64),
                       ctypes.POINTER(_I64)]),
    "salr_format_view": (_I, [_P, ctypes.POINTER(_P), ctypes.POINTER(_I64), ctypes.POINTER(_P),
                              ctypes.POINTER(_I64)]),
    "salr_save_size": (_I, [_P, ctypes.POINTER(_I64)]),
    "salr_save": (_I, [_P, _P, _I64, _P]),
    "salr_load": (_I, [_P, _I64, _P, ctypes.POINTER(_P)]),
    "salr_residual_adapter": (_I, [_P, _P, _I64, _P, _I64, _I, _P, _P, _P, _P]),
    "salr_linear_plan": (_I, [_I64, _I64, _I64, _I64, ctypes.c_int32, ctypes.POINTER(SalrPlan)]),
    "salr_sync_status": (_I, [_P, _P]),
    "salr_status_string": (ctypes.c_char_p, [_I]),
}

_lib = None


class SalrError(RuntimeError):
    def __init__(self, fn: str, code: int):
        self.code = code
        super().__init__(f"{fn} failed: {status_string(code)} ({code})")


def load_library(path: str = LIB_PATH) -> ctypes.CDLL:
    """Load the CUDA library; raises if it has not been built (no silent fallback)."""
    global _lib
    if _lib is not None:
        return _lib
    if not os.path.exists(path):
        raise RuntimeError(f"SALR CUDA library not built: {path} is missing "
                           "(run python -m sparse_rank_linear_b200.build)")
    lib = ctypes.CDLL(path)
    for name, (res, args) in SIGNATURES.items():
        f = getattr(lib, name)
        f.restype = res
        f.argtypes = args
    _lib = lib
    return lib


def status_string(code: int) -> str:
    return load_library().salr_status_string(int(code)).decode()


def _check(fn: str, code: int):
    if code != SALR_OK:
        raise SalrError(fn, code)


def _stream_ptr(stream=None):
    import torch
    s = stream if stream is not None else torch.cuda.current_stream()
    return ctypes.c_void_p(s.cuda_stream)


def _ptr(t):
    return ctypes.c_void_p(t.data_ptr()) if t is not None else ctypes.c_void_p(0)


def _require(t, name, shape=None, device=True):
    import torch
    if t.dtype != torch.bfloat16:
        raise TypeError(f"{name} must be bfloat16")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous (row-major)")
    if device and not t.is_cuda:
        raise ValueError(f"{name} must be a CUDA tensor")
    if shape is not None and tuple(t.shape) != tuple(shape):
        raise ValueError(f"{name} has shape {tuple(t.shape)}, expected {tuple(shape)}")


class Weight:
    """An encoded (pruned, bitmap-stored) weight: owns a ``salr_handle``."""

    def __init__(self, handle: ctypes.c_void_p):
        self._h = handle

    @property
    def handle(self):
        if self._h is None:
            raise RuntimeError("weight has been freed")
        return self._h

    def info(self):
        n, k, nnz, nbytes = _I64(), _I64(), _I64(), _I64()
        _check("salr_info", load_library().salr_info(self.handle, ctypes.byref(n), ctypes.byref(k),
                                                     ctypes.byref(nnz), ctypes.byref(nbytes)))
        return {"N": n.value, "K": k.value, "nnz": nnz.value, "bytes": nbytes.value}

    def format_view(self):
        """(blob_ptr, blob_bytes, offsets_ptr, n_offsets): device pointers, read only."""
        b, bb, o, no = _P(), _I64(), _P(), _I64()
        _check("salr_format_view", load_library().salr_format_view(
            self.handle, ctypes.byref(b), ctypes.byref(bb), ctypes.byref(o), ctypes.byref(no)))
        return b.value, bb.value, o.value, no.value

    def format_tensors(self):
        """Copies of the encoded blob (uint8) and offset table (int32 holding the uint32
        entries), made by torch from views of the handle's device memory."""
        b, bb, o, no = self.format_view()
        return (_device_view(b, bb, "|u1").clone(), _device_view(o, no, "<i4").clone())

    def decode(self, out=None, stream=None):
        import torch
        inf = self.info()
        if out is None:
            out = torch.empty(inf["N"], inf["K"], dtype=torch.bfloat16, device="cuda")
        _require(out, "W_out", (inf["N"], inf["K"]))
        _check("salr_decode", load_library().salr_decode(self.handle, _ptr(out), _stream_ptr(stream)))
        return out

    def to_bytes(self, stream=None) -> bytes:
        """salr_save: the serialised image of this weight (layout in include/salr.h)."""
        lib = load_library()
        n = _I64()
        _check("salr_save_size", lib.salr_save_size(self.handle, ctypes.byref(n)))
        buf = ctypes.create_string_buffer(n.value)
        _check("salr_save", lib.salr_save(self.handle, ctypes.cast(buf, _P), n.value,
                                          _stream_ptr(stream)))
        return buf.raw

    def sync_status(self, stream=None) -> int:
        return load_library().salr_sync_status(self.handle, _stream_ptr(stream))

    def free(self):
        if self._h is not None:
            _check("salr_free", load_library().salr_free(self._h))
            self._h = None

    def __del__(self):
        try:
            if self._h is not None and _lib is not None:
                _lib.salr_free(self._h)
                self._h = None
        except Exception:
            pass


class _DevArray:
    """Minimal __cuda_array_interface__ exporter of a device range (only ever cloned)."""

    def __init__(self, ptr: int, n: int, typestr: str):
        self.__cuda_array_interface__ = {"shape": (n,), "typestr": typestr,
                                         "data": (ptr, False), "version": 2, "strides": None}


def _device_view(ptr: int, n: int, typestr: str):
    import torch
    return torch.as_tensor(_DevArray(ptr, n, typestr), device="cuda")


def encode(W, sparsity: float = 0.5, stream=None) -> Weight:
    """salr_encode: prune ``W`` (N x K bf16, CUDA) per row and bitmap-encode it."""
    _require(W, "W")
    N, K = W.shape
    h = _P()
    _check("salr_encode", load_library().salr_encode(_ptr(W), N, K, float(sparsity),
                                                     _stream_ptr(stream), ctypes.byref(h)))
    return Weight(h)


def load(image: bytes, stream=None) -> Weight:
    """salr_load: a weight on the current CUDA device from a serialised image."""
    data = bytes(image)
    h = _P()
    _check("salr_load", load_library().salr_load(ctypes.cast(ctypes.c_char_p(data), _P),
                                                 len(data), _stream_ptr(stream),
                                                 ctypes.byref(h)))
    return Weight(h)


def residual_adapter(W, weight: Weight, r: int, q: int = 2, oversample: int = 16, omega=None,
                     seed: int = 0, stream=None):
    """salr_residual_adapter: the rank-r adapter (A' K x r, B' r x N, bf16) of W minus its
    pruned form, and the estimated singular values (r, fp32).  ``omega`` (K x l fp32,
    CUDA) is the random test matrix; by default a seeded standard normal one with
    l = r + oversample columns (capped at 160 and at min(N, K))."""
    import torch
    inf = weight.info()
    N, K = inf["N"], inf["K"]
    _require(W, "W", (N, K))
    if omega is None:
        l = min(r + oversample, 160, N, K)
        g = torch.Generator(device=W.device)
        g.manual_seed(seed)
        omega = torch.randn(K, l, generator=g, device=W.device, dtype=torch.float32)
    if omega.dtype != torch.float32 or not omega.is_contiguous() or omega.shape[0] != K:
        raise ValueError("omega must be a contiguous K x l float32 tensor")
    A = torch.empty(K, r, dtype=torch.bfloat16, device=W.device)
    B = torch.empty(r, N, dtype=torch.bfloat16, device=W.device)
    sigma = torch.empty(r, dtype=torch.float32, device=W.device)
    _check("salr_residual_adapter", load_library().salr_residual_adapter(
        _ptr(W), weight.handle, r, _ptr(omega), omega.shape[1], q, _ptr(A), _ptr(B),
        _ptr(sigma), _stream_ptr(stream)))
    return A, B, sigma


def linear(X, weight: Weight, A_cat=None, B_cat=None, Y=None, stream=None):
    """salr_linear: Y = X (M.W)^T + (X A_cat) B_cat; returns Y (M x N bf16)."""
    import torch
    inf = weight.info()
    _require(X, "X")
    M = X.shape[0]
    if X.shape[1] != inf["K"]:
        raise ValueError("X has the wrong number of columns")
    R = 0
    if A_cat is not None:
        R = A_cat.shape[1]
        _require(A_cat, "A_cat", (inf["K"], R))
        _require(B_cat, "B_cat", (R, inf["N"]))
    if Y is None:
        Y = torch.empty(M, inf["N"], dtype=torch.bfloat16, device=X.device)
    _require(Y, "Y", (M, inf["N"]))
    _check("salr_linear", load_library().salr_linear(_ptr(X), M, weight.handle, _ptr(A_cat),
                                                     _ptr(B_cat), R, _ptr(Y), _stream_ptr(stream)))
    return Y


def linear_host(X_host, weight: Weight, A_cat, B_cat, Y_host, stream=None):
    """salr_linear_host: X_host / Y_host are pinned CPU bf16 tensors; adapters on device."""
    inf = weight.info()
    _require(X_host, "X_host", device=False)
    _require(Y_host, "Y_host", (X_host.shape[0], inf["N"]), device=False)
    R = 0 if A_cat is None else A_cat.shape[1]
    _check("salr_linear_host", load_library().salr_linear_host(
        _ptr(X_host), X_host.shape[0], weight.handle, _ptr(A_cat), _ptr(B_cat), R, _ptr(Y_host),
        _stream_ptr(stream)))
    return Y_host


def plan(N: int, K: int, M: int, R: int = 0, sms: int = 0) -> dict:
    """salr_linear_plan: the kernels, tiles, work split and extra device memory that
    salr_linear uses for M tokens on an N x K weight (sms = 0: the current device's)."""
    out = SalrPlan()
    _check("salr_linear_plan", load_library().salr_linear_plan(N, K, M, R, sms, ctypes.byref(out)))
    return {name: getattr(out, name) for name, _ in SalrPlan._fields_}

"""Python binding of ``libqlora_nf4.so`` (the C ABI in ``include/qlora_nf4.h``).

Argument marshalling only: every step of the computation runs in the
library's CUDA kernels.  PyTorch provides device memory and the current
stream.  There is no CPU fallback: if the shared library is missing the
import fails, and every non-OK status raises :class:`QloraError`.

Functions keep the C names:

* :func:`nf4_quantize` / :func:`nf4_dequantize`
* :func:`qlora_linear_fwd` / :func:`qlora_linear_bwd`
* :func:`qlora_fwd_workspace_size` / :func:`qlora_bwd_workspace_size`
* :func:`nf4_levels`, :func:`qlora_strerror`
"""

import ctypes
import os
from collections import namedtuple

import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libqlora_nf4.so")

if not os.path.exists(LIB_PATH):
    raise ImportError(
        f"{LIB_PATH} is missing: build it with `python -m bit_nf4_quantized_26_b200.build`")

_lib = ctypes.CDLL(LIB_PATH)

DTYPE_BF16 = 0
DTYPE_F32 = 1
DEV_NONFINITE = 1
DEV_TIMEOUT = 2

STATUS = {0: "QLORA_OK", 1: "QLORA_ERR_NULL", 2: "QLORA_ERR_SHAPE", 3: "QLORA_ERR_ALIGN",
          4: "QLORA_ERR_WORKSPACE", 5: "QLORA_ERR_NONFINITE", 6: "QLORA_ERR_TIMEOUT",
          7: "QLORA_ERR_CUDA", 8: "QLORA_ERR_ARCH", 9: "QLORA_ERR_DTYPE"}


class QloraError(RuntimeError):
    def __init__(self, code, where):
        self.code = code
        super().__init__(f"{where}: {STATUS.get(code, code)} ({qlora_strerror(code)})")


class _NF4Weight(ctypes.Structure):
    _fields_ = [("codes", ctypes.c_void_p), ("c8", ctypes.c_void_p), ("s2", ctypes.c_void_p),
                ("n_out", ctypes.c_int64), ("k_in", ctypes.c_int64)]


_P = ctypes.c_void_p
_I64 = ctypes.c_int64
_I32 = ctypes.c_int32
_SZ = ctypes.c_size_t

_lib.nf4_quantize.argtypes = [_P, _I64, _P, _P, _P, _P, _P]
_lib.nf4_quantize.restype = ctypes.c_int
_lib.nf4_dequantize.argtypes = [_P, _P, _P, _I64, _P, _P]
_lib.nf4_dequantize.restype = ctypes.c_int
_lib.qlora_linear_fwd.argtypes = [_P, _I64, _NF4Weight, _P, _P, _I32, ctypes.c_float, _P, _I32, _P, _P, _SZ,
                                  _P, _P]
_lib.qlora_linear_fwd.restype = ctypes.c_int
_lib.qlora_linear_bwd.argtypes = [_P, _P, _P, _I64, _NF4Weight, _P, _P, _I32, ctypes.c_float, _P, _I32, _P, _P,
                                  _P, _SZ, _P, _P]
_lib.qlora_linear_bwd.restype = ctypes.c_int
_lib.qlora_fwd_workspace_size.argtypes = [_I64, _I64, _I64, _I32]
_lib.qlora_fwd_workspace_size.restype = _SZ
_lib.qlora_bwd_workspace_size.argtypes = [_I64, _I64, _I64, _I32]
_lib.qlora_bwd_workspace_size.restype = _SZ
_lib.nf4_levels.argtypes = [_P]
_lib.nf4_levels.restype = None
_lib.qlora_strerror.argtypes = [ctypes.c_int]
_lib.qlora_strerror.restype = ctypes.c_char_p
_lib.qlora_linear_fwd_noalloc.argtypes = [_P, _I64, _NF4Weight, _P, _P, _I32, ctypes.c_float, _P, _I32, _P, _P,
                                          _P]
_lib.qlora_linear_fwd_noalloc.restype = ctypes.c_int
_lib.qlora_profile_enable.argtypes = [_I32]
_lib.qlora_profile_enable.restype = None
_lib.qlora_profile_collect.argtypes = [_P, _P, _I32]
_lib.qlora_profile_collect.restype = _I32
_lib.qlora_kernel_name.argtypes = [_I32]
_lib.qlora_kernel_name.restype = ctypes.c_char_p

EXPORTED = ("nf4_quantize", "nf4_dequantize", "qlora_linear_fwd", "qlora_linear_bwd",
            "qlora_fwd_workspace_size", "qlora_bwd_workspace_size", "nf4_levels", "qlora_strerror",
            "qlora_profile_enable", "qlora_profile_collect", "qlora_kernel_name", "qlora_linear_fwd_noalloc")

NF4Weight = namedtuple("NF4Weight", "codes c8 s2 n_out k_in")


def qlora_strerror(code):
    return _lib.qlora_strerror(int(code)).decode()


def nf4_levels():
    """The 16 fp32 NF4 levels the library's kernels use (host-only query)."""
    buf = (ctypes.c_float * 16)()
    _lib.nf4_levels(ctypes.cast(buf, _P))
    return [float(v) for v in buf]


def qlora_fwd_workspace_size(M, N, K, r):
    return int(_lib.qlora_fwd_workspace_size(M, N, K, r))


def qlora_bwd_workspace_size(M, N, K, r):
    return int(_lib.qlora_bwd_workspace_size(M, N, K, r))


def _ptr(t):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _stream(stream=None):
    s = torch.cuda.current_stream() if stream is None else stream
    return ctypes.c_void_p(s.cuda_stream)


def _check(code, where):
    if code != 0:
        raise QloraError(code, where)


def _weight(W):
    return _NF4Weight(W.codes.data_ptr(), W.c8.data_ptr(), W.s2.data_ptr(), int(W.n_out), int(W.k_in))


def nf4_sizes(numel):
    """(codes bytes, c8 bytes, s2 floats) of the NF4 storage of ``numel`` elements."""
    nb = -(-numel // 64)
    return nb * 32, nb, -(-nb // 256)


def nf4_quantize(w, codes=None, c8=None, s2=None, status=None, stream=None):
    """Quantise a bf16 CUDA tensor; returns ``(codes, c8, s2)`` (allocated if not given)."""
    assert w.dtype == torch.bfloat16 and w.is_cuda and w.is_contiguous()
    numel = w.numel()
    nc, nb, ns = nf4_sizes(numel)
    dev = w.device
    codes = torch.empty(nc, dtype=torch.uint8, device=dev) if codes is None else codes
    c8 = torch.empty(nb, dtype=torch.uint8, device=dev) if c8 is None else c8
    s2 = torch.empty(ns, dtype=torch.float32, device=dev) if s2 is None else s2
    _check(_lib.nf4_quantize(_ptr(w), numel, _ptr(codes), _ptr(c8), _ptr(s2), _ptr(status), _stream(stream)),
           "nf4_quantize")
    return codes, c8, s2


def quantize_weight(w, stream=None):
    """NF4-quantise a bf16 weight [n_out, k_in]; returns an :class:`NF4Weight`."""
    codes, c8, s2 = nf4_quantize(w, stream=stream)
    return NF4Weight(codes, c8, s2, w.shape[0], w.shape[1])


def nf4_dequantize(codes, c8, s2, numel, out=None, stream=None):
    """bf16 tensor of ``numel`` dequantised values."""
    out = torch.empty(numel, dtype=torch.bfloat16, device=codes.device) if out is None else out
    _check(_lib.nf4_dequantize(_ptr(codes), _ptr(c8), _ptr(s2), numel, _ptr(out), _stream(stream)),
           "nf4_dequantize")
    return out


def qlora_linear_fwd(X, W, A, B, s, y_dtype=DTYPE_BF16, Y=None, U=None, ws=None, status=None, stream=None):
    """Forward of the adapter-augmented NF4 linear; returns ``(Y, U)``."""
    M = X.shape[0]
    N, K, r = int(W.n_out), int(W.k_in), A.shape[0]
    dev = X.device
    if Y is None:
        Y = torch.empty((M, N), dtype=torch.float32 if y_dtype == DTYPE_F32 else torch.bfloat16, device=dev)
    if U is None:
        U = torch.empty((M, r), dtype=torch.float32, device=dev)
    if ws is None:
        ws = torch.empty(max(qlora_fwd_workspace_size(M, N, K, r), 16), dtype=torch.uint8, device=dev)
    _check(_lib.qlora_linear_fwd(_ptr(X), M, _weight(W), _ptr(A), _ptr(B), r, float(s), _ptr(Y), y_dtype,
                                 _ptr(U), _ptr(ws), ws.numel(), _ptr(status), _stream(stream)),
           "qlora_linear_fwd")
    return Y, U


def qlora_linear_fwd_noalloc(X, W, A, B, s, y_dtype=DTYPE_BF16, Y=None, U=None, status=None, stream=None):
    """Forward without a workspace, for callers that cannot allocate device
    memory at call time (the library keeps a fixed 16 MiB scratch array per
    device; problems that need more are rejected).  Returns ``(Y, U)``.  The
    output tensors are allocated here only when not given."""
    M = X.shape[0]
    N, r = int(W.n_out), A.shape[0]
    dev = X.device
    if Y is None:
        Y = torch.empty((M, N), dtype=torch.float32 if y_dtype == DTYPE_F32 else torch.bfloat16, device=dev)
    if U is None:
        U = torch.empty((M, r), dtype=torch.float32, device=dev)
    _check(_lib.qlora_linear_fwd_noalloc(_ptr(X), M, _weight(W), _ptr(A), _ptr(B), r, float(s), _ptr(Y), y_dtype,
                                         _ptr(U), _ptr(status), _stream(stream)),
           "qlora_linear_fwd_noalloc")
    return Y, U


def qlora_linear_bwd(dY, X, U, W, A, B, s, dx_dtype=DTYPE_BF16, dX=None, dA=None, dB=None, ws=None,
                     status=None, stream=None):
    """Backward through the frozen NF4 weight; returns ``(dX, dA, dB)``."""
    M = X.shape[0]
    N, K, r = int(W.n_out), int(W.k_in), A.shape[0]
    dev = X.device
    if dX is None:
        dX = torch.empty((M, K), dtype=torch.float32 if dx_dtype == DTYPE_F32 else torch.bfloat16, device=dev)
    if dA is None:
        dA = torch.empty((r, K), dtype=torch.float32, device=dev)
    if dB is None:
        dB = torch.empty((N, r), dtype=torch.float32, device=dev)
    if ws is None:
        ws = torch.empty(max(qlora_bwd_workspace_size(M, N, K, r), 16), dtype=torch.uint8, device=dev)
    _check(_lib.qlora_linear_bwd(_ptr(dY), _ptr(X), _ptr(U), M, _weight(W), _ptr(A), _ptr(B), r, float(s),
                                 _ptr(dX), dx_dtype, _ptr(dA), _ptr(dB), _ptr(ws), ws.numel(), _ptr(status),
                                 _stream(stream)),
           "qlora_linear_bwd")
    return dX, dA, dB


def profile_enable(on=True):
    """Bracket every library kernel launch with CUDA events (diagnostics)."""
    _lib.qlora_profile_enable(1 if on else 0)


def profile_collect(capacity=1 << 16):
    """[(kernel name, ms)] of the launches recorded since the last collect."""
    ids = (ctypes.c_int32 * capacity)()
    ms = (ctypes.c_float * capacity)()
    n = _lib.qlora_profile_collect(ctypes.cast(ids, _P), ctypes.cast(ms, _P), capacity)
    if n < 0:
        raise QloraError(7, "qlora_profile_collect")
    return [(_lib.qlora_kernel_name(ids[i]).decode(), float(ms[i])) for i in range(min(n, capacity))]


def raw():
    """The loaded ``ctypes.CDLL`` (for callers that pass raw pointers)."""
    return _lib

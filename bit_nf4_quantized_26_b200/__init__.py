"""Python binding of ``libqlora_nf4.so`` (the C ABI in ``include/qlora_nf4.h`` and
``include/qlora_optim.h``).

Argument marshalling only: every step of the computation runs in the
library's CUDA kernels.  PyTorch provides device memory and the current
stream.  There is no CPU fallback: if the shared library is missing the
import fails, and every non-OK status raises :class:`QloraError`.

Functions keep the C names:

* :func:`nf4_quantize` / :func:`nf4_dequantize`
* :func:`qlora_linear_fwd` / :func:`qlora_linear_bwd`
* :func:`qlora_fwd_workspace_size` / :func:`qlora_bwd_workspace_size`
* :func:`nf4_levels`, :func:`qlora_strerror`
* :func:`qlora_adamw8_step` with :class:`AdamW8State` (``include/qlora_optim.h``)
"""

import ctypes
import os
from collections import namedtuple

import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libqlora_nf4.so")

if not os.path.exists(LIB_PATH):
    raise ImportError(
        f"{LIB_PATH} is missing: build it with `python bit_nf4_quantized_26_b200/build.py`")

_lib = ctypes.CDLL(LIB_PATH)

DTYPE_BF16 = 0
DTYPE_F32 = 1
DEV_NONFINITE = 1
DEV_TIMEOUT = 2

STATUS = {0: "QLORA_OK", 1: "QLORA_ERR_NULL", 2: "QLORA_ERR_SHAPE", 3: "QLORA_ERR_ALIGN",
          4: "QLORA_ERR_WORKSPACE", 5: "QLORA_ERR_NONFINITE", 6: "QLORA_ERR_TIMEOUT",
          7: "QLORA_ERR_CUDA", 8: "QLORA_ERR_ARCH", 9: "QLORA_ERR_DTYPE", 10: "QLORA_ERR_INTERNAL"}


class QloraError(RuntimeError):
    def __init__(self, code, where):
        self.code = code
        super().__init__(f"{where}: {STATUS.get(code, code)} ({qlora_strerror(code)})")


class _NF4Weight(ctypes.Structure):
    _fields_ = [("codes", ctypes.c_void_p), ("c8", ctypes.c_void_p), ("s2", ctypes.c_void_p),
                ("n_out", ctypes.c_int64), ("k_in", ctypes.c_int64), ("mean", ctypes.c_void_p)]


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

# mean: None for the plain double quantisation, or the 1-element fp32 device
# tensor of a weight quantised with nf4_quantize_centered.
NF4Weight = namedtuple("NF4Weight", "codes c8 s2 n_out k_in mean", defaults=(None,))


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
    mean = getattr(W, "mean", None)
    return _NF4Weight(W.codes.data_ptr(), W.c8.data_ptr(), W.s2.data_ptr(), int(W.n_out), int(W.k_in),
                      None if mean is None else mean.data_ptr())


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


# ------------------------------------------------------------ optimizer step
# (include/qlora_optim.h: AdamW with 8-bit states in paged memory)

_F = ctypes.c_float
_lib.qlora_adamw8_step.argtypes = [_P, _P, _P, _P, _P, _P, _I64, _F, _F, _F, _F, _F, _I64, _P, _P]
_lib.qlora_adamw8_step.restype = ctypes.c_int
_lib.qlora_paged_alloc.argtypes = [ctypes.POINTER(ctypes.c_void_p), _SZ]
_lib.qlora_paged_alloc.restype = ctypes.c_int
_lib.qlora_paged_prefetch.argtypes = [_P, _SZ, _I32, _P]
_lib.qlora_paged_prefetch.restype = ctypes.c_int
_lib.qlora_paged_free.argtypes = [_P]
_lib.qlora_paged_free.restype = ctypes.c_int

EXPORTED = EXPORTED + ("qlora_adamw8_step", "qlora_paged_alloc", "qlora_paged_prefetch", "qlora_paged_free")

STATE_BLOCK = 256  # parameters per fp32 state scale


def _al(b):
    return (b + 255) & ~255


class AdamW8State:
    """8-bit AdamW state of an ``n``-parameter tensor: E4M3 codes of m and of
    sqrt(v) (one byte each per parameter) and one fp32 scale per 256
    parameters for each.  ``paged=True`` puts all four arrays in one CUDA
    managed allocation (``qlora_paged_alloc``: resident in HBM, evicted to
    host RAM under memory pressure, migrated back when touched); otherwise
    they live in a torch device tensor.  A fresh state is all zeros."""

    def __init__(self, n, paged=True, device=None):
        self.n = int(n)
        self.nb = -(-self.n // STATE_BLOCK)
        self._offs = (0, _al(self.n), 2 * _al(self.n), 2 * _al(self.n) + _al(4 * self.nb))
        self.bytes = self._offs[3] + _al(4 * self.nb)
        self.paged = paged
        self._buf = None
        self._base = None
        if paged:
            ptr = ctypes.c_void_p()
            _check(_lib.qlora_paged_alloc(ctypes.byref(ptr), self.bytes), "qlora_paged_alloc")
            self._base = ptr.value
        else:
            self._buf = torch.zeros(self.bytes, dtype=torch.uint8, device=device or "cuda")
            self._base = self._buf.data_ptr()

    def pointers(self):
        """Device-usable addresses of (m8, u8, m_scale, u_scale)."""
        return tuple(self._base + o for o in self._offs)

    def prefetch(self, to_host=False, stream=None):
        """Migrate a paged state to the device (or to host RAM) on ``stream``."""
        if self.paged:
            _check(_lib.qlora_paged_prefetch(ctypes.c_void_p(self._base), self.bytes, 1 if to_host else 0,
                                             _stream(stream)), "qlora_paged_prefetch")

    def host_arrays(self):
        """Copies of (m8, u8, m_scale, u_scale) as numpy arrays (synchronises)."""
        import numpy as np
        torch.cuda.synchronize()
        if self.paged:
            def grab(off, n, ct, dt):
                return np.ctypeslib.as_array((ct * n).from_address(self._base + off)).astype(dt, copy=True)
            return (grab(self._offs[0], self.n, ctypes.c_uint8, np.uint8),
                    grab(self._offs[1], self.n, ctypes.c_uint8, np.uint8),
                    grab(self._offs[2], self.nb, ctypes.c_float, np.float32),
                    grab(self._offs[3], self.nb, ctypes.c_float, np.float32))
        b = self._buf.cpu().numpy()
        o = self._offs
        return (b[o[0]:o[0] + self.n].copy(), b[o[1]:o[1] + self.n].copy(),
                b[o[2]:o[2] + 4 * self.nb].view(np.float32).copy(), b[o[3]:o[3] + 4 * self.nb].view(np.float32).copy())

    def close(self):
        if self.paged and self._base is not None:
            torch.cuda.synchronize()
            _check(_lib.qlora_paged_free(ctypes.c_void_p(self._base)), "qlora_paged_free")
        self._base = None
        self._buf = None

    def __del__(self):
        try:
            self.close()
        except Exception:
            pass


def qlora_adamw8_step(p, grad, state, lr, beta1=0.9, beta2=0.999, eps=1e-8, weight_decay=0.0, step=1,
                      status=None, stream=None):
    """One AdamW step in place on the bf16 parameter tensor ``p`` with fp32
    gradient ``grad`` and the 8-bit :class:`AdamW8State` ``state``."""
    assert p.dtype == torch.bfloat16 and grad.dtype == torch.float32
    assert p.is_contiguous() and grad.is_contiguous() and p.numel() == grad.numel() == state.n
    m8, u8, ms, us = state.pointers()
    _check(_lib.qlora_adamw8_step(_ptr(p), _ptr(grad), ctypes.c_void_p(m8), ctypes.c_void_p(u8),
                                  ctypes.c_void_p(ms), ctypes.c_void_p(us), state.n, lr, beta1, beta2, eps,
                                  weight_decay, int(step), _ptr(status), _stream(stream)), "qlora_adamw8_step")
    return p


# ------------------------------------------------------------ LoRA dropout
# (include/qlora_nf4.h: dropout on the adapter input, Philox-4x32-10 mask)

_U64 = ctypes.c_uint64
_lib.qlora_bwd_dropout_workspace_size.argtypes = [_I64, _I64, _I64, _I32]
_lib.qlora_bwd_dropout_workspace_size.restype = _SZ
_lib.qlora_linear_fwd_dropout.argtypes = [_P, _I64, _NF4Weight, _P, _P, _I32, ctypes.c_float, ctypes.c_float, _U64,
                                          _P, _P, _I32, _P, _P, _SZ, _P, _P]
_lib.qlora_linear_fwd_dropout.restype = ctypes.c_int
_lib.qlora_linear_bwd_dropout.argtypes = [_P, _P, _P, _I64, _NF4Weight, _P, _P, _I32, ctypes.c_float, ctypes.c_float,
                                          _U64, _P, _I32, _P, _P, _P, _SZ, _P, _P]
_lib.qlora_linear_bwd_dropout.restype = ctypes.c_int

EXPORTED = EXPORTED + ("qlora_bwd_dropout_workspace_size", "qlora_linear_fwd_dropout", "qlora_linear_bwd_dropout")


def qlora_bwd_dropout_workspace_size(M, N, K, r):
    return int(_lib.qlora_bwd_dropout_workspace_size(M, N, K, r))


def qlora_linear_fwd_dropout(X, W, A, B, s, p, seed, y_dtype=DTYPE_BF16, Y=None, U=None, X_drop=None, ws=None,
                             status=None, stream=None):
    """Forward with dropout (probability ``p``, Philox ``seed``) on the adapter
    input; returns ``(Y, U, X_drop)`` (keep X_drop for the backward)."""
    M = X.shape[0]
    N, K, r = int(W.n_out), int(W.k_in), A.shape[0]
    dev = X.device
    if Y is None:
        Y = torch.empty((M, N), dtype=torch.float32 if y_dtype == DTYPE_F32 else torch.bfloat16, device=dev)
    if U is None:
        U = torch.empty((M, r), dtype=torch.float32, device=dev)
    if X_drop is None:
        X_drop = torch.empty((M, K), dtype=torch.bfloat16, device=dev)
    if ws is None:
        ws = torch.empty(max(qlora_fwd_workspace_size(M, N, K, r), 16), dtype=torch.uint8, device=dev)
    _check(_lib.qlora_linear_fwd_dropout(_ptr(X), M, _weight(W), _ptr(A), _ptr(B), r, float(s), float(p), int(seed),
                                         _ptr(X_drop), _ptr(Y), y_dtype, _ptr(U), _ptr(ws), ws.numel(), _ptr(status),
                                         _stream(stream)),
           "qlora_linear_fwd_dropout")
    return Y, U, X_drop


def qlora_linear_bwd_dropout(dY, X_drop, U, W, A, B, s, p, seed, dx_dtype=DTYPE_BF16, dX=None, dA=None, dB=None,
                             ws=None, status=None, stream=None):
    """Backward of :func:`qlora_linear_fwd_dropout` (same ``p`` and ``seed``);
    returns ``(dX, dA, dB)``."""
    M = X_drop.shape[0]
    N, K, r = int(W.n_out), int(W.k_in), A.shape[0]
    dev = X_drop.device
    if dX is None:
        dX = torch.empty((M, K), dtype=torch.float32 if dx_dtype == DTYPE_F32 else torch.bfloat16, device=dev)
    if dA is None:
        dA = torch.empty((r, K), dtype=torch.float32, device=dev)
    if dB is None:
        dB = torch.empty((N, r), dtype=torch.float32, device=dev)
    if ws is None:
        ws = torch.empty(max(qlora_bwd_dropout_workspace_size(M, N, K, r), 16), dtype=torch.uint8, device=dev)
    _check(_lib.qlora_linear_bwd_dropout(_ptr(dY), _ptr(X_drop), _ptr(U), M, _weight(W), _ptr(A), _ptr(B), r,
                                         float(s), float(p), int(seed), _ptr(dX), dx_dtype, _ptr(dA), _ptr(dB),
                                         _ptr(ws), ws.numel(), _ptr(status), _stream(stream)),
           "qlora_linear_bwd_dropout")
    return dX, dA, dB


# ------------------------------------------------------ bounded-wait self-test

_lib.qlora_selftest_timeout.argtypes = [_P, _I64, _P]
_lib.qlora_selftest_timeout.restype = ctypes.c_int
EXPORTED = EXPORTED + ("qlora_selftest_timeout",)


def qlora_selftest_timeout(status, limit_ns, stream=None):
    """Run the kernels' bounded wait against a barrier nothing completes, with
    a ``limit_ns`` limit; sets DEV_TIMEOUT in the int32 device tensor ``status``."""
    _check(_lib.qlora_selftest_timeout(_ptr(status), int(limit_ns), _stream(stream)), "qlora_selftest_timeout")


# ------------------------------------------------------ few-token kernel choice

_lib.qlora_set_few_token_threshold.argtypes = [_I64]
_lib.qlora_set_few_token_threshold.restype = _I64
EXPORTED = EXPORTED + ("qlora_set_few_token_threshold",)
DEFAULT_FEW_TOKEN_THRESHOLD = 1 << 26


def qlora_set_few_token_threshold(min_weight_elems):
    """Weights of at least this many elements run the few-token kernel for
    M <= 16 tokens (0: always, a huge value: never); returns the previous value."""
    return int(_lib.qlora_set_few_token_threshold(int(min_weight_elems)))


# ------------------------------------------------------ grouped projections
# (include/qlora_nf4.h: linears sharing one input, stacked along the outputs)

_lib.qlora_group_fwd_workspace_size.argtypes = [_I64, _I64, _I64, _I32, _I32]
_lib.qlora_group_fwd_workspace_size.restype = _SZ
_lib.qlora_group_bwd_workspace_size.argtypes = [_I64, _I64, _I64, _I32, _I32]
_lib.qlora_group_bwd_workspace_size.restype = _SZ
_lib.qlora_group_fwd.argtypes = [_P, _I64, _NF4Weight, _I32, _P, _P, _P, _I32, ctypes.c_float, _P, _I32, _P, _P,
                                 _SZ, _P, _P]
_lib.qlora_group_fwd.restype = ctypes.c_int
_lib.qlora_group_bwd.argtypes = [_P, _P, _P, _I64, _NF4Weight, _I32, _P, _P, _P, _I32, ctypes.c_float, _P, _I32,
                                 _P, _P, _P, _SZ, _P, _P]
_lib.qlora_group_bwd.restype = ctypes.c_int

EXPORTED = EXPORTED + ("qlora_group_fwd_workspace_size", "qlora_group_bwd_workspace_size", "qlora_group_fwd",
                       "qlora_group_bwd")


def qlora_group_fwd_workspace_size(M, N, K, members, r):
    return int(_lib.qlora_group_fwd_workspace_size(M, N, K, members, r))


def qlora_group_bwd_workspace_size(M, N, K, members, r):
    return int(_lib.qlora_group_bwd_workspace_size(M, N, K, members, r))


def _members(n_member):
    arr = (ctypes.c_int64 * len(n_member))(*[int(n) for n in n_member])
    return len(n_member), arr


def quantize_group(weights, stream=None):
    """NF4-quantise the members of a group (bf16 [n_g, K] each) as one stacked
    weight; returns ``(NF4Weight [sum n_g, K], [n_g ...])``."""
    stacked = torch.cat([w.reshape(w.shape[0], -1) for w in weights], 0).contiguous()
    return quantize_weight(stacked, stream=stream), [int(w.shape[0]) for w in weights]


def qlora_group_fwd(X, W, n_member, A, B, s, y_dtype=DTYPE_BF16, Y=None, U=None, ws=None, status=None, stream=None):
    """Forward of a group of linears sharing ``X``: W stacked [N, K], A [G r, K],
    B [N, r]; returns ``(Y [M, N], U [M, G r])``."""
    M = X.shape[0]
    G, arr = _members(n_member)
    N, K, r = int(W.n_out), int(W.k_in), A.shape[0] // G
    dev = X.device
    if Y is None:
        Y = torch.empty((M, N), dtype=torch.float32 if y_dtype == DTYPE_F32 else torch.bfloat16, device=dev)
    if U is None:
        U = torch.empty((M, G * r), dtype=torch.float32, device=dev)
    if ws is None:
        ws = torch.empty(max(qlora_group_fwd_workspace_size(M, N, K, G, r), 16), dtype=torch.uint8, device=dev)
    _check(_lib.qlora_group_fwd(_ptr(X), M, _weight(W), G, ctypes.cast(arr, _P), _ptr(A), _ptr(B), r, float(s),
                                _ptr(Y), y_dtype, _ptr(U), _ptr(ws), ws.numel(), _ptr(status), _stream(stream)),
           "qlora_group_fwd")
    return Y, U


def qlora_group_bwd(dY, X, U, W, n_member, A, B, s, dx_dtype=DTYPE_BF16, dX=None, dA=None, dB=None, ws=None,
                    status=None, stream=None):
    """Backward of :func:`qlora_group_fwd`; returns ``(dX [M, K] summed over the
    members, dA [G r, K], dB [N, r])``."""
    M = X.shape[0]
    G, arr = _members(n_member)
    N, K, r = int(W.n_out), int(W.k_in), A.shape[0] // G
    dev = X.device
    if dX is None:
        dX = torch.empty((M, K), dtype=torch.float32 if dx_dtype == DTYPE_F32 else torch.bfloat16, device=dev)
    if dA is None:
        dA = torch.empty((G * r, K), dtype=torch.float32, device=dev)
    if dB is None:
        dB = torch.empty((N, r), dtype=torch.float32, device=dev)
    if ws is None:
        ws = torch.empty(max(qlora_group_bwd_workspace_size(M, N, K, G, r), 16), dtype=torch.uint8, device=dev)
    _check(_lib.qlora_group_bwd(_ptr(dY), _ptr(X), _ptr(U), M, _weight(W), G, ctypes.cast(arr, _P), _ptr(A),
                                _ptr(B), r, float(s), _ptr(dX), dx_dtype, _ptr(dA), _ptr(dB), _ptr(ws), ws.numel(),
                                _ptr(status), _stream(stream)),
           "qlora_group_bwd")
    return dX, dA, dB


# ------------------------------------------ mean-centred double quantisation

_lib.nf4_centered_workspace_size.argtypes = [_I64]
_lib.nf4_centered_workspace_size.restype = _SZ
_lib.nf4_quantize_centered.argtypes = [_P, _I64, _P, _P, _P, _P, _P, _SZ, _P, _P]
_lib.nf4_quantize_centered.restype = ctypes.c_int
_lib.nf4_dequantize_centered.argtypes = [_P, _P, _P, _P, _I64, _P, _P]
_lib.nf4_dequantize_centered.restype = ctypes.c_int

EXPORTED = EXPORTED + ("nf4_centered_workspace_size", "nf4_quantize_centered", "nf4_dequantize_centered")


def nf4_centered_workspace_size(numel):
    return int(_lib.nf4_centered_workspace_size(numel))


def nf4_quantize_centered(w, codes=None, c8=None, s2=None, mean=None, ws=None, status=None, stream=None):
    """Quantise a bf16 CUDA tensor with mean-centred constants; returns
    ``(codes, c8, s2, mean)`` (allocated if not given; mean is fp32 [1])."""
    assert w.dtype == torch.bfloat16 and w.is_cuda and w.is_contiguous()
    numel = w.numel()
    nc, nb, ns = nf4_sizes(numel)
    dev = w.device
    codes = torch.empty(nc, dtype=torch.uint8, device=dev) if codes is None else codes
    c8 = torch.empty(nb, dtype=torch.uint8, device=dev) if c8 is None else c8
    s2 = torch.empty(ns, dtype=torch.float32, device=dev) if s2 is None else s2
    mean = torch.empty(4, dtype=torch.float32, device=dev)[:1] if mean is None else mean
    if ws is None:
        ws = torch.empty(max(nf4_centered_workspace_size(numel), 16), dtype=torch.uint8, device=dev)
    _check(_lib.nf4_quantize_centered(_ptr(w), numel, _ptr(codes), _ptr(c8), _ptr(s2), _ptr(mean), _ptr(ws),
                                      ws.numel(), _ptr(status), _stream(stream)), "nf4_quantize_centered")
    return codes, c8, s2, mean


def quantize_weight_centered(w, stream=None):
    """NF4-quantise a bf16 weight [n_out, k_in] with mean-centred constants;
    returns an :class:`NF4Weight` whose ``mean`` is set."""
    codes, c8, s2, mean = nf4_quantize_centered(w, stream=stream)
    return NF4Weight(codes, c8, s2, w.shape[0], w.shape[1], mean)


def nf4_dequantize_centered(codes, c8, s2, mean, numel, out=None, stream=None):
    """bf16 tensor of ``numel`` values dequantised with mean-centred constants."""
    out = torch.empty(numel, dtype=torch.bfloat16, device=codes.device) if out is None else out
    _check(_lib.nf4_dequantize_centered(_ptr(codes), _ptr(c8), _ptr(s2), _ptr(mean), numel, _ptr(out),
                                        _stream(stream)), "nf4_dequantize_centered")
    return out

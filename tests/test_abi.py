"""Host-only checks of the C ABI: the library loads, exports every declared
symbol, derives the same NF4 levels as the oracle, sizes its workspaces, and
rejects bad arguments before touching a device.  No GPU needed; no test here
enqueues device work."""

import ctypes
import os
import re

import numpy as np
import pytest
import torch

import bit_nf4_quantized_26_b200 as q
from oracle import nf4

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADERS = [os.path.join(ROOT, "include", h) for h in ("qlora_nf4.h", "qlora_optim.h")]

OK, NULL, SHAPE, ALIGN, WS, CUDA, ARCH, DTYPE = 0, 1, 2, 3, 4, 7, 8, 9


def declared_functions():
    text = "".join(open(h).read() for h in HEADERS)
    return sorted(set(re.findall(r"QLORA_API\s+[\w\s\*]+?\b(\w+)\s*\(", text)))


def test_header_declarations_are_exported():
    names = declared_functions()
    assert len(names) == 28
    lib = q.raw()
    for n in names:
        assert hasattr(lib, n), n
    assert sorted(q.EXPORTED) == names


def test_library_levels_equal_oracle_codebook():
    """The library's codebook (bisection on erfc, C++) and the oracle's
    (Wichura AS241, Python) are independent derivations of the same levels."""
    lib_levels = np.array(q.nf4_levels(), dtype=np.float32)
    assert np.array_equal(lib_levels.view(np.uint32), nf4.codebook().view(np.uint32))


def test_strerror():
    for code in range(11):
        assert isinstance(q.qlora_strerror(code), str) and q.qlora_strerror(code)
    assert q.qlora_strerror(0) == "ok"


def test_workspace_sizes():
    assert q.qlora_fwd_workspace_size(0, 4096, 4096, 64) == 0
    assert q.qlora_bwd_workspace_size(0, 4096, 4096, 64) == 0
    a = q.qlora_fwd_workspace_size(4096, 4096, 4096, 64)
    b = q.qlora_fwd_workspace_size(8192, 4096, 4096, 64)
    assert 0 < a <= b
    assert q.qlora_fwd_workspace_size(4096, 4096, 4096, 64) % 256 == 0
    assert q.qlora_bwd_workspace_size(4096, 4096, 4096, 64) >= 4096 * 2 * 64 * 2 * 2
    # small M uses split-K partials: still bounded by S * M * N * 4
    assert q.qlora_fwd_workspace_size(1, 22016, 8192, 64) < 300 * 22016 * 4 + (1 << 20)


# ----------------------------------------------------------- argument checks

FAKE = 1 << 20  # a 16-byte aligned non-null value; never dereferenced


def _w(codes=FAKE, c8=FAKE, s2=FAKE, n=4096, k=4096):
    return q._NF4Weight(codes, c8, s2, n, k)


def _fwd(X=FAKE, M=64, W=None, A=FAKE, B=FAKE, r=64, Y=FAKE, ydt=0, U=FAKE, ws=FAKE, wsb=1 << 40,
         status=None):
    W = _w() if W is None else W
    return q.raw().qlora_linear_fwd(X, M, W, A, B, r, 0.25, Y, ydt, U, ws, wsb, status, None)


def _bwd(dY=FAKE, X=FAKE, U=FAKE, M=64, W=None, A=FAKE, B=FAKE, r=64, dX=FAKE, dxdt=0, dA=FAKE, dB=FAKE,
         ws=FAKE, wsb=1 << 40):
    W = _w() if W is None else W
    return q.raw().qlora_linear_bwd(dY, X, U, M, W, A, B, r, 0.25, dX, dxdt, dA, dB, ws, wsb, None, None)


def test_fwd_argument_errors():
    assert _fwd(X=None) == NULL
    assert _fwd(W=_w(codes=None)) == NULL
    assert _fwd(U=None) == NULL
    assert _fwd(W=_w(k=4096 + 32)) == SHAPE          # K % 64 != 0
    assert _fwd(W=_w(n=4096 + 16)) == SHAPE          # N % 64 != 0
    assert _fwd(r=8) == SHAPE and _fwd(r=24) == SHAPE and _fwd(r=320) == SHAPE and _fwd(r=272) == SHAPE
    for r in (80, 128, 144, 192, 240, 256):
        assert _fwd(M=0, r=r, X=None, Y=None, U=None, ws=None) == OK   # accepted: no-op
        assert _bwd(M=0, r=r, dY=None) == OK
    assert _fwd(M=-1) == SHAPE
    assert _fwd(X=FAKE + 8) == ALIGN
    assert _fwd(W=_w(c8=FAKE + 4)) == ALIGN
    assert _fwd(ydt=7) == DTYPE
    assert _fwd(ws=None) == WS
    assert _fwd(wsb=16) == WS
    assert _fwd(M=0, X=None, Y=None, U=None, ws=None) == OK   # no-op


def _noalloc(X=FAKE, M=64, W=None, A=FAKE, B=FAKE, r=64, Y=FAKE, ydt=0, U=FAKE, status=None):
    W = _w() if W is None else W
    return q.raw().qlora_linear_fwd_noalloc(X, M, W, A, B, r, 0.25, Y, ydt, U, status, None)


def test_noalloc_argument_errors_match_the_forward():
    """The allocation-free forward makes the forward's checks in the same
    order, and refuses a problem whose workspace exceeds its fixed 16 MiB
    scratch, all before touching a device."""
    wsmall = _w(n=128, k=128)
    assert q.qlora_fwd_workspace_size(70000, 128, 128, 64) > 16 << 20
    assert _noalloc(M=70000, W=wsmall) == WS
    assert _noalloc(r=8) == SHAPE
    assert _noalloc(M=1 << 31) == SHAPE
    assert _noalloc(M=0, ydt=7) == DTYPE == _fwd(M=0, ydt=7)
    assert _noalloc(M=0, X=None, Y=None, U=None) == OK
    assert _noalloc(X=None) == NULL
    assert _noalloc(X=FAKE + 8) == ALIGN
    assert _noalloc(W=_w(codes=None)) == NULL


def test_group_argument_errors():
    """Grouped projections: 1..4 members, each a multiple of 128 rows (64 for
    one member), summing to the stacked weight's rows; checked on the host."""
    f = q.raw().qlora_group_fwd
    b = q.raw().qlora_group_bwd

    def members(*n):
        return ctypes.cast((ctypes.c_int64 * len(n))(*n), ctypes.c_void_p)

    def fwd(G, nm, W=None, M=64, ydt=0):
        W = _w(n=4096 * 3) if W is None else W
        return f(FAKE, M, W, G, nm, FAKE, FAKE, 64, 0.25, FAKE, ydt, FAKE, FAKE, 1 << 40, None, None)

    assert fwd(3, None) == NULL
    assert fwd(0, members(4096)) == SHAPE and fwd(5, members(*[2048] * 5)) == SHAPE
    assert fwd(3, members(4096, 4096, 4032)) == SHAPE          # sum != stacked rows
    assert fwd(2, members(6080, 6208), W=_w(n=12288)) == SHAPE  # 6080 % 128 != 0
    assert fwd(3, members(4096, 4096, 4096), ydt=5) == DTYPE
    assert fwd(3, members(4096, 4096, 4096), M=0) == OK
    assert b(FAKE, FAKE, FAKE, 64, _w(n=8192), 2, members(4096, 4096), FAKE, FAKE, 8, 0.25, FAKE, 0, FAKE, FAKE,
             FAKE, 1 << 40, None, None) == SHAPE                # r = 8
    # members of a real group take r <= 64; one member is a single linear
    assert b(FAKE, FAKE, FAKE, 64, _w(n=8192), 2, members(4096, 4096), FAKE, FAKE, 128, 0.25, FAKE, 0, FAKE, FAKE,
             FAKE, 1 << 40, None, None) == SHAPE
    assert f(FAKE, 64, _w(n=8192), 2, members(4096, 4096), FAKE, FAKE, 128, 0.25, FAKE, 0, FAKE, FAKE, 1 << 40,
             None, None) == SHAPE
    assert f(FAKE, 0, _w(n=8192), 1, members(8192), FAKE, FAKE, 128, 0.25, FAKE, 0, FAKE, FAKE, 1 << 40,
             None, None) == OK
    assert b(FAKE, FAKE, FAKE, 64, _w(n=8192), 2, members(4096, 4096), FAKE, FAKE, 64, 0.25, FAKE, 0, FAKE, FAKE,
             FAKE, 16, None, None) == WS
    assert q.qlora_group_fwd_workspace_size(4096, 12288, 4096, 1, 64) == q.qlora_fwd_workspace_size(4096, 12288,
                                                                                                    4096, 64)
    assert q.qlora_group_bwd_workspace_size(4096, 12288, 4096, 3, 64) > q.qlora_bwd_workspace_size(4096, 12288,
                                                                                                   4096, 64)


def test_centred_quantize_argument_errors():
    lib = q.raw()
    assert q.nf4_centered_workspace_size(0) == 0
    assert q.nf4_centered_workspace_size(16384 * 3) == 256 * 3 * 4 + 256 + 2 * 256  # constants, group sums, two pass buffers
    assert lib.nf4_quantize_centered(FAKE, 64, FAKE, FAKE, FAKE, None, FAKE, 1 << 20, None, None) == NULL  # mean
    assert lib.nf4_quantize_centered(FAKE, 64, FAKE, FAKE, FAKE, FAKE + 4, FAKE, 1 << 20, None, None) == ALIGN
    assert lib.nf4_quantize_centered(FAKE, 64, FAKE, FAKE, FAKE, FAKE, FAKE, 16, None, None) == WS
    assert lib.nf4_quantize_centered(FAKE, -1, FAKE, FAKE, FAKE, FAKE, FAKE, 1 << 20, None, None) == SHAPE
    assert lib.nf4_quantize_centered(None, 0, None, None, None, None, None, 0, None, None) == OK
    assert lib.nf4_dequantize_centered(FAKE, FAKE, FAKE, None, 64, FAKE, None) == NULL
    w = q._NF4Weight(FAKE, FAKE, FAKE, 4096, 4096, FAKE + 8)   # misaligned mean pointer
    assert q.raw().qlora_linear_fwd(FAKE, 64, w, FAKE, FAKE, 64, 0.25, FAKE, 0, FAKE, FAKE, 1 << 40, None,
                                    None) == ALIGN


def test_bwd_argument_errors():
    assert _bwd(dY=None) == NULL
    assert _bwd(dB=None) == NULL
    assert _bwd(W=_w(k=100)) == SHAPE
    assert _bwd(dA=FAKE + 2) == ALIGN
    assert _bwd(dxdt=3) == DTYPE
    assert _bwd(wsb=0) == WS
    assert _bwd(M=0, dY=None) == OK


def test_quantize_argument_errors():
    lib = q.raw()
    assert lib.nf4_quantize(None, 64, FAKE, FAKE, FAKE, None, None) == NULL
    assert lib.nf4_quantize(FAKE, -5, FAKE, FAKE, FAKE, None, None) == SHAPE
    assert lib.nf4_quantize(FAKE + 2, 64, FAKE, FAKE, FAKE, None, None) == ALIGN
    assert lib.nf4_quantize(None, 0, None, None, None, None, None) == OK
    assert lib.nf4_dequantize(FAKE, None, FAKE, 64, FAKE, None) == NULL
    assert lib.nf4_dequantize(FAKE, FAKE, FAKE, 64, FAKE + 1, None) == ALIGN


@pytest.mark.skipif(torch.cuda.is_available(), reason="would reach the device with fake pointers")
def test_valid_arguments_without_device_fail_cleanly():
    """With every argument valid but no usable sm_100 device the call returns an
    error status (never crashes, never falls back)."""
    assert _fwd() in (CUDA, ARCH)
    assert q.raw().nf4_quantize(FAKE, 64, FAKE, FAKE, FAKE, None, None) in (CUDA, ARCH)


def test_adamw8_rejects_bad_arguments_before_touching_a_device():
    """Sizes, step and hyper-parameters are checked first, then pointers and
    alignment; none of these reach the device."""
    f = q._lib.qlora_adamw8_step
    P = ctypes.c_void_p
    good = [P(256)] * 6
    def call(ptrs=good, n=10, lr=1e-3, b1=0.9, b2=0.999, eps=1e-8, wd=0.0, step=1):
        return f(*ptrs, n, lr, b1, b2, eps, wd, step, None, None)
    assert call(n=-1) == SHAPE
    assert call(n=1 << 40) == SHAPE
    assert call(step=0) == SHAPE
    assert call(b1=1.0) == SHAPE and call(b2=-0.1) == SHAPE and call(b1=float("nan")) == SHAPE
    assert call(eps=-1e-8) == SHAPE and call(lr=float("inf")) == SHAPE and call(wd=float("nan")) == SHAPE
    assert call(n=0) == OK
    assert call(ptrs=[None] + good[1:]) == NULL
    assert call(ptrs=good[:3] + [None] + good[4:]) == NULL
    assert call(ptrs=[P(256 + 8)] + good[1:]) == ALIGN
    assert call(ptrs=good[:5] + [P(256 + 4)]) == ALIGN


def test_paged_calls_reject_null_pointers():
    assert q._lib.qlora_paged_alloc(None, 16) == NULL
    assert q._lib.qlora_paged_prefetch(None, 16, 0, None) == NULL
    assert q._lib.qlora_paged_free(None) == OK


def test_dropout_rejects_bad_probability_before_touching_a_device():
    f = q._lib.qlora_linear_fwd_dropout
    P = ctypes.c_void_p
    w = q._NF4Weight(256, 256, 256, 4096, 4096)
    for p in (-0.1, 1.0, float("nan")):
        assert f(P(256), 64, w, P(256), P(256), 16, 1.0, p, 7, P(256), P(256), 0, P(256), P(256), 1 << 20,
                 None, None) == SHAPE
    g = q._lib.qlora_linear_bwd_dropout
    assert g(P(256), P(256), P(256), 64, w, P(256), P(256), 16, 1.0, 1.5, 7, P(256), 0, P(256), P(256), P(256),
             1 << 20, None, None) == SHAPE
    assert f(P(256), 64, w, P(256), P(256), 16, 1.0, 0.1, 7, None, P(256), 0, P(256), P(256), 1 << 20,
             None, None) == NULL
    # ranks as for the plain linear: up to 256 in steps of 16
    assert f(P(256), 64, w, P(256), P(256), 272, 1.0, 0.1, 7, P(256), P(256), 0, P(256), P(256), 1 << 20,
             None, None) == SHAPE
    assert f(P(256), 0, w, P(256), P(256), 144, 1.0, 0.1, 7, P(256), P(256), 0, P(256), P(256), 1 << 20,
             None, None) == OK
    assert g(P(256), P(256), P(256), 64, w, P(256), P(256), 80 + 4, 1.0, 0.1, 7, P(256), 0, P(256), P(256),
             P(256), 1 << 20, None, None) == SHAPE
    assert q.qlora_bwd_dropout_workspace_size(4096, 4096, 4096, 64) == \
        q.qlora_bwd_workspace_size(4096, 4096, 4096, 64) + 4096 * 4096 * 4


def test_selftest_timeout_argument_checks():
    f = q._lib.qlora_selftest_timeout
    P = ctypes.c_void_p
    assert f(None, 5_000_000, None) == NULL
    assert f(P(256), 10, None) == SHAPE
    assert f(P(256), 3_000_000_000, None) == SHAPE
    assert f(P(260), 5_000_000, None) == ALIGN


def test_few_token_threshold_setting():
    """The setter returns the previous value (default 2^26 elements) and
    changes the forward's plan: M <= 16 on a small weight uses the few-token
    kernel's partial buffers only when forced (host-only workspace queries)."""
    prev = q.qlora_set_few_token_threshold(0)
    assert prev == q.DEFAULT_FEW_TOKEN_THRESHOLD
    try:
        forced = q.qlora_fwd_workspace_size(8, 512, 512, 16)
        assert q.qlora_set_few_token_threshold(1 << 62) == 0
        mid = q.qlora_fwd_workspace_size(8, 512, 512, 16)
        assert forced != mid
        assert q.qlora_set_few_token_threshold(-5) == 1 << 62
        assert q.qlora_set_few_token_threshold(prev) == 0  # negative counts as 0
    finally:
        q.qlora_set_few_token_threshold(prev)

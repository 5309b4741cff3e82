"""The allocation-free forward, qlora_linear_fwd_noalloc, through the C ABI.

Callers that may not allocate device memory at call time (a plugin that a
host framework hands only its input and output buffers, or a loop that must
not let cudaMalloc/cudaFree synchronise the device) use this entry point: its
scratch is a fixed 16 MiB device array inside the library.  Calls in a row,
on different inputs and through different kernel paths, must each give
bitwise the same Y and U as qlora_linear_fwd (which takes a caller-provided
workspace and runs the same kernels), and match the fp64 oracle within the
tolerances of the other parity tests; a problem that needs more scratch than
the array holds must be refused before any work is enqueued.
"""

import ctypes

import numpy as np
import pytest
import torch

import synth
from oracle import linear as ol
from tests._util import bits, oracle_dequant_full, rel

pytestmark = pytest.mark.gpu

TOL_BF16 = 2e-3
TOL_F32 = 1e-4
ERR_WORKSPACE = 4


def _lib():
    import bit_nf4_quantized_26_b200 as lib
    return lib


def _p(t):
    return ctypes.c_void_p(t.data_ptr())


def _noalloc_raw(lib, X, W, A, B, s, Y, U, status):
    stream = ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    return lib.raw().qlora_linear_fwd_noalloc(_p(X), X.shape[0], lib._weight(W), _p(A), _p(B), A.shape[0],
                                              float(s), _p(Y), 0, _p(U), _p(status), stream)


def test_noalloc_forward_matches_workspace_forward_and_oracle(few_token_kernel):
    lib = _lib()
    # few-token kernel (split partials in the scratch), 64-token tiles with a
    # split contraction, and the CTA-pair kernel; one call after another
    cases = [(8, 2048, 4096, 64, 2), (64, 512, 512, 16, 0), (4096, 4096, 4096, 64, 1)]
    for M, N, K, r, seed in cases:
        cpu = synth.linear_inputs(synth.Linear("na", N, K), M, r, seed)
        d = {k: v.cuda() for k, v in cpu.items()}
        s = 16.0 / r
        W = lib.quantize_weight(d["W"])
        Y_ref, U_ref = lib.qlora_linear_fwd(d["X"], W, d["A"], d["B"], s)
        Y = torch.full((M, N), float("nan"), dtype=torch.bfloat16, device="cuda")
        U = torch.full((M, r), float("nan"), dtype=torch.float32, device="cuda")
        status = torch.zeros(4, dtype=torch.int32, device="cuda")
        assert _noalloc_raw(lib, d["X"], W, d["A"], d["B"], s, Y, U, status) == 0
        torch.cuda.synchronize()
        assert int(status[0].item()) == 0
        assert torch.equal(Y.view(torch.int16), Y_ref.view(torch.int16)), (M, N, K)
        assert torch.equal(U.view(torch.int32), U_ref.view(torch.int32)), (M, N, K)
        rows = np.unique(np.linspace(0, M - 1, min(M, 64)).astype(np.int64))
        Wd = oracle_dequant_full(bits(cpu["W"]))
        Ur, Yr = ol.linear_fwd(bits(cpu["X"])[rows], Wd, bits(cpu["A"]), bits(cpu["B"]), s)
        assert rel(Y.float().cpu().numpy()[rows], Yr) <= TOL_BF16
        assert rel(U.cpu().numpy()[rows], Ur) <= TOL_F32


def test_noalloc_refuses_problem_beyond_scratch():
    lib = _lib()
    M, N, K, r = 70000, 128, 128, 64
    assert lib.qlora_fwd_workspace_size(M, N, K, r) > 16 << 20
    d = {k: v.cuda() for k, v in synth.linear_inputs(synth.Linear("big", N, K), M, r, 3).items()}
    W = lib.quantize_weight(d["W"])
    Y = torch.empty((M, N), dtype=torch.bfloat16, device="cuda")
    U = torch.empty((M, r), dtype=torch.float32, device="cuda")
    status = torch.zeros(4, dtype=torch.int32, device="cuda")
    assert _noalloc_raw(lib, d["X"], W, d["A"], d["B"], 0.25, Y, U, status) == ERR_WORKSPACE

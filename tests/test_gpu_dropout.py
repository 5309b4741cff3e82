"""GPU parity of the LoRA-dropout forward and backward against the CPU oracle
(oracle/dropout.py): X_drop bit for bit, U / dA / dB within 1e-4 and Y / dX
within 2e-3 relative Frobenius error, on the few-token, split-K, CTA-pair and
single-CTA wide paths, and for ranks above 64."""

import numpy as np
import pytest
import torch

import bit_nf4_quantized_26_b200 as q
import synth
from oracle import dropout as dr
from oracle import linear as ol
from oracle import nf4

pytestmark = pytest.mark.gpu


def _bits(t):
    return t.detach().cpu().contiguous().view(torch.int16).numpy().view(np.uint16)


def _case(M, N, K, r, seed=0):
    d = synth.linear_inputs(synth.Linear("drop", N, K), M, r, seed)
    g = {k: v.cuda() for k, v in d.items() if k in ("W", "X", "dY", "A", "B")}
    W = q.quantize_weight(g["W"])
    codes, c8, s2 = nf4.quantize(_bits(d["W"]).reshape(-1))
    wd = nf4.dequantize(codes, c8, s2, d["W"].numel()).reshape(d["W"].shape)
    return d, g, W, wd


SHAPES = [(16, 320, 512, 16),     # few tokens (register path)
          (200, 512, 640, 32),    # split-K fused kernel
          (600, 512, 768, 64),    # CTA-pair kernels (rows % 256 == 0)
          (1000, 384, 512, 64),   # single-CTA wide kernel for the forward (384 rows)
          (150, 384, 448, 144),   # a rank above 64 (chunks of 64 and 16; dX pass over three rank blocks)
          (700, 512, 768, 256)]   # the widest rank on the CTA-pair kernels


@pytest.mark.parametrize("shape", SHAPES)
@pytest.mark.parametrize("p", [0.05, 0.5])
def test_dropout_forward_backward_match_oracle(shape, p, few_token_kernel):
    M, N, K, r = shape
    d, g, W, wd = _case(M, N, K, r)
    s, seed = 0.25, 1234567 + (1 << 33)
    Y, U, Xd = q.qlora_linear_fwd_dropout(g["X"], W, g["A"], g["B"], s, p, seed)
    dX, dA, dB = q.qlora_linear_bwd_dropout(g["dY"], Xd, U, W, g["A"], g["B"], s, p, seed)
    torch.cuda.synchronize()
    Xd_ref, U_ref, Y_ref = dr.linear_fwd_dropout(_bits(d["X"]), wd, _bits(d["A"]), _bits(d["B"]), s, p, seed)
    assert np.array_equal(_bits(Xd), Xd_ref)
    assert ol.rel_frobenius(U.cpu().numpy(), U_ref) <= 1e-4
    assert ol.rel_frobenius(Y.float().cpu().numpy(), Y_ref) <= 2e-3
    dX_ref, dA_ref, dB_ref, _ = dr.linear_bwd_dropout(_bits(d["dY"]), _bits(d["X"]), wd, _bits(d["A"]),
                                                      _bits(d["B"]), s, p, seed)
    assert ol.rel_frobenius(dX.float().cpu().numpy(), dX_ref) <= 2e-3
    assert ol.rel_frobenius(dA.cpu().numpy(), dA_ref) <= 1e-4
    assert ol.rel_frobenius(dB.cpu().numpy(), dB_ref) <= 1e-4


def test_dropout_adapter_term_of_dx_matches_oracle_in_fp32():
    """The masked dU A term alone (dX with dropout minus dX without it, both
    in fp32) against the oracle's keep * c * (dU A)."""
    M, N, K, r = 600, 512, 768, 64
    d, g, W, wd = _case(M, N, K, r, seed=3)
    s, p, seed = 1.0, 0.3, 99
    Y, U, Xd = q.qlora_linear_fwd_dropout(g["X"], W, g["A"], g["B"], s, p, seed)
    dX, _, _ = q.qlora_linear_bwd_dropout(g["dY"], Xd, U, W, g["A"], g["B"], s, p, seed, dx_dtype=q.DTYPE_F32)
    dX0, _, _ = q.qlora_linear_bwd(g["dY"], g["X"], U, W, g["A"], g["B"] * 0, s, dx_dtype=q.DTYPE_F32)
    torch.cuda.synchronize()
    dX_ref, _, _, dU = dr.linear_bwd_dropout(_bits(d["dY"]), _bits(d["X"]), wd, _bits(d["A"]), _bits(d["B"]), s, p,
                                             seed)
    term_ref = dX_ref - ol._f64(_bits(d["dY"])) @ ol._f64(wd)
    term = dX.cpu().numpy().astype(np.float64) - dX0.cpu().numpy().astype(np.float64)
    assert ol.rel_frobenius(term, term_ref) <= 1e-3


def test_dropout_p_zero_forward_equals_plain_forward(few_token_kernel):
    M, N, K, r = 600, 512, 768, 64
    d, g, W, wd = _case(M, N, K, r, seed=5)
    Y, U, Xd = q.qlora_linear_fwd_dropout(g["X"], W, g["A"], g["B"], 0.5, 0.0, 1)
    Y0, U0 = q.qlora_linear_fwd(g["X"], W, g["A"], g["B"], 0.5)
    torch.cuda.synchronize()
    assert torch.equal(Xd, g["X"])
    assert torch.equal(Y, Y0) and torch.equal(U, U0)

"""GPU parity of the fused QLoRA linear (forward and backward) against the fp64 oracle.

Bar (stated by the method's accuracy target): relative Frobenius error
<= 2e-3 for every output against the fp64 product on the same dequantised
weights.  bf16 rounding of Y or dX alone costs about 1.5e-3 of that budget on
Gaussian data.  fp32 outputs carry no such rounding, so they are held to a
tighter 1e-4, which catches mistakes that would hide under the bf16 bar.
Large shapes compare sampled token rows of Y and dX (each row is computed
independently) and the full dA, dB.
"""

import numpy as np
import pytest
import torch

import synth
from oracle import linear as ol
from tests._util import bits, oracle_dequant_full, oracle_dequant_rows, rel

pytestmark = pytest.mark.gpu

TOL_BF16 = 2e-3
TOL_F32 = 1e-4


def _lib():
    import bit_nf4_quantized_26_b200 as lib
    return lib


def _inputs(M, N, K, r, seed, outliers=False, w_zero=False, b_zero=False):
    d = synth.linear_inputs(synth.Linear("t", N, K), M, r, seed, outliers=outliers)
    if w_zero:
        d["W"] = torch.zeros_like(d["W"])
    if b_zero:
        d["B"] = torch.zeros_like(d["B"])
    return d


def _run_gpu(d, s, out_dtype):
    lib = _lib()
    g = {k: v.cuda() for k, v in d.items()}
    W = lib.quantize_weight(g["W"])
    status = torch.zeros(4, dtype=torch.int32, device="cuda")
    Y, U = lib.qlora_linear_fwd(g["X"], W, g["A"], g["B"], s, y_dtype=out_dtype, status=status)
    dX, dA, dB = lib.qlora_linear_bwd(g["dY"], g["X"], U, W, g["A"], g["B"], s, dx_dtype=out_dtype,
                                      status=status)
    torch.cuda.synchronize()
    assert int(status[0].item()) == 0
    return {k: v.float().cpu().numpy() for k, v in dict(Y=Y, U=U, dX=dX, dA=dA, dB=dB).items()}


def _check_full(M, N, K, r, s, seed, out_dtype=0, **kw):
    d = _inputs(M, N, K, r, seed, **kw)
    got = _run_gpu(d, s, out_dtype)
    Wd = oracle_dequant_full(bits(d["W"]))
    U, Y = ol.linear_fwd(bits(d["X"]), Wd, bits(d["A"]), bits(d["B"]), s)
    dX, dA, dB, _ = ol.linear_bwd(bits(d["dY"]), bits(d["X"]), Wd, bits(d["A"]), bits(d["B"]), s)
    tol = TOL_F32 if out_dtype == 1 else TOL_BF16
    errs = dict(Y=rel(got["Y"], Y), dX=rel(got["dX"], dX), U=rel(got["U"], U), dA=rel(got["dA"], dA),
                dB=rel(got["dB"], dB))
    assert errs["Y"] <= tol and errs["dX"] <= tol, errs
    assert errs["U"] <= TOL_F32 and errs["dA"] <= TOL_F32 and errs["dB"] <= TOL_F32, errs
    return errs


# ---------------------------------------------------------------- small, full

def test_c1_full_bf16():
    """512x512 linear, 64 tokens, r=16, alpha=16 (s=1), seed 0."""
    _check_full(64, 512, 512, 16, 1.0, 0)


def test_c1_full_f32_outputs():
    _check_full(64, 512, 512, 16, 1.0, 0, out_dtype=1)


@pytest.mark.parametrize("M,N,K,r", [
    (1, 192, 256, 16), (16, 256, 192, 32), (63, 320, 448, 48), (65, 128, 128, 64),
    (300, 192, 320, 64), (128, 64, 64, 16), (257, 384, 576, 64), (33, 64, 1024, 32),
    (700, 320, 448, 48), (1000, 192, 576, 16), (513, 128, 128, 64), (2000, 384, 192, 32),
    (700, 256, 512, 48), (1300, 512, 256, 16), (600, 768, 1024, 64),
    # extremes of the shape rules: K = 64 (one block per row: two 32-deep
    # stages in the CTA pair, one 64-deep stage in the mid-size kernel),
    # N = 64 (a single half-filled W tile), an odd large M
    (1024, 256, 64, 16), (257, 256, 64, 64), (100, 512, 64, 32), (300, 64, 4096, 64),
    (4097, 128, 128, 16),
])
def test_ragged_shapes(M, N, K, r):
    _check_full(M, N, K, r, 16.0 / r, M + N + K, out_dtype=1)
    _check_full(M, N, K, r, 16.0 / r, M + N + K, out_dtype=0)


@pytest.mark.parametrize("M,N,K,r", [
    (100, 512, 384, 128),     # mid-size forward and dX
    (12, 4096, 16384, 128),   # few tokens on a 2^26 weight: the mid-size kernel (the few-token one takes r <= 64)
    (700, 512, 768, 256),     # CTA-pair forward and dX (W rows and K multiples of 256)
    (600, 320, 448, 192),     # the 512-token single-CTA kernels both ways
    (257, 256, 64, 256),      # K = 64 with the widest rank
    (80, 384, 320, 80),       # a last chunk of 16 (mid-size kernels)
    (900, 768, 512, 160),     # a last chunk of 32 (CTA pair both ways)
    (520, 448, 704, 240),     # a last chunk of 48 (the 512-token single-CTA kernels)
])
def test_ranks_above_64(M, N, K, r):
    """Ranks above 64 run U, dU, dB and dA as chunks of 64 (the layout of a
    group's members; the last chunk r - 64 (chunks - 1) wide) and the whole
    rank in the GEMMs' adapter stages: the same tolerances against the
    oracle, fp32 and bf16 outputs."""
    _check_full(M, N, K, r, 16.0 / r, 11 * M + N + K + r, out_dtype=1)
    _check_full(M, N, K, r, 16.0 / r, 11 * M + N + K + r, out_dtype=0)


@pytest.mark.parametrize("M,N,K,r", [
    (1, 64, 64, 16), (3, 320, 832, 48), (8, 448, 1344, 64), (9, 128, 64, 16),
    (12, 1088, 2112, 32), (16, 960, 4160, 64), (5, 4096, 256, 16), (7, 2048, 8192, 64),
    (11, 1024, 16384, 48), (16, 4096, 4096, 32), (17, 320, 832, 48), (24, 1088, 2112, 64),
    (32, 960, 4160, 16), (29, 2048, 8192, 32),
])
def test_few_tokens(M, N, K, r, few_token_kernel):
    """M <= 16: the few-token kernel, forced whatever the weight's size: row
    tiles with a half-empty last tile (N % 128 = 64), K chunks with 1..3 of
    their 4 blocks present, 1..19 units per CTA, ranges that start and end
    inside a tile, r = 16..64, 1 and 2 token tiles of 8.  M = 17..32: the
    mid-size kernel with 32-token tiles."""
    _check_full(M, N, K, r, 16.0 / r, 3 * M + N + K, out_dtype=1)
    _check_full(M, N, K, r, 16.0 / r, 3 * M + N + K, out_dtype=0)


@pytest.mark.parametrize("M,N,K,r", [(1, 64, 64, 16), (12, 1088, 2112, 32), (16, 4096, 4096, 32), (9, 4096, 11008, 64)])
def test_few_tokens_default_dispatch(M, N, K, r):
    """With the library's default threshold a weight below 2^26 elements runs
    few tokens on the mid-size kernel: the same tolerances."""
    _check_full(M, N, K, r, 16.0 / r, 5 * M + N + K, out_dtype=1)


def test_few_tokens_forward_is_deterministic(few_token_kernel):
    lib = _lib()
    d = {k: v.cuda() for k, v in _inputs(13, 2048, 8192, 64, 12).items()}
    W = lib.quantize_weight(d["W"])
    y1, u1 = lib.qlora_linear_fwd(d["X"], W, d["A"], d["B"], 0.25)
    y2, u2 = lib.qlora_linear_fwd(d["X"], W, d["A"], d["B"], 0.25)
    torch.cuda.synchronize()
    assert torch.equal(y1.view(torch.int16), y2.view(torch.int16))
    assert torch.equal(u1.view(torch.int32), u2.view(torch.int32))


@pytest.mark.parametrize("M,N,K,r", [(9, 4096, 11008, 64), (100, 4096, 11008, 64), (48, 2048, 8192, 32)])
def test_mid_size_repeatable_under_churn(M, N, K, r):
    """Mid-size GEMMs with split contractions and two dequantiser groups over
    a three-stage ring: every repetition, with other work between them to
    shift the copies' timing, gives the same bits (a stage dequantised from a
    stale ring slot shows as a tile that differs), and the first matches the
    oracle."""
    lib = _lib()
    d = {k: v.cuda() for k, v in _inputs(M, N, K, r, 7 * M + r).items()}
    W = lib.quantize_weight(d["W"])
    churn = torch.empty(64 << 20, dtype=torch.float32, device="cuda")  # 256 MB: more than L2
    y0, u0 = lib.qlora_linear_fwd(d["X"], W, d["A"], d["B"], 0.5)
    g0 = lib.qlora_linear_bwd(d["dY"], d["X"], u0, W, d["A"], d["B"], 0.5)
    for i in range(12):
        churn.add_(1.0)
        y, u = lib.qlora_linear_fwd(d["X"], W, d["A"], d["B"], 0.5)
        g = lib.qlora_linear_bwd(d["dY"], d["X"], u, W, d["A"], d["B"], 0.5)
        torch.cuda.synchronize()
        assert torch.equal(y.view(torch.int16), y0.view(torch.int16)), f"Y differs at repetition {i}"
        assert torch.equal(g[0].view(torch.int16), g0[0].view(torch.int16)), f"dX differs at repetition {i}"
    got = {"Y": y0.float().cpu().numpy(), "dX": g0[0].float().cpu().numpy()}
    Wd = oracle_dequant_full(bits(d["W"]))
    _, Y = ol.linear_fwd(bits(d["X"]), Wd, bits(d["A"]), bits(d["B"]), 0.5)
    assert rel(got["Y"], Y) <= TOL_BF16
    dX = ol.linear_bwd(bits(d["dY"]), bits(d["X"]), Wd, bits(d["A"]), bits(d["B"]), 0.5)[0]
    assert rel(got["dX"], dX) <= TOL_BF16


def test_lora_path_alone_w_zero():
    """W = 0: Y, dX come from the adapters alone (all codes 7, constants 0)."""
    _check_full(96, 256, 384, 64, 0.25, 7, out_dtype=1, w_zero=True)
    _check_full(96, 256, 384, 16, 1.0, 7, out_dtype=0, w_zero=True)


def test_base_path_alone_b_zero():
    """B = 0: Y = X W'^T, dU = 0, so dA must be exactly zero."""
    d = _inputs(80, 320, 256, 32, 8, b_zero=True)
    got = _run_gpu(d, 0.5, 1)
    assert np.all(got["dA"] == 0.0)
    Wd = oracle_dequant_full(bits(d["W"]))
    _, Y = ol.linear_fwd(bits(d["X"]), Wd, bits(d["A"]), bits(d["B"]), 0.5)
    assert rel(got["Y"], Y) <= TOL_F32


def test_backward_is_deterministic():
    lib = _lib()
    d = {k: v.cuda() for k, v in _inputs(1000, 512, 768, 64, 11).items()}
    W = lib.quantize_weight(d["W"])
    _, U = lib.qlora_linear_fwd(d["X"], W, d["A"], d["B"], 0.25)
    r1 = lib.qlora_linear_bwd(d["dY"], d["X"], U, W, d["A"], d["B"], 0.25)
    r2 = lib.qlora_linear_bwd(d["dY"], d["X"], U, W, d["A"], d["B"], 0.25)
    torch.cuda.synchronize()
    for a, b in zip(r1, r2):
        assert torch.equal(a.view(torch.int16) if a.dtype == torch.bfloat16 else a.view(torch.int32),
                           b.view(torch.int16) if b.dtype == torch.bfloat16 else b.view(torch.int32))


# ------------------------------------------------------- full-size, sampled

def _check_sampled(N, K, M, r, s, seed, outliers=False, nrows=96, bwd=True, ncols=192):
    lib = _lib()
    d = _inputs(M, N, K, r, seed, outliers=outliers)
    g = {k: v.cuda() for k, v in d.items()}
    W = lib.quantize_weight(g["W"])
    Y, U = lib.qlora_linear_fwd(g["X"], W, g["A"], g["B"], s)
    rng = np.random.default_rng(seed)
    rows = np.unique(np.concatenate([rng.integers(0, M, nrows), [0, M - 1]]))
    Xb, Ab, Bb = bits(d["X"]), bits(d["A"]), bits(d["B"])
    if bwd:
        Wd = oracle_dequant_full(bits(d["W"]))
        cols = np.arange(N)
    else:
        # forward only: sampled output features need only their W rows
        cols = np.unique(np.concatenate([rng.integers(0, N, ncols), [0, N - 1]]))
        Wd = oracle_dequant_rows(bits(d["W"]), cols)
    Ur, Yr = ol.linear_fwd(Xb[rows], Wd, Ab, Bb[cols], s)
    Yg = Y.float().cpu().numpy()[rows][:, cols]
    Ug = U.cpu().numpy()[rows]
    errs = {"Y": rel(Yg, Yr), "U": rel(Ug, Ur)}
    if bwd:
        dX, dA, dB = lib.qlora_linear_bwd(g["dY"], g["X"], U, W, g["A"], g["B"], s)
        torch.cuda.synchronize()
        dYb = bits(d["dY"])
        dXr, _, _, _ = ol.linear_bwd(dYb[rows], Xb[rows], Wd, Ab, Bb, s)
        _, dAr, dBr, _ = ol.linear_bwd(dYb, Xb, None, Ab, Bb, s, want_dx=False)
        errs.update(dX=rel(dX.float().cpu().numpy()[rows], dXr), dA=rel(dA.cpu().numpy(), dAr),
                    dB=rel(dB.cpu().numpy(), dBr))
    assert errs["Y"] <= TOL_BF16 and errs["U"] <= TOL_F32, errs
    if bwd:
        assert errs["dX"] <= TOL_BF16 and errs["dA"] <= TOL_F32 and errs["dB"] <= TOL_F32, errs
    return errs


def test_c2_attention_projection():
    """4096x4096, 4 x 1024 tokens, r=64, alpha=16."""
    _check_sampled(4096, 4096, 4096, 64, 0.25, 2)


@pytest.mark.parametrize("N,K", [(11008, 4096), (4096, 11008)])
def test_c3_mlp_with_outliers(N, K):
    _check_sampled(N, K, 8192, 64, 0.25, 3, outliers=True, nrows=48)


@pytest.mark.parametrize("M", [1, 16, 32, 128, 2048])
@pytest.mark.parametrize("N,K", [(22016, 8192), (8192, 22016)])
def test_c5_forward_sweep(N, K, M):
    _check_sampled(N, K, M, 64, 0.25, 5, nrows=32, bwd=False)


@pytest.mark.parametrize("N,K", [(22016, 8192), (8192, 22016)])
def test_c5_forward_largest_m(N, K):
    """65B-shaped up (8192 -> 22016) and down (22016 -> 8192) at 16384 tokens."""
    _check_sampled(N, K, 16384, 64, 0.25, 6, nrows=16, bwd=False)


@pytest.mark.parametrize("index", range(len(synth.LLAMA7B_LAYER)))
def test_c4_decoder_layer_linear(index):
    """c4: each of the seven linears of the LLaMA-7B-shaped decoder layer (q, k,
    v, o 4096x4096; gate, up 4096->11008; down 11008->4096) at 8 x 2048 =
    16384 tokens, r=64, alpha=16, forward and backward: 32 sampled token rows
    of Y and dX against the oracle, and the full dA and dB."""
    lin = synth.LLAMA7B_LAYER[index]
    _check_sampled(lin.n_out, lin.k_in, 16384, 64, 0.25, 40 + index, nrows=32)

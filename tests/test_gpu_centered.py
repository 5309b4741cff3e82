"""GPU parity of mean-centred double quantisation: the quantiser's codes, FP8
constants, group scales and tensor mean bit-exact against the oracle
(oracle.dq_centered), the standalone dequantiser bit-exact, the dequantisation
inside every GEMM path bit-exact (one-hot inputs, as in
test_gpu_dequant_exact), and the GEMMs within the usual tolerances."""

import numpy as np
import pytest
import torch

import synth
from oracle import dq_centered as dqc
from oracle import linear as ol
from tests._util import bits, np_u8, rel

pytestmark = pytest.mark.gpu


def _lib():
    import bit_nf4_quantized_26_b200 as lib
    return lib


def _f32(bf16_bits):
    return (np.asarray(bf16_bits, dtype=np.uint16).astype(np.uint32) << 16).view(np.float32)


def _check_quant(w):
    lib = _lib()
    status = torch.zeros(4, dtype=torch.int32, device="cuda")
    codes, c8, s2, mean = lib.nf4_quantize_centered(w.reshape(-1).contiguous().cuda(), status=status)
    torch.cuda.synchronize()
    assert int(status[0].item()) == 0
    rc, r8, rs2, rmean = dqc.quantize_centered(bits(w).reshape(-1))
    assert np.array_equal(np_u8(codes), rc), "codes differ"
    assert np.array_equal(mean.cpu().numpy().view(np.uint32), np.array([rmean], np.float32).view(np.uint32))
    assert np.array_equal(np_u8(c8), r8), "FP8 constants differ"
    assert np.array_equal(s2.cpu().numpy().view(np.uint32), rs2.view(np.uint32)), "group scales differ"
    return (codes, c8, s2, mean), (rc, r8, rs2, rmean)


@pytest.mark.parametrize("shape,outliers,seed", [
    ((512, 512), False, 0), ((4096, 4096), False, 1), ((11008, 4096), True, 2)])
def test_centred_quantize_bit_exact(shape, outliers, seed):
    _check_quant(synth.weight_bf16(*shape, seed, outliers=outliers))


@pytest.mark.parametrize("numel", [1, 63, 65, 16384 + 17, 3 * 16384 + 64 * 7 + 3, 1500 * 16384 + 5])
def test_centred_quantize_ragged_sizes(numel):
    """Short last blocks and groups (zero-padded constants stay out of the
    group maximum), and more than 1024 groups (the mean kernel's chunks)."""
    _check_quant(synth.normal_bf16((numel,), 0.02, seed=numel))


def test_centred_dequantize_bit_exact():
    lib = _lib()
    w = synth.weight_bf16(2048, 1024, seed=5, outliers=True)
    (codes, c8, s2, mean), (rc, r8, rs2, rmean) = _check_quant(w)
    out = lib.nf4_dequantize_centered(codes, c8, s2, mean, w.numel())
    torch.cuda.synchronize()
    assert np.array_equal(bits(out), dqc.dequantize_centered(rc, r8, rs2, rmean, w.numel()))


# ----------------------------------------------- inside the GEMMs, one-hot

N_W, K_W = 1920, 1088   # neither a multiple of 256: the single-CTA wide kernels


@pytest.fixture(scope="module")
def centred():
    lib = _lib()
    w = synth.weight_bf16(N_W, K_W, seed=6, outliers=True)
    rc, r8, rs2, rmean = dqc.quantize_centered(bits(w).reshape(-1))
    ref = dqc.dequantize_centered(rc, r8, rs2, rmean, w.numel()).reshape(N_W, K_W)
    W = lib.quantize_weight_centered(w.cuda())
    torch.cuda.synchronize()
    return {"W": W, "ref": ref, "w": w}


def _onehot(M, width, cols):
    X = torch.zeros((M, width), dtype=torch.bfloat16, device="cuda")
    X[torch.arange(M, device="cuda"), torch.as_tensor(cols, device="cuda")] = 1.0
    return X


def _sub(lib, W, n):
    """The first n rows of an NF4 weight (n * K a multiple of 16384 elements)."""
    K = int(W.k_in)
    return lib.NF4Weight(W.codes[: n * K // 2], W.c8[: n * K // 64], W.s2[: n * K // 16384], n, K, W.mean)


@pytest.mark.parametrize("M", [8, 32, 64, 200, 1024])
def test_centred_forward_dequant_is_exact(centred, M, few_token_kernel):
    """Y = one-hot X W'^T with B = 0 equals W'[:, cols]^T: few tokens, 64- and
    256-token tiles, and above 256 tokens both the single-CTA kernel (1920
    rows) and the CTA pairs (the first 1792 rows)."""
    lib = _lib()
    for W, n in ((centred["W"], N_W), (_sub(lib, centred["W"], 1792), 1792)):
        if M <= 256 and n != N_W:
            continue
        cols = (np.arange(M) * 37) % K_W
        A = synth.normal_bf16((64, K_W), 1.0 / K_W, seed=1).cuda()
        B = torch.zeros((n, 64), dtype=torch.bfloat16, device="cuda")
        Y, _ = lib.qlora_linear_fwd(_onehot(M, K_W, cols), W, A, B, 0.25, y_dtype=1)
        torch.cuda.synchronize()
        assert np.array_equal(Y.cpu().numpy(), _f32(centred["ref"][:n][:, cols].T)), (M, n)


@pytest.mark.parametrize("M", [64, 200, 1920])
def test_centred_dx_dequant_is_exact(centred, M):
    """dX = one-hot dY W' with B = 0 equals W'[rows, :] (K = 1088: the
    single-CTA kernel above 256 tokens)."""
    lib = _lib()
    W = centred["W"]
    rows = (np.arange(M) * 29) % N_W
    A = synth.normal_bf16((64, K_W), 1.0 / K_W, seed=2).cuda()
    B = torch.zeros((N_W, 64), dtype=torch.bfloat16, device="cuda")
    X = synth.normal_bf16((M, K_W), 1.0, seed=3).cuda()
    _, U = lib.qlora_linear_fwd(X, W, A, B, 0.25)
    dX, _, _ = lib.qlora_linear_bwd(_onehot(M, N_W, rows), X, U, W, A, B, 0.25, dx_dtype=1)
    torch.cuda.synchronize()
    assert np.array_equal(dX.cpu().numpy(), _f32(centred["ref"][rows]))


def test_centred_pair_dx_dequant_is_exact():
    """dX through the CTA-pair kernel (K % 256 == 0)."""
    lib = _lib()
    w = synth.weight_bf16(1024, 1280, seed=7, outliers=True)
    rc, r8, rs2, rmean = dqc.quantize_centered(bits(w).reshape(-1))
    ref = dqc.dequantize_centered(rc, r8, rs2, rmean, w.numel()).reshape(1024, 1280)
    W = lib.quantize_weight_centered(w.cuda())
    A = synth.normal_bf16((16, 1280), 1.0 / 1280, seed=2).cuda()
    B = torch.zeros((1024, 16), dtype=torch.bfloat16, device="cuda")
    X = synth.normal_bf16((1024, 1280), 1.0, seed=3).cuda()
    _, U = lib.qlora_linear_fwd(X, W, A, B, 1.0)
    dX, _, _ = lib.qlora_linear_bwd(_onehot(1024, 1024, np.arange(1024)), X, U, W, A, B, 1.0, dx_dtype=1)
    torch.cuda.synchronize()
    assert np.array_equal(dX.cpu().numpy(), _f32(ref))


@pytest.mark.parametrize("M", [16, 128, 700])
def test_centred_linear_matches_oracle(M, few_token_kernel):
    """Forward and backward on a mean-centred weight against the fp64 oracle
    on the oracle's centred dequantised weight."""
    lib = _lib()
    N, K, r, s = 768, 1024, 64, 0.25
    d = synth.linear_inputs(synth.Linear("c", N, K), M, r, 40 + M, outliers=True)
    g = {k: v.cuda() for k, v in d.items()}
    W = lib.quantize_weight_centered(g["W"])
    Y, U = lib.qlora_linear_fwd(g["X"], W, g["A"], g["B"], s, y_dtype=1)
    dX, dA, dB = lib.qlora_linear_bwd(g["dY"], g["X"], U, W, g["A"], g["B"], s, dx_dtype=1)
    torch.cuda.synchronize()
    rc, r8, rs2, rmean = dqc.quantize_centered(bits(d["W"]).reshape(-1))
    Wd = dqc.dequantize_centered(rc, r8, rs2, rmean, N * K).reshape(N, K)
    Ur, Yr = ol.linear_fwd(bits(d["X"]), Wd, bits(d["A"]), bits(d["B"]), s)
    dXr, dAr, dBr, _ = ol.linear_bwd(bits(d["dY"]), bits(d["X"]), Wd, bits(d["A"]), bits(d["B"]), s)
    for got, ref in ((Y, Yr), (U, Ur), (dX, dXr), (dA, dAr), (dB, dBr)):
        assert rel(got.cpu().numpy(), ref) <= 1e-4

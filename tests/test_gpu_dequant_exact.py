"""Bit-exact check of the dequantisation each GEMM path does in its own tiles.

The method fixes the dequantised weight exactly ("QLoRA" encyclopedia entry,
tonho.wtf, "a ideia": the 4-bit weight becomes a BFloat16 weight at the
moment of use), and the standalone dequantiser is held to that bit for bit.
The GEMM kernels do not call it: they dequantise inside their own tiles
(byte-permute tables written into swizzled shared-memory tiles for the
tensor-core paths, register tables in the few-token kernel).  A wrong table
entry there is one bf16 ulp on a few weights, far below the Frobenius bar of
the other parity tests, so this file isolates the weight:

* forward, B = 0, row m of X one-hot at feature k_m:  Y[m, n] = W'[n, k_m]
  exactly (one nonzero product; U B^T is zero; an fp32 sum of one bf16 value
  and zeros is that value; split-contraction partial sums only add zeros);
* dX, B = 0 (so dU = s dY B = 0), row m of dY one-hot at output n_m:
  dX[m, :] = W'[n_m, :] exactly.

Outputs are fp32, so nothing rounds after the product, and each path's result
is compared with the oracle's dequantised bf16 weight bit for bit (as
values: -0 and +0 compare equal; no block here has a zero constant, so the
oracle has no -0 weights).  The weight is the 65B-shaped 22016 x 8192 matrix
with the outlier recipe (0.1% of elements at +-10 sigma), and the chosen
features cover every residue of the contraction index modulo 256 (every
position within an NF4 block and within a kernel's contraction chunk), where
the test also checks that all 16 codes occur.

Paths, by the library's dispatch rules:
  forward  M <= 16 on a weight of at least 2^26 elements (this one): the
           few-token kernel (8, 16 token rows); other M <= 256: tcgen05
           kernel with 32, 64, 128 and 256 token columns and a split
           contraction;  > 256: CTA-pair kernel (W rows % 256 == 0) or the
           single-CTA 512-token kernel (other W row counts);
  dX       M <= 256: tcgen05 kernel, 128 / 256 token columns, MN-major tiles;
           > 256: CTA-pair kernel (K % 256 == 0) or the 512-token kernel;
  dX with LoRA dropout: the GEMM without its adapter stages into fp32, then
           the dropout pass.
"""

import numpy as np
import pytest
import torch

import synth
from oracle import nf4
from tests._util import bits, oracle_dequant_full

pytestmark = pytest.mark.gpu

N_BIG, K_BIG = 22016, 8192


def _lib():
    import bit_nf4_quantized_26_b200 as lib
    return lib


def _f32(bf16_bits):
    return (np.asarray(bf16_bits, dtype=np.uint16).astype(np.uint32) << 16).view(np.float32)


@pytest.fixture(scope="module")
def big():
    """The 22016 x 8192 outlier weight: bf16 on the GPU, its NF4 storage from
    the library, and the oracle's dequantised weight and codes."""
    lib = _lib()
    w = synth.weight_bf16(N_BIG, K_BIG, seed=2201, outliers=True)
    wb = bits(w)
    ref = oracle_dequant_full(wb)
    W = lib.quantize_weight(w.cuda())
    torch.cuda.synchronize()
    return {"W": W, "ref": ref, "wb": wb}


def _features(M, K, call):
    """One-hot features of `call`: residues (call*M + m) mod 256 spread over
    the 256-wide chunks of K, so ceil(256 / M) calls cover every residue."""
    m = np.arange(M)
    res = (call * M + m) % 256
    chunk = (m * 37 + call * 11) % (K // 256)
    return res + 256 * chunk


def _onehot(M, width, cols):
    X = torch.zeros((M, width), dtype=torch.bfloat16, device="cuda")
    X[torch.arange(M, device="cuda"), torch.as_tensor(cols, device="cuda")] = 1.0
    return X


def _adapters(K, N, r=64, seed=7):
    A = synth.normal_bf16((r, K), 1.0 / K, seed=seed).cuda()
    B = torch.zeros((N, r), dtype=torch.bfloat16, device="cuda")
    return A, B


def _fwd_exact(lib, W, ref, M, cols, y_dtype=1):
    """Y = X W'^T with one-hot X at `cols` must equal W'[:, cols]^T exactly."""
    N, K = int(W.n_out), int(W.k_in)
    A, B = _adapters(K, N)
    X = _onehot(M, K, cols)
    status = torch.zeros(4, dtype=torch.int32, device="cuda")
    Y, _ = lib.qlora_linear_fwd(X, W, A, B, 0.25, y_dtype=y_dtype, status=status)
    torch.cuda.synchronize()
    assert int(status[0].item()) == 0
    got = Y.float().cpu().numpy()
    want = _f32(ref[:N][:, cols].T)
    bad = np.argwhere(got != want)
    assert bad.size == 0, f"{len(bad)} weights differ, first (token, row) {bad[:4].tolist()}"


def _dx_exact(lib, W, ref, M, rows, dropout=False):
    """dX = dY W' with one-hot dY at `rows` must equal W'[rows, :] exactly."""
    N, K = int(W.n_out), int(W.k_in)
    A, B = _adapters(K, N)
    dY = _onehot(M, N, rows)
    X = synth.normal_bf16((M, K), 1.0, seed=M).cuda()
    status = torch.zeros(4, dtype=torch.int32, device="cuda")
    if dropout:
        _, U, Xd = lib.qlora_linear_fwd_dropout(X, W, A, B, 0.25, 0.05, 3, status=status)
        dX, _, _ = lib.qlora_linear_bwd_dropout(dY, Xd, U, W, A, B, 0.25, 0.05, 3, dx_dtype=1, status=status)
    else:
        _, U = lib.qlora_linear_fwd(X, W, A, B, 0.25, status=status)
        dX, _, _ = lib.qlora_linear_bwd(dY, X, U, W, A, B, 0.25, dx_dtype=1, status=status)
    torch.cuda.synchronize()
    assert int(status[0].item()) == 0
    got = dX.cpu().numpy()
    want = _f32(ref[rows])
    bad = np.argwhere(got != want)
    assert bad.size == 0, f"{len(bad)} weights differ, first (token, column) {bad[:4].tolist()}"


def test_every_code_occurs_at_every_block_position(big):
    """Coverage of the inputs below: all 16 codes at every position 0..63 of
    a block (checked on the oracle's codes of the weight)."""
    codes = nf4.quantize(big["wb"][:4096].reshape(-1))[0]
    per_elem = nf4.unpack_codes(codes, 4096 * K_BIG).reshape(-1, 64)
    for pos in range(64):
        assert np.unique(per_elem[:, pos]).size == 16, pos


@pytest.mark.parametrize("M", [8, 16, 32])
def test_few_token_forward_dequant_is_exact(big, M):
    lib = _lib()
    for call in range(-(-256 // M)):
        _fwd_exact(lib, big["W"], big["ref"], M, _features(M, K_BIG, call))


@pytest.mark.parametrize("M", [64, 128, 200])
def test_mid_token_forward_dequant_is_exact(big, M):
    lib = _lib()
    for call in range(-(-256 // M)):
        _fwd_exact(lib, big["W"], big["ref"], M, _features(M, K_BIG, call))


def test_pair_forward_dequant_is_exact(big):
    """8192 one-hot tokens over all 8192 features: Y is the whole W'^T."""
    _fwd_exact(_lib(), big["W"], big["ref"], K_BIG, np.arange(K_BIG))


def test_pair_forward_bf16_output_is_exact(big):
    """bf16 output of a bf16-representable accumulator is the same value."""
    _fwd_exact(_lib(), big["W"], big["ref"], 1024, _features(1024, K_BIG, 0), y_dtype=0)


def test_single_cta_wide_forward_dequant_is_exact(big):
    """W rows 21952 (not a multiple of 256): the 512-token single-CTA kernel.
    The first 21952 rows of the NF4 storage are the NF4 storage of those rows
    (each row is 128 blocks, so double-quantisation groups end on row pairs)."""
    lib = _lib()
    n = 21952
    W = big["W"]
    Ws = lib.NF4Weight(W.codes[: n * K_BIG // 2], W.c8[: n * K_BIG // 64], W.s2[: n * K_BIG // 16384], n, K_BIG)
    _fwd_exact(lib, Ws, big["ref"], K_BIG, np.arange(K_BIG))


@pytest.mark.parametrize("M", [64, 200])
def test_small_dx_dequant_is_exact(big, M):
    lib = _lib()
    for call in range(-(-64 // min(M, 64))):
        m = np.arange(M)
        rows = (m % 64) + 64 * ((m * 29 + call * 5) % (N_BIG // 64))
        _dx_exact(lib, big["W"], big["ref"], M, rows)


def test_pair_dx_dequant_is_exact(big):
    """22016 one-hot gradient rows: dX is the whole W'."""
    _dx_exact(_lib(), big["W"], big["ref"], N_BIG, np.arange(N_BIG))


def test_single_cta_wide_dx_dequant_is_exact():
    """K = 4160 (not a multiple of 256): the 512-token single-CTA dX kernel."""
    lib = _lib()
    w = synth.weight_bf16(2048, 4160, seed=2202, outliers=True)
    ref = oracle_dequant_full(bits(w))
    W = lib.quantize_weight(w.cuda())
    _dx_exact(lib, W, ref, 2048, np.arange(2048))


@pytest.mark.parametrize("M", [64, 512])
def test_dropout_dx_dequant_is_exact(big, M):
    m = np.arange(M)
    rows = (m * 43) % N_BIG
    _dx_exact(_lib(), big["W"], big["ref"], M, rows, dropout=True)

"""GPU parity of grouped projections (linears sharing one input, stacked
along the output dimension) against the oracle's group forward/backward.

Tolerances as for the single linear: Y, dX within 2e-3 (bf16) or 1e-4
(fp32), U, dA, dB within 1e-4 (relative Frobenius), per member for Y, U, dA,
dB and on the summed dX.  Shapes reach every kernel path with member
boundaries inside the stacked weight: few tokens, mid-size token tiles with a
split contraction, CTA pairs (every boundary on 256 rows) and the single-CTA
512-token kernel (a boundary on 128 rows).  Where the grouped call runs the
same tiles as a call on the member alone (the CTA-pair forward and the
unsplit rank-r product above 256 tokens), Y and U must match that call bit
for bit.
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


def _inputs(M, members, K, r, seed, outliers=False):
    """Member weights and adapters, one shared X and a stacked dY (CPU bf16)."""
    Ws, As, Bs = [], [], []
    for g, n in enumerate(members):
        d = synth.linear_inputs(synth.Linear(f"m{g}", n, K), 1, r, seed * 10 + g, outliers=outliers)
        Ws.append(d["W"])
        As.append(d["A"])
        Bs.append(d["B"])
    X = synth.normal_bf16((M, K), 1.0, seed * 10 + 7)
    dY = synth.normal_bf16((M, sum(members)), 1.0, seed * 10 + 8)
    return {"W": torch.cat(Ws, 0), "A": torch.cat(As, 0), "B": torch.cat(Bs, 0), "X": X, "dY": dY}


def _run(d, members, s, dtype):
    lib = _lib()
    g = {k: v.cuda() for k, v in d.items()}
    W = lib.quantize_weight(g["W"])
    status = torch.zeros(4, dtype=torch.int32, device="cuda")
    Y, U = lib.qlora_group_fwd(g["X"], W, members, g["A"], g["B"], s, y_dtype=dtype, status=status)
    dX, dA, dB = lib.qlora_group_bwd(g["dY"], g["X"], U, W, members, g["A"], g["B"], s, dx_dtype=dtype,
                                     status=status)
    torch.cuda.synchronize()
    assert int(status[0].item()) == 0
    return W, {k: v.float().cpu().numpy() for k, v in dict(Y=Y, U=U, dX=dX, dA=dA, dB=dB).items()}


@pytest.mark.parametrize("M,members,K,r", [
    (8, (256, 128, 384), 512, 16),      # few-token kernel, three members
    (29, (128, 128), 1024, 64),         # few-token kernel, four token tiles
    (100, (128, 256), 1024, 64),        # 128-token tiles, split contraction
    (200, (384, 128, 256), 768, 32),    # 256-token tiles
    (700, (512, 256, 256), 768, 64),    # CTA pairs (boundaries on 256 rows)
    (600, (384, 128), 512, 48),         # single-CTA 512-token kernel (boundary on 384)
])
def test_group_matches_oracle(M, members, K, r, few_token_kernel):
    s = 16.0 / r
    d = _inputs(M, members, K, r, seed=M + K)
    for dtype, tol in ((1, TOL_F32), (0, TOL_BF16)):
        _, got = _run(d, list(members), s, dtype)
        Wd = oracle_dequant_full(bits(d["W"]))
        U, Y = ol.group_fwd(bits(d["X"]), Wd, bits(d["A"]), bits(d["B"]), s, members)
        dX, dA, dB = ol.group_bwd(bits(d["dY"]), bits(d["X"]), Wd, bits(d["A"]), bits(d["B"]), s, members)
        off = np.concatenate([[0], np.cumsum(members)])
        for g in range(len(members)):
            cols = slice(off[g], off[g + 1])
            assert rel(got["Y"][:, cols], Y[:, cols]) <= tol, ("Y", g)
            assert rel(got["U"][:, g * r:(g + 1) * r], U[:, g * r:(g + 1) * r]) <= TOL_F32, ("U", g)
            assert rel(got["dA"][g * r:(g + 1) * r], dA[g * r:(g + 1) * r]) <= TOL_F32, ("dA", g)
            assert rel(got["dB"][cols], dB[cols]) <= TOL_F32, ("dB", g)
        assert rel(got["dX"], dX) <= tol


def test_group_of_one_is_the_single_linear():
    lib = _lib()
    d = {k: v.cuda() for k, v in synth.linear_inputs(synth.Linear("one", 512, 768), 300, 64, 5).items()}
    W = lib.quantize_weight(d["W"])
    Y1, U1 = lib.qlora_linear_fwd(d["X"], W, d["A"], d["B"], 0.25)
    Yg, Ug = lib.qlora_group_fwd(d["X"], W, [512], d["A"], d["B"], 0.25)
    r1 = lib.qlora_linear_bwd(d["dY"], d["X"], U1, W, d["A"], d["B"], 0.25)
    rg = lib.qlora_group_bwd(d["dY"], d["X"], Ug, W, [512], d["A"], d["B"], 0.25)
    torch.cuda.synchronize()
    assert torch.equal(Y1.view(torch.int16), Yg.view(torch.int16))
    assert torch.equal(U1.view(torch.int32), Ug.view(torch.int32))
    for a, b in zip(r1, rg):
        assert torch.equal(a.view(torch.int16) if a.dtype == torch.bfloat16 else a.view(torch.int32),
                           b.view(torch.int16) if b.dtype == torch.bfloat16 else b.view(torch.int32))


def test_pair_group_forward_equals_members_alone():
    """Above 256 tokens with boundaries on 256 rows, each member's tiles of the
    grouped forward are the tiles of the member's own forward: same bits."""
    lib = _lib()
    members, K, r, M = (512, 256, 768), 512, 64, 1024
    d = {k: v.cuda() for k, v in _inputs(M, members, K, r, seed=11).items()}
    W = lib.quantize_weight(d["W"])
    Yg, Ug = lib.qlora_group_fwd(d["X"], W, list(members), d["A"], d["B"], 0.25)
    off = np.concatenate([[0], np.cumsum(members)])
    for g, n in enumerate(members):
        Wg = lib.NF4Weight(W.codes[off[g] * K // 2: off[g + 1] * K // 2], W.c8[off[g] * K // 64: off[g + 1] * K // 64],
                           W.s2[off[g] * K // 16384: off[g + 1] * K // 16384], n, K)
        Y1, U1 = lib.qlora_linear_fwd(d["X"], Wg, d["A"][g * r:(g + 1) * r].contiguous(),
                                      d["B"][off[g]:off[g + 1]].contiguous(), 0.25)
        torch.cuda.synchronize()
        assert torch.equal(Yg[:, off[g]:off[g + 1]].contiguous().view(torch.int16), Y1.view(torch.int16)), g
        assert torch.equal(Ug[:, g * r:(g + 1) * r].contiguous().view(torch.int32), U1.view(torch.int32)), g


@pytest.mark.parametrize("members", [(4096, 4096, 4096), (11008, 11008)])
def test_c4_groups_at_full_size(members):
    """The decoder layer's q/k/v and gate/up groups at 16384 tokens: sampled
    token rows of Y (all members) and dX, the full dA and dB."""
    lib = _lib()
    M, K, r, s = 16384, 4096, 64, 0.25
    d = _inputs(M, members, K, r, seed=len(members))
    g = {k: v.cuda() for k, v in d.items()}
    W = lib.quantize_weight(g["W"])
    status = torch.zeros(4, dtype=torch.int32, device="cuda")
    Y, U = lib.qlora_group_fwd(g["X"], W, list(members), g["A"], g["B"], s, status=status)
    dX, dA, dB = lib.qlora_group_bwd(g["dY"], g["X"], U, W, list(members), g["A"], g["B"], s, status=status)
    torch.cuda.synchronize()
    assert int(status[0].item()) == 0
    rng = np.random.default_rng(0)
    rows = np.unique(np.concatenate([rng.integers(0, M, 24), [0, M - 1]]))
    Xb, Ab, Bb, dYb = bits(d["X"]), bits(d["A"]), bits(d["B"]), bits(d["dY"])
    Wd = oracle_dequant_full(bits(d["W"]))
    Ur, Yr = ol.group_fwd(Xb[rows], Wd, Ab, Bb, s, members)
    dXr, _, _ = ol.group_bwd(dYb[rows], Xb[rows], Wd, Ab, Bb, s, members)
    _, dAr, dBr = ol.group_bwd(dYb, Xb, None, Ab, Bb, s, members, want_dx=False)
    assert rel(Y.float().cpu().numpy()[rows], Yr) <= TOL_BF16
    assert rel(U.cpu().numpy()[rows], Ur) <= TOL_F32
    assert rel(dX.float().cpu().numpy()[rows], dXr) <= TOL_BF16
    assert rel(dA.cpu().numpy(), dAr) <= TOL_F32
    assert rel(dB.cpu().numpy(), dBr) <= TOL_F32

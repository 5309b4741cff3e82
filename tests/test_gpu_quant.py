"""GPU parity of NF4 quantisation and dequantisation: bit-exact against the oracle."""

import numpy as np
import pytest
import torch

import synth
from oracle import nf4
from oracle import numerics as nm
from tests._util import bits, np_u8, oracle_quantize_chunked

pytestmark = pytest.mark.gpu

def _lib():
    import bit_nf4_quantized_26_b200 as lib
    return lib


def _gpu_quant(w_cpu_bf16):
    lib = _lib()
    w = w_cpu_bf16.reshape(-1).contiguous().cuda()
    status = torch.zeros(4, dtype=torch.int32, device="cuda")
    codes, c8, s2 = lib.nf4_quantize(w, status=status)
    torch.cuda.synchronize()
    return np_u8(codes), np_u8(c8), s2.cpu().numpy(), int(status[0].item())


def _check_quant(w_cpu_bf16):
    codes, c8, s2, st = _gpu_quant(w_cpu_bf16)
    ref_codes, ref_c8, ref_s2 = oracle_quantize_chunked(bits(w_cpu_bf16))
    assert st == 0
    assert np.array_equal(codes, ref_codes), "codes differ"
    assert np.array_equal(c8, ref_c8), "FP8 constants differ"
    assert np.array_equal(s2.view(np.uint32), ref_s2.view(np.uint32)), "group scales differ"
    return codes, c8, s2


@pytest.mark.parametrize("shape,outliers,seed", [
    ((512, 512), False, 0),
    ((4096, 4096), False, 1),
    ((11008, 4096), True, 2),
    ((4096, 11008), True, 3),
])
def test_quantize_bit_exact(shape, outliers, seed):
    _check_quant(synth.weight_bf16(*shape, seed, outliers=outliers))


@pytest.mark.parametrize("numel", [1, 5, 63, 64, 65, 16384 - 1, 16384 + 17, 3 * 16384 + 64 * 7 + 3, 1 << 20])
def test_quantize_ragged_sizes(numel):
    _check_quant(synth.normal_bf16((numel,), 0.02, seed=numel))


def test_quantize_special_values():
    rng = np.random.default_rng(5)
    parts = [
        np.zeros(64 * 3, dtype=np.uint16),                                   # zero blocks
        np.full(64, 0x8000, dtype=np.uint16),                                # -0 block
        rng.integers(0, 0x0080, 64 * 4).astype(np.uint16),                   # subnormals / tiny c
        np.tile(nm.f32_to_bf16_bits(nf4.codebook()), 4),                     # codebook values, c = 1
        (rng.integers(0, 0x7F7F, 64 * 8) | (rng.integers(0, 2, 64 * 8) << 15)).astype(np.uint16),  # wide range
        np.array([0x7F7F, 0xFF7F] * 32, dtype=np.uint16),                    # +-max bf16
    ]
    w = np.concatenate(parts)
    w = np.concatenate([w, synth.random_bf16_bits((16384 * 2 - w.size,), seed=9)])
    t = torch.from_numpy(w.view(np.int16).copy()).view(torch.bfloat16)
    _check_quant(t)


def test_quantize_65b_shape_sampled_groups():
    """Full [22016, 8192] matrix on the GPU; 48 random groups checked against the oracle."""
    lib = _lib()
    w = synth.weight_bf16(22016, 8192, seed=65, device="cuda")
    codes, c8, s2 = lib.nf4_quantize(w.reshape(-1))
    torch.cuda.synchronize()
    flat = bits(w).reshape(-1)
    ngroups = s2.numel()
    rng = np.random.default_rng(0)
    picks = sorted(set(rng.integers(0, ngroups, 46).tolist()) | {0, ngroups - 1})
    codes_h, c8_h, s2_h = np_u8(codes), np_u8(c8), s2.cpu().numpy()
    for g in picks:
        seg = flat[g * 16384:(g + 1) * 16384]
        p, c, s = nf4.quantize(seg)
        assert np.array_equal(codes_h[g * 8192:(g + 1) * 8192], p), g
        assert np.array_equal(c8_h[g * 256:(g + 1) * 256], c), g
        assert s2_h[g].view(np.uint32) == s[0].view(np.uint32), g


@pytest.mark.parametrize("numel", [64 * 256 * 8, 5000, 16384 * 3 + 100, 1, 5, 63, 64, 65, 127, 64 * 32 + 3,
                                   64 * 33, 16384 * 2 + 64 * 33 + 7])
def test_dequantize_bit_exact(numel):
    """Sizes: no full block (no tensor-map store), a partial last block, warps
    whose 32-row store box runs past the last full row."""
    lib = _lib()
    w = synth.normal_bf16((numel,), 0.02, seed=numel + 1)
    ref_codes, ref_c8, ref_s2 = nf4.quantize(bits(w))
    ref = nf4.dequantize(ref_codes, ref_c8, ref_s2, numel)
    codes = torch.from_numpy(ref_codes).cuda()
    c8 = torch.from_numpy(ref_c8).cuda()
    s2 = torch.from_numpy(ref_s2).cuda()
    out = lib.nf4_dequantize(codes, c8, s2, numel)
    torch.cuda.synchronize()
    assert np.array_equal(bits(out), ref)


def test_dequantize_all_codes_and_constants():
    """Every (code, c8) pair once, with a group scale that exercises rounding."""
    lib = _lib()
    nblocks = 256
    codes = np.zeros(nblocks * 32, dtype=np.uint8)
    cod = np.tile(np.arange(16, dtype=np.uint8), nblocks * 4)
    codes[:] = cod[0::2] | (cod[1::2] << 4)
    c8 = (np.arange(nblocks) % 127).astype(np.uint8)     # every finite non-negative E4M3 code
    s2 = np.array([np.float32(0.0123456789)], dtype=np.float32)
    ref = nf4.dequantize(codes, c8, s2, nblocks * 64)
    out = lib.nf4_dequantize(torch.from_numpy(codes).cuda(), torch.from_numpy(c8).cuda(),
                             torch.from_numpy(s2).cuda(), nblocks * 64)
    torch.cuda.synchronize()
    assert np.array_equal(bits(out), ref)


def test_round_trip_matches_oracle_dequant():
    lib = _lib()
    w = synth.weight_bf16(4096, 4096, seed=21, device="cuda")
    codes, c8, s2 = lib.nf4_quantize(w.reshape(-1))
    out = lib.nf4_dequantize(codes, c8, s2, w.numel())
    torch.cuda.synchronize()
    rc, rc8, rs2 = oracle_quantize_chunked(bits(w))
    assert np.array_equal(bits(out), nf4.dequantize(rc, rc8, rs2, w.numel()))


def test_nonfinite_input_sets_status():
    lib = _lib()
    w = synth.normal_bf16((64 * 512,), 0.02, seed=3).cuda()
    w[777] = float("inf")
    status = torch.zeros(4, dtype=torch.int32, device="cuda")
    lib.nf4_quantize(w, status=status)
    torch.cuda.synchronize()
    assert int(status[0].item()) & lib.DEV_NONFINITE


def test_nan_input_sets_status_and_other_groups_stay_exact():
    """A NaN makes its block's codes unspecified (never a stray table access);
    the other groups of the call are still exact."""
    lib = _lib()
    w = synth.normal_bf16((16384 * 4,), 0.02, seed=4)
    w[16384 * 2 + 100] = float("nan")
    status = torch.zeros(4, dtype=torch.int32, device="cuda")
    codes, c8, s2 = lib.nf4_quantize(w.cuda(), status=status)
    torch.cuda.synchronize()
    assert int(status[0].item()) & lib.DEV_NONFINITE
    flat = bits(w)
    for g in (0, 1, 3):
        p, c, s = nf4.quantize(flat[g * 16384:(g + 1) * 16384])
        assert np.array_equal(np_u8(codes)[g * 8192:(g + 1) * 8192], p)
        assert np.array_equal(np_u8(c8)[g * 256:(g + 1) * 256], c)


def test_c5_quantize_sweep_all_layers_sampled_groups():
    """The 65B-shaped sweep: every linear weight of 80 layers (hidden 8192,
    intermediate 22016; 64.76 G parameters) drawn on the device, quantised,
    and dropped, keeping only the 33.4 GB of NF4 resident.  Then the weights
    of the first, the last and three random layers are drawn again from the
    same seeds and 6 random double-quantisation groups of each matrix (plus
    its first and last) are checked bit for bit against the oracle."""
    lib = _lib()
    kept = []
    for layer in range(synth.C5_LAYERS):
        for j, lin in enumerate(synth.c5_layer_linears()):
            w = synth.weight_bf16(lin.n_out, lin.k_in, seed=650000 + 10 * layer + j, device="cuda")
            kept.append(lib.nf4_quantize(w.reshape(-1)))
            del w
    torch.cuda.synchronize()
    resident = sum(c.numel() + c8.numel() + 4 * s2.numel() for c, c8, s2 in kept)
    assert resident == 33407713280
    rng = np.random.default_rng(80)
    layers = sorted({0, synth.C5_LAYERS - 1, *rng.integers(1, synth.C5_LAYERS - 1, 3).tolist()})
    for layer in layers:
        for j, lin in enumerate(synth.c5_layer_linears()):
            codes, c8, s2 = kept[layer * 7 + j]
            w = synth.weight_bf16(lin.n_out, lin.k_in, seed=650000 + 10 * layer + j, device="cuda").reshape(-1)
            ngroups = s2.numel()
            picks = sorted({0, ngroups - 1, *rng.integers(0, ngroups, 6).tolist()})
            for g in picks:
                seg = bits(w[g * 16384:(g + 1) * 16384])
                p, c, s = nf4.quantize(seg)
                assert np.array_equal(np_u8(codes[g * 8192:(g + 1) * 8192]), p), (layer, j, g)
                assert np.array_equal(np_u8(c8[g * 256:(g + 1) * 256]), c), (layer, j, g)
                assert s2[g].item() == float(s[0]), (layer, j, g)
            del w
    del kept

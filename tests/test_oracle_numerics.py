"""Pins for oracle.numerics: bf16 and FP8 E4M3 against library casts and closed forms."""

import numpy as np
import torch

from oracle import numerics as nm


def _torch_bf16_bits(x32):
    t = torch.from_numpy(np.ascontiguousarray(x32, dtype=np.float32)).to(torch.bfloat16)
    return t.view(torch.int16).numpy().view(np.uint16)


def test_bf16_round_matches_torch_cast():
    rng = np.random.default_rng(0)
    x = rng.standard_normal(200_000).astype(np.float32) * np.float32(37.0)
    # exact ties: low 16 bits = 0x8000 with both parities of bit 16
    ties = (rng.integers(0, 2**31, 5000, dtype=np.uint32) & np.uint32(0xFFFF0000)) | np.uint32(0x8000)
    x = np.concatenate([x, ties.view(np.float32), np.float32([0.0, -0.0, 1e-40, -3e38, 3.3e38])])
    x = x[np.isfinite(x)]
    assert np.array_equal(nm.f32_to_bf16_bits(x), _torch_bf16_bits(x))


def test_bf16_tie_goes_to_even():
    # 1 + 2^-8 is exactly between bf16 1.0 (even) and 1 + 2^-7 (odd)
    assert nm.f32_to_bf16_bits(np.float32(1 + 2**-8)) == 0x3F80
    # 1 + 3*2^-8 is between 1+2^-7 (odd) and 1+2^-6 (even)
    assert nm.f32_to_bf16_bits(np.float32(1 + 3 * 2**-8)) == 0x3F82


def test_bf16_widen_is_exact():
    b = np.arange(2**16, dtype=np.uint32).astype(np.uint16)
    f = nm.bf16_bits_to_f32(b)
    ok = np.isfinite(f)
    assert np.array_equal(nm.f32_to_bf16_bits(f[ok]), b[ok])


def test_e4m3_decode_all_codes_match_torch():
    codes = np.arange(256, dtype=np.uint8)
    ours = nm.e4m3_decode(codes)
    ref = torch.from_numpy(codes.copy()).view(torch.float8_e4m3fn).to(torch.float32).numpy()
    assert np.array_equal(np.isnan(ours), np.isnan(ref))
    ok = ~np.isnan(ref)
    assert np.array_equal(ours[ok], ref[ok])


def test_e4m3_closed_forms():
    d = nm.e4m3_decode(np.uint8([0x7E, 0x01, 0x08, 0x38, 0x00, 0x80, 0xFE]))
    assert d[0] == 448.0 and d[1] == 2.0**-9 and d[2] == 2.0**-6 and d[3] == 1.0
    assert d[4] == 0.0 and d[6] == -448.0
    assert np.isnan(nm.e4m3_decode(np.uint8([0x7F]))[0])


def test_e4m3_encode_round_trips_every_finite_value():
    codes = np.array([c for c in range(256) if (c & 0x7F) != 0x7F], dtype=np.uint8)
    vals = nm.e4m3_decode(codes)
    enc = nm.e4m3_encode(vals)
    # -0 encodes as +0; every other value returns its own code
    nz = vals != 0
    assert np.array_equal(enc[nz], codes[nz])


def test_e4m3_encode_midpoints_and_neighbours():
    pos = nm.e4m3_decode(np.arange(0x7F, dtype=np.uint8)).astype(np.float64)
    mids = ((pos[:-1] + pos[1:]) / 2).astype(np.float32)
    assert np.array_equal(mids.astype(np.float64), (pos[:-1] + pos[1:]) / 2)  # exact in fp32
    enc = nm.e4m3_encode(mids)
    lo = np.arange(0x7E)
    expect = np.where(lo % 2 == 0, lo, lo + 1)  # ties to the even code
    assert np.array_equal(enc, expect)
    up = np.nextafter(mids, np.float32(np.inf))
    dn = np.nextafter(mids, np.float32(0))
    assert np.array_equal(nm.e4m3_encode(up), lo + 1)
    assert np.array_equal(nm.e4m3_encode(dn), lo)


def test_e4m3_encode_matches_torch_in_range():
    rng = np.random.default_rng(1)
    x = np.concatenate([
        rng.uniform(0, 464, 100_000), np.exp(rng.uniform(np.log(1e-9), np.log(464), 100_000)),
    ]).astype(np.float32)
    x = np.concatenate([x, -x])
    ref = torch.from_numpy(x).to(torch.float8_e4m3fn).view(torch.uint8).numpy()
    ours = nm.e4m3_encode(x)
    # torch encodes -0 (tiny negatives that round to zero) as 0x80; ours as 0x00
    ref = np.where(ref == 0x80, 0x00, ref)
    assert np.array_equal(ours, ref)


def test_e4m3_encode_saturates():
    x = np.float32([464.0, 464.01, 480.0, 1e6, 3e38, -1e6])
    assert list(nm.e4m3_encode(x)) == [0x7E, 0x7E, 0x7E, 0x7E, 0x7E, 0xFE]

"""Bit-level number formats used by the oracle (test infrastructure only).

bfloat16
    IEEE-754 binary32 with the low 16 bits dropped: 1 sign, 8 exponent,
    7 stored mantissa bits.  Conversion from fp32 rounds to nearest, ties to
    even (the compute type named in the "QLoRA" encyclopedia entry, section
    "a ideia": weights are dequantised to BFloat16 for the matmul).

FP8 E4M3 (OCP 8-bit floating point, "fn" flavour)
    1 sign, 4 exponent bits (bias 7), 3 mantissa bits; no infinities;
    S.1111.111 is NaN, so the largest finite magnitude is 1.75 * 2**8 = 448;
    exponent field 0 encodes subnormals m/8 * 2**-6.  The pages name only
    "FP8" for the double-quantised constants ("como funciona"); the E4M3
    flavour with round-to-nearest-even and saturation to +-448 is this
    build's reading.

Parity status: pinned (exhaustive decode and encode checks against
torch's float8_e4m3fn / bfloat16 CPU casts and closed forms in
tests/test_oracle_numerics.py).
"""

import numpy as np

# ---------------------------------------------------------------- bfloat16


def f32_to_bf16_bits(x):
    """Round fp32 values to bfloat16 (RNE); return the 16-bit patterns.

    NaN inputs map to a quiet NaN with the input's sign.
    """
    x = np.ascontiguousarray(np.asarray(x, dtype=np.float32))
    u = x.view(np.uint32).astype(np.uint64)
    lsb = (u >> np.uint64(16)) & np.uint64(1)
    rounded = ((u + np.uint64(0x7FFF) + lsb) >> np.uint64(16)).astype(np.uint16)
    nan = np.isnan(x)
    if nan.any():
        sign = ((u >> np.uint64(16)) & np.uint64(0x8000)).astype(np.uint16)
        rounded = np.where(nan, sign | np.uint16(0x7FC0), rounded)
    return rounded.astype(np.uint16)


def bf16_bits_to_f32(b):
    """Widen bfloat16 bit patterns to fp32 (exact)."""
    b = np.asarray(b, dtype=np.uint16)
    return (b.astype(np.uint32) << np.uint32(16)).view(np.float32)


# ------------------------------------------------------------ FP8 E4M3


def e4m3_decode(codes):
    """Decode E4M3 bytes to fp32 (exact; NaN for S.1111.111)."""
    c = np.asarray(codes, dtype=np.uint8).astype(np.int64)
    sign = np.where(c & 0x80, -1.0, 1.0)
    e = (c >> 3) & 0xF
    m = c & 0x7
    normal = sign * np.ldexp(1.0 + m / 8.0, e - 7)
    subnormal = sign * np.ldexp(m / 8.0, -6)
    out = np.where(e == 0, subnormal, normal)
    out = np.where((e == 15) & (m == 7), np.nan, out)
    return out.astype(np.float32)


# The 127 non-negative finite E4M3 values, ascending, indexed by their code.
_E4M3_POS = e4m3_decode(np.arange(0x7F, dtype=np.uint8)).astype(np.float64)


def e4m3_encode(x):
    """Encode fp32 values to E4M3: round to nearest, ties to even, saturate.

    Written as the definition: among the finite E4M3 magnitudes pick the
    nearest one to |x| (exact comparison in fp64, where every fp32 value,
    every E4M3 value and every midpoint between two E4M3 values is exact);
    when |x| is exactly half way, pick the code with an even mantissa
    (even code, since the mantissa is the code's low bits).  Magnitudes above
    448 saturate to 448.  Non-finite input is a caller error.
    """
    x = np.asarray(x, dtype=np.float32)
    if not np.all(np.isfinite(x)):
        raise ValueError("e4m3_encode: non-finite input")
    a = np.abs(x.astype(np.float64))
    hi = np.searchsorted(_E4M3_POS, a, side="left")  # first value >= a
    hi = np.minimum(hi, len(_E4M3_POS) - 1)
    lo = np.maximum(hi - 1, 0)
    d_lo = a - _E4M3_POS[lo]
    d_hi = _E4M3_POS[hi] - a
    pick_hi = (d_hi < d_lo) | ((d_hi == d_lo) & (hi % 2 == 0))
    code = np.where(pick_hi, hi, lo)
    code = np.where(a >= _E4M3_POS[-1], len(_E4M3_POS) - 1, code)  # saturate
    code = np.where(a == 0.0, 0, code)
    sign = np.signbit(x) & (code != 0)
    return (code | np.where(sign, 0x80, 0)).astype(np.uint8)

"""NF4 codebook, blockwise quantisation, double quantisation, dequantisation.

TEST INFRASTRUCTURE ONLY (see the package header).  Each step follows the
"QLoRA" encyclopedia entry (tonho.wtf), section "como funciona", in the order
the page gives it; where the page is silent the plainest reading is taken and
named in the function's docstring.

Storage format produced for a tensor of ``numel`` bf16 elements, flattened in
row-major order:

* ``codes``  uint8[ceil(numel/64) * 32]: two 4-bit codes per byte, element 2j
  in the LOW nibble of byte j, element 2j+1 in the high nibble;
* ``c8``     uint8[ceil(numel/64)]: one FP8 E4M3 constant per 64-element block;
* ``s2``     float32[ceil(numel/16384)]: one fp32 scale per group of 256 blocks.

That is 4 + 8/64 + 32/16384 bits per parameter, the 0.127-bit constant
overhead of "como funciona".

Parity status: codebook — pinned by the invariants the page fixes (16
levels, [-1, 1], exact 0, asymmetry) plus a forward-CDF check of the
quantile construction; the choice of the outermost probability ``DELTA`` is
a reading (any value passes the page's invariants), so the codebook is
"parity unpinned beyond these invariants".  quantize/double-quantize/
dequantize — pinned (brute-force nearest level, exhaustive FP8, bit-cost
closed forms, zero padding, codebook round trip, idempotence, locality).
"""

import statistics

import numpy as np

from .numerics import bf16_bits_to_f32, e4m3_decode, e4m3_encode, f32_to_bf16_bits

BLOCK = 64          # elements per absmax constant ("como funciona")
GROUP = 256         # constants per FP8 double-quantisation group ("como funciona")
FP8_MAX = 448.0     # largest finite E4M3 magnitude

# Outermost probability of the quantile grid.  The pages fix only "quantiles
# of the standard normal"; this value (the mean of 1-1/30 and 1-1/32) is the
# one published with the original NF4 construction and is a reading.
DELTA = 0.5 * ((1.0 - 1.0 / 30.0) + (1.0 - 1.0 / 32.0))


def codebook_f64():
    """The 16 NF4 levels in fp64, ascending, before rounding to fp32.

    Construction ("como funciona": 4-bit type from standard-normal quantiles,
    normalised to [-1, 1] by the absolute maximum, asymmetric so that zero is
    represented exactly):

    * 8 positive levels: the N(0,1) quantiles at 8 probabilities evenly
      spaced from DELTA down towards 1/2 (9 points from DELTA to 1/2, the
      last one — the median — dropped);
    * 7 negative levels: minus the quantiles at 7 probabilities evenly spaced
      the same way (8 points, the median dropped);
    * the level 0 (exact);
    * everything divided by the largest magnitude, so the ends are -1 and +1.

    The inverse normal CDF is Python's ``statistics.NormalDist.inv_cdf``
    (Wichura's algorithm AS241, accurate to about 1e-16).
    """
    nd = statistics.NormalDist(0.0, 1.0)
    p_pos = np.linspace(DELTA, 0.5, 9)[:-1]
    p_neg = np.linspace(DELTA, 0.5, 8)[:-1]
    pos = [nd.inv_cdf(float(p)) for p in p_pos]
    neg = [-nd.inv_cdf(float(p)) for p in p_neg]
    levels = np.array(sorted(neg + [0.0] + pos), dtype=np.float64)
    return levels / np.max(np.abs(levels))


def codebook():
    """The 16 NF4 levels as fp32 (one rounding of :func:`codebook_f64`).

    Code i is the i-th level in ascending order, so code 7 is the exact zero
    (the pages do not fix a code order; ascending is the plainest one).
    """
    return codebook_f64().astype(np.float32)


def midpoints():
    """The 15 decision thresholds m_i between level i and level i+1, fp32.

    m_i is the exact midpoint (q_i + q_{i+1}) / 2, computed exactly in fp64
    from the fp32 levels and rounded once to fp32.
    """
    q = codebook().astype(np.float64)
    return ((q[:-1] + q[1:]) / 2.0).astype(np.float32)


def _blocks(w_bits, numel):
    """bf16 bits -> fp32 array [nblocks, 64], zero padded at the tail."""
    w_bits = np.asarray(w_bits, dtype=np.uint16).reshape(-1)
    if w_bits.size != numel:
        raise ValueError("numel mismatch")
    nblocks = -(-numel // BLOCK)
    padded = np.zeros(nblocks * BLOCK, dtype=np.uint16)  # +0.0 padding
    padded[:numel] = w_bits
    return bf16_bits_to_f32(padded).reshape(nblocks, BLOCK)


def absmax_constants(w_bits, numel):
    """Per-block absmax constant c (fp32, exact: the max of |bf16| values).

    "como funciona": one constant per block of 64, the absolute maximum used
    to normalise the block to [-1, 1].  Raises on non-finite input (the
    output would be unspecified).
    """
    w = _blocks(w_bits, numel)
    if not np.all(np.isfinite(w)):
        raise ValueError("non-finite weight")
    return np.max(np.abs(w), axis=1).astype(np.float32)


def encode_codes(w_bits, numel, c):
    """4-bit codes (one uint8 per element, 0..15) given the block constants.

    Normalise: x = RN32(w * RN32(1/c)) — one correctly rounded reciprocal per
    block, then one rounded product per element (the page says "normalise by
    the absolute maximum" without fixing the arithmetic; this is the reading).
    Nearest level: code = #{i : x > m_i}.  A value exactly on a midpoint goes
    to the lower code.  A zero weight (+0 or -0) is always code 7, the exact
    zero level ("como funciona": zero padding quantises without error); this
    also covers blocks with c = 0 and blocks so small that RN32(1/c)
    overflows, where the product would be 0 * inf.
    """
    w = _blocks(w_bits, numel)
    c = np.asarray(c, dtype=np.float32)
    with np.errstate(divide="ignore", invalid="ignore", over="ignore"):
        rc = np.float32(1.0) / c
        x = (w * rc[:, None]).astype(np.float32)
    codes = nearest_code(x)
    codes[w == 0] = 7
    return codes


def nearest_code(x):
    """Index of the nearest level for normalised fp32 values: #{i : x > m_i}.

    Exactly on a midpoint the lower code wins; NaN gives 0 (callers exclude
    it).
    """
    x = np.asarray(x, dtype=np.float32)
    m = midpoints()
    return np.sum(x[..., None] > m, axis=-1).astype(np.uint8)


def pack_codes(codes):
    """Pack codes [nblocks, 64] two per byte: element 2j -> low nibble."""
    flat = np.asarray(codes, dtype=np.uint8).reshape(-1)
    return (flat[0::2] | (flat[1::2] << 4)).astype(np.uint8)


def unpack_codes(packed, numel):
    """Inverse of :func:`pack_codes`; returns one code per element."""
    packed = np.asarray(packed, dtype=np.uint8)
    out = np.empty(packed.size * 2, dtype=np.uint8)
    out[0::2] = packed & 0xF
    out[1::2] = packed >> 4
    return out[:numel]


def double_quantize(c):
    """FP8 double quantisation of the block constants ("como funciona").

    Groups of 256 consecutive constants (the last group zero padded).  Per
    group: amax = max c; s2 = RN32(amax / 448); c8 = E4M3(RN32(c / s2)) with
    round-to-nearest-even and saturation.  amax = 0 gives s2 = 0 and c8 = 0.
    The page says only "quantise the constants to FP8 in blocks of 256"; the
    absmax scale onto the E4M3 range, the fp32 scale and the absence of mean
    centring are this build's reading.
    """
    c = np.asarray(c, dtype=np.float32)
    nblocks = c.size
    ngroups = -(-nblocks // GROUP)
    cp = np.zeros(ngroups * GROUP, dtype=np.float32)
    cp[:nblocks] = c
    cg = cp.reshape(ngroups, GROUP)
    amax = np.max(cg, axis=1)
    s2 = (amax / np.float32(FP8_MAX)).astype(np.float32)
    with np.errstate(divide="ignore", invalid="ignore"):
        y = (cg / s2[:, None]).astype(np.float32)
    y[s2 == 0] = 0.0
    c8 = e4m3_encode(y).reshape(-1)[:nblocks]
    return c8, s2


def quantize(w_bits, numel=None):
    """Full NF4 quantisation of a bf16 tensor (flattened row-major).

    Returns ``(codes_packed, c8, s2)``: codes from the exact fp32 constants,
    then the constants double-quantised (the page describes double
    quantisation as a later step applied to the constants).
    """
    w_bits = np.asarray(w_bits, dtype=np.uint16).reshape(-1)
    numel = w_bits.size if numel is None else numel
    c = absmax_constants(w_bits, numel)
    codes = encode_codes(w_bits, numel, c)
    c8, s2 = double_quantize(c)
    return pack_codes(codes), c8, s2


def dequantized_constants(c8, s2):
    """c_hat = RN32(e4m3_to_f32(c8) * s2[group]) for every block."""
    c8 = np.asarray(c8, dtype=np.uint8)
    s2 = np.asarray(s2, dtype=np.float32)
    g = np.arange(c8.size) // GROUP
    return (e4m3_decode(c8) * s2[g]).astype(np.float32)


def dequantize(codes_packed, c8, s2, numel):
    """bf16 bit patterns of w' = bf16(RN32(q[code] * c_hat)).

    "a ideia": each weight is dequantised to BFloat16 at the moment of use.
    Two separate roundings (fp32 product, then bf16), no fused multiply-add.
    """
    nblocks = -(-numel // BLOCK)
    codes = unpack_codes(codes_packed, nblocks * BLOCK).reshape(nblocks, BLOCK)
    chat = dequantized_constants(c8, s2)
    q = codebook()
    vals = (q[codes] * chat[:, None]).astype(np.float32)
    return f32_to_bf16_bits(vals).reshape(-1)[:numel]


def bits_per_param(block=BLOCK, group=GROUP, const_bits=8, scale_bits=32):
    """Constant overhead in bits per parameter of the two-level scheme."""
    return const_bits / block + scale_bits / (block * group)

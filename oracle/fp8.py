"""FP8 (E4M3) quantisation of Q and K for the FP8 forward — TEST INFRASTRUCTURE ONLY.

The FP8 forward variant computes S = Q K^T on the tensor core from E4M3 codes
(the quantised-attention line of work, e.g. SageAttention2 in the related-paper
list of the scifaro.com related-papers page for arXiv 2411.10958: quantised
Q / K, exact attention otherwise).  What it must reach exactly is
masked softmax attention of the *dequantised* inputs, so the oracle is

    q_hat = decode(q8) * q_descale[b, h],   k_hat = decode(k8) * k_descale[b, h]
    O, LSE = forward_rows(q_hat, k_hat, v, ...)          (oracle.attention)

with the codes and scales produced by the quantiser below.

E4M3 is the OCP 8-bit floating-point format: 1 sign bit, 4 exponent bits
(bias 7), 3 mantissa bits; exponent field 0 holds the subnormals
2^-6 * m / 8; there are no infinities, and S.1111.111 is NaN, so the largest
finite magnitude is 2^8 * 1.75 = 448.  Conversion from float32 rounds to the
nearest representable value, ties to the even code, and saturates finite
values beyond 448 to +-448.

The quantiser (per batch*head slice of a [bh, rows, D] bf16 tensor) works in
float32 throughout:
    amax    = max |x| over the slice (exact: a maximum of bf16 values)
    inv     = float32(448) / amax          (1 if amax == 0)
    code    = encode(float32(x) * inv)
    descale = amax / float32(448)          (1 if amax == 0)
Each step is one correctly rounded float32 operation, so a device
implementation that performs the same operations reproduces the codes bit
for bit.
"""

import numpy as np

E4M3_MAX = 448.0


def e4m3_decode_table():
    """Value of each of the 256 codes (NaN for the two NaN codes), float64."""
    vals = np.empty(256, np.float64)
    for c in range(256):
        s = -1.0 if c & 0x80 else 1.0
        e = (c >> 3) & 0xF
        m = c & 0x7
        if e == 0xF and m == 0x7:
            vals[c] = np.nan
        elif e == 0:
            vals[c] = s * (2.0 ** -6) * (m / 8.0)
        else:
            vals[c] = s * (2.0 ** (e - 7)) * (1.0 + m / 8.0)
    return vals


_TABLE = e4m3_decode_table()
# non-negative finite codes in increasing order of value: 0x00 .. 0x7E
_POS_CODES = np.arange(0x7F, dtype=np.int64)
_POS_VALS = _TABLE[:0x7F]


def e4m3_decode(codes):
    """float64 values of uint8 codes."""
    return _TABLE[np.asarray(codes, dtype=np.uint8)]


def e4m3_encode(y):
    """Round float32 values to E4M3 codes: nearest, ties to the even code,
    finite values saturate to +-448, NaN maps to 0x7F."""
    y = np.asarray(y, dtype=np.float32).astype(np.float64)
    out = np.empty(y.shape, np.uint8)
    nan = np.isnan(y)
    a = np.minimum(np.abs(np.where(nan, 0.0, y)), E4M3_MAX)
    # the two neighbouring representable magnitudes lo <= a <= hi
    hi_i = np.searchsorted(_POS_VALS, a, side="left")
    hi_i = np.minimum(hi_i, len(_POS_VALS) - 1)
    lo_i = np.where(_POS_VALS[hi_i] == a, hi_i, np.maximum(hi_i - 1, 0))
    lo, hi = _POS_VALS[lo_i], _POS_VALS[hi_i]
    d_lo, d_hi = a - lo, hi - a
    pick_hi = (d_hi < d_lo) | ((d_hi == d_lo) & (hi_i % 2 == 0) & (hi_i != lo_i))
    mag = np.where(pick_hi, hi_i, lo_i).astype(np.uint8)
    neg = np.signbit(y) & ~nan
    out[...] = np.where(neg, mag | 0x80, mag)
    out[nan] = 0x7F
    return out


def quantize_e4m3(x):
    """Quantise a [bh, rows, D] array (bf16 values, any float dtype) per
    slice; returns (codes uint8 [bh, rows, D], descale float32 [bh])."""
    x = np.asarray(x, dtype=np.float32)
    codes = np.empty(x.shape, np.uint8)
    descale = np.empty(x.shape[0], np.float32)
    for i in range(x.shape[0]):
        amax = np.float32(np.max(np.abs(x[i]))) if x[i].size else np.float32(0)
        if amax > 0:
            inv = np.float32(E4M3_MAX) / amax
            descale[i] = amax / np.float32(E4M3_MAX)
        else:
            inv = np.float32(1.0)
            descale[i] = np.float32(1.0)
        codes[i] = e4m3_encode(x[i] * inv)
    return codes, descale


def dequantize_e4m3(codes, descale):
    """float64 [bh, rows, D] values of per-slice quantised codes."""
    v = e4m3_decode(codes)
    return v * np.asarray(descale, np.float64).reshape((-1,) + (1,) * (v.ndim - 1))

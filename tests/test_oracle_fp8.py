"""Pins of the E4M3 oracle (oracle/fp8.py) against the format's definition.

The values below come from the OCP 8-bit floating-point format (E4M3:
sign, 4 exponent bits with bias 7, 3 mantissa bits, subnormals at exponent
field 0, S.1111.111 = NaN, no infinities), not from the oracle's own code:
hand-computed codes, a brute-force nearest-value search over the 254 finite
values, and the half-ulp error bound of a 3-bit mantissa.
"""

import numpy as np
import pytest

from oracle import fp8

pytestmark = pytest.mark.filterwarnings("ignore::RuntimeWarning")


def test_decode_table_matches_hand_values():
    t = fp8.e4m3_decode_table()
    hand = {
        0x00: 0.0, 0x01: 2.0 ** -9, 0x07: 7 * 2.0 ** -9, 0x08: 2.0 ** -6, 0x30: 0.5, 0x38: 1.0, 0x39: 1.125,
        0x3F: 1.875, 0x40: 2.0, 0x48: 4.0, 0x70: 128.0, 0x78: 256.0, 0x7E: 448.0, 0xB8: -1.0, 0xFE: -448.0,
    }
    for c, v in hand.items():
        assert t[c] == v, hex(c)
    assert np.isnan(t[0x7F]) and np.isnan(t[0xFF])
    assert np.isfinite(t).sum() == 254
    assert t[0x80] == 0.0 and np.signbit(t[0x80])
    # the positive codes 0x00..0x7E are strictly increasing in value
    assert np.all(np.diff(t[:0x7F]) > 0)
    # negative codes mirror the positive ones
    assert np.array_equal(t[0x81:0xFF], -t[0x01:0x7F])


def test_encode_round_trips_every_finite_code():
    t = fp8.e4m3_decode_table()
    codes = np.array([c for c in range(256) if np.isfinite(t[c])], np.uint8)
    assert np.array_equal(fp8.e4m3_encode(t[codes].astype(np.float32)), codes)


def test_encode_is_nearest_with_ties_to_even_by_brute_force():
    t = fp8.e4m3_decode_table()
    finite = np.array([c for c in range(256) if np.isfinite(t[c]) and c != 0x80])  # +0 stands for both zeros
    rng = np.random.default_rng(8)
    y = np.concatenate([rng.uniform(-460, 460, 4000), rng.uniform(-2.0 ** -5, 2.0 ** -5, 2000),
                        np.array([1.0625, 1.1875, 3.5 * 2 ** -9, 2.0 ** -10, 240.0, 464.0, -1e9, 1e9])]).astype(np.float32)
    got = fp8.e4m3_encode(y)
    yc = np.clip(y.astype(np.float64), -448.0, 448.0)
    for yi, g in zip(yc, got):
        d = np.abs(t[finite] - yi)
        best = d.min()
        cands = finite[d == best]
        gv = t[g]
        assert abs(gv - yi) == best or (gv == 0.0 and best == abs(yi))
        if len(cands) == 2:  # a tie: the even code wins
            assert (g & 0x7F) % 2 == 0


def test_encode_special_cases():
    got = fp8.e4m3_encode(np.array([1.0625, 1.1875, 500.0, -1e9, 2.0 ** -10, 1.5 * 2.0 ** -10, 0.0], np.float32))
    # ties to even (1.0, 1.25), saturation (+-448), the half-way point below the
    # smallest subnormal goes to zero, just above it to the subnormal
    assert got.tolist() == [0x38, 0x3A, 0x7E, 0xFE, 0x00, 0x01, 0x00]
    assert fp8.e4m3_encode(np.array([-0.0], np.float32))[0] == 0x80


def test_quantize_scales_and_error_bound():
    rng = np.random.default_rng(3)
    x = rng.standard_normal((3, 40, 16)).astype(np.float32)
    x[1] *= 1e-3
    x[2] = 0.0
    codes, descale = fp8.quantize_e4m3(x)
    # the element of largest magnitude lands on +-448 exactly
    for i in range(2):
        j = np.unravel_index(np.argmax(np.abs(x[i])), x[i].shape)
        assert fp8.e4m3_decode(codes[i][j]) == np.sign(x[i][j]) * 448.0
        assert descale[i] == np.float32(np.max(np.abs(x[i]))) / np.float32(448.0)
    assert descale[2] == 1.0 and not codes[2].any()
    # relative error of a normal E4M3 value is at most half an ulp: 2^-4
    deq = fp8.dequantize_e4m3(codes, descale)
    for i in range(2):
        big = np.abs(x[i]) * (448.0 / np.abs(x[i]).max()) >= 2.0 ** -6
        rel = np.abs(deq[i][big] - x[i][big]) / np.abs(x[i][big])
        assert rel.max() <= 2.0 ** -4 + 1e-7

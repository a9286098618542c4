"""Pins for the oracle's FP8 (E4M3) cache quantiser.

The quantiser is this build's own definition (the pages fix no KV-cache
quantisation); these tests pin it against a brute-force nearest-code search
over all 256 E4M3 codes with ties to even, against exactly representable
rows, and against the E4M3 error bound.
"""

import numpy as np
import pytest

from oracle import star_oracle as so


def brute_force_codes(y):
    """Nearest E4M3 code to each float32 value, ties to the even code."""
    codes = np.arange(256)
    vals = so.e4m3_value(codes)
    ok = ~(((codes >> 3) & 0xF) == 0xF) | ((codes & 7) != 7)        # drop the NaN codes
    codes, vals = codes[ok], vals[ok]
    out = np.empty(y.shape, dtype=np.uint8)
    for idx, v in np.ndenumerate(y.astype(np.float64)):
        d = np.abs(vals - v)
        best = np.nonzero(d == d.min())[0]
        if len(best) > 1:                     # tie: even mantissa, and +0 over -0
            even = [b for b in best if (codes[b] & 1) == 0]
            best = even if even else best
            best = [b for b in best if codes[b] != 0x80] or best
        out[idx] = codes[best[0]]
    return out


def test_quantiser_matches_brute_force_rounding(rng):
    x = (rng.standard_normal((6, 64)) * rng.choice([1e-3, 1.0, 40.0], size=(6, 1))).astype(np.float32)
    codes, s = so.fp8_quantize_rows(x)
    inv = (np.float32(1) / s).astype(np.float32)
    y = (x * inv[:, None]).astype(np.float32)
    assert np.array_equal(codes, brute_force_codes(y))
    assert (np.abs(y).max(axis=1) <= 448.0 * (1 + 2 ** -20)).all()


def test_representable_rows_round_trip_exactly():
    vals = so.e4m3_value(np.array([0x7E, 0x38, 0x01, 0x45, 0xC0, 0x00, 0x2A, 0x7E]))   # 448 is the max
    for k in (-3, 0, 5):
        x = (vals * 2.0 ** k).astype(np.float32)[None]
        codes, s = so.fp8_quantize_rows(x)
        assert s[0] == np.float32(2.0 ** k)
        np.testing.assert_array_equal(so.fp8_dequantize_rows(codes, s), x.astype(np.float64))


def test_error_bound_and_zero_rows(rng):
    x = rng.standard_normal((50, 128)).astype(np.float32)
    x[3] = 0.0
    codes, s = so.fp8_quantize_rows(x)
    assert s[3] == 1.0 and not codes[3].any()
    xh = so.fp8_dequantize_rows(codes, s)
    # E4M3: 3 mantissa bits (half-ulp 2^-4 relative) down to 2^-6, subnormal step 2^-9
    bound = np.maximum(np.abs(x) * 2.0 ** -4, s[:, None] * 2.0 ** -10) * (1 + 1e-6)
    assert (np.abs(xh - x) <= bound).all()


def test_planted_rounding_mistake_is_caught(rng, monkeypatch):
    good = so.fp8_quantize_rows

    def truncating(x):      # round toward zero instead of to nearest
        import torch
        codes, s = good(x)
        x32 = np.asarray(x, np.float32)
        y = (x32 * (np.float32(1) / s)[:, None]).astype(np.float32)
        v = so.e4m3_value(codes)
        over = np.abs(v) > np.abs(y)
        codes = codes.copy()
        codes[over & (codes & 7 != 0)] -= 1
        return codes, s

    monkeypatch.setattr(so, "fp8_quantize_rows", truncating)
    with pytest.raises(AssertionError):
        test_quantiser_matches_brute_force_rounding(rng)

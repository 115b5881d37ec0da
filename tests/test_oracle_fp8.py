"""Pins for the oracle's e4m3 codec: textbook code values, exact round trips, brute
force over all codes, ties, saturation, and torch's own float8_e4m3fn cast."""
import numpy as np
import torch

from oracle import fp8


def test_textbook_values():
    assert fp8.e4m3_value(0x38) == 1.0            # exponent 7 = bias, mantissa 0
    assert fp8.e4m3_value(0x7E) == 448.0          # largest finite
    assert fp8.e4m3_value(0x01) == 2.0 ** -9      # smallest subnormal
    assert fp8.e4m3_value(0x08) == 2.0 ** -6      # smallest normal
    assert fp8.e4m3_value(0xB8) == -1.0
    assert np.isnan(fp8.e4m3_value(0x7F)) and np.isnan(fp8.e4m3_value(0xFF))
    assert fp8.MAX_FINITE == 448.0


def test_every_code_round_trips():
    for c in range(256):
        v = fp8.e4m3_value(c)
        if np.isnan(v):
            continue
        got = fp8.encode_one(v)
        assert fp8.e4m3_value(got) == v and (got == c or v == 0.0)


def test_nearest_by_brute_force():
    g = np.random.default_rng(0)
    vals = np.array([fp8.e4m3_value(c) for c in range(256)])
    finite = vals[~np.isnan(vals)]
    for x in np.concatenate([g.standard_normal(300) * 50, g.uniform(-0.02, 0.02, 100)]):
        code = fp8.encode_one(x)
        best = np.abs(finite - x).min()
        assert abs(fp8.e4m3_value(code) - x) == best


def test_ties_go_to_even_mantissa_and_overflow_saturates():
    assert fp8.encode_one(1.0625) == 0x38          # between 1.0 (m=0) and 1.125 (m=1)
    assert fp8.encode_one(1.1875) == 0x3A          # between 1.125 (m=1) and 1.25 (m=2)
    assert fp8.encode_one(1000.0) == 0x7E and fp8.encode_one(-1e9) == 0xFE
    assert fp8.encode_one(float("nan")) == 0x7F


def test_matches_torch_float8_cast_in_range():
    g = np.random.default_rng(1)
    x = np.concatenate([g.standard_normal(2000) * 30, g.standard_normal(500) * 1e-3])
    x = np.clip(x, -448, 448).astype(np.float32)
    ref = torch.from_numpy(x).to(torch.float8_e4m3fn).view(torch.uint8).numpy()
    assert np.array_equal(fp8.encode(x), ref)


def test_quantize_uses_float32_reciprocal():
    x = np.float32([0.3, -2.5, 7.0])
    s = 0.037
    inv = np.float32(1) / np.float32(s)
    assert np.array_equal(fp8.quantize(x, s), fp8.encode(x * inv))
    back = fp8.dequantize(fp8.quantize(x, s), s)
    assert np.all(np.abs(back - x) <= np.abs(x) * 2.0 ** -4 + 2.0 ** -9 * s)

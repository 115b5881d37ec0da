"""Plant plausible mistakes in the oracle's e4m3 codec and show that a pin of
``test_oracle_fp8`` catches each one (CPU only; every mutation is undone after its
test by pytest's monkeypatch)."""
import numpy as np
import pytest

import test_oracle_fp8 as pins
from oracle import fp8

PINS = [pins.test_textbook_values, pins.test_every_code_round_trips,
        pins.test_nearest_by_brute_force, pins.test_ties_go_to_even_mantissa_and_overflow_saturates,
        pins.test_matches_torch_float8_cast_in_range, pins.test_quantize_uses_float32_reciprocal]


def _caught() -> bool:
    for pin in PINS:
        try:
            pin()
        except AssertionError:
            return True
    return False


def _use_value_function(monkeypatch, value):
    """Replace the code -> value definition and every table built from it."""
    vals = np.array([value(c) for c in range(256)])
    pos = np.array([c for c in range(0x80) if not np.isnan(vals[c])], dtype=np.int64)
    monkeypatch.setattr(fp8, "e4m3_value", value)
    monkeypatch.setattr(fp8, "_VALUES", vals)
    monkeypatch.setattr(fp8, "_POS", pos)
    monkeypatch.setattr(fp8, "_POS_VAL", vals[pos])
    monkeypatch.setattr(fp8, "MAX_FINITE", float(vals[pos].max()))


def test_unmutated_codec_passes():
    assert not _caught()


def test_catches_wrong_exponent_bias(monkeypatch):
    def value(code):
        sign = -1.0 if code & 0x80 else 1.0
        e, m = (code >> 3) & 0xF, code & 0x7
        if e == 0xF and m == 0x7:
            return float("nan")
        if e == 0:
            return sign * (m / 8.0) * 2.0 ** -7
        return sign * (1.0 + m / 8.0) * 2.0 ** (e - 8)
    _use_value_function(monkeypatch, value)
    assert _caught()


def test_catches_wrong_subnormal_step(monkeypatch):
    def value(code):
        sign = -1.0 if code & 0x80 else 1.0
        e, m = (code >> 3) & 0xF, code & 0x7
        if e == 0xF and m == 0x7:
            return float("nan")
        if e == 0:
            return sign * (m / 8.0) * 2.0 ** -7         # half the true step
        return sign * (1.0 + m / 8.0) * 2.0 ** (e - 7)
    _use_value_function(monkeypatch, value)
    assert _caught()


def test_catches_ties_away_from_zero(monkeypatch):
    orig = fp8.encode_one

    def bad(x):
        code = orig(x)
        a = abs(float(x))
        i = int(np.searchsorted(fp8._POS_VAL, a))
        if 0 < i < len(fp8._POS_VAL) and a - fp8._POS_VAL[i - 1] == fp8._POS_VAL[i] - a:
            return (code & 0x80) | int(fp8._POS[i])          # always the larger magnitude
        return code
    monkeypatch.setattr(fp8, "encode_one", bad)
    assert _caught()


def test_catches_subnormals_flushed_to_zero(monkeypatch):
    orig = fp8.encode_one
    monkeypatch.setattr(fp8, "encode_one",
                        lambda x: (0x80 if x < 0 else 0) if abs(x) < 2.0 ** -6 else orig(x))
    assert _caught()


def test_catches_overflow_to_nan(monkeypatch):
    orig = fp8.encode_one
    monkeypatch.setattr(fp8, "encode_one", lambda x: 0x7F if abs(x) > 448.0 else orig(x))
    assert _caught()


def test_catches_scale_multiplied_instead_of_divided(monkeypatch):
    monkeypatch.setattr(fp8, "quantize",
                        lambda x, s: fp8.encode(np.asarray(x, np.float32) * np.float32(s)))
    assert _caught()

"""Pins for the oracle's number formats: bf16 rounding and the E4M3FN codec.

bf16: torch's fp32->bf16 cast (a library routine, round-to-nearest-even).
E4M3FN: facts of the OCP FP8 format (bias 7, max 448, smallest normal 2**-6,
smallest subnormal 2**-9, NaN = S.1111.111, no infinities), round trips of
all 256 codes, torch's float8_e4m3fn cast inside the finite range, and
saturation beyond it.
"""
import numpy as np
import pytest
import torch

from oracle import bf16_round, e4m3_decode, e4m3_encode, e4m3_values, quant_rows_e4m3


def test_bf16_round_matches_torch_cast():
    rng = np.random.default_rng(1)
    parts = [
        rng.standard_normal(200000).astype(np.float32),
        (rng.standard_normal(20000) * 1e30).astype(np.float32),
        (rng.standard_normal(20000) * 1e-38).astype(np.float32),   # bf16 subnormals
        np.array([0.0, -0.0, 1.0, -1.0, 3.0e38, -3.0e38, 1.00390625, 1.01171875], np.float32),
    ]
    # exact halfway cases between neighbouring bf16 values
    base = rng.standard_normal(5000).astype(np.float32)
    bits = base.view(np.uint32) & np.uint32(0xFFFF0000)
    parts.append((bits | np.uint32(0x8000)).view(np.float32))
    v = np.concatenate(parts)
    ref = torch.from_numpy(v).to(torch.bfloat16).float().numpy().astype(np.float64)
    got = bf16_round(v.astype(np.float64))
    np.testing.assert_array_equal(got, ref)


def test_e4m3_format_facts():
    assert e4m3_decode(0x7E) == 448.0
    assert e4m3_decode(0xFE) == -448.0
    assert e4m3_decode(0x38) == 1.0
    assert e4m3_decode(0x08) == 2.0 ** -6
    assert e4m3_decode(0x01) == 2.0 ** -9
    assert e4m3_decode(0x07) == 7 * 2.0 ** -9
    assert e4m3_decode(0x00) == 0.0
    assert np.isnan(e4m3_decode(0x7F)) and np.isnan(e4m3_decode(0xFF))
    vals = e4m3_values()
    assert vals.size == 127 and np.all(np.diff(vals) > 0)


def test_e4m3_round_trip_all_codes():
    codes = np.array([c for c in range(256) if c not in (0x7F, 0xFF)])
    back = e4m3_encode(e4m3_decode(codes))
    np.testing.assert_array_equal(back, codes.astype(np.uint8))


def test_e4m3_ties_to_even_and_saturation():
    # 1.0625 lies halfway between 1.0 (0x38) and 1.125 (0x39): even code wins
    assert e4m3_encode(1.0625) == 0x38
    assert e4m3_encode(1.1875) == 0x3A
    assert e4m3_encode(-1.0625) == 0xB8
    # beyond 448 saturates (satfinite), both signs
    assert e4m3_encode(449.0) == 0x7E
    assert e4m3_encode(1e9) == 0x7E
    assert e4m3_encode(-1e9) == 0xFE
    # 464 is halfway between 448 and the (non-existent) 480: saturate
    assert e4m3_encode(464.0) == 0x7E
    # below half the smallest subnormal rounds to zero
    assert e4m3_encode(2.0 ** -11) == 0x00
    assert e4m3_encode(2.0 ** -10 * 1.0001) == 0x01
    assert e4m3_encode(float("nan")) == 0x7F


def test_e4m3_encode_matches_torch_in_range():
    rng = np.random.default_rng(2)
    v = np.concatenate([
        rng.uniform(-448, 448, 100000),
        rng.standard_normal(100000) * 0.01,
        # midpoints of neighbouring codes
        (e4m3_values()[:-1] + e4m3_values()[1:]) / 2,
        -(e4m3_values()[:-1] + e4m3_values()[1:]) / 2,
    ]).astype(np.float32)
    ref = torch.from_numpy(v).to(torch.float8_e4m3fn).view(torch.uint8).numpy()
    got = e4m3_encode(v.astype(np.float64))
    np.testing.assert_array_equal(got, ref)


def test_quant_rows_scale_and_zero_row():
    a = np.zeros((3, 16), np.float32)
    a[1] = np.linspace(-3, 5, 16)
    a[2, 3] = -7.0
    q, s = quant_rows_e4m3(a)
    assert s.dtype == np.float32
    assert s[0] == 1.0 and np.all(q[0] == 0)
    assert s[1] == np.float32(5.0) / np.float32(448.0)
    # the row's max magnitude maps to the largest code
    assert q[1, 15] == 0x7E and q[2, 3] == 0xFE
    # decoded codes times the scale stay within half a code step (rel 1/16)
    back = e4m3_decode(q) * s[:, None]
    nz = np.abs(a) > 1e-2
    assert np.all(np.abs(back[nz] - a[nz]) <= np.abs(a[nz]) / 16 + 1e-7)


@pytest.mark.parametrize("bad", ["drop_subnormal", "ties_up"])
def test_planted_codec_mistakes_are_caught(bad, monkeypatch):
    """A wrong codec (planted in the oracle, on the CPU) fails the pins."""
    import oracle.moe_oracle as mo
    orig = mo.e4m3_encode

    def broken(v):
        v = np.asarray(v, dtype=np.float64)
        if bad == "drop_subnormal":
            v = np.where(np.abs(v) < 2.0 ** -6, 0.0, v)
            return orig(v)
        tab = mo.e4m3_values()
        a = np.minimum(np.abs(v), 448.0)
        hi = np.clip(np.searchsorted(tab, a), 0, 126)
        lo = np.clip(hi - 1, 0, 126)
        code = np.where(tab[hi] - a <= a - tab[lo], hi, lo)   # ties away
        return np.where(np.signbit(v), code | 0x80, code).astype(np.uint8)

    monkeypatch.setattr(mo, "e4m3_encode", broken)
    with pytest.raises(AssertionError):
        _check_round_trip(mo.e4m3_encode)
        _check_ties(mo.e4m3_encode)


def _check_round_trip(enc):
    codes = np.array([c for c in range(256) if c not in (0x7F, 0xFF)])
    np.testing.assert_array_equal(enc(e4m3_decode(codes)), codes.astype(np.uint8))


def _check_ties(enc):
    assert enc(1.0625) == 0x38 and enc(1.1875) == 0x3A

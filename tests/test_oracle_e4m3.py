"""Pins of the oracle's E4M3 encoder/decoder against things other than itself:
the OCP FP8 format's characteristic values (tests/golden), torch's independent
float8_e4m3fn implementation, and an exhaustive nearest-code search in exact
rational arithmetic."""

import math
import os
from fractions import Fraction

import numpy as np
import pytest
import torch

GOLDEN = os.path.join(os.path.dirname(__file__), "golden", "e4m3_special_values.txt")


def _golden():
    rows = []
    for line in open(GOLDEN):
        line = line.split("#")[0].strip()
        if line:
            code, val = line.split()
            rows.append((int(code, 16), float(val)))
    return rows


def test_decode_golden_values(oracle):
    for code, val in _golden():
        got = oracle.e4m3_decode(code)
        if math.isnan(val):
            assert math.isnan(got), hex(code)
        else:
            assert got == val and math.copysign(1, got) == math.copysign(1, val), hex(code)


def test_decode_matches_torch_for_all_codes(oracle):
    codes = torch.arange(256, dtype=torch.int32).to(torch.uint8)
    ref = codes.view(torch.float8_e4m3fn).to(torch.float64).numpy()
    got = oracle.e4m3_decode_table()
    nan = np.isnan(ref)
    assert np.array_equal(nan, np.isnan(got))
    assert np.array_equal(ref[~nan], got[~nan])
    assert np.array_equal(np.signbit(ref[~nan]), np.signbit(got[~nan]))
    assert nan.sum() == 2  # only S.1111.111


def test_decode_monotonic_and_spacing(oracle):
    mags = oracle.e4m3_decode_table()[:127]
    assert np.all(np.diff(mags) > 0)
    # 8 values per binade, spacing 2^(e-3) inside binade [2^e, 2^(e+1)), subnormal step 2^-9
    for c in range(1, 127):
        step = mags[c] - mags[c - 1]
        if c <= 8:
            assert step == 2.0 ** -9
        else:
            e = math.floor(math.log2(mags[c - 1]))
            assert step == 2.0 ** (e - 3)


def _nearest_code_exact(v: float) -> int:
    """Brute force over all finite codes in exact rationals; ties to the even code;
    magnitudes >= 448 saturate."""
    mags = [Fraction(x) for x in np.array([
        (m * 2.0 ** -9) if e == 0 else (1 + m / 8) * 2.0 ** (e - 7)
        for e in range(16) for m in range(8)])[:127]]
    a = Fraction(abs(v))
    sign = 0x80 if math.copysign(1.0, v) < 0 else 0
    if a >= 448:
        return 0x7E | sign
    best, best_d = None, None
    for c, m in enumerate(mags):
        d = abs(a - m)
        if best is None or d < best_d or (d == best_d and c % 2 == 0):
            best, best_d = c, d
    return best | sign


def _torch_encode(v: np.ndarray) -> np.ndarray:
    t = torch.from_numpy(np.ascontiguousarray(v, dtype=np.float32))
    t = t.clamp(-448.0, 448.0)  # torch's cast does not saturate
    return t.to(torch.float8_e4m3fn).view(torch.uint8).numpy()


def test_encode_golden_roundtrip(oracle):
    for code, val in _golden():
        if not math.isnan(val):
            assert oracle.e4m3_encode(val) == code


def test_encode_all_bf16_values_vs_torch(oracle):
    bits = np.arange(1 << 16, dtype=np.uint32) << 16
    v = bits.view(np.float32)
    v = v[np.isfinite(v)]
    assert np.array_equal(oracle.e4m3_encode_array(v), _torch_encode(v))


def test_encode_midpoints_and_neighbours_vs_torch(oracle):
    mags = oracle.e4m3_decode_table()[:127]
    mids = (mags[:-1] + mags[1:]) / 2
    vals = [np.float32(m) for m in np.concatenate([mids, mags])]
    out = []
    for x in vals:
        u = int(np.array([x], dtype=np.float32).view(np.uint32)[0])
        for d in range(-3, 4):
            if 0 <= u + d < 0x7F800000:
                out.append(np.array([u + d], np.uint32).view(np.float32)[0])
    v = np.array(out, dtype=np.float32)
    v = np.concatenate([v, -v, np.array([448.0, 449.0, 463.9, 464.0, 470.0, 1e30], np.float32)])
    got = oracle.e4m3_encode_array(v)
    assert np.array_equal(got, _torch_encode(v))


def test_encode_strided_fp32_patterns_vs_torch(oracle):
    # every 4099th finite fp32 bit pattern (~1M values spread over all binades)
    u = np.arange(0, 1 << 32, 4099, dtype=np.uint64).astype(np.uint32)
    v = u.view(np.float32)
    v = v[np.isfinite(v)]
    assert np.array_equal(oracle.e4m3_encode_array(v), _torch_encode(v))


def test_encode_vs_exact_brute_force(oracle):
    rng = np.random.default_rng(7)
    mags = oracle.e4m3_decode_table()[:127]
    mids = (mags[:-1] + mags[1:]) / 2
    v = np.concatenate([
        rng.standard_normal(300).astype(np.float32) * 50,
        rng.uniform(0, 2.0 ** -6, 100).astype(np.float32),
        mids.astype(np.float32),
        np.array([0.0, -0.0, 1e-30, -1e-30, 2.0 ** -10, 3 * 2.0 ** -11], np.float32),
    ])
    for x in v:
        assert oracle.e4m3_encode(float(x)) == _nearest_code_exact(float(x)), float(x)


def test_sign_of_zero(oracle):
    assert oracle.e4m3_encode(0.0) == 0x00
    assert oracle.e4m3_encode(-0.0) == 0x80
    assert oracle.e4m3_encode(-1e-12) == 0x80
    assert oracle.e4m3_encode(2.0 ** -11) == 0x00   # below half the subnormal step
    assert oracle.e4m3_encode(2.0 ** -10) == 0x00   # exact tie 0 vs 2^-9 -> even code 0x00
    assert oracle.e4m3_encode(3 * 2.0 ** -10) == 0x02  # tie 2^-9 vs 2*2^-9 -> even code 0x02


@pytest.mark.parametrize("amax", [1.0, 448.0, 1e-3, 3.0e38, 2.0 ** -133, 0.7109375])
def test_tile_scale_is_correctly_rounded_quotient(oracle, amax):
    """s is the fp32 value nearest to amax/448 (checked in exact rationals
    against both fp32 neighbours), and an all-zero tile has s = 1."""
    a = float(np.float32(amax))
    s = np.float32(oracle.tile_scale(a))
    exact = Fraction(a) / 448
    d = abs(Fraction(float(s)) - exact)
    for nb in (np.nextafter(s, np.float32(np.inf)), np.nextafter(s, np.float32(0))):
        assert d <= abs(Fraction(float(nb)) - exact)
    assert s > 0.0
    assert oracle.tile_scale(0.0) == 1.0

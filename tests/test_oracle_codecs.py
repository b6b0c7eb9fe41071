"""Pins for the oracle's number formats: e4m3fn and bf16.

The e4m3fn codec is pinned by exhaustion against the format definition
(1 sign, 4 exponent bits with bias 7, 3 mantissa bits, S.1111.111 = NaN) and
against torch's float8_e4m3fn conversion (a library routine); bf16 rounding
against torch's bfloat16 conversion and, for the single fp64 rounding of the
rotary table, against exact rational arithmetic.
"""

from fractions import Fraction

import numpy as np
import pytest
import torch


def _lib_decode_all():
    codes = torch.arange(256, dtype=torch.int32).to(torch.uint8)
    return codes.view(torch.float8_e4m3fn).float().numpy()


def test_e4m3_decode_every_code(oracle_mod):
    ours = oracle_mod.e4m3_to_f32(np.arange(256, dtype=np.uint8))
    lib = _lib_decode_all()
    nan = np.isnan(lib)
    assert nan.sum() == 2 and nan[0x7F] and nan[0xFF]
    assert np.isnan(ours[0x7F]) and np.isnan(ours[0xFF])
    assert np.array_equal(ours[~nan], lib[~nan])
    # hand values from the format definition
    assert ours[0x7E] == 448.0 and ours[0xFE] == -448.0
    assert ours[0x38] == 1.0 and ours[0xB8] == -1.0
    assert ours[0x08] == 2.0 ** -6          # smallest normal
    assert ours[0x01] == 2.0 ** -9          # smallest subnormal
    assert ours[0x07] == 7 * 2.0 ** -9      # largest subnormal
    assert ours[0x00] == 0.0 and np.signbit(ours[0x80])


def test_e4m3_round_trip_and_ties(oracle_mod):
    vals = oracle_mod.e4m3_to_f32(np.arange(256, dtype=np.uint8))
    finite = [c for c in range(256) if c not in (0x7F, 0xFF)]
    back = oracle_mod.f32_to_e4m3(vals[finite])
    assert np.array_equal(back, np.array(finite, dtype=np.uint8))
    # midpoints between neighbouring magnitudes go to the even code
    mids, want = [], []
    for c in range(0x00, 0x7E):
        lo, hi = float(vals[c]), float(vals[c + 1])
        mids += [(lo + hi) / 2, -(lo + hi) / 2]
        even = c if c % 2 == 0 else c + 1
        want += [even, even | 0x80]
    got = oracle_mod.f32_to_e4m3(np.array(mids, np.float32))
    assert np.array_equal(got, np.array(want, np.uint8))


def test_e4m3_saturates_and_keeps_sign(oracle_mod):
    got = oracle_mod.f32_to_e4m3(np.array(
        [449.0, 464.0, 1e6, -500.0, -1e-12, 1e-12, 0.0, -0.0], np.float32))
    assert list(got) == [0x7E, 0x7E, 0x7E, 0xFE, 0x80, 0x00, 0x00, 0x80]


def test_e4m3_matches_library_cast_on_sweep(oracle_mod):
    rng = np.random.default_rng(5)
    x = np.concatenate([
        rng.standard_normal(20000).astype(np.float32) * 30,
        rng.uniform(-2e-3, 2e-3, 5000).astype(np.float32),
        rng.uniform(-448, 448, 5000).astype(np.float32)])
    ours = oracle_mod.f32_to_e4m3(x)
    lib = torch.from_numpy(np.clip(x, -448, 448)).to(
        torch.float8_e4m3fn).view(torch.uint8).numpy()
    assert np.array_equal(ours, lib)


def test_bf16_matches_library(oracle_mod):
    rng = np.random.default_rng(6)
    x = rng.standard_normal(20000).astype(np.float32) * 10
    # exact ties: bf16 value plus half a unit in the last place
    base = torch.from_numpy(x[:2000]).to(torch.bfloat16).float().numpy()
    ties = (base.view(np.uint32) | np.uint32(0x8000)).view(np.float32)
    x = np.concatenate([x, ties])
    ours = oracle_mod.f32_to_bf16(x)
    lib = torch.from_numpy(x).to(torch.bfloat16).view(torch.int16).numpy()
    assert np.array_equal(ours, lib.view(np.uint16))


def _exact_bf16_of(d: float) -> int:
    """Nearest-even bf16 code of a double, by exact rational comparison."""
    if d == 0:
        return 0
    sign = 0x8000 if d < 0 else 0
    a = Fraction(abs(d))
    best = None
    # scan the bf16 codes around the float32 neighbourhood
    f = np.float32(abs(d))
    c0 = int(np.array([f], np.float32).view(np.uint32)[0] >> 16)
    for c in range(max(c0 - 2, 0), c0 + 3):
        v = Fraction(float(np.array([c << 16], np.uint32).view(np.float32)[0]))
        key = (abs(v - a), c % 2)
        if best is None or key < best[0]:
            best = (key, c)
    return best[1] | sign


def test_bf16_from_f64_single_rounding(oracle_mod):
    rng = np.random.default_rng(7)
    xs = list(rng.uniform(-1, 1, 400))
    # a double just above a bf16 midpoint whose float32 rounding lands on the
    # midpoint: a double rounding would tie to even (1.0), one rounding goes up
    xs += [1.0 + 2.0 ** -8 + 2.0 ** -40, -(1.0 + 2.0 ** -8 + 2.0 ** -40),
           1.0 + 2.0 ** -8]
    ours = oracle_mod.f64_to_bf16(np.array(xs))
    want = [_exact_bf16_of(v) for v in xs]
    assert list(ours) == want
    assert ours[-3] == 0x3F81 and ours[-1] == 0x3F80

"""The parity helpers' own behaviour (CPU): the e4m3 step distance that the
code bar counts with, checked against the e4m3fn format's code order."""

import numpy as np

from parity import e4m3_step_distance


def test_step_distance_adjacent_codes():
    # magnitudes are ordered by code: neighbours are one step apart
    a = np.arange(0, 0x7E, dtype=np.uint8)
    assert (e4m3_step_distance(a, a + 1) == 1).all()
    assert (e4m3_step_distance(a | 0x80, (a + 1) | 0x80) == 1).all()
    assert (e4m3_step_distance(a, a) == 0).all()


def test_step_distance_signed_zero_and_smallest_subnormal():
    assert e4m3_step_distance([0x00], [0x80])[0] == 1       # +0 vs -0
    assert e4m3_step_distance([0x00], [0x01])[0] == 1       # 0 vs 2^-9
    assert e4m3_step_distance([0x80], [0x01])[0] == 1       # -0 vs +2^-9
    assert e4m3_step_distance([0x81], [0x01])[0] == 2       # -2^-9 vs +2^-9
    assert e4m3_step_distance([0x05], [0x85])[0] == 2       # opposite signs


def test_step_distance_nan_is_never_one_step():
    # 0x7E / 0xFE are +-448 (the saturation value); 0x7F / 0xFF are NaN
    assert e4m3_step_distance([0x7F], [0x7E])[0] == 2
    assert e4m3_step_distance([0x7E], [0x7F])[0] == 2
    assert e4m3_step_distance([0xFF], [0xFE])[0] == 2
    assert e4m3_step_distance([0xFE], [0xFF])[0] == 2
    assert e4m3_step_distance([0x7F], [0x7F])[0] == 0


def test_rms_bar_accepts_one_bf16_step_only():
    import pytest
    from parity import assert_rms
    from fp8_transformer_block_b200.synth import bf16_bits
    rng = np.random.default_rng(0)
    ref = bf16_bits(rng.standard_normal(4096).astype(np.float32))
    big = int(np.argmax(np.abs(ref.view(np.int16).astype(np.int32) & 0x7FFF)))
    got = ref.copy()
    got[big] += 1                     # one step at the largest value: accepted
    assert_rms(got, ref)
    got[big] += 1                     # two steps (> 2e-2 * rms there): rejected
    with pytest.raises(AssertionError):
        assert_rms(got, ref)
    got = ref.copy()
    small = int(np.argmin(np.abs(ref.view(np.int16).astype(np.int32) & 0x7FFF)))
    got[small] = bf16_bits(np.array([0.5], np.float32))[0]   # far off at a small value: rejected
    with pytest.raises(AssertionError):
        assert_rms(got, ref)

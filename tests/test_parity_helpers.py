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

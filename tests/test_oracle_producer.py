"""Pins for the oracle's producers (AdaRMS and per-token-table LayerNorm).

Hand-enumerated D=8 rows, closed forms and invariants; each case is chosen
so that a plausible slip (a dropped gate term, swapped scale/shift chunks,
eps outside the root, weight not applied, wrong chunk index, unbiased
variance) fails it.
"""

import math

import numpy as np
import pytest

from fp8_transformer_block_b200.synth import bf16_bits, bf16_value


def _bf(x):
    return bf16_bits(np.asarray(x, np.float32))


def _style(scale, shift, gate, D):
    s = np.zeros((1, 3 * D), np.float32)
    s[0, :D], s[0, D:2 * D], s[0, 2 * D:] = scale, shift, gate
    return _bf(s)


def test_adarms_unit_rms_row(oracle_mod):
    D = 8
    res = _bf([[1, -1] * 4])
    z = _bf(np.zeros((1, D)))
    out = oracle_mod.ada_rms_norm_quant(res, z, _bf(np.zeros((1, D))),
                                        _style(0, 0, 0, D), 1.0, want_y=True)
    want = np.array([1, -1] * 4) / math.sqrt(1 + 1e-6)
    assert np.allclose(out["y"][0], want, rtol=1e-7, atol=0)
    assert list(out["x8"][0]) == [0x38, 0xB8] * 4       # +-1.0
    assert np.array_equal(out["res"], res)               # no gate, no change


def test_adarms_gated_residual_update(oracle_mod):
    D = 8
    res = _bf(np.ones((2, D)))
    delta = _bf(np.full((2, D), 0.5))
    gate = _bf(np.full((1, D), 2.0))
    out = oracle_mod.ada_rms_norm_quant(res, delta, gate, _style(0, 0, 0, D),
                                        1.0)
    assert np.all(bf16_value(out["res"]) == 2.0)         # 1 + 2 * 0.5
    # per-row gate: row 1 gate 0 leaves the residual alone
    g2 = _bf(np.stack([np.full(D, 2.0), np.zeros(D)]))
    out = oracle_mod.ada_rms_norm_quant(res, delta, g2, _style(0, 0, 0, D), 1.0)
    assert np.all(bf16_value(out["res"][0]) == 2.0)
    assert np.all(bf16_value(out["res"][1]) == 1.0)


def test_adarms_zero_input_gives_shift(oracle_mod):
    D = 8
    z = _bf(np.zeros((3, D)))
    shift = np.linspace(-3, 3, D).astype(np.float32)
    out = oracle_mod.ada_rms_norm_quant(z, z, _bf(np.zeros((1, D))),
                                        _style(0.7, shift, 0, D), 0.25,
                                        want_y=True)
    assert np.array_equal(out["y"], np.tile(bf16_value(_bf(shift)), (3, 1)))


def test_adarms_scale_shift_chunk_order_and_gate_out(oracle_mod):
    D = 8
    res = _bf([[2, -2] * 4])
    z = _bf(np.zeros((1, D)))
    r = 1 / math.sqrt(4 + 1e-6)                           # ms = 4
    a = oracle_mod.ada_rms_norm_quant(res, z, z, _style(3, 0, 0, D), 1.0,
                                      want_y=True)
    assert np.allclose(a["y"][0], np.array([2, -2] * 4) * r * 4, rtol=1e-6)
    b = oracle_mod.ada_rms_norm_quant(res, z, z, _style(0, 3, 0, D), 1.0,
                                      want_y=True)
    assert np.allclose(b["y"][0], np.array([2, -2] * 4) * r + 3, rtol=1e-6)
    gate = np.arange(D, dtype=np.float32) - 4
    c = oracle_mod.ada_rms_norm_quant(res, z, z, _style(0, 0, gate, D), 1.0)
    assert np.array_equal(c["gate_out"][0], _bf(gate))


def test_adarms_eps_inside_root(oracle_mod):
    D = 8
    v = 2.0 ** -10
    res = _bf(np.full((1, D), v))
    z = _bf(np.zeros((1, D)))
    out = oracle_mod.ada_rms_norm_quant(res, z, z, _style(0, 0, 0, D), 1.0,
                                        want_y=True)
    want = v / math.sqrt(v * v + 1e-6)                    # ~0.6987, not 1
    assert abs(out["y"][0, 0] - want) < 1e-6 * want


def test_adarms_weight_and_quant_scale(oracle_mod):
    D = 8
    res = _bf([[1, -1] * 4])
    z = _bf(np.zeros((1, D)))
    w = _bf(np.full(D, 2.0))
    out = oracle_mod.ada_rms_norm_quant(res, z, z, _style(0.5, 0.25, 0, D),
                                        0.5, weight=w, want_y=True)
    x_hat = np.array([1, -1] * 4) / math.sqrt(1 + 1e-6)
    y = x_hat * 2 * 1.5 + 0.25
    assert np.allclose(out["y"][0], y, rtol=1e-6)
    # y / 0.5 = 6.5 / -5.5: 6.5 = 1.625 * 2^2 -> exponent field 9, mantissa 5
    # (0x4D); -5.5 = -1.375 * 2^2 -> mantissa 3, sign set (0xCB)
    assert list(out["x8"][0]) == [0x4D, 0xCB] * 4


def test_adarms_unit_rms_and_scale_invariance(oracle_mod):
    rng = np.random.default_rng(11)
    D = 512
    x = rng.standard_normal((4, D)).astype(np.float32)
    z = _bf(np.zeros((1, D)))
    zz = _bf(np.zeros((4, D)))
    a = oracle_mod.ada_rms_norm_quant(_bf(x), zz, z, _style(0, 0, 0, D),
                                      1.0, want_y=True)
    rms = np.sqrt((a["y"].astype(np.float64) ** 2).mean(axis=1))
    assert np.allclose(rms, 1.0, atol=1e-5)
    b = oracle_mod.ada_rms_norm_quant(_bf(x * 16), zz, z, _style(0, 0, 0, D),
                                      1.0, want_y=True)
    assert np.allclose(a["y"], b["y"], rtol=1e-5, atol=1e-6)
    assert b["amax"] == np.abs(b["y"]).max()


def test_layer_norm_hand_row(oracle_mod):
    D = 8
    x = _bf([np.arange(1, 9)])
    temb = _bf(np.zeros((1, 6, D)))
    table = np.zeros((6, D), np.float32)
    out = oracle_mod.ada_layer_norm_quant_table(x, temb, table, 0, 1, 1.0,
                                                want_y=True)
    want = (np.arange(1, 9) - 4.5) / math.sqrt(5.25 + 1e-6)   # biased var
    assert np.allclose(out["y"][0], want, rtol=1e-6)


def test_layer_norm_chunk_selection(oracle_mod):
    D = 8
    x = _bf([np.arange(1, 9)])
    table = np.full((6, D), 100.0, np.float32)
    table[3], table[4] = 0.5, 1.0                  # FFN site: shift 3, scale 4
    temb = np.zeros((1, 6, D), np.float32)
    temb[0, 3] = 0.25                              # per-token shift add
    out = oracle_mod.ada_layer_norm_quant_table(x, _bf(temb), table, 3, 4,
                                                1.0, want_y=True)
    x_hat = (np.arange(1, 9) - 4.5) / math.sqrt(5.25 + 1e-6)
    assert np.allclose(out["y"][0], x_hat * 2.0 + 0.75, rtol=1e-6)


def test_layer_norm_constant_row_and_moments(oracle_mod):
    D = 64
    x = _bf(np.full((1, D), 3.0))
    shift = np.linspace(-1, 1, D).astype(np.float32)
    table = np.zeros((6, D), np.float32)
    table[0] = shift
    temb = _bf(np.zeros((1, 6, D)))
    out = oracle_mod.ada_layer_norm_quant_table(x, temb, table, 0, 1, 1.0,
                                                want_y=True)
    assert np.array_equal(out["y"][0], shift)
    rng = np.random.default_rng(12)
    xr = _bf(rng.standard_normal((3, 1024)) * 5 + 2)
    out = oracle_mod.ada_layer_norm_quant_table(
        xr, _bf(np.zeros((3, 6, 1024))), np.zeros((6, 1024), np.float32),
        0, 1, 1.0, want_y=True)
    y = out["y"].astype(np.float64)
    assert np.allclose(y.mean(axis=1), 0, atol=1e-5)
    assert np.allclose(y.var(axis=1), 1, atol=1e-4)

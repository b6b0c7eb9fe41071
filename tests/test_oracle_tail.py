"""Pins of the oracle's output-side pieces of the AdaRMS layer: the static
quantize in front of the output projection and the stack's final AdaRMS
tail (impls/adarms_stack/fp8_chain.py: `out_project`, and the "ad:tail"
range of `_make_run`).  Each check is a value the definitions fix."""

import numpy as np

import oracle


def _bf16(x):
    return oracle.f32_to_bf16(np.asarray(x, dtype=np.float32))


def test_quant_roundtrips_every_finite_code():
    # dec(c) * 2^-3 is exact in bf16 for every finite e4m3 code c, so the
    # quantizer must return c itself (signed zero included)
    codes = np.array([c for c in range(256) if c not in (0x7F, 0xFF)], np.uint8)
    vals = oracle.e4m3_to_f32(codes) * np.float32(0.125)
    x = _bf16(vals).reshape(1, -1)
    assert np.array_equal(oracle.bf16_to_f32(x[0]), vals)
    x8, amax = oracle.quant_fp8_static(x, 0.125)
    assert np.array_equal(x8[0], codes)
    assert amax == 448.0 * 0.125


def test_quant_saturates_and_keeps_sign():
    s = 0.25
    x = _bf16([[449 * s, -449 * s, 1000 * s, -1000 * s, 0.0, -0.0, 3e-7, -3e-7]])
    x8, amax = oracle.quant_fp8_static(x, s)
    assert list(x8[0]) == [0x7E, 0xFE, 0x7E, 0xFE, 0x00, 0x80, 0x00, 0x80]
    assert amax == float(oracle.bf16_to_f32(x[0, 2]))


def _tail(res, delta, gate, scale, shift, eps=1e-6):
    res, delta, gate = (np.atleast_2d(np.asarray(a, np.uint16)) for a in (res, delta, gate))
    D = res.shape[1]
    fin = np.stack([np.broadcast_to(np.float32(scale), (D,)),
                    np.broadcast_to(np.float32(shift), (D,))]).astype(np.float32)
    return oracle.ada_rms_tail(res, delta, gate, fin, eps)


def test_tail_unit_rms_row_maps_to_plus_minus_one():
    h = _bf16([1, -1, 1, -1, 1, -1, 1, -1]).reshape(1, 8)
    z = np.zeros((1, 8), np.uint16)
    out = _tail(h, z, z, 0.0, 0.0)
    # ms = 1, 1/sqrt(1 + 1e-6) rounds, after the product, to +-1 in bf16
    assert list(out[0]) == [0x3F80, 0xBF80] * 4


def test_tail_gated_delta_equals_the_same_residual():
    rng = np.random.default_rng(3)
    x = _bf16(rng.normal(size=(4, 64)))
    half = _bf16(oracle.bf16_to_f32(x) * np.float32(0.5))   # exact: a power of two
    two = _bf16(np.full((1, 64), 2.0))
    z = np.zeros((4, 64), np.uint16)
    a = _tail(x, z, np.zeros((1, 64), np.uint16), 0.3, -0.2)
    b = _tail(z, half, two, 0.3, -0.2)
    assert np.array_equal(a, b)


def test_tail_scale_minus_one_leaves_the_shift():
    rng = np.random.default_rng(4)
    x = _bf16(rng.normal(size=(3, 32)))
    z = np.zeros((3, 32), np.uint16)
    out = _tail(x, z, np.zeros((1, 32), np.uint16), -1.0, 0.375)
    assert np.all(out == _bf16(0.375))


def test_tail_output_has_unit_rms():
    rng = np.random.default_rng(5)
    x = _bf16(rng.normal(size=(16, 512)) * 3.0)
    z = np.zeros((16, 512), np.uint16)
    y = oracle.bf16_to_f32(_tail(x, z, np.zeros((1, 512), np.uint16), 0.0, 0.0))
    ms = (y.astype(np.float64) ** 2).mean(axis=1)
    assert np.all(np.abs(ms - 1.0) < 1e-2)


def test_tail_norm_sees_the_unrounded_sum():
    # h = (1 + 2^-9, 1) is not a bf16 pair: rms(h) = 1 + 2^-10 (to first
    # order), so h / rms(h) - 1 = (+2^-10, -2^-10); rounding h to bf16 first
    # would give (1, 1) and an output of ~0 in both columns
    res = _bf16([[1.0, 1.0]])
    delta = _bf16([[2.0 ** -9, 0.0]])
    gate = _bf16([[1.0, 1.0]])
    out = oracle.bf16_to_f32(_tail(res, delta, gate, 0.0, -1.0))
    assert abs(out[0, 0] - 2.0 ** -10) < 1e-4 and abs(out[0, 1] + 2.0 ** -10) < 1e-4


def test_layer_stack_wiring_with_silent_projections():
    # with zero o and down weights the FFN half adds nothing: the residual
    # leaving the layer is the one the q/k/v norm stored, and the tail sees
    # a zero delta (checks the loop's order and which tensor feeds which)
    rng = np.random.default_rng(8)
    D, M, H = 64, 4, 128
    dims = {"B": 1, "M": M, "D": D, "hq": 1, "hkv": 1, "hd": 64, "P": 0, "T": M, "H": H}
    wq = [oracle.f32_to_bf16(rng.normal(0, 0.05, size=(64, D)).astype(np.float32))
          for _ in range(3)]
    zero_o = np.zeros((D, D), np.uint16)
    mlp = [oracle.f32_to_bf16(rng.normal(0, 0.05, size=(H, D)).astype(np.float32))
           for _ in range(2)]
    layer = {"qkv": oracle.pack_weights_fp8(wq, layout=1, hd=64),
             "o": oracle.pack_weights_fp8([zero_o]),
             "gu": oracle.pack_weights_fp8(mlp),
             "dn": oracle.pack_weights_fp8([np.zeros((D, H), np.uint16)]),
             "styles": oracle.f32_to_bf16(rng.normal(0, 0.2, size=(2, 3 * D))
                                          .astype(np.float32))}
    x = oracle.f32_to_bf16(rng.normal(size=(M, D)).astype(np.float32))
    fin = rng.normal(0, 0.1, size=(3, D)).astype(np.float32)
    out, recs, scales = oracle.adarms_layer_stack(x, [layer], fin, dims)
    r = recs[0]
    assert not np.any(r["dn_o"]) and not np.any(r["dn"])
    first = oracle.ada_rms_norm_quant(x, np.zeros((M, D), np.uint16),
                                      np.zeros((1, D), np.uint16), layer["styles"][0:1],
                                      scales[0]["a_qkv"])
    assert np.array_equal(r["res"], first["res"])
    assert np.array_equal(r["x8"], first["x8"])
    want = oracle.ada_rms_tail(first["res"], np.zeros((M, D), np.uint16), r["g2"], fin, 1e-6)
    assert np.array_equal(out, want)


def _gelu_vals(x, scale=1.0 / 32):
    u = _bf16(np.asarray(x, np.float32).reshape(1, -1))
    hid, amax = oracle.gelu_quant(u, scale)
    return oracle.e4m3_to_f32(hid[0]) * np.float32(scale), amax


def test_gelu_quant_fixed_points():
    # gelu(0) = 0; gelu(x) -> x for large x and -> 0 for large -x; the
    # odd-part identity gelu(x) - gelu(-x) = x (the tanh factor is odd)
    v, _ = _gelu_vals([0.0, 6.0, -6.0, 10.0, -10.0])
    assert v[0] == 0.0 and v[2] == 0.0 and v[4] == 0.0
    assert abs(v[1] - 6.0) <= 6.0 / 8 and abs(v[3] - 10.0) <= 10.0 / 8  # one e4m3 step
    xs = np.array([0.25, 0.5, 1.0, 1.5, 2.0, 3.0], np.float32)
    u = _bf16(np.concatenate([xs, -xs]).reshape(1, -1))
    hid, _ = oracle.gelu_quant(u, 1.0 / 128)     # 3 * 128 < 448: no saturation
    g = oracle.e4m3_to_f32(hid[0]).astype(np.float64) / 128
    diff = g[:6] - g[6:]
    assert np.all(np.abs(diff - xs) <= 0.07 * xs + 2e-3)   # within e4m3 rounding


def test_gelu_quant_amax_is_the_largest_output():
    u = _bf16(np.array([[-3.0, -0.5, 0.0, 0.7, 2.5]], np.float32))
    _, amax = oracle.gelu_quant(u, 1.0)
    # gelu is increasing for x > -0.75: the largest value is gelu(2.5) ~ 2.48
    assert 2.45 < amax < 2.5


def test_dit_ffn_wiring_zero_up_projection_gives_the_down_bias():
    # u = 0 -> gelu(0) = 0 -> hid8 = 0 -> ff = bf16(0 * alpha + bias_dn)
    from fp8_transformer_block_b200 import synth
    rng = np.random.default_rng(12)
    D, H, rows = 64, 128, 5
    inp = synth.dit_inputs(rows, D, 3)
    up = oracle.pack_weights_fp8([np.zeros((H, D), np.uint16)], [np.zeros(H, np.uint16)])
    bias_dn = _bf16(rng.normal(0, 0.3, size=D).astype(np.float32))
    dn = oracle.pack_weights_fp8([_bf16(rng.normal(0, 0.02, size=(D, H)).astype(np.float32))],
                                 [bias_dn])
    r = oracle.dit_ffn(inp["x"], inp["temb"], inp["table"], up, dn, 0.02, a_hid=0.01)
    assert not np.any(r["hid8"])
    assert np.array_equal(r["ff"], np.broadcast_to(bias_dn, (rows, D)))

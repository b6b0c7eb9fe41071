"""Pins for the oracle's pack, GEMM, rotary table, split+RoPE+KV write,
prefix copy and GEGLU requant.

Pins come from outside the oracle: library routines (numpy fp64 matmul,
numpy cos/sin, torch's tanh-GELU), closed forms (zero input gives the bias,
position 0 is the identity, GELU odd-part identity), invariants the pages
rely on (packed GEMM equals the sibling GEMMs; attention scores unchanged
by the shared q/k permutation that maps rotate-half onto adjacent pairs;
RoPE keeps norms and depends on relative position only) and brute force.
"""

import math

import numpy as np
import pytest
import torch

from fp8_transformer_block_b200.synth import bf16_bits, bf16_value


def _bf(x):
    return bf16_bits(np.asarray(x, np.float32))


def _rand_bf(rng, shape, std=1.0):
    return _bf(rng.standard_normal(shape) * std)


# ---------------------------------------------------------------- pack ----

def test_pack_scale_and_extreme_codes(oracle_mod):
    rng = np.random.default_rng(21)
    ws = [_rand_bf(rng, (16, 32), 0.02), _rand_bf(rng, (8, 32), 0.05)]
    p = oracle_mod.pack_weights_fp8(ws)
    allw = np.concatenate([bf16_value(w) for w in ws])
    amax = np.abs(allw).max()
    assert p["w_scale"] == np.float32(amax) / np.float32(448.0)
    i = np.unravel_index(np.abs(allw).argmax(), allw.shape)
    assert p["w8"][i] in (0x7E, 0xFE)
    dq = oracle_mod.e4m3_to_f32(p["w8"]) * p["w_scale"]
    # nearest-code rounding: within half a step (2^-4 relative for normals,
    # 2^-10 * scale absolute in the subnormal range)
    err = np.abs(dq - allw)
    bound = np.maximum(np.abs(allw) * 2.0 ** -4, 2.0 ** -10 * p["w_scale"])
    assert np.all(err <= bound * (1 + 1e-6))
    assert np.array_equal(p["bias"], np.zeros(24, np.uint16))


def test_pack_all_zero_floor(oracle_mod):
    p = oracle_mod.pack_weights_fp8([np.zeros((4, 16), np.uint16)])
    assert p["w_scale"] == np.float32(1e-8)
    assert not p["w8"].any()


def test_pack_qk_interleave_map(oracle_mod):
    hd, K = 4, 16
    # row r of each sibling carries the constant r+1 (distinct codes)
    q = _bf(np.repeat(np.arange(1, 9)[:, None], K, 1) * 0.01)      # 2 heads
    k = _bf(np.repeat(np.arange(1, 5)[:, None], K, 1) * 0.01)      # 1 head
    v = _bf(np.repeat(np.arange(1, 5)[:, None], K, 1) * 0.01)
    plain = oracle_mod.pack_weights_fp8([q, k, v])
    inter = oracle_mod.pack_weights_fp8([q, k, v], layout=1, hd=hd)
    # per head [a0, a1, a2, a3] -> [a0, a2, a1, a3]; v unchanged
    order = [0, 2, 1, 3, 4, 6, 5, 7, 8, 10, 9, 11, 12, 13, 14, 15]
    assert np.array_equal(inter["w8"], plain["w8"][order])
    # the chain's kperm gather (kperm[2i]=i, kperm[2i+1]=hd/2+i) undoes it
    kperm = np.empty(hd, int)
    kperm[0::2], kperm[1::2] = np.arange(hd // 2), np.arange(hd // 2, hd)
    inv = np.argsort(kperm)
    assert np.array_equal(inter["w8"][:4][inv], plain["w8"][:4])


def test_pack_bias_concat_and_layouts(oracle_mod):
    rng = np.random.default_rng(22)
    g, u = _rand_bf(rng, (256, 16), 0.02), _rand_bf(rng, (256, 16), 0.02)
    bg = _rand_bf(rng, (256,), 0.01)
    plain = oracle_mod.pack_weights_fp8([g, u], [bg, None])
    assert np.array_equal(plain["bias"][:256], bg)
    assert not plain["bias"][256:].any()
    # the oracle packs only the pages' two orders (concatenation, q/k
    # interleave); the library's gate/up block order is a test-side
    # permutation of the concatenation
    with pytest.raises(ValueError):
        oracle_mod.pack_weights_fp8([g, u], layout=2)


def test_gate_up_block_order_by_enumeration():
    from parity import gate_up_block_order
    o = gate_up_block_order(256)
    want = list(range(0, 128)) + list(range(256, 384)) + \
        list(range(128, 256)) + list(range(384, 512))
    assert o.tolist() == want
    assert sorted(gate_up_block_order(1024).tolist()) == list(range(2048))


# ---------------------------------------------------------------- gemm ----

def test_gemm_zero_input_gives_bias(oracle_mod):
    rng = np.random.default_rng(23)
    w8 = rng.integers(0, 0x7E, (40, 64), dtype=np.uint8)
    bias = _rand_bf(rng, (40,), 0.5)
    y = oracle_mod.fp8_gemm(np.zeros((5, 64), np.uint8), w8, 0.3, 0.01, bias)
    assert np.array_equal(y, np.tile(bias, (5, 1)))


def test_gemm_single_hot_column(oracle_mod):
    rng = np.random.default_rng(24)
    w8 = rng.integers(0, 0x7E, (24, 32), dtype=np.uint8)
    x8 = np.zeros((1, 32), np.uint8)
    x8[0, 5] = 0x38                                   # 1.0 at k = 5
    y = oracle_mod.fp8_gemm(x8, w8, 0.5, 0.25)
    want = _bf(oracle_mod.e4m3_to_f32(w8[:, 5]) * np.float32(0.125))
    assert np.array_equal(y[0], want)


def test_gemm_against_fp64_matmul(oracle_mod):
    rng = np.random.default_rng(25)
    M, N, K = 33, 48, 256
    x8 = oracle_mod.f32_to_e4m3(rng.standard_normal((M, K)) * 50)
    w8 = oracle_mod.f32_to_e4m3(rng.standard_normal((N, K)) * 100)
    bias = _rand_bf(rng, (N,), 1.0)
    a, s = 0.011, 0.0007
    y = bf16_value(oracle_mod.fp8_gemm(x8, w8, a, s, bias))
    ref = (oracle_mod.e4m3_to_f32(x8).astype(np.float64)
           @ oracle_mod.e4m3_to_f32(w8).astype(np.float64).T
           ) * float(np.float32(a) * np.float32(s)) + bf16_value(bias)
    # one bf16 rounding (2^-9 relative) plus fp32 accumulation slack
    assert np.all(np.abs(y - ref) <= np.abs(ref) * 2.0 ** -8 + 1e-4 *
                  np.abs(ref).max())
    sub = oracle_mod.fp8_gemm(x8, w8, a, s, bias, rows=[3, 0, 32])
    full = oracle_mod.fp8_gemm(x8, w8, a, s, bias)
    assert np.array_equal(sub, full[[3, 0, 32]])


def test_gemm_packed_equals_siblings(oracle_mod):
    rng = np.random.default_rng(26)
    ws = [_rand_bf(rng, (n, 64), 0.02) for n in (32, 8, 8)]
    p = oracle_mod.pack_weights_fp8(ws)
    x8 = oracle_mod.f32_to_e4m3(rng.standard_normal((7, 64)) * 40)
    full = oracle_mod.fp8_gemm(x8, p["w8"], 0.02, p["w_scale"])
    lo = 0
    for w in ws:
        n = w.shape[0]
        part = oracle_mod.fp8_gemm(x8, p["w8"][lo:lo + n], 0.02, p["w_scale"])
        assert np.array_equal(part, full[:, lo:lo + n])
        lo += n


# ---------------------------------------------------------------- rope ----

def test_rope_table_library_values(oracle_mod):
    M, hd, P = 40, 64, 816
    t = oracle_mod.rope_table(M, hd, P)
    assert t.shape == (M, hd)
    pos = np.arange(P, P + M, dtype=np.float64)[:, None]
    ang = pos * 10000.0 ** (-np.arange(0, hd, 2, dtype=np.float64) / hd)
    cosv, sinv = bf16_value(t[:, 0::2]), bf16_value(t[:, 1::2])
    # within half a bf16 step of numpy's fp64 cos/sin
    assert np.all(np.abs(cosv - np.cos(ang)) <= np.abs(np.cos(ang)) * 2 ** -8
                  + 1e-30)
    assert np.all(np.abs(sinv - np.sin(ang)) <= np.abs(np.sin(ang)) * 2 ** -8
                  + 1e-30)
    t0 = oracle_mod.rope_table(2, 8, 0)
    assert np.all(t0[0, 0::2] == 0x3F80) and np.all(t0[0, 1::2] == 0)


def _split(oracle_mod, qkv, rope, B, M, hq, hkv, hd, P, T, fill=0x7FC1):
    kc = np.full((B, T, hkv, hd), fill, np.uint16)
    vc = np.full((B, T, hkv, hd), fill, np.uint16)
    return oracle_mod.split_rope_kvcache(qkv, rope, B, M, hq, hkv, hd, P,
                                         kc, vc)


def test_split_position_zero_identity_and_v_copy(oracle_mod):
    rng = np.random.default_rng(27)
    B, M, hq, hkv, hd, P, T = 2, 3, 2, 1, 8, 0, 5
    N = (hq + 2 * hkv) * hd
    qkv = _rand_bf(rng, (B * M, N))
    rope = oracle_mod.rope_table(M, hd, P)
    q, kc, vc = _split(oracle_mod, qkv, rope, B, M, hq, hkv, hd, P, T)
    for b in range(B):
        row = qkv[b * M]                           # s = 0: position 0
        assert np.array_equal(q[b, 0].ravel(), row[:hq * hd])
        assert np.array_equal(kc[b, 0, 0], row[hq * hd:(hq + 1) * hd])
        for s in range(M):
            assert np.array_equal(vc[b, s, 0], qkv[b * M + s, (hq + 1) * hd:])
    # rows P+M.. untouched (sentinel survives)
    assert np.all(kc[:, M:] == 0x7FC1) and np.all(vc[:, M:] == 0x7FC1)


def test_split_keeps_norms_and_relative_positions(oracle_mod):
    rng = np.random.default_rng(28)
    hq, hkv, hd = 1, 1, 64
    N = (hq + 2 * hkv) * hd
    M, P, T = 12, 100, 112
    base = rng.standard_normal(N)
    qkv = _bf(np.tile(base, (M, 1)))               # same q, k at every row
    rope = oracle_mod.rope_table(M, hd, P)
    q, kc, _ = _split(oracle_mod, qkv, rope, 1, M, hq, hkv, hd, P, T)
    qv, kv = bf16_value(q[0, :, 0]), bf16_value(kc[0, P:, 0])
    x = bf16_value(qkv[0, :hd]).reshape(-1, 2)
    for s in range(M):
        pair = qv[s].reshape(-1, 2)
        assert np.allclose((pair ** 2).sum(1), (x ** 2).sum(1), rtol=2e-2,
                           atol=1e-3)
    # score between query at s and key at s+d depends on d only
    d = 3
    scores = [qv[s] @ kv[s + d] for s in range(M - d)]
    scale = np.linalg.norm(qv[0]) * np.linalg.norm(kv[0])
    assert max(scores) - min(scores) <= 2e-2 * scale


def test_interleave_maps_rotate_half_to_adjacent_pairs(oracle_mod):
    """Attention scores of the host's rotate-half RoPE equal those of the
    adjacent-pair RoPE on the interleaved q/k (the bind-time equivalence)."""
    rng = np.random.default_rng(29)
    hd, M, P = 64, 6, 7
    q = rng.standard_normal((M, hd))
    k = rng.standard_normal((M, hd))
    pos = np.arange(P, P + M, dtype=np.float64)[:, None]
    inv = 10000.0 ** (-np.arange(0, hd, 2, dtype=np.float64) / hd)
    cos = np.cos(pos * inv)
    sin = np.sin(pos * inv)

    def rotate_half(x):                        # host convention, fp64
        c, s = np.concatenate([cos, cos], 1), np.concatenate([sin, sin], 1)
        h = hd // 2
        rot = np.concatenate([-x[:, h:], x[:, :h]], 1)
        return x * c + rot * s
    host = rotate_half(q) @ rotate_half(k).T
    perm = np.empty(hd, int)                   # interleave: kperm gather
    perm[0::2], perm[1::2] = np.arange(hd // 2), np.arange(hd // 2, hd)
    qkv = _bf(np.concatenate([q[:, perm], k[:, perm], k[:, perm]], 1))
    rope = oracle_mod.rope_table(M, hd, P)
    qo, kc, _ = _split(oracle_mod, qkv, rope, 1, M, 1, 1, hd, P, P + M)
    ours = bf16_value(qo[0, :, 0]) @ bf16_value(kc[0, P:, 0]).T
    assert np.allclose(ours, host, atol=3e-2 * np.abs(host).max())


def test_prefix_copy_gather(oracle_mod):
    rng = np.random.default_rng(30)
    B, hkv, Ts, hd, P, T = 1, 2, 10, 8, 6, 9
    pk, pv = _rand_bf(rng, (B, hkv, Ts, hd)), _rand_bf(rng, (B, hkv, Ts, hd))
    kc0 = np.full((B, T, hkv, hd), 0x7FC1, np.uint16)
    kc, vc = oracle_mod.prefix_copy(pk, pv, P, kc0, kc0, interleave=True)
    perm = [0, 4, 1, 5, 2, 6, 3, 7]
    for p in range(P):
        for h in range(hkv):
            assert np.array_equal(kc[0, p, h], pk[0, h, p, perm])
            assert np.array_equal(vc[0, p, h], pv[0, h, p])
    assert np.all(kc[:, P:] == 0x7FC1) and np.all(vc[:, P:] == 0x7FC1)
    kc2, _ = oracle_mod.prefix_copy(pk, pv, P, kc0, kc0, interleave=False)
    assert np.array_equal(kc2[0, :P, 1], pk[0, 1, :P])


# --------------------------------------------------------------- geglu ----

def test_geglu_against_library_and_closed_forms(oracle_mod):
    rng = np.random.default_rng(31)
    M, H = 4, 256
    g = rng.standard_normal((M, H)) * 3
    u = rng.standard_normal((M, H))
    gu = _bf(np.concatenate([g, u], 1))
    hid8, amax = oracle_mod.geglu_quant(gu, 1.0 / 8)    # no saturation
    gf, uf = bf16_value(gu[:, :H]), bf16_value(gu[:, H:])
    lib = torch.nn.functional.gelu(torch.from_numpy(gf).double(),
                                   approximate="tanh").numpy() * uf
    assert abs(amax - np.abs(lib).max()) <= 1e-5 * np.abs(lib).max()
    # every code is the nearest (or a tie-neighbour) of the library value
    assert np.abs(lib).max() < 448 / 8
    dq = oracle_mod.e4m3_to_f32(hid8) / 8
    step = np.maximum(np.abs(lib) * 2 ** -3, 2 ** -9 / 8)
    assert np.all(np.abs(dq - lib) <= step * 0.5 * (1 + 1e-3) + 1e-7)
    # zero gate gives zero, and gelu(x) - gelu(-x) = x (odd-part identity)
    z, _ = oracle_mod.geglu_quant(_bf(np.concatenate(
        [np.zeros((1, H)), np.ones((1, H))], 1)), 1.0)
    assert not (z & 0x7F).any()
    x = np.linspace(-4, 4, 64)
    xb = bf16_value(_bf(x))
    pos = []
    neg = []
    for v in xb:
        pos.append(oracle_mod.geglu_quant(_bf([[v, 1.0]]), 1.0)[1])
        neg.append(oracle_mod.geglu_quant(_bf([[-v, 1.0]]), 1.0)[1])
    # amax gives |gelu|; recover signed values from the sign of x
    gp = np.where(xb >= 0, pos, -np.array(pos))
    gn = np.where(-xb >= 0, neg, -np.array(neg))
    assert np.allclose(gp - gn, xb, atol=1e-5)
    # within the tanh form's known distance of the exact erf GELU
    erf_gelu = 0.5 * xb * (1 + np.vectorize(math.erf)(xb / math.sqrt(2)))
    assert np.all(np.abs(gp - erf_gelu) < 1e-3)

"""GPU parity of every kernel against the CPU oracle, through the C ABI.

Each test draws seeded inputs, runs the oracle and the CUDA path on the same
bytes and applies the stated bar (see tests/parity.py).  Output buffers and
caches are pre-filled with a NaN sentinel so stray writes are caught.
"""

import numpy as np
import pytest

import oracle
from fp8_transformer_block_b200 import synth
from fp8_transformer_block_b200.synth import bf16_bits, normal_bf16
from parity import assert_codes, assert_rms, bf16_ulps, gate_up_block_order
from chain_cases import SENTINEL, calibrate_adarms, calibrate_dit

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def rt():
    import torch
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"
    from fp8_transformer_block_b200 import build
    build.build()
    from fp8_transformer_block_b200 import frt, runtime
    return frt, runtime, torch


def _sync(torch):
    torch.cuda.synchronize()


# ------------------------------------------------------------ bounded wait --

def test_bounded_wait_reports_timeout(rt):
    frt, runtime, torch = rt
    rc = frt.frt_selftest_bounded_wait(20000)
    assert rc == frt.FRT_ETIMEOUT
    assert frt.frt_device_status(True) == frt.FRT_OK
    x = torch.ones(4, device="cuda")
    assert float(x.sum()) == 4.0            # the context is still usable


# ---------------------------------------------------------------- producer --

def _gpu_adarms(rt, inp, act_scale, eps=1e-6, weight=None, amax=False):
    frt, runtime, torch = rt
    res = runtime.bf16_dev(inp["res"])
    delta = runtime.bf16_dev(inp["delta"])
    gate = runtime.bf16_dev(inp["prev_gate"])
    style = runtime.bf16_dev(inp["style"])
    rows, D = inp["res"].shape
    x8 = runtime.empty_u8(rows, D)
    gate_out = runtime.empty_bf16(rows, D)
    sc = runtime.scale_dev(act_scale)
    am = torch.zeros(1, dtype=torch.float32, device="cuda") if amax else None
    w = None if weight is None else runtime.bf16_dev(weight)
    frt.frt_ada_norm_quant_fp8(
        frt.FRT_NORM_ADARMS, rows, D, eps, res, delta, gate,
        0 if inp["prev_gate"].shape[0] == 1 else D, w, style,
        0 if inp["style"].shape[0] == 1 else 3 * D, None, None, 0, None, 0, 0,
        sc, x8, gate_out, am)
    _sync(torch)
    return {"res": runtime.bf16_host(res), "x8": runtime.u8_host(x8),
            "gate_out": runtime.bf16_host(gate_out),
            "amax": None if am is None else float(am.item())}


@pytest.mark.parametrize("rows,D,outliers,per_row", [
    (64, 512, False, False),      # tiny AdaRMS layer
    (50, 2048, True, False),      # VLA action expert, 1 % outlier rows x20
    (37, 776, False, True),       # ragged: D = 97 chunks, per-row style/gate
    (5, 16384, False, False),     # widest D
    (3, 8, False, False),         # narrowest D
    (1024, 2048, True, True),     # gate/up MLP producer site
    (4096, 512, False, True),     # many narrow rows: register groups, not the staged ring
    (700, 512, False, False),     # narrow rows, staged ring
])
def test_producer_adarms_parity(rt, rows, D, outliers, per_row):
    inp = synth.adarms_inputs(rows, D, 4242 + D, outliers=outliers)
    if per_row:
        rng = np.random.default_rng(D)
        inp["prev_gate"] = normal_bf16(rng, (rows, D))
        inp["style"] = normal_bf16(rng, (rows, 3 * D), 0.5)
    ref1 = oracle.ada_rms_norm_quant(inp["res"], inp["delta"],
                                     inp["prev_gate"], inp["style"], 1.0)
    a = ref1["amax"] / 448.0
    ref = oracle.ada_rms_norm_quant(inp["res"], inp["delta"],
                                    inp["prev_gate"], inp["style"], a)
    got = _gpu_adarms(rt, inp, a, amax=True)
    assert np.array_equal(got["res"], ref["res"]), "residual update"
    assert np.array_equal(got["gate_out"], ref["gate_out"]), "gate_out"
    assert_codes(got["x8"], ref["x8"], what="x8")
    assert abs(got["amax"] - ref1["amax"]) <= 1e-5 * ref1["amax"]


@pytest.mark.parametrize("rows,D,chunks,sidx,cidx", [
    (256, 3072, 6, 0, 1),         # video-DiT attention site
    (33, 1000, 6, 3, 4),          # ragged, FFN-site chunks
    (4096, 1000, 6, 3, 4),        # many narrow rows (register groups)
    (2, 16384, 6, 0, 1),
])
def test_producer_layernorm_parity(rt, rows, D, chunks, sidx, cidx):
    frt, runtime, torch = rt
    inp = synth.dit_inputs(rows, D, 777 + D, chunks)
    a = oracle.ada_layer_norm_quant_table(inp["x"], inp["temb"], inp["table"],
                                          sidx, cidx, 1.0)["amax"] / 448.0
    ref = oracle.ada_layer_norm_quant_table(inp["x"], inp["temb"],
                                            inp["table"], sidx, cidx, a)
    x8 = runtime.empty_u8(rows, D)
    am = torch.zeros(1, dtype=torch.float32, device="cuda")
    frt.frt_ada_norm_quant_fp8(
        frt.FRT_NORM_LAYERNORM_TABLE, rows, D, 1e-6, None, None, None, 0,
        None, None, 0, runtime.bf16_dev(inp["x"]),
        runtime.bf16_dev(inp["temb"]), chunks, runtime.f32_dev(inp["table"]),
        sidx, cidx, runtime.scale_dev(a), x8, None, am)
    _sync(torch)
    assert_codes(runtime.u8_host(x8), ref["x8"], what="x8")
    assert abs(float(am.item()) - a * 448.0) <= 1e-5 * a * 448.0


def test_producer_layernorm_full_dit(rt):
    frt, runtime, torch = rt
    w = synth.WORKLOADS["video_dit"]
    inp = synth.dit_inputs(w.rows, w.D, w.seed)
    a = calibrate_dit(w, inp["table"])
    ref = oracle.ada_layer_norm_quant_table(inp["x"], inp["temb"],
                                            inp["table"], 0, 1, a)
    x8 = runtime.empty_u8(w.rows, w.D)
    frt.frt_ada_norm_quant_fp8(
        frt.FRT_NORM_LAYERNORM_TABLE, w.rows, w.D, w.eps, None, None, None,
        0, None, None, 0, runtime.bf16_dev(inp["x"]),
        runtime.bf16_dev(inp["temb"]), 6, runtime.f32_dev(inp["table"]), 0,
        1, runtime.scale_dev(a), x8, None, None)
    _sync(torch)
    assert_codes(runtime.u8_host(x8), ref["x8"], what="video-DiT x8")


# -------------------------------------------------------------------- pack --

@pytest.mark.parametrize("case", ["qk_interleave", "bias_concat",
                                  "gate_up_blocks"])
def test_pack_bit_exact(rt, case):
    frt, runtime, torch = rt
    if case == "qk_interleave":
        ws, bs = synth.qkv_weights(8, 1, 64, 512, 11)
        layout, hd = frt.FRT_PACK_QK_INTERLEAVE, 64
    elif case == "bias_concat":
        ws, bs = synth.qkv_weights(4, 4, 128, 1024, 12, bias=True)
        bs[1] = None
        layout, hd = frt.FRT_PACK_CONCAT, 0
    else:
        mw = synth.mlp_weights(512, 2048, 13)
        ws, bs = [mw["gate"], mw["up"]], None
        layout, hd = frt.FRT_PACK_GATE_UP_BLOCKS, 0
    if case == "gate_up_blocks":
        # the pages' concatenation, permuted into the library's block order
        ref = oracle.pack_weights_fp8(ws, bs)
        order = gate_up_block_order(ws[0].shape[0])
        ref = dict(ref, w8=ref["w8"][order], bias=ref["bias"][order])
    else:
        ref = oracle.pack_weights_fp8(ws, bs, layout=layout, hd=hd)
    pk = runtime.pack(ws, bs, layout=layout, hd=hd)
    _sync(torch)
    assert float(pk.w_scale.item()) == ref["w_scale"]
    assert np.array_equal(runtime.u8_host(pk.w8), ref["w8"])
    if pk.bias is not None:
        assert np.array_equal(runtime.bf16_host(pk.bias), ref["bias"])


# -------------------------------------------------------------------- GEMM --

def _x8_codes(rows, K, seed):
    inp = synth.adarms_inputs(rows, K, seed)
    return oracle.ada_rms_norm_quant(inp["res"], inp["delta"],
                                     inp["prev_gate"], inp["style"],
                                     0.02)["x8"]


GEMM_CASES = [
    # M, N, K, bias   (M <= 128 runs the swapped schedule, K split in clusters)
    (1, 640, 512, False),
    (16, 640, 512, False),
    (50, 2560, 2048, False),
    (64, 640, 512, True),
    (100, 672, 528, True),         # ragged N tile, K tail (528 = 4*128 + 16)
    (128, 2560, 2048, False),
    (129, 640, 512, False),        # first normal-orientation size
    (300, 672, 528, True),         # ragged everywhere, BN = 128
    (1000, 2560, 2048, True),      # 128-wide tiles (256-wide would underfill)
    (256, 9216, 3072, True),       # video-DiT projection width
    (1200, 4096, 1024, False),     # 256-wide tiles, persistent
    (64, 2048, 16384, False),      # long K: K split in a 4-CTA cluster
    (100, 1024, 4096, True),       # 128-token tiles: 4-CTA clusters, ragged
    (32, 1024, 4096, True),        # clusters at the split cap (4)
    (50, 1056, 2048, True),        # 4-CTA clusters, ragged last weight tile
    (16, 512, 1024, False),        # 2-CTA clusters, 8 weight tiles
    (200, 256, 16384, True),       # 128-row tiles, K split via workspace
    # CTA pairs (256-row tiles over two SMs)
    (300, 4096, 528, True),        # BN = 128; the odd CTA of the last pair
                                   # holds rows past M only; K tail
    (1100, 4096, 1024, True),      # BN = 256, ragged last 256-row tile
    (2048, 4096, 512, False),      # several tiles per pair, K < ring depth
    (1024, 640, 512, False),       # 160-wide pair tiles (one wave where 128 needs two)
    (1100, 640, 1024, True),       # 160-wide, ragged 256-row tile
    (2048, 1536, 512, True),       # 192-wide pair tiles
    (1024, 1024, 4096, True),      # K in halves over two 128-wide pairs (clusters of 4)
    (1024, 2048, 4096, False),     # K in halves over two 256-wide pairs
    (1100, 1024, 4096, True),      # K in halves, ragged 256-row tile
    (1100, 2304, 1024, True),      # BN = 256 pairs (N not a multiple of 512)
    (2560, 8192, 256, True),       # several tiles per pair, K < ring depth
    (1300, 5120, 1152, False),     # ragged last 256-row tile, K tail of 1 block
    (3000, 2048, 2048, True),      # ragged rows, K beyond the ring
]


# wide CTA pairs (256 x 512 tiles, two 256-column MMAs per K-step): long K
# only, so the oracle checks seeded sampled rows (rows are independent)
WIDE_CASES = [
    # M, N, K, bias, epilogue
    (2048, 4096, 8192, True, "bf16"),      # one tile per pair
    (4000, 4096, 8192, False, "bf16"),     # two tiles on most pairs, ragged rows
    (2048, 8192, 8192, False, "geglu"),    # gate/up blocks, two per wide tile
    (2048, 4096, 8192, True, "gelu"),
]


@pytest.mark.parametrize("M,N,K,bias,epi", WIDE_CASES)
def test_gemm_wide_parity_sampled(rt, M, N, K, bias, epi):
    frt, runtime, torch = rt
    code = {"bf16": frt.FRT_EPI_BF16, "geglu": frt.FRT_EPI_GEGLU_E4M3,
            "gelu": frt.FRT_EPI_GELU_E4M3}[epi]
    plan = frt.frt_gemm_plan_info(M, N, K, code)
    assert plan["pair"] == 1 and plan["tile_cols"] == 512, plan
    rng = np.random.default_rng(M + N + K)
    x8 = _x8_codes(M, K, 300 + M)
    w = normal_bf16(rng, (N, K), 0.02)
    b = normal_bf16(rng, (N,), 0.5) if bias else None
    a = 0.0173
    sel = np.unique(np.concatenate([[0, M - 1], rng.choice(M, 62, replace=False)]))
    if epi == "geglu":
        H = N // 2
        ws = [w[:H], w[H:]]
        cat = oracle.pack_weights_fp8(ws)
        pk = runtime.pack(ws, layout=frt.FRT_PACK_GATE_UP_BLOCKS)
        gu = oracle.fp8_gemm(x8, cat["w8"], a, cat["w_scale"], rows=sel)
        s_out = max(oracle.geglu_quant(gu, 1.0)[1] / 448.0, 1e-8)
        ref, _ = oracle.geglu_quant(gu, s_out)
        out = torch.full((M, H), 0x7F, dtype=torch.uint8, device="cuda")
        ldo = H
    else:
        pk_ref = oracle.pack_weights_fp8([w], [b])
        pk = runtime.pack([w], [b] if bias else None)
        y = oracle.fp8_gemm(x8, pk_ref["w8"], a, pk_ref["w_scale"],
                            pk_ref["bias"] if bias else None, rows=sel)
        if epi == "gelu":
            s_out = max(oracle.gelu_quant(y, 1.0)[1] / 448.0, 1e-8)
            ref, _ = oracle.gelu_quant(y, s_out)
            out = torch.full((M, N), 0x7F, dtype=torch.uint8, device="cuda")
        else:
            s_out, ref = None, y
            out = torch.full((M, N), float("nan"), dtype=torch.bfloat16, device="cuda")
        ldo = N
    wsb = frt.frt_gemm_workspace_size(M, N, K, code)
    frt.frt_packed_fp8_gemm(M, N, K, runtime.u8_dev(x8), pk.w8, runtime.scale_dev(a),
                            pk.w_scale, pk.bias if bias else None, code, out, ldo,
                            None if s_out is None else runtime.scale_dev(s_out),
                            runtime.workspace(wsb), wsb)
    _sync(torch)
    assert frt.frt_device_status(True) == frt.FRT_OK
    if epi == "bf16":
        got = runtime.bf16_host(out)[sel]
        assert_rms(got, ref, what=f"wide GEMM {M}x{N}x{K}")
        assert np.percentile(bf16_ulps(got, ref), 99.9) <= 1
        # rows past the sample are written too (no NaN left anywhere)
        assert not torch.isnan(out).any().item()
    else:
        assert_codes(runtime.u8_host(out)[sel], ref, what=f"wide {epi} {M}x{N}x{K}")
        assert not (out == 0x7F).all(dim=1).any().item()


@pytest.mark.parametrize("M,N,K,bias", GEMM_CASES)
def test_gemm_parity(rt, M, N, K, bias):
    frt, runtime, torch = rt
    rng = np.random.default_rng(M * 7 + N)
    x8 = _x8_codes(M, K, 100 + M)
    w = normal_bf16(rng, (N, K), 0.02)
    b = normal_bf16(rng, (N,), 0.5) if bias else None
    pk_ref = oracle.pack_weights_fp8([w], [b])
    a = 0.0173
    ref = oracle.fp8_gemm(x8, pk_ref["w8"], a, pk_ref["w_scale"],
                          pk_ref["bias"] if bias else None)
    w8 = runtime.u8_dev(pk_ref["w8"])
    ws = runtime.scale_dev(pk_ref["w_scale"])
    bd = runtime.bf16_dev(pk_ref["bias"]) if bias else None
    out = torch.full((M, N), float("nan"), dtype=torch.bfloat16,
                     device="cuda")
    wsb = frt.frt_gemm_workspace_size(M, N, K)
    wsp = runtime.workspace(wsb)
    for _ in range(2):   # a second call reuses the zeroed split counters
        frt.frt_packed_fp8_gemm(M, N, K, runtime.u8_dev(x8), w8,
                                runtime.scale_dev(a), ws, bd, frt.FRT_EPI_BF16,
                                out, N, None, wsp, wsb)
    _sync(torch)
    got = runtime.bf16_host(out)
    assert_rms(got, ref, what=f"GEMM {M}x{N}x{K}")
    assert np.percentile(bf16_ulps(got, ref), 99.9) <= 1
    if wsp is not None:
        assert not wsp[:256].any().item(), "split counters left non-zero"


def test_gemm_zero_input_gives_bias(rt):
    frt, runtime, torch = rt
    for M in (7, 200):
        N, K = 640, 512
        rng = np.random.default_rng(M)
        b = normal_bf16(rng, (N,), 1.0)
        w8 = runtime.u8_dev(rng.integers(0, 0x7E, (N, K), dtype=np.uint8))
        out = runtime.empty_bf16(M, N)
        wsb = frt.frt_gemm_workspace_size(M, N, K)
        frt.frt_packed_fp8_gemm(M, N, K, runtime.empty_u8(M, K).zero_(), w8,
                                runtime.scale_dev(0.5), runtime.scale_dev(0.01),
                                runtime.bf16_dev(b), frt.FRT_EPI_BF16, out, N,
                                None, runtime.workspace(wsb), wsb)
        _sync(torch)
        assert np.array_equal(runtime.bf16_host(out), np.tile(b, (M, 1)))


# ------------------------------------------------- rope table / split / KV --

@pytest.mark.parametrize("M,hd,P", [(50, 256, 816), (4096, 128, 0), (64, 64, 0)])
def test_rope_table(rt, M, hd, P):
    frt, runtime, torch = rt
    t = runtime.empty_bf16(M, hd)
    frt.frt_build_rope_table(M, hd, P, 10000.0, t)
    _sync(torch)
    ref = oracle.rope_table(M, hd, P)
    got = runtime.bf16_host(t)
    d = bf16_ulps(got, ref)
    assert d.max() <= 1 and (d == 0).mean() >= 0.9999


def _caches(runtime, torch, B, T, hkv, hd):
    kc = torch.full((B, T, hkv, hd), 0, dtype=torch.int16, device="cuda")
    kc.fill_(np.int16(np.uint16(SENTINEL).view(np.int16)).item())
    vc = kc.clone()
    return kc.view(torch.bfloat16), vc.view(torch.bfloat16)


@pytest.mark.parametrize("B,M,hq,hkv,hd,P,T,bias,prefix", [
    (1, 64, 8, 1, 64, 0, 64, False, False),      # tiny AdaRMS
    (1, 50, 8, 1, 256, 816, 1024, False, True),  # VLA action expert
    (2, 200, 4, 4, 128, 0, 256, True, False),    # DiT-shaped, normal tiles
    (1, 1, 8, 1, 64, 816, 817, False, True),     # one token
])
def test_split_rope_fused_and_unfused(rt, B, M, hq, hkv, hd, P, T, bias,
                                      prefix):
    frt, runtime, torch = rt
    K = 512
    N = (hq + 2 * hkv) * hd
    rows = B * M
    x8 = _x8_codes(rows, K, 500 + M)
    ws_, bs_ = synth.qkv_weights(hq, hkv, hd, K, 900 + M, bias=bias)
    pk_ref = oracle.pack_weights_fp8(ws_, bs_, layout=1, hd=hd)
    pk = runtime.pack(ws_, bs_, layout=frt.FRT_PACK_QK_INTERLEAVE, hd=hd)
    a = 0.02
    sc = runtime.scale_dev(a)
    x8d = runtime.u8_dev(x8)
    rope = runtime.empty_bf16(M, hd)
    frt.frt_build_rope_table(M, hd, P, 10000.0, rope)
    pkh = pvh = None
    if prefix:
        pkh, pvh = synth.prefix_cache(B, hkv, P + 8, hd, 31)
    wsb = frt.frt_gemm_workspace_size(rows, N, K)
    wsp = runtime.workspace(wsb)
    # unfused: GEMM -> qkv -> split (+ prefix in the same launch)
    qkv = runtime.empty_bf16(rows, N)
    frt.frt_packed_fp8_gemm(rows, N, K, x8d, pk.w8, sc, pk.w_scale, pk.bias,
                            frt.FRT_EPI_BF16, qkv, N, None, wsp, wsb)
    q1 = runtime.empty_bf16(B, M, hq, hd)
    k1, v1 = _caches(runtime, torch, B, T, hkv, hd)
    pkd = runtime.bf16_dev(pkh) if prefix else None
    pvd = runtime.bf16_dev(pvh) if prefix else None
    frt.frt_split_rope_kvcache(B, M, hq, hkv, hd, P, T, qkv, rope, q1, k1, v1,
                               pkd, pvd, P + 8 if prefix else 0, 1)
    # fused: GEMM epilogue does split + RoPE + KV; prefix copied separately
    q2 = runtime.empty_bf16(B, M, hq, hd)
    k2, v2 = _caches(runtime, torch, B, T, hkv, hd)
    if prefix:
        frt.frt_prefix_copy_kv(B, hkv, hd, P, T, P + 8, pkd, pvd, 1, k2, v2)
    frt.frt_packed_fp8_gemm_rope_kvcache(B, M, K, hq, hkv, hd, P, T, x8d,
                                         pk.w8, sc, pk.w_scale, pk.bias, rope,
                                         q2, k2, v2, wsp, wsb)
    _sync(torch)
    h = runtime.bf16_host
    assert np.array_equal(h(q1), h(q2)), "fused q differs from unfused"
    assert np.array_equal(h(k1), h(k2)), "fused k cache differs"
    assert np.array_equal(h(v1), h(v2)), "fused v cache differs"
    # unfused split vs the oracle split on the GPU's own qkv: bit-exact
    kc0 = np.full((B, T, hkv, hd), SENTINEL, np.uint16)
    if prefix:
        kc0a, vc0a = oracle.prefix_copy(pkh, pvh, P, kc0, kc0, True)
    else:
        kc0a, vc0a = kc0, kc0
    qo, ko, vo = oracle.split_rope_kvcache(h(qkv), oracle.rope_table(M, hd, P),
                                           B, M, hq, hkv, hd, P, kc0a, vc0a)
    assert np.array_equal(h(q1), qo)
    assert np.array_equal(h(k1), ko)
    assert np.array_equal(h(v1), vo)
    # GEMM vs oracle GEMM on the same codes, then end to end
    ref_qkv = oracle.fp8_gemm(x8, pk_ref["w8"], a, pk_ref["w_scale"],
                              pk_ref["bias"] if bias else None)
    assert_rms(h(qkv), ref_qkv, what="qkv")
    qr, kr, vr = oracle.split_rope_kvcache(ref_qkv, oracle.rope_table(M, hd, P),
                                           B, M, hq, hkv, hd, P, kc0a, vc0a)
    assert_rms(h(q2), qr, what="q_out")
    sl = slice(P, P + M)
    assert_rms(h(k2)[:, sl], kr[:, sl], what="k rows")
    assert np.array_equal(h(k2)[:, P + M:], kr[:, P + M:])   # untouched
    assert np.array_equal(h(k2)[:, :P], kr[:, :P])           # prefix


# ------------------------------------------------------------------- GEGLU --

def test_geglu_standalone_parity(rt):
    frt, runtime, torch = rt
    rng = np.random.default_rng(5)
    M, H = 96, 1024
    gu = bf16_bits(np.concatenate([rng.standard_normal((M, H)) * 2,
                                   rng.standard_normal((M, H))], 1))
    _, amax = oracle.geglu_quant(gu, 1.0)
    a = amax / 448.0
    ref, _ = oracle.geglu_quant(gu, a)
    hid = runtime.empty_u8(M, H)
    am = torch.zeros(1, dtype=torch.float32, device="cuda")
    frt.frt_geglu_quant_fp8(M, H, runtime.bf16_dev(gu), 2 * H,
                            runtime.scale_dev(a), hid, am)
    _sync(torch)
    assert_codes(runtime.u8_host(hid), ref, what="hid8")
    assert abs(float(am.item()) - amax) <= 1e-5 * amax


@pytest.mark.parametrize("M,H", [(64, 1024), (300, 1024), (1100, 1024), (2048, 8192)])
def test_geglu_fused_epilogue(rt, M, H):
    """The GEMM's GEGLU + requant epilogue against the oracle, two ways:
    (a) element-wise on its own input: the oracle's GEGLU applied to the
    bf16 gate/up values the same GEMM writes with the plain epilogue (the
    fused epilogue rounds its accumulators to those bf16 values first);
    (b) end to end: the oracle's GEMM and GEGLU from the same x8 codes.
    Both at the code bar (99.99 % identical, the rest one step)."""
    frt, runtime, torch = rt
    D = 512
    mw = synth.mlp_weights(D, H, 21)
    x8h = _x8_codes(M, D, 77)
    x8 = runtime.u8_dev(x8h)
    sc = runtime.scale_dev(0.02)
    blk = runtime.pack([mw["gate"], mw["up"]],
                       layout=frt.FRT_PACK_GATE_UP_BLOCKS)
    order = gate_up_block_order(H)
    # the plain epilogue on the same block-ordered weights: gu in block order
    gu = runtime.empty_bf16(M, 2 * H)
    wsb = frt.frt_gemm_workspace_size(M, 2 * H, D)
    frt.frt_packed_fp8_gemm(M, 2 * H, D, x8, blk.w8, sc, blk.w_scale, None,
                            frt.FRT_EPI_BF16, gu, 2 * H, None,
                            runtime.workspace(wsb), wsb)
    out_scale = runtime.scale_dev(0.01)
    h2 = torch.full((M, H), 0x7F, dtype=torch.uint8, device="cuda")
    wsb2 = frt.frt_gemm_workspace_size(M, 2 * H, D, frt.FRT_EPI_GEGLU_E4M3)
    frt.frt_packed_fp8_gemm(M, 2 * H, D, x8, blk.w8, sc, blk.w_scale, None,
                            frt.FRT_EPI_GEGLU_E4M3, h2, H, out_scale,
                            runtime.workspace(wsb2), wsb2)
    _sync(torch)
    assert frt.frt_device_status(True) == frt.FRT_OK
    fused = runtime.u8_host(h2)
    # back to the pages' [gate | up] column order
    gu_cat = np.empty((M, 2 * H), np.uint16)
    gu_cat[:, order] = runtime.bf16_host(gu)
    ref_a, _ = oracle.geglu_quant(gu_cat, 0.01)
    assert_codes(fused, ref_a, what="fused GEGLU vs oracle on the GEMM's gu")
    cat = oracle.pack_weights_fp8([mw["gate"], mw["up"]])
    assert np.array_equal(runtime.u8_host(blk.w8), cat["w8"][order])
    gu_ref = oracle.fp8_gemm(x8h, cat["w8"], 0.02, cat["w_scale"])
    assert_rms(gu_cat, gu_ref, what="gate/up projection")
    ref_b, _ = oracle.geglu_quant(gu_ref, 0.01)
    assert_codes(fused, ref_b, what="fused GEGLU vs oracle end to end")
    # the standalone kernel on the same gu: the same codes as the oracle's
    h1 = runtime.empty_u8(M, H)
    gu_dev = runtime.bf16_dev(gu_cat)
    frt.frt_geglu_quant_fp8(M, H, gu_dev, 2 * H, out_scale, h1)
    _sync(torch)
    assert_codes(runtime.u8_host(h1), ref_a, what="standalone GEGLU vs oracle")


@pytest.mark.parametrize("scale_div", [8.0, 64.0])
def test_gelu_requant_saturates(rt, scale_div):
    """Output scales at amax / 448 / scale_div: a large share of the GEGLU and
    GELU values lie beyond +-448 and must saturate to codes 0x7E / 0xFE (the
    pages' clamp-then-round quantizer), never the NaN codes 0x7F / 0xFF; the
    rest, down to e4m3's subnormal codes, at the code bar against the
    oracle.  The standalone kernels and the fused GEGLU epilogue (the same
    device GELU) on the same values."""
    frt, runtime, torch = rt
    rng = np.random.default_rng(41)
    M, H = 128, 1024
    gu = bf16_bits(np.concatenate([rng.standard_normal((M, H)) * 3,
                                   rng.standard_normal((M, H)) * 2], 1))

    def gelu64(x):  # values well past the clamp, where no rounding can matter
        return 0.5 * x * (1.0 + np.tanh(np.sqrt(2.0 / np.pi) * (x + 0.044715 * x ** 3)))

    def f64(bits):
        return (bits.astype(np.uint32) << 16).view(np.float32).astype(np.float64)

    _, amax = oracle.geglu_quant(gu, 1.0)
    a = amax / 448.0 / scale_div
    ref, _ = oracle.geglu_quant(gu, a)
    sat = np.abs(gelu64(f64(gu[:, :H])) * f64(gu[:, H:])) / a > 460.0
    assert sat.mean() > 0.005, sat.mean()      # the case is exercised
    assert ((ref[sat] & 0x7F) == 0x7E).all()
    hid = runtime.empty_u8(M, H)
    frt.frt_geglu_quant_fp8(M, H, runtime.bf16_dev(gu), 2 * H, runtime.scale_dev(a), hid)
    _sync(torch)
    got = runtime.u8_host(hid)
    assert not ((got & 0x7F) == 0x7F).any(), "GEGLU produced NaN codes"
    assert np.array_equal(got[sat], ref[sat])
    assert_codes(got, ref, what="saturating GEGLU vs oracle")
    # GELU alone on the gate half
    u = np.ascontiguousarray(gu[:, :H])
    _, amax_u = oracle.gelu_quant(u, 1.0)
    au = amax_u / 448.0 / scale_div
    ref_u, _ = oracle.gelu_quant(u, au)
    sat_u = np.abs(gelu64(f64(u))) / au > 460.0
    assert sat_u.mean() > 0.005, sat_u.mean()
    assert ((ref_u[sat_u] & 0x7F) == 0x7E).all()
    hu = runtime.empty_u8(M, H)
    frt.frt_gelu_quant_fp8(M, H, runtime.bf16_dev(u), H, runtime.scale_dev(au), hu)
    _sync(torch)
    got_u = runtime.u8_host(hu)
    assert not ((got_u & 0x7F) == 0x7F).any(), "GELU produced NaN codes"
    assert np.array_equal(got_u[sat_u], ref_u[sat_u])
    assert_codes(got_u, ref_u, what="saturating GELU vs oracle")
    # the fused GEGLU epilogue at the same kind of scale, against the
    # oracle's GEGLU on the bf16 gate/up values the same GEMM writes
    D = 512
    mw = synth.mlp_weights(D, H, 23)
    x8 = runtime.u8_dev(_x8_codes(M, D, 79))
    sc = runtime.scale_dev(0.02)
    blk = runtime.pack([mw["gate"], mw["up"]], layout=frt.FRT_PACK_GATE_UP_BLOCKS)
    order = gate_up_block_order(H)
    g2 = runtime.empty_bf16(M, 2 * H)
    wsb = frt.frt_gemm_workspace_size(M, 2 * H, D)
    frt.frt_packed_fp8_gemm(M, 2 * H, D, x8, blk.w8, sc, blk.w_scale, None,
                            frt.FRT_EPI_BF16, g2, 2 * H, None, runtime.workspace(wsb), wsb)
    _sync(torch)
    gu_cat = np.empty((M, 2 * H), np.uint16)
    gu_cat[:, order] = runtime.bf16_host(g2)
    _, amax2 = oracle.geglu_quant(gu_cat, 1.0)
    a2 = amax2 / 448.0 / scale_div
    ref2, _ = oracle.geglu_quant(gu_cat, a2)
    h2 = torch.full((M, H), 0x7F, dtype=torch.uint8, device="cuda")
    wsb2 = frt.frt_gemm_workspace_size(M, 2 * H, D, frt.FRT_EPI_GEGLU_E4M3)
    frt.frt_packed_fp8_gemm(M, 2 * H, D, x8, blk.w8, sc, blk.w_scale, None,
                            frt.FRT_EPI_GEGLU_E4M3, h2, H, runtime.scale_dev(a2),
                            runtime.workspace(wsb2), wsb2)
    _sync(torch)
    assert frt.frt_device_status(True) == frt.FRT_OK
    fused = runtime.u8_host(h2)
    sat2 = np.abs(gelu64(f64(gu_cat[:, :H])) * f64(gu_cat[:, H:])) / a2 > 460.0
    assert sat2.mean() > 0.005, sat2.mean()
    assert not ((fused & 0x7F) == 0x7F).any(), "fused GEGLU produced NaN codes"
    assert np.array_equal(fused[sat2], ref2[sat2])
    assert_codes(fused, ref2, what="saturating fused GEGLU vs oracle")


def test_device_gelu_error_bound(rt):
    """The device GELU (tanh from the exponential) against an fp64
    evaluation of the tanh-form GELU: within 5e-7 * max(1, |x|) plus four
    fp32 ulps of the value over [-12, 12] and at small magnitudes; exactly x
    once tanh saturates (x >= 10) and signed zero at zero."""
    frt, runtime, torch = rt
    x = np.concatenate([np.linspace(-12.0, 12.0, 240001),
                        [0.0, -0.0, 1e-30, -1e-30, 1e-5, -1e-5, 3e-3, -3e-3]]).astype(np.float32)
    xd = torch.from_numpy(x).cuda()
    yd = torch.empty_like(xd)
    frt.frt_selftest_gelu(xd, yd, x.size)
    _sync(torch)
    y = yd.cpu().numpy().astype(np.float64)
    xx = x.astype(np.float64)
    ref = 0.5 * xx * (1.0 + np.tanh(np.sqrt(2.0 / np.pi) * (xx + 0.044715 * xx ** 3)))
    ulp = np.spacing(np.abs(ref).astype(np.float32)).astype(np.float64)
    err = np.abs(y - ref)
    bound = 5e-7 * np.maximum(1.0, np.abs(xx)) + 4 * ulp
    assert (err <= bound).all(), f"worst {(err / bound).max():.2f} of the bound at x={xx[np.argmax(err / bound)]}"
    big = xx >= 10
    assert np.array_equal(y[big], xx[big])
    assert y[x.size - 8] == 0.0 and np.signbit(yd.cpu().numpy()[x.size - 7])


# ------------------------------------------------------------ peak probes --
def test_peak_probes_run_and_are_plausible(rt):
    frt, runtime, torch = rt
    sms = torch.cuda.get_device_properties(0).multi_processor_count
    ev = [torch.cuda.Event(enable_timing=True) for _ in range(2)]
    for operands in (frt.FRT_PEAK_OPERANDS_GAUSSIAN, frt.FRT_PEAK_OPERANDS_LOW_TOGGLE):
        frt.frt_peak_fp8_mma(sms, 200, operands)
        ev[0].record()
        frt.frt_peak_fp8_mma(sms, 2000, operands)
        ev[1].record()
        _sync(torch)
        assert frt.frt_device_status(True) == frt.FRT_OK
        tflops = 2.0 * 128 * 256 * 128 * 2000 * sms / (ev[0].elapsed_time(ev[1]) * 1e-3) / 1e12
        assert 300 < tflops < 6000, tflops   # dense e4m3 on one B200: a few PFLOP/s
    n = 64 << 20
    src = torch.randint(0, 255, (n,), dtype=torch.uint8, device="cuda")
    dst = torch.zeros_like(src)
    frt.frt_peak_copy(src, dst, n)
    _sync(torch)
    assert torch.equal(src, dst)


# -------------------------------------------------------- GELU epilogue --
@pytest.mark.parametrize("M,D,H", [(64, 512, 1024), (300, 512, 1024), (1100, 512, 2048),
                                   (200, 4096, 256), (2048, 512, 8192)])
def test_gelu_fused_epilogue(rt, M, D, H):
    """The GEMM's GELU + requant epilogue (the DiT FFN's up projection)
    against the unfused GEMM -> GELU kernel, and that against the oracle."""
    frt, runtime, torch = rt
    rng = np.random.default_rng(M + H)
    w = normal_bf16(rng, (H, D), 0.02)
    b = normal_bf16(rng, (H,), 0.01)
    x8 = runtime.u8_dev(_x8_codes(M, D, 91))
    sc = runtime.scale_dev(0.02)
    pk = runtime.pack([w], [b])
    u = runtime.empty_bf16(M, H)
    wsb = frt.frt_gemm_workspace_size(M, H, D)
    frt.frt_packed_fp8_gemm(M, H, D, x8, pk.w8, sc, pk.w_scale, pk.bias, frt.FRT_EPI_BF16,
                            u, H, None, runtime.workspace(wsb), wsb)
    am = torch.zeros(1, dtype=torch.float32, device="cuda")
    h1 = runtime.empty_u8(M, H)
    frt.frt_gelu_quant_fp8(M, H, u, H, runtime.scale_dev(1.0), h1, am)
    torch.cuda.synchronize()
    s_h = float(am.item()) / 448.0
    out_scale = runtime.scale_dev(s_h)
    frt.frt_gelu_quant_fp8(M, H, u, H, out_scale, h1)
    h2 = torch.full((M, H), 0x7F, dtype=torch.uint8, device="cuda")
    wsb2 = frt.frt_gemm_workspace_size(M, H, D, frt.FRT_EPI_GELU_E4M3)
    frt.frt_packed_fp8_gemm(M, H, D, x8, pk.w8, sc, pk.w_scale, pk.bias,
                            frt.FRT_EPI_GELU_E4M3, h2, H, out_scale,
                            runtime.workspace(wsb2), wsb2)
    _sync(torch)
    assert frt.frt_device_status(True) == frt.FRT_OK
    u_host = runtime.bf16_host(u)
    ref_u = oracle.fp8_gemm(runtime.u8_host(x8), runtime.u8_host(pk.w8), 0.02,
                            float(pk.w_scale.item()), runtime.bf16_host(pk.bias))
    assert_rms(u_host, ref_u, what="up projection")
    assert_codes(runtime.u8_host(h2), runtime.u8_host(h1), match=0.9999,
                 what="fused vs unfused GELU")
    ref, amax = oracle.gelu_quant(u_host, s_h)
    assert_codes(runtime.u8_host(h1), ref, what="unfused GELU vs oracle")
    assert abs(float(am.item()) - amax) <= 1e-6 * amax

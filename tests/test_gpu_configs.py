"""Parity at the configurations' own sizes, step by step.

* The gate/up MLP (1024 tokens, D 2048, gate and up 16384 each, the fused
  GEGLU requant, the 2048 x 16384 down projection on its K-halves schedule)
  at full size on the GPU, with the oracle on seeded sampled rows (rows are
  independent through the producer, both GEMMs and the GEGLU).
* The 18-layer AdaRMS stack over its whole row-count sweep (1 .. 4096
  tokens behind the 816-token prefix).

Each step is held to the single-step bar in isolation: the oracle's step is
fed the GPU's own inputs to that step (the residual, delta and gate the GPU
carried into a layer; the x8 codes the GPU's producer wrote; the hidden
codes its GEGLU wrote).  Beside it, the oracle runs the whole sequence from
the seeded inputs on its own, held to the norm-wise end-to-end bar (a
one-step code flip earlier in the sequence legitimately moves what follows).

Code bar: every code within one e4m3 step, >= 99.99 % identical, counted
over all codes a test compares (a single layer of the 1-token stack holds
only 512 codes, too few for a per-layer percentage).
"""

import numpy as np
import pytest

import oracle
from fp8_transformer_block_b200 import synth
from fp8_transformer_block_b200.synth import bf16_value
from parity import CODE_MATCH, assert_codes, assert_rms, e4m3_step_distance
from chain_cases import calibrate_adarms

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def rt():
    import torch
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"
    from fp8_transformer_block_b200 import build
    build.build()
    from fp8_transformer_block_b200 import frt, runtime
    return frt, runtime, torch


def _rel_l2(got_bf16, ref_bf16):
    g = bf16_value(got_bf16).astype(np.float64)
    r = bf16_value(ref_bf16).astype(np.float64)
    return float(np.linalg.norm(g - r) / np.linalg.norm(r))


def _rowwise_split(qkv_rows, positions, table, hq, hkv, hd):
    """The oracle's split + RoPE on single rows: row i at table row
    positions[i] (the table already holds the absolute positions P + s).
    Returns q [n, hq, hd], k [n, hkv, hd], v [n, hkv, hd]."""
    q, k, v = [], [], []
    for i, s in enumerate(positions):
        one = np.zeros((1, 1, hkv, hd), np.uint16)
        qo, ko, vo = oracle.split_rope_kvcache(qkv_rows[i:i + 1], table[s:s + 1], 1, 1,
                                               hq, hkv, hd, 0, one, one)
        q.append(qo[0, 0])
        k.append(ko[0, 0])
        v.append(vo[0, 0])
    return np.stack(q), np.stack(k), np.stack(v)


class CodeTally:
    """Codes compared across a test: none more than one step apart, and the
    identical fraction over all of them at the code bar."""

    def __init__(self):
        self.same = 0
        self.total = 0

    def add(self, got, ref, what):
        d = e4m3_step_distance(got, ref)
        bad = int((d > 1).sum())
        assert bad == 0, f"{what}: {bad} codes more than one step apart"
        self.same += int((d == 0).sum())
        self.total += d.size

    def check(self, what):
        frac = self.same / max(self.total, 1)
        assert frac >= CODE_MATCH, f"{what}: {frac:.6f} identical (< {CODE_MATCH})"
        return frac


# ------------------------------------------------------------ gate/up MLP --

def test_gateup_mlp_full_size_sampled(rt):
    """1024 x 2048 -> gate/up 32768 (fused GEGLU requant) -> 2048 x 16384."""
    frt, runtime, torch = rt
    w = synth.WORKLOADS["gateup_mlp"]
    M, D, H = w.M, w.D, w.H
    mw = synth.mlp_weights(D, H, w.seed)
    inp = synth.adarms_inputs(M, D, w.seed)
    cat = oracle.pack_weights_fp8([mw["gate"], mw["up"]])
    dnp = oracle.pack_weights_fp8([mw["down"]])
    # static scales: the oracle's calibration on the seed + 500 batch
    a_gu = calibrate_adarms(w)
    cal = synth.adarms_inputs(w.cal_rows, D, w.seed + synth.CAL_OFFSET)
    prc = oracle.ada_rms_norm_quant(cal["res"], cal["delta"], cal["prev_gate"],
                                    cal["style"], a_gu, eps=w.eps)
    guc = oracle.fp8_gemm(prc["x8"], cat["w8"], a_gu, cat["w_scale"])
    a_dn = max(oracle.geglu_quant(guc, 1.0)[1] / 448.0, 1e-8)
    del guc

    blk = runtime.pack([mw["gate"], mw["up"]], layout=frt.FRT_PACK_GATE_UP_BLOCKS)
    dn = runtime.pack([mw["down"]])
    plan_gu = frt.frt_gemm_plan_info(M, 2 * H, D, frt.FRT_EPI_GEGLU_E4M3)
    plan_dn = frt.frt_gemm_plan_info(M, D, H)
    assert plan_gu["pair"] == 1 and plan_dn["split2"] == 1   # the schedules of the config
    res = runtime.bf16_dev(inp["res"])
    x8 = runtime.empty_u8(M, D)
    g_out = runtime.empty_bf16(M, D)
    hid = torch.full((M, H), 0x7F, dtype=torch.uint8, device="cuda")
    out = runtime.empty_bf16(M, D)
    s_gu, s_dn = runtime.scale_dev(a_gu), runtime.scale_dev(a_dn)
    frt.frt_ada_norm_quant_fp8(frt.FRT_NORM_ADARMS, M, D, w.eps, res,
                               runtime.bf16_dev(inp["delta"]),
                               runtime.bf16_dev(inp["prev_gate"]), 0, None,
                               runtime.bf16_dev(inp["style"]), 0, None, None,
                               0, None, 0, 0, s_gu, x8, g_out, None)
    ws1 = frt.frt_gemm_workspace_size(M, 2 * H, D, frt.FRT_EPI_GEGLU_E4M3)
    frt.frt_packed_fp8_gemm(M, 2 * H, D, x8, blk.w8, s_gu, blk.w_scale, None,
                            frt.FRT_EPI_GEGLU_E4M3, hid, H, s_dn,
                            runtime.workspace(ws1), ws1)
    ws2 = frt.frt_gemm_workspace_size(M, D, H)
    frt.frt_packed_fp8_gemm(M, D, H, hid, dn.w8, s_dn, dn.w_scale, None,
                            frt.FRT_EPI_BF16, out, D, None,
                            runtime.workspace(ws2), ws2)
    torch.cuda.synchronize()
    assert frt.frt_device_status(True) == frt.FRT_OK

    # producer: every row
    pr = oracle.ada_rms_norm_quant(inp["res"], inp["delta"], inp["prev_gate"],
                                   inp["style"], a_gu, eps=w.eps)
    gx8 = runtime.u8_host(x8)
    assert np.array_equal(runtime.bf16_host(res), pr["res"])
    assert np.array_equal(runtime.bf16_host(g_out), pr["gate_out"])
    assert_codes(gx8, pr["x8"], what="producer x8")
    # sampled rows through both GEMMs (first, last, the rest seeded)
    rng = np.random.default_rng(4)
    sel = np.unique(np.concatenate([[0, M - 1], rng.choice(M, 62, replace=False)]))
    ghid = runtime.u8_host(hid)[sel]
    gout = runtime.bf16_host(out)[sel]
    # isolated: the oracle's gate/up GEMM + GEGLU on the GPU's x8, the
    # oracle's down GEMM on the GPU's hidden codes
    gu_i = oracle.fp8_gemm(gx8[sel], cat["w8"], a_gu, cat["w_scale"])
    hid_i, _ = oracle.geglu_quant(gu_i, a_dn)
    assert_codes(ghid, hid_i, what="GEGLU hid8 (GPU x8)")
    out_i = oracle.fp8_gemm(ghid, dnp["w8"], a_dn, dnp["w_scale"])
    assert_rms(gout, out_i, what="down projection (GPU hid8)")
    # end to end from the oracle's own codes
    gu_e = oracle.fp8_gemm(pr["x8"][sel], cat["w8"], a_gu, cat["w_scale"])
    hid_e, _ = oracle.geglu_quant(gu_e, a_dn)
    out_e = oracle.fp8_gemm(hid_e, dnp["w8"], a_dn, dnp["w_scale"])
    d = e4m3_step_distance(ghid, hid_e)
    rel = _rel_l2(gout, out_e)
    print(f"gate/up MLP full size: hid8 identical {(d == 0).mean():.6f} (isolated "
          f"{(e4m3_step_distance(ghid, hid_i) == 0).mean():.6f}), out rel-L2 {rel:.3e}")
    assert (d == 0).mean() >= 0.99 and rel <= 2e-2


# -------------------------------------------------------- 18-layer stack --

def _oracle_stack_rows(w, lays, packs, table, res, positions, scales=None):
    """The oracle's stack on independent rows (row i at position
    positions[i]): per layer the producer, the packed q/k/v GEMM and the
    split + RoPE; layer l + 1 takes layer l's q rows as delta and its gate
    rows as gate (layer 0: zeros).  scales None calibrates each layer's
    static scale on these rows (amax / 448).  Returns per layer
    (res, x8, q, k, v) and the scales."""
    n, D = res.shape
    delta = np.zeros((n, D), np.uint16)
    gate = np.zeros((1, D), np.uint16)
    out, used = [], []
    for l in range(w.layers):
        st = lays[l]["style"]
        if scales is None:
            a = oracle.ada_rms_norm_quant(res, delta, gate, st, 1.0, eps=w.eps)["amax"] / 448.0
        else:
            a = scales[l]
        used.append(a)
        pr = oracle.ada_rms_norm_quant(res, delta, gate, st, a, eps=w.eps)
        qkv = oracle.fp8_gemm(pr["x8"], packs[l]["w8"], a, packs[l]["w_scale"])
        q, k, v = _rowwise_split(qkv, positions, table, w.hq, w.hkv, w.hd)
        out.append((pr["res"], pr["x8"], q, k, v))
        res, delta, gate = pr["res"], q.reshape(n, D), pr["gate_out"]
    return out, used


@pytest.mark.parametrize("M", [1, 16, 50, 256, 1024, 4096])
def test_stack_sweep_per_layer_isolated(rt, M):
    """The 18-layer stack through frt_chain_layer at one row count of the
    sweep.  Per layer: the residual update and the gate bit-exact, the x8
    codes at the code bar, q/k/v at the GEMM/RoPE bar, all against the
    oracle's layer fed the GPU's own layer inputs; the prefix rows
    bit-exact.  Up to 256 tokens every row is compared; above, a seeded
    sample (first and last rows included).  End to end, the oracle's own
    stack on the same rows: q norm-wise within 2e-2 at every layer."""
    frt, runtime, torch = rt
    w = synth.WORKLOADS["adarms_stack18"].with_M(M)
    L, D, rows, P = w.layers, w.D, w.rows, w.P
    inp = synth.adarms_inputs(rows, D, w.seed)
    lays = [synth.stack_layer_inputs(w, l) for l in range(L)]
    packs = [oracle.pack_weights_fp8(li["w"], layout=1, hd=w.hd) for li in lays]
    table = oracle.rope_table(M, w.hd, P)
    # static scales calibrated by the oracle's stack on the seed + 500 batch
    n_cal = min(rows, 256)
    cal = synth.adarms_inputs(n_cal, D, w.seed + synth.CAL_OFFSET)
    _, scales = _oracle_stack_rows(w, lays, packs, table, cal["res"], np.arange(n_cal))
    if rows <= 256:
        sel = np.arange(rows)
    else:
        rng = np.random.default_rng(M)
        sel = np.unique(np.concatenate([[0, rows - 1], rng.choice(rows, 94, replace=False)]))
    e2e, _ = _oracle_stack_rows(w, lays, packs, table, inp["res"][sel], sel, scales)

    res = runtime.bf16_dev(inp["res"])
    zero = torch.zeros(rows, D, dtype=torch.bfloat16, device="cuda")
    x8 = runtime.empty_u8(rows, D)
    q = [runtime.empty_bf16(1, M, w.hq, w.hd) for _ in range(2)]
    g = [runtime.empty_bf16(rows, D) for _ in range(2)]
    rope = runtime.empty_bf16(M, w.hd)
    frt.frt_build_rope_table(M, w.hd, P, w.theta, rope)
    keep, descs = [], []
    for l in range(L):
        pk = runtime.pack(lays[l]["w"], layout=frt.FRT_PACK_QK_INTERLEAVE, hd=w.hd)
        kc = torch.zeros(1, w.T, w.hkv, w.hd, dtype=torch.bfloat16, device="cuda")
        vc = torch.zeros_like(kc)
        pkd = runtime.bf16_dev(lays[l]["prefix_k"])
        pvd = runtime.bf16_dev(lays[l]["prefix_v"])
        sc = runtime.scale_dev(scales[l])
        st = runtime.bf16_dev(lays[l]["style"])
        keep += [pk, pkd, pvd, sc, st]
        d = runtime.chain_desc(
            B=1, M=M, D=D, hq=w.hq, hkv=w.hkv, hd=w.hd, P=P, T=w.T,
            eps=w.eps, norm_mode=frt.FRT_NORM_ADARMS,
            flags=frt.FRT_CHAIN_FUSED_ROPE, res=res,
            delta=zero if l == 0 else q[(l - 1) % 2],
            prev_gate=zero if l == 0 else g[(l - 1) % 2],
            gate_row_stride=0 if l == 0 else D, style=st, gate_out=g[l % 2],
            act_scale=sc, x8=x8, w8=pk.w8, w_scale=pk.w_scale, rope=rope,
            q_out=q[l % 2], k_cache=kc, v_cache=vc, prefix_k=pkd,
            prefix_v=pvd, prefix_T_src=P, prefix_interleave=1)
        descs.append((d, kc, vc))
    wsb = frt.frt_chain_workspace_size(descs[0][0])
    wsp = runtime.workspace(wsb)
    h = runtime.bf16_host
    tally_iso, tally_e2e = CodeTally(), CodeTally()
    stats = []
    res_in = inp["res"][sel]
    delta_in = np.zeros((len(sel), D), np.uint16)
    gate_in = np.zeros((1, D), np.uint16)
    for l, (d, kc, vc) in enumerate(descs):
        d.workspace, d.workspace_bytes = frt.ptr(wsp), wsb
        frt.frt_chain_layer(d)
        torch.cuda.synchronize()
        assert frt.frt_device_status(True) == frt.FRT_OK
        g_res = h(res)[sel]
        g_x8 = runtime.u8_host(x8)[sel]
        g_gate = h(g[l % 2])[sel]
        g_q = h(q[l % 2]).reshape(rows, w.hq, w.hd)[sel]
        kch, vch = h(kc), h(vc)
        g_k = kch[0, P + sel]
        g_v = vch[0, P + sel]
        # isolated: the oracle's layer on this layer's GPU inputs
        pr = oracle.ada_rms_norm_quant(res_in, delta_in, gate_in, lays[l]["style"],
                                       scales[l], eps=w.eps)
        assert np.array_equal(g_res, pr["res"]), f"layer {l}: residual"
        assert np.array_equal(g_gate, pr["gate_out"]), f"layer {l}: gate"
        tally_iso.add(g_x8, pr["x8"], f"layer {l} x8")
        qkv_i = oracle.fp8_gemm(g_x8, packs[l]["w8"], scales[l], packs[l]["w_scale"])
        qi, ki, vi = _rowwise_split(qkv_i, sel, table, w.hq, w.hkv, w.hd)
        assert_rms(g_q, qi, what=f"layer {l} q_out (GPU x8)")
        assert_rms(g_k, ki, what=f"layer {l} k rows (GPU x8)")
        assert_rms(g_v, vi, what=f"layer {l} v rows (GPU x8)")
        # the prefix rows are copies: bit-exact
        zc = np.zeros((1, w.T, w.hkv, w.hd), np.uint16)
        kp, vp = oracle.prefix_copy(lays[l]["prefix_k"], lays[l]["prefix_v"], P, zc, zc, True)
        assert np.array_equal(kch[:, :P], kp[:, :P]), f"layer {l}: k prefix"
        assert np.array_equal(vch[:, :P], vp[:, :P]), f"layer {l}: v prefix"
        # end to end against the oracle's own stack on the same rows
        e_res, e_x8, e_q, _, _ = e2e[l]
        tally_e2e.same += int((g_x8 == e_x8).sum())
        tally_e2e.total += g_x8.size
        rel = _rel_l2(g_q, e_q)
        stats.append((l, round(rel, 6)))
        assert rel <= 2e-2, f"layer {l}: q_out end to end rel-L2 {rel}"
        # the next layer's GPU inputs
        res_in, delta_in, gate_in = g_res, g_q.reshape(len(sel), D), g_gate
    frac = tally_iso.check(f"stack M={M}: x8 over all layers")
    e2e_frac = tally_e2e.same / tally_e2e.total
    print(f"stack M={M}: isolated x8 identical {frac:.7f} over {tally_iso.total} codes; "
          f"end-to-end x8 identical {e2e_frac:.5f}; q rel-L2 per layer {stats}")
    assert e2e_frac >= 0.97

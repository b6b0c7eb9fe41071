"""The AdaRMS layer loop except attention, on the GPU through the C ABI
(fp8_transformer_block_b200.stack: frt_chain_layer, the output projection's
static quantize + GEMM on the attention stand-in, frt_ffn_layer, and the
final frt_ada_rms_tail), against the oracle's composition of the same steps
(impls/adarms_stack/fp8_chain.py `_make_run`)."""

import numpy as np
import pytest

import oracle
from fp8_transformer_block_b200 import synth
from fp8_transformer_block_b200.synth import bf16_value
from parity import assert_rms

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def rt():
    import torch
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"
    from fp8_transformer_block_b200 import build
    build.build()
    from fp8_transformer_block_b200 import frt, runtime, stack
    return frt, runtime, stack, torch


def _rel_l2(got, ref):
    g = bf16_value(got).astype(np.float64)
    r = bf16_value(ref).astype(np.float64)
    return float(np.linalg.norm(g - r) / np.linalg.norm(r))


def _oracle_layers(lays, w):
    return [{"qkv": oracle.pack_weights_fp8(li["w"], layout=1, hd=w.hd),
             "o": oracle.pack_weights_fp8([li["o"]]),
             "gu": oracle.pack_weights_fp8([li["mlp"]["gate"], li["mlp"]["up"]]),
             "dn": oracle.pack_weights_fp8([li["mlp"]["down"]]),
             "styles": li["styles"], "prefix_k": li["prefix_k"],
             "prefix_v": li["prefix_v"]} for li in lays]


def test_layer_stack_matches_oracle(rt):
    frt, runtime, stack, torch = rt
    w = synth.WORKLOADS["adarms_layer18"].with_M(16)
    L = 3
    lays = [synth.full_layer_inputs(w, l) for l in range(L)]
    fin = synth.final_norm_rows(w)
    x = synth.adarms_inputs(w.rows, w.D, w.seed)["res"]
    cal = synth.adarms_inputs(w.rows, w.D, w.seed + synth.CAL_OFFSET)["res"]
    dims = {"B": w.B, "M": w.M, "D": w.D, "hq": w.hq, "hkv": w.hkv, "hd": w.hd,
            "P": w.P, "T": w.T, "H": w.H, "theta": w.theta}
    ol = _oracle_layers(lays, w)
    _, _, scales = oracle.adarms_layer_stack(cal, ol, fin, dims)
    ref, recs, _ = oracle.adarms_layer_stack(x, ol, fin, dims, scales=scales)

    st = stack.AdaRmsLayerStack(w, lays, fin, scales=scales)
    st.load(x)
    st.step()
    torch.cuda.synchronize()
    assert frt.frt_device_status(True) == frt.FRT_OK
    h = runtime.bf16_host
    for l in range(L):
        kc, vc = h(st.lay[l]["kc"]), h(st.lay[l]["vc"])
        # the prefix rows are copies at every depth
        assert np.array_equal(kc[:, :w.P], recs[l]["k"][:, :w.P]), f"layer {l} prefix k"
        assert np.array_equal(vc[:, :w.P], recs[l]["v"][:, :w.P]), f"layer {l} prefix v"
        if l == 0:
            assert_rms(kc[:, w.P:], recs[l]["k"][:, w.P:], what="layer 0 k rows")
            assert_rms(vc[:, w.P:], recs[l]["v"][:, w.P:], what="layer 0 v rows")
        else:
            # later layers carry the earlier layers' rounding in the residual
            assert _rel_l2(kc[:, w.P:], recs[l]["k"][:, w.P:]) <= 2e-2, f"layer {l} k"
            assert _rel_l2(vc[:, w.P:], recs[l]["v"][:, w.P:]) <= 2e-2, f"layer {l} v"
    assert _rel_l2(h(st.res), recs[-1]["res"]) <= 1e-2, "residual after the stack"
    e = _rel_l2(h(st.out), ref)
    print(f"whole-layer stack, {L} layers: final output rel-L2 {e:.3e}")
    assert e <= 2e-2, "final tail output"


def test_layer_stack_gpu_calibration_runs(rt):
    frt, runtime, stack, torch = rt
    w = synth.WORKLOADS["adarms_layer18"]
    lays = [synth.full_layer_inputs(w, l) for l in range(2)]
    cal = synth.adarms_inputs(w.rows, w.D, w.seed + synth.CAL_OFFSET)["res"]
    st = stack.AdaRmsLayerStack(w, lays, synth.final_norm_rows(w), x=cal)
    for sc in st.scales:
        assert all(0 < v < 1e3 for v in sc.values()), sc
    st.load(synth.adarms_inputs(w.rows, w.D, w.seed)["res"])
    st.step()
    torch.cuda.synchronize()
    assert frt.frt_device_status(True) == frt.FRT_OK
    out = bf16_value(runtime.bf16_host(st.out))
    assert np.all(np.isfinite(out)) and 0.5 < float(np.sqrt((out ** 2).mean())) < 50


def test_layer_stack_modulation_on_device(rt):
    """Every step computes all norms' (scale, shift, gate) rows from the
    conditioning row on the device (`_style_stack`): the projection's rows
    against the oracle's, then the whole stack against the oracle's
    composition fed the oracle's rows, for two conditioning rows in turn."""
    frt, runtime, stack, torch = rt
    w = synth.WORKLOADS["adarms_layer18"].with_M(16)
    L = 3
    lays = [synth.full_layer_inputs(w, l) for l in range(L)]
    mod = synth.modulation_inputs(2, w.D, 2 * L + 1, w.seed)
    x = synth.adarms_inputs(w.rows, w.D, w.seed)["res"]
    dims = {"B": w.B, "M": w.M, "D": w.D, "hq": w.hq, "hkv": w.hkv, "hd": w.hd,
            "P": w.P, "T": w.T, "H": w.H, "theta": w.theta}
    fin_col0 = 3 * w.D * 2 * L
    st = None
    for i in range(2):
        cond = mod["cond"][i:i + 1]
        style_ref, fin_ref = oracle.style_project(cond, mod["w"], mod["bias"], fin_col0=fin_col0)
        lays_i = [dict(li, styles=style_ref[0, 3 * w.D * 2 * l:3 * w.D * (2 * l + 2)]
                       .reshape(2, 3 * w.D)) for l, li in enumerate(lays)]
        ol = _oracle_layers(lays_i, w)
        fin = fin_ref.reshape(3, w.D)
        if st is None:
            _, _, scales = oracle.adarms_layer_stack(x, ol, fin, dims)
            st = stack.AdaRmsLayerStack(w, lays, None, scales=scales,
                                        modulation={"w": mod["w"], "bias": mod["bias"],
                                                    "cond": cond})
        else:
            st.set_cond(cond)
        ref, _, _ = oracle.adarms_layer_stack(x, ol, fin, dims, scales=scales)
        st.load(x)
        st.step()
        torch.cuda.synchronize()
        assert frt.frt_device_status(True) == frt.FRT_OK
        gs = runtime.bf16_host(st.styles)
        same = float((gs == style_ref).mean())
        assert same >= 0.999, f"cond {i}: style rows {same:.5f} identical"
        assert np.all(np.abs(bf16_value(gs) - bf16_value(style_ref))
                      <= 2.0 ** -7 * np.abs(bf16_value(style_ref)) + 1e-6), f"cond {i}: style"
        fg = st.fin.cpu().numpy().reshape(1, -1)
        assert np.allclose(fg, fin_ref, rtol=0, atol=1e-5), f"cond {i}: final rows"
        e = _rel_l2(runtime.bf16_host(st.out), ref)
        print(f"modulated stack, cond {i}: final output rel-L2 {e:.3e}")
        assert e <= 2e-2, f"cond {i}: final tail output"

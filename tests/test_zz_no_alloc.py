"""frt_packed_fp8_gemm_noalloc: the GEMM entry point for callers that cannot
allocate device memory (a plug-in whose host engine owns all device memory,
a real-time loop that must stay out of the CUDA allocator, code running
during stream capture).  It uses the library's static scratch instead of a
caller workspace, and runs the same schedule as frt_packed_fp8_gemm, so its
output must be bit-identical to the workspace entry's on every call.  This
file is collected last so that a run stopping at the first failure has
already run every other test.
"""

import numpy as np
import pytest

import oracle
from fp8_transformer_block_b200 import synth
from fp8_transformer_block_b200.synth import normal_bf16
from parity import assert_codes, assert_rms

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def rt():
    import torch
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"
    from fp8_transformer_block_b200 import build
    build.build()
    from fp8_transformer_block_b200 import frt, runtime
    return frt, runtime, torch


def _x8(M, K, seed):
    inp = synth.adarms_inputs(M, K, seed)
    return oracle.ada_rms_norm_quant(inp["res"], inp["delta"], inp["prev_gate"],
                                     inp["style"], 0.02)["x8"]


@pytest.mark.parametrize("M,N,K,bias", [
    (200, 256, 16384, True),    # splits K through the workspace (8 splits)
    (50, 2560, 2048, False),    # cluster schedule, no workspace needed
])
def test_noalloc_matches_workspace_entry(rt, M, N, K, bias):
    frt, runtime, torch = rt
    rng = np.random.default_rng(M + N)
    x8 = _x8(M, K, 9)
    w = normal_bf16(rng, (N, K), 0.02)
    b = normal_bf16(rng, (N,), 0.5) if bias else None
    pk = runtime.pack([w], [b] if bias else None)
    x8d = runtime.u8_dev(x8)
    sc = runtime.scale_dev(0.0173)
    need = frt.frt_gemm_workspace_size(M, N, K)
    assert (need > 0) == (M == 200)
    ref = runtime.empty_bf16(M, N)
    frt.frt_packed_fp8_gemm(M, N, K, x8d, pk.w8, sc, pk.w_scale, pk.bias,
                            frt.FRT_EPI_BF16, ref, N, None,
                            runtime.workspace(need), need)
    torch.cuda.synchronize()
    want = ref.clone()
    for call in range(2):   # the static scratch keeps the last call's state
        out = torch.full((M, N), float("nan"), dtype=torch.bfloat16,
                         device="cuda")
        frt.frt_packed_fp8_gemm_noalloc(M, N, K, x8d, pk.w8, sc, pk.w_scale,
                                        pk.bias, frt.FRT_EPI_BF16, out, N)
        torch.cuda.synchronize()
        assert frt.frt_device_status(True) == frt.FRT_OK
        # same plan, kernel and split order: bit for bit
        assert torch.equal(out.view(torch.int16), want.view(torch.int16)), \
            f"noalloc call {call} differs from the workspace entry"
    # and both against the oracle's GEMM on the same codes (the GEMM bar)
    ref_o = oracle.fp8_gemm(x8, runtime.u8_host(pk.w8), 0.0173,
                            float(pk.w_scale.item()),
                            runtime.bf16_host(pk.bias) if bias else None)
    assert_rms(runtime.bf16_host(out), ref_o, what="noalloc vs oracle")


def test_noalloc_geglu_through_the_scratch(rt):
    """A gated (GEGLU + e4m3) shape whose K split uses the static scratch:
    codes identical to the workspace entry's, and within the code bar of the
    oracle's GEGLU on the oracle's GEMM."""
    frt, runtime, torch = rt
    M, H, K = 128, 256, 8192
    plan = frt.frt_gemm_plan_info(M, 2 * H, K, frt.FRT_EPI_GEGLU_E4M3)
    assert plan["splits"] > 1 and plan["swap"] == 0 and plan["pair"] == 0
    need = frt.frt_gemm_workspace_size(M, 2 * H, K, frt.FRT_EPI_GEGLU_E4M3)
    assert 0 < need <= 8 << 20
    mw = synth.mlp_weights(K, H, 31)
    x8 = _x8(M, K, 33)
    x8d = runtime.u8_dev(x8)
    sc, os_ = runtime.scale_dev(0.02), runtime.scale_dev(0.004)
    blk = runtime.pack([mw["gate"], mw["up"]],
                       layout=frt.FRT_PACK_GATE_UP_BLOCKS)
    ref = runtime.empty_u8(M, H)
    frt.frt_packed_fp8_gemm(M, 2 * H, K, x8d, blk.w8, sc, blk.w_scale, None,
                            frt.FRT_EPI_GEGLU_E4M3, ref, H, os_,
                            runtime.workspace(need), need)
    torch.cuda.synchronize()
    want = ref.clone()
    for call in range(2):
        out = torch.full((M, H), 0x7F, dtype=torch.uint8, device="cuda")
        frt.frt_packed_fp8_gemm_noalloc(M, 2 * H, K, x8d, blk.w8, sc,
                                        blk.w_scale, None,
                                        frt.FRT_EPI_GEGLU_E4M3, out, H, os_)
        torch.cuda.synchronize()
        assert frt.frt_device_status(True) == frt.FRT_OK
        assert torch.equal(out, want), f"noalloc GEGLU call {call}"
    cat = oracle.pack_weights_fp8([mw["gate"], mw["up"]])
    gu = oracle.fp8_gemm(x8, cat["w8"], 0.02, cat["w_scale"])
    hid, _ = oracle.geglu_quant(gu, 0.004)
    assert_codes(runtime.u8_host(out), hid, what="noalloc GEGLU vs oracle")


def test_noalloc_rejects_shapes_beyond_its_scratch(rt):
    frt, runtime, torch = rt
    M, N, K = 1024, 256, 65536
    assert frt.frt_gemm_workspace_size(M, N, K) > 8 << 20
    rc = frt.raw_call("frt_packed_fp8_gemm_noalloc", M, N, K, 0x10000, 0x10000,
                      0x10000, 0x10000, None, 0, 0x10000, N, None, None)
    assert rc == frt.FRT_ERANGE
    assert "static scratch" in frt.last_error()

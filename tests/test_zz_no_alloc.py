"""frt_packed_fp8_gemm_noalloc: the GEMM entry point for callers that cannot
allocate device memory (a plug-in whose host engine owns all device memory,
a real-time loop that must stay out of the CUDA allocator, code running
during stream capture).  It uses the library's static scratch instead of a
caller workspace.  This file is collected last so that a run stopping at the
first failure has already run every other test.
"""

import numpy as np
import pytest

import oracle
from fp8_transformer_block_b200 import synth
from fp8_transformer_block_b200.synth import normal_bf16
from parity import assert_rms

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def rt():
    import torch
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"
    from fp8_transformer_block_b200 import build
    build.build()
    from fp8_transformer_block_b200 import frt, runtime
    return frt, runtime, torch


@pytest.mark.parametrize("M,N,K,bias", [
    (200, 256, 16384, True),    # splits K through the workspace (8 splits)
    (50, 2560, 2048, False),    # cluster schedule, no workspace needed
])
def test_noalloc_matches_workspace_entry(rt, M, N, K, bias):
    frt, runtime, torch = rt
    rng = np.random.default_rng(M + N)
    inp = synth.adarms_inputs(M, K, 9)
    x8 = oracle.ada_rms_norm_quant(inp["res"], inp["delta"], inp["prev_gate"],
                                   inp["style"], 0.02)["x8"]
    w = normal_bf16(rng, (N, K), 0.02)
    b = normal_bf16(rng, (N,), 0.5) if bias else None
    pk = runtime.pack([w], [b] if bias else None)
    x8d = runtime.u8_dev(x8)
    sc = runtime.scale_dev(0.0173)
    need = frt.frt_gemm_workspace_size(M, N, K)
    ref = runtime.empty_bf16(M, N)
    frt.frt_packed_fp8_gemm(M, N, K, x8d, pk.w8, sc, pk.w_scale, pk.bias,
                            frt.FRT_EPI_BF16, ref, N, None,
                            runtime.workspace(need), need)
    torch.cuda.synchronize()
    want = runtime.bf16_host(ref)
    for call in range(2):   # the static scratch keeps the last call's state
        out = torch.full((M, N), float("nan"), dtype=torch.bfloat16,
                         device="cuda")
        frt.frt_packed_fp8_gemm_noalloc(M, N, K, x8d, pk.w8, sc, pk.w_scale,
                                        pk.bias, frt.FRT_EPI_BF16, out, N)
        torch.cuda.synchronize()
        assert frt.frt_device_status(True) == frt.FRT_OK
        assert_rms(runtime.bf16_host(out), want,
                   what=f"noalloc call {call} vs workspace entry")


def test_noalloc_rejects_shapes_beyond_its_scratch(rt):
    frt, runtime, torch = rt
    M, N, K = 1024, 256, 65536
    assert frt.frt_gemm_workspace_size(M, N, K) > 8 << 20
    rc = frt.raw_call("frt_packed_fp8_gemm_noalloc", M, N, K, 0x10000, 0x10000,
                      0x10000, 0x10000, None, 0, 0x10000, N, None, None)
    assert rc == frt.FRT_ERANGE
    assert "static scratch" in frt.last_error()

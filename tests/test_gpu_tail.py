"""GPU parity of the AdaRMS layer's output side against the oracle: the
static quantize in front of the output projection and the stack's final
AdaRMS tail (impls/adarms_stack/fp8_chain.py `out_project` and the
"ad:tail" range of `_make_run`), through the C ABI."""

import numpy as np
import pytest

import oracle
from fp8_transformer_block_b200.synth import bf16_value, normal_bf16
from parity import assert_codes, bf16_ulps

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def rt():
    import torch
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"
    from fp8_transformer_block_b200 import build
    build.build()
    from fp8_transformer_block_b200 import frt, runtime
    return frt, runtime, torch


@pytest.mark.parametrize("rows,D,ld", [(1, 512, 512), (50, 2048, 2048), (1024, 512, 512),
                                       (300, 3072, 3200), (7, 8, 8)])
def test_quantize_static_parity(rt, rows, D, ld):
    frt, runtime, torch = rt
    rng = np.random.default_rng(rows * 31 + D)
    full = normal_bf16(rng, (rows, ld), 1.0)
    full[rng.random(rows) < 0.02] = normal_bf16(rng, (1, ld), 20.0)  # outlier rows
    x = full[:, :D]
    _, amax = oracle.quant_fp8_static(x, 1.0)
    scale = max(amax / 448.0, 1e-8)
    ref, _ = oracle.quant_fp8_static(x, scale)
    xd = runtime.bf16_dev(full)
    out = torch.full((rows, D), 0x7F, dtype=torch.uint8, device="cuda")
    am = torch.zeros(1, dtype=torch.float32, device="cuda")
    frt.frt_quantize_fp8_static(rows, D, xd, ld, runtime.scale_dev(scale), out, am)
    torch.cuda.synchronize()
    assert_codes(runtime.u8_host(out), ref, what="o_proj input codes")
    assert float(am.item()) == amax


@pytest.mark.parametrize("rows,D,per_row_gate", [(1, 512, False), (50, 2048, True),
                                                 (300, 3072, True), (64, 1024, False),
                                                 (129, 8192, True)])
def test_ada_rms_tail_parity(rt, rows, D, per_row_gate):
    frt, runtime, torch = rt
    rng = np.random.default_rng(rows + D)
    res = normal_bf16(rng, (rows, D), 1.0)
    delta = normal_bf16(rng, (rows, D), 0.5)
    gate = normal_bf16(rng, (rows if per_row_gate else 1, D), 0.3)
    fin = rng.normal(0.0, 0.1, size=(3, D)).astype(np.float32)
    ref = oracle.ada_rms_tail(res, delta, gate, fin, 1e-6)
    out = torch.full((rows, D), float("nan"), dtype=torch.bfloat16, device="cuda")
    frt.frt_ada_rms_tail(rows, D, 1e-6, runtime.bf16_dev(res), runtime.bf16_dev(delta),
                         runtime.bf16_dev(gate), D if per_row_gate else 0,
                         runtime.f32_dev(fin), D, out)
    torch.cuda.synchronize()
    got = runtime.bf16_host(out)
    # same fp32 operations; the row sum runs in another order, so the
    # statistic may differ by a few ulps: an output is then one bf16 step
    # off, or, where (1 + scale) * h / rms cancels against the shift, a few
    # steps of a value near zero (absolute error tiny against the row rms)
    u = bf16_ulps(got, ref)
    err = np.abs(bf16_value(got).astype(np.float64) - bf16_value(ref).astype(np.float64))
    rms = float(np.sqrt((bf16_value(ref).astype(np.float64) ** 2).mean()))
    assert bool(np.all((u <= 1) | (err <= 1e-4 * rms)))
    assert float((u == 0).mean()) >= 0.999

"""GPU parity of the modulation projection (impls/adarms_stack/fp8_chain.py
`_style_stack` and the binder's per-step bake) against the oracle, through
the C ABI.

Bar, derived from the arithmetic: both sides sum K fp32 products, in
different orders, so each fp32 result lies within (K + 2) * 2^-24 *
(sum_k |cond * w| + |bias|) of the exact value, and the two within twice
that of each other (the fp32 rows).  A bf16 row value then lies within half
a bf16 step of its own fp32 value: where the two sides' bf16 values differ,
the GPU's is within half a step plus twice the bound of the oracle's fp32
value.  Bit-identical bf16 for all but the few values that sit on a bf16
rounding boundary (>= 99.9 %)."""

import numpy as np
import pytest

import oracle
from fp8_transformer_block_b200 import synth
from fp8_transformer_block_b200.synth import bf16_bits, bf16_value

pytestmark = pytest.mark.gpu

U = 2.0 ** -24


@pytest.fixture(scope="module")
def rt():
    import torch
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"
    from fp8_transformer_block_b200 import build
    build.build()
    from fp8_transformer_block_b200 import frt, runtime
    return frt, runtime, torch


def _half_step(v32):
    """Half a bf16 step at each fp32 value."""
    ex = (np.asarray(v32, np.float32).view(np.uint32) >> 23) & 0xFF
    return np.ldexp(1.0, np.maximum(ex.astype(np.int64), 1) - 127 - 8)


def _check(style_gpu, fin_gpu, cond, w, b, fin_col0):
    """GPU rows against the oracle's on the same inputs (w: the weight rows
    of the compared columns, in order)."""
    K = cond.shape[1]
    style_ref, fin_ref = oracle.style_project(cond, w, b, fin_col0=0)
    c64, w64 = cond.astype(np.float64), bf16_value(w).astype(np.float64)
    scale = np.abs(c64) @ np.abs(w64).T
    if b is not None:
        scale += np.abs(b.astype(np.float64))
    bound = 2 * (K + 2) * U * scale
    if fin_gpu is not None:
        err = np.abs(fin_gpu.astype(np.float64)[:, :] - fin_ref[:, fin_col0:])
        assert np.all(err <= bound[:, fin_col0:]), f"fin: worst {float((err - bound[:, fin_col0:]).max()):.3e} past the bound"
    same = style_gpu == style_ref
    frac = float(same.mean())
    gv = bf16_value(style_gpu).astype(np.float64)
    off = np.abs(gv - fin_ref.astype(np.float64))
    lim = _half_step(fin_ref) + _half_step(gv.astype(np.float32)) + bound
    assert np.all(same | (off <= lim)), "style: a bf16 value past half a step plus the bound"
    assert frac >= 0.999, f"style: only {frac:.5f} bit-identical"
    return frac


def _inputs(rows, K, N, seed, bias=True):
    rng = np.random.Generator(np.random.PCG64(seed))
    cond = bf16_value(bf16_bits(rng.standard_normal((rows, K), dtype=np.float32)))
    w = bf16_bits(rng.standard_normal((N, K), dtype=np.float32) * np.float32(0.02))
    b = bf16_value(bf16_bits(rng.standard_normal(N, dtype=np.float32) * np.float32(0.01)))
    return cond, w, (b if bias else None)


def _launch(rt, cond, w, b, fin_col0, pad_cond=0, pad_w=0, pad_style=0, with_fin=True):
    frt, runtime, torch = rt
    rows, K = cond.shape
    N = w.shape[0]
    cpad = np.zeros((rows, K + pad_cond), np.float32)
    cpad[:, :K] = cond
    wpad = np.zeros((N, K + pad_w), np.uint16)
    wpad[:, :K] = w
    cd = runtime.f32_dev(cpad)
    wd = runtime.bf16_dev(wpad)
    bd = None if b is None else runtime.f32_dev(b)
    ld_style = N + pad_style
    st = torch.full((rows, ld_style), float("nan"), dtype=torch.bfloat16, device="cuda")
    nf = N - fin_col0
    fin = (torch.full((rows, max(nf, 1)), float("nan"), dtype=torch.float32, device="cuda")
           if with_fin else None)
    frt.frt_style_project(rows, K, N, cd, K + pad_cond, wd, K + pad_w, bd, st, ld_style,
                          fin, max(nf, 1), fin_col0)
    torch.cuda.synchronize()
    assert frt.frt_device_status(True) == frt.FRT_OK
    sh = runtime.bf16_host(st)
    # columns past N in each row (the stride's padding) stay untouched
    assert np.all(sh[:, N:] == 0x7FC0)
    fh = None if fin is None else fin.cpu().numpy()[:, :nf]
    return sh[:, :N], fh


@pytest.mark.parametrize("rows,K,N,fin_col0,pads,bias", [
    (1, 512, 37 * 1536, 36 * 1536, (0, 0, 0), True),   # 18-layer stack width
    (1, 2048, 3 * 6144, 2 * 6144, (0, 0, 0), True),     # action-expert width
    (3, 1024, 1005, 0, (4, 8, 3), True),                # ragged N, 3 rows, strides
    (2, 8, 7, 7, (0, 0, 0), False),                     # one chunk, no fin columns
    (5, 24, 77, 40, (12, 16, 1), True),                 # 3 chunks, 2 row groups
    (1, 16384, 96, 48, (0, 0, 0), True),                # long K: 64 chunks per lane
    (8, 256, 4099, 4000, (0, 0, 0), True),              # full row groups, ragged N
])
def test_style_project_parity(rt, rows, K, N, fin_col0, pads, bias):
    cond, w, b = _inputs(rows, K, N, 7 * rows + K + N, bias)
    style, fin = _launch(rt, cond, w, b, fin_col0, *pads)
    _check(style, fin, cond, w, b, fin_col0)


def test_style_project_zero_cond_is_the_bias(rt):
    w = synth.WORKLOADS["style_stack18"]
    n_norms = 2 * w.layers + 1
    inp = synth.modulation_inputs(1, w.D, n_norms, w.seed)
    fin_col0 = 3 * w.D * (n_norms - 1)
    style, fin = _launch(rt, np.zeros_like(inp["cond"]), inp["w"], inp["bias"], fin_col0)
    assert np.array_equal(style[0], bf16_bits(inp["bias"]))
    assert np.array_equal(fin[0], inp["bias"][fin_col0:])


def test_style_project_no_fin_output(rt):
    cond, w, b = _inputs(1, 512, 1536, 11)
    style, _ = _launch(rt, cond, w, b, 0, with_fin=False)
    _check(style, None, cond, w, b, 0)


@pytest.mark.parametrize("name", ["style_stack18", "style_vla18"])
def test_style_workload_sampled(rt, name):
    """The workload at full size, launched as the benchmark launches it;
    the oracle computes a sample of columns (every column is independent):
    the final norm's rows whole and a seeded spread over the rest."""
    wl = synth.WORKLOADS[name]
    n_norms = 2 * wl.layers + 1
    inp = synth.modulation_inputs(wl.rows, wl.D, n_norms, wl.seed)
    fin_col0 = 3 * wl.D * (n_norms - 1)
    style, fin = _launch(rt, inp["cond"], inp["w"], inp["bias"], fin_col0)
    rng = np.random.Generator(np.random.PCG64(5))
    cols = np.unique(np.concatenate([rng.choice(fin_col0, 4096, replace=False),
                                     np.arange(fin_col0, wl.N)]))
    tail = cols >= fin_col0
    n_tail = int(tail.sum())
    # fin covers the sampled tail columns, which come last in `cols`
    _check(style[:, cols], fin[:, cols[tail] - fin_col0], inp["cond"], inp["w"][cols],
           inp["bias"][cols], len(cols) - n_tail)

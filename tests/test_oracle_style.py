"""Pins of the oracle's modulation projection (impls/adarms_stack/fp8_chain.py
`_style_stack` and the binder's per-step bake: st = cond @ W.T + b in fp32,
the rows cast to bf16, the final norm's rows kept fp32).

Each pin fails on a plausible mistake: a dropped bias or a bias added
twice (zero conditioning), a transposed or shifted weight (one-hot
conditioning, column-index weights), a wrong chunk order or norm offset
(the layout pin), a lost or doubled term in the sum (fp64 matmul within the
fp32 error bound), a wrong rounding (bf16 values against numpy's own
round-to-nearest-even of the fp32 result)."""

import numpy as np
import pytest

from oracle import oracle
from fp8_transformer_block_b200 import synth

U = 2.0 ** -24


def _bf16(x):
    return synth.bf16_bits(np.asarray(x, np.float32))


def _val(h):
    return synth.bf16_value(h)


def _inputs(rows, K, N, seed):
    rng = np.random.Generator(np.random.PCG64(seed))
    cond = _val(_bf16(rng.standard_normal((rows, K), dtype=np.float32)))
    w = _bf16(rng.standard_normal((N, K), dtype=np.float32) * np.float32(0.02))
    b = _val(_bf16(rng.standard_normal(N, dtype=np.float32) * np.float32(0.01)))
    return cond, w, b


def test_zero_conditioning_gives_the_bias():
    cond, w, b = _inputs(2, 64, 96, 1)
    style, fin = oracle.style_project(np.zeros_like(cond), w, b, fin_col0=32)
    assert np.array_equal(style, np.broadcast_to(_bf16(b), style.shape))
    assert np.array_equal(fin, np.broadcast_to(b[32:], fin.shape))
    style0, fin0 = oracle.style_project(np.zeros_like(cond), w, None, fin_col0=0)
    assert not np.any(style0 & 0x7FFF) and not np.any(fin0)


@pytest.mark.parametrize("k", [0, 5, 63])
def test_one_hot_conditioning_picks_a_weight_column(k):
    cond, w, b = _inputs(1, 64, 48, 2)
    hot = np.zeros_like(cond)
    hot[0, k] = 4.0  # a power of two: the product is exact
    style, fin = oracle.style_project(hot, w, b, fin_col0=0)
    exact = (4.0 * _val(w[:, k]).astype(np.float64) + b.astype(np.float64)).astype(np.float32)
    assert np.array_equal(fin[0], exact)
    assert np.array_equal(style[0], _bf16(exact))


def test_layout_norm_chunks_and_final_rows():
    """Weights whose first column encodes the output index: with cond = e_0
    every output names its own column, so norm i's (scale, shift, gate)
    land at 3*D*i + {0, D, 2*D} and fin holds the last norm's three rows."""
    D, n_norms = 16, 5
    N = 3 * D * n_norms
    idx = np.arange(N, dtype=np.float32)
    w = np.zeros((N, D), np.uint16)
    w[:, 0] = _bf16(idx / 256.0)  # exact in bf16 for idx < 256
    cond = np.zeros((1, D), np.float32)
    cond[0, 0] = 1.0
    style, fin = oracle.style_project(cond, w, None, fin_col0=3 * D * (n_norms - 1))
    got = _val(style[0]).reshape(n_norms, 3, D) * 256.0
    for i in range(n_norms):
        for chunk in range(3):
            assert np.array_equal(got[i, chunk], idx[3 * D * i + chunk * D:3 * D * i + (chunk + 1) * D])
    assert fin.shape == (1, 3 * D)
    assert np.array_equal(fin[0].reshape(3, D) * 256.0, idx[-3 * D:].reshape(3, D))


@pytest.mark.parametrize("rows,K,N", [(1, 512, 1536), (3, 2048, 200), (2, 8, 7)])
def test_against_fp64_matmul_within_the_fp32_bound(rows, K, N):
    cond, w, b = _inputs(rows, K, N, 3 + K)
    style, fin = oracle.style_project(cond, w, b, fin_col0=0)
    c64, w64 = cond.astype(np.float64), _val(w).astype(np.float64)
    exact = c64 @ w64.T + b.astype(np.float64)
    scale = np.abs(c64) @ np.abs(w64).T + np.abs(b.astype(np.float64))
    bound = (K + 2) * U * scale
    assert np.all(np.abs(fin - exact) <= bound)
    # the bf16 rows are the fp32 rows rounded to nearest even
    assert np.array_equal(style, _bf16(fin))


def test_brute_force_tiny():
    """Pure-Python fp32 evaluation in k order, bias last: bit-identical."""
    rows, K, N = 2, 8, 5
    cond, w, b = _inputs(rows, K, N, 9)
    style, fin = oracle.style_project(cond, w, b, fin_col0=2)
    wv = _val(w)
    for r in range(rows):
        for n in range(N):
            acc = np.float32(0.0)
            for k in range(K):
                acc = np.float32(acc + np.float32(cond[r, k] * wv[n, k]))
            st = np.float32(acc + b[n])
            assert style[r, n] == _bf16(st)
            if n >= 2:
                assert fin[r, n - 2] == st


def test_synthetic_recipe_shapes():
    w = synth.WORKLOADS["style_stack18"]
    inp = synth.modulation_inputs(1, w.D, 2 * w.layers + 1, w.seed)
    assert inp["w"].shape == (w.N, w.D) and w.N == 37 * 3 * 512
    assert inp["cond"].dtype == np.float32 and inp["bias"].shape == (w.N,)
    # cond and bias are values on the bf16 grid
    assert np.array_equal(_val(_bf16(inp["cond"])), inp["cond"])
    assert np.array_equal(_val(_bf16(inp["bias"])), inp["bias"])

"""Shared set-up for the GPU parity tests: seeded inputs of a workload, the
oracle's run of the chain on them, and the GPU run through the C ABI.

The oracle side only calls ``oracle``; the GPU side only calls the binding.
Static activation scales come from the oracle's calibration on the
workload's calibration batch (seed + 500) and are passed identically to both
sides.
"""

from __future__ import annotations

import numpy as np

import oracle
from fp8_transformer_block_b200 import synth

SENTINEL = 0x7FC1  # a bf16 NaN pattern no kernel writes


def calibrate_adarms(w: synth.Workload) -> float:
    cal = synth.adarms_inputs(w.cal_rows, w.D, w.seed + synth.CAL_OFFSET,
                              outliers=w.outliers)
    out = oracle.ada_rms_norm_quant(cal["res"], cal["delta"],
                                    cal["prev_gate"], cal["style"], 1.0,
                                    eps=w.eps)
    return out["amax"] / 448.0


def calibrate_dit(w: synth.Workload, table) -> float:
    cal = synth.dit_inputs(w.cal_rows, w.D, w.seed + synth.CAL_OFFSET,
                           with_table=False)
    out = oracle.ada_layer_norm_quant_table(cal["x"], cal["temb"], table, 0,
                                            1, 1.0, eps=w.eps)
    return out["amax"] / 448.0


def oracle_attn_chain(inp, x8, pk, w: synth.Workload, rows_sel=None):
    """GEMM -> split + RoPE + KV of the oracle on the given x8 codes.

    Returns (qkv, q_out, k_cache, v_cache) with caches of capacity T whose
    rows outside [P, P + M) hold the sentinel (or the copied prefix)."""
    B, M = w.B, w.M
    qkv = oracle.fp8_gemm(x8, pk["w8"], inp["act_scale"], pk["w_scale"],
                          pk["bias"] if w.bias else None, rows=rows_sel)
    rope = oracle.rope_table(M, w.hd, w.P, w.theta)
    kc = np.full((B, w.T, w.hkv, w.hd), SENTINEL, np.uint16)
    vc = np.full((B, w.T, w.hkv, w.hd), SENTINEL, np.uint16)
    if inp.get("prefix_k") is not None:
        kc, vc = oracle.prefix_copy(inp["prefix_k"], inp["prefix_v"], w.P,
                                    kc, vc, interleave=True)
    if rows_sel is not None:
        return qkv, None, kc, vc
    q, kc, vc = oracle.split_rope_kvcache(qkv, rope, B, M, w.hq, w.hkv, w.hd,
                                          w.P, kc, vc)
    return qkv, q, kc, vc

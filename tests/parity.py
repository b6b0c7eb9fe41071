"""Comparison helpers for the GPU-vs-oracle parity tests.

Tolerances are the chain's stated bar:
  * indices, copies, caches: bit-exact;
  * e4m3 activation codes: >= 99.99 % identical, every other code exactly one
    step away (adjacent magnitude with the same sign, or +-0 against the
    smallest subnormal, or +0 against -0);
  * GEMM / RoPE outputs: max |err| <= 2e-2 * rms(ref), fp32 accumulation.
"""

import numpy as np

from fp8_transformer_block_b200.synth import bf16_value

CODE_MATCH = 0.9999
RMS_TOL = 2e-2


def e4m3_step_distance(a, b):
    a = np.asarray(a, np.uint8).astype(np.int32)
    b = np.asarray(b, np.uint8).astype(np.int32)
    ma, mb = a & 0x7F, b & 0x7F
    sa, sb = a >> 7, b >> 7
    same = a == b
    adjacent = (sa == sb) & (np.abs(ma - mb) == 1)
    zero_cross = ((ma == 0) & (mb <= 1)) | ((mb == 0) & (ma <= 1))
    # 0x7F / 0xFF are e4m3fn's NaN: never one step from a finite code (the
    # quantizer saturates at +-448, so a NaN is an error, not a rounding)
    nan = (ma == 0x7F) | (mb == 0x7F)
    near = (adjacent | zero_cross) & ~nan
    dist = np.where(same, 0, np.where(near, 1, 2))
    return dist


def assert_codes(got, ref, match=CODE_MATCH, what="codes"):
    d = e4m3_step_distance(got, ref)
    frac = float((d == 0).mean()) if d.size else 1.0
    bad = int((d > 1).sum())
    assert bad == 0, f"{what}: {bad} codes differ by more than one step"
    assert frac >= match, f"{what}: only {frac:.6f} identical (< {match})"
    return frac


def rel_rms_err(got_bf16, ref_bf16):
    g = bf16_value(got_bf16).astype(np.float64)
    r = bf16_value(ref_bf16).astype(np.float64)
    rms = np.sqrt((r ** 2).mean()) if r.size else 1.0
    return float(np.abs(g - r).max() / rms) if r.size else 0.0


def assert_rms(got_bf16, ref_bf16, tol=RMS_TOL, what="values"):
    """max|err| <= tol * rms(ref), where an element that differs from the
    reference by exactly one bf16 step is always within the bar.  Both
    sides round an fp32 value to bf16, and the two fp32 values (sums taken
    in different orders) can straddle a rounding boundary; one bf16 step is
    2^-8 .. 2^-7 of the value, which exceeds 2e-2 * rms for outputs beyond
    about 5 * rms (present at these sizes).  Every element off by more than
    one step must meet the bar."""
    g = bf16_value(got_bf16).astype(np.float64)
    r = bf16_value(ref_bf16).astype(np.float64)
    if not r.size:
        return 0.0
    rms = np.sqrt((r ** 2).mean())
    err = np.abs(g - r)
    over = err > tol * rms
    if over.any():
        steps = bf16_ulps(np.asarray(got_bf16)[over], np.asarray(ref_bf16)[over])
        bad = int((steps > 1).sum())
        worst = float(err[over][steps > 1].max() / rms) if bad else 0.0
        assert bad == 0, (f"{what}: {bad} values beyond {tol} * rms(ref) and more than "
                          f"one bf16 step off (worst {worst:.3e} * rms)")
    return float(err.max() / rms)


def bf16_ulps(got_bf16, ref_bf16):
    """Distance in bf16 units of the last place (same-sign values)."""
    g = np.asarray(got_bf16, np.uint16).astype(np.int32)
    r = np.asarray(ref_bf16, np.uint16).astype(np.int32)
    # map sign-magnitude to a monotone integer line
    g = np.where(g & 0x8000, -(g & 0x7FFF), g)
    r = np.where(r & 0x8000, -(r & 0x7FFF), r)
    return np.abs(g - r)


def gate_up_block_order(H, block=128):
    """Row order of the library's gate/up block layout as indices into the
    pages' concatenation [gate; up] (H rows each): packed row r of 256-row
    block b holds gate row 128b + r for r < 128 and up row 128b + r - 128
    after it.  Test-side only: the oracle packs in the pages' order and the
    tests permute its rows to compare with the device layout."""
    order = np.empty(2 * H, np.int64)
    for b in range(H // block):
        order[2 * block * b: 2 * block * b + block] = np.arange(block * b, block * (b + 1))
        order[2 * block * b + block: 2 * block * (b + 1)] = H + np.arange(block * b, block * (b + 1))
    return order

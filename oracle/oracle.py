"""ctypes front end of the C oracle (``frt_oracle.c``).

Test infrastructure only (see the package docstring).  Every function takes
and returns numpy arrays: bf16 tensors travel as ``uint16`` bit patterns,
e4m3 tensors as ``uint8`` codes, scales as Python floats.  The arithmetic is
all in the C file; this module only marshals arguments and composes the
chain's steps in the pages' order.
"""

from __future__ import annotations

import ctypes as C
import os
import subprocess

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "frt_oracle.c")
_BUILD = os.path.join(_HERE, "_build")
_LIB_PATH = os.path.join(_BUILD, "liboracle.so")

__all__ = [
    "build_oracle", "num_threads",
    "bf16_to_f32", "f32_to_bf16", "f64_to_bf16", "e4m3_to_f32", "f32_to_e4m3",
    "ada_rms_norm_quant", "ada_layer_norm_quant_table", "pack_weights_fp8",
    "fp8_gemm", "rope_table", "split_rope_kvcache", "prefix_copy",
    "geglu_quant", "quant_fp8_static", "ada_rms_tail", "adarms_layer_stack",
    "gelu_quant", "dit_ffn", "style_project",
]


def build_oracle(force: bool = False) -> str:
    """Compile the oracle with gcc (fp32 ops exactly as written: no FMA
    contraction, no fast-math) and return the shared-object path."""
    os.makedirs(_BUILD, exist_ok=True)
    if (not force and os.path.exists(_LIB_PATH)
            and os.path.getmtime(_LIB_PATH) >= os.path.getmtime(_SRC)):
        return _LIB_PATH
    tmp = _LIB_PATH + f".tmp{os.getpid()}"
    subprocess.check_call([
        "gcc", "-O2", "-ffp-contract=off", "-fno-fast-math", "-fopenmp",
        "-fPIC", "-shared", "-o", tmp, _SRC, "-lm"])
    os.replace(tmp, _LIB_PATH)
    return _LIB_PATH


_lib = None


def _L():
    global _lib
    if _lib is None:
        lib = C.CDLL(build_oracle())
        p = C.c_void_p
        i, l, f, d = C.c_int, C.c_long, C.c_float, C.c_double
        sig = {
            "or_bf16_to_f32": (f, [C.c_uint16]),
            "or_bf16_from_f32": (C.c_uint16, [f]),
            "or_bf16_from_f64": (C.c_uint16, [d]),
            "or_e4m3_to_f32": (f, [C.c_uint8]),
            "or_e4m3_from_f32": (C.c_uint8, [f]),
            "or_ada_rms_norm_quant": (None, [i, i, f, p, p, p, l, p, p, l, f,
                                             p, p, p, p]),
            "or_ada_layer_norm_quant_table": (None, [i, i, f, p, p, i, p, i, i,
                                                     f, p, p, p]),
            "or_pack_weights_fp8": (None, [i, p, p, i, p, i, i, p, p, p]),
            "or_fp8_gemm": (None, [i, i, i, p, p, f, f, p, p, l, p, i]),
            "or_rope_table": (None, [i, i, i, d, p]),
            "or_split_rope_kvcache": (None, [i, i, i, i, i, i, i, p, p, p, p,
                                             p]),
            "or_prefix_copy": (None, [i, i, i, i, i, i, p, p, i, p, p]),
            "or_geglu_quant": (None, [i, i, p, f, p, p]),
            "or_quant_fp8_static": (None, [i, i, p, l, f, p, p]),
            "or_gelu_quant": (None, [i, i, p, l, f, p, p]),
            "or_ada_rms_tail": (None, [i, i, f, p, p, p, l, p, l, p]),
            "or_style_project": (None, [i, i, i, p, p, p, p, p, i]),
            "or_num_threads": (i, []),
        }
        for name, (res, args) in sig.items():
            fn = getattr(lib, name)
            fn.restype = res
            fn.argtypes = args
        _lib = lib
    return _lib


def _ptr(a):
    return None if a is None else a.ctypes.data_as(C.c_void_p)


def _c(a, dtype):
    a = np.ascontiguousarray(a, dtype=dtype)
    return a


def num_threads() -> int:
    return int(_L().or_num_threads())


# ---- scalar codecs (vectorised by looping in C one value at a time) ----

def bf16_to_f32(h):
    h = np.asarray(h, dtype=np.uint16)
    return (h.astype(np.uint32) << 16).view(np.float32)


def f32_to_bf16(x):
    x = np.asarray(x, dtype=np.float32)
    fn = _L().or_bf16_from_f32
    return np.array([fn(float(v)) for v in x.ravel()],
                    dtype=np.uint16).reshape(x.shape)


def f64_to_bf16(x):
    x = np.asarray(x, dtype=np.float64)
    fn = _L().or_bf16_from_f64
    return np.array([fn(float(v)) for v in x.ravel()],
                    dtype=np.uint16).reshape(x.shape)


def e4m3_to_f32(c):
    c = np.asarray(c, dtype=np.uint8)
    fn = _L().or_e4m3_to_f32
    table = np.array([fn(k) for k in range(256)], dtype=np.float32)
    return table[c]


def f32_to_e4m3(x):
    x = np.asarray(x, dtype=np.float32)
    fn = _L().or_e4m3_from_f32
    return np.array([fn(float(v)) for v in x.ravel()],
                    dtype=np.uint8).reshape(x.shape)


# ---- chain steps ----

def ada_rms_norm_quant(res, delta, prev_gate, style, act_scale, eps=1e-6,
                       weight=None, want_gate=True, want_y=False):
    """AdaRMS producer.  ``res`` [rows, D] is NOT modified; the updated
    residual is returned.  prev_gate / style with one row broadcast.
    Returns dict(res, x8, gate_out, y, amax)."""
    res = _c(res, np.uint16).copy()
    rows, D = res.shape
    delta = _c(delta, np.uint16)
    prev_gate = _c(prev_gate, np.uint16)
    style = _c(style, np.uint16)
    gstride = 0 if prev_gate.shape[0] == 1 else D
    sstride = 0 if style.shape[0] == 1 else 3 * D
    x8 = np.empty((rows, D), np.uint8)
    gate = np.empty((rows, D), np.uint16) if want_gate else None
    y = np.empty((rows, D), np.float32) if want_y else None
    amax = np.zeros(1, np.float32)
    w = None if weight is None else _c(weight, np.uint16)
    _L().or_ada_rms_norm_quant(rows, D, eps, _ptr(res), _ptr(delta),
                               _ptr(prev_gate), gstride, _ptr(w), _ptr(style),
                               sstride, float(act_scale), _ptr(x8), _ptr(gate),
                               _ptr(y), _ptr(amax))
    return {"res": res, "x8": x8, "gate_out": gate, "y": y,
            "amax": float(amax[0])}


def ada_layer_norm_quant_table(x, temb, table, shift_idx, scale_idx,
                               act_scale, eps=1e-6, want_y=False):
    """Per-token-table LayerNorm producer.  x [rows, D]; temb
    [rows, chunks, D] bf16; table [chunks, D] fp32."""
    x = _c(x, np.uint16)
    rows, D = x.shape
    temb = _c(temb, np.uint16).reshape(rows, -1, D)
    chunks = temb.shape[1]
    table = _c(table, np.float32).reshape(chunks, D)
    x8 = np.empty((rows, D), np.uint8)
    y = np.empty((rows, D), np.float32) if want_y else None
    amax = np.zeros(1, np.float32)
    _L().or_ada_layer_norm_quant_table(rows, D, eps, _ptr(x), _ptr(temb),
                                       chunks, _ptr(table), shift_idx,
                                       scale_idx, float(act_scale), _ptr(x8),
                                       _ptr(y), _ptr(amax))
    return {"x8": x8, "y": y, "amax": float(amax[0])}


def pack_weights_fp8(ws, biases=None, layout=0, hd=0):
    """Joint pack of sibling weights (list of [n_i, K] uint16).  Returns
    dict(w8 [N, K], w_scale float, bias [N] uint16).  layout 0 stacks the
    siblings in order (the pages' torch.cat); layout 1 interleaves the q and
    k rows per head (the chain's `_interleave_rows`)."""
    if layout not in (0, 1):
        raise ValueError(f"layout must be 0 (concatenation) or 1 (q/k interleave), got {layout}")
    ws = [_c(w, np.uint16) for w in ws]
    K = ws[0].shape[1]
    n_i = np.array([w.shape[0] for w in ws], dtype=np.int32)
    N = int(n_i.sum())
    if biases is None:
        biases = [None] * len(ws)
    biases = [None if b is None else _c(b, np.uint16) for b in biases]
    wp = (C.c_void_p * len(ws))(*[w.ctypes.data for w in ws])
    bp = (C.c_void_p * len(ws))(*[0 if b is None else b.ctypes.data
                                  for b in biases])
    w8 = np.empty((N, K), np.uint8)
    scale = np.zeros(1, np.float32)
    bias = np.empty(N, np.uint16)
    _L().or_pack_weights_fp8(len(ws), C.cast(wp, C.c_void_p), _ptr(n_i), K,
                             C.cast(bp, C.c_void_p), layout, hd, _ptr(w8),
                             _ptr(scale), _ptr(bias))
    return {"w8": w8, "w_scale": float(scale[0]), "bias": bias}


def fp8_gemm(x8, w8, act_scale, w_scale, bias=None, rows=None):
    """Y = bf16(alpha * x8 @ w8^T + bias).  ``rows`` (optional) selects rows
    of x8; the result then has len(rows) rows."""
    x8 = _c(x8, np.uint8)
    w8 = _c(w8, np.uint8)
    M, K = x8.shape
    N = w8.shape[0]
    idx = None if rows is None else _c(rows, np.int32)
    n_rows = M if idx is None else len(idx)
    out = np.empty((n_rows, N), np.uint16)
    b = None if bias is None else _c(bias, np.uint16)
    _L().or_fp8_gemm(M, N, K, _ptr(x8), _ptr(w8), float(act_scale),
                     float(w_scale), _ptr(b), _ptr(out), N, _ptr(idx), n_rows)
    return out


def rope_table(M, hd, P, theta=10000.0):
    out = np.empty((M, hd), np.uint16)
    _L().or_rope_table(M, hd, P, float(theta), _ptr(out))
    return out


def split_rope_kvcache(qkv, rope, B, M, hq, hkv, hd, P, k_cache, v_cache):
    """Returns (q_out [B, M, hq, hd], k_cache, v_cache); the caches passed
    in are copied, then written at rows P..P+M-1."""
    qkv = _c(qkv, np.uint16)
    rope = _c(rope, np.uint16)
    k_cache = _c(k_cache, np.uint16).copy()
    v_cache = _c(v_cache, np.uint16).copy()
    T = k_cache.shape[1]
    q = np.empty((B, M, hq, hd), np.uint16)
    _L().or_split_rope_kvcache(B, M, hq, hkv, hd, P, T, _ptr(qkv), _ptr(rope),
                               _ptr(q), _ptr(k_cache), _ptr(v_cache))
    return q, k_cache, v_cache


def prefix_copy(prefix_k, prefix_v, P, k_cache, v_cache, interleave=True):
    """prefix_k/v [B, hkv, T_src, hd]; caches [B, T, hkv, hd] (copied)."""
    prefix_k = _c(prefix_k, np.uint16)
    prefix_v = _c(prefix_v, np.uint16)
    B, hkv, T_src, hd = prefix_k.shape
    k_cache = _c(k_cache, np.uint16).copy()
    v_cache = _c(v_cache, np.uint16).copy()
    T = k_cache.shape[1]
    _L().or_prefix_copy(B, hkv, hd, P, T, T_src, _ptr(prefix_k),
                        _ptr(prefix_v), int(bool(interleave)), _ptr(k_cache),
                        _ptr(v_cache))
    return k_cache, v_cache


def gelu_quant(u, out_scale):
    """[ptok_table] fp8_gelu_mlp's middle step: hid8 = q8(gelu_tanh(u);
    out_scale) for bf16 bits u [M, H]; returns (hid8, amax)."""
    u = _c(u, np.uint16)
    M, H = u.shape
    hid8 = np.empty((M, H), np.uint8)
    amax = np.zeros(1, np.float32)
    _L().or_gelu_quant(M, H, _ptr(u), H, float(out_scale), _ptr(hid8), _ptr(amax))
    return hid8, float(amax[0])


def quant_fp8_static(x, scale):
    """[fp8_chain] out_project's static quantize: x8 = q8(x; scale) for a
    bf16-bits array x [rows, D]; returns (x8, amax of |x|)."""
    x = _c(x, np.uint16)
    rows, D = x.shape
    x8 = np.empty((rows, D), np.uint8)
    amax = np.zeros(1, np.float32)
    _L().or_quant_fp8_static(rows, D, _ptr(x), D, float(scale), _ptr(x8), _ptr(amax))
    return x8, float(amax[0])


def ada_rms_tail(res, delta, gate, fin, eps):
    """[fp8_chain] _make_run's final tail: bf16 bits [rows, D] of
    RMSnorm(res + gate*delta) * (1 + fin[0]) + fin[1] (fp32 throughout).
    gate is [1, D] (broadcast) or [rows, D]; fin is fp32 [2 or 3, D]."""
    res = _c(res, np.uint16)
    delta = _c(delta, np.uint16)
    gate = _c(gate, np.uint16)
    fin = _c(fin, np.float32)
    rows, D = res.shape
    out = np.empty((rows, D), np.uint16)
    gs = 0 if gate.shape[0] == 1 else D
    _L().or_ada_rms_tail(rows, D, float(eps), _ptr(res), _ptr(delta), _ptr(gate), gs,
                         _ptr(fin), fin.shape[1], _ptr(out))
    return out


def style_project(cond, w, bias=None, fin_col0=None):
    """[fp8_chain] _style_stack and the binder's per-step bake: the stacked
    modulation projection st = cond @ w.T + bias in fp32 (k order, bias
    last).  cond fp32 [rows, K]; w bf16 bits [N, K]; bias fp32 [N] or None.
    Returns (style bf16 bits [rows, N], fin fp32 [rows, N - fin_col0] or
    None when fin_col0 is None)."""
    cond = _c(np.atleast_2d(cond), np.float32)
    w = _c(w, np.uint16)
    rows, K = cond.shape
    N = w.shape[0]
    assert w.shape[1] == K
    b = None if bias is None else _c(bias, np.float32)
    style = np.empty((rows, N), np.uint16)
    fin = None if fin_col0 is None else np.empty((rows, N - fin_col0), np.float32)
    _L().or_style_project(rows, K, N, _ptr(cond), _ptr(w),
                          None if b is None else _ptr(b), _ptr(style),
                          None if fin is None else _ptr(fin),
                          0 if fin_col0 is None else int(fin_col0))
    return style, fin


def geglu_quant(gu, out_scale):
    gu = _c(gu, np.uint16)
    M, H2 = gu.shape
    H = H2 // 2
    hid8 = np.empty((M, H), np.uint8)
    amax = np.zeros(1, np.float32)
    _L().or_geglu_quant(M, H, _ptr(gu), float(out_scale), _ptr(hid8),
                        _ptr(amax))
    return hid8, float(amax[0])


def adarms_layer_stack(x, layers, fin, dims, scales=None, eps=1e-6):
    """Every step of the AdaRMS layer loop except attention, in the order of
    [fp8_chain] `_make_run`, then the final tail.  Per layer l:
      norm_project(slot 2l, "qkv"): producer (res += gate * delta, AdaRMS,
        quantize) into the packed q/k/v GEMM; the prefix copy and the split +
        RoPE + KV write;
      attention stand-in: att2 = q_out viewed as [rows, hq * hd] (attention
        itself is outside the path);
      out_project: static quantize of att2, o GEMM -> dn;
      norm_project(slot 2l + 1, "gu"): producer (delta = dn, gate = the qkv
        norm's gate) into the packed gate/up GEMM;
      down_project: GEGLU requant, down GEMM -> dn;
      delta, gate = dn, the gu norm's gate.
    Then ada_rms_tail(res, delta, gate, fin).

    layers[l]: dict(qkv, o, gu, dn: pack_weights_fp8 results (qkv with the
    q/k interleave, gu in concatenated [gate; up] order), styles [2, 3D]
    (attention site, FFN site), prefix_k, prefix_v host caches).
    dims: dict(B, M, D, hq, hkv, hd, P, T, H, theta).  scales: per layer
    dict(a_qkv, a_o, a_gu, a_dn); None calibrates them on this batch, each
    site's scale = amax / 448 of its quantizer input, in order.
    Returns (out, records, scales)."""
    B, M, D = dims["B"], dims["M"], dims["D"]
    rows = B * M
    table = rope_table(M, dims["hd"], dims["P"], dims.get("theta", 10000.0))
    res = _c(x, np.uint16).copy()
    delta = np.zeros((rows, D), np.uint16)
    gate = np.zeros((1, D), np.uint16)
    recs, used = [], []

    def scale_of(site, l, amax):
        if scales is not None:
            return scales[l][site]
        return max(amax / 448.0, 1e-8)

    for l, ly in enumerate(layers):
        sc = {}
        st_attn, st_ffn = ly["styles"][0:1], ly["styles"][1:2]
        a = scale_of("a_qkv", l, None if scales else
                     ada_rms_norm_quant(res, delta, gate, st_attn, 1.0, eps)["amax"])
        sc["a_qkv"] = a
        pr = ada_rms_norm_quant(res, delta, gate, st_attn, a, eps)
        qkv = fp8_gemm(pr["x8"], ly["qkv"]["w8"], a, ly["qkv"]["w_scale"])
        kc = np.zeros((B, dims["T"], dims["hkv"], dims["hd"]), np.uint16)
        vc = kc
        if ly.get("prefix_k") is not None:
            kc, vc = prefix_copy(ly["prefix_k"], ly["prefix_v"], dims["P"], kc, vc, True)
        q, kc, vc = split_rope_kvcache(qkv, table, B, M, dims["hq"], dims["hkv"],
                                       dims["hd"], dims["P"], kc, vc)
        att2 = q.reshape(rows, dims["hq"] * dims["hd"])
        a_o = scale_of("a_o", l, None if scales else quant_fp8_static(att2, 1.0)[1])
        sc["a_o"] = a_o
        o8, _ = quant_fp8_static(att2, a_o)
        dn_o = fp8_gemm(o8, ly["o"]["w8"], a_o, ly["o"]["w_scale"])
        a_gu = scale_of("a_gu", l, None if scales else
                        ada_rms_norm_quant(pr["res"], dn_o, pr["gate_out"], st_ffn, 1.0,
                                           eps)["amax"])
        sc["a_gu"] = a_gu
        pf = ada_rms_norm_quant(pr["res"], dn_o, pr["gate_out"], st_ffn, a_gu, eps)
        gu = fp8_gemm(pf["x8"], ly["gu"]["w8"], a_gu, ly["gu"]["w_scale"])
        a_dn = scale_of("a_dn", l, None if scales else geglu_quant(gu, 1.0)[1])
        sc["a_dn"] = a_dn
        hid8, _ = geglu_quant(gu, a_dn)
        dn = fp8_gemm(hid8, ly["dn"]["w8"], a_dn, ly["dn"]["w_scale"])
        recs.append({"x8": pr["x8"], "q": q, "k": kc, "v": vc, "o8": o8, "dn_o": dn_o,
                     "x8_ffn": pf["x8"], "hid8": hid8, "dn": dn, "res": pf["res"],
                     "g1": pr["gate_out"], "g2": pf["gate_out"]})
        used.append(sc)
        res, delta, gate = pf["res"], dn, pf["gate_out"]
    out = ada_rms_tail(res, delta, gate, fin, eps)
    return out, recs, used


def dit_ffn(x, temb, table, up, dn, a_in, a_hid=None, eps=1e-6, shift_idx=3, scale_idx=4):
    """The video-DiT block's FFN half ([ptok_table] PerTokenModChainBlock.
    forward): the per-token-table producer at the FFN site (chunks 3, 4)
    into the fp8_gelu_mlp pair: up GEMM (+ bias), GELU + static requant,
    down GEMM (+ bias).  up / dn: pack_weights_fp8 results with bias.
    a_hid None calibrates it on this batch (amax of the GELU output / 448).
    Returns dict(x8, u, hid8, ff, a_hid)."""
    pr = ada_layer_norm_quant_table(x, temb, table, shift_idx, scale_idx, a_in, eps=eps)
    u = fp8_gemm(pr["x8"], up["w8"], a_in, up["w_scale"], up["bias"])
    if a_hid is None:
        a_hid = max(gelu_quant(u, 1.0)[1] / 448.0, 1e-8)
    hid8, _ = gelu_quant(u, a_hid)
    ff = fp8_gemm(hid8, dn["w8"], a_hid, dn["w_scale"], dn["bias"])
    return {"x8": pr["x8"], "u": u, "hid8": hid8, "ff": ff, "a_hid": a_hid, "amax_in": pr["amax"]}

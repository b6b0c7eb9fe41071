"""ctypes binding of libfrt (the C ABI declared in ``include/frt.h``).

Argument marshalling only: every function below forwards to the C entry
point of the same name.  Tensor arguments may be torch tensors (their
``data_ptr()`` is passed), plain integers (device addresses) or None (NULL).
``stream`` defaults to torch's current CUDA stream.  A negative status
raises :class:`FrtError` with the library's reason string.

There is no fallback: if ``libfrt.so`` is missing or cannot be loaded the
import fails with an error naming the build command.
"""

from __future__ import annotations

import ctypes as C
import os

_HERE = os.path.dirname(os.path.abspath(__file__))
# FRT_LIBRARY may name another build of the same ABI (e.g. an instrumented
# one); by default the in-tree libfrt.so is loaded.
LIB_PATH = os.environ.get("FRT_LIBRARY") or os.path.join(_HERE, "libfrt.so")

FRT_OK, FRT_EINVAL, FRT_ESHAPE, FRT_EALIGN, FRT_ERANGE, FRT_ECUDA, \
    FRT_ETIMEOUT = 0, -1, -2, -3, -4, -5, -6
FRT_NORM_ADARMS, FRT_NORM_LAYERNORM_TABLE = 0, 1
FRT_PACK_CONCAT, FRT_PACK_QK_INTERLEAVE, FRT_PACK_GATE_UP_BLOCKS = 0, 1, 2
FRT_EPI_BF16, FRT_EPI_GEGLU_E4M3, FRT_EPI_GELU_E4M3 = 0, 1, 2
FRT_CHAIN_FUSED_ROPE, FRT_CHAIN_UNFUSED = 0, 1
FRT_PEAK_OPERANDS_GAUSSIAN, FRT_PEAK_OPERANDS_LOW_TOGGLE = 0, 1

STATUS_NAMES = {0: "FRT_OK", -1: "FRT_EINVAL", -2: "FRT_ESHAPE",
                -3: "FRT_EALIGN", -4: "FRT_ERANGE", -5: "FRT_ECUDA",
                -6: "FRT_ETIMEOUT"}


class FrtError(RuntimeError):
    def __init__(self, code: int, fn: str, reason: str):
        self.code = code
        super().__init__(f"{fn} -> {STATUS_NAMES.get(code, code)}: {reason}")


def _load():
    if not os.path.exists(LIB_PATH):
        raise ImportError(
            f"libfrt.so not found at {LIB_PATH}; build it with "
            "`python -m fp8_transformer_block_b200.build` (nvcc, sm_100a)")
    return C.CDLL(LIB_PATH)


_lib = _load()

_p, _i, _l, _f, _d, _z = (C.c_void_p, C.c_int, C.c_long, C.c_float,
                          C.c_double, C.c_size_t)


class frt_chain_desc(C.Structure):
    """Mirror of ``frt_chain_desc`` in include/frt.h (same field order)."""
    _fields_ = [
        ("B", _i), ("M", _i), ("D", _i), ("hq", _i), ("hkv", _i), ("hd", _i),
        ("P", _i), ("T", _i), ("eps", _f), ("norm_mode", _i), ("flags", _i),
        ("res", _p), ("delta", _p), ("prev_gate", _p), ("gate_row_stride", _l),
        ("norm_weight", _p), ("style", _p), ("style_row_stride", _l),
        ("gate_out", _p),
        ("x", _p), ("temb", _p), ("chunks", _i), ("table", _p),
        ("shift_idx", _i), ("scale_idx", _i),
        ("act_scale", _p), ("x8", _p),
        ("w8", _p), ("w_scale", _p), ("bias", _p),
        ("rope", _p), ("q_out", _p), ("k_cache", _p), ("v_cache", _p),
        ("prefix_k", _p), ("prefix_v", _p), ("prefix_T_src", _i),
        ("prefix_interleave", _i),
        ("qkv", _p), ("workspace", _p), ("workspace_bytes", _z),
    ]


class frt_ffn_desc(C.Structure):
    """Mirror of ``frt_ffn_desc`` in include/frt.h (same field order)."""
    _fields_ = [
        ("rows", _i), ("D", _i), ("H", _i), ("eps", _f),
        ("res", _p), ("delta", _p), ("prev_gate", _p), ("gate_row_stride", _l),
        ("norm_weight", _p), ("style", _p), ("style_row_stride", _l),
        ("gate_out", _p), ("act_scale", _p), ("x8", _p),
        ("w8_gu", _p), ("w_scale_gu", _p), ("bias_gu", _p), ("hid_scale", _p),
        ("hid8", _p), ("w8_dn", _p), ("w_scale_dn", _p), ("bias_dn", _p),
        ("out", _p), ("workspace", _p), ("workspace_bytes", _z),
    ]


_SIGS = {
    "frt_last_error": (C.c_char_p, []),
    "frt_version": (_i, []),
    "frt_device_status": (_i, [_i, _p]),
    "frt_ada_norm_quant_fp8": (_i, [_i, _i, _i, _f, _p, _p, _p, _l, _p, _p, _l,
                                    _p, _p, _i, _p, _i, _i, _p, _p, _p, _p,
                                    _p]),
    "frt_pack_weights_fp8": (_i, [_i, _p, _p, _i, _p, _i, _i, _p, _p, _p, _p]),
    "frt_gemm_workspace_size": (_z, [_i, _i, _i, _i]),
    "frt_packed_fp8_gemm": (_i, [_i, _i, _i, _p, _p, _p, _p, _p, _i, _p, _l,
                                 _p, _p, _z, _p]),
    "frt_packed_fp8_gemm_noalloc": (_i, [_i, _i, _i, _p, _p, _p, _p, _p, _i,
                                         _p, _l, _p, _p]),
    "frt_packed_fp8_gemm_rope_kvcache": (_i, [_i, _i, _i, _i, _i, _i, _i, _i,
                                              _p, _p, _p, _p, _p, _p, _p, _p,
                                              _p, _p, _z, _p]),
    "frt_build_rope_table": (_i, [_i, _i, _i, _d, _p, _p]),
    "frt_split_rope_kvcache": (_i, [_i, _i, _i, _i, _i, _i, _i, _p, _p, _p,
                                    _p, _p, _p, _p, _i, _i, _p]),
    "frt_prefix_copy_kv": (_i, [_i, _i, _i, _i, _i, _i, _p, _p, _i, _p, _p,
                                _p]),
    "frt_geglu_quant_fp8": (_i, [_i, _i, _p, _l, _p, _p, _p, _p]),
    "frt_chain_workspace_size": (_z, [C.POINTER(frt_chain_desc)]),
    "frt_chain_layer": (_i, [C.POINTER(frt_chain_desc), _p]),
    "frt_ffn_workspace_size": (_z, [C.POINTER(frt_ffn_desc)]),
    "frt_ffn_layer": (_i, [C.POINTER(frt_ffn_desc), _p]),
    "frt_selftest_bounded_wait": (_i, [_i, _p]),
    "frt_selftest_gelu": (_i, [_p, _p, _l, _p]),
    "frt_quantize_fp8_static": (_i, [_i, _i, _p, _l, _p, _p, _p, _p]),
    "frt_gelu_quant_fp8": (_i, [_i, _i, _p, _l, _p, _p, _p, _p]),
    "frt_ada_rms_tail": (_i, [_i, _i, _f, _p, _p, _p, _l, _p, _l, _p, _p]),
    "frt_style_project": (_i, [_i, _i, _i, _p, _l, _p, _l, _p, _p, _l, _p, _l, _i, _p]),
    "frt_gemm_plan_info": (_i, [_i, _i, _i, _i, _p, _i]),
    "frt_peak_fp8_mma": (_i, [_i, _i, _i, _p]),
    "frt_peak_copy": (_i, [_p, _p, C.c_size_t, _p]),
}

for _name, (_res, _args) in _SIGS.items():
    _fn = getattr(_lib, _name)
    _fn.restype = _res
    _fn.argtypes = _args

EXPORTED = tuple(_SIGS)


def ptr(x):
    """Device address of a tensor, an int, or None."""
    if x is None:
        return None
    if isinstance(x, int):
        return x or None
    return x.data_ptr() or None


def _stream(stream):
    if stream is None:
        import torch
        return torch.cuda.current_stream().cuda_stream or None
    if isinstance(stream, int):
        return stream or None
    return stream.cuda_stream or None


def last_error() -> str:
    return (_lib.frt_last_error() or b"").decode()


def _check(rc: int, name: str) -> int:
    if rc != FRT_OK:
        raise FrtError(rc, name, last_error())
    return rc


def frt_version() -> int:
    return _lib.frt_version()


def frt_device_status(reset=True, stream=None) -> int:
    """Returns the status code (does not raise)."""
    return _lib.frt_device_status(int(reset), _stream(stream))


def frt_ada_norm_quant_fp8(mode, rows, D, eps, res, delta, prev_gate,
                           gate_row_stride, weight, style, style_row_stride,
                           x, temb, chunks, table, shift_idx, scale_idx,
                           act_scale, x8_out, gate_out=None, amax_out=None,
                           stream=None):
    return _check(_lib.frt_ada_norm_quant_fp8(
        mode, rows, D, eps, ptr(res), ptr(delta), ptr(prev_gate),
        gate_row_stride, ptr(weight), ptr(style), style_row_stride, ptr(x),
        ptr(temb), chunks, ptr(table), shift_idx, scale_idx, ptr(act_scale),
        ptr(x8_out), ptr(gate_out), ptr(amax_out), _stream(stream)),
        "frt_ada_norm_quant_fp8")


def frt_pack_weights_fp8(ws, n_rows, K, biases, layout, hd, w8_out,
                         w_scale_out, bias_out=None, stream=None):
    n = len(ws)
    wp = (C.c_void_p * n)(*[ptr(w) for w in ws])
    npp = (C.c_int * n)(*[int(v) for v in n_rows])
    bp = None
    if biases is not None:
        bp = (C.c_void_p * n)(*[ptr(b) for b in biases])
    return _check(_lib.frt_pack_weights_fp8(
        n, C.cast(wp, C.c_void_p), C.cast(npp, C.c_void_p), K,
        None if bp is None else C.cast(bp, C.c_void_p), layout, hd,
        ptr(w8_out), ptr(w_scale_out), ptr(bias_out), _stream(stream)),
        "frt_pack_weights_fp8")


def frt_gemm_workspace_size(M, N, K, epilogue=FRT_EPI_BF16) -> int:
    return int(_lib.frt_gemm_workspace_size(M, N, K, epilogue))


def frt_packed_fp8_gemm(M, N, K, x8, w8, act_scale, w_scale, bias, epilogue,
                        out, ldo, out_scale=None, workspace=None,
                        workspace_bytes=0, stream=None):
    return _check(_lib.frt_packed_fp8_gemm(
        M, N, K, ptr(x8), ptr(w8), ptr(act_scale), ptr(w_scale), ptr(bias),
        epilogue, ptr(out), ldo, ptr(out_scale), ptr(workspace),
        workspace_bytes, _stream(stream)), "frt_packed_fp8_gemm")


def frt_packed_fp8_gemm_noalloc(M, N, K, x8, w8, act_scale, w_scale, bias,
                                epilogue, out, ldo, out_scale=None,
                                stream=None):
    """frt_packed_fp8_gemm without a workspace argument: for callers that
    cannot allocate device memory (the library's static scratch is used)."""
    return _check(_lib.frt_packed_fp8_gemm_noalloc(
        M, N, K, ptr(x8), ptr(w8), ptr(act_scale), ptr(w_scale), ptr(bias),
        epilogue, ptr(out), ldo, ptr(out_scale), _stream(stream)),
        "frt_packed_fp8_gemm_noalloc")


def frt_packed_fp8_gemm_rope_kvcache(B, M, K, hq, hkv, hd, P, T, x8, w8,
                                     act_scale, w_scale, bias, rope, q_out,
                                     k_cache, v_cache, workspace=None,
                                     workspace_bytes=0, stream=None):
    return _check(_lib.frt_packed_fp8_gemm_rope_kvcache(
        B, M, K, hq, hkv, hd, P, T, ptr(x8), ptr(w8), ptr(act_scale),
        ptr(w_scale), ptr(bias), ptr(rope), ptr(q_out), ptr(k_cache),
        ptr(v_cache), ptr(workspace), workspace_bytes, _stream(stream)),
        "frt_packed_fp8_gemm_rope_kvcache")


def frt_build_rope_table(M, hd, P, theta, rope_out, stream=None):
    return _check(_lib.frt_build_rope_table(M, hd, P, float(theta),
                                            ptr(rope_out), _stream(stream)),
                  "frt_build_rope_table")


def frt_split_rope_kvcache(B, M, hq, hkv, hd, P, T, qkv, rope, q_out, k_cache,
                           v_cache, prefix_k=None, prefix_v=None,
                           prefix_T_src=0, prefix_interleave=0, stream=None):
    return _check(_lib.frt_split_rope_kvcache(
        B, M, hq, hkv, hd, P, T, ptr(qkv), ptr(rope), ptr(q_out),
        ptr(k_cache), ptr(v_cache), ptr(prefix_k), ptr(prefix_v),
        prefix_T_src, prefix_interleave, _stream(stream)),
        "frt_split_rope_kvcache")


def frt_prefix_copy_kv(B, hkv, hd, P, T, T_src, prefix_k, prefix_v,
                       interleave, k_cache, v_cache, stream=None):
    return _check(_lib.frt_prefix_copy_kv(
        B, hkv, hd, P, T, T_src, ptr(prefix_k), ptr(prefix_v), interleave,
        ptr(k_cache), ptr(v_cache), _stream(stream)), "frt_prefix_copy_kv")


def frt_geglu_quant_fp8(M, H, gu, ld_gu, out_scale, hid8, amax_out=None,
                        stream=None):
    return _check(_lib.frt_geglu_quant_fp8(
        M, H, ptr(gu), ld_gu, ptr(out_scale), ptr(hid8), ptr(amax_out),
        _stream(stream)), "frt_geglu_quant_fp8")


def frt_chain_workspace_size(desc: frt_chain_desc) -> int:
    return int(_lib.frt_chain_workspace_size(C.byref(desc)))


def frt_chain_layer(desc: frt_chain_desc, stream=None):
    return _check(_lib.frt_chain_layer(C.byref(desc), _stream(stream)),
                  "frt_chain_layer")


def frt_ffn_workspace_size(desc: frt_ffn_desc) -> int:
    return int(_lib.frt_ffn_workspace_size(C.byref(desc)))


def frt_ffn_layer(desc: frt_ffn_desc, stream=None):
    return _check(_lib.frt_ffn_layer(C.byref(desc), _stream(stream)), "frt_ffn_layer")


def frt_gelu_quant_fp8(M, H, u, ld_u, out_scale, hid8, amax_out=None, stream=None) -> None:
    """GELU + static e4m3 requant (the DiT FFN's middle step, unfused)."""
    _check(_lib.frt_gelu_quant_fp8(M, H, ptr(u), ld_u, ptr(out_scale), ptr(hid8),
                                   ptr(amax_out), _stream(stream)), "frt_gelu_quant_fp8")


def frt_quantize_fp8_static(rows, D, x, ldx, act_scale, x8_out, amax_out=None,
                            stream=None) -> None:
    """Static e4m3 quantize of a bf16 activation (the o_proj input)."""
    _check(_lib.frt_quantize_fp8_static(rows, D, ptr(x), ldx, ptr(act_scale), ptr(x8_out),
                                        ptr(amax_out), _stream(stream)),
           "frt_quantize_fp8_static")


def frt_ada_rms_tail(rows, D, eps, res, delta, gate, gate_row_stride, fin, fin_row_stride,
                     out, stream=None) -> None:
    """The stack's final AdaRMS tail: bf16(RMSnorm(res + gate*delta) *
    (1 + fin[0]) + fin[1])."""
    _check(_lib.frt_ada_rms_tail(rows, D, eps, ptr(res), ptr(delta), ptr(gate),
                                 gate_row_stride, ptr(fin), fin_row_stride, ptr(out),
                                 _stream(stream)),
           "frt_ada_rms_tail")


def frt_style_project(rows, K, N, cond, ld_cond, w, ldw, bias, style_out, ld_style,
                      fin_out=None, ld_fin=0, fin_col0=0, stream=None) -> None:
    """The stacked modulation projection: style = bf16(cond @ w.T + bias),
    and the fp32 values of columns >= fin_col0 into fin_out."""
    _check(_lib.frt_style_project(rows, K, N, ptr(cond), ld_cond, ptr(w), ldw, ptr(bias),
                                  ptr(style_out), ld_style, ptr(fin_out), ld_fin, fin_col0,
                                  _stream(stream)),
           "frt_style_project")


FRT_PLAN_INFO_LEN = 10
_PLAN_KEYS = ("swap", "pair", "split2", "cluster", "tile_rows", "tile_cols", "splits",
              "units", "grid", "k_blocks")


def frt_gemm_plan_info(M, N, K, epilogue=0) -> dict:
    """The GEMM schedule the library picks for this shape (host-side)."""
    buf = (C.c_int * FRT_PLAN_INFO_LEN)()
    _check(_lib.frt_gemm_plan_info(M, N, K, epilogue, buf, FRT_PLAN_INFO_LEN),
           "frt_gemm_plan_info")
    return dict(zip(_PLAN_KEYS, list(buf)))


def frt_peak_fp8_mma(ctas: int, iters: int,
                     operands: int = FRT_PEAK_OPERANDS_GAUSSIAN, stream=None) -> None:
    """Launch the dense FP8 tensor-core loop (the library's peak probe) on the
    operand codes `operands` names."""
    _check(_lib.frt_peak_fp8_mma(ctas, iters, operands, _stream(stream)), "frt_peak_fp8_mma")


def frt_peak_copy(src, dst, nbytes: int, stream=None) -> None:
    """Launch the device-to-device copy probe over `nbytes`."""
    _check(_lib.frt_peak_copy(ptr(src), ptr(dst), nbytes, _stream(stream)),
           "frt_peak_copy")


def frt_selftest_bounded_wait(timeout_us: int, stream=None) -> int:
    """Returns the status (FRT_ETIMEOUT expected); does not raise."""
    return _lib.frt_selftest_bounded_wait(timeout_us, _stream(stream))


def frt_selftest_gelu(x, y, n: int, stream=None) -> None:
    """y = the device GELU of x (n fp32 values each)."""
    _check(_lib.frt_selftest_gelu(ptr(x), ptr(y), n, _stream(stream)), "frt_selftest_gelu")


def raw_call(name: str, *args) -> int:
    """Call an entry point with already-marshalled arguments and return the
    status code without raising (used to test argument validation)."""
    return getattr(_lib, name)(*args)

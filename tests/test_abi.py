"""The C ABI without a GPU: the library loads, exports every entry point
include/frt.h declares, and rejects bad arguments on the host with the
documented status codes before touching the device."""

import ctypes as C
import os
import re

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def frt():
    from fp8_transformer_block_b200 import build
    build.build()
    from fp8_transformer_block_b200 import frt as mod
    return mod


def _declared():
    names = set()
    for fn in os.listdir(os.path.join(ROOT, "include")):
        if fn.endswith(".h"):
            src = open(os.path.join(ROOT, "include", fn)).read()
            src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
            names |= set(re.findall(r"\b(frt_[a-z0-9_]+)\s*\(", src))
    return names


def test_every_declared_symbol_is_exported(frt):
    declared = _declared()
    assert len(declared) >= 14
    lib = C.CDLL(frt.LIB_PATH)
    for name in sorted(declared):
        assert hasattr(lib, name), name
    assert declared == set(frt.EXPORTED)
    assert frt.frt_version() == 100


A16 = 0x10000  # a fake, 16-byte aligned, never dereferenced address


def _norm(frt, **kw):
    args = dict(mode=0, rows=4, D=512, eps=1e-6, res=A16, delta=A16,
                prev_gate=A16, gate_row_stride=0, weight=None, style=A16,
                style_row_stride=0, x=None, temb=None, chunks=0, table=None,
                shift_idx=0, scale_idx=0, act_scale=A16, x8_out=A16,
                gate_out=None, amax_out=None, stream=None)
    args.update(kw)
    return frt.raw_call("frt_ada_norm_quant_fp8", *args.values())


def test_producer_validation(frt):
    assert _norm(frt, D=7) == frt.FRT_ESHAPE
    assert _norm(frt, D=16392) == frt.FRT_ESHAPE
    assert _norm(frt, mode=5) == frt.FRT_EINVAL
    assert _norm(frt, res=None) == frt.FRT_EINVAL
    assert _norm(frt, delta=A16 + 2) == frt.FRT_EALIGN
    assert _norm(frt, gate_row_stride=12) == frt.FRT_EALIGN
    assert _norm(frt, style_row_stride=512) == frt.FRT_ESHAPE
    assert _norm(frt, mode=1, x=A16, temb=A16, table=A16, chunks=6,
                 shift_idx=6) == frt.FRT_EINVAL
    assert _norm(frt, rows=-1) == frt.FRT_ESHAPE
    assert "D must be" in (_norm(frt, D=7) and frt.last_error())
    # rows == 0 is a valid no-op (nothing launched)
    assert _norm(frt, rows=0) == frt.FRT_OK


def _gemm(frt, **kw):
    args = dict(M=64, N=640, K=512, x8=A16, w8=A16, act_scale=A16,
                w_scale=A16, bias=None, epilogue=0, out=A16, ldo=640,
                out_scale=None, workspace=None, workspace_bytes=0,
                stream=None)
    args.update(kw)
    return frt.raw_call("frt_packed_fp8_gemm", *args.values())


def test_gemm_validation(frt):
    assert _gemm(frt, N=33) == frt.FRT_ESHAPE
    assert _gemm(frt, K=520) == frt.FRT_ESHAPE
    assert _gemm(frt, x8=A16 + 8) == frt.FRT_EALIGN
    assert _gemm(frt, ldo=600) == frt.FRT_EALIGN
    assert _gemm(frt, epilogue=9) == frt.FRT_EINVAL
    assert _gemm(frt, epilogue=1, N=640, ldo=320) == frt.FRT_ESHAPE
    assert _gemm(frt, epilogue=1, N=512, ldo=256) == frt.FRT_EINVAL
    assert _gemm(frt, M=0) == frt.FRT_OK
    # few 128-row tiles over a long K split K through a global workspace
    need = frt.frt_gemm_workspace_size(200, 256, 16384)
    assert need > 0
    assert _gemm(frt, M=200, N=256, K=16384, ldo=256) == frt.FRT_EINVAL
    assert _gemm(frt, M=200, N=256, K=16384, ldo=256, workspace=A16 * 16,
                 workspace_bytes=need - 1) == frt.FRT_ERANGE
    # small M splits K inside thread-block clusters: no workspace
    assert frt.frt_gemm_workspace_size(50, 2560, 2048) == 0
    assert frt.frt_gemm_workspace_size(64, 2048, 16384) == 0
    assert frt.frt_gemm_workspace_size(8192, 9216, 3072) == 0


def _noalloc(frt, **kw):
    args = dict(M=200, N=256, K=16384, x8=A16, w8=A16, act_scale=A16,
                w_scale=A16, bias=None, epilogue=0, out=A16, ldo=256,
                out_scale=None, stream=None)
    args.update(kw)
    return frt.raw_call("frt_packed_fp8_gemm_noalloc", *args.values())


def test_noalloc_rejects_before_touching_the_device(frt):
    """Bad arguments to the no-allocation entry come back with the
    workspace entry's codes before any CUDA call: with no device here, a
    call that reached the scratch set-up or its counter memset would report
    FRT_ECUDA instead.  The shape (200 x 256 x 16384) splits K through the
    scratch, so a valid call would clear its counters."""
    assert frt.frt_gemm_workspace_size(200, 256, 16384) > 0
    assert _noalloc(frt, epilogue=9) == frt.FRT_EINVAL
    assert _noalloc(frt, out=A16 + 2) == frt.FRT_EALIGN
    assert _noalloc(frt, ldo=200) == frt.FRT_EALIGN
    assert _noalloc(frt, bias=A16 + 4) == frt.FRT_EALIGN
    assert _noalloc(frt, x8=A16 + 8) == frt.FRT_EALIGN
    assert _noalloc(frt, epilogue=2) == frt.FRT_EINVAL        # no out_scale
    assert _noalloc(frt, epilogue=1, N=512, ldo=256) == frt.FRT_EINVAL
    assert _noalloc(frt, K=520) == frt.FRT_ESHAPE
    assert _noalloc(frt, M=0) == frt.FRT_OK                    # nothing to do


def test_rope_and_cache_validation(frt):
    r = frt.raw_call("frt_packed_fp8_gemm_rope_kvcache", 1, 50, 2048, 8, 1,
                     256, 1000, 1024, A16, A16, A16, A16, None, A16, A16,
                     A16, A16, None, 0, None)
    assert r == frt.FRT_ERANGE                      # P + M > T
    r = frt.raw_call("frt_packed_fp8_gemm_rope_kvcache", 1, 50, 2048, 8, 1,
                     40, 0, 64, A16, A16, A16, A16, None, A16, A16, A16, A16,
                     None, 0, None)
    assert r == frt.FRT_ESHAPE                      # hd % 32 != 0
    r = frt.raw_call("frt_split_rope_kvcache", 1, 10, 2, 1, 12, 0, 10, A16,
                     A16, A16, A16, A16, None, None, 0, 0, None)
    assert r == frt.FRT_ESHAPE                      # hd % 8 != 0
    r = frt.raw_call("frt_prefix_copy_kv", 1, 1, 64, 900, 1024, 816, A16,
                     A16, 1, A16, A16, None)
    assert r == frt.FRT_ERANGE                      # P > T_src
    r = frt.raw_call("frt_geglu_quant_fp8", 4, 100, A16, 200, A16, A16, None,
                     None)
    assert r == frt.FRT_ESHAPE                      # H % 8 != 0
    r = frt.raw_call("frt_build_rope_table", 4, 7, 0, 1e4, A16, None)
    assert r == frt.FRT_ESHAPE


def test_pack_validation(frt):
    w = (C.c_void_p * 2)(A16, A16)
    n = (C.c_int * 2)(256, 128)
    r = frt.raw_call("frt_pack_weights_fp8", 2, C.cast(w, C.c_void_p),
                     C.cast(n, C.c_void_p), 64, None, 2, 0, A16, A16, None,
                     None)
    assert r == frt.FRT_ESHAPE        # gate/up blocks need equal siblings
    r = frt.raw_call("frt_pack_weights_fp8", 5, C.cast(w, C.c_void_p),
                     C.cast(n, C.c_void_p), 64, None, 0, 0, A16, A16, None,
                     None)
    assert r == frt.FRT_EINVAL
    r = frt.raw_call("frt_pack_weights_fp8", 2, C.cast(w, C.c_void_p),
                     C.cast(n, C.c_void_p), 40, None, 0, 0, A16, A16, None,
                     None)
    assert r == frt.FRT_ESHAPE        # K % 16


def test_chain_desc_layout_matches_header(frt):
    src = open(os.path.join(ROOT, "include", "frt.h")).read()
    body = src[src.index("typedef struct frt_chain_desc"):]
    body = body[:body.index("} frt_chain_desc;")]
    body = re.sub(r"/\*.*?\*/", "", body, flags=re.S)
    names = re.findall(r"\**\s*([A-Za-z_][A-Za-z0-9_]*)\s*(?=[,;])", body)
    assert names == [f for f, _ in frt.frt_chain_desc._fields_]


def test_ffn_desc_layout_matches_header(frt):
    src = open(os.path.join(ROOT, "include", "frt.h")).read()
    body = src[src.index("typedef struct frt_ffn_desc"):]
    body = body[:body.index("} frt_ffn_desc;")]
    body = re.sub(r"/\*.*?\*/", "", body, flags=re.S)
    names = re.findall(r"\**\s*([A-Za-z_][A-Za-z0-9_]*)\s*(?=[,;])", body)
    assert names == [f for f, _ in frt.frt_ffn_desc._fields_]


def test_output_side_validation(frt):
    q = frt.raw_call
    # static quantize: D % 8, ldx < D, misaligned input
    assert q("frt_quantize_fp8_static", 4, 12, A16, 12, A16, A16, None, None) == frt.FRT_ESHAPE
    assert q("frt_quantize_fp8_static", 4, 64, A16, 32, A16, A16, None, None) == frt.FRT_EALIGN
    assert q("frt_quantize_fp8_static", 4, 64, A16 + 8, 64, A16, A16, None, None) == \
        frt.FRT_EALIGN
    assert q("frt_quantize_fp8_static", 0, 64, A16, 64, A16, A16, None, None) == frt.FRT_OK
    # final tail: D beyond 8192, a gate stride below D, a missing fin
    assert q("frt_ada_rms_tail", 4, 8200, C.c_float(1e-6), A16, A16, A16, 0, A16, 8200, A16,
             None) == frt.FRT_ESHAPE
    assert q("frt_ada_rms_tail", 4, 64, C.c_float(1e-6), A16, A16, A16, 32, A16, 64, A16,
             None) == frt.FRT_EALIGN
    assert q("frt_ada_rms_tail", 4, 64, C.c_float(1e-6), A16, A16, A16, 0, None, 64, A16,
             None) == frt.FRT_EINVAL
    # GELU requant: H % 8
    assert q("frt_gelu_quant_fp8", 4, 12, A16, 16, A16, A16, None, None) == frt.FRT_ESHAPE
    # GEMM with the GELU epilogue needs out_scale
    assert q("frt_packed_fp8_gemm", 4, 256, 512, A16, A16, A16, A16, None,
             frt.FRT_EPI_GELU_E4M3, A16, 256, None, None, 0, None) == frt.FRT_EINVAL
    assert q("frt_packed_fp8_gemm", 4, 256, 512, A16, A16, A16, A16, None, 9, A16, 256,
             A16, None, 0, None) == frt.FRT_EINVAL
    # modulation projection: K % 8, a row stride below K, misalignment,
    # fin_col0 past N, a missing operand; no rows is a no-op
    sp = "frt_style_project"
    assert q(sp, 1, 12, 64, A16, 12, A16, 16, None, A16, 64, None, 0, 0, None) == frt.FRT_ESHAPE
    assert q(sp, 1, 64, 64, A16, 64, A16, 32, None, A16, 64, None, 0, 0, None) == frt.FRT_EALIGN
    assert q(sp, 1, 64, 64, A16, 66, A16, 64, None, A16, 64, None, 0, 0, None) == frt.FRT_EALIGN
    assert q(sp, 1, 64, 64, A16, 64, A16 + 8, 64, None, A16, 64, None, 0, 0, None) == \
        frt.FRT_EALIGN
    assert q(sp, 1, 64, 64, A16, 64, A16, 64, None, A16, 64, A16, 64, 65, None) == frt.FRT_ERANGE
    assert q(sp, 1, 64, 64, None, 64, A16, 64, None, A16, 64, None, 0, 0, None) == frt.FRT_EINVAL
    assert q(sp, 1, 64, 64, A16, 64, A16, 64, None, A16, 32, None, 0, 0, None) == frt.FRT_ESHAPE
    assert q(sp, 0, 64, 64, A16, 64, A16, 64, None, A16, 64, A16, 192, 0, None) == frt.FRT_OK
    # FFN half: no descriptor; the peak probe: no CTAs
    assert q("frt_ffn_layer", None, None) == frt.FRT_EINVAL
    assert q("frt_peak_fp8_mma", 0, 10, 0, None) == frt.FRT_EINVAL
    assert q("frt_peak_fp8_mma", 1, 10, 2, None) == frt.FRT_EINVAL
    assert q("frt_peak_copy", A16 + 4, A16, 64, None) == frt.FRT_EALIGN

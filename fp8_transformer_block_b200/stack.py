"""Whole AdaRMS layers except attention, as a sequence of the library's
C-ABI calls (impls/adarms_stack/fp8_chain.py `_make_run`, the layer loop
and the final tail).  Per layer l, on the current stream:

  frt_chain_layer           producer at norm slot 2l -> packed q/k/v GEMM
                            with the split + RoPE + KV write (+ prefix copy)
  frt_quantize_fp8_static   the attention output's static quantize, on the
                            attention stand-in att2 = q_out as [rows, hq*hd]
  frt_packed_fp8_gemm       the output projection -> dn_o
  frt_ffn_layer             producer at slot 2l + 1 (delta dn_o, gate g1)
                            -> gate/up GEMM with the GEGLU requant -> down
then frt_ada_rms_tail on (res, dn, g2).  With on-device modulation, each
step opens with frt_style_project: the conditioning row through the stacked
dense projection of all 2L + 1 norms (`_style_stack`), whose bf16 rows the
layers' producers read at norm slots 2l and 2l + 1 and whose final fp32
rows the tail reads.  Attention itself is outside this
library; the stand-in keeps every tensor's shape and the residual moving.
Argument marshalling only: every step runs in the CUDA library.
"""

from __future__ import annotations

import numpy as np
import torch

from . import frt
from . import runtime as rt


class AdaRmsLayerStack:
    def __init__(self, w, layers, fin, scales=None, x=None, modulation=None):
        """w: a "full" Workload; layers: synth.full_layer_inputs per layer;
        fin: fp32 [3, D] rows of the final norm; scales: per layer dict
        (a_qkv, a_o, a_gu, a_dn), or None to calibrate on the GPU from the
        quantizers' amax outputs over `x` (bf16 bits [rows, D]).
        modulation: None (the layers' own style rows and `fin`), or a dict
        of the stacked projection "w" (bf16 bits [(2L + 1) * 3D, D]), its
        fp32 "bias" and one fp32 conditioning row "cond" [1, D]: every step
        then computes all norms' rows on the device (`fin` is unused)."""
        assert w.hq * w.hd == w.D, "the attention stand-in needs hq * hd == D"
        self.w = w
        B, M, D, H = w.B, w.M, w.D, w.H
        rows = B * M
        self.rows = rows
        self.L = len(layers)
        dev = "cuda"
        self.res = torch.empty(rows, D, dtype=torch.bfloat16, device=dev)
        self.zero = torch.zeros(rows, D, dtype=torch.bfloat16, device=dev)
        self.x8 = rt.empty_u8(rows, D)
        self.q = rt.empty_bf16(B, M, w.hq, w.hd)
        self.g1 = rt.empty_bf16(rows, D)
        self.g2 = [rt.empty_bf16(rows, D) for _ in range(2)]
        self.o8 = rt.empty_u8(rows, D)
        self.dn_o = rt.empty_bf16(rows, D)
        self.dn = [rt.empty_bf16(rows, D) for _ in range(2)]
        self.x8f = rt.empty_u8(rows, D)
        self.hid8 = rt.empty_u8(rows, H)
        self.gu = rt.empty_bf16(rows, 2 * H)     # calibration only
        self.out = rt.empty_bf16(rows, D)
        self.rope = rt.empty_bf16(M, w.hd)
        frt.frt_build_rope_table(M, w.hd, w.P, w.theta, self.rope)
        self.mod = None
        if modulation is None:
            self.fin = rt.f32_dev(fin)
        else:
            n_norms = 2 * self.L + 1
            Nm = n_norms * 3 * D
            assert modulation["w"].shape == (Nm, D), "one (scale, shift, gate) block per norm"
            self.mod = {"w": rt.bf16_dev(modulation["w"]),
                        "bias": rt.f32_dev(modulation["bias"]),
                        "cond": rt.f32_dev(np.asarray(modulation["cond"], np.float32)
                                           .reshape(1, D)),
                        "N": Nm, "fin_col0": 3 * D * (n_norms - 1)}
            self.styles = rt.empty_bf16(1, Nm)
            self.fin = torch.empty(3, D, dtype=torch.float32, device=dev)
            self._project()
        self.lay = []
        for l, li in enumerate(layers):
            self.lay.append({
                "qkv": rt.pack(li["w"], layout=frt.FRT_PACK_QK_INTERLEAVE, hd=w.hd),
                "o": rt.pack([li["o"]]),
                "gu": rt.pack([li["mlp"]["gate"], li["mlp"]["up"]],
                              layout=frt.FRT_PACK_GATE_UP_BLOCKS),
                "dn": rt.pack([li["mlp"]["down"]]),
                "st_attn": (rt.bf16_dev(li["styles"][0:1]) if self.mod is None
                            else self.styles[:, 3 * D * (2 * l):3 * D * (2 * l + 1)]),
                "st_ffn": (rt.bf16_dev(li["styles"][1:2]) if self.mod is None
                           else self.styles[:, 3 * D * (2 * l + 1):3 * D * (2 * l + 2)]),
                "pk": rt.bf16_dev(li["prefix_k"]) if w.P else None,
                "pv": rt.bf16_dev(li["prefix_v"]) if w.P else None,
                "kc": torch.zeros(B, w.T, w.hkv, w.hd, dtype=torch.bfloat16, device=dev),
                "vc": torch.zeros(B, w.T, w.hkv, w.hd, dtype=torch.bfloat16, device=dev),
            })
        self.layers_host = layers
        N = (w.hq + 2 * w.hkv) * w.hd
        self.ws_bytes = max(frt.frt_chain_workspace_size(rt.chain_desc(
                                B=w.B, M=w.M, D=D, hq=w.hq, hkv=w.hkv, hd=w.hd,
                                norm_mode=frt.FRT_NORM_ADARMS,
                                flags=frt.FRT_CHAIN_FUSED_ROPE)),
                            frt.frt_gemm_workspace_size(rows, N, D),
                            frt.frt_gemm_workspace_size(rows, D, D),
                            frt.frt_gemm_workspace_size(rows, 2 * H, D, frt.FRT_EPI_GEGLU_E4M3),
                            frt.frt_gemm_workspace_size(rows, 2 * H, D),
                            frt.frt_gemm_workspace_size(rows, D, H))
        self.ws = rt.workspace(self.ws_bytes)
        if scales is None:
            scales = self.calibrate(x)
        self.scales = scales
        self.sdev = [{k: rt.scale_dev(v) for k, v in sc.items()} for sc in scales]
        self._build()

    # ------------------------------------------------------------------
    def _build(self):
        w, D, H, rows = self.w, self.w.D, self.w.H, self.rows
        self.cdesc, self.fdesc = [], []
        for l, ly in enumerate(self.lay):
            sc = self.sdev[l]
            self.cdesc.append(rt.chain_desc(
                B=w.B, M=w.M, D=D, hq=w.hq, hkv=w.hkv, hd=w.hd, P=w.P, T=w.T, eps=w.eps,
                norm_mode=frt.FRT_NORM_ADARMS, flags=frt.FRT_CHAIN_FUSED_ROPE,
                res=self.res, delta=self.zero if l == 0 else self.dn[(l - 1) % 2],
                prev_gate=self.zero if l == 0 else self.g2[(l - 1) % 2],
                gate_row_stride=0 if l == 0 else D, style=ly["st_attn"], style_row_stride=0,
                gate_out=self.g1, act_scale=sc["a_qkv"], x8=self.x8, w8=ly["qkv"].w8,
                w_scale=ly["qkv"].w_scale, bias=None, rope=self.rope, q_out=self.q,
                k_cache=ly["kc"], v_cache=ly["vc"], prefix_k=ly["pk"], prefix_v=ly["pv"],
                prefix_T_src=w.P, prefix_interleave=1, workspace=self.ws,
                workspace_bytes=self.ws_bytes))
            self.fdesc.append(rt.ffn_desc(
                rows=rows, D=D, H=H, eps=w.eps, res=self.res, delta=self.dn_o,
                prev_gate=self.g1, gate_row_stride=D, norm_weight=None, style=ly["st_ffn"],
                style_row_stride=0, gate_out=self.g2[l % 2], act_scale=sc["a_gu"],
                x8=self.x8f, w8_gu=ly["gu"].w8, w_scale_gu=ly["gu"].w_scale, bias_gu=None,
                hid_scale=sc["a_dn"], hid8=self.hid8, w8_dn=ly["dn"].w8,
                w_scale_dn=ly["dn"].w_scale, bias_dn=None, out=self.dn[l % 2],
                workspace=self.ws, workspace_bytes=self.ws_bytes))

    def _out_project(self, l, scale):
        D, rows = self.w.D, self.rows
        frt.frt_quantize_fp8_static(rows, D, self.q, D, scale, self.o8)
        ly = self.lay[l]
        frt.frt_packed_fp8_gemm(rows, D, D, self.o8, ly["o"].w8, scale, ly["o"].w_scale, None,
                                frt.FRT_EPI_BF16, self.dn_o, D, None, self.ws, self.ws_bytes)

    def _project(self):
        m, D = self.mod, self.w.D
        frt.frt_style_project(1, D, m["N"], m["cond"], D, m["w"], D, m["bias"], self.styles,
                              m["N"], self.fin, 3 * D, m["fin_col0"])

    def set_cond(self, cond):
        """Load a new conditioning row (fp32 [1, D]) for the next steps."""
        self.mod["cond"].copy_(torch.from_numpy(np.asarray(cond, np.float32)
                                                .reshape(1, self.w.D)))

    def step(self):
        """One pass of the whole stack on the current stream."""
        if self.mod is not None:
            self._project()
        for l in range(self.L):
            frt.frt_chain_layer(self.cdesc[l])
            self._out_project(l, self.sdev[l]["a_o"])
            frt.frt_ffn_layer(self.fdesc[l])
        last = (self.L - 1) % 2
        frt.frt_ada_rms_tail(self.rows, self.w.D, self.w.eps, self.res, self.dn[last],
                             self.g2[last], self.w.D, self.fin, self.w.D, self.out)

    def load(self, x):
        """Set the stack's input rows (bf16 bits [rows, D])."""
        self.res.copy_(rt.bf16_dev(x))

    # ------------------------------------------------------------------
    def calibrate(self, x):
        """Static scales per site, layer by layer in order: each quantizer
        first runs with scale 1 and an amax output, its scale is amax / 448,
        then the site runs with it to produce the next site's input.  The
        fused GEGLU epilogue has no amax output: its site is calibrated on
        the unfused GEMM + GEGLU kernel."""
        w, D, H, rows = self.w, self.w.D, self.w.H, self.rows
        one = rt.scale_dev(1.0)
        am = torch.zeros(1, dtype=torch.float32, device="cuda")
        junk = rt.empty_u8(rows, max(D, H))

        def amax_of(fn):
            am.zero_()
            fn(am)
            torch.cuda.synchronize()
            return max(float(am.item()) / 448.0, 1e-8)

        self.load(x)
        scales = []
        delta, gate, gs = self.zero, self.zero, 0
        for l, ly in enumerate(self.lay):
            sc = {}

            def producer(style, d, g, stride, s, out8, gout, amax=None):
                frt.frt_ada_norm_quant_fp8(frt.FRT_NORM_ADARMS, rows, D, w.eps, self.res, d, g,
                                           stride, None, style, 0, None, None, 0, None, 0, 0,
                                           s, out8, gout, amax)
            snap = self.res.clone()
            sc["a_qkv"] = amax_of(lambda a: producer(ly["st_attn"], delta, gate, gs, one,
                                                     junk, None, a))
            self.res.copy_(snap)
            producer(ly["st_attn"], delta, gate, gs, rt.scale_dev(sc["a_qkv"]), self.x8, self.g1)
            frt.frt_packed_fp8_gemm_rope_kvcache(
                w.B, w.M, D, w.hq, w.hkv, w.hd, w.P, w.T, self.x8, ly["qkv"].w8,
                rt.scale_dev(sc["a_qkv"]), ly["qkv"].w_scale, None, self.rope, self.q,
                ly["kc"], ly["vc"], self.ws, self.ws_bytes)
            sc["a_o"] = amax_of(lambda a: frt.frt_quantize_fp8_static(rows, D, self.q, D, one,
                                                                      junk, a))
            self._out_project(l, rt.scale_dev(sc["a_o"]))
            snap = self.res.clone()
            sc["a_gu"] = amax_of(lambda a: producer(ly["st_ffn"], self.dn_o, self.g1, D, one,
                                                    junk, None, a))
            self.res.copy_(snap)
            producer(ly["st_ffn"], self.dn_o, self.g1, D, rt.scale_dev(sc["a_gu"]), self.x8f,
                     self.g2[l % 2])
            gu_cat = rt.pack([self.layers_host[l]["mlp"]["gate"],
                              self.layers_host[l]["mlp"]["up"]])
            frt.frt_packed_fp8_gemm(rows, 2 * H, D, self.x8f, gu_cat.w8,
                                    rt.scale_dev(sc["a_gu"]), gu_cat.w_scale, None,
                                    frt.FRT_EPI_BF16, self.gu, 2 * H, None, self.ws,
                                    self.ws_bytes)
            sc["a_dn"] = amax_of(lambda a: frt.frt_geglu_quant_fp8(rows, H, self.gu, 2 * H, one,
                                                                   junk, a))
            frt.frt_geglu_quant_fp8(rows, H, self.gu, 2 * H, rt.scale_dev(sc["a_dn"]), self.hid8)
            frt.frt_packed_fp8_gemm(rows, D, H, self.hid8, ly["dn"].w8, rt.scale_dev(sc["a_dn"]),
                                    ly["dn"].w_scale, None, frt.FRT_EPI_BF16, self.dn[l % 2], D,
                                    None, self.ws, self.ws_bytes)
            torch.cuda.synchronize()
            scales.append(sc)
            delta, gate, gs = self.dn[l % 2], self.g2[l % 2], D
        return scales

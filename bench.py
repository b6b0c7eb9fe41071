"""Benchmark of the fused static-FP8 attention-input chain on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--config NAME]
                    [--impl reference] [--repeats R] [--no-subconfigs]

One step = one pass of the chain over one batch of the workload, all inputs
resident in HBM.  The default workload is the video-DiT block form (B=2 x
4096 tokens, D=3072, the per-token-table LayerNorm producer, the packed
q/k/v FP8 GEMM (N=9216, bias) with the split + RoPE + KV write in its
epilogue): the two launches frt_chain_layer makes.  The same JSON line
carries one record per other configuration under "configs": the tiny
AdaRMS layer, the action-expert layer (50 tokens behind an 816-token
prefix), the gate/up MLP (producer, gate/up GEMM with the GEGLU requant,
down GEMM) and the 18-layer AdaRMS stack at every row count of its sweep.
Other workloads (--config): video_dit_ffn, adarms_layer18[_live],
style_stack18, style_vla18, adarms_stack18:M.

Timing: W untimed warm-up steps, then R timed regions of exactly K steps,
each bracketed by a barrier and a synchronize, K steps replayed back to
back from CUDA graphs over independent copies of the workload (inputs
larger than L2), CUDA events on the launching stream, max over ranks; the
value comes from the median region, the spread is reported.  Each kernel is
timed alone the same way.  `e2e` runs the step through the entry points
with pinned host buffers copied in and the outputs copied back, timed on
the host clock per step.  With N > 1 (torchrun) every rank runs an
independent replica on its own batch (no data-path collective); value =
all ranks' tokens / max rank time.

--impl reference times the CPU oracle (the reference arm: plain C, OpenMP
over rows) on the host cores on the same workload.
"""

from __future__ import annotations

import argparse
import hashlib
import json
import os
import statistics
import sys
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = ("chain tokens/s & µs/layer; GEMM % FP8 tensor peak, "
          "producer % HBM GB/s")
DEFAULT_CONFIG = "video_dit"
FLUSH_BYTES = 256 << 20
FALLBACK_HBM_GBS = 6650.0
FALLBACK_BF16_TFLOPS = 1590.0
FP8_PER_BF16 = 2.0  # nominal dense ratio (4.5 / 2.25 PFLOP/s)

# DRAM bytes (read + write) per launch of the dominant kernel from the ncu
# captures summarised under profiles/, keyed by (workload, kernel); a value
# counts only while the hash of the kernel's sources matches the one the
# counters were taken on (else the line reports traffic null).
KERNEL_SOURCES = {
    "gemm": ("gemm.cu", "frt_sm100.cuh", "frt_common.cuh"),
    "producer": ("producer.cu", "frt_common.cuh", "frt_sm100.cuh", "frt_prefix.cuh"),
    "prefix_copy": ("rope.cu", "frt_prefix.cuh"),
    "style": ("style.cu", "frt_common.cuh"),
}
NCU_TRAFFIC = {
    ("vla_action_expert", "gemm_rope_kv"): (5_427_968, "61e0f042b56e0b91"),
    ("video_dit", "gemm_rope_kv"): (58_575_616 + 110_788_352, "61e0f042b56e0b91"),
    ("gateup_mlp", "gemm_gateup_geglu"): (69_275_648 + 4_848_128, "61e0f042b56e0b91"),
    ("style_stack18", "style_project"): (58_446_336 + 5_888, "41d4aa014b38bc81"),
    ("style_vla18", "style_project"): (932_082_432 + 1_793_024, "41d4aa014b38bc81"),
}


def _src_hash(kernel_name):
    kind = ("gemm" if kernel_name.startswith("gemm") else
            "producer" if kernel_name == "producer" else
            "style" if kernel_name == "style_project" else "prefix_copy")
    h = hashlib.sha256()
    for f in KERNEL_SOURCES[kind]:
        with open(os.path.join(ROOT, "fp8_transformer_block_b200", "csrc", f),
                  "rb") as fh:
            h.update(fh.read())
    return h.hexdigest()[:16]


def max_over_ranks(ms, torch, dist, world, device):
    """The slowest rank's time: every rank's device-timed milliseconds,
    all-reduced with MAX (the identity on one rank)."""
    t = torch.tensor([float(ms)], dtype=torch.float64, device=device)
    if world > 1:
        dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def job_throughput(tokens_per_rank, steps, max_ms, world):
    """Whole-job tokens/s: every rank's tokens over the slowest rank's time
    (replicas: each rank runs its own copy of the workload)."""
    return world * tokens_per_rank * steps / (max_ms / 1e3)


def own_peaks(torch, frt):
    """The library's own probes (frt_peak_fp8_mma, frt_peak_copy): best of
    three timed launches each, CUDA events on the current stream."""
    sms = torch.cuda.get_device_properties(0).multi_processor_count
    iters = 20000
    flops = 2.0 * 128 * 256 * 128 * iters * sms

    def best(fn, n=3):
        fn()
        torch.cuda.synchronize()
        out = []
        for _ in range(n):
            a = torch.cuda.Event(enable_timing=True)
            b = torch.cuda.Event(enable_timing=True)
            a.record()
            fn()
            b.record()
            torch.cuda.synchronize()
            out.append(a.elapsed_time(b) * 1e-3)
        return min(out)
    t_mma = best(lambda: frt.frt_peak_fp8_mma(sms, iters, frt.FRT_PEAK_OPERANDS_GAUSSIAN))
    t_mma_lt = best(lambda: frt.frt_peak_fp8_mma(sms, iters, frt.FRT_PEAK_OPERANDS_LOW_TOGGLE))
    nbytes = 1 << 30
    src = torch.empty(nbytes, dtype=torch.uint8, device="cuda")
    dst = torch.empty_like(src)
    src.fill_(1)
    t_cp = best(lambda: frt.frt_peak_copy(src, dst, nbytes))
    del src, dst
    assert frt.frt_device_status(True) == frt.FRT_OK
    return {"fp8_dense_tflops": round(flops / t_mma / 1e12, 1),
            "fp8_dense_tflops_low_toggle": round(flops / t_mma_lt / 1e12, 1),
            "hbm_copy_gbs": round(2.0 * nbytes / t_cp / 1e9, 1),
            "method": f"tcgen05 e4m3 MMA loop, {sms} CTAs x {4 * iters} "
                      "M128xN256xK32 MMAs from shared memory on the e4m3 codes of "
                      "N(0, 100^2) values (like statically quantised operands; "
                      "fp8_dense_tflops) and on low-toggle non-negative codes "
                      "(fp8_dense_tflops_low_toggle: less power, higher clock); "
                      "1 GiB device copy (read + write bytes); best of 3",
            "datasheet": {"fp8_dense_tflops": 4500.0, "hbm_gbs": 7700.0}}


def _peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(p) as fh:
            d = json.load(fh)
        return (float(d["hbm_gbs"]), float(d["bf16_tflops"]),
                float(d.get("bf16_tflops_sustained", d["bf16_tflops"])),
                "measured")
    except (OSError, KeyError, ValueError):
        return (FALLBACK_HBM_GBS, FALLBACK_BF16_TFLOPS, 1400.0, "fallback")


# ---------------------------------------------------------------- clocks ----

class ClockSampler:
    """NVML samples of the SM clock and the clock-event (throttle) reasons,
    taken every millisecond by a thread while the timed region runs (the
    region is a few milliseconds long, too short for nvidia-smi's loop)."""

    NAMES = ("hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown",
             "sw_power_cap")

    def __init__(self, gpu_uuid: str | None):
        self.handle = None
        self.samples: list[tuple[float, int]] = []
        self.thread = None
        self.stop_flag = False
        try:
            import pynvml
            pynvml.nvmlInit()
            self.nv = pynvml
            self.handle = pynvml.nvmlDeviceGetHandleByUUID(gpu_uuid)
            self.max_mhz = float(pynvml.nvmlDeviceGetMaxClockInfo(
                self.handle, pynvml.NVML_CLOCK_SM))
            self.bits = dict(zip(self.NAMES, (
                pynvml.nvmlClocksEventReasonHwSlowdown,
                pynvml.nvmlClocksEventReasonHwThermalSlowdown,
                pynvml.nvmlClocksEventReasonSwThermalSlowdown,
                pynvml.nvmlClocksEventReasonSwPowerCap)))
        except Exception as exc:  # noqa: BLE001
            self.handle = None
            self.why = f"no NVML: {exc}"[:80]

    def _sample(self):
        nv = self.nv
        sm = nv.nvmlDeviceGetClockInfo(self.handle, nv.NVML_CLOCK_SM)
        rs = nv.nvmlDeviceGetCurrentClocksEventReasons(self.handle)
        self.samples.append((float(sm), int(rs)))

    def _loop(self):
        while not self.stop_flag:
            try:
                self._sample()
            except Exception:  # noqa: BLE001
                return
            time.sleep(0.001)

    def start(self):
        if self.handle is None:
            return
        import threading
        self.stop_flag = False
        self.thread = threading.Thread(target=self._loop, daemon=True)
        self.thread.start()

    def stop(self):
        if self.handle is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": [self.why],
                    "samples": 0}
        self.stop_flag = True
        self.thread.join(timeout=5)
        if not self.samples:   # the region ended before the first sample
            self._sample()
        reasons = sorted(n for n, b in self.bits.items()
                         if any(r & b for _, r in self.samples))
        return {"sm_mhz": statistics.median(sm for sm, _ in self.samples),
                "sm_max_mhz": self.max_mhz, "reasons": reasons,
                "samples": len(self.samples), "source": "nvml, 1 ms"}


# --------------------------------------------------------------- runners ----

class Kern:
    """One kind of launch in a step, with its algorithmic work per launch."""

    def __init__(self, name, bound, algo_bytes=0.0, flops=0.0, per_step=1):
        self.name, self.bound = name, bound
        self.algo_bytes, self.flops = float(algo_bytes), float(flops)
        self.per_step = per_step


class ChainRunner:
    """Attention-input chain layers: prefix copy, producer (AdaRMS or
    per-token-table LayerNorm), packed q/k/v GEMM with the fused split +
    RoPE + KV epilogue.  With layers > 1 the residual is carried and layer
    l+1 takes layer l's q_out (viewed [rows, D]) as delta and its gate_out
    as gate; layer 0 sees delta = gate = 0."""

    def __init__(self, w, torch, frt, rt, synth):
        self.w, self.torch, self.frt, self.rt = w, torch, frt, rt
        self.dit = w.kind == "dit"
        self.L = w.layers
        B, M, D = w.B, w.M, w.D
        self.rows = rows = B * M
        N = w.N
        self.layers = []
        for l in range(self.L):
            if self.L > 1:
                li = synth.stack_layer_inputs(w, l)
                ws, bs, style = li["w"], li["b"], li["style"]
                pkh, pvh = li["prefix_k"], li["prefix_v"]
            else:
                ws, bs = synth.qkv_weights(w.hq, w.hkv, w.hd, D, w.seed,
                                           bias=w.bias)
                style, pkh, pvh = None, None, None
                if w.P > 0:
                    pkh, pvh = synth.prefix_cache(B, w.hkv, max(1024, w.P),
                                                  w.hd, w.seed)
            layout = (frt.FRT_PACK_CONCAT if self.dit
                      else frt.FRT_PACK_QK_INTERLEAVE)
            pk = rt.pack(ws, bs if w.bias else None, layout=layout, hd=w.hd)
            self.layers.append({
                "pk": pk,
                "kc": torch.zeros(B, w.T, w.hkv, w.hd, dtype=torch.bfloat16,
                                  device="cuda"),
                "vc": torch.zeros(B, w.T, w.hkv, w.hd, dtype=torch.bfloat16,
                                  device="cuda"),
                "style": None if style is None else rt.bf16_dev(style),
                "pkd": None if pkh is None else rt.bf16_dev(pkh),
                "pvd": None if pvh is None else rt.bf16_dev(pvh),
                "T_src": 0 if pkh is None else int(pkh.shape[2])})
        self.rope = rt.empty_bf16(M, w.hd)
        frt.frt_build_rope_table(M, w.hd, w.P, w.theta, self.rope)
        if self.dit:
            inp = synth.dit_inputs(rows, D, w.seed)
            self.x = rt.bf16_dev(inp["x"])
            self.temb = rt.bf16_dev(inp["temb"])
            self.table = rt.f32_dev(inp["table"])
            self.host_in = {"x": inp["x"], "temb": inp["temb"]}
        else:
            inp = synth.adarms_inputs(rows, D, w.seed, outliers=w.outliers)
            self.res0 = rt.bf16_dev(inp["res"])
            self.res = self.res0.clone()
            self.delta = rt.bf16_dev(inp["delta"])
            self.gate = rt.bf16_dev(inp["prev_gate"])
            self.style1 = rt.bf16_dev(inp["style"])
            self.zero = torch.zeros(rows, D, dtype=torch.bfloat16, device="cuda")
            self.gate_out = [rt.empty_bf16(rows, D) for _ in range(2)]
            self.host_in = {k: inp[k] for k in
                            ("res", "delta", "prev_gate", "style")}
        self.x8 = rt.empty_u8(rows, D)
        self.q = [rt.empty_bf16(B, M, w.hq, w.hd) for _ in range(2)]
        # the chain's own workspace size (its GEMM's split-K, or the counters
        # of the producer-in-the-grid form at small M)
        self.ws_bytes = frt.frt_chain_workspace_size(rt.chain_desc(
            B=B, M=M, D=D, hq=w.hq, hkv=w.hkv, hd=w.hd,
            norm_mode=(frt.FRT_NORM_LAYERNORM_TABLE if self.dit else frt.FRT_NORM_ADARMS),
            flags=frt.FRT_CHAIN_FUSED_ROPE))
        self.ws = rt.workspace(self.ws_bytes)
        self.calibrate(synth)
        ks = []
        if self.layers[0]["pkd"] is not None:
            ks.append(Kern("prefix_copy", "hbm",
                           4.0 * B * w.P * w.hkv * w.hd * 2, per_step=self.L))
        prod = (rows * D * (2 + 2 * 2 + 1) if self.dit
                else rows * D * (4 + 2 + 1 + 2) + 4 * D * 2)
        ks.append(Kern("producer", "hbm", prod, per_step=self.L))
        gbytes = (N * D + rows * D + M * w.hd * 2 + rows * N * 2
                  + (N * 2 if w.bias else 0))
        gflops = 2.0 * rows * N * D
        ks.append(Kern("gemm_rope_kv",
                       "tensor" if gflops / gbytes > 560 else "hbm",
                       gbytes, gflops, per_step=self.L))
        self.kerns = ks
        self.tokens = rows
        self.launches = 2 * self.L   # frt_chain_layer: producer(+prefix), GEMM
        self._build_descs()

    # ----------------------------------------------------------------------
    def _inputs(self, l):
        """(delta, gate, gate_stride, style) of layer l."""
        if self.L == 1:
            return self.delta, self.gate, 0, self.style1
        if l == 0:
            return self.zero, self.zero, 0, self.layers[0]["style"]
        return (self.q[(l - 1) % 2], self.gate_out[(l - 1) % 2], self.w.D,
                self.layers[l]["style"])

    def _producer(self, l, scale, amax=None):
        frt, w = self.frt, self.w
        if self.dit:
            frt.frt_ada_norm_quant_fp8(
                frt.FRT_NORM_LAYERNORM_TABLE, self.rows, w.D, w.eps, None,
                None, None, 0, None, None, 0, self.x, self.temb, 6,
                self.table, 0, 1, scale, self.x8, None, amax)
        else:
            d, g, gs, st = self._inputs(l)
            frt.frt_ada_norm_quant_fp8(
                frt.FRT_NORM_ADARMS, self.rows, w.D, w.eps, self.res, d, g,
                gs, None, st, 0, None, None, 0, None, 0, 0, scale, self.x8,
                self.gate_out[l % 2], amax)

    def _gemm(self, l, scale):
        w, lay = self.w, self.layers[l]
        self.frt.frt_packed_fp8_gemm_rope_kvcache(
            w.B, w.M, w.D, w.hq, w.hkv, w.hd, w.P, w.T, self.x8,
            lay["pk"].w8, scale, lay["pk"].w_scale, lay["pk"].bias,
            self.rope, self.q[l % 2], lay["kc"], lay["vc"], self.ws,
            self.ws_bytes)

    def _prefix(self, l):
        w, lay = self.w, self.layers[l]
        if lay["pkd"] is not None:
            self.frt.frt_prefix_copy_kv(w.B, w.hkv, w.hd, w.P, w.T,
                                        lay["T_src"], lay["pkd"], lay["pvd"],
                                        1, lay["kc"], lay["vc"])

    def calibrate(self, synth):
        """Static activation scale per layer = amax / 448 of the producer's
        output on the calibration batch (seed + 500), from the GPU
        producer's amax output; stacked layers are calibrated in order, each
        on the output of the already-calibrated layers before it."""
        torch, frt, rt, w = self.torch, self.frt, self.rt, self.w
        am = torch.zeros(1, dtype=torch.float32, device="cuda")
        one = rt.scale_dev(1.0)
        self.act = []
        if self.dit:
            cal = synth.dit_inputs(w.cal_rows, w.D, w.seed + synth.CAL_OFFSET,
                                   with_table=False)
            x8 = rt.empty_u8(w.cal_rows, w.D)
            frt.frt_ada_norm_quant_fp8(
                frt.FRT_NORM_LAYERNORM_TABLE, w.cal_rows, w.D, w.eps, None,
                None, None, 0, None, None, 0, rt.bf16_dev(cal["x"]),
                rt.bf16_dev(cal["temb"]), 6, self.table, 0, 1, one, x8, None,
                am)
            self.act = [rt.scale_dev(float(am.item()) / 448.0)]
            return
        if self.L == 1:
            cal = synth.adarms_inputs(w.cal_rows, w.D,
                                      w.seed + synth.CAL_OFFSET,
                                      outliers=w.outliers)
            x8 = rt.empty_u8(w.cal_rows, w.D)
            frt.frt_ada_norm_quant_fp8(
                frt.FRT_NORM_ADARMS, w.cal_rows, w.D, w.eps,
                rt.bf16_dev(cal["res"]), rt.bf16_dev(cal["delta"]),
                rt.bf16_dev(cal["prev_gate"]), 0, None,
                rt.bf16_dev(cal["style"]), 0, None, None, 0, None, 0, 0, one,
                x8, None, am)
            self.act = [rt.scale_dev(float(am.item()) / 448.0)]
            return
        cal = synth.adarms_inputs(self.rows, w.D, w.seed + synth.CAL_OFFSET)
        self.res.copy_(rt.bf16_dev(cal["res"]))
        snap = torch.empty_like(self.res)
        for l in range(self.L):
            snap.copy_(self.res)
            am.zero_()
            self._producer(l, one, am)
            a = rt.scale_dev(max(float(am.item()), 1e-30) / 448.0)
            self.act.append(a)
            self.res.copy_(snap)
            self._producer(l, a)
            self._gemm(l, a)
        self.res.copy_(self.res0)

    # ----------------------------------------------------------------------
    def _build_descs(self):
        frt, rt, w = self.frt, self.rt, self.w
        self.descs = []
        for l, lay in enumerate(self.layers):
            d, g, gs, st = self._inputs(l) if not self.dit else (None,) * 4
            self.descs.append(rt.chain_desc(
                B=w.B, M=w.M, D=w.D, hq=w.hq, hkv=w.hkv, hd=w.hd, P=w.P,
                T=w.T, eps=w.eps,
                norm_mode=(frt.FRT_NORM_LAYERNORM_TABLE if self.dit
                           else frt.FRT_NORM_ADARMS),
                flags=frt.FRT_CHAIN_FUSED_ROPE,
                res=None if self.dit else self.res, delta=d, prev_gate=g,
                gate_row_stride=gs or 0, style=st, style_row_stride=0,
                gate_out=None if self.dit else self.gate_out[l % 2],
                x=self.x if self.dit else None,
                temb=self.temb if self.dit else None,
                chunks=6 if self.dit else 0,
                table=self.table if self.dit else None, shift_idx=0,
                scale_idx=1, act_scale=self.act[l if not self.dit else 0],
                x8=self.x8, w8=lay["pk"].w8, w_scale=lay["pk"].w_scale,
                bias=lay["pk"].bias, rope=self.rope, q_out=self.q[l % 2],
                k_cache=lay["kc"], v_cache=lay["vc"], prefix_k=lay["pkd"],
                prefix_v=lay["pvd"], prefix_T_src=lay["T_src"],
                prefix_interleave=1, workspace=self.ws,
                workspace_bytes=self.ws_bytes))

    def reset(self):
        """Restore the state a step mutates (the residual); untimed."""
        if not self.dit:
            self.res.copy_(self.res0)

    def step(self):
        """One step through the public entry point: frt_chain_layer per
        layer (producer + prefix in one launch, then the fused GEMM)."""
        for d in self.descs:
            self.frt.frt_chain_layer(d)

    def kernel_calls(self):
        """(Kern, call) pairs timing each kernel alone through the C ABI."""
        kc = []
        by = {k.name: k for k in self.kerns}
        if "prefix_copy" in by:
            kc.append((by["prefix_copy"], lambda: self._prefix(0)))
        kc.append((by["producer"],
                   lambda: self._producer(0, self.act[0])))
        kc.append((by["gemm_rope_kv"], lambda: self._gemm(0, self.act[0])))
        return kc

    def aux_calls(self):
        """Kernels timed beside the step (not part of it), video-DiT form:
        the standalone split + RoPE + KV write on a bf16 q/k/v buffer (the
        unfused page form; HBM-bound, rows * (4N + 2hd) bytes per launch) and
        the same GEMM with the plain bf16 epilogue (its time against the
        fused one prices the split/RoPE/KV epilogue)."""
        if not self.dit:
            return []
        frt, w, lay = self.frt, self.w, self.layers[0]
        N = w.N
        if not hasattr(self, "qkv_bf16"):
            self.qkv_bf16 = self.rt.empty_bf16(self.rows, N)
            frt.frt_packed_fp8_gemm(self.rows, N, w.D, self.x8, lay["pk"].w8, self.act[0],
                                    lay["pk"].w_scale, lay["pk"].bias, frt.FRT_EPI_BF16,
                                    self.qkv_bf16, N, None, self.ws, self.ws_bytes)

        def split():
            frt.frt_split_rope_kvcache(w.B, w.M, w.hq, w.hkv, w.hd, w.P, w.T, self.qkv_bf16,
                                       self.rope, self.q[0], lay["kc"], lay["vc"])

        def gemm_plain():
            frt.frt_packed_fp8_gemm(self.rows, N, w.D, self.x8, lay["pk"].w8, self.act[0],
                                    lay["pk"].w_scale, lay["pk"].bias, frt.FRT_EPI_BF16,
                                    self.qkv_bf16, N, None, self.ws, self.ws_bytes)
        rows = self.rows
        return [
            (Kern("split_rope_kv", "hbm", rows * (4.0 * N + 2 * w.hd)), split),
            (Kern("gemm_bf16", "tensor", N * w.D + rows * w.D + rows * N * 2 + N * 2,
                  2.0 * rows * N * w.D), gemm_plain),
        ]

    # ---------------------------------------------------------------- e2e --
    def e2e_setup(self):
        """Host-buffer form of the step: the step's token inputs sit back to
        back in one pinned host buffer and one device arena (the chain's
        input tensors become views of it), so a step copies them in with one
        host->device copy; the residual, the last layer's q and gate outputs
        follow them in the arena and come back with one device->host copy,
        the new K/V cache rows with one copy each.  The prefix K/V stays in
        device memory, like the weights: it is the host model's own cache,
        which the chain gathers from on the device."""
        torch, w, L = self.torch, self.w, self.L
        lq = (L - 1) % 2
        # (name, device tensor, host array or None, setter)
        ins = []
        if self.dit:
            ins.append(("x", self.x, self.host_in["x"],
                        lambda t: setattr(self, "x", t)))
            ins.append(("temb", self.temb, self.host_in["temb"],
                        lambda t: setattr(self, "temb", t)))
        else:
            ins.append(("delta", self.delta, self.host_in["delta"],
                        lambda t: setattr(self, "delta", t)))
            ins.append(("prev_gate", self.gate, self.host_in["prev_gate"],
                        lambda t: setattr(self, "gate", t)))
            ins.append(("style", self.style1, self.host_in["style"],
                        lambda t: setattr(self, "style1", t)))
        outs = []
        if not self.dit:   # the residual is both an input and an output
            ins.append(("res", self.res, self.host_in["res"],
                        lambda t: setattr(self, "res", t)))
        outs.append(("q", self.q[lq], lambda t: self.q.__setitem__(lq, t)))
        if not self.dit:
            outs.append(("gate", self.gate_out[lq],
                         lambda t: self.gate_out.__setitem__(lq, t)))
        offs, n = {}, 0
        for name, t, *_ in ins + outs:
            offs[name] = n
            n += (t.numel() + 127) // 128 * 128   # 256-byte aligned slices
        arena = torch.empty(n, dtype=torch.int16, device="cuda")
        pin = torch.empty(n, dtype=torch.int16).pin_memory()
        for name, t, host, setter in ins:
            v = arena[offs[name]:offs[name] + t.numel()].view(t.dtype).view(t.shape)
            v.copy_(t)
            pin[offs[name]:offs[name] + t.numel()].copy_(
                torch.from_numpy(np.ascontiguousarray(host).view(np.int16).reshape(-1)))
            setter(v)
        for name, t, setter in outs:
            v = arena[offs[name]:offs[name] + t.numel()].view(t.dtype).view(t.shape)
            setter(v)
        self._build_descs()
        self.arena, self.pin_arena = arena, pin
        self.in_elems = offs["res"] + self.res.numel() if not self.dit else offs["q"]
        self.out_lo = offs["res"] if not self.dit else offs["q"]
        self.out_hi = n
        self.pin_back = torch.empty(n - self.out_lo, dtype=torch.int16).pin_memory()
        self.kv_out = []
        for lay in self.layers:
            for c in ("kc", "vc"):
                src = lay[c][:, w.P:w.P + w.M]
                self.kv_out.append((src, torch.empty(src.shape, dtype=src.dtype).pin_memory()))
        self.h2d_bytes = 2 * self.in_elems
        self.d2h_bytes = (2 * (self.out_hi - self.out_lo) +
                          sum(t.numel() * t.element_size() for _, t in self.kv_out))

    def e2e_step(self):
        self.arena[:self.in_elems].copy_(self.pin_arena[:self.in_elems], non_blocking=True)
        self.step()
        self.pin_back.copy_(self.arena[self.out_lo:self.out_hi], non_blocking=True)
        for src, dst in self.kv_out:
            dst.copy_(src, non_blocking=True)


class MlpRunner:
    """Gate/up sibling MLP: AdaRMS producer -> packed gate/up FP8 GEMM with
    the GEGLU + static requant epilogue -> down-projection FP8 GEMM."""

    def __init__(self, w, torch, frt, rt, synth):
        self.w, self.torch, self.frt, self.rt = w, torch, frt, rt
        M, D, H = w.M, w.D, w.H
        self.rows = M
        mw = synth.mlp_weights(D, H, w.seed)
        self.gu = rt.pack([mw["gate"], mw["up"]],
                          layout=frt.FRT_PACK_GATE_UP_BLOCKS)
        self.dn = rt.pack([mw["down"]])
        inp = synth.adarms_inputs(M, D, w.seed)
        self.host_in = {k: inp[k] for k in ("res", "delta", "prev_gate", "style")}
        self.res0 = rt.bf16_dev(inp["res"])
        self.res = self.res0.clone()
        self.delta = rt.bf16_dev(inp["delta"])
        self.gate = rt.bf16_dev(inp["prev_gate"])
        self.style = rt.bf16_dev(inp["style"])
        self.gate_out = rt.empty_bf16(M, D)
        self.x8 = rt.empty_u8(M, D)
        self.hid8 = rt.empty_u8(M, H)
        self.out = rt.empty_bf16(M, D)
        self.ws1 = frt.frt_gemm_workspace_size(M, 2 * H, D, frt.FRT_EPI_GEGLU_E4M3)
        self.ws2 = frt.frt_gemm_workspace_size(M, D, H)
        self.wsp1, self.wsp2 = rt.workspace(self.ws1), rt.workspace(self.ws2)
        self.calibrate(synth, mw)
        self.kerns = [
            Kern("producer", "hbm", M * D * 9 + 4 * D * 2),
            Kern("gemm_gateup_geglu", "tensor", 2 * H * D + M * D + M * H,
                 2.0 * M * 2 * H * D),
            Kern("gemm_down", "tensor", D * H + M * H + M * D * 2,
                 2.0 * M * D * H),
        ]
        self.tokens = M
        self.launches = 3

    def calibrate(self, synth, mw):
        torch, frt, rt, w = self.torch, self.frt, self.rt, self.w
        C, D, H = w.cal_rows, w.D, w.H
        cal = synth.adarms_inputs(C, D, w.seed + synth.CAL_OFFSET)
        am = torch.zeros(1, dtype=torch.float32, device="cuda")
        x8 = rt.empty_u8(C, D)
        res = rt.bf16_dev(cal["res"])
        frt.frt_ada_norm_quant_fp8(
            frt.FRT_NORM_ADARMS, C, D, w.eps, res, rt.bf16_dev(cal["delta"]),
            rt.bf16_dev(cal["prev_gate"]), 0, None, rt.bf16_dev(cal["style"]),
            0, None, None, 0, None, 0, 0, rt.scale_dev(1.0), x8, None, am)
        self.a_gu = rt.scale_dev(float(am.item()) / 448.0)
        res = rt.bf16_dev(cal["res"])
        frt.frt_ada_norm_quant_fp8(
            frt.FRT_NORM_ADARMS, C, D, w.eps, res, rt.bf16_dev(cal["delta"]),
            rt.bf16_dev(cal["prev_gate"]), 0, None, rt.bf16_dev(cal["style"]),
            0, None, None, 0, None, 0, 0, self.a_gu, x8, None, None)
        cat = rt.pack([mw["gate"], mw["up"]])
        gu = rt.empty_bf16(C, 2 * H)
        wsb = frt.frt_gemm_workspace_size(C, 2 * H, D)
        frt.frt_packed_fp8_gemm(C, 2 * H, D, x8, cat.w8, self.a_gu,
                                cat.w_scale, None, frt.FRT_EPI_BF16, gu,
                                2 * H, None, rt.workspace(wsb), wsb)
        am.zero_()
        hid = rt.empty_u8(C, H)
        frt.frt_geglu_quant_fp8(C, H, gu, 2 * H, rt.scale_dev(1.0), hid, am)
        self.a_dn = rt.scale_dev(float(am.item()) / 448.0)
        del cat, gu

    def reset(self):
        self.res.copy_(self.res0)

    def _producer(self):
        frt, w = self.frt, self.w
        frt.frt_ada_norm_quant_fp8(
            frt.FRT_NORM_ADARMS, w.M, w.D, w.eps, self.res, self.delta,
            self.gate, 0, None, self.style, 0, None, None, 0, None, 0, 0,
            self.a_gu, self.x8, self.gate_out, None)

    def _gateup(self):
        frt, w = self.frt, self.w
        frt.frt_packed_fp8_gemm(w.M, 2 * w.H, w.D, self.x8, self.gu.w8,
                                self.a_gu, self.gu.w_scale, None,
                                frt.FRT_EPI_GEGLU_E4M3, self.hid8, w.H,
                                self.a_dn, self.wsp1, self.ws1)

    def _down(self):
        frt, w = self.frt, self.w
        frt.frt_packed_fp8_gemm(w.M, w.D, w.H, self.hid8, self.dn.w8,
                                self.a_dn, self.dn.w_scale, None,
                                frt.FRT_EPI_BF16, self.out, w.D, None,
                                self.wsp2, self.ws2)

    def step(self):
        self._producer()
        self._gateup()
        self._down()

    def kernel_calls(self):
        return list(zip(self.kerns, (self._producer, self._gateup,
                                     self._down)))

    def e2e_setup(self):
        torch = self.torch
        self.pin_in = {k: torch.from_numpy(v.view(np.int16)).pin_memory()
                       for k, v in self.host_in.items()}
        self.dev_in = {"res": self.res, "delta": self.delta,
                       "prev_gate": self.gate, "style": self.style}
        self.dev_out = {"out": self.out, "res": self.res,
                        "gate": self.gate_out}
        self.pin_out = {k: torch.empty(v.shape, dtype=v.dtype).pin_memory()
                        for k, v in self.dev_out.items()}
        self.h2d_bytes = sum(t.numel() * 2 for t in self.pin_in.values())
        self.d2h_bytes = sum(t.numel() * 2 for t in self.pin_out.values())

    def e2e_step(self):
        for k, t in self.pin_in.items():
            d = self.dev_in[k]
            d.view(self.torch.int16).copy_(t.view(d.shape), non_blocking=True)
        self.step()
        for k, t in self.pin_out.items():
            t.copy_(self.dev_out[k], non_blocking=True)


class FullRunner:
    """Whole AdaRMS layers except attention (fp8_transformer_block_b200.stack):
    per layer the q/k/v chain layer, the output projection's static quantize
    and GEMM on the attention stand-in, the FFN half; then the final tail."""

    def __init__(self, w, torch, frt, rt, synth):
        from fp8_transformer_block_b200 import stack
        self.w, self.torch, self.frt, self.rt = w, torch, frt, rt
        L, rows, D, H = w.layers, w.rows, w.D, w.H
        self.L = L
        lays = [synth.full_layer_inputs(w, l) for l in range(L)]
        fin = synth.final_norm_rows(w)
        cal = synth.adarms_inputs(rows, D, w.seed + synth.CAL_OFFSET)["res"]
        mod = None
        if w.live:
            m = synth.modulation_inputs(1, D, 2 * L + 1, w.seed)
            mod = {"w": m["w"], "bias": m["bias"], "cond": m["cond"]}
            self.cond_host = m["cond"]
        self.st = stack.AdaRmsLayerStack(w, lays, fin, x=cal, modulation=mod)
        self.x_host = synth.adarms_inputs(rows, D, w.seed)["res"]
        self.x0 = rt.bf16_dev(self.x_host)
        self.st.res.copy_(self.x0)
        N = (w.hq + 2 * w.hkv) * w.hd
        gb = N * D + rows * D + w.M * w.hd * 2 + rows * N * 2
        gf = 2.0 * rows * N * D
        self.kerns = [
            Kern("prefix_copy", "hbm", 4.0 * w.B * w.P * w.hkv * w.hd * 2, per_step=L),
            Kern("producer", "hbm", rows * D * 11 + 6 * D, per_step=2 * L),
            Kern("gemm_rope_kv", "tensor" if gf / gb > 560 else "hbm", gb, gf, per_step=L),
            Kern("quantize_o", "hbm", rows * D * 3, per_step=L),
            Kern("gemm_o", "tensor" if rows > 560 else "hbm", D * D + rows * D * 3,
                 2.0 * rows * D * D, per_step=L),
            Kern("gemm_gateup_geglu", "tensor" if rows > 560 else "hbm",
                 2 * H * D + rows * D + rows * H, 2.0 * rows * 2 * H * D, per_step=L),
            Kern("gemm_down", "tensor" if rows > 560 else "hbm",
                 D * H + rows * H + rows * D * 2, 2.0 * rows * D * H, per_step=L),
            Kern("tail", "hbm", rows * D * 8 + 8 * D, per_step=1),
        ]
        self.tokens = rows
        self.launches = 7 * L + 1
        if w.live:
            Nm = (2 * L + 1) * 3 * D
            self.kerns.insert(0, Kern("style_project", "hbm",
                                      Nm * D * 2 + Nm * 4 + D * 4 + Nm * 2 + 12 * D))
            self.launches += 1

    def footprint(self):
        st, seen, total = self.st, set(), 0
        ts = [v for v in vars(st).values() if isinstance(v, self.torch.Tensor)]
        for v in vars(st).values():
            if isinstance(v, list):
                ts += [x for x in v if isinstance(x, self.torch.Tensor)]
            elif isinstance(v, dict):
                ts += [x for x in v.values() if isinstance(x, self.torch.Tensor)]
        for ly in st.lay:
            for v in ly.values():
                if isinstance(v, self.torch.Tensor):
                    ts.append(v)
                elif hasattr(v, "w8"):
                    ts.append(v.w8)
        for t in ts:
            if t.data_ptr() not in seen:
                seen.add(t.data_ptr())
                total += t.numel() * t.element_size()
        return total

    def reset(self):
        self.st.res.copy_(self.x0)

    def step(self):
        self.st.step()

    def kernel_calls(self):
        st, w, frt = self.st, self.w, self.frt
        ly, sc = st.lay[0], st.sdev[0]
        D, H, rows = w.D, w.H, st.rows

        def prefix():
            frt.frt_prefix_copy_kv(w.B, w.hkv, w.hd, w.P, w.T, w.P, ly["pk"], ly["pv"], 1,
                                   ly["kc"], ly["vc"])

        def producer():
            frt.frt_ada_norm_quant_fp8(frt.FRT_NORM_ADARMS, rows, D, w.eps, st.res, st.dn_o,
                                       st.g1, D, None, ly["st_ffn"], 0, None, None, 0, None,
                                       0, 0, sc["a_gu"], st.x8f, st.g2[0], None)

        def gemm_rope():
            frt.frt_packed_fp8_gemm_rope_kvcache(
                w.B, w.M, D, w.hq, w.hkv, w.hd, w.P, w.T, st.x8, ly["qkv"].w8, sc["a_qkv"],
                ly["qkv"].w_scale, None, st.rope, st.q, ly["kc"], ly["vc"], st.ws, st.ws_bytes)

        def quant():
            frt.frt_quantize_fp8_static(rows, D, st.q, D, sc["a_o"], st.o8)

        def gemm_o():
            frt.frt_packed_fp8_gemm(rows, D, D, st.o8, ly["o"].w8, sc["a_o"], ly["o"].w_scale,
                                    None, frt.FRT_EPI_BF16, st.dn_o, D, None, st.ws,
                                    st.ws_bytes)

        def gemm_gu():
            frt.frt_packed_fp8_gemm(rows, 2 * H, D, st.x8f, ly["gu"].w8, sc["a_gu"],
                                    ly["gu"].w_scale, None, frt.FRT_EPI_GEGLU_E4M3, st.hid8, H,
                                    sc["a_dn"], st.ws, st.ws_bytes)

        def gemm_dn():
            frt.frt_packed_fp8_gemm(rows, D, H, st.hid8, ly["dn"].w8, sc["a_dn"],
                                    ly["dn"].w_scale, None, frt.FRT_EPI_BF16, st.dn[0], D,
                                    None, st.ws, st.ws_bytes)

        def tail():
            frt.frt_ada_rms_tail(rows, D, w.eps, st.res, st.dn[0], st.g2[0], D, st.fin, D,
                                 st.out)
        calls = [prefix, producer, gemm_rope, quant, gemm_o, gemm_gu, gemm_dn, tail]
        if w.live:
            calls.insert(0, st._project)
        return list(zip(self.kerns, calls))

    # ---------------------------------------------------------------- e2e --
    def e2e_setup(self):
        """The step's input (the rows entering the stack) in a pinned buffer
        and a device arena the stack reads directly (one host->device copy);
        the output rows and each layer's new K/V rows come back with one copy
        each.  Every layer's prefix K/V stays in device memory, like the
        weights (the host model's own cache)."""
        torch, st, w = self.torch, self.st, self.w
        ins = [("x", st.res, self.x_host)]
        if w.live:   # the step's conditioning row (fp32) comes in with it
            ins.append(("cond", st.mod["cond"], self.cond_host))
        offs, n = {}, 0
        for name, t, _ in ins:
            offs[name] = n
            n += (t.numel() * t.element_size() // 2 + 127) // 128 * 128
        arena = torch.empty(n, dtype=torch.int16, device="cuda")
        pin = torch.empty(n, dtype=torch.int16).pin_memory()
        views = {}
        for name, t, host in ins:
            m = t.numel() * t.element_size() // 2
            v = arena[offs[name]:offs[name] + m].view(t.dtype).view(t.shape)
            v.copy_(t)
            pin[offs[name]:offs[name] + m].copy_(
                torch.from_numpy(np.ascontiguousarray(host).view(np.int16).reshape(-1)))
            views[name] = v
        st.res = views["x"]
        if w.live:
            st.mod["cond"] = views["cond"]
        st._build()
        self.arena, self.pin_arena, self.n_in = arena, pin, n
        self.outs = [(st.out, torch.empty(st.out.shape, dtype=st.out.dtype).pin_memory())]
        for ly in st.lay:
            for c in ("kc", "vc"):
                src = ly[c][:, w.P:w.P + w.M]
                self.outs.append((src, torch.empty(src.shape, dtype=src.dtype).pin_memory()))
        self.h2d_bytes = 2 * n
        self.d2h_bytes = sum(t.numel() * t.element_size() for t, _ in self.outs)

    def e2e_step(self):
        self.arena.copy_(self.pin_arena, non_blocking=True)
        self.step()
        for src, dst in self.outs:
            dst.copy_(src, non_blocking=True)


class DitFfnRunner:
    """The video-DiT block's FFN half: the per-token-table producer at the
    FFN site (chunks 3/4) -> up projection with the GELU + static requant
    epilogue -> down projection, both with bias."""

    def __init__(self, w, torch, frt, rt, synth):
        self.w, self.torch, self.frt, self.rt = w, torch, frt, rt
        rows, D, H = w.rows, w.D, w.H
        self.rows = rows
        fw = synth.dit_ffn_weights(D, H, w.seed)
        self.up = rt.pack([fw["up"]], [fw["up_b"]])
        self.dn = rt.pack([fw["dn"]], [fw["dn_b"]])
        inp = synth.dit_inputs(rows, D, w.seed)
        self.host_in = {"x": inp["x"], "temb": inp["temb"]}
        self.x = rt.bf16_dev(inp["x"])
        self.temb = rt.bf16_dev(inp["temb"])
        self.table = rt.f32_dev(inp["table"])
        self.x8 = rt.empty_u8(rows, D)
        self.hid8 = rt.empty_u8(rows, H)
        self.ff = rt.empty_bf16(rows, D)
        self.ws1 = frt.frt_gemm_workspace_size(rows, H, D, frt.FRT_EPI_GELU_E4M3)
        self.ws2 = frt.frt_gemm_workspace_size(rows, D, H)
        self.wsp1, self.wsp2 = rt.workspace(self.ws1), rt.workspace(self.ws2)
        self.calibrate(synth, fw)
        self.kerns = [
            Kern("producer", "hbm", rows * D * (2 + 2 * 2 + 1)),
            Kern("gemm_up_gelu", "tensor", H * D + rows * D + rows * H + 2 * H,
                 2.0 * rows * H * D),
            Kern("gemm_down", "tensor", D * H + rows * H + rows * D * 2 + 2 * D,
                 2.0 * rows * D * H),
        ]
        self.tokens = rows
        self.launches = 3

    def calibrate(self, synth, fw):
        """a_in from the producer's amax and a_hid from the unfused GELU
        kernel's amax, on a seeded calibration batch (seed + 500)."""
        torch, frt, rt, w = self.torch, self.frt, self.rt, self.w
        C, D, H = w.cal_rows, w.D, w.H
        cal = synth.dit_inputs(C, D, w.seed + synth.CAL_OFFSET)
        am = torch.zeros(1, dtype=torch.float32, device="cuda")
        x8 = rt.empty_u8(C, D)
        frt.frt_ada_norm_quant_fp8(frt.FRT_NORM_LAYERNORM_TABLE, C, D, w.eps, None, None, None,
                                   0, None, None, 0, rt.bf16_dev(cal["x"]),
                                   rt.bf16_dev(cal["temb"]), 6, rt.f32_dev(cal["table"]), 3, 4,
                                   rt.scale_dev(1.0), x8, None, am)
        torch.cuda.synchronize()
        self.a_in = max(float(am.item()) / 448.0, 1e-8)
        s_in = rt.scale_dev(self.a_in)
        frt.frt_ada_norm_quant_fp8(frt.FRT_NORM_LAYERNORM_TABLE, C, D, w.eps, None, None, None,
                                   0, None, None, 0, rt.bf16_dev(cal["x"]),
                                   rt.bf16_dev(cal["temb"]), 6, rt.f32_dev(cal["table"]), 3, 4,
                                   s_in, x8, None, None)
        u = rt.empty_bf16(C, H)
        wsb = frt.frt_gemm_workspace_size(C, H, D)
        frt.frt_packed_fp8_gemm(C, H, D, x8, self.up.w8, s_in, self.up.w_scale, self.up.bias,
                                frt.FRT_EPI_BF16, u, H, None, rt.workspace(wsb), wsb)
        am.zero_()
        frt.frt_gelu_quant_fp8(C, H, u, H, rt.scale_dev(1.0), rt.empty_u8(C, H), am)
        torch.cuda.synchronize()
        self.a_hid = max(float(am.item()) / 448.0, 1e-8)
        self.s_in, self.s_hid = s_in, rt.scale_dev(self.a_hid)

    def _producer(self):
        w, frt = self.w, self.frt
        frt.frt_ada_norm_quant_fp8(frt.FRT_NORM_LAYERNORM_TABLE, self.rows, w.D, w.eps, None,
                                   None, None, 0, None, None, 0, self.x, self.temb, 6,
                                   self.table, 3, 4, self.s_in, self.x8, None, None)

    def _up(self):
        w, frt = self.w, self.frt
        frt.frt_packed_fp8_gemm(self.rows, w.H, w.D, self.x8, self.up.w8, self.s_in,
                                self.up.w_scale, self.up.bias, frt.FRT_EPI_GELU_E4M3,
                                self.hid8, w.H, self.s_hid, self.wsp1, self.ws1)

    def _down(self):
        w, frt = self.w, self.frt
        frt.frt_packed_fp8_gemm(self.rows, w.D, w.H, self.hid8, self.dn.w8, self.s_hid,
                                self.dn.w_scale, self.dn.bias, frt.FRT_EPI_BF16, self.ff, w.D,
                                None, self.wsp2, self.ws2)

    def reset(self):
        pass

    def step(self):
        self._producer()
        self._up()
        self._down()

    def kernel_calls(self):
        return list(zip(self.kerns, (self._producer, self._up, self._down)))

    def e2e_setup(self):
        torch = self.torch
        self.pin_in = {k: torch.from_numpy(np.ascontiguousarray(v).view(np.int16)).pin_memory()
                       for k, v in self.host_in.items()}
        self.dev_in = {"x": self.x, "temb": self.temb}
        self.pin_out = torch.empty(self.ff.shape, dtype=self.ff.dtype).pin_memory()
        self.h2d_bytes = sum(t.numel() * 2 for t in self.pin_in.values())
        self.d2h_bytes = self.ff.numel() * 2

    def e2e_step(self):
        for k, t in self.pin_in.items():
            d = self.dev_in[k]
            d.view(self.torch.int16).copy_(t.view(d.shape), non_blocking=True)
        self.step()
        self.pin_out.copy_(self.ff, non_blocking=True)


class StyleRunner:
    """Modulation projection: the conditioning rows into the (scale, shift,
    gate) rows of all 2L + 1 norms (bf16), the final norm's rows also in
    fp32: one launch, bound by reading the stacked bf16 weights."""

    dtype = "bf16 weights/fp32 accumulate"

    def __init__(self, w, torch, frt, rt, synth):
        self.w, self.torch, self.frt, self.rt = w, torch, frt, rt
        self.n_norms = 2 * w.layers + 1
        rows, K, N = w.rows, w.D, w.N
        inp = synth.modulation_inputs(rows, K, self.n_norms, w.seed)
        self.host_in = {"cond": inp["cond"]}
        self.cond = rt.f32_dev(inp["cond"])
        self.wm = rt.bf16_dev(inp["w"])
        self.bias = rt.f32_dev(inp["bias"])
        del inp
        self.fin_col0 = 3 * K * (self.n_norms - 1)
        self.style = rt.empty_bf16(rows, N)
        self.fin = torch.empty((rows, N - self.fin_col0), dtype=torch.float32,
                               device="cuda")
        self.kerns = [Kern("style_project", "hbm",
                           N * K * 2 + N * 4 + rows * K * 4 + rows * N * 2
                           + rows * (N - self.fin_col0) * 4)]
        self.tokens = rows
        self.launches = 1

    def reset(self):
        pass

    def _project(self):
        w = self.w
        self.frt.frt_style_project(w.rows, w.D, w.N, self.cond, w.D, self.wm, w.D,
                                   self.bias, self.style, w.N, self.fin,
                                   w.N - self.fin_col0, self.fin_col0)

    def step(self):
        self._project()

    def kernel_calls(self):
        return list(zip(self.kerns, (self._project,)))

    def e2e_setup(self):
        torch = self.torch
        self.pin_cond = torch.from_numpy(self.host_in["cond"]).pin_memory()
        self.pin_style = torch.empty(self.style.shape, dtype=self.style.dtype).pin_memory()
        self.pin_fin = torch.empty(self.fin.shape, dtype=self.fin.dtype).pin_memory()
        self.h2d_bytes = self.pin_cond.numel() * 4
        self.d2h_bytes = self.pin_style.numel() * 2 + self.pin_fin.numel() * 4

    def e2e_step(self):
        self.cond.copy_(self.pin_cond, non_blocking=True)
        self.step()
        self.pin_style.copy_(self.style, non_blocking=True)
        self.pin_fin.copy_(self.fin, non_blocking=True)


def make_runner(name, torch, frt, rt, synth):
    base, _, m = name.partition(":")
    w = synth.WORKLOADS[base]
    if m:
        w = w.with_M(int(m))
    if w.kind == "mlp":
        return MlpRunner(w, torch, frt, rt, synth)
    if w.kind == "full":
        return FullRunner(w, torch, frt, rt, synth)
    if w.kind == "ditffn":
        return DitFfnRunner(w, torch, frt, rt, synth)
    if w.kind == "style":
        return StyleRunner(w, torch, frt, rt, synth)
    return ChainRunner(w, torch, frt, rt, synth)


def workload_text(w):
    if w.kind == "style":
        return (f"{w.name}: {w.rows} conditioning row(s) of D={w.D} into the "
                f"(scale, shift, gate) rows of {2 * w.layers + 1} norms "
                f"(N={w.N}, bf16 weights {w.N * w.D * 2 / 2**20:.0f} MiB, fp32 bias); "
                "tokens = conditioning rows")
    if w.kind == "ditffn":
        return (f"{w.name}: B={w.B} M={w.M} D={w.D} FFN {w.H}: table producer at the FFN "
                "site (chunks 3/4) + up GEMM with GELU requant + down GEMM, both biased")
    if w.kind == "full":
        return (f"{w.name}: B={w.B} M={w.M} D={w.D} Hq={w.hq}x{w.hd} Hkv={w.hkv}x{w.hd} "
                f"P={w.P} T={w.T} FFN {w.H}, {w.layers} whole layers except attention "
                "(q/k/v chain, output projection on the attention stand-in q_out, "
                "FFN half) + final tail"
                + (", every step opening with the modulation projection of one "
                   f"conditioning row into all {2 * w.layers + 1} norms' rows"
                   if w.live else ""))
    if w.kind == "mlp":
        return (f"{w.name}: M={w.M} D={w.D} gate/up {w.H} each (packed "
                f"N={2 * w.H}) + GEGLU requant + down [{w.D},{w.H}]")
    s = (f"{w.name}: B={w.B} M={w.M} D={w.D} Hq={w.hq}x{w.hd} "
         f"Hkv={w.hkv}x{w.hd} N={w.N} P={w.P} T={w.T}")
    if w.layers > 1:
        s += f", {w.layers} layers, residual carried"
    return s + (" bias" if w.bias else "")


# ------------------------------------------------------- CPU oracle arm ----

def oracle_sampler(name, synth, rows_cap=None):
    """Closure running the CPU oracle on a bounded sample of the workload:
    all tokens when that is cheap, else a seeded subset of rows (rows are
    independent through the whole chain).  Returns (fn, tokens, text)."""
    import oracle
    base, _, m = name.partition(":")
    w = synth.WORKLOADS[base]
    if m:
        w = w.with_M(int(m))
    rng = np.random.default_rng(7)
    if w.kind == "mlp":
        n = rows_cap or 256
        sel = np.sort(rng.choice(w.M, size=min(n, w.M), replace=False))
        mw = synth.mlp_weights(w.D, w.H, w.seed)
        gu_p = oracle.pack_weights_fp8([mw["gate"], mw["up"]])
        dn_p = oracle.pack_weights_fp8([mw["down"]])
        inp = synth.adarms_inputs(w.M, w.D, w.seed)
        sub = {k: (v[sel] if v.shape[0] == w.M else v) for k, v in inp.items()}

        def fn():
            pr = oracle.ada_rms_norm_quant(sub["res"], sub["delta"],
                                           sub["prev_gate"], sub["style"],
                                           0.01, eps=w.eps)
            gu = oracle.fp8_gemm(pr["x8"], gu_p["w8"], 0.01, gu_p["w_scale"])
            hid, _ = oracle.geglu_quant(gu, 0.05)
            oracle.fp8_gemm(hid, dn_p["w8"], 0.05, dn_p["w_scale"])
        return fn, len(sel), f"{len(sel)} of {w.M} rows, full MLP per row"

    if w.kind == "style":
        # columns are independent: a leading block of output columns, for
        # every conditioning row; tokens scale with the share of columns
        n_norms = 2 * w.layers + 1
        inp = synth.modulation_inputs(w.rows, w.D, n_norms, w.seed)
        n = w.N if rows_cap is None else max(1, min(w.N, rows_cap))
        if rows_cap is None:
            n = min(w.N, max(3 * w.D, (1 << 27) // (w.D * w.rows)))
        wsub, bsub = inp["w"][:n].copy(), inp["bias"][:n].copy()
        cond = inp["cond"]
        del inp

        def fn():
            oracle.style_project(cond, wsub, bsub, fin_col0=0)
        return fn, w.rows * n / w.N, f"{n} of {w.N} output columns, all conditioning rows"

    if w.kind == "ditffn":
        n = rows_cap or 32
        sel = np.sort(rng.choice(w.rows, size=min(n, w.rows), replace=False))
        fw = synth.dit_ffn_weights(w.D, w.H, w.seed)
        up = oracle.pack_weights_fp8([fw["up"]], [fw["up_b"]])
        dnp = oracle.pack_weights_fp8([fw["dn"]], [fw["dn_b"]])
        inp = synth.dit_inputs(w.rows, w.D, w.seed)
        x, temb, table = inp["x"][sel], inp["temb"][sel], inp["table"]

        def fn():
            oracle.dit_ffn(x, temb, table, up, dnp, 0.02, a_hid=0.01, eps=w.eps)
        return fn, len(sel), f"{len(sel)} of {w.rows} rows, the FFN half per row"

    if w.kind == "full":
        # rows stay independent through the whole loop (the attention
        # stand-in is the row's own q): a leading block of rows, the stack
        # at its own positions, static scales fixed
        n = w.rows if rows_cap is None else max(1, min(w.rows, rows_cap))
        wl = w.with_M(n)
        lays = [synth.full_layer_inputs(w, l) for l in range(w.layers)]
        ol = [{"qkv": oracle.pack_weights_fp8(li["w"], layout=1, hd=w.hd),
               "o": oracle.pack_weights_fp8([li["o"]]),
               "gu": oracle.pack_weights_fp8([li["mlp"]["gate"], li["mlp"]["up"]]),
               "dn": oracle.pack_weights_fp8([li["mlp"]["down"]]),
               "styles": li["styles"], "prefix_k": li["prefix_k"],
               "prefix_v": li["prefix_v"]} for li in lays]
        fin = synth.final_norm_rows(w)
        x = synth.adarms_inputs(w.rows, w.D, w.seed)["res"][:n]
        dims = {"B": 1, "M": n, "D": w.D, "hq": w.hq, "hkv": w.hkv, "hd": w.hd,
                "P": w.P, "T": wl.T, "H": w.H, "theta": w.theta}
        fixed = [{"a_qkv": 0.01, "a_o": 0.01, "a_gu": 0.01, "a_dn": 0.05}] * w.layers
        mod = synth.modulation_inputs(1, w.D, 2 * w.layers + 1, w.seed) if w.live else None

        def fn():
            f, layers = fin, ol
            if mod is not None:
                st, f = oracle.style_project(mod["cond"], mod["w"], mod["bias"],
                                             fin_col0=3 * w.D * 2 * w.layers)
                f = f.reshape(3, w.D)
                layers = [dict(li, styles=st[0, 6 * w.D * l:6 * w.D * (l + 1)].reshape(2, 3 * w.D))
                          for l, li in enumerate(ol)]
            oracle.adarms_layer_stack(x, layers, f, dims, scales=fixed, eps=w.eps)
        return fn, n, (f"{n} of {w.rows} rows, {w.layers} whole layers except attention "
                       "+ tail" + (", with the modulation projection" if w.live else ""))

    L = w.layers
    rows = w.rows
    n = rows if rows_cap is None else min(rows, rows_cap)
    if rows > 256 and rows_cap is None:
        n = 64 if w.kind == "dit" else 256
    sel = np.sort(rng.choice(rows, size=n, replace=False)) if n < rows \
        else np.arange(rows)
    layers = []
    for l in range(L):
        if L > 1:
            li = synth.stack_layer_inputs(w, l)
            ws, bs, style = li["w"], li["b"], li["style"]
            pkh, pvh = li["prefix_k"], li["prefix_v"]
        else:
            ws, bs = synth.qkv_weights(w.hq, w.hkv, w.hd, w.D, w.seed,
                                       bias=w.bias)
            style, pkh, pvh = None, None, None
            if w.P > 0:
                pkh, pvh = synth.prefix_cache(w.B, w.hkv, max(1024, w.P),
                                              w.hd, w.seed)
        pk = oracle.pack_weights_fp8(ws, bs, layout=0 if w.kind == "dit" else 1,
                                     hd=w.hd)
        layers.append((pk, style, pkh, pvh))
    rope = oracle.rope_table(w.M, w.hd, w.P, w.theta)
    kc0 = np.zeros((w.B, w.T, w.hkv, w.hd), np.uint16)
    if w.kind == "dit":
        inp = synth.dit_inputs(rows, w.D, w.seed)
        x, temb, table = inp["x"][sel], inp["temb"][sel], inp["table"]
    else:
        inp = synth.adarms_inputs(rows, w.D, w.seed, outliers=w.outliers)
        sub = {k: (v[sel] if v.shape[0] == rows else v) for k, v in inp.items()}
    s_of = sel % w.M

    def fn():
        res = None if w.kind == "dit" else sub["res"]
        delta = gate = None
        for l, (pk, style, pkh, pvh) in enumerate(layers):
            if pkh is not None:
                oracle.prefix_copy(pkh, pvh, w.P, kc0, kc0, interleave=True)
            if w.kind == "dit":
                x8 = oracle.ada_layer_norm_quant_table(x, temb, table, 0, 1,
                                                       0.01, eps=w.eps)["x8"]
            else:
                if L == 1:
                    d, g, st = sub["delta"], sub["prev_gate"], sub["style"]
                elif l == 0:
                    d = np.zeros_like(res)
                    g, st = np.zeros((1, w.D), np.uint16), style
                else:
                    d, g, st = delta, gate, style
                pr = oracle.ada_rms_norm_quant(res, d, g, st, 0.01, eps=w.eps)
                res, x8, gate = pr["res"], pr["x8"], pr["gate_out"]
            qkv = oracle.fp8_gemm(x8, pk["w8"], 0.01, pk["w_scale"],
                                  pk["bias"] if w.bias else None)
            # split + RoPE row by row (each sampled row has its own position)
            qs = []
            for i in range(len(sel)):
                s = int(s_of[i])
                kk = np.zeros((1, 1, w.hkv, w.hd), np.uint16)
                q, _, _ = oracle.split_rope_kvcache(
                    qkv[i:i + 1], rope[s:s + 1], 1, 1, w.hq, w.hkv, w.hd, 0,
                    kk, kk)
                qs.append(q.reshape(-1))
            delta = np.stack(qs) if w.hq * w.hd == w.D else None
    return fn, len(sel) * 1, (f"{len(sel)} of {rows} rows, {L} layer(s) "
                              "of prefix copy + producer + GEMM + split/RoPE")


def cpu_baseline(name, synth, seconds=12.0):
    import oracle
    fn, tokens, text = oracle_sampler(name, synth)
    fn()  # warm
    n, t0 = 0, time.perf_counter()
    while True:
        fn()
        n += 1
        el = time.perf_counter() - t0
        if el >= seconds or n >= 2000:
            break
    return {"value": tokens * n / el, "unit": "tokens/s",
            "cores": oracle.num_threads(), "kind": "oracle",
            "sample": f"{text}; {n} repetitions in {el:.1f} s"}


def run_reference(args):
    """The reference arm: the CPU oracle, as it stands, on the host cores."""
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return 0
    from fp8_transformer_block_b200 import synth
    import oracle
    fn, tokens, text = oracle_sampler(args.config, synth)
    t0 = time.perf_counter()
    fn()
    t1 = time.perf_counter() - t0
    cap = None
    if args.steps * t1 > 150.0:   # keep the whole run within a few minutes
        base, _, m = args.config.partition(":")
        w = synth.WORKLOADS[base]
        full = w.M if w.kind == "mlp" else w.rows
        if w.kind == "ditffn":
            full = 32
        if w.kind == "style":
            full = min(w.N, max(3 * w.D, (1 << 27) // (w.D * w.rows)))
        cap = max(1, int(full * 150.0 / (args.steps * t1) * 0.5))
        fn, tokens, text = oracle_sampler(args.config, synth, rows_cap=cap)
    for _ in range(args.warmup):
        fn()
    t0 = time.perf_counter()
    for _ in range(args.steps):
        fn()
    el = time.perf_counter() - t0
    v = tokens * args.steps / el
    base, _, m = args.config.partition(":")
    w = synth.WORKLOADS[base].with_M(int(m)) if m else synth.WORKLOADS[base]
    line = {"metric": METRIC, "value": v, "unit": "tokens/s", "n_gpus": args.gpus,
            "steps": args.steps, "warmup": args.warmup,
            "ms_per_step": 1e3 * el / args.steps, "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None,
            "dtype": StyleRunner.dtype if w.kind == "style" else "e4m3/fp32",
            "data": "synthetic", "impl": "reference",
            "config": {"workload": workload_text(w),
                       "sample_per_step": text},
            "cpu_baseline": {"value": v, "unit": "tokens/s",
                             "cores": oracle.num_threads(), "kind": "oracle",
                             "sample": text},
            "e2e": {"value": v, "unit": "tokens/s", "h2d_bytes_per_step": 0,
                    "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)
    return 0


# ----------------------------------------------------------------- GPU arm --

L2_BYTES = 126 << 20


def _footprint(runner, torch):
    """Device bytes a step of this runner reads or writes (its own tensors)."""
    if hasattr(runner, "footprint"):
        return runner.footprint()
    seen, total = set(), 0
    for v in vars(runner).values():
        ts = []
        if isinstance(v, torch.Tensor):
            ts = [v]
        elif isinstance(v, (list, tuple)):
            ts = [x for x in v if isinstance(x, torch.Tensor)]
            for x in v:
                if isinstance(x, dict):
                    ts += [y for y in x.values() if isinstance(y, torch.Tensor)]
                    pk = x.get("pk")
                    if pk is not None:
                        ts += [pk.w8]
        elif hasattr(v, "w8"):
            ts = [v.w8]
        for t in ts:
            if t.data_ptr() not in seen:
                seen.add(t.data_ptr())
                total += t.numel() * t.element_size()
    return total


def _smallest_divisor_at_least(K, r):
    for d in range(max(1, r), K + 1):
        if K % d == 0:
            return d
    return K


SUB_CONFIGS = ("tiny_adarms", "vla_action_expert", "gateup_mlp") + tuple(
    f"adarms_stack18:{m}" for m in (1, 16, 50, 256, 1024, 4096))


class GpuEnv:
    """What every measurement of one run shares: torch, the process group,
    the binding, the L2 flush buffer and the peaks."""

    def __init__(self, args):
        import torch
        import torch.distributed as dist
        self.torch, self.dist, self.args = torch, dist, args
        self.world = int(os.environ.get("WORLD_SIZE", "1"))
        self.rank = int(os.environ.get("RANK", "0"))
        local = int(os.environ.get("LOCAL_RANK", "0"))
        torch.cuda.set_device(local)
        self.dev = torch.device("cuda", local)
        if self.world > 1:
            from datetime import timedelta
            dist.init_process_group("nccl", timeout=timedelta(seconds=120),
                                    device_id=self.dev)
        from fp8_transformer_block_b200 import build
        if self.rank == 0 or self.world == 1:
            build.build()
        self.barrier()
        from fp8_transformer_block_b200 import frt, synth
        from fp8_transformer_block_b200 import runtime as rt
        self.frt, self.synth, self.rt = frt, synth, rt
        self.flush = torch.empty(FLUSH_BYTES, dtype=torch.uint8, device=self.dev)
        self.gpu_id = None
        try:
            self.gpu_id = "GPU-" + str(torch.cuda.get_device_properties(self.dev).uuid)
        except Exception:  # noqa: BLE001
            pass
        self.peaks = _peaks()
        self.own = None

    def barrier(self):
        if self.world > 1:
            self.dist.barrier()

    def max_ms(self, ms):
        return max_over_ranks(ms, self.torch, self.dist, self.world, self.dev)

    def capture(self, calls):
        torch = self.torch
        cap = torch.cuda.Stream(device=self.dev)
        cap.wait_stream(torch.cuda.current_stream())
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g, stream=cap):
            for c in calls:
                c()
        torch.cuda.current_stream().wait_stream(cap)
        return g


def _kern_entry(ms, k, hbm, fp8_peak, own):
    e = {"kernel": k.name, "us": round(ms * 1e3, 3),
         "launches_per_step": k.per_step, "bound": k.bound,
         "algo_bytes": int(k.algo_bytes),
         "GB_s": round(k.algo_bytes / (ms * 1e-3) / 1e9, 1),
         "hbm_frac": round(k.algo_bytes / (ms * 1e-3) / 1e9 / hbm, 4)}
    if k.flops:
        e["TFLOP_s"] = round(k.flops / (ms * 1e-3) / 1e12, 2)
        e["fp8_frac"] = round(e["TFLOP_s"] / fp8_peak, 4)
        e["fp8_frac_own"] = round(e["TFLOP_s"] / own["fp8_dense_tflops"], 4)
        e["fp8_frac_own_low_toggle"] = round(
            e["TFLOP_s"] / own["fp8_dense_tflops_low_toggle"], 4)
    e["hbm_frac_own"] = round(e["GB_s"] / own["hbm_copy_gbs"], 4)
    return e


def measure(env, name, n_rep, cpu_seconds):
    """One workload: R independent copies stepped in rotation (inputs larger
    than L2), n_rep timed regions of exactly K steps each (CUDA events on
    the launching stream around K steps replayed from CUDA graphs, a barrier
    and a synchronize on both sides, max over ranks), each kernel alone the
    same way, an isolated step after an L2 flush, the end-to-end step with
    host buffers on the host clock, and the oracle on the host cores."""
    torch, frt, args = env.torch, env.frt, env.args
    first = make_runner(name, torch, frt, env.rt, env.synth)
    w = first.w
    L = getattr(first, "L", 1)
    fp = _footprint(first, torch)
    K = args.steps
    r_min = 1 if fp >= 1.5 * L2_BYTES else -(-int(1.5 * L2_BYTES) // fp)
    R = _smallest_divisor_at_least(K, min(r_min, K))
    runners = [first] + [make_runner(name, torch, frt, env.rt, env.synth)
                         for _ in range(R - 1)]
    torch.cuda.synchronize()
    for _ in range(args.warmup):
        for r in runners:
            r.step()
    torch.cuda.synchronize()
    assert frt.frt_device_status(True) == frt.FRT_OK
    g_steps = env.capture([r.step for r in runners])
    for _ in range(2):
        g_steps.replay()
    torch.cuda.synchronize()
    assert frt.frt_device_status(True) == frt.FRT_OK

    mk = lambda: torch.cuda.Event(enable_timing=True)  # noqa: E731
    reps = K // R
    clocks = ClockSampler(env.gpu_id)
    region_ms = []
    env.barrier()
    torch.cuda.synchronize()
    clocks.start()
    t_wall = time.perf_counter()
    for _ in range(n_rep):
        e0, e1 = mk(), mk()
        env.barrier()
        torch.cuda.synchronize()
        torch.cuda._sleep(2_000_000)   # hold the GPU while the replays queue
        torch.cuda.nvtx.range_push("timed_steps")
        e0.record()
        for _ in range(reps):
            g_steps.replay()
        e1.record()
        torch.cuda.nvtx.range_pop()
        torch.cuda.synchronize()
        env.barrier()
        region_ms.append(env.max_ms(e0.elapsed_time(e1)))
    wall = time.perf_counter() - t_wall
    clk = clocks.stop()
    assert frt.frt_device_status(True) == frt.FRT_OK
    med_ms = statistics.median(region_ms)
    ms_per_step = med_ms / K
    value = job_throughput(first.tokens, K, med_ms, env.world)

    # ---- each kernel alone (and the aux kernels), back to back over the R copies
    def time_alone(calls, label):
        gk = env.capture(calls)
        gk.replay()
        torch.cuda.synchronize()
        a, b = mk(), mk()
        torch.cuda._sleep(2_000_000)
        torch.cuda.nvtx.range_push(f"kernel_{label}")
        a.record()
        for _ in range(reps):
            gk.replay()
        b.record()
        torch.cuda.nvtx.range_pop()
        torch.cuda.synchronize()
        return env.max_ms(a.elapsed_time(b)) / (reps * R)

    kinds, kern_ms = [], []
    for kk in range(len(first.kernel_calls())):
        kinds.append(first.kernel_calls()[kk][0])
        kern_ms.append(time_alone([r.kernel_calls()[kk][1] for r in runners],
                                  kinds[-1].name))
    aux = []
    if hasattr(first, "aux_calls"):
        n_aux = len(first.aux_calls())
        for kk in range(n_aux):
            k = first.aux_calls()[kk][0]
            aux.append((k, time_alone([r.aux_calls()[kk][1] for r in runners], k.name)))
    assert frt.frt_device_status(True) == frt.FRT_OK

    # ---- one step per event pair after an L2 flush: the latency of an
    # isolated step as a stream sees it (event and launch costs included)
    flush = env.flush
    g_one = env.capture([first.step])
    n_iso = min(K, 100)
    iso = [(mk(), mk()) for _ in range(n_iso)]
    for i in range(n_iso):
        flush.fill_(i & 0xFF)
        torch.cuda._sleep(1_000_000)
        iso[i][0].record()
        g_one.replay()
        iso[i][1].record()
        torch.cuda.synchronize()
    iso_us = 1e3 * sum(a.elapsed_time(b) for a, b in iso) / n_iso
    del g_one, g_steps

    # ---- e2e through the public entry points with host buffers: every
    # step copies its inputs in from pinned host memory, runs, and reads its
    # outputs back; timed on the host clock from the first call to the
    # synchronize after the read-back (host-side launch and marshalling
    # included), after an L2 flush that has completed
    first.e2e_setup()
    for _ in range(3):
        first.e2e_step()
    torch.cuda.synchronize()
    KE = min(K, 100)
    host_s = 0.0
    env.barrier()
    for i in range(KE):
        flush.fill_(i & 0xFF)
        torch.cuda.synchronize()
        t0 = time.perf_counter()
        first.e2e_step()
        torch.cuda.synchronize()
        host_s += time.perf_counter() - t0
    e_ms = env.max_ms(1e3 * host_s)
    e2e_value = job_throughput(first.tokens, KE, e_ms, env.world)
    # the same steps' device time alone (the GPU held by a spin while the
    # host enqueues, so host-side costs are not in it)
    e_ev = [(mk(), mk()) for _ in range(KE)]
    for i in range(KE):
        flush.fill_(i & 0xFF)
        torch.cuda._sleep(1_000_000)
        e_ev[i][0].record()
        first.e2e_step()
        e_ev[i][1].record()
    torch.cuda.synchronize()
    ed_ms = env.max_ms(sum(a.elapsed_time(b) for a, b in e_ev))
    assert frt.frt_device_status(True) == frt.FRT_OK

    # ---- roofline of the dominant kernel (largest share of a step)
    hbm, bf16_burst, _, src = env.peaks
    fp8_peak = bf16_burst * FP8_PER_BF16
    own = env.own
    shares = [ms * k.per_step for ms, k in zip(kern_ms, kinds)]
    dom = int(np.argmax(shares))
    kd = kinds[dom]
    if kd.bound == "tensor":
        achieved = kd.flops / (kern_ms[dom] * 1e-3) / 1e12
        peak, unit, peak_own = fp8_peak, "TFLOP/s", own["fp8_dense_tflops"]
    else:
        achieved = kd.algo_bytes / (kern_ms[dom] * 1e-3) / 1e9
        peak, unit, peak_own = hbm, "GB/s", own["hbm_copy_gbs"]
    base = name.partition(":")[0]
    tr = NCU_TRAFFIC.get((name, kd.name)) or NCU_TRAFFIC.get((base, kd.name))
    traffic = tr[0] if tr and tr[1] == _src_hash(kd.name) else None
    roof = {"bound": kd.bound, "kernel": kd.name, "achieved": achieved,
            "peak": peak, "unit": unit, "frac": achieved / peak, "traffic": traffic,
            "peak_source": f"{src} " + ("(bf16 burst x 2, nominal fp8/bf16 ratio)"
                                        if unit == "TFLOP/s" else "(HBM copy)"),
            "algo_per_launch": kd.flops if unit == "TFLOP/s" else kd.algo_bytes,
            "peak_own": peak_own, "frac_own": achieved / peak_own,
            "peak_own_source": ("the library's own tcgen05 e4m3 MMA loop on Gaussian "
                                "operand codes" if unit == "TFLOP/s"
                                else "the library's own device copy")}
    if unit == "TFLOP/s":
        roof["fp8_frac_own"] = roof["frac_own"]
        roof["peak_own_low_toggle"] = own["fp8_dense_tflops_low_toggle"]
        roof["fp8_frac_own_low_toggle"] = achieved / own["fp8_dense_tflops_low_toggle"]
    kern_list = [_kern_entry(ms, k, hbm, fp8_peak, own) for ms, k in zip(kern_ms, kinds)]
    aux_list = [_kern_entry(ms, k, hbm, fp8_peak, own) for k, ms in aux]
    if aux:
        by = {e["kernel"]: e for e in aux_list}
        if "gemm_bf16" in by and kd.name == "gemm_rope_kv":
            by["gemm_bf16"]["fused_epilogue_cost_us"] = round(
                kern_ms[dom] * 1e3 - by["gemm_bf16"]["us"], 3)

    cpu = None
    if env.rank == 0 and env.world == 1 and not args.no_cpu and cpu_seconds > 0:
        cpu = cpu_baseline(name, env.synth, seconds=cpu_seconds)
    rec = {
        "workload": workload_text(w), "value": value, "unit": "tokens/s",
        "steps": K, "ms_per_step": ms_per_step, "us_per_layer": 1e3 * ms_per_step / L,
        "timed_regions": {"n": n_rep, "steps_each": K,
                          "ms_per_step": [round(m / K, 6) for m in region_ms],
                          "median": round(ms_per_step, 6),
                          "min": round(min(region_ms) / K, 6),
                          "max": round(max(region_ms) / K, 6),
                          "spread": round((max(region_ms) - min(region_ms)) / med_ms, 4)},
        "dtype": getattr(first, "dtype", "e4m3/fp32"),
        "l2": (f"inputs larger than L2: {R} independent copies of the workload "
               f"({R * fp / 2**20:.0f} MiB) rotated step by step" if R > 1 else
               f"inputs larger than L2 ({fp / 2**20:.0f} MiB per step)"),
        "isolated_step_us_after_l2_flush": round(iso_us, 3),
        "roofline": roof, "kernels": kern_list,
        "cpu_baseline": cpu,
        "e2e": {"value": e2e_value, "unit": "tokens/s",
                "h2d_bytes_per_step": int(first.h2d_bytes),
                "d2h_bytes_per_step": int(first.d2h_bytes),
                "clock": "host (perf_counter), call to synchronize, per step",
                "us_per_step": round(1e3 * e_ms / KE, 3), "steps": KE},
        "e2e_device": {"value": job_throughput(first.tokens, KE, ed_ms, env.world),
                       "unit": "tokens/s", "us_per_step": round(1e3 * ed_ms / KE, 3),
                       "clock": "CUDA events around each step, GPU held while it queued"},
        "gpu_launches": first.launches * K * n_rep,
        "gpu_launches_per_region": first.launches * K,
        "clocks": clk, "wall_s_timed_loop": round(wall, 3),
    }
    if aux_list:
        rec["aux_kernels"] = aux_list
    for r in runners:
        for attr in list(vars(r)):
            setattr(r, attr, None)
    del runners, first
    torch.cuda.synchronize()
    torch.cuda.empty_cache()
    return rec


def run_gpu(args):
    env = GpuEnv(args)
    torch = env.torch
    env.own = own_peaks(torch, env.frt)
    main_rec = measure(env, args.config, args.repeats, args.cpu_seconds)
    subs = {}
    if args.config == DEFAULT_CONFIG and not args.no_subconfigs:
        for name in SUB_CONFIGS:
            subs[name] = measure(env, name, 3, args.cpu_seconds_sub)
    if env.rank != 0:
        if env.world > 1:
            env.dist.destroy_process_group()
        return 0
    line = {
        "metric": METRIC, "value": main_rec["value"], "unit": "tokens/s",
        "n_gpus": env.world, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": main_rec["ms_per_step"], "us_per_layer": main_rec["us_per_layer"],
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
        "dtype": main_rec["dtype"], "data": "synthetic",
        "config": {"workload": main_rec["workload"], "l2": main_rec["l2"],
                   "parallelism": "replicas" if env.world > 1 else "single",
                   "timing": (f"{args.repeats} timed regions of exactly K steps each "
                              "(K back-to-back steps replayed from CUDA graphs, CUDA "
                              "events on the launching stream, barrier + synchronize "
                              "on both sides, max over ranks); value from the median "
                              "region; kernels timed the same way"),
                   "isolated_step_us_after_l2_flush":
                       main_rec["isolated_step_us_after_l2_flush"],
                   "e2e_scope": "each step copies the tokens' input rows in from pinned "
                                "host memory and reads its output rows (and new K/V rows) "
                                "back; weights, tables and the prefix K/V cache (the host "
                                "model's device-resident cache) stay in device memory; "
                                "timed on the host clock"},
        "timed_regions": main_rec["timed_regions"],
        "roofline": main_rec["roofline"], "kernels": main_rec["kernels"],
        "peaks_own": env.own, "cpu_baseline": main_rec["cpu_baseline"],
        "e2e": main_rec["e2e"], "e2e_device": main_rec["e2e_device"],
        "gpu_launches": main_rec["gpu_launches"],
        "gpu_launches_per_region": main_rec["gpu_launches_per_region"],
        "clocks": main_rec["clocks"], "wall_s_timed_loop": main_rec["wall_s_timed_loop"],
    }
    if "aux_kernels" in main_rec:
        line["aux_kernels"] = main_rec["aux_kernels"]
    if subs:
        line["configs"] = subs
    print(json.dumps(line), flush=True)
    if env.world > 1:
        env.dist.destroy_process_group()
    return 0


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=1000)
    ap.add_argument("--warmup", type=int, default=10)
    ap.add_argument("--config", default=DEFAULT_CONFIG)
    ap.add_argument("--impl", default="frt", choices=["frt", "reference"])
    ap.add_argument("--no-cpu", action="store_true")
    ap.add_argument("--cpu-seconds", type=float, default=12.0)
    ap.add_argument("--cpu-seconds-sub", type=float, default=3.0,
                    help="oracle seconds per sub-configuration record")
    ap.add_argument("--repeats", type=int, default=5,
                    help="timed regions of K steps for the main line (median reported)")
    ap.add_argument("--no-subconfigs", action="store_true",
                    help="only the selected workload (no per-configuration records)")
    args = ap.parse_args()
    if args.warmup < 3:
        ap.error("--warmup must be >= 3")
    if args.impl == "reference":
        return run_reference(args)
    return run_gpu(args)


if __name__ == "__main__":
    sys.exit(main())

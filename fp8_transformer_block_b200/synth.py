"""Seeded synthetic inputs for the chain's five workloads.

This module only draws numbers: seeded normal samples, rounded to bf16 bit
patterns, in the shapes and distributions the workloads name.  It holds none
of the chain's arithmetic, so both the CUDA path and the CPU oracle take
their inputs from here (identical bytes to both).

Recipe (all draws fp32 from ``numpy.random.Generator(PCG64(seed))`` in the
order listed, rounded to bf16 by round-to-nearest-even on the bit pattern):

* AdaRMS producer inputs: residual ``res`` N(0,1), sublayer output ``delta``
  N(0,1), previous gate ``prev_gate`` N(0,1) (one broadcast row), and the
  modulation row ``style`` = (scale, shift, gate) N(0, 0.02*sqrt(D)), the
  spread of an N(0,1) conditioning vector through an N(0, 0.02) [3D, D]
  projection (the projection itself is not drawn).  Outlier rows (1 % of
  rows, at least one, seeded choice) of ``res`` are scaled by 20.
* Weights N(0, 0.02); biases N(0, 0.01) where a workload has them.
* Per-token-table LayerNorm inputs: ``x`` N(0,1), ``temb`` N(0,1),
  ``table`` fp32 N(0, 0.1).
* Prefix K/V of the host cache N(0,1).
* Modulation projection (every norm's (scale, shift, gate) from one
  conditioning row): ``cond`` N(0,1) kept as fp32 values on the bf16 grid,
  the stacked dense weights [(2L+1)*3D, D] N(0, 0.02) bf16, their fp32
  bias N(0, 0.01) on the bf16 grid.
* The calibration batch of a workload uses seed + 500.
"""

from __future__ import annotations

from dataclasses import dataclass, field

import numpy as np

SEED_BASE = 1000
CAL_OFFSET = 500


def bf16_bits(x: np.ndarray) -> np.ndarray:
    """fp32 -> bf16 bit pattern (uint16), nearest-even; finite input only:
    adding 0x7FFF plus the kept part's lowest bit carries into the kept
    half exactly when the dropped half is above one half, or equal to it
    with an odd kept part."""
    u = np.ascontiguousarray(x, dtype=np.float32).view(np.uint32)
    r = u + np.uint32(0x7FFF) + ((u >> np.uint32(16)) & np.uint32(1))
    return (r >> np.uint32(16)).astype(np.uint16)


def bf16_value(h: np.ndarray) -> np.ndarray:
    """bf16 bit pattern -> fp32 value (exact)."""
    return (np.asarray(h, dtype=np.uint16).astype(np.uint32) << 16).view(
        np.float32)


def normal_bf16(rng: np.random.Generator, shape, std: float = 1.0):
    """N(0, std) draws rounded to bf16 bit patterns.  Large arrays are drawn
    in blocks of leading rows: the generator's stream, and so every value,
    is the same as one draw of the whole shape."""
    shape = tuple(np.atleast_1d(shape)) if not isinstance(shape, tuple) else shape
    n = int(np.prod(shape))
    if len(shape) < 2 or n <= (1 << 24):
        return bf16_bits(rng.standard_normal(size=shape, dtype=np.float32)
                         * np.float32(std))
    out = np.empty(shape, np.uint16)
    step = max(1, (1 << 24) // int(np.prod(shape[1:])))
    for i in range(0, shape[0], step):
        blk = (min(step, shape[0] - i),) + shape[1:]
        out[i:i + blk[0]] = bf16_bits(rng.standard_normal(size=blk, dtype=np.float32)
                                      * np.float32(std))
    return out


def outlier_rows(rng: np.random.Generator, rows: int, frac: float = 0.01):
    n = max(1, int(round(frac * rows)))
    return np.sort(rng.choice(rows, size=n, replace=False))


@dataclass(frozen=True)
class Workload:
    """One of the five shapes.  ``kind`` is "adarms" (AdaRMS producer +
    q/k/v chain), "dit" (per-token-table LayerNorm + biased q/k/v),
    "mlp" (AdaRMS producer + gate/up GEMM + GEGLU + down GEMM),
    "style" (the modulation projection of ``M`` conditioning rows into the
    (scale, shift, gate) rows of all 2 * ``layers`` + 1 norms),
    "stack" (``layers`` AdaRMS chain layers, residual carried) or "full"
    (``layers`` whole AdaRMS layers except attention: the q/k/v chain, the
    output projection, the FFN half; then the final tail) or "ditffn" (the
    video-DiT block's FFN half)."""
    name: str
    cid: int
    kind: str
    B: int
    M: int
    D: int
    hq: int = 0
    hkv: int = 0
    hd: int = 0
    P: int = 0
    T: int = 0
    bias: bool = False
    H: int = 0
    layers: int = 1
    outliers: bool = False
    cal_rows: int = 64
    theta: float = 10000.0
    eps: float = 1e-6
    m_sweep: tuple = field(default_factory=tuple)
    live: bool = False  # "full": every step projects the norms' rows from cond

    @property
    def seed(self) -> int:
        return SEED_BASE + self.cid

    @property
    def rows(self) -> int:
        return self.B * self.M

    @property
    def N(self) -> int:
        if self.kind == "mlp":
            return 2 * self.H
        if self.kind == "style":
            return (2 * self.layers + 1) * 3 * self.D
        return (self.hq + 2 * self.hkv) * self.hd

    def with_M(self, M: int) -> "Workload":
        T = self.P + M if self.kind in ("stack", "full") else self.T
        return Workload(**{**self.__dict__, "M": M, "T": T})


WORKLOADS = {
    "tiny_adarms": Workload("tiny_adarms", 0, "adarms", B=1, M=64, D=512,
                            hq=8, hkv=1, hd=64, P=0, T=64, cal_rows=64),
    "vla_action_expert": Workload("vla_action_expert", 1, "adarms", B=1, M=50,
                                  D=2048, hq=8, hkv=1, hd=256, P=816, T=1024,
                                  outliers=True, cal_rows=4096),
    "video_dit": Workload("video_dit", 2, "dit", B=2, M=4096, D=3072, hq=24,
                          hkv=24, hd=128, P=0, T=4096, bias=True,
                          cal_rows=512),
    "gateup_mlp": Workload("gateup_mlp", 3, "mlp", B=1, M=1024, D=2048,
                           H=16384, cal_rows=128),
    "adarms_stack18": Workload("adarms_stack18", 4, "stack", B=1, M=50, D=512,
                               hq=8, hkv=1, hd=64, P=816, T=866, layers=18,
                               cal_rows=64,
                               m_sweep=(1, 16, 50, 256, 1024, 4096)),
    # not one of the five configurations: the stack's layers made whole
    # except attention (FFN hidden 4 * D, a reading: the pages give none
    # for this shape)
    "adarms_layer18": Workload("adarms_layer18", 5, "full", B=1, M=50, D=512,
                               hq=8, hkv=1, hd=64, P=816, T=866, H=2048,
                               layers=18, cal_rows=64),
    # the same loop with the modulation projection on device at the head of
    # every step (one conditioning row into all 2 * 18 + 1 norms' rows)
    "adarms_layer18_live": Workload("adarms_layer18_live", 9, "full", B=1, M=50, D=512,
                                    hq=8, hkv=1, hd=64, P=816, T=866, H=2048,
                                    layers=18, cal_rows=64, live=True),
    # not one of the five configurations: the video-DiT block's FFN half
    # (producer at the FFN site, chunks 3/4; up projection + GELU requant;
    # down projection; both with bias), FFN hidden 4 * D (a reading)
    "video_dit_ffn": Workload("video_dit_ffn", 6, "ditffn", B=2, M=4096, D=3072,
                              H=12288, bias=True, cal_rows=256),
    # not one of the five configurations: the modulation projection on
    # device, one conditioning row into the rows of all 2 * 18 + 1 norms, at
    # the stack's width and at the action expert's width
    "style_stack18": Workload("style_stack18", 7, "style", B=1, M=1, D=512,
                              layers=18, bias=True),
    "style_vla18": Workload("style_vla18", 8, "style", B=1, M=1, D=2048,
                            layers=18, bias=True),
}


def adarms_inputs(rows: int, D: int, seed: int, outliers: bool = False):
    """Producer inputs of the AdaRMS form (see the module recipe)."""
    rng = np.random.Generator(np.random.PCG64(seed))
    res = rng.standard_normal(size=(rows, D), dtype=np.float32)
    if outliers:
        res[outlier_rows(rng, rows)] *= np.float32(20.0)
    return {
        "res": bf16_bits(res),
        "delta": normal_bf16(rng, (rows, D)),
        "prev_gate": normal_bf16(rng, (1, D)),
        "style": normal_bf16(rng, (1, 3 * D), 0.02 * np.sqrt(D)),
    }


def dit_inputs(rows: int, D: int, seed: int, chunks: int = 6,
               with_table: bool = True):
    rng = np.random.Generator(np.random.PCG64(seed))
    out = {
        "x": normal_bf16(rng, (rows, D)),
        "temb": normal_bf16(rng, (rows, chunks, D)),
    }
    if with_table:
        out["table"] = (rng.standard_normal(size=(chunks, D), dtype=np.float32)
                        * np.float32(0.1))
    return out


def qkv_weights(hq: int, hkv: int, hd: int, K: int, seed: int,
                bias: bool = False):
    rng = np.random.Generator(np.random.PCG64(seed + 7919))
    ws = [normal_bf16(rng, (n * hd, K), 0.02) for n in (hq, hkv, hkv)]
    bs = ([normal_bf16(rng, (n * hd,), 0.01) for n in (hq, hkv, hkv)]
          if bias else [None, None, None])
    return ws, bs


def mlp_weights(D: int, H: int, seed: int):
    rng = np.random.Generator(np.random.PCG64(seed + 7919))
    return {
        "gate": normal_bf16(rng, (H, D), 0.02),
        "up": normal_bf16(rng, (H, D), 0.02),
        "down": normal_bf16(rng, (D, H), 0.02),
    }


def prefix_cache(B: int, hkv: int, T_src: int, hd: int, seed: int):
    """Host-layout prefix cache [B, hkv, T_src, hd] for K and V."""
    rng = np.random.Generator(np.random.PCG64(seed + 104729))
    return (normal_bf16(rng, (B, hkv, T_src, hd)),
            normal_bf16(rng, (B, hkv, T_src, hd)))


def stack_layer_inputs(w: Workload, layer: int):
    """Per-layer fresh weights, style and prefix of the stacked workload."""
    s = w.seed + 1000 * (layer + 1)
    ws, bs = qkv_weights(w.hq, w.hkv, w.hd, w.D, s)
    rng = np.random.Generator(np.random.PCG64(s))
    style = normal_bf16(rng, (1, 3 * w.D), 0.02 * np.sqrt(w.D))
    pk, pv = prefix_cache(w.B, w.hkv, w.P, w.hd, s)
    return {"w": ws, "b": bs, "style": style, "prefix_k": pk, "prefix_v": pv}


def full_layer_inputs(w: Workload, layer: int):
    """Per-layer fresh weights of a whole AdaRMS layer (q/k/v, o, gate/up,
    down), the two norms' styles (attention site, FFN site) and the prefix."""
    s = w.seed + 1000 * (layer + 1)
    ws, bs = qkv_weights(w.hq, w.hkv, w.hd, w.D, s)
    rng = np.random.Generator(np.random.PCG64(s))
    styles = normal_bf16(rng, (2, 3 * w.D), 0.02 * np.sqrt(w.D))
    o = normal_bf16(np.random.Generator(np.random.PCG64(s + 17)), (w.D, w.hq * w.hd), 0.02)
    mw = mlp_weights(w.D, w.H, s)
    pk, pv = prefix_cache(w.B, w.hkv, w.P, w.hd, s)
    return {"w": ws, "b": bs, "o": o, "mlp": mw, "styles": styles,
            "prefix_k": pk, "prefix_v": pv}


def final_norm_rows(w: Workload):
    """fp32 (scale, shift, gate) rows of the final norm, the modulation
    projection's distribution."""
    rng = np.random.Generator(np.random.PCG64(w.seed + 31337))
    return (rng.standard_normal(size=(3, w.D), dtype=np.float32)
            * np.float32(0.02 * np.sqrt(w.D)))


def modulation_inputs(rows: int, D: int, n_norms: int, seed: int):
    """Conditioning rows, stacked modulation weights [n_norms * 3D, D] and
    their bias (see the module recipe); norm i's (scale, shift, gate) are
    output columns 3*D*i + {0, D, 2*D}."""
    rng = np.random.Generator(np.random.PCG64(seed + 4241))
    cond = bf16_value(normal_bf16(rng, (rows, D)))
    w = normal_bf16(rng, (n_norms * 3 * D, D), 0.02)
    bias = bf16_value(normal_bf16(rng, (n_norms * 3 * D,), 0.01))
    return {"cond": cond, "w": w, "bias": bias}


def dit_ffn_weights(D: int, H: int, seed: int):
    """Up [H, D] and down [D, H] projections N(0, 0.02) with bf16 biases
    N(0, 0.01) (the DiT block's FFN, biased like its q/k/v)."""
    rng = np.random.Generator(np.random.PCG64(seed + 7919))
    return {"up": normal_bf16(rng, (H, D), 0.02), "up_b": normal_bf16(rng, (H,), 0.01),
            "dn": normal_bf16(rng, (D, H), 0.02), "dn_b": normal_bf16(rng, (D,), 0.01)}

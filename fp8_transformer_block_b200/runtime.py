"""Device-buffer plumbing around the C ABI: torch provides the memory and
the stream, libfrt does every step of the chain.

Nothing here computes a result of the chain: it converts host arrays to
device tensors (bf16 bit patterns travel as uint16 numpy arrays), allocates
outputs, and calls the binding in ``frt``.
"""

from __future__ import annotations

from dataclasses import dataclass

import numpy as np
import torch

from . import frt


# ---------------------------------------------------------------- tensors ---

def bf16_dev(a: np.ndarray, device="cuda") -> torch.Tensor:
    a = np.ascontiguousarray(a, dtype=np.uint16)
    return torch.from_numpy(a.view(np.int16)).to(device).view(torch.bfloat16)


def u8_dev(a: np.ndarray, device="cuda") -> torch.Tensor:
    return torch.from_numpy(np.ascontiguousarray(a, dtype=np.uint8)).to(device)


def f32_dev(a, device="cuda") -> torch.Tensor:
    return torch.from_numpy(np.ascontiguousarray(a, dtype=np.float32)).to(device)


def bf16_host(t: torch.Tensor) -> np.ndarray:
    return t.detach().contiguous().view(torch.int16).cpu().numpy().view(np.uint16)


def u8_host(t: torch.Tensor) -> np.ndarray:
    return t.detach().contiguous().view(torch.uint8).cpu().numpy()


def empty_bf16(*shape, device="cuda"):
    return torch.empty(*shape, dtype=torch.bfloat16, device=device)


def empty_u8(*shape, device="cuda"):
    return torch.empty(*shape, dtype=torch.uint8, device=device)


def scale_dev(v: float, device="cuda") -> torch.Tensor:
    return torch.tensor([float(v)], dtype=torch.float32, device=device)


# ------------------------------------------------------------------ pack ---

@dataclass
class PackedWeight:
    w8: torch.Tensor        # [N, K] uint8 (e4m3 codes)
    w_scale: torch.Tensor   # [1] fp32
    bias: torch.Tensor | None  # [N] bf16
    N: int
    K: int


def pack(ws, biases=None, layout=frt.FRT_PACK_CONCAT, hd=0, device="cuda",
         stream=None) -> PackedWeight:
    """Joint FP8 pack of sibling weights given as device bf16 tensors (or
    uint16 numpy arrays, uploaded first)."""
    ws = [bf16_dev(w, device) if isinstance(w, np.ndarray) else w for w in ws]
    if biases is not None:
        biases = [None if b is None else
                  (bf16_dev(b, device) if isinstance(b, np.ndarray) else b)
                  for b in biases]
    K = int(ws[0].shape[1])
    n_rows = [int(w.shape[0]) for w in ws]
    N = sum(n_rows)
    w8 = empty_u8(N, K, device=device)
    sc = torch.zeros(1, dtype=torch.float32, device=device)
    has_bias = biases is not None and any(b is not None for b in biases)
    bias = empty_bf16(N, device=device) if has_bias else None
    frt.frt_pack_weights_fp8(ws, n_rows, K, biases, layout, hd, w8, sc, bias,
                             stream=stream)
    return PackedWeight(w8, sc, bias, N, K)


def workspace(nbytes: int, device="cuda") -> torch.Tensor | None:
    """Zero-filled split-K workspace (the library keeps its counters at
    zero after every completed call)."""
    if nbytes <= 0:
        return None
    return torch.zeros(nbytes, dtype=torch.uint8, device=device)


# --------------------------------------------------------------- chain ----

def chain_desc(**kw) -> frt.frt_chain_desc:
    """Build an frt_chain_desc; tensor fields accept tensors/ints/None."""
    d = frt.frt_chain_desc()
    ptr_fields = {name for name, typ in frt.frt_chain_desc._fields_
                  if typ is frt._p}
    for k, v in kw.items():
        if k in ptr_fields:
            setattr(d, k, frt.ptr(v))
        else:
            setattr(d, k, v)
    return d


def ffn_desc(**kw) -> frt.frt_ffn_desc:
    """Build an frt_ffn_desc; tensor fields accept tensors/ints/None."""
    d = frt.frt_ffn_desc()
    ptr_fields = {name for name, typ in frt.frt_ffn_desc._fields_ if typ is frt._p}
    for k, v in kw.items():
        setattr(d, k, frt.ptr(v) if k in ptr_fields else v)
    return d

"""Shared helpers of the GPU tests: run one Sparse-BitLinear layer through the
C ABI (via the Python binding) and hand back numpy arrays, and compare them
with the oracle.  Inputs always come from sparsity_sbl_quantize_b200.workloads
and are copied byte for byte to the GPU."""
from __future__ import annotations

import numpy as np
import torch

import oracle


def sbl_mod():
    from sparsity_sbl_quantize_b200 import build
    build.build()
    from sparsity_sbl_quantize_b200 import sbl
    return sbl


def to_dev(a: np.ndarray, dtype=None) -> torch.Tensor:
    t = torch.from_numpy(np.ascontiguousarray(a))
    if dtype is not None:
        t = t.view(dtype)
    return t.cuda()


def bf16_dev(bits: np.ndarray) -> torch.Tensor:
    return to_dev(bits.view(np.int16), torch.bfloat16)


def bits_of(t: torch.Tensor) -> np.ndarray:
    """bf16 tensor -> uint16 bit patterns on the host."""
    return t.view(torch.int16).cpu().numpy().view(np.uint16)


ALL_FORMATS = 1 | 2 | 4 | 8


class GpuLayer:
    """Pack a layer on the GPU and keep its buffers."""

    def __init__(self, w: np.ndarray, n: int, m: int, formats: int = ALL_FORMATS):
        self.sbl = sbl = sbl_mod()
        o, k = w.shape
        self.desc = sbl.desc(o, k, n, m)
        self.w_dev = to_dev(w)
        self.packed = sbl.alloc_packed(self.desc, formats)
        self.ws = sbl.alloc_workspace(sbl.sbl_workspace_bytes(self.desc, 0, sbl.SBL_OP_QUANTIZE_MASK_PACK))
        self.formats = formats
        sbl.sbl_quantize_mask_pack(self.desc, self.w_dev, formats, self.packed, self.ws)

    def host(self):
        p = self.packed
        out = {"gamma": np.float32(p.gamma[0].item())}
        if p.pk2 is not None:
            out["pk2"] = p.pk2.cpu().numpy()
        if p.nm_values is not None:
            out["nm_values"] = p.nm_values.cpu().numpy()
            out["nm_bitmap"] = p.nm_bitmap.cpu().numpy()
        if p.i8 is not None:
            out["i8"] = p.i8.cpu().numpy()
        if p.bf16t is not None:
            out["bf16t"] = bits_of(p.bf16t)
        if p.sp24_values is not None:
            out["sp24_values"] = p.sp24_values.cpu().numpy()
            out["sp24_meta"] = p.sp24_meta.cpu().numpy()
        if p.t24_lo is not None:
            out["t24_lo"] = p.t24_lo.cpu().numpy()
            out["t24_hi"] = p.t24_hi.cpu().numpy()
        return out


def quantize_act(x_bits: np.ndarray):
    sbl = sbl_mod()
    t, k = x_bits.shape
    x = bf16_dev(x_bits)
    q = torch.empty((t, k), dtype=torch.int8, device="cuda")
    d = torch.empty((max(t, 1),), dtype=torch.float32, device="cuda")
    sbl.sbl_quantize_act(x, t, k, q, d)
    return q, d


def forward(layer: GpuLayer, q: torch.Tensor, d: torch.Tensor, fmt: int, fp32: bool = False,
            want_acc: bool = True):
    sbl = layer.sbl
    t = q.shape[0]
    o = layer.desc.out_features
    y = torch.empty((t, o), dtype=torch.float32 if fp32 else torch.bfloat16, device="cuda")
    acc = torch.empty((t, o), dtype=torch.int32, device="cuda") if want_acc else None
    sbl.sbl_forward(layer.desc, q, d, t, layer.packed, fmt, y, fp32, acc)
    return y, acc


def normwise(gpu: np.ndarray, ref: np.ndarray) -> float:
    ref = np.asarray(ref, dtype=np.float64)
    den = np.abs(ref).max()
    return float(np.abs(np.asarray(gpu, dtype=np.float64) - ref).max() / (den if den > 0 else 1.0))


def elementwise_rel(gpu: np.ndarray, ref: np.ndarray, floor: float = 1e-2) -> float:
    """Largest elementwise relative error over the entries with |ref| >= floor * max|ref|
    (reported beside the normwise figure; cancellation makes it ill-posed below the floor)."""
    ref = np.asarray(ref, dtype=np.float64)
    gpu = np.asarray(gpu, dtype=np.float64)
    big = np.abs(ref) >= floor * np.abs(ref).max()
    if not big.any():
        return 0.0
    return float((np.abs(gpu[big] - ref[big]) / np.abs(ref[big])).max())


def bf16_ulp(x: np.ndarray) -> np.ndarray:
    """One bf16 ulp at |x| (8 significant bits: 2^(E-7) for |x| in [2^E, 2^(E+1)))."""
    _, e = np.frexp(np.abs(np.asarray(x, dtype=np.float64)))
    return np.ldexp(1.0, (e - 8).astype(np.int64))


def bf16_bits_to_f64(bits: np.ndarray) -> np.ndarray:
    return (np.asarray(bits, dtype=np.uint16).astype(np.uint32) << 16).view(np.float32).astype(np.float64)


def f32_to_bf16_bits(x: np.ndarray) -> np.ndarray:
    """Exact conversion for values that are already bf16 numbers (checked)."""
    b = np.ascontiguousarray(x, dtype=np.float32).view(np.uint32)
    assert not (b & 0xFFFF).any(), "not a bf16 value"
    return (b >> 16).astype(np.uint16)


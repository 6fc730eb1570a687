"""CPU oracle of the Sparse-BitLinear layer -- TEST INFRASTRUCTURE ONLY.

Only ``tests/``, ``__graft_entry__.smoke()`` and the CPU-baseline leg of
``bench.py`` may import this package.  The CUDA library never links, loads or
calls it, and it shares no code with the CUDA path.  The arithmetic lives in
``sbl_oracle.c`` (plain C loops written from the Sparse-BitNet and BitNet
b1.58 2B4T definitions, cited there); this module only marshals numpy arrays.

Parity pins for every function are in ``tests/test_oracle_pins.py``.
"""
from __future__ import annotations

import ctypes

import numpy as np

from .build import build_oracle, library_path

_lib = None


def _load():
    global _lib
    if _lib is None:
        path = build_oracle()
        lib = ctypes.CDLL(path)
        i64, f32, i32 = ctypes.c_int64, ctypes.c_float, ctypes.c_int
        p = ctypes.c_void_p
        lib.sbl_oracle_abs_sum.restype = ctypes.c_double
        lib.sbl_oracle_abs_sum.argtypes = [p, i64]
        lib.sbl_oracle_gamma.restype = f32
        lib.sbl_oracle_gamma.argtypes = [p, i64, i64]
        lib.sbl_oracle_ternarize.argtypes = [p, i64, f32, p]
        lib.sbl_oracle_nm_mask.argtypes = [p, i64, i64, i32, i32, p]
        lib.sbl_oracle_apply_mask.argtypes = [p, p, i64, p]
        lib.sbl_oracle_pk2_row_bytes.restype = i64
        lib.sbl_oracle_pk2_row_bytes.argtypes = [i64]
        lib.sbl_oracle_pack_pk2.argtypes = [p, i64, i64, p]
        lib.sbl_oracle_nm_value_row_bytes.restype = i64
        lib.sbl_oracle_nm_value_row_bytes.argtypes = [i64, i32, i32]
        lib.sbl_oracle_nm_bitmap_row_bytes.restype = i64
        lib.sbl_oracle_nm_bitmap_row_bytes.argtypes = [i64]
        lib.sbl_oracle_pack_nm.argtypes = [p, p, i64, i64, i32, i32, p, p]
        lib.sbl_oracle_sp24_value_row_bytes.restype = i64
        lib.sbl_oracle_sp24_value_row_bytes.argtypes = [i64]
        lib.sbl_oracle_sp24_meta_row_bytes.restype = i64
        lib.sbl_oracle_sp24_meta_row_bytes.argtypes = [i64]
        lib.sbl_oracle_pack_sp24.restype = ctypes.c_int
        lib.sbl_oracle_pack_sp24.argtypes = [p, p, i64, i64, p, p]
        lib.sbl_oracle_t24_lo_row_bytes.restype = i64
        lib.sbl_oracle_t24_lo_row_bytes.argtypes = [i64]
        lib.sbl_oracle_t24_hi_row_bytes.restype = i64
        lib.sbl_oracle_t24_hi_row_bytes.argtypes = [i64]
        lib.sbl_oracle_pack_t24.restype = ctypes.c_int
        lib.sbl_oracle_pack_t24.argtypes = [p, i64, i64, p, p]
        lib.sbl_oracle_epilogue.argtypes = [p, i64, i64, i32, p, p, p]
        lib.sbl_oracle_rmsnorm_quantize_act.argtypes = [p, i64, i64, p, f32, p, p]
        lib.sbl_oracle_gamma_survivors.restype = f32
        lib.sbl_oracle_gamma_survivors.argtypes = [p, p, i64, i64]
        lib.sbl_oracle_nm_mask_quantized.argtypes = [p, i64, i64, i32, i32, p]
        lib.sbl_oracle_mask_flips.restype = i64
        lib.sbl_oracle_mask_flips.argtypes = [p, p, i64]
        lib.sbl_oracle_near_zero.restype = i64
        lib.sbl_oracle_near_zero.argtypes = [p, i64, f32]
        lib.sbl_oracle_block_threshold.argtypes = [p, p, i64, i64, i32, p]
        lib.sbl_oracle_quantize_act.argtypes = [p, i64, i64, p, p]
        lib.sbl_oracle_gemm_acc.restype = i32
        lib.sbl_oracle_gemm_acc.argtypes = [p, p, i64, i64, i64, p]
        lib.sbl_oracle_dequant.argtypes = [p, i64, i64, f32, p, p, p]
        lib.sbl_oracle_backward.argtypes = [p, p, f32, p, p, i64, i64, i64, p, p]
        lib.sbl_oracle_acc_samples.argtypes = [p, p, i64, p, p, i64, p]
        lib.sbl_oracle_dx_samples.argtypes = [p, p, f32, i64, i64, p, p, i64, p]
        lib.sbl_oracle_dw_samples.argtypes = [p, p, p, i64, i64, i64, p, p, i64, p]
        lib.sbl_oracle_rounding_is_nearest.restype = i32
        _lib = lib
    return _lib


class use_library:
    """Context manager that points this wrapper at another build of the oracle
    source (used by the planted-mistake tests to run the pins against a
    deliberately broken copy)."""

    def __init__(self, path: str):
        self.path = path

    def __enter__(self):
        global _lib
        self._saved = _load()
        _lib = None
        real_build = build_oracle
        globals()["build_oracle"] = lambda: self.path
        try:
            _load()
        finally:
            globals()["build_oracle"] = real_build
        return self

    def __exit__(self, *exc):
        global _lib
        _lib = self._saved
        return False


def _ptr(a: np.ndarray):
    assert a.flags["C_CONTIGUOUS"], "oracle inputs must be C-contiguous"
    return a.ctypes.data_as(ctypes.c_void_p)


def _f32(a):
    return np.ascontiguousarray(a, dtype=np.float32)


def _u16(a):
    return np.ascontiguousarray(a, dtype=np.uint16)


def _i8(a):
    return np.ascontiguousarray(a, dtype=np.int8)


def abs_sum(w) -> float:
    """fp64 pairwise-tree sum of |w| over the flat row-major order."""
    w = _f32(w)
    return float(_load().sbl_oracle_abs_sum(_ptr(w), w.size))


def gamma(w) -> np.float32:
    """Absmean weight scale of a [d_out, d_in] fp32 matrix."""
    w = _f32(w)
    d_out, d_in = w.shape
    return np.float32(_load().sbl_oracle_gamma(_ptr(w), d_out, d_in))


def ternarize(w, g) -> np.ndarray:
    w = _f32(w)
    out = np.empty(w.shape, dtype=np.int8)
    _load().sbl_oracle_ternarize(_ptr(w), w.size, float(np.float32(g)), _ptr(out))
    return out


def nm_mask(w, n: int, m: int) -> np.ndarray:
    w = _f32(w)
    d_out, d_in = w.shape
    assert d_in % m == 0
    out = np.empty(w.shape, dtype=np.uint8)
    _load().sbl_oracle_nm_mask(_ptr(w), d_out, d_in, n, m, _ptr(out))
    return out


def apply_mask(wq, mask) -> np.ndarray:
    wq = _i8(wq)
    mask = np.ascontiguousarray(mask, dtype=np.uint8)
    out = np.empty(wq.shape, dtype=np.int8)
    _load().sbl_oracle_apply_mask(_ptr(wq), _ptr(mask), wq.size, _ptr(out))
    return out


def pk2_row_bytes(d_in: int) -> int:
    return int(_load().sbl_oracle_pk2_row_bytes(d_in))


def pack_pk2(weff) -> np.ndarray:
    weff = _i8(weff)
    d_out, d_in = weff.shape
    out = np.empty((d_out, pk2_row_bytes(d_in)), dtype=np.uint8)
    _load().sbl_oracle_pack_pk2(_ptr(weff), d_out, d_in, _ptr(out))
    return out


def nm_value_row_bytes(d_in: int, n: int, m: int) -> int:
    return int(_load().sbl_oracle_nm_value_row_bytes(d_in, n, m))


def nm_bitmap_row_bytes(d_in: int) -> int:
    return int(_load().sbl_oracle_nm_bitmap_row_bytes(d_in))


def pack_nm(weff, mask, n: int, m: int):
    weff = _i8(weff)
    mask = np.ascontiguousarray(mask, dtype=np.uint8)
    d_out, d_in = weff.shape
    vals = np.empty((d_out, nm_value_row_bytes(d_in, n, m)), dtype=np.uint8)
    bm = np.empty((d_out, nm_bitmap_row_bytes(d_in)), dtype=np.uint8)
    _load().sbl_oracle_pack_nm(_ptr(weff), _ptr(mask), d_out, d_in, n, m, _ptr(vals), _ptr(bm))
    return vals, bm


def sp24_value_row_bytes(d_in: int) -> int:
    return int(_load().sbl_oracle_sp24_value_row_bytes(d_in))


def sp24_meta_row_bytes(d_in: int) -> int:
    return int(_load().sbl_oracle_sp24_meta_row_bytes(d_in))


def pack_sp24(weff, mask):
    """2:4-compressed values int8 [O, value_row_bytes] and metadata uint8
    [O, meta_row_bytes]; raises ValueError when the mask is not 2:4."""
    weff = _i8(weff)
    mask = np.ascontiguousarray(mask, dtype=np.uint8)
    d_out, d_in = weff.shape
    vals = np.empty((d_out, sp24_value_row_bytes(d_in)), dtype=np.int8)
    meta = np.empty((d_out, sp24_meta_row_bytes(d_in)), dtype=np.uint8)
    if _load().sbl_oracle_pack_sp24(_ptr(weff), _ptr(mask), d_out, d_in, _ptr(vals), _ptr(meta)) != 0:
        raise ValueError("mask keeps more than two positions in a group of four")
    return vals, meta


def t24_lo_row_bytes(d_in: int) -> int:
    return int(_load().sbl_oracle_t24_lo_row_bytes(d_in))


def t24_hi_row_bytes(d_in: int) -> int:
    return int(_load().sbl_oracle_t24_hi_row_bytes(d_in))


def pack_t24(weff):
    """6-bit group codes of W_eff: low plane uint8 [O, lo_row_bytes] and high
    plane uint8 [O, hi_row_bytes]; raises ValueError when a group of four
    holds more than two nonzeros."""
    weff = _i8(weff)
    d_out, d_in = weff.shape
    lo = np.empty((d_out, t24_lo_row_bytes(d_in)), dtype=np.uint8)
    hi = np.empty((d_out, t24_hi_row_bytes(d_in)), dtype=np.uint8)
    if _load().sbl_oracle_pack_t24(_ptr(weff), d_out, d_in, _ptr(lo), _ptr(hi)) != 0:
        raise ValueError("a group of four holds more than two nonzeros")
    return lo, hi


def gamma_survivors(w, mask) -> np.float32:
    w = _f32(w)
    mask = np.ascontiguousarray(mask, dtype=np.uint8)
    d_out, d_in = w.shape
    return np.float32(_load().sbl_oracle_gamma_survivors(_ptr(w), _ptr(mask), d_out, d_in))


def nm_mask_quantized(wq, n: int, m: int) -> np.ndarray:
    wq = _i8(wq)
    d_out, d_in = wq.shape
    mask = np.empty((d_out, d_in), dtype=np.uint8)
    _load().sbl_oracle_nm_mask_quantized(_ptr(wq), d_out, d_in, n, m, _ptr(mask))
    return mask


def mask_flips(mask_prev, mask) -> int:
    a = np.ascontiguousarray(mask_prev, dtype=np.uint8)
    b = np.ascontiguousarray(mask, dtype=np.uint8)
    assert a.shape == b.shape
    return int(_load().sbl_oracle_mask_flips(_ptr(a), _ptr(b), a.size))


def near_zero(w, g) -> int:
    w = _f32(w)
    return int(_load().sbl_oracle_near_zero(_ptr(w), w.size, float(g)))


def block_threshold(w, mask, m: int) -> np.ndarray:
    w = _f32(w)
    mask = np.ascontiguousarray(mask, dtype=np.uint8)
    d_out, d_in = w.shape
    t = np.empty((d_out, d_in // m), dtype=np.float32)
    _load().sbl_oracle_block_threshold(_ptr(w), _ptr(mask), d_out, d_in, m, _ptr(t))
    return t


def quantize_act(x_bf16_bits):
    """x as uint16 bf16 bit patterns [T, K] -> (q int8 [T, K], d fp32 [T])."""
    x = _u16(x_bf16_bits)
    t, k = x.shape
    q = np.empty((t, k), dtype=np.int8)
    d = np.empty((t,), dtype=np.float32)
    _load().sbl_oracle_quantize_act(_ptr(x), t, k, _ptr(q), _ptr(d))
    return q, d


def gemm_acc(q, weff) -> np.ndarray:
    q, weff = _i8(q), _i8(weff)
    t, k = q.shape
    o, k2 = weff.shape
    assert k == k2
    acc = np.empty((t, o), dtype=np.int32)
    st = _load().sbl_oracle_gemm_acc(_ptr(q), _ptr(weff), t, o, k, _ptr(acc))
    if st != 0:
        raise OverflowError("accumulator does not fit int32")
    return acc


def dequant(acc, g, d):
    """-> (y fp32 [T, O], y bf16 bit patterns uint16 [T, O])."""
    acc = np.ascontiguousarray(acc, dtype=np.int32)
    d = _f32(d)
    t, o = acc.shape
    y = np.empty((t, o), dtype=np.float32)
    yb = np.empty((t, o), dtype=np.uint16)
    _load().sbl_oracle_dequant(_ptr(acc), t, o, float(np.float32(g)), _ptr(d), _ptr(y), _ptr(yb))
    return y, yb


def rmsnorm_quantize_act(x_bf16_bits, g_bf16_bits=None, eps: float = 1e-5):
    """RMSNorm fused with the activation quantiser -> (q int8 [T, K], d fp32 [T])."""
    x = _u16(x_bf16_bits)
    t, k = x.shape
    g = None if g_bf16_bits is None else _u16(g_bf16_bits)
    q = np.empty((t, k), dtype=np.int8)
    d = np.empty((t,), dtype=np.float32)
    _load().sbl_oracle_rmsnorm_quantize_act(_ptr(x), t, k, _ptr(g) if g is not None else None, float(eps),
                                            _ptr(q), _ptr(d))
    return q, d


def epilogue(y, relu2: bool = False, residual_bf16_bits=None):
    """Squared-ReLU and residual epilogue on the fp32 output y -> (fp32,
    bf16 bit patterns)."""
    y = _f32(y)
    t, o = y.shape
    out = np.empty((t, o), dtype=np.float32)
    ob = np.empty((t, o), dtype=np.uint16)
    res = None if residual_bf16_bits is None else _u16(residual_bf16_bits)
    _load().sbl_oracle_epilogue(_ptr(y), t, o, 1 if relu2 else 0, _ptr(res) if res is not None else None,
                                _ptr(out), _ptr(ob))
    return out, ob


def backward(dy_bf16_bits, weff, g, q, d, want_dx=True, want_dw=True):
    """Dual-STE backward in fp64 -> (dX [T, K] or None, dW [O, K] or None)."""
    dy, weff, q, d = _u16(dy_bf16_bits), _i8(weff), _i8(q), _f32(d)
    t, o = dy.shape
    o2, k = weff.shape
    assert o == o2 and q.shape == (t, k) and d.shape == (t,)
    dx = np.empty((t, k), dtype=np.float64) if want_dx else None
    dw = np.empty((o, k), dtype=np.float64) if want_dw else None
    _load().sbl_oracle_backward(
        _ptr(dy), _ptr(weff), float(np.float32(g)), _ptr(q), _ptr(d), t, o, k,
        _ptr(dx) if dx is not None else None, _ptr(dw) if dw is not None else None)
    return dx, dw


def acc_samples(q, weff, idx_t, idx_o) -> np.ndarray:
    q, weff = _i8(q), _i8(weff)
    it = np.ascontiguousarray(idx_t, dtype=np.int64)
    io = np.ascontiguousarray(idx_o, dtype=np.int64)
    out = np.empty(it.shape, dtype=np.int64)
    _load().sbl_oracle_acc_samples(_ptr(q), _ptr(weff), q.shape[1], _ptr(it), _ptr(io), it.size, _ptr(out))
    return out


def dx_samples(dy_bf16_bits, weff, g, idx_t, idx_k) -> np.ndarray:
    dy, weff = _u16(dy_bf16_bits), _i8(weff)
    it = np.ascontiguousarray(idx_t, dtype=np.int64)
    ik = np.ascontiguousarray(idx_k, dtype=np.int64)
    out = np.empty(it.shape, dtype=np.float64)
    _load().sbl_oracle_dx_samples(_ptr(dy), _ptr(weff), float(np.float32(g)), weff.shape[0],
                                  weff.shape[1], _ptr(it), _ptr(ik), it.size, _ptr(out))
    return out


def dw_samples(dy_bf16_bits, q, d, idx_o, idx_k) -> np.ndarray:
    dy, q, d = _u16(dy_bf16_bits), _i8(q), _f32(d)
    io = np.ascontiguousarray(idx_o, dtype=np.int64)
    ik = np.ascontiguousarray(idx_k, dtype=np.int64)
    out = np.empty(io.shape, dtype=np.float64)
    t, o = dy.shape
    _load().sbl_oracle_dw_samples(_ptr(dy), _ptr(q), _ptr(d), t, o, q.shape[1], _ptr(io),
                                  _ptr(ik), io.size, _ptr(out))
    return out


def rounding_is_nearest() -> bool:
    return bool(_load().sbl_oracle_rounding_is_nearest())


class Layer:
    """The whole forward of one Sparse-BitLinear layer, step by step, as the
    oracle computes it (a convenience bundle for tests and the bench)."""

    def __init__(self, w, n: int, m: int, mask_source: str = "master", order: str = "quant_then_mask"):
        """mask_source "master" ranks |W| (the method) or "quantized" ranks
        |W_q|; order "quant_then_mask" takes gamma over all weights (the
        method) or "mask_then_quant" over the survivors ([P1] "Composition
        Order" ablations).  w may be bf16 bits (uint16), read as fp32 exactly."""
        w = np.asarray(w)
        if w.dtype == np.uint16:
            w = (w.astype(np.uint32) << 16).view(np.float32)
        self.w = _f32(w)
        self.n, self.m = n, m
        if mask_source == "quantized" and order == "mask_then_quant":
            raise ValueError("a mask from W_q needs gamma, which mask-then-quant takes from the mask")
        if order == "mask_then_quant":
            self.mask = nm_mask(self.w, n, m)
            self.gamma = gamma_survivors(self.w, self.mask)
            self.wq = ternarize(self.w, self.gamma)
        else:
            self.gamma = gamma(self.w)
            self.wq = ternarize(self.w, self.gamma)
            self.mask = nm_mask(self.w, n, m) if mask_source == "master" else nm_mask_quantized(self.wq, n, m)
        self.weff = apply_mask(self.wq, self.mask)

    def forward(self, x_bf16_bits):
        q, d = quantize_act(x_bf16_bits)
        acc = gemm_acc(q, self.weff)
        y, yb = dequant(acc, self.gamma, d)
        return q, d, acc, y, yb


__all__ = [
    "abs_sum", "gamma", "ternarize", "nm_mask", "apply_mask", "pk2_row_bytes", "pack_pk2",
    "nm_value_row_bytes", "nm_bitmap_row_bytes", "pack_nm", "quantize_act", "gemm_acc",
    "dequant", "backward", "acc_samples", "dx_samples", "dw_samples", "rounding_is_nearest",
    "Layer", "build_oracle", "library_path",
]

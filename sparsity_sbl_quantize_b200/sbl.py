"""Python binding of libsbl.so (include/sbl.h): argument marshalling only.

Every function keeps the C name and takes torch tensors that already live on
the current CUDA device; the work runs in the library's sm_100a kernels on
torch's current stream.  Importing this module loads ``libsbl.so`` from this
directory and raises if it is missing -- there is no CPU fallback.
"""
from __future__ import annotations

import ctypes
import os
from dataclasses import dataclass
from typing import Optional

import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libsbl.so")

if not os.path.exists(LIB_PATH):
    raise ImportError(
        f"{LIB_PATH} is missing: build it with `python -m sparsity_sbl_quantize_b200.build`")

_lib = ctypes.CDLL(LIB_PATH)

SBL_OK = 0
SBL_FMT_PK2, SBL_FMT_NM, SBL_FMT_I8, SBL_FMT_BF16T, SBL_FMT_SP24, SBL_FMT_T24 = 1, 2, 4, 8, 16, 32
SBL_BUF_MAIN, SBL_BUF_NM_BITMAP, SBL_BUF_SP24_META, SBL_BUF_T24_HI = 0, 1, 2, 3
SBL_OP_QUANTIZE_MASK_PACK, SBL_OP_BACKWARD = 0, 1

STATUS_NAMES = {0: "SBL_OK", 1: "SBL_ERR_INVALID_ARG", 2: "SBL_ERR_SHAPE", 3: "SBL_ERR_ALIGNMENT",
                4: "SBL_ERR_UNSUPPORTED", 5: "SBL_ERR_WORKSPACE", 6: "SBL_ERR_CUDA",
                7: "SBL_ERR_DEVICE"}


class sbl_layer_desc(ctypes.Structure):
    _fields_ = [("out_features", ctypes.c_int32), ("in_features", ctypes.c_int32),
                ("n", ctypes.c_int32), ("m", ctypes.c_int32)]


class sbl_packed(ctypes.Structure):
    _fields_ = [("pk2", ctypes.c_void_p), ("nm_values", ctypes.c_void_p),
                ("nm_bitmap", ctypes.c_void_p), ("i8", ctypes.c_void_p),
                ("bf16t", ctypes.c_void_p), ("gamma", ctypes.c_void_p),
                ("sp24_values", ctypes.c_void_p), ("sp24_meta", ctypes.c_void_p),
                ("t24_lo", ctypes.c_void_p), ("t24_hi", ctypes.c_void_p)]


class sbl_pack_variant(ctypes.Structure):
    _fields_ = [("master_dtype", ctypes.c_int32), ("mask_source", ctypes.c_int32), ("order", ctypes.c_int32)]


SBL_GROUP_MAX = 4  # layers of one sbl_forward_group launch

SBL_MASTER_FP32, SBL_MASTER_BF16 = 0, 1
SBL_MASK_FROM_MASTER, SBL_MASK_FROM_QUANTIZED = 0, 1
SBL_QUANT_THEN_MASK, SBL_MASK_THEN_QUANT = 0, 1


class sbl_epilogue(ctypes.Structure):
    _fields_ = [("relu2", ctypes.c_int32), ("residual", ctypes.c_void_p)]


class sbl_mask_stats(ctypes.Structure):
    _fields_ = [("prev_keep", ctypes.c_void_p), ("keep", ctypes.c_void_p), ("flips", ctypes.c_void_p),
                ("near_zero", ctypes.c_void_p), ("block_threshold", ctypes.c_void_p)]


class sbl_host_buffers(ctypes.Structure):
    _fields_ = [(name, ctypes.c_void_p) for name in
                ("pk2", "nm_values", "nm_bitmap", "i8", "bf16t", "sp24_values", "sp24_meta", "t24_lo", "t24_hi")]


class sbl_batch_layer(ctypes.Structure):
    _fields_ = [("desc", sbl_layer_desc), ("pk2", ctypes.c_void_p), ("gamma", ctypes.c_void_p),
                ("xq", ctypes.c_void_p), ("d", ctypes.c_void_p), ("y", ctypes.c_void_p),
                ("y_is_fp32", ctypes.c_int32), ("input_is_previous_output", ctypes.c_int32),
                ("xq_out", ctypes.c_void_p), ("d_out", ctypes.c_void_p)]


SBL_BATCH_MAX_LAYERS = 256

_P = ctypes.c_void_p
_D = ctypes.POINTER(sbl_layer_desc)
_W = ctypes.POINTER(sbl_packed)
_i32, _u32, _sz = ctypes.c_int32, ctypes.c_uint32, ctypes.c_size_t

_lib.sbl_status_string.restype = ctypes.c_char_p
_lib.sbl_status_string.argtypes = [ctypes.c_int]
_lib.sbl_version.restype = _i32
_lib.sbl_packed_row_bytes.restype = _sz
_lib.sbl_packed_row_bytes.argtypes = [_D, ctypes.c_int, ctypes.c_int]
_lib.sbl_workspace_bytes.restype = _sz
_lib.sbl_workspace_bytes.argtypes = [_D, _i32, ctypes.c_int]
_lib.sbl_quantize_mask_pack.restype = ctypes.c_int
_lib.sbl_quantize_mask_pack.argtypes = [_D, _P, _u32, _W, _P, _sz, _P]
_lib.sbl_quantize_mask_pack_stats.restype = ctypes.c_int
_lib.sbl_quantize_mask_pack_stats.argtypes = [_D, _P, _u32, _W, ctypes.POINTER(sbl_mask_stats), _P, _sz, _P]
_lib.sbl_quantize_mask_pack_ex.restype = ctypes.c_int
_lib.sbl_quantize_mask_pack_ex.argtypes = [_D, _P, ctypes.POINTER(sbl_pack_variant), _u32, _W,
                                           ctypes.POINTER(sbl_mask_stats), _P, _sz, _P]
_lib.sbl_backward_dual_ste_ex.restype = ctypes.c_int
_lib.sbl_backward_dual_ste_ex.argtypes = [_D, _P, _P, _P, _i32, _W, _P, _i32, _P, _P, _P, _sz, _P]
_lib.sbl_quantize_mask_pack_noalloc.restype = ctypes.c_int
_lib.sbl_quantize_mask_pack_noalloc.argtypes = [_D, _P, _u32, _W, _P]
_lib.sbl_quantize_act.restype = ctypes.c_int
_lib.sbl_quantize_act.argtypes = [_P, _i32, _i32, _P, _P, _P]
_lib.sbl_quantize_act_rmsnorm.restype = ctypes.c_int
_lib.sbl_quantize_act_rmsnorm.argtypes = [_P, _i32, _i32, _P, ctypes.c_float, _P, _P, _P]
_lib.sbl_forward.restype = ctypes.c_int
_lib.sbl_forward.argtypes = [_D, _P, _P, _i32, _W, ctypes.c_int, _P, _i32, _P, _P]
_lib.sbl_backward_dual_ste.restype = ctypes.c_int
_lib.sbl_forward_group.restype = ctypes.c_int
_lib.sbl_forward_group.argtypes = [ctypes.POINTER(_D), _i32, _P, _P, _i32, ctypes.POINTER(_W), ctypes.POINTER(_P),
                                   _i32, _P]
_lib.sbl_backward_dual_ste.argtypes = [_D, _P, _P, _P, _i32, _W, _P, _i32, _P, _P, _sz, _P]
_lib.sbl_forward_ex.restype = ctypes.c_int
_lib.sbl_forward_ex.argtypes = [_D, _P, _P, _i32, _W, ctypes.c_int, _P, _i32, _P, ctypes.POINTER(sbl_epilogue), _P]
_lib.sbl_linear_forward.restype = ctypes.c_int
_lib.sbl_linear_forward.argtypes = [_D, _P, _i32, _W, ctypes.c_int, _P, _P, _P, _i32,
                                    ctypes.POINTER(sbl_epilogue), _P]
_lib.sbl_forward_batch_workspace_bytes.restype = _sz
_lib.sbl_forward_batch_workspace_bytes.argtypes = [ctypes.POINTER(sbl_batch_layer), _i32, _i32]
_lib.sbl_forward_batch.restype = ctypes.c_int
_lib.sbl_forward_batch.argtypes = [ctypes.POINTER(sbl_batch_layer), _i32, _i32, _P, _sz, _P]
_lib.sbl_gamma_node_count.restype = _sz
_lib.sbl_gamma_node_count.argtypes = [_D]
_lib.sbl_gamma_partials.restype = ctypes.c_int
_lib.sbl_gamma_partials.argtypes = [_D, _P, ctypes.c_int64, _P, _P, _sz, _P]
_lib.sbl_gamma_combine.restype = ctypes.c_int
_lib.sbl_gamma_combine.argtypes = [_P, ctypes.c_int64, ctypes.c_int64, _P, _P]
_lib.sbl_quantize_mask_pack_shard.restype = ctypes.c_int
_lib.sbl_quantize_mask_pack_shard.argtypes = [_D, _P, _u32, _W, _P]
_lib.sbl_forward_format.restype = ctypes.c_int
_lib.sbl_forward_format.argtypes = [_D, _i32]
_lib.sbl_device_error.restype = ctypes.c_int
_lib.sbl_device_error.argtypes = [ctypes.POINTER(_u32), _i32]
_lib.sbl_selftest_wait_expiry.restype = ctypes.c_int
_lib.sbl_selftest_wait_expiry.argtypes = [_P]
_lib.sbl_container_bytes.restype = _sz
_lib.sbl_container_bytes.argtypes = [_D, _u32]
_lib.sbl_container_write.restype = ctypes.c_int
_lib.sbl_container_write.argtypes = [_D, _u32, ctypes.c_float, ctypes.POINTER(sbl_host_buffers), _P, _sz]
_lib.sbl_container_info.restype = ctypes.c_int
_lib.sbl_container_info.argtypes = [_P, _sz, _D, ctypes.POINTER(_u32), ctypes.POINTER(ctypes.c_float)]
_lib.sbl_container_read.restype = ctypes.c_int
_lib.sbl_container_read.argtypes = [_P, _sz, ctypes.POINTER(sbl_host_buffers)]

EXPORTED = ["sbl_status_string", "sbl_version", "sbl_packed_row_bytes", "sbl_workspace_bytes",
            "sbl_quantize_mask_pack", "sbl_quantize_mask_pack_stats", "sbl_quantize_mask_pack_noalloc", "sbl_quantize_act", "sbl_quantize_act_rmsnorm", "sbl_forward", "sbl_linear_forward",
            "sbl_forward_ex", "sbl_forward_group", "sbl_forward_format", "sbl_forward_batch",
            "sbl_forward_batch_workspace_bytes",
            "sbl_gamma_node_count", "sbl_gamma_partials", "sbl_gamma_combine", "sbl_quantize_mask_pack_shard",
            "sbl_backward_dual_ste", "sbl_backward_dual_ste_ex",
            "sbl_quantize_mask_pack_ex", "sbl_device_error", "sbl_selftest_wait_expiry", "sbl_container_bytes",
            "sbl_container_write",
            "sbl_container_info", "sbl_container_read"]


class SblError(RuntimeError):
    def __init__(self, status: int, call: str):
        self.status = status
        msg = _lib.sbl_status_string(status).decode()
        super().__init__(f"{call}: {STATUS_NAMES.get(status, status)} ({msg})")


def _check(status: int, call: str):
    if status != SBL_OK:
        raise SblError(status, call)


def _ptr(t: Optional[torch.Tensor]):
    if t is None:
        return None
    return ctypes.c_void_p(t.data_ptr())


def _stream():
    return ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)


def desc(out_features: int, in_features: int, n: int, m: int) -> sbl_layer_desc:
    return sbl_layer_desc(out_features, in_features, n, m)


@dataclass
class Packed:
    """Device buffers of one packed layer (torch tensors; None = absent)."""
    gamma: torch.Tensor
    pk2: Optional[torch.Tensor] = None
    nm_values: Optional[torch.Tensor] = None
    nm_bitmap: Optional[torch.Tensor] = None
    i8: Optional[torch.Tensor] = None
    bf16t: Optional[torch.Tensor] = None
    sp24_values: Optional[torch.Tensor] = None
    sp24_meta: Optional[torch.Tensor] = None
    t24_lo: Optional[torch.Tensor] = None
    t24_hi: Optional[torch.Tensor] = None

    def c(self) -> sbl_packed:
        return sbl_packed(*[(t.data_ptr() if t is not None else None)
                            for t in (self.pk2, self.nm_values, self.nm_bitmap, self.i8, self.bf16t,
                                      self.gamma, self.sp24_values, self.sp24_meta, self.t24_lo, self.t24_hi)])


# ------------------------------------------------------------------ C calls

def sbl_status_string(status: int) -> str:
    return _lib.sbl_status_string(status).decode()


def sbl_version() -> int:
    return int(_lib.sbl_version())


def sbl_packed_row_bytes(d: sbl_layer_desc, fmt: int, which: int = SBL_BUF_MAIN) -> int:
    return int(_lib.sbl_packed_row_bytes(ctypes.byref(d), fmt, which))


def sbl_workspace_bytes(d: sbl_layer_desc, tokens: int, op: int) -> int:
    return int(_lib.sbl_workspace_bytes(ctypes.byref(d), tokens, op))


def sbl_quantize_mask_pack(d: sbl_layer_desc, W: torch.Tensor, formats: int, out: Packed,
                           workspace: torch.Tensor) -> None:
    cp = out.c()
    _check(_lib.sbl_quantize_mask_pack(ctypes.byref(d), _ptr(W), formats, ctypes.byref(cp),
                                       _ptr(workspace), workspace.numel() * workspace.element_size(),
                                       _stream()), "sbl_quantize_mask_pack")


def sbl_quantize_mask_pack_stats(d: sbl_layer_desc, W: torch.Tensor, formats: int, p: Packed,
                                 workspace: torch.Tensor, prev_keep: Optional[torch.Tensor] = None,
                                 keep: Optional[torch.Tensor] = None, flips: Optional[torch.Tensor] = None,
                                 near_zero: Optional[torch.Tensor] = None,
                                 block_threshold: Optional[torch.Tensor] = None):
    """sbl_quantize_mask_pack plus re-mask statistics; flips / near_zero are
    one-element int64 device tensors (read as uint64)."""
    st = sbl_mask_stats(*[(t.data_ptr() if t is not None else None)
                          for t in (prev_keep, keep, flips, near_zero, block_threshold)])
    cp = p.c()
    _check(_lib.sbl_quantize_mask_pack_stats(ctypes.byref(d), _ptr(W), formats, ctypes.byref(cp), ctypes.byref(st),
                                             _ptr(workspace), workspace.numel() * workspace.element_size(), _stream()),
           "sbl_quantize_mask_pack_stats")


def sbl_quantize_mask_pack_ex(d: sbl_layer_desc, W: torch.Tensor, formats: int, p: Packed, workspace: torch.Tensor,
                              mask_source: int = SBL_MASK_FROM_MASTER, order: int = SBL_QUANT_THEN_MASK,
                              prev_keep: Optional[torch.Tensor] = None, keep: Optional[torch.Tensor] = None,
                              flips: Optional[torch.Tensor] = None, near_zero: Optional[torch.Tensor] = None,
                              block_threshold: Optional[torch.Tensor] = None):
    """Packing with a weight-side variant; W is float32 or bfloat16."""
    dtype = SBL_MASTER_BF16 if W.dtype == torch.bfloat16 else SBL_MASTER_FP32
    v = sbl_pack_variant(dtype, mask_source, order)
    st = sbl_mask_stats(*[(t.data_ptr() if t is not None else None)
                          for t in (prev_keep, keep, flips, near_zero, block_threshold)])
    cp = p.c()
    _check(_lib.sbl_quantize_mask_pack_ex(ctypes.byref(d), _ptr(W), ctypes.byref(v), formats, ctypes.byref(cp),
                                          ctypes.byref(st), _ptr(workspace), workspace.numel() * workspace.element_size(),
                                          _stream()), "sbl_quantize_mask_pack_ex")


def keep_bitmap_bytes(d: sbl_layer_desc) -> int:
    """Bytes per row of the keep bitmap of sbl_mask_stats (the NM bitmap layout)."""
    return sbl_packed_row_bytes(d, SBL_FMT_NM, SBL_BUF_NM_BITMAP)


def sbl_quantize_mask_pack_noalloc(d: sbl_layer_desc, W: torch.Tensor, formats: int, out: Packed) -> None:
    """sbl_quantize_mask_pack without a caller workspace: for callers that
    cannot obtain device memory where they call the layer (the library uses
    its own static per-device scratch; calls must not overlap on the GPU)."""
    cp = out.c()
    _check(_lib.sbl_quantize_mask_pack_noalloc(ctypes.byref(d), _ptr(W), formats, ctypes.byref(cp),
                                               _stream()), "sbl_quantize_mask_pack_noalloc")


def sbl_quantize_act(X: torch.Tensor, T: int, K: int, Xq: torch.Tensor, d: torch.Tensor) -> None:
    _check(_lib.sbl_quantize_act(_ptr(X), T, K, _ptr(Xq), _ptr(d), _stream()), "sbl_quantize_act")


def sbl_quantize_act_rmsnorm(X: torch.Tensor, T: int, K: int, g: Optional[torch.Tensor], eps: float,
                             Xq: torch.Tensor, d: torch.Tensor) -> None:
    _check(_lib.sbl_quantize_act_rmsnorm(_ptr(X), T, K, _ptr(g), float(eps), _ptr(Xq), _ptr(d), _stream()),
           "sbl_quantize_act_rmsnorm")


def sbl_forward(dsc: sbl_layer_desc, Xq: torch.Tensor, d: torch.Tensor, T: int, w: Packed, fmt: int,
                Y: torch.Tensor, y_is_fp32: bool = False, acc_out: Optional[torch.Tensor] = None) -> None:
    cp = w.c()
    _check(_lib.sbl_forward(ctypes.byref(dsc), _ptr(Xq), _ptr(d), T, ctypes.byref(cp), fmt, _ptr(Y),
                            1 if y_is_fp32 else 0, _ptr(acc_out), _stream()), "sbl_forward")


def sbl_forward_group(descs, Xq: torch.Tensor, d: torch.Tensor, T: int, ws, Ys, y_is_fp32: bool = False) -> None:
    """The SBL_FMT_I8 forward of several layers on the same activations in
    one launch: descs, ws (Packed) and Ys are equal-length sequences."""
    n = len(descs)
    cps = [w.c() for w in ws]
    darr = (_D * n)(*[ctypes.pointer(x) for x in descs])
    warr = (_W * n)(*[ctypes.pointer(c) for c in cps])
    yarr = (_P * n)(*[_ptr(y) for y in Ys])
    _check(_lib.sbl_forward_group(darr, n, _ptr(Xq), _ptr(d), T, warr, yarr, 1 if y_is_fp32 else 0, _stream()),
           "sbl_forward_group")


def sbl_forward_ex(dsc: sbl_layer_desc, Xq: torch.Tensor, d: torch.Tensor, T: int, w: Packed, fmt: int,
                   Y: torch.Tensor, relu2: bool = False, residual: Optional[torch.Tensor] = None,
                   acc_out: Optional[torch.Tensor] = None) -> None:
    """sbl_forward with the Squared-ReLU / residual output epilogue."""
    cp = w.c()
    epi = sbl_epilogue(1 if relu2 else 0, residual.data_ptr() if residual is not None else None)
    y_fp32 = 1 if Y.dtype == torch.float32 else 0
    _check(_lib.sbl_forward_ex(ctypes.byref(dsc), _ptr(Xq), _ptr(d), T, ctypes.byref(cp), fmt, _ptr(Y), y_fp32,
                               _ptr(acc_out), ctypes.byref(epi), _stream()), "sbl_forward_ex")


def sbl_linear_forward(dsc: sbl_layer_desc, X: torch.Tensor, T: int, w: Packed, fmt: int, Xq: torch.Tensor,
                       d: torch.Tensor, Y: torch.Tensor, relu2: bool = False,
                       residual: Optional[torch.Tensor] = None) -> None:
    """Q_a(X) -> Xq, d, then the forward into Y (one launch for the PK2 decode)."""
    cp = w.c()
    epi = sbl_epilogue(1 if relu2 else 0, residual.data_ptr() if residual is not None else None)
    y_fp32 = 1 if Y.dtype == torch.float32 else 0
    _check(_lib.sbl_linear_forward(ctypes.byref(dsc), _ptr(X), T, ctypes.byref(cp), fmt, _ptr(Xq), _ptr(d),
                                   _ptr(Y), y_fp32, ctypes.byref(epi), _stream()), "sbl_linear_forward")


def sbl_backward_dual_ste(dsc: sbl_layer_desc, dY: torch.Tensor, Xq: Optional[torch.Tensor],
                          d: Optional[torch.Tensor], T: int, w: Packed, dX: Optional[torch.Tensor],
                          dx_is_fp32: bool, dW: Optional[torch.Tensor],
                          workspace: Optional[torch.Tensor]) -> None:
    cp = w.c()
    nbytes = 0 if workspace is None else workspace.numel() * workspace.element_size()
    _check(_lib.sbl_backward_dual_ste(ctypes.byref(dsc), _ptr(dY), _ptr(Xq), _ptr(d), T,
                                      ctypes.byref(cp), _ptr(dX), 1 if dx_is_fp32 else 0, _ptr(dW),
                                      _ptr(workspace), nbytes, _stream()), "sbl_backward_dual_ste")


def sbl_backward_dual_ste_ex(d: sbl_layer_desc, dY: torch.Tensor, Xq: torch.Tensor, dvec: torch.Tensor, T: int,
                             p: Packed, dX: Optional[torch.Tensor], dx_fp32: bool, dW: Optional[torch.Tensor],
                             dw_keep: Optional[torch.Tensor], workspace: Optional[torch.Tensor]):
    """The backward with dW gated by a keep bitmap (the pages' mask-gated ablation)."""
    cp = p.c()
    ws_bytes = workspace.numel() * workspace.element_size() if workspace is not None else 0
    _check(_lib.sbl_backward_dual_ste_ex(ctypes.byref(d), _ptr(dY), _ptr(Xq), _ptr(dvec), T, ctypes.byref(cp),
                                         _ptr(dX), 1 if dx_fp32 else 0, _ptr(dW), _ptr(dw_keep), _ptr(workspace),
                                         ws_bytes, _stream()), "sbl_backward_dual_ste_ex")


def sbl_device_error(clear: bool = False) -> int:
    code = _u32(0)
    _check(_lib.sbl_device_error(ctypes.byref(code), 1 if clear else 0), "sbl_device_error")
    return int(code.value)


SBL_DEVICE_ERROR_SELFTEST = 0x80000000


def sbl_selftest_wait_expiry() -> None:
    """Enqueue the bounded-wait self-test; its bit appears in sbl_device_error."""
    _check(_lib.sbl_selftest_wait_expiry(_stream()), "sbl_selftest_wait_expiry")


# ------------------------------------------------- allocation helpers (torch)

def batch_layer(dsc: sbl_layer_desc, w: "Packed", Y: torch.Tensor, Xq: Optional[torch.Tensor] = None,
                d: Optional[torch.Tensor] = None, y_is_fp32: bool = False, chained: bool = False,
                xq_out: Optional[torch.Tensor] = None, d_out: Optional[torch.Tensor] = None) -> sbl_batch_layer:
    """One entry of a batched decode forward (the tensors must outlive the call)."""
    def addr(t):
        return t.data_ptr() if t is not None else None
    return sbl_batch_layer(dsc, w.pk2.data_ptr(), w.gamma.data_ptr(), addr(Xq), addr(d), Y.data_ptr(),
                           1 if y_is_fp32 else 0, 1 if chained else 0, addr(xq_out), addr(d_out))


def batch_array(layers) -> ctypes.Array:
    return (sbl_batch_layer * len(layers))(*layers)


def sbl_forward_batch_workspace_bytes(layers: ctypes.Array, count: int, T: int) -> int:
    return int(_lib.sbl_forward_batch_workspace_bytes(layers, count, T))


def sbl_forward_batch(layers: ctypes.Array, count: int, T: int, workspace: Optional[torch.Tensor] = None) -> None:
    nbytes = workspace.numel() * workspace.element_size() if workspace is not None else 0
    _check(_lib.sbl_forward_batch(layers, count, T, _ptr(workspace), nbytes, _stream()), "sbl_forward_batch")


def sbl_gamma_node_count(shard: sbl_layer_desc) -> int:
    return int(_lib.sbl_gamma_node_count(ctypes.byref(shard)))


def sbl_gamma_partials(shard: sbl_layer_desc, W: torch.Tensor, first_row: int, node_sums: torch.Tensor,
                       workspace: torch.Tensor) -> None:
    _check(_lib.sbl_gamma_partials(ctypes.byref(shard), _ptr(W), first_row, _ptr(node_sums), _ptr(workspace),
                                   workspace.numel() * workspace.element_size(), _stream()), "sbl_gamma_partials")


def sbl_gamma_combine(node_sums: torch.Tensor, nodes: int, total_weights: int, gamma: torch.Tensor) -> None:
    _check(_lib.sbl_gamma_combine(_ptr(node_sums), nodes, total_weights, _ptr(gamma), _stream()),
           "sbl_gamma_combine")


def sbl_quantize_mask_pack_shard(shard: sbl_layer_desc, W: torch.Tensor, formats: int, out: "Packed") -> None:
    cp = out.c()
    _check(_lib.sbl_quantize_mask_pack_shard(ctypes.byref(shard), _ptr(W), formats, ctypes.byref(cp), _stream()),
           "sbl_quantize_mask_pack_shard")


def sbl_forward_format(d: sbl_layer_desc, tokens: int) -> int:
    return int(_lib.sbl_forward_format(ctypes.byref(d), tokens))


def alloc_packed(d: sbl_layer_desc, formats: int, device="cuda") -> Packed:
    """Allocate (with torch) the buffers sbl_quantize_mask_pack writes."""
    O, K = d.out_features, d.in_features
    p = Packed(gamma=torch.empty(4, dtype=torch.float32, device=device))
    if formats & SBL_FMT_PK2:
        p.pk2 = torch.empty((O, sbl_packed_row_bytes(d, SBL_FMT_PK2)), dtype=torch.uint8, device=device)
    if formats & SBL_FMT_NM:
        p.nm_values = torch.empty((O, sbl_packed_row_bytes(d, SBL_FMT_NM)), dtype=torch.uint8, device=device)
        p.nm_bitmap = torch.empty((O, sbl_packed_row_bytes(d, SBL_FMT_NM, SBL_BUF_NM_BITMAP)),
                                  dtype=torch.uint8, device=device)
    if formats & SBL_FMT_I8:
        p.i8 = torch.empty((O, K), dtype=torch.int8, device=device)
    if formats & SBL_FMT_BF16T:
        p.bf16t = torch.empty((K, O), dtype=torch.bfloat16, device=device)
    if formats & SBL_FMT_SP24:
        p.sp24_values = torch.empty((O, sbl_packed_row_bytes(d, SBL_FMT_SP24)), dtype=torch.int8, device=device)
        p.sp24_meta = torch.empty((O, sbl_packed_row_bytes(d, SBL_FMT_SP24, SBL_BUF_SP24_META)),
                                  dtype=torch.uint8, device=device)
    if formats & SBL_FMT_T24:
        p.t24_lo = torch.empty((O, sbl_packed_row_bytes(d, SBL_FMT_T24)), dtype=torch.uint8, device=device)
        p.t24_hi = torch.empty((O, sbl_packed_row_bytes(d, SBL_FMT_T24, SBL_BUF_T24_HI)),
                               dtype=torch.uint8, device=device)
    return p


def alloc_workspace(nbytes: int, device="cuda") -> torch.Tensor:
    """Workspace as a 256-byte aligned torch buffer (torch's allocator aligns to 512)."""
    return torch.empty(max(nbytes, 256), dtype=torch.uint8, device=device)


# ------------------------------------------- packed-layer container (host)

_BUFFERS = ("pk2", "nm_values", "nm_bitmap", "i8", "bf16t", "sp24_values", "sp24_meta", "t24_lo", "t24_hi")


def _host_buffers(p: Packed) -> sbl_host_buffers:
    """sbl_host_buffers over the host (CPU, contiguous) tensors of p."""
    ptrs = []
    for name in _BUFFERS:
        t = getattr(p, name)
        if t is not None and (t.is_cuda or not t.is_contiguous()):
            raise ValueError(f"{name}: the container works on contiguous host tensors")
        ptrs.append(t.data_ptr() if t is not None else None)
    return sbl_host_buffers(*ptrs)


def sbl_container_bytes(d: sbl_layer_desc, formats: int) -> int:
    return int(_lib.sbl_container_bytes(ctypes.byref(d), formats))


def sbl_container_write(d: sbl_layer_desc, formats: int, gamma: float, src: Packed) -> bytes:
    """The container image of a packed layer whose buffers are host tensors."""
    n = sbl_container_bytes(d, formats)  # 0 for an invalid descriptor or mask: the call reports which
    buf = ctypes.create_string_buffer(max(n, 1))
    hb = _host_buffers(src)
    _check(_lib.sbl_container_write(ctypes.byref(d), formats, float(gamma), ctypes.byref(hb), buf, n),
           "sbl_container_write")
    return buf.raw


def sbl_container_info(image: bytes):
    """(desc, formats, gamma) of a checked container image."""
    d = sbl_layer_desc()
    f = _u32(0)
    g = ctypes.c_float(0.0)
    _check(_lib.sbl_container_info(image, len(image), ctypes.byref(d), ctypes.byref(f), ctypes.byref(g)),
           "sbl_container_info")
    return d, int(f.value), float(g.value)


def sbl_container_read(image: bytes, dst: Packed) -> None:
    """Copy the stored buffers of a checked image into dst's host tensors."""
    hb = _host_buffers(dst)
    _check(_lib.sbl_container_read(image, len(image), ctypes.byref(hb)), "sbl_container_read")


def save_packed(path: str, d: sbl_layer_desc, formats: int, p: Packed) -> None:
    """Store a packed layer (device or host tensors) with its descriptor and
    gamma; the device buffers are copied to host memory first."""
    host = Packed(gamma=p.gamma.detach().cpu(),
                  **{name: (getattr(p, name).detach().cpu().contiguous() if getattr(p, name) is not None else None)
                     for name in _BUFFERS})
    image = sbl_container_write(d, formats, float(host.gamma.reshape(-1)[0]), host)
    with open(path, "wb") as f:
        f.write(image)


def load_packed(path: str, device="cuda"):
    """Read a stored packed layer: (desc, formats, Packed on `device`)."""
    with open(path, "rb") as f:
        image = f.read()
    d, formats, gamma = sbl_container_info(image)
    host = alloc_packed(d, formats, device="cpu")
    sbl_container_read(image, host)
    host.gamma.zero_()
    host.gamma[0] = gamma
    if device == "cpu":
        return d, formats, host
    dev = Packed(gamma=host.gamma.to(device),
                 **{name: (getattr(host, name).to(device) if getattr(host, name) is not None else None)
                    for name in _BUFFERS})
    return d, formats, dev

"""Python binding of libsp24 (the C ABI declared in include/sp24.h).

Argument marshalling only: every step of the pipeline runs in the CUDA kernels of
``libsp24.so``.  PyTorch supplies device memory and the current stream.  There is no CPU path:
the functions accept CUDA tensors only and raise when the library cannot be loaded.

Pipeline ([P1] "NVFP4 vs 2:4 sparse: where the other half of the petaflop went",
[P2] "Sparse GPU FLOPS Need the Right Zeros in the Right Places", [P5] "NVFP4 Without FP4
Hardware"):

    check_24 -> prune_compress_24 -> quantize_nvfp4 -> gemm_dense / gemm_sparse24
"""
from __future__ import annotations

import ctypes
import os
import threading
from typing import NamedTuple, Optional

import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libsp24.so")

# status codes (include/sp24.h)
OK, ERR_INVALID_ARG, ERR_SHAPE, ERR_DTYPE, ERR_ALIGN, ERR_UNSUPPORTED, ERR_CUDA, \
    ERR_DEVICE_TIMEOUT, ERR_WORKSPACE = range(9)
F16, BF16, F32, NVFP4, NVFP4_B32, NVFP4_MMA, NVFP4_B32_MMA = 0, 1, 2, 3, 4, 5, 6
OP_MATMUL, OP_CONV = 0, 1
ALGO_AUTO, ALGO_SKINNY, ALGO_TILED = 0, 1, 2

EXPORTS = ("sp24_status_string", "sp24_abi_version", "sp24_sizes", "sp24_check_24",
           "sp24_prune_compress_24", "sp24_decompress_24", "sp24_quantize_nvfp4_workspace_size",
           "sp24_quantize_nvfp4", "sp24_dequantize_nvfp4", "sp24_gemm_workspace_size",
           "sp24_gemm_dense", "sp24_gemm_sparse24", "sp24_kernel_launches",
           "sp24_last_device_error", "sp24_quantize_nvfp4_noalloc", "sp24_gemm_grouped_workspace_size",
           "sp24_gemm_grouped", "sp24_prepare_24_workspace_size", "sp24_prepare_24",
           "sp24_quantize_nvfp4_pair", "sp24_nvfp4_group_tensor_scale_workspace_size",
           "sp24_nvfp4_group_tensor_scale", "sp24_gemm_select", "sp24_gemm_choice", "sp24_gemm_auto",
           "sp24_gemm_choice_reset", "sp24_moe_block_workspace_size", "sp24_moe_block",
           "sp24_interleave_rows", "sp24_check_48", "sp24_prune_compress_48", "sp24_decompress_48",
           "sp24_quantize_nvfp4_block32", "sp24_gemm_sparse48")

_lock = threading.Lock()
_lib = None


class SP24Error(RuntimeError):
    def __init__(self, status: int, where: str):
        self.status = status
        msg = _lib.sp24_status_string(status).decode() if _lib is not None else str(status)
        super().__init__(f"{where}: {msg} (status {status})")


class _Operand(ctypes.Structure):
    _fields_ = [("format", ctypes.c_int32), ("data", ctypes.c_void_p),
                ("scales", ctypes.c_void_p), ("tensor_scale", ctypes.c_void_p)]


class _SparseOperand(ctypes.Structure):
    _fields_ = [("format", ctypes.c_int32), ("values", ctypes.c_void_p),
                ("scales", ctypes.c_void_p), ("tensor_scale", ctypes.c_void_p),
                ("meta", ctypes.c_void_p)]


def lib() -> ctypes.CDLL:
    """Loads libsp24.so (building it in-tree first if it is missing or older than a source)."""
    global _lib
    with _lock:
        if _lib is None:
            from . import build as _build
            if _build.stale():
                _build.build()
            L = ctypes.CDLL(LIB_PATH)
            P, I, I64 = ctypes.c_void_p, ctypes.c_int, ctypes.c_int64
            L.sp24_status_string.restype = ctypes.c_char_p
            L.sp24_status_string.argtypes = [I]
            L.sp24_sizes.argtypes = [I, I, P, I, P, P, P, P, P]
            L.sp24_check_24.argtypes = [P, I, I, P, I, P, P, P]
            L.sp24_prune_compress_24.argtypes = [P, I, I, P, I, P, P, P]
            L.sp24_decompress_24.argtypes = [P, P, I, I, P, I, P, P]
            L.sp24_quantize_nvfp4_workspace_size.argtypes = [I64, I64, P]
            L.sp24_quantize_nvfp4.argtypes = [P, I, I64, I64, P, P, P, P, P, I64, P]
            L.sp24_dequantize_nvfp4.argtypes = [P, P, P, I64, I64, I, P, P]
            L.sp24_quantize_nvfp4_noalloc.argtypes = [P, I, I64, I64, P, P, P, P, P]
            L.sp24_gemm_workspace_size.argtypes = [I, I, I, I64, I64, I64, I, P]
            L.sp24_gemm_dense.argtypes = [ctypes.POINTER(_Operand), ctypes.POINTER(_Operand), I64,
                                          I64, I64, P, P, I64, I, P]
            L.sp24_gemm_sparse24.argtypes = [ctypes.POINTER(_Operand),
                                             ctypes.POINTER(_SparseOperand), I64, I64, I64, P, P,
                                             I64, I, P]
            L.sp24_last_device_error.argtypes = [P]
            L.sp24_gemm_grouped_workspace_size.argtypes = [I64, I, I64, P]
            L.sp24_gemm_grouped.argtypes = [ctypes.POINTER(_Operand), P, I64, I, ctypes.POINTER(_Operand),
                                             ctypes.POINTER(_SparseOperand), I64, I64, I64, P, P, I64, P]
            L.sp24_prepare_24_workspace_size.argtypes = [I64, I64, P]
            L.sp24_prepare_24.argtypes = [P, I, I64, I64, P, P, P, P, P, P, P, I64, P]
            L.sp24_quantize_nvfp4_pair.argtypes = [P, I, I64, I64, P, P, P, P, P, I64, I64, P, P, P, P, P]
            L.sp24_nvfp4_group_tensor_scale_workspace_size.argtypes = [P]
            L.sp24_nvfp4_group_tensor_scale.argtypes = [P, P, I, I, P, P, I64, P]
            L.sp24_gemm_select.argtypes = [ctypes.POINTER(_Operand), ctypes.POINTER(_Operand),
                                           ctypes.POINTER(_SparseOperand), I64, I64, I64, P, P, I64, I,
                                           P, P, P, P]
            L.sp24_gemm_choice.argtypes = [I, I, I64, I64, I64, P, P]
            L.sp24_gemm_auto.argtypes = [ctypes.POINTER(_Operand), ctypes.POINTER(_Operand),
                                         ctypes.POINTER(_SparseOperand), I64, I64, I64, P, P, I64, P, P]
            L.sp24_gemm_choice_reset.argtypes = []
            L.sp24_moe_block_workspace_size.argtypes = [I64, I, I64, I64, I64, P]
            L.sp24_moe_block.argtypes = [ctypes.POINTER(_Operand), P, P, I64, I, ctypes.POINTER(_Operand),
                                         ctypes.POINTER(_SparseOperand), ctypes.POINTER(_Operand),
                                         ctypes.POINTER(_SparseOperand), I64, I64, I64, P, P, I64, P]
            L.sp24_interleave_rows.argtypes = [P, P, I64, I64, I64, P, P]
            L.sp24_check_48.argtypes = [P, I, I64, I64, P, P, P]
            L.sp24_prune_compress_48.argtypes = [P, I, I64, I64, P, P, P]
            L.sp24_decompress_48.argtypes = [P, P, I, I64, I64, P, P]
            L.sp24_quantize_nvfp4_block32.argtypes = [P, I, I64, I64, P, P, P, P, P, I64, P]
            L.sp24_gemm_sparse48.argtypes = [ctypes.POINTER(_Operand), ctypes.POINTER(_SparseOperand), I64, I64,
                                             I64, P, P]
            L.sp24_nvfp4_mma_size.argtypes = [I64, I64, P, P]
            L.sp24_nvfp4_to_mma.argtypes = [P, P, I64, I64, P, P, P]
            L.sp24_set_wait_limit.argtypes = [ctypes.c_ulonglong]
            L.sp24_get_wait_limit.argtypes = [P]
            L.sp24_selftest_wait_timeout.argtypes = [P, P, P]
            L.sp24_nvfp4_b32_mma_size.argtypes = [I64, I64, P, P]
            L.sp24_nvfp4_b32_to_mma.argtypes = [P, P, I64, I64, P, P, P]
            L.sp24_sparse48_mma_size.argtypes = [I64, I64, P, P, P]
            L.sp24_prepare_sparse_size.argtypes = [I64, I64, P]
            L.sp24_prepare_sparse.argtypes = [P, I64, I64, P, P]
            L.sp24_sparse48_to_mma.argtypes = [P, P, P, I64, I64, P, P, P, P]
            L.sp24_peak_mma.argtypes = [I, I, P, P]
            L.sp24_peak_ctas.argtypes = [I]
            L.sp24_peak_read.argtypes = [P, I64, P, P]
            L.sp24_kernel_launches.restype = I64
            L.sp24_kernel_launches.argtypes = []
            _lib = L
    return _lib


# ---------------------------------------------------------------------------- marshalling

_DT = {torch.float16: F16, torch.bfloat16: BF16, torch.float32: F32}
_TORCH = {F16: torch.float16, BF16: torch.bfloat16, F32: torch.float32}


def _dtype_code(t: torch.Tensor) -> int:
    try:
        return _DT[t.dtype]
    except KeyError:
        raise TypeError(f"unsupported dtype {t.dtype}") from None


def _cuda(t: torch.Tensor, name: str) -> torch.Tensor:
    if not isinstance(t, torch.Tensor) or not t.is_cuda:
        raise ValueError(f"{name} must be a CUDA tensor (this library has no CPU path)")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")
    return t


def _ptr(t: Optional[torch.Tensor]):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _stream(stream=None):
    s = stream if stream is not None else torch.cuda.current_stream()
    return ctypes.c_void_p(s.cuda_stream)


def _shape(shape) -> ctypes.Array:
    arr = (ctypes.c_int64 * 4)()
    for i, s in enumerate(shape):
        arr[i] = int(s)
    return arr


def _call(fn: str, *args) -> None:
    st = getattr(lib(), fn)(*args)
    if st != OK:
        raise SP24Error(st, fn)


def _groups(op: int, shape) -> int:
    shape = tuple(int(s) for s in shape)
    if op == OP_MATMUL:
        n = 1
        for s in shape:
            n *= s
        return n // 4
    K, C, R, S = shape
    return K * (C // 4) * R * S


def group_shape(op: int, shape) -> tuple:
    shape = tuple(int(s) for s in shape)
    if op == OP_MATMUL:
        return shape[:-1] + (shape[-1] // 4,)
    K, C, R, S = shape
    return (K, C // 4, R, S)


def values_shape(op: int, shape) -> tuple:
    shape = tuple(int(s) for s in shape)
    if op == OP_MATMUL:
        return shape[:-1] + (shape[-1] // 2,)
    K, C, R, S = shape
    return (K, C // 2, R, S)


class NVFP4Tensor(NamedTuple):
    """codes uint8 [rows, cols/2], scales uint8 [rows, cols/16], tensor_scale fp32 [1]."""
    codes: torch.Tensor
    scales: torch.Tensor
    tensor_scale: torch.Tensor


class NVFP4MMA(NamedTuple):
    """An NVFP4 tensor as the W4A4 GEMM's tile images (see to_mma): codes and scales are flat
    uint8 tensors (rows padded to a multiple of 128), tensor_scale fp32 [1]; rows, cols the
    logical shape."""
    codes: torch.Tensor
    scales: torch.Tensor
    tensor_scale: torch.Tensor
    rows: int
    cols: int


class Sparse24(NamedTuple):
    """A 2:4-compressed weight [N, K]: values ([N, K/2] 16-bit, or NVFP4 of them) + meta."""
    values: object  # torch.Tensor (16-bit) or NVFP4Tensor
    meta: torch.Tensor


# ---------------------------------------------------------------------------- a1 .. a3

def check_24(w: torch.Tensor, op: int = OP_MATMUL, pass_out=None, n_fail_out=None, stream=None):
    """Per-group eligibility (uint8 0/1) and the failing-group count (int32 [1], device)."""
    _cuda(w, "w")
    if pass_out is None:
        pass_out = torch.empty(group_shape(op, w.shape), dtype=torch.uint8, device=w.device)
    if n_fail_out is None:
        n_fail_out = torch.empty(1, dtype=torch.int32, device=w.device)
    _call("sp24_check_24", _ptr(w), _dtype_code(w), op, _shape(w.shape), w.dim(),
          _ptr(pass_out), _ptr(n_fail_out), _stream(stream))
    return pass_out, n_fail_out


def prune_compress_24(w: torch.Tensor, op: int = OP_MATMUL, values_out=None, meta_out=None,
                      stream=None):
    """(values, meta): kept entries [.., K/2] (or [K, C/2, R, S]) and the nibble stream."""
    _cuda(w, "w")
    if values_out is None:
        values_out = torch.empty(values_shape(op, w.shape), dtype=w.dtype, device=w.device)
    if meta_out is None:
        meta_out = torch.empty((_groups(op, w.shape) + 1) // 2, dtype=torch.uint8, device=w.device)
    _call("sp24_prune_compress_24", _ptr(w), _dtype_code(w), op, _shape(w.shape), w.dim(),
          _ptr(values_out), _ptr(meta_out), _stream(stream))
    return values_out, meta_out


def decompress_24(values: torch.Tensor, meta: torch.Tensor, shape, op: int = OP_MATMUL,
                  out=None, stream=None):
    _cuda(values, "values")
    _cuda(meta, "meta")
    if out is None:
        out = torch.empty(tuple(shape), dtype=values.dtype, device=values.device)
    _call("sp24_decompress_24", _ptr(values), _ptr(meta), _dtype_code(values), op, _shape(shape),
          len(shape), _ptr(out), _stream(stream))
    return out


def _rows_k48(shape) -> tuple:
    shape = tuple(int(d) for d in shape)
    if not shape:
        raise ValueError("pairwise 4:8 needs at least one axis")
    K = shape[-1]
    rows = 1
    for d in shape[:-1]:
        rows *= d
    return rows, K


def check_48(w: torch.Tensor, pass_out=None, n_fail_out=None, stream=None):
    """Pairwise 4:8 eligibility per chunk of 8 along K (uint8 0/1, [.., K/8]) and the failing
    chunk count (int32 [1], device)."""
    _cuda(w, "w")
    rows, K = _rows_k48(w.shape)
    if pass_out is None:
        pass_out = torch.empty(tuple(w.shape[:-1]) + (K // 8,), dtype=torch.uint8, device=w.device)
    if n_fail_out is None:
        n_fail_out = torch.empty(1, dtype=torch.int32, device=w.device)
    _call("sp24_check_48", _ptr(w), _dtype_code(w), rows, K, _ptr(pass_out), _ptr(n_fail_out), _stream(stream))
    return pass_out, n_fail_out


def prune_compress_48(w: torch.Tensor, values_out=None, meta_out=None, stream=None):
    """(values [.., K/2], meta): the two kept pairs of every chunk of 8 and the nibble stream."""
    _cuda(w, "w")
    rows, K = _rows_k48(w.shape)
    if values_out is None:
        values_out = torch.empty(tuple(w.shape[:-1]) + (K // 2,), dtype=w.dtype, device=w.device)
    if meta_out is None:
        meta_out = torch.empty((rows * (K // 8) + 1) // 2, dtype=torch.uint8, device=w.device)
    _call("sp24_prune_compress_48", _ptr(w), _dtype_code(w), rows, K, _ptr(values_out), _ptr(meta_out),
          _stream(stream))
    return values_out, meta_out


def decompress_48(values: torch.Tensor, meta: torch.Tensor, shape, out=None, stream=None):
    _cuda(values, "values")
    _cuda(meta, "meta")
    rows, K = _rows_k48(shape)
    if out is None:
        out = torch.empty(tuple(shape), dtype=values.dtype, device=values.device)
    _call("sp24_decompress_48", _ptr(values), _ptr(meta), _dtype_code(values), rows, K, _ptr(out),
          _stream(stream))
    return out


def quantize_workspace_bytes(rows: int, cols: int) -> int:
    n = ctypes.c_int64(0)
    _call("sp24_quantize_nvfp4_workspace_size", rows, cols, ctypes.byref(n))
    return n.value


def quantize_nvfp4(t: torch.Tensor, tensor_scale: Optional[torch.Tensor] = None, out=None,
                   workspace: Optional[torch.Tensor] = None, stream=None) -> NVFP4Tensor:
    """NVFP4 of a 2-D tensor; `tensor_scale` (fp32 [1], device) shares a scale across tensors."""
    _cuda(t, "t")
    if t.dim() != 2:
        raise ValueError("quantize_nvfp4 wants a 2-D tensor")
    R, L = t.shape
    if out is None:
        out = NVFP4Tensor(torch.empty((R, L // 2), dtype=torch.uint8, device=t.device),
                          torch.empty((R, L // 16), dtype=torch.uint8, device=t.device),
                          torch.empty(1, dtype=torch.float32, device=t.device))
    if workspace is None and tensor_scale is None:
        workspace = torch.empty(quantize_workspace_bytes(R, L), dtype=torch.uint8, device=t.device)
    _call("sp24_quantize_nvfp4", _ptr(t), _dtype_code(t), R, L, _ptr(tensor_scale),
          _ptr(out.codes), _ptr(out.scales), _ptr(out.tensor_scale), _ptr(workspace),
          0 if workspace is None else workspace.numel(), _stream(stream))
    return out


def quantize_nvfp4_block32(t: torch.Tensor, tensor_scale: Optional[torch.Tensor] = None, out=None,
                           workspace: Optional[torch.Tensor] = None, stream=None) -> NVFP4Tensor:
    """E2M1 codes with one E4M3 scale per 32 entries (scales [R, L/32]): the activation form of
    the pairwise-4:8 FP4 GEMM (gemm_sparse48)."""
    _cuda(t, "t")
    if t.dim() != 2:
        raise ValueError("quantize_nvfp4_block32 wants a 2-D tensor")
    R, L = t.shape
    if out is None:
        out = NVFP4Tensor(torch.empty((R, L // 2), dtype=torch.uint8, device=t.device),
                          torch.empty((R, L // 32), dtype=torch.uint8, device=t.device),
                          torch.empty(1, dtype=torch.float32, device=t.device))
    if workspace is None and tensor_scale is None:
        workspace = torch.empty(quantize_workspace_bytes(R, L), dtype=torch.uint8, device=t.device)
    _call("sp24_quantize_nvfp4_block32", _ptr(t), _dtype_code(t), R, L, _ptr(tensor_scale),
          _ptr(out.codes), _ptr(out.scales), _ptr(out.tensor_scale), _ptr(workspace),
          0 if workspace is None else workspace.numel(), _stream(stream))
    return out


def nvfp4_group_tensor_scale(tensors, out: Optional[torch.Tensor] = None,
                             workspace: Optional[torch.Tensor] = None, stream=None) -> torch.Tensor:
    """One NVFP4 tensor scale (fp32 [1], device) shared by a group of tensors of one dtype:
    max amax / 2688 over all of them.  Pass it to quantize_nvfp4(t, tensor_scale=...)."""
    tensors = list(tensors)
    if not tensors:
        raise ValueError("nvfp4_group_tensor_scale wants at least one tensor")
    for i, t in enumerate(tensors):
        _cuda(t, f"tensors[{i}]")
        if not t.is_contiguous() or t.dtype != tensors[0].dtype:
            raise ValueError("nvfp4_group_tensor_scale wants contiguous tensors of one dtype")
    dev = tensors[0].device
    if out is None:
        out = torch.empty(1, dtype=torch.float32, device=dev)
    if workspace is None:
        nb = ctypes.c_int64(0)
        _call("sp24_nvfp4_group_tensor_scale_workspace_size", ctypes.byref(nb))
        workspace = torch.empty(nb.value, dtype=torch.uint8, device=dev)
    n = len(tensors)
    ptrs = (ctypes.c_void_p * n)(*[t.data_ptr() for t in tensors])
    numels = (ctypes.c_int64 * n)(*[t.numel() for t in tensors])
    _call("sp24_nvfp4_group_tensor_scale", ptrs, numels, n, _dtype_code(tensors[0]), _ptr(out),
          _ptr(workspace), workspace.numel(), _stream(stream))
    return out


def quantize_nvfp4_pair(t0: torch.Tensor, ts0: torch.Tensor, t1: torch.Tensor, ts1: torch.Tensor,
                        out0=None, out1=None, stream=None):
    """NVFP4 of two 2-D tensors of one dtype in one launch, each with its supplied tensor scale
    (fp32 [1], device); identical to quantize_nvfp4(t0, ts0) and quantize_nvfp4(t1, ts1)."""
    _cuda(t0, "t0")
    _cuda(t1, "t1")
    if t0.dim() != 2 or t1.dim() != 2 or t0.dtype != t1.dtype:
        raise ValueError("quantize_nvfp4_pair wants two 2-D tensors of one dtype")
    outs = []
    for t, o in ((t0, out0), (t1, out1)):
        R, L = t.shape
        outs.append(o if o is not None else NVFP4Tensor(
            torch.empty((R, L // 2), dtype=torch.uint8, device=t.device),
            torch.empty((R, L // 16), dtype=torch.uint8, device=t.device),
            torch.empty(1, dtype=torch.float32, device=t.device)))
    a, b = outs
    _call("sp24_quantize_nvfp4_pair", _ptr(t0), _dtype_code(t0), t0.shape[0], t0.shape[1], _ptr(ts0),
          _ptr(a.codes), _ptr(a.scales), _ptr(a.tensor_scale), _ptr(t1), t1.shape[0], t1.shape[1],
          _ptr(ts1), _ptr(b.codes), _ptr(b.scales), _ptr(b.tensor_scale), _stream(stream))
    return a, b


def quantize_nvfp4_noalloc(t: torch.Tensor, tensor_scale: Optional[torch.Tensor] = None, out=None,
                           stream=None) -> NVFP4Tensor:
    """quantize_nvfp4 without a workspace: the library's own per-device scratch is used, so the
    call needs no device allocation (for callers that cannot allocate, e.g. during graph
    capture).  Calls whose GPU work overlaps race on that scratch."""
    _cuda(t, "t")
    if t.dim() != 2:
        raise ValueError("quantize_nvfp4_noalloc wants a 2-D tensor")
    R, L = t.shape
    if out is None:
        out = NVFP4Tensor(torch.empty((R, L // 2), dtype=torch.uint8, device=t.device),
                          torch.empty((R, L // 16), dtype=torch.uint8, device=t.device),
                          torch.empty(1, dtype=torch.float32, device=t.device))
    _call("sp24_quantize_nvfp4_noalloc", _ptr(t), _dtype_code(t), R, L, _ptr(tensor_scale),
          _ptr(out.codes), _ptr(out.scales), _ptr(out.tensor_scale), _stream(stream))
    return out


def dequantize_nvfp4(q: NVFP4Tensor, dtype=torch.float32, stream=None) -> torch.Tensor:
    R, L2 = q.codes.shape
    out = torch.empty((R, 2 * L2), dtype=dtype, device=q.codes.device)
    _call("sp24_dequantize_nvfp4", _ptr(q.codes), _ptr(q.scales), _ptr(q.tensor_scale), R, 2 * L2,
          _DT[dtype], _ptr(out), _stream(stream))
    return out


class Prepared24(NamedTuple):
    """What sp24_prepare_24 produces for a weight W[rows, K]."""
    pass_map: Optional[torch.Tensor]   # uint8 [rows, K/4] or None
    n_fail: torch.Tensor               # int32 [1]
    values: torch.Tensor               # kept entries [rows, K/2], W's dtype
    meta: torch.Tensor                 # uint8 [rows, K/8] nibble stream
    w_tensor_scale: torch.Tensor       # fp32 [1]: amax|W| / 2688
    v_tensor_scale: torch.Tensor       # fp32 [1]: amax|values| / 2688


def prepare_workspace_bytes(rows: int, K: int) -> int:
    n = ctypes.c_int64(0)
    _call("sp24_prepare_24_workspace_size", rows, K, ctypes.byref(n))
    return n.value


def prepare_24(w: torch.Tensor, with_pass: bool = True, out: Optional[Prepared24] = None,
               workspace=None, stream=None) -> Prepared24:
    """check_24 + prune_compress_24 + both NVFP4 tensor scales of a matmul weight w[rows, K]
    (K % 16 == 0) with one read of w; identical to the separate calls."""
    _cuda(w, "w")
    if w.dim() != 2:
        raise ValueError("prepare_24 wants a 2-D weight")
    R, K = w.shape
    dev = w.device
    if out is None:
        out = Prepared24(
            torch.empty((R, K // 4), dtype=torch.uint8, device=dev) if with_pass else None,
            torch.empty(1, dtype=torch.int32, device=dev),
            torch.empty((R, K // 2), dtype=w.dtype, device=dev),
            torch.empty((R, K // 8), dtype=torch.uint8, device=dev),
            torch.empty(1, dtype=torch.float32, device=dev),
            torch.empty(1, dtype=torch.float32, device=dev))
    if workspace is None:
        workspace = torch.empty(prepare_workspace_bytes(R, K), dtype=torch.uint8, device=dev)
    _call("sp24_prepare_24", _ptr(w), _dtype_code(w), R, K, _ptr(out.pass_map), _ptr(out.n_fail),
          _ptr(out.values), _ptr(out.meta), _ptr(out.w_tensor_scale), _ptr(out.v_tensor_scale),
          _ptr(workspace), workspace.numel(), _stream(stream))
    return out


def prepare_nvfp4_24(w: torch.Tensor, stream=None):
    """The whole weight side of both GEMM paths: prepare_24, then NVFP4 of w and of its kept
    values with the tensor scales prepare_24 derived.  Returns (Prepared24, dense NVFP4Tensor,
    Sparse24 with NVFP4 values)."""
    p = prepare_24(w, stream=stream)
    wq, vq = quantize_nvfp4_pair(w, p.w_tensor_scale, p.values, p.v_tensor_scale, stream=stream)
    return p, wq, Sparse24(vq, p.meta)


# ---------------------------------------------------------------------------- a4 .. a6

def to_mma(q: NVFP4Tensor, stream=None) -> NVFP4MMA:
    """The same NVFP4 tensor rewritten as the tile images the W4A4 GEMM loads whole
    (sp24_nvfp4_to_mma; cols % 256 == 0); the tensor scale is shared, not copied."""
    rows, cols = q.codes.shape[0], 2 * q.codes.shape[1]
    nc, ns = ctypes.c_int64(0), ctypes.c_int64(0)
    _call("sp24_nvfp4_mma_size", rows, cols, ctypes.byref(nc), ctypes.byref(ns))
    codes = torch.empty(nc.value, dtype=torch.uint8, device=q.codes.device)
    scales = torch.empty(ns.value, dtype=torch.uint8, device=q.codes.device)
    _call("sp24_nvfp4_to_mma", _ptr(q.codes), _ptr(q.scales), rows, cols, _ptr(codes), _ptr(scales),
          _stream(stream))
    return NVFP4MMA(codes, scales, q.tensor_scale, rows, cols)


def _operand(t) -> _Operand:
    if isinstance(t, NVFP4Tensor):
        return _Operand(NVFP4, t.codes.data_ptr(), t.scales.data_ptr(), t.tensor_scale.data_ptr())
    if isinstance(t, NVFP4MMA):
        return _Operand(NVFP4_MMA, t.codes.data_ptr(), t.scales.data_ptr(), t.tensor_scale.data_ptr())
    _cuda(t, "operand")
    return _Operand(_dtype_code(t), t.data_ptr(), None, None)


def _rows_k(t) -> tuple:
    if isinstance(t, NVFP4MMA):
        return t.rows, t.cols
    if isinstance(t, NVFP4Tensor):
        return t.codes.shape[0], 2 * t.codes.shape[1]
    return t.shape[0], t.shape[1]


def gemm_workspace_bytes(x, w, sparse: bool, M: int, N: int, K: int, algo: int = ALGO_AUTO) -> int:
    fmt = lambda t: NVFP4 if isinstance(t, NVFP4Tensor) else NVFP4_MMA if isinstance(t, NVFP4MMA) else _DT[t.dtype]
    xf = fmt(x)
    wf = fmt(w.values if sparse else w)
    n = ctypes.c_int64(0)
    _call("sp24_gemm_workspace_size", xf, wf, int(sparse), M, N, K, algo, ctypes.byref(n))
    return n.value


def gemm_dense(x, w, out=None, algo: int = ALGO_AUTO, workspace=None, stream=None) -> torch.Tensor:
    """Y[M, N] fp32 = x[M, K] @ w[N, K]^T; x, w: 16-bit tensors or NVFP4Tensor."""
    M, K = _rows_k(x)
    N, Kw = _rows_k(w)
    if K != Kw:
        raise ValueError(f"K mismatch: {K} vs {Kw}")
    dev = (x.codes if isinstance(x, (NVFP4Tensor, NVFP4MMA)) else x).device
    if out is None:
        out = torch.empty((M, N), dtype=torch.float32, device=dev)
    ws_bytes = gemm_workspace_bytes(x, w, False, M, N, K, algo)
    if workspace is None and ws_bytes:
        workspace = torch.empty(ws_bytes, dtype=torch.uint8, device=dev)
    xo, wo = _operand(x), _operand(w)
    _call("sp24_gemm_dense", ctypes.byref(xo), ctypes.byref(wo), M, N, K, _ptr(out),
          _ptr(workspace), 0 if workspace is None else workspace.numel(), algo, _stream(stream))
    return out


def gemm_sparse24(x, w: Sparse24, K: int, out=None, algo: int = ALGO_AUTO, workspace=None,
                  stream=None) -> torch.Tensor:
    """The same product with w 2:4-compressed (values 16-bit or NVFP4 + meta)."""
    M, Kx = _rows_k(x)
    if Kx != K:
        raise ValueError(f"K mismatch: {Kx} vs {K}")
    v = w.values
    if isinstance(v, NVFP4Tensor):
        N = v.codes.shape[0]
        wo = _SparseOperand(NVFP4, v.codes.data_ptr(), v.scales.data_ptr(),
                            v.tensor_scale.data_ptr(), w.meta.data_ptr())
    else:
        _cuda(v, "values")
        N = v.shape[0]
        wo = _SparseOperand(_dtype_code(v), v.data_ptr(), None, None, w.meta.data_ptr())
    dev = w.meta.device
    if out is None:
        out = torch.empty((M, N), dtype=torch.float32, device=dev)
    ws_bytes = gemm_workspace_bytes(x, w, True, M, N, K, algo)
    if workspace is None and ws_bytes:
        workspace = torch.empty(ws_bytes, dtype=torch.uint8, device=dev)
    xo = _operand(x)
    _call("sp24_gemm_sparse24", ctypes.byref(xo), ctypes.byref(wo), M, N, K, _ptr(out),
          _ptr(workspace), 0 if workspace is None else workspace.numel(), algo, _stream(stream))
    return out


class Sparse48(NamedTuple):
    """A pairwise-4:8 weight [N, K] for the sparse FP4 MMA: the kept values [N, K/2] as NVFP4
    (16-value blocks: codes [N, K/4], scales [N, K/32]) + the nibble stream of prune_compress_48."""
    values: NVFP4Tensor
    meta: torch.Tensor


class Sparse48MMA(NamedTuple):
    """A pairwise-4:8 weight [rows, K] as the sparse FP4 pair kernel's tile images (flat uint8:
    values, scales, metadata; rows padded to 256), with its tensor scale."""
    values: torch.Tensor
    scales: torch.Tensor
    meta: torch.Tensor
    tensor_scale: torch.Tensor
    rows: int
    K: int


def sparse48_to_mma(w: Sparse48, K: int, stream=None) -> Sparse48MMA:
    """The weight rewritten as tile images (sp24_sparse48_to_mma), once per weight."""
    v = w.values
    rows = v.codes.shape[0]
    nv, ns, nm = ctypes.c_int64(0), ctypes.c_int64(0), ctypes.c_int64(0)
    _call("sp24_sparse48_mma_size", rows, K, ctypes.byref(nv), ctypes.byref(ns), ctypes.byref(nm))
    dev = v.codes.device
    vo = torch.empty(nv.value, dtype=torch.uint8, device=dev)
    so = torch.empty(ns.value, dtype=torch.uint8, device=dev)
    mo = torch.empty(nm.value, dtype=torch.uint8, device=dev)
    _call("sp24_sparse48_to_mma", _ptr(v.codes), _ptr(v.scales), _ptr(w.meta), rows, K, _ptr(vo), _ptr(so), _ptr(mo),
          _stream(stream))
    return Sparse48MMA(vo, so, mo, v.tensor_scale, rows, K)


def prepare_sparse(meta: torch.Tensor, rows: int, K: int, stream=None) -> torch.Tensor:
    """The 2:4 nibble stream of a [rows, K] weight in the tensor cores' metadata layout
    (sp24_prepare_sparse): uint8 tiles of 2 KB per 128 rows and 128 K, rows padded to 256."""
    n = ctypes.c_int64(0)
    _call("sp24_prepare_sparse_size", rows, K, ctypes.byref(n))
    out = torch.empty(n.value, dtype=torch.uint8, device=meta.device)
    _call("sp24_prepare_sparse", _ptr(meta), rows, K, _ptr(out), _stream(stream))
    return out


def b32_to_mma(q: NVFP4Tensor, stream=None) -> NVFP4MMA:
    """Activations from quantize_nvfp4_block32 rewritten as tile images (sp24_nvfp4_b32_to_mma)."""
    rows, cols = q.codes.shape[0], 2 * q.codes.shape[1]
    nc, ns = ctypes.c_int64(0), ctypes.c_int64(0)
    _call("sp24_nvfp4_b32_mma_size", rows, cols, ctypes.byref(nc), ctypes.byref(ns))
    codes = torch.empty(nc.value, dtype=torch.uint8, device=q.codes.device)
    scales = torch.empty(ns.value, dtype=torch.uint8, device=q.codes.device)
    _call("sp24_nvfp4_b32_to_mma", _ptr(q.codes), _ptr(q.scales), rows, cols, _ptr(codes), _ptr(scales),
          _stream(stream))
    return NVFP4MMA(codes, scales, q.tensor_scale, rows, cols)


def gemm_sparse48(x, w, K: int, out=None, stream=None) -> torch.Tensor:
    """y[M, N] = x w^T on the sparse FP4 MMA: x from quantize_nvfp4_block32 ([M, K]), w a
    pairwise-4:8 weight; K % 512 == 0.  With both operands as tile images (b32_to_mma,
    sparse48_to_mma) the persistent CTA-pair kernel runs."""
    if isinstance(x, NVFP4MMA) or isinstance(w, Sparse48MMA):
        if not (isinstance(x, NVFP4MMA) and isinstance(w, Sparse48MMA)):
            raise ValueError("tile images are taken for both operands or neither")
        M, N = x.rows, w.rows
        if x.cols != K or w.K != K:
            raise ValueError(f"K mismatch: {x.cols}, {w.K} vs {K}")
        if out is None:
            out = torch.empty((M, N), dtype=torch.float32, device=w.meta.device)
        xo = _Operand(NVFP4_B32_MMA, x.codes.data_ptr(), x.scales.data_ptr(), x.tensor_scale.data_ptr())
        wo = _SparseOperand(NVFP4_MMA, w.values.data_ptr(), w.scales.data_ptr(), w.tensor_scale.data_ptr(),
                            w.meta.data_ptr())
        _call("sp24_gemm_sparse48", ctypes.byref(xo), ctypes.byref(wo), M, N, K, _ptr(out), _stream(stream))
        return out
    M = x.codes.shape[0]
    if x.codes.shape[1] * 2 != K:
        raise ValueError(f"K mismatch: {x.codes.shape[1] * 2} vs {K}")
    v = w.values
    N = v.codes.shape[0]
    if out is None:
        out = torch.empty((M, N), dtype=torch.float32, device=w.meta.device)
    xo = _Operand(NVFP4_B32, x.codes.data_ptr(), x.scales.data_ptr(), x.tensor_scale.data_ptr())
    wo = _SparseOperand(NVFP4, v.codes.data_ptr(), v.scales.data_ptr(), v.tensor_scale.data_ptr(), w.meta.data_ptr())
    _call("sp24_gemm_sparse48", ctypes.byref(xo), ctypes.byref(wo), M, N, K, _ptr(out), _stream(stream))
    return out


def _sparse_operand(w: "Sparse24") -> _SparseOperand:
    v = w.values
    if isinstance(v, NVFP4Tensor):
        return _SparseOperand(NVFP4, v.codes.data_ptr(), v.scales.data_ptr(), v.tensor_scale.data_ptr(),
                              w.meta.data_ptr())
    _cuda(v, "values")
    return _SparseOperand(_dtype_code(v), v.data_ptr(), None, None, w.meta.data_ptr())


def _both_forms(x, w_dense, w_sparse: "Sparse24"):
    M, K = _rows_k(x)
    N, Kw = _rows_k(w_dense)
    if K != Kw:
        raise ValueError(f"K mismatch: {K} vs {Kw}")
    ws = max(gemm_workspace_bytes(x, w_dense, False, M, N, K), gemm_workspace_bytes(x, w_sparse, True, M, N, K))
    return M, N, K, ws


def gemm_choice(x_format: int, w_format: int, M: int, N: int, K: int) -> tuple:
    """(use_sparse, measured): the dense / 2:4 decision for a shape (host only)."""
    u, m = ctypes.c_int(0), ctypes.c_int(0)
    _call("sp24_gemm_choice", x_format, w_format, M, N, K, ctypes.byref(u), ctypes.byref(m))
    return bool(u.value), bool(m.value)


def gemm_choice_reset() -> None:
    _call("sp24_gemm_choice_reset")


def gemm_select(x, w_dense, w_sparse: "Sparse24", reps: int = 10, out=None, workspace=None, stream=None) -> dict:
    """Times the dense and the 2:4 GEMM of this shape, records the faster one (synchronises)."""
    M, N, K, ws_bytes = _both_forms(x, w_dense, w_sparse)
    dev = w_sparse.meta.device
    if out is None:
        out = torch.empty((M, N), dtype=torch.float32, device=dev)
    if workspace is None and ws_bytes:
        workspace = torch.empty(ws_bytes, dtype=torch.uint8, device=dev)
    xo, wd, wsp = _operand(x), _operand(w_dense), _sparse_operand(w_sparse)
    u, td, tsp = ctypes.c_int(0), ctypes.c_float(0), ctypes.c_float(0)
    _call("sp24_gemm_select", ctypes.byref(xo), ctypes.byref(wd), ctypes.byref(wsp), M, N, K, _ptr(out),
          _ptr(workspace), 0 if workspace is None else workspace.numel(), reps, ctypes.byref(u),
          ctypes.byref(td), ctypes.byref(tsp), _stream(stream))
    return {"use_sparse": bool(u.value), "us_dense": td.value, "us_sparse": tsp.value}


def gemm_auto(x, w_dense, w_sparse: "Sparse24", out=None, workspace=None, stream=None):
    """Y[M, N] from whichever form sp24_gemm_choice names; returns (Y, used_sparse)."""
    M, N, K, ws_bytes = _both_forms(x, w_dense, w_sparse)
    dev = w_sparse.meta.device
    if out is None:
        out = torch.empty((M, N), dtype=torch.float32, device=dev)
    if workspace is None and ws_bytes:
        workspace = torch.empty(ws_bytes, dtype=torch.uint8, device=dev)
    xo, wd, wsp = _operand(x), _operand(w_dense), _sparse_operand(w_sparse)
    u = ctypes.c_int(0)
    _call("sp24_gemm_auto", ctypes.byref(xo), ctypes.byref(wd), ctypes.byref(wsp), M, N, K, _ptr(out),
          _ptr(workspace), 0 if workspace is None else workspace.numel(), ctypes.byref(u), _stream(stream))
    return out, bool(u.value)


def grouped_workspace_bytes(T: int, topk: int, E: int) -> int:
    n = ctypes.c_int64(0)
    _call("sp24_gemm_grouped_workspace_size", T, topk, E, ctypes.byref(n))
    return n.value


def gemm_grouped(x, routing: torch.Tensor, w, E: int, N: int, K: int, out=None, workspace=None,
                 stream=None) -> torch.Tensor:
    """Routed-expert GEMM: Y[t, s, :] = x[t] @ W[routing[t, s]]^T with the E experts stacked as
    one [E*N, K] operand (16-bit tensor, NVFP4Tensor, or Sparse24 of those)."""
    _cuda(routing, "routing")
    T, topk = routing.shape
    dev = routing.device
    if out is None:
        out = torch.empty((T, topk, N), dtype=torch.float32, device=dev)
    if workspace is None:
        workspace = torch.empty(grouped_workspace_bytes(T, topk, E), dtype=torch.uint8, device=dev)
    xo = _operand(x)
    if isinstance(w, Sparse24):
        v = w.values
        if isinstance(v, NVFP4Tensor):
            so = _SparseOperand(NVFP4, v.codes.data_ptr(), v.scales.data_ptr(), v.tensor_scale.data_ptr(),
                                w.meta.data_ptr())
        else:
            so = _SparseOperand(_dtype_code(v), v.data_ptr(), None, None, w.meta.data_ptr())
        dense_p, sparse_p = None, ctypes.byref(so)
    else:
        do = _operand(w)
        dense_p, sparse_p = ctypes.byref(do), None
    _call("sp24_gemm_grouped", ctypes.byref(xo), _ptr(routing), T, topk, dense_p, sparse_p, E, N, K,
          _ptr(out), _ptr(workspace), workspace.numel(), _stream(stream))
    return out


def kernel_launches() -> int:
    """Kernels this library has launched in this process (host-side count)."""
    return int(lib().sp24_kernel_launches())


def last_device_error(stream=None) -> int:
    return int(lib().sp24_last_device_error(_stream(stream)))


def sizes(op: int, dtype: int, shape) -> dict:
    """Host-side size arithmetic of the compressed and NVFP4 forms (no device access)."""
    out = [ctypes.c_int64(0) for _ in range(5)]
    _call("sp24_sizes", op, dtype, _shape(shape), len(shape), *[ctypes.byref(o) for o in out])
    keys = ("groups", "values_bytes", "meta_bytes", "nvfp4_codes_bytes", "nvfp4_scales_bytes")
    return {k: o.value for k, o in zip(keys, out)}


def _interleave(a: torch.Tensor, b: torch.Tensor, rows: int, block_rows: int = 16, stream=None) -> torch.Tensor:
    _cuda(a, "a")
    _cuda(b, "b")
    if a.shape != b.shape or a.dtype != b.dtype:
        raise ValueError("interleave wants two tensors of one shape and dtype")
    row_bytes = a.numel() * a.element_size() // rows
    out = torch.empty((2 * rows, row_bytes), dtype=torch.uint8, device=a.device)
    _call("sp24_interleave_rows", _ptr(a), _ptr(b), rows, row_bytes, block_rows, _ptr(out), _stream(stream))
    return out


def pack_gate_up(gate, up, stream=None):
    """The expert block's gate / up operand: the stacked gate and up weights [E*F, H] (NVFP4Tensor,
    or Sparse24 of NVFP4Tensor values, sharing one tensor scale) packed in 16-row blocks."""
    if isinstance(gate, Sparse24):
        gv, uv = gate.values, up.values
        rows = gv.codes.shape[0]
        vals = NVFP4Tensor(_interleave(gv.codes, uv.codes, rows, stream=stream),
                           _interleave(gv.scales, uv.scales, rows, stream=stream), gv.tensor_scale.clone())
        return Sparse24(vals, _interleave(gate.meta, up.meta, rows, stream=stream).reshape(-1))
    rows = gate.codes.shape[0]
    return NVFP4Tensor(_interleave(gate.codes, up.codes, rows, stream=stream),
                       _interleave(gate.scales, up.scales, rows, stream=stream), gate.tensor_scale.clone())


def moe_block_workspace_bytes(T: int, topk: int, E: int, H: int, F: int) -> int:
    n = ctypes.c_int64(0)
    _call("sp24_moe_block_workspace_size", T, topk, E, H, F, ctypes.byref(n))
    return n.value


def moe_block(x: torch.Tensor, routing: torch.Tensor, router_w: torch.Tensor, w_gate_up, w_down, E: int, H: int,
              F: int, out=None, workspace=None, stream=None) -> torch.Tensor:
    """y[T, H] fp32 = sum_s r[t, s] * (SiLU(x Wg^T) * (x Wu^T)) Wd^T over the routed experts;
    w_gate_up from pack_gate_up, w_down [E*H, F]; each an NVFP4Tensor or a Sparse24 of one."""
    _cuda(routing, "routing")
    _cuda(router_w, "router_w")
    T, topk = routing.shape
    dev = routing.device
    if out is None:
        out = torch.empty((T, H), dtype=torch.float32, device=dev)
    if workspace is None:
        workspace = torch.empty(moe_block_workspace_bytes(T, topk, E, H, F), dtype=torch.uint8, device=dev)
    xo = _operand(x)
    gd = gs = dd = ds = None
    if isinstance(w_gate_up, Sparse24):
        gs = ctypes.byref(_sparse_operand(w_gate_up))
    else:
        gd = ctypes.byref(_operand(w_gate_up))
    if isinstance(w_down, Sparse24):
        ds = ctypes.byref(_sparse_operand(w_down))
    else:
        dd = ctypes.byref(_operand(w_down))
    _call("sp24_moe_block", ctypes.byref(xo), _ptr(routing), _ptr(router_w), T, topk, gd, gs, dd, ds, E, H, F,
          _ptr(out), _ptr(workspace), workspace.numel(), _stream(stream))
    return out

"""CPU oracle for the 2:4 sparsity / NVFP4 pipeline -- TEST INFRASTRUCTURE ONLY.

Only ``tests/``, ``__graft_entry__.smoke()`` and ``bench.py``'s CPU-baseline leg may import
this package.  The product library (``fp16_gemm_b200``) never imports, links or calls it, and
the two share no code.

The arithmetic lives in ``sp24_oracle.c`` (plain scalar C, fp64 GEMM sums, IEEE fp32 for the
NVFP4 scale decisions); this module compiles it with gcc on first use and wraps it with
ctypes over numpy arrays.  Pages followed, by title:

* "NVFP4 vs 2:4 sparse: where the other half of the petaflop went" -- "What 2:4 actually is",
  "The byte saving is about a quarter, not a half".
* "Sparse GPU FLOPS Need the Right Zeros in the Right Places" -- "The operation determines
  which four entries belong together", "Two half-zero vectors produce different pattern
  answers".
* "NVFP4 Without FP4 Hardware" -- "Convert BF16 to NVFP4 yourself", "The shared global
  scale", "Bit-exact check against lyf's ModelOpt output".

Pairwise 4:8 (``check_48`` / ``compress_48`` / ``decompress_48``) and the 32-value NVFP4 block
(``nvfp4_encode(..., block=32)``) follow readings R21 / R22 of the same pages ("What 2:4
actually is", carried over to pairs; the block size the sparse FP4 MMA reads); they are pinned
against brute force over the six pair choices and against ml_dtypes' roundings.

The NVFP4 scale and rounding formulae (tensor scale = amax / 2688, block scale =
E4M3(bmax / (6 s_t)), code = E2M1(|t| / (dec(sb) s_t)), all RNE) are a reading: the pages
state the format but print no worked example.  They are pinned to the recipe the pages'
converter reproduces bit for bit (ModelOpt's), as compressed-tensors (global scale) and vLLM
(reference quantiser) implement it, up to one rounding step next to a rounding boundary, and
by their properties (sizes, re-quantisation stability, negative zero, exhaustive rounding).
"""
from __future__ import annotations

import ctypes
import os
import subprocess
import threading

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "sp24_oracle.c")
_LIB = os.path.join(_HERE, "libsp24_oracle.so")
_lock = threading.Lock()
_lib = None

F16, BF16, F32 = 0, 1, 2
MATMUL, CONV = 0, 1

_DT = {F16: np.uint16, BF16: np.uint16, F32: np.float32}


def build(force: bool = False) -> str:
    """Compile the oracle into ``libsp24_oracle.so`` (gcc, -O2, OpenMP, no FMA contraction)."""
    stale = (not os.path.exists(_LIB)) or os.path.getmtime(_LIB) < os.path.getmtime(_SRC)
    if force or stale:
        tmp = _LIB + f".tmp{os.getpid()}"
        cmd = ["gcc", "-std=c11", "-O2", "-fPIC", "-shared", "-fopenmp", "-ffp-contract=off",
               "-fno-fast-math", "-Wall", "-o", tmp, _SRC, "-lm"]
        subprocess.run(cmd, check=True)
        os.replace(tmp, _LIB)
    return _LIB


def lib():
    global _lib
    with _lock:
        if _lib is None:
            build()
            L = ctypes.CDLL(_LIB)
            P, I64, I = ctypes.c_void_p, ctypes.c_int64, ctypes.c_int
            L.sp24o_check_24.restype = I64
            L.sp24o_check_24.argtypes = [P, I, I, P, I, P]
            for f in ("sp24o_prune_24",):
                getattr(L, f).argtypes = [P, I, I, P, I, P]
            L.sp24o_compress_24.argtypes = [P, I, I, P, I, P, P]
            L.sp24o_decompress_24.argtypes = [P, P, I, I, P, I, P]
            L.sp24o_check_48.restype = I64
            L.sp24o_check_48.argtypes = [P, I, I64, I64, P]
            L.sp24o_compress_48.argtypes = [P, I, I64, I64, P, P]
            L.sp24o_decompress_48.argtypes = [P, P, I, I64, I64, P]
            L.sp24o_e2m1_value.restype = ctypes.c_double
            L.sp24o_e2m1_value.argtypes = [I]
            L.sp24o_e4m3_value.restype = ctypes.c_double
            L.sp24o_e4m3_value.argtypes = [I]
            L.sp24o_e2m1_round.argtypes = [ctypes.c_double]
            L.sp24o_e4m3_round.argtypes = [ctypes.c_double]
            L.sp24o_nvfp4_tensor_scale.restype = ctypes.c_float
            L.sp24o_nvfp4_tensor_scale.argtypes = [P, I, I64]
            L.sp24o_nvfp4_encode.argtypes = [P, I, I64, I64, P, P, P, P]
            L.sp24o_nvfp4_decode.argtypes = [P, P, ctypes.c_float, I64, I64, P]
            L.sp24o_nvfp4_encode_blk.argtypes = [P, I, I64, I64, I, P, P, P, P]
            L.sp24o_nvfp4_decode_blk.argtypes = [P, P, ctypes.c_float, I64, I64, I, P]
            L.sp24o_to_double.argtypes = [P, I, I64, P]
            L.sp24o_gemm.argtypes = [P, P, I64, I64, I64, P, P, I]
            L.sp24o_gemm_sparse.argtypes = [P, P, P, I64, I64, I64, P, P, I]
            L.sp24o_moe.argtypes = [P, P, P, I64, I, I64, I64, I64, P, P, I]
            _lib = L
    return _lib


class OracleError(RuntimeError):
    pass


def _ptr(a: np.ndarray | None):
    if a is None:
        return None
    assert a.flags["C_CONTIGUOUS"], "oracle arrays must be C-contiguous"
    return a.ctypes.data


def _check(rc: int, what: str) -> None:
    if rc != 0:
        raise OracleError(f"{what}: oracle returned {rc}")


def _shape(shape) -> np.ndarray:
    s = np.zeros(4, dtype=np.int64)
    s[: len(shape)] = shape
    return s


def _bits(t: np.ndarray, dtype: int) -> np.ndarray:
    want = _DT[dtype]
    t = np.ascontiguousarray(t)
    if t.dtype == np.float16:
        t = t.view(np.uint16)
    if t.dtype != want:
        raise TypeError(f"dtype code {dtype} wants {want}, got {t.dtype}")
    return t


def groups(op: int, shape) -> int:
    """Number of groups of four along the reduction axis (K for matmul, C for conv)."""
    shape = tuple(int(s) for s in shape)
    if op == MATMUL:
        return int(np.prod(shape)) // 4
    K, C, R, S = shape
    return K * (C // 4) * R * S


def group_shape(op: int, shape) -> tuple:
    shape = tuple(int(s) for s in shape)
    if op == MATMUL:
        return shape[:-1] + (shape[-1] // 4,)
    K, C, R, S = shape
    return (K, C // 4, R, S)


def values_shape(op: int, shape) -> tuple:
    shape = tuple(int(s) for s in shape)
    if op == MATMUL:
        return shape[:-1] + (shape[-1] // 2,)
    K, C, R, S = shape
    return (K, C // 2, R, S)


def check_24(w: np.ndarray, dtype: int, op: int = MATMUL):
    """Per-group pass map (uint8, group axis replacing K or C) and the failing-group count."""
    w = _bits(w, dtype)
    pass_ = np.zeros(group_shape(op, w.shape), dtype=np.uint8)
    n = lib().sp24o_check_24(_ptr(w), dtype, op, _ptr(_shape(w.shape)), w.ndim, _ptr(pass_))
    if n < 0:
        raise OracleError(f"check_24: oracle returned {n}")
    return pass_, int(n)


def prune_24(w: np.ndarray, dtype: int, op: int = MATMUL) -> np.ndarray:
    kind = np.asarray(w).dtype
    w = _bits(w, dtype)
    out = np.empty_like(w)
    _check(lib().sp24o_prune_24(_ptr(w), dtype, op, _ptr(_shape(w.shape)), w.ndim, _ptr(out)),
           "prune_24")
    return out.view(kind)


def compress_24(w: np.ndarray, dtype: int, op: int = MATMUL):
    """(values, meta): values in the caller's storage type, meta a flat nibble stream."""
    kind = np.asarray(w).dtype
    w = _bits(w, dtype)
    G = groups(op, w.shape)
    values = np.empty(values_shape(op, w.shape), dtype=w.dtype)
    meta = np.zeros((G + 1) // 2, dtype=np.uint8)
    _check(lib().sp24o_compress_24(_ptr(w), dtype, op, _ptr(_shape(w.shape)), w.ndim,
                                   _ptr(values), _ptr(meta)), "compress_24")
    return values.view(kind), meta


def decompress_24(values: np.ndarray, meta: np.ndarray, dtype: int, shape, op: int = MATMUL):
    kind = np.asarray(values).dtype
    values = _bits(values, dtype)
    meta = np.ascontiguousarray(meta, dtype=np.uint8)
    out = np.empty(tuple(shape), dtype=values.dtype)
    _check(lib().sp24o_decompress_24(_ptr(values), _ptr(meta), dtype, op, _ptr(_shape(shape)),
                                     len(shape), _ptr(out)), "decompress_24")
    return out.view(kind)


def check_48(w: np.ndarray, dtype: int):
    """Pairwise 4:8 eligibility of W[rows, K] (chunks of 8 along K): pass map [rows, K/8], fails."""
    w = _bits(w, dtype)
    rows, K = w.shape
    pass_ = np.zeros((rows, K // 8), dtype=np.uint8)
    n = lib().sp24o_check_48(_ptr(w), dtype, rows, K, _ptr(pass_))
    if n < 0:
        raise OracleError(f"check_48: oracle returned {n}")
    return pass_, int(n)


def compress_48(w: np.ndarray, dtype: int):
    """(values [rows, K/2] in the caller's storage type, meta nibble stream) of pairwise 4:8."""
    kind = np.asarray(w).dtype
    w = _bits(w, dtype)
    rows, K = w.shape
    values = np.empty((rows, K // 2), dtype=w.dtype)
    meta = np.empty((rows * (K // 8) + 1) // 2, dtype=np.uint8)
    _check(lib().sp24o_compress_48(_ptr(w), dtype, rows, K, _ptr(values), _ptr(meta)), "compress_48")
    return values.view(kind), meta


def decompress_48(values: np.ndarray, meta: np.ndarray, dtype: int, shape):
    kind = np.asarray(values).dtype
    values = _bits(values, dtype)
    meta = np.ascontiguousarray(meta, dtype=np.uint8)
    rows, K = shape
    out = np.empty((rows, K), dtype=values.dtype)
    _check(lib().sp24o_decompress_48(_ptr(values), _ptr(meta), dtype, rows, K, _ptr(out)), "decompress_48")
    return out.view(kind)


def e2m1_value(code: int) -> float:
    return lib().sp24o_e2m1_value(int(code))


def e4m3_value(code: int) -> float:
    return lib().sp24o_e4m3_value(int(code))


def e2m1_round(x: float) -> int:
    return lib().sp24o_e2m1_round(float(x))


def e4m3_round(x: float) -> int:
    return lib().sp24o_e4m3_round(float(x))


def nvfp4_tensor_scale(t: np.ndarray, dtype: int) -> float:
    t = _bits(t, dtype)
    return float(np.float32(lib().sp24o_nvfp4_tensor_scale(_ptr(t), dtype, t.size)))


def nvfp4_group_tensor_scale(tensors, dtype: int) -> float:
    """One tensor scale for a group of tensors read together ([P5] "The shared global scale"):
    the scale of the group's entries taken as one tensor, max amax / 2688."""
    flat = [np.ascontiguousarray(t).ravel() for t in tensors]
    if not flat or sum(f.size for f in flat) == 0:
        return 0.0
    return nvfp4_tensor_scale(np.concatenate([f for f in flat if f.size]), dtype)


def nvfp4_encode(t: np.ndarray, dtype: int, tensor_scale: float | None = None, block: int = 16):
    """(codes [R, L/2] u8, scales [R, L/block] u8, tensor_scale f32) of a 2-D tensor T[R, L];
    block 16 is NVFP4, block 32 the activation form of the sparse FP4 MMA."""
    t = _bits(t, dtype)
    if t.ndim != 2:
        raise ValueError("nvfp4_encode wants a 2-D tensor")
    R, L = t.shape
    codes = np.zeros((R, L // 2), dtype=np.uint8)
    scales = np.zeros((R, L // block), dtype=np.uint8)
    ts_out = np.zeros(1, dtype=np.float32)
    ts_in = None if tensor_scale is None else np.array([tensor_scale], dtype=np.float32)
    _check(lib().sp24o_nvfp4_encode_blk(_ptr(t), dtype, R, L, block, _ptr(ts_in), _ptr(codes), _ptr(scales),
                                        _ptr(ts_out)), "nvfp4_encode")
    return codes, scales, np.float32(ts_out[0])


def nvfp4_decode(codes: np.ndarray, scales: np.ndarray, tensor_scale, block: int = 16) -> np.ndarray:
    codes = np.ascontiguousarray(codes, dtype=np.uint8)
    scales = np.ascontiguousarray(scales, dtype=np.uint8)
    R, L2 = codes.shape
    out = np.empty((R, 2 * L2), dtype=np.float64)
    _check(lib().sp24o_nvfp4_decode_blk(_ptr(codes), _ptr(scales), float(np.float32(tensor_scale)),
                                        R, 2 * L2, block, _ptr(out)), "nvfp4_decode")
    return out


def to_double(t: np.ndarray, dtype: int) -> np.ndarray:
    t = _bits(t, dtype)
    out = np.empty(t.shape, dtype=np.float64)
    _check(lib().sp24o_to_double(_ptr(t), dtype, t.size, _ptr(out)), "to_double")
    return out


def gemm(X: np.ndarray, W: np.ndarray, nthreads: int = 0):
    """(Y, S) with Y = X W^T in fp64 and S = |X| |W|^T (per-output tolerance scale)."""
    X = np.ascontiguousarray(X, dtype=np.float64)
    W = np.ascontiguousarray(W, dtype=np.float64)
    M, K = X.shape
    N = W.shape[0]
    Y = np.empty((M, N), dtype=np.float64)
    S = np.empty((M, N), dtype=np.float64)
    _check(lib().sp24o_gemm(_ptr(X), _ptr(W), M, N, K, _ptr(Y), _ptr(S), nthreads), "gemm")
    return Y, S


def gemm_sparse(X: np.ndarray, V: np.ndarray, meta: np.ndarray, nthreads: int = 0):
    """(Y, S) for W given as decoded kept values V [N, K/2] plus its nibble stream."""
    X = np.ascontiguousarray(X, dtype=np.float64)
    V = np.ascontiguousarray(V, dtype=np.float64)
    meta = np.ascontiguousarray(meta, dtype=np.uint8)
    M, K = X.shape
    N = V.shape[0]
    Y = np.empty((M, N), dtype=np.float64)
    S = np.empty((M, N), dtype=np.float64)
    _check(lib().sp24o_gemm_sparse(_ptr(X), _ptr(V), _ptr(meta), M, N, K, _ptr(Y), _ptr(S),
                                   nthreads), "gemm_sparse")
    return Y, S


def moe(X: np.ndarray, routing: np.ndarray, W: np.ndarray, nthreads: int = 0):
    """(Y [T, topk, N], S) for decoded expert weights W [E, N, K] and routing [T, topk]."""
    X = np.ascontiguousarray(X, dtype=np.float64)
    W = np.ascontiguousarray(W, dtype=np.float64)
    routing = np.ascontiguousarray(routing, dtype=np.int32)
    T, K = X.shape
    E, N, _ = W.shape
    topk = routing.shape[1]
    Y = np.empty((T, topk, N), dtype=np.float64)
    S = np.empty((T, topk, N), dtype=np.float64)
    _check(lib().sp24o_moe(_ptr(X), _ptr(routing), _ptr(W), T, topk, E, N, K, _ptr(Y), _ptr(S),
                           nthreads), "moe")
    return Y, S


def max_threads() -> int:
    return int(lib().sp24o_max_threads())


def within_tolerance(y_gpu: np.ndarray, y_ref: np.ndarray, s_ref: np.ndarray, rel: float = 1e-3):
    """Per-output acceptance: |y_gpu - y_ref| <= rel * S, and y_gpu == 0 where S == 0."""
    y_gpu = np.asarray(y_gpu, dtype=np.float64)
    err = np.abs(y_gpu - y_ref)
    ok = np.where(s_ref > 0, err <= rel * s_ref, y_gpu == 0)
    return ok


def round_to_16(x: np.ndarray, dtype: int) -> np.ndarray:
    """fp64 values held in a 16-bit type (round to nearest even; through fp32 for bf16), as fp64."""
    x = np.asarray(x, dtype=np.float64)
    if dtype == F16:
        return x.astype(np.float16).astype(np.float64)
    u = x.astype(np.float32).view(np.uint32).astype(np.uint64)
    r = ((u + 0x7FFF + ((u >> 16) & 1)) >> 16) << 16
    return r.astype(np.uint32).view(np.float32).astype(np.float64)


def moe_block(X: np.ndarray, routing: np.ndarray, router_w: np.ndarray, Wg: np.ndarray, Wu: np.ndarray,
              Wd: np.ndarray, hdtype: int):
    """(Y, S) of the routed expert block on decoded fp64 operands ([P1] "Concurrency, not sparsity,
    is the lever"): for each token t and slot s with expert e = routing[t, s],
    h = SiLU(Wg[e] x_t) * (Wu[e] x_t) held in the 16-bit type `hdtype`, and
    Y[t] = sum_s router_w[t, s] * Wd[e] h;  S[t] = sum_s |router_w| |Wd[e]| |h| (tolerance scale).
    X [T, H]; Wg, Wu [E, F, H]; Wd [E, H, F]."""
    T, topk = routing.shape
    H = X.shape[1]
    Y = np.zeros((T, H))
    S = np.zeros((T, H))
    for t in range(T):
        for s in range(topk):
            e = int(routing[t, s])
            r = float(router_w[t, s])
            g = Wg[e] @ X[t]
            u = Wu[e] @ X[t]
            h = round_to_16(g / (1.0 + np.exp(-g)) * u, hdtype)
            Y[t] += r * (Wd[e] @ h)
            S[t] += abs(r) * (np.abs(Wd[e]) @ np.abs(h))
    return Y, S

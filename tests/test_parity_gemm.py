"""GPU parity of the dense and 2:4-sparse GEMM/GEMV against the oracle's fp64 GEMM on decoded
operands: |y - y_ref| <= 1e-3 * sum_k |x||w| per output.  Each side runs the whole pipeline
(prune -> compress -> NVFP4) from the same seeded inputs on its own."""
import numpy as np
import pytest
import torch

import fp16_gemm_b200 as sp
import oracle
import synth
from helpers import ORACLE_DT, assert_gemm_close, to_dev

pytestmark = pytest.mark.gpu

REL = 1e-3  # the tolerance the method's statement fixes for GEMM outputs


def make_case(xfmt, wfmt, M, N, K, seed, w_sigma=1.0):
    """Raw inputs: x and w drawn in a 16-bit source type (bf16 for NVFP4 operands)."""
    g = synth.rng(seed)
    xsrc = "f16" if xfmt == "f16" else "bf16"
    wsrc = "f16" if wfmt == "f16" or (wfmt == "nvfp4" and xfmt == "f16") else "bf16"
    if xfmt == "nvfp4":
        wsrc = "bf16"
    X = synth.draw(g, (M, K), xsrc)
    W = synth.draw(g, (N, K), wsrc, w_sigma)
    return X, xsrc, W, wsrc


def oracle_side(X, xsrc, xfmt, W, wsrc, wfmt, sparse):
    if xfmt == "nvfp4":
        c, s, ts = oracle.nvfp4_encode(X, ORACLE_DT[xsrc])
        Xd = oracle.nvfp4_decode(c, s, ts)
    else:
        Xd = oracle.to_double(X, ORACLE_DT[xsrc])
    od = ORACLE_DT[wsrc]
    if sparse:
        V, meta = oracle.compress_24(W, od)
        if wfmt == "nvfp4":
            c, s, ts = oracle.nvfp4_encode(V, od)
            Vd = oracle.nvfp4_decode(c, s, ts)
        else:
            Vd = oracle.to_double(V, od)
        return oracle.gemm_sparse(Xd, Vd, meta)
    if wfmt == "nvfp4":
        c, s, ts = oracle.nvfp4_encode(W, od)
        Wd = oracle.nvfp4_decode(c, s, ts)
    else:
        Wd = oracle.to_double(W, od)
    return oracle.gemm(Xd, Wd)


def gpu_side(X, xsrc, xfmt, W, wsrc, wfmt, sparse, algo=sp.ALGO_AUTO):
    x = to_dev(X, xsrc)
    if xfmt == "nvfp4":
        x = sp.quantize_nvfp4(x)
    w = to_dev(W, wsrc)
    K = W.shape[1]
    if sparse:
        v, m = sp.prune_compress_24(w)
        if wfmt == "nvfp4":
            v = sp.quantize_nvfp4(v)
        return sp.gemm_sparse24(x, sp.Sparse24(v, m.view(W.shape[0], K // 8)), K, algo=algo)
    if wfmt == "nvfp4":
        w = sp.quantize_nvfp4(w)
    return sp.gemm_dense(x, w, algo=algo)


FORMATS = [("f16", "f16"), ("bf16", "bf16"), ("bf16", "nvfp4"), ("f16", "nvfp4"), ("nvfp4", "nvfp4")]
SHAPES = [(16, 256, 512), (1, 64, 256), (5, 72, 384), (33, 130, 640), (64, 96, 1024), (100, 64, 512)]


@pytest.mark.parametrize("sparse", [False, True], ids=["dense", "sparse24"])
@pytest.mark.parametrize("fmt", FORMATS, ids=lambda f: f"x{f[0]}-w{f[1]}")
@pytest.mark.parametrize("shape", SHAPES, ids=lambda s: "x".join(map(str, s)))
def test_gemm_parity(fmt, shape, sparse):
    xfmt, wfmt = fmt
    M, N, K = shape
    X, xs, W, ws = make_case(xfmt, wfmt, M, N, K, seed=M * 1000 + N + K)
    Y, S = oracle_side(X, xs, xfmt, W, ws, wfmt, sparse)
    y = gpu_side(X, xs, xfmt, W, ws, wfmt, sparse)
    assert_gemm_close(y, Y, S, REL)
    assert sp.last_device_error() == sp.OK


def test_fp16_toy_sparse_vs_dense_on_pruned():
    """W fp16 [256, 512], X fp16 [16, 512]: check -> prune -> compress -> sparse GEMM, against
    the dense GEMM on the pruned W, both on the GPU and against the oracle."""
    d = synth.fp16_toy()
    X, W = d["X"], d["W"]
    x, w = to_dev(X, "f16"), to_dev(W, "f16")
    p, n = sp.check_24(w)
    assert int(n.item()) == oracle.check_24(W, oracle.F16)[1]
    v, m = sp.prune_compress_24(w)
    y_sp = sp.gemm_sparse24(x, sp.Sparse24(v, m), 512)
    y_dn = sp.gemm_dense(x, sp.decompress_24(v, m, W.shape))
    Y, S = oracle.gemm(oracle.to_double(X, oracle.F16),
                       oracle.to_double(oracle.prune_24(W, oracle.F16), oracle.F16))
    assert_gemm_close(y_sp, Y, S)
    assert_gemm_close(y_dn, Y, S)


@pytest.mark.parametrize("sparse", [False, True], ids=["dense", "sparse24"])
def test_decode_workload_full_size(sparse):
    """bf16 x [8, 5120], NVFP4 w [5120, 5120] (N(0, 0.02)), every output checked."""
    d = synth.decode_nvfp4()
    Y, S = oracle_side(d["X"], "bf16", "bf16", d["W"], "bf16", "nvfp4", sparse)
    y = gpu_side(d["X"], "bf16", "bf16", d["W"], "bf16", "nvfp4", sparse)
    assert_gemm_close(y, Y, S)


def test_k_zero_writes_zeros():
    x = torch.zeros((4, 0), dtype=torch.float16, device="cuda")
    w = torch.zeros((8, 0), dtype=torch.float16, device="cuda")
    y = torch.full((4, 8), 7.0, device="cuda")
    sp.gemm_dense(x, w, out=y)
    assert not y.any()


ALGO_SHAPES = [(16, 256, 512), (130, 200, 640), (512, 384, 1024), (200, 136, 192)]


@pytest.mark.parametrize("algo", [sp.ALGO_SKINNY, sp.ALGO_TILED], ids=["skinny", "tiled"])
@pytest.mark.parametrize("sparse", [False, True], ids=["dense", "sparse24"])
@pytest.mark.parametrize("fmt", FORMATS, ids=lambda f: f"x{f[0]}-w{f[1]}")
@pytest.mark.parametrize("shape", ALGO_SHAPES, ids=lambda s: "x".join(map(str, s)))
def test_gemm_both_kernels(fmt, shape, sparse, algo):
    """The skinny (warp-MMA) and the tiled (tcgen05) kernels on the same problems, with token
    and weight-row tails that do not fill a tile."""
    xfmt, wfmt = fmt
    M, N, K = shape
    if K % 64 and (wfmt == "nvfp4" or xfmt == "nvfp4"):
        pytest.skip("NVFP4 2:4 operands need K % 64")
    X, xs, W, ws = make_case(xfmt, wfmt, M, N, K, seed=M * 7 + N * 3 + K)
    Y, S = oracle_side(X, xs, xfmt, W, ws, wfmt, sparse)
    y = gpu_side(X, xs, xfmt, W, ws, wfmt, sparse, algo=algo)
    assert_gemm_close(y, Y, S, REL)
    assert sp.last_device_error() == sp.OK


def _sampled(xfmt, wfmt, sparse, M, N, K, rows, seed=0, w_sigma=1.0):
    X, xs, W, ws = make_case(xfmt, wfmt, M, N, K, seed=seed, w_sigma=w_sigma)
    y = gpu_side(X, xs, xfmt, W, ws, wfmt, sparse)
    torch.cuda.synchronize()
    # the oracle on a seeded subset of output rows (x quantisation is per tensor, so NVFP4 x is
    # encoded whole and the sampled rows decoded from it)
    if xfmt == "nvfp4":
        c, s, ts = oracle.nvfp4_encode(X, ORACLE_DT[xs])
        Xd = oracle.nvfp4_decode(c[rows], s[rows], ts)
    else:
        Xd = oracle.to_double(np.ascontiguousarray(X[rows]), ORACLE_DT[xs])
    od = ORACLE_DT[ws]
    if sparse:
        V, meta = oracle.compress_24(W, od)
        if wfmt == "nvfp4":
            c, s, ts = oracle.nvfp4_encode(V, od)
            Vd = oracle.nvfp4_decode(c, s, ts)
        else:
            Vd = oracle.to_double(V, od)
        Y, S = oracle.gemm_sparse(Xd, Vd, meta)
    else:
        if wfmt == "nvfp4":
            c, s, ts = oracle.nvfp4_encode(W, od)
            Wd = oracle.nvfp4_decode(c, s, ts)
        else:
            Wd = oracle.to_double(W, od)
        Y, S = oracle.gemm(Xd, Wd)
    assert_gemm_close(y[torch.as_tensor(rows, device=y.device)], Y, S)


@pytest.mark.parametrize("sparse", [False, True], ids=["dense", "sparse24"])
def test_prefill_w4a4_4096_sampled(sparse):
    """NVFP4 x and w at M = N = K = 4096 (the prefill shape), 24 sampled token rows x all 4096
    outputs checked against the oracle."""
    rows = np.sort(synth.rng(77).choice(4096, 24, replace=False))
    _sampled("nvfp4", "nvfp4", sparse, 4096, 4096, 4096, rows)


@pytest.mark.parametrize("M", [1024, 16384])
@pytest.mark.parametrize("sparse", [False, True], ids=["dense", "sparse24"])
def test_fp16_msweep_sampled(M, sparse):
    """FP16 W [5120, 5120] and X [M, 5120] of the M sweep, sampled token rows."""
    rows = np.sort(synth.rng(M).choice(M, 8, replace=False))
    _sampled("f16", "f16", sparse, M, 5120, 5120, rows, seed=5)

"""GPU parity of the persistent decode GEMV (16-bit x of at most 8 tokens, NVFP4 weights dense
or 2:4) against the oracle's fp64 GEMM, on shapes that stress how it splits work: rows of
weight units shared between neighbouring CTAs, many tiles per CTA (short K), fewer than 8
tokens (the missing token rows of x read as zeros), K at the kernel's limit (8192), and fewer
units than SMs.  Also checks that the skinny and decode paths agree with each other."""
import numpy as np
import pytest
import torch

import fp16_gemm_b200 as sp
from helpers import assert_gemm_close
from test_parity_gemm import gpu_side, make_case, oracle_side

pytestmark = pytest.mark.gpu

DECODE_SHAPES = [
    (8, 5120, 1024),   # 4 or 2 units per tile, tiles split across CTAs
    (1, 2048, 512),    # one or two units per tile: many tiles per CTA
    (3, 1040, 2560),   # 3 tokens; 65 tiles; odd unit counts per CTA
    (8, 48, 8192),     # largest K: x fills 128 KB of shared memory; fewer units than SMs
    (5, 16, 512),      # a single tile
    (8, 4096, 4608),   # 18 / 9 units per tile
    (3, 2560, 2048),   # 3 tokens on the whole-tile kernel (160 tiles)
    (8, 4736, 7168),   # K above the whole-tile kernel's 5120: the k-group decode kernel
]


@pytest.mark.parametrize("sparse", [False, True], ids=["dense", "sparse24"])
@pytest.mark.parametrize("xdt", ["bf16", "f16"])
@pytest.mark.parametrize("shape", DECODE_SHAPES, ids=lambda s: "x".join(map(str, s)))
def test_decode_gemv_parity(shape, xdt, sparse):
    M, N, K = shape
    X, xs, W, ws = make_case(xdt, "nvfp4", M, N, K, seed=M * 7919 + N * 31 + K, w_sigma=0.02)
    Y, S = oracle_side(X, xs, xdt, W, ws, "nvfp4", sparse)
    y = gpu_side(X, xs, xdt, W, ws, "nvfp4", sparse)
    assert_gemm_close(y, Y, S)
    assert sp.last_device_error() == sp.OK


@pytest.mark.parametrize("sparse", [False, True], ids=["dense", "sparse24"])
@pytest.mark.parametrize("shift", [-100, 60])
def test_decode_tile_bf16_far_from_unit_range(shift, sparse):
    """bf16 x times 2^shift (every value still a normal bf16 number, far outside f16's range):
    the whole-tile kernel runs its MMAs in f16 on x times a power of two that each warp picks
    for its K range, so the result still meets the oracle's tolerance at both ends."""
    M, N, K = 8, 2560, 1024
    X, xs, W, ws = make_case("bf16", "nvfp4", M, N, K, seed=4242 + shift, w_sigma=0.02)
    f = (X.astype(np.uint32) << 16).view(np.float32) * np.float32(2.0 ** shift)
    X = (f.view(np.uint32) >> 16).astype(np.uint16)
    Y, S = oracle_side(X, xs, "bf16", W, ws, "nvfp4", sparse)
    y = gpu_side(X, xs, "bf16", W, ws, "nvfp4", sparse)
    assert_gemm_close(y, Y, S)
    assert sp.last_device_error() == sp.OK


@pytest.mark.parametrize("sparse", [False, True], ids=["dense", "sparse24"])
def test_decode_matches_tiled_kernel(sparse):
    """The same NVFP4 product through the decode GEMV (AUTO at M = 8) and the tensor-core tiled
    kernel (ALGO_TILED): both within the oracle tolerance of each other's inputs."""
    M, N, K = 8, 1024, 2048
    X, xs, W, ws = make_case("bf16", "nvfp4", M, N, K, seed=99, w_sigma=0.02)
    Y, S = oracle_side(X, xs, "bf16", W, ws, "nvfp4", sparse)
    y_auto = gpu_side(X, xs, "bf16", W, ws, "nvfp4", sparse)
    y_tiled = gpu_side(X, xs, "bf16", W, ws, "nvfp4", sparse, algo=sp.ALGO_TILED)
    assert_gemm_close(y_auto, Y, S)
    assert_gemm_close(y_tiled, Y, S)


def test_repeated_launches_reuse_no_state():
    """Two back-to-back calls, the second into an output pre-filled with 7.0: the results agree
    to fp32 summation-order noise (the output is cleared by each call and no shared-memory
    state leaks between launches; partial sums meet through fp32 atomics, whose order varies)."""
    M, N, K = 8, 2048, 1024
    X, xs, W, ws = make_case("bf16", "nvfp4", M, N, K, seed=5, w_sigma=0.02)
    x = torch.from_numpy(X.view("int16")).view(torch.bfloat16).cuda()
    w = sp.quantize_nvfp4(torch.from_numpy(W.view("int16")).view(torch.bfloat16).cuda())
    y1 = sp.gemm_dense(x, w)
    y2 = sp.gemm_dense(x, w, out=torch.full_like(y1, 7.0))
    torch.cuda.synchronize()
    assert torch.allclose(y1, y2, rtol=1e-5, atol=1e-5)

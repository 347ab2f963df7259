"""GPU parity of the 16-bit CTA-pair tensor-core GEMM (tcgen05 cta_group::2, kind::f16), dense
and 2:4, against the oracle's fp64 GEMM on shapes that span several 256-row weight tiles and
token tiles with ragged edges in both, and of the 2:4 metadata image it reads
(sp24_prepare_sparse) against that image's definition, byte for byte."""
import numpy as np
import pytest
import torch

import fp16_gemm_b200 as sp
from helpers import assert_gemm_close
from test_parity_gemm import gpu_side, make_case, oracle_side

pytestmark = pytest.mark.gpu


def image_definition(meta: np.ndarray, rows: int, K: int) -> np.ndarray:
    """The metadata image as sp24.h defines it: per 128-row block rb and 128-K chunk kc a 2 KB
    tile; its 16-byte row l holds, for rows m = 128 rb + 16 (l // 16) + l % 8 and m + 8 and half
    h = (l // 8) % 2, in word t the nibble bytes 16 kc + 4 t + 2 h, +1 of row m (low half) and of
    row m + 8 (high half); rows past `rows` read as 0x44."""
    rp = (rows + 255) // 256 * 256
    padded = np.full((rp, K // 8), 0x44, np.uint8)
    padded[:rows] = meta
    kcs = K // 128
    out = np.zeros((rp // 128, kcs, 128, 4, 4), np.uint8)
    lanes = np.arange(128)
    for rb in range(rp // 128):
        m = 128 * rb + 16 * (lanes // 16) + lanes % 8
        h = (lanes // 8) % 2
        for kc in range(kcs):
            for t in range(4):
                b = 16 * kc + 4 * t + 2 * h
                out[rb, kc, :, t, 0] = padded[m, b]
                out[rb, kc, :, t, 1] = padded[m, b + 1]
                out[rb, kc, :, t, 2] = padded[m + 8, b]
                out[rb, kc, :, t, 3] = padded[m + 8, b + 1]
    return out.reshape(-1)


@pytest.mark.parametrize("rows,K", [(300, 256), (512, 384), (40, 128)])
def test_metadata_image_matches_its_definition(rows, K):
    g = torch.Generator(device="cuda")
    g.manual_seed(rows + K)
    w = torch.randn((rows, K), generator=g, device="cuda").half()
    _, meta = sp.prune_compress_24(w)
    meta = meta.view(rows, K // 8)
    img = sp.prepare_sparse(meta, rows, K)
    torch.cuda.synchronize()
    assert np.array_equal(img.cpu().numpy(), image_definition(meta.cpu().numpy(), rows, K))


PAIR_SHAPES = [
    (200, 520, 384),    # 2 x 3 pair tiles (BN 256 / 128-token halves), ragged N and M
    (1000, 768, 1024),  # 4 token tiles, 3 weight tiles, several tiles per pair
    (65, 300, 256),     # BN = 128, one partial token tile
]


@pytest.mark.parametrize("sparse", [False, True], ids=["dense", "sparse24"])
@pytest.mark.parametrize("dt", ["f16", "bf16"])
@pytest.mark.parametrize("shape", PAIR_SHAPES, ids=lambda s: "x".join(map(str, s)))
def test_pair_gemm_parity(shape, dt, sparse):
    M, N, K = shape
    X, xs, W, ws = make_case(dt, dt, M, N, K, seed=M * 131 + N * 7 + K)
    Y, S = oracle_side(X, xs, dt, W, ws, dt, sparse)
    y = gpu_side(X, xs, dt, W, ws, dt, sparse)
    assert_gemm_close(y, Y, S)
    assert sp.last_device_error() == sp.OK

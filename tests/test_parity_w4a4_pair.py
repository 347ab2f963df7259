"""The W4A4 GEMM on the persistent CTA-pair kernel (tcgen05 cta_group::2, block-scaled FP4
MMA) against the oracle's fp64 GEMM on decoded operands, |y - y_ref| <= 1e-3 sum_k |x||w| per
output, and the block-scale tile rearrangement it reads ("NVFP4 vs 2:4 sparse: where the other
half of the petaflop went", "The ladder, top to bottom": the dense NVFP4 GEMM at prefill sizes).
Shapes cover both token-tile widths (128 at M <= 128, 256 above), weight-row tails that leave
the odd CTA of a pair with no rows, token tails, and more tiles than CTA pairs so that pairs
reuse both TMEM accumulators (the 256-wide ones overlap in 64 columns)."""
import numpy as np
import pytest
import torch

import fp16_gemm_b200 as sp
import oracle
import synth
from helpers import assert_gemm_close, to_dev

pytestmark = pytest.mark.gpu


def _scale_tiles(scales: np.ndarray) -> np.ndarray:
    """The scale tile order written out from its definition: tile (rb, kc) holds, for row r of
    the 128-row block rb, the four scales of 64-column chunk kc at byte 16 (r % 32) + 4 (r / 32)."""
    rows, kb = scales.shape
    kc = kb // 4
    rb_n = -(-rows // 128)
    out = np.zeros(rb_n * kc * 512, dtype=np.uint8)
    for r in range(rows):
        rb, rr = divmod(r, 128)
        for c in range(kc):
            base = (rb * kc + c) * 512 + 16 * (rr % 32) + 4 * (rr // 32)
            out[base:base + 4] = scales[r, 4 * c:4 * c + 4]
    return out


def _code_tiles(codes: np.ndarray) -> np.ndarray:
    """The code image from its definition: tile (rb, kc) of 16 KB holds row r of the block at
    byte 128 r, its 16-byte piece c at 16 (c ^ (r % 8))."""
    rows, half = codes.shape
    kc = half // 128
    rb_n = -(-rows // 128)
    out = np.zeros(rb_n * kc * 16384, dtype=np.uint8)
    for r in range(rows):
        rb, rr = divmod(r, 128)
        for k in range(kc):
            for c in range(8):
                dst = (rb * kc + k) * 16384 + 128 * rr + 16 * (c ^ (rr % 8))
                out[dst:dst + 16] = codes[r, 128 * k + 16 * c:128 * k + 16 * c + 16]
    return out


@pytest.mark.parametrize("rows,cols", [(1, 256), (128, 256), (200, 512), (300, 1024)])
def test_tile_images_match_their_definition(rows, cols):
    g = synth.rng(rows + cols)
    c = g.integers(0, 256, size=(rows, cols // 2), dtype=np.uint8)
    s = g.integers(0, 256, size=(rows, cols // 16), dtype=np.uint8)
    q = sp.NVFP4Tensor(to_dev(c, "u8"), to_dev(s, "u8"), torch.ones(1, dtype=torch.float32, device="cuda"))
    t = sp.to_mma(q)
    torch.cuda.synchronize()
    assert np.array_equal(t.codes.cpu().numpy(), _code_tiles(c))
    assert np.array_equal(t.scales.cpu().numpy(), _scale_tiles(s))


def _oracle(X, W):
    cx, sx, tx = oracle.nvfp4_encode(X, oracle.BF16)
    cw, sw, tw = oracle.nvfp4_encode(W, oracle.BF16)
    return oracle.gemm(oracle.nvfp4_decode(cx, sx, tx), oracle.nvfp4_decode(cw, sw, tw))


SHAPES = [
    (65, 2000, 512),     # 128-wide token tiles, weight tail of 208 rows
    (128, 256, 256),     # one tile, one 256-K stage
    (300, 520, 768),     # 256-wide token tiles, token tail 44, weight tail 8 (odd CTA empty)
    (1280, 4096, 256),   # 80 tiles over at most 74 pairs: accumulators reused
    (520, 2304, 1024),   # 27 tiles, several K stages, both tails
]


@pytest.mark.parametrize("shape", SHAPES, ids=lambda s: "x".join(map(str, s)))
def test_pair_kernel_every_output(shape):
    M, N, K = shape
    g = synth.rng(M * 31 + N * 7 + K)
    X = synth.draw(g, (M, K), "bf16")
    W = synth.draw(g, (N, K), "bf16")
    Y, S = _oracle(X, W)
    x, w = sp.quantize_nvfp4(to_dev(X, "bf16")), sp.quantize_nvfp4(to_dev(W, "bf16"))
    # plain NVFP4 operands (scales relaid in the workspace) and pre-tiled ones give the same bits
    y_plain = sp.gemm_dense(x, w)
    y_mma = sp.gemm_dense(sp.to_mma(x), sp.to_mma(w))
    y_mixed = sp.gemm_dense(x, sp.to_mma(w))
    torch.cuda.synchronize()
    assert sp.last_device_error() == sp.OK
    assert_gemm_close(y_mma, Y, S)
    assert torch.equal(y_plain, y_mma) and torch.equal(y_mixed, y_mma)


def test_pair_kernel_repeatable_and_zero_scale():
    """Every output is written by exactly one thread (no atomics): two runs are bit-identical;
    an all-zero activation tensor (tensor scale 0, scales 0) gives exact zeros."""
    M, N, K = 512, 1024, 512
    g = synth.rng(3)
    x = sp.quantize_nvfp4(to_dev(synth.draw(g, (M, K), "bf16"), "bf16"))
    w = sp.to_mma(sp.quantize_nvfp4(to_dev(synth.draw(g, (N, K), "bf16"), "bf16")))
    xm = sp.to_mma(x)
    a, b = sp.gemm_dense(xm, w), sp.gemm_dense(xm, w)
    z = sp.to_mma(sp.quantize_nvfp4(torch.zeros((M, K), dtype=torch.bfloat16, device="cuda")))
    y0 = torch.full((M, N), 5.0, device="cuda")
    sp.gemm_dense(z, w, out=y0)
    torch.cuda.synchronize()
    assert torch.equal(a, b)
    assert not y0.any()
    assert sp.last_device_error() == sp.OK

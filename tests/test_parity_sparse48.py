"""GPU parity of the W4A4 GEMM on the sparse FP4 MMA: a pairwise-4:8 weight (kept values as
NVFP4) times activations in 32-value blocks, against the oracle's fp64 product of the decoded
operands, plus the bit-exact 32-value-block activation quantiser."""
import numpy as np
import pytest
import torch

import fp16_gemm_b200 as sp
import oracle
import synth
from helpers import ORACLE_DT, assert_gemm_close, bits, to_dev, to_host

pytestmark = pytest.mark.gpu


def _bits32(x) -> int:
    return int(np.float32(x).view(np.uint32))


@pytest.mark.parametrize("dtype", ["f16", "bf16", "f32"])
@pytest.mark.parametrize("shape", [(1, 32), (7, 96), (130, 512), (33, 2048)], ids=lambda s: "x".join(map(str, s)))
def test_block32_quantiser_bit_exact(dtype, shape):
    g = synth.rng(500 + shape[0])
    x = synth.normal(g, shape) * np.exp(synth.normal(g, (shape[0], 1)))
    t = synth.as_storage(x, dtype)
    c_ref, s_ref, ts_ref = oracle.nvfp4_encode(t, ORACLE_DT[dtype], block=32)
    q = sp.quantize_nvfp4_block32(to_dev(t, dtype))
    torch.cuda.synchronize()
    assert _bits32(q.tensor_scale.item()) == _bits32(ts_ref)
    assert np.array_equal(to_host(q.scales), s_ref)
    assert np.array_equal(to_host(q.codes), c_ref)
    # with a supplied (shared) scale
    ts = torch.tensor([float(ts_ref) * 3], dtype=torch.float32, device="cuda")
    q2 = sp.quantize_nvfp4_block32(to_dev(t, dtype), tensor_scale=ts)
    c2, s2, _ = oracle.nvfp4_encode(t, ORACLE_DT[dtype], tensor_scale=float(ts_ref) * 3, block=32)
    torch.cuda.synchronize()
    assert np.array_equal(to_host(q2.scales), s2) and np.array_equal(to_host(q2.codes), c2)
    assert sp.last_device_error() == sp.OK


def test_block32_quantiser_zero_and_rejects():
    z = torch.zeros((2, 64), dtype=torch.bfloat16, device="cuda")
    q = sp.quantize_nvfp4_block32(z)
    torch.cuda.synchronize()
    assert q.tensor_scale.item() == 0 and not q.scales.any() and not q.codes.any()
    with pytest.raises(sp.SP24Error) as e:
        sp.quantize_nvfp4_block32(torch.zeros((2, 48), dtype=torch.bfloat16, device="cuda"))
    assert e.value.status == sp.ERR_SHAPE


def _decompress48_f64(vals: np.ndarray, meta: np.ndarray, N: int, K: int) -> np.ndarray:
    """Dense fp64 [N, K] from decoded kept values [N, K/2] and the nibble stream."""
    nib = np.stack([meta & 0xF, meta >> 4], 1).ravel()[: N * K // 8].reshape(N, K // 8)
    out = np.zeros((N, K // 8, 4, 2))
    v = vals.reshape(N, K // 8, 2, 2)
    rows = np.arange(N)[:, None]
    ch = np.arange(K // 8)[None, :]
    out[rows, ch, nib & 3] = v[:, :, 0]
    out[rows, ch, nib >> 2] = v[:, :, 1]
    return out.reshape(N, K)


def _case(M, N, K, seed):
    g = synth.rng(seed)
    X = synth.draw(g, (M, K), "bf16")
    W = synth.draw(g, (N, K), "bf16", 0.02)
    return X, W


def _run(M, N, K, seed):
    X, W = _case(M, N, K, seed)
    # oracle
    v_ref, m_ref = oracle.compress_48(W, oracle.BF16)
    vc, vs, vts = oracle.nvfp4_encode(v_ref, oracle.BF16)
    Wd = _decompress48_f64(oracle.nvfp4_decode(vc, vs, vts), m_ref, N, K)
    xc, xs, xts = oracle.nvfp4_encode(X, oracle.BF16, block=32)
    Xd = oracle.nvfp4_decode(xc, xs, xts, block=32)
    Y, S = oracle.gemm(Xd, Wd)
    # CUDA path
    v, m = sp.prune_compress_48(to_dev(W, "bf16"))
    vq = sp.quantize_nvfp4(v)
    xq = sp.quantize_nvfp4_block32(to_dev(X, "bf16"))
    y = sp.gemm_sparse48(xq, sp.Sparse48(vq, m), K)
    torch.cuda.synchronize()
    assert sp.last_device_error() == sp.OK
    # the operands are the oracle's, byte for byte
    assert np.array_equal(bits(to_host(v)), bits(v_ref)) and np.array_equal(to_host(m), m_ref)
    assert np.array_equal(to_host(vq.codes), vc) and np.array_equal(to_host(vq.scales), vs)
    assert np.array_equal(to_host(xq.codes), xc) and np.array_equal(to_host(xq.scales), xs)
    assert_gemm_close(y, Y, S)
    # the same product on the CTA-pair kernel from tile images of the same operands
    y2 = sp.gemm_sparse48(sp.b32_to_mma(xq), sp.sparse48_to_mma(sp.Sparse48(vq, m), K), K)
    torch.cuda.synchronize()
    assert sp.last_device_error() == sp.OK
    assert_gemm_close(y2, Y, S)


@pytest.mark.parametrize("mnk", [(1, 128, 512), (96, 200, 1024), (128, 256, 512), (300, 384, 1536),
                                 (129, 129, 2048), (512, 130, 1024), (1280, 4096, 512)],
                         ids=lambda t: "x".join(map(str, t)))
def test_gemm_sparse48(mnk):
    """Every output, at sizes spanning several 128-row weight tiles, both activation tile widths
    (128 for M <= 256, 256 above), ragged M and N, and several 512-wide K stages; on tile images
    also more pair tiles (80) than CTA pairs, so pairs reuse both TMEM accumulators."""
    _run(*mnk, seed=510 + sum(mnk))


def test_gemm_sparse48_rejects():
    X, W = _case(4, 128, 512, 520)
    v, m = sp.prune_compress_48(to_dev(W, "bf16"))
    vq = sp.quantize_nvfp4(v)
    xq16 = sp.quantize_nvfp4(to_dev(X, "bf16"))
    xo = sp._Operand(sp.NVFP4, xq16.codes.data_ptr(), xq16.scales.data_ptr(), xq16.tensor_scale.data_ptr())
    wo = sp._SparseOperand(sp.NVFP4, vq.codes.data_ptr(), vq.scales.data_ptr(), vq.tensor_scale.data_ptr(),
                           m.data_ptr())
    y = torch.empty((4, 128), dtype=torch.float32, device="cuda")
    L = sp.lib()
    import ctypes
    assert L.sp24_gemm_sparse48(ctypes.byref(xo), ctypes.byref(wo), 4, 128, 512, y.data_ptr(), None) == sp.ERR_DTYPE
    xo.format = sp.NVFP4_B32
    assert L.sp24_gemm_sparse48(ctypes.byref(xo), ctypes.byref(wo), 4, 128, 256, y.data_ptr(), None) == sp.ERR_SHAPE
    assert L.sp24_gemm_sparse48(ctypes.byref(xo), ctypes.byref(wo), 0, 128, 512, y.data_ptr(), None) == sp.OK
    torch.cuda.synchronize()
    assert sp.last_device_error() == sp.OK


def _sampled48(M, N, K, rows, d):
    X, W = d["X"], d["W"]
    v_ref, m_ref = oracle.compress_48(W, oracle.BF16)
    vc, vs, vts = oracle.nvfp4_encode(v_ref, oracle.BF16)
    Wd = _decompress48_f64(oracle.nvfp4_decode(vc, vs, vts), m_ref, N, K)
    # the tensor scale of x is the whole tensor's; the sampled rows are encoded with it
    _, _, xts = oracle.nvfp4_encode(X, oracle.BF16, block=32)
    Xs = np.ascontiguousarray(X[rows])
    xc, xs, _ = oracle.nvfp4_encode(Xs, oracle.BF16, tensor_scale=float(xts), block=32)
    Y, S = oracle.gemm(oracle.nvfp4_decode(xc, xs, xts, block=32), Wd)
    v, m = sp.prune_compress_48(to_dev(W, "bf16"))
    xq = sp.quantize_nvfp4_block32(to_dev(X, "bf16"))
    w48 = sp.Sparse48(sp.quantize_nvfp4(v), m)
    y = sp.gemm_sparse48(xq, w48, K)
    y2 = sp.gemm_sparse48(sp.b32_to_mma(xq), sp.sparse48_to_mma(w48, K), K)
    torch.cuda.synchronize()
    assert sp.last_device_error() == sp.OK
    assert _bits32(xq.tensor_scale.item()) == _bits32(xts)
    sel = torch.as_tensor(rows, device=y.device)
    assert_gemm_close(y[sel], Y, S)
    assert_gemm_close(y2[sel], Y, S)


def test_prefill_4096_sampled():
    """The W4A4 prefill shape M = N = K = 4096 in the configuration the sweep times (256-wide
    activation tiles): 24 sampled token rows x all 4096 outputs against the oracle."""
    rows = np.sort(synth.rng(78).choice(4096, 24, replace=False))
    _sampled48(4096, 4096, 4096, rows, synth.prefill_w4a4())


def test_msweep_16384_sampled():
    """The largest M of the sweep's W4A4 lines: x [16384, 5120], w [5120, 5120], 8 sampled rows."""
    rows = np.sort(synth.rng(79).choice(16384, 8, replace=False))
    d = {"X": synth.draw(synth.rng(16384), (16384, 5120), "bf16"), "W": synth.draw(synth.rng(0), (5120, 5120), "bf16")}
    _sampled48(16384, 5120, 5120, rows, d)


def _tiles(a: np.ndarray, rows_pad: int, words: int) -> np.ndarray:
    """Scale tiles from their definition: per 128-row block, `words` 4-byte groups per row, tile
    (rb, w) holding row r's group w at byte 16 (r % 32) + 4 (r / 32)."""
    rows = a.shape[0]
    out = np.zeros(rows_pad // 128 * words * 512, dtype=np.uint8)
    for r in range(rows):
        rb, rr = divmod(r, 128)
        for w in range(words):
            base = (rb * words + w) * 512 + 16 * (rr % 32) + 4 * (rr // 32)
            out[base:base + 4] = a[r, 4 * w:4 * w + 4]
    return out


def _code_image(c: np.ndarray, rows_pad: int) -> np.ndarray:
    rows, half = c.shape
    kc = half // 128
    out = np.zeros(rows_pad // 128 * kc * 16384, dtype=np.uint8)
    for r in range(rows):
        rb, rr = divmod(r, 128)
        for k in range(kc):
            for p in range(8):
                dst = (rb * kc + k) * 16384 + 128 * rr + 16 * (p ^ (rr % 8))
                out[dst:dst + 16] = c[r, 128 * k + 16 * p:128 * k + 16 * p + 16]
    return out


@pytest.mark.parametrize("rows,K", [(1, 512), (130, 1024), (300, 512)])
def test_pair_images_match_their_definition(rows, K):
    """Tile images of a pairwise-4:8 weight (rows padded to 256, metadata padding 0x44) and of
    block-32 activations, byte for byte against their definitions."""
    g = synth.rng(rows + K)
    vc = g.integers(0, 256, size=(rows, K // 4), dtype=np.uint8)
    vs = g.integers(0, 256, size=(rows, K // 32), dtype=np.uint8)
    mt = g.integers(0, 256, size=(rows, K // 16), dtype=np.uint8)
    one = torch.ones(1, dtype=torch.float32, device="cuda")
    w = sp.Sparse48(sp.NVFP4Tensor(to_dev(vc, "u8"), to_dev(vs, "u8"), one), to_dev(mt.reshape(-1), "u8"))
    im = sp.sparse48_to_mma(w, K)
    rp = -(-rows // 256) * 256
    meta_ref = np.full(rp // 128 * (K // 256) * 2048, 0x44, dtype=np.uint8)
    for r in range(rows):
        rb, rr = divmod(r, 128)
        for t in range(K // 256):
            dst = (rb * (K // 256) + t) * 2048 + 16 * rr
            meta_ref[dst:dst + 16] = mt[r, 16 * t:16 * t + 16]
    xc = g.integers(0, 256, size=(rows, K // 2), dtype=np.uint8)
    xs = g.integers(0, 256, size=(rows, K // 32), dtype=np.uint8)
    xi = sp.b32_to_mma(sp.NVFP4Tensor(to_dev(xc, "u8"), to_dev(xs, "u8"), one))
    torch.cuda.synchronize()
    assert np.array_equal(to_host(im.values), _code_image(vc, rp))
    assert np.array_equal(to_host(im.scales), _tiles(vs, rp, K // 128))
    assert np.array_equal(to_host(im.meta), meta_ref)
    xp = -(-rows // 128) * 128
    assert np.array_equal(to_host(xi.codes), _code_image(xc, xp))
    assert np.array_equal(to_host(xi.scales), _tiles(xs, xp, K // 128))

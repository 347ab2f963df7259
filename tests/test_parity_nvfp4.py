"""GPU parity of a3 (NVFP4 quantisation): codes, block scales and tensor scale bit-exact against
the oracle on the same seeded inputs; decode against the oracle's fp64 decode."""
import numpy as np
import pytest
import torch

import fp16_gemm_b200 as sp
import oracle
import synth
from helpers import ORACLE_DT, f64_to_bf16_bits, to_dev, to_host

pytestmark = pytest.mark.gpu


def _compare(t_np, dtype, ts=None):
    od = ORACLE_DT[dtype]
    c_ref, s_ref, ts_ref = oracle.nvfp4_encode(t_np, od, ts)
    t = to_dev(t_np, dtype)
    ts_dev = None if ts is None else torch.tensor([ts], dtype=torch.float32, device="cuda")
    q = sp.quantize_nvfp4(t, tensor_scale=ts_dev)
    torch.cuda.synchronize()
    assert np.float32(q.tensor_scale.item()).view(np.uint32) == np.float32(ts_ref).view(np.uint32)
    s = to_host(q.scales)
    c = to_host(q.codes)
    bad_s = np.argwhere(s != s_ref)
    assert bad_s.size == 0, f"{len(bad_s)} scale mismatches, first {bad_s[:3].tolist()}"
    bad_c = np.argwhere(c != c_ref)
    assert bad_c.size == 0, f"{len(bad_c)} code mismatches, first {bad_c[:3].tolist()}"
    return q, (c_ref, s_ref, ts_ref)


@pytest.mark.parametrize("dtype", ["f16", "bf16", "f32"])
@pytest.mark.parametrize("shape", [(1, 16), (3, 48), (64, 512), (129, 1040)])
def test_random_rows_of_varied_scale(dtype, shape):
    g = synth.rng(shape[0] * 31 + shape[1])
    x = synth.normal(g, shape) * np.exp(2 * synth.normal(g, (shape[0], 1)))
    _compare(synth.as_storage(x, dtype), dtype)


@pytest.mark.parametrize("dtype", ["bf16", "f32"])
def test_subnormal_block_scales(dtype):
    """Blocks far below the tensor max get E4M3 subnormal scales (and E2M1 half steps)."""
    g = synth.rng(5)
    x = synth.normal(g, (16, 256))
    x[:, :128] *= 1e-3
    x[0, 0] = 40.0
    x[3, 16:32] = 0.0
    _compare(synth.as_storage(x, dtype), dtype)


def test_fp32_tiny_tensor_scale():
    """amax ~1e-36: the tensor scale is an fp32 subnormal; no flush to zero on the GPU."""
    x = synth.normal(synth.rng(6), (4, 64)).astype(np.float32) * np.float32(1e-37)
    _compare(x, "f32")


def test_supplied_shared_scale_and_saturation():
    x = synth.normal(synth.rng(7), (8, 128)).astype(np.float32)
    ts = float(oracle.nvfp4_encode(x, oracle.F32)[2])
    _compare(x, "f32", ts)
    _compare(x, "f32", ts * 8)        # scale of a larger partner tensor
    _compare(x, "f32", ts / 1000.0)   # saturating: codes at 6, scales at 448


def test_zeros_and_negative_zero():
    x = np.zeros((2, 32), np.float32)
    x[1, 3] = -0.0
    x[0, 5] = -1e-9
    x[0, 6] = 1.0
    q, _ = _compare(x, "f32")
    z = np.zeros((2, 32), np.float32)
    z[0, 1] = -0.0
    _compare(z, "f32")


def test_decode_workload_dense_and_sparse():
    """The decode workload's weight, bf16 [5120, 5120] N(0, 0.02): dense NVFP4, and NVFP4 of its
    2:4-compressed values [5120, 2560] (one scale per 16 stored values)."""
    w_np = synth.decode_nvfp4()["W"]
    _compare(w_np, "bf16")
    v_np, _ = oracle.compress_24(w_np, oracle.BF16)
    q, ref = _compare(v_np, "bf16")
    # amax survives pruning: the two tensor scales agree
    assert ref[2] == oracle.nvfp4_encode(w_np, oracle.BF16)[2]


@pytest.mark.parametrize("out", [torch.float32, torch.bfloat16, torch.float16])
def test_dequantize(out):
    x = synth.normal(synth.rng(8), (24, 160)).astype(np.float32)
    c, s, ts = oracle.nvfp4_encode(x, oracle.F32)
    ref = oracle.nvfp4_decode(c, s, ts)
    q = sp.NVFP4Tensor(to_dev(c, "u8"), to_dev(s, "u8"),
                       torch.tensor([ts], dtype=torch.float32, device="cuda"))
    d = to_host(sp.dequantize_nvfp4(q, out))
    if out == torch.float32:
        assert np.array_equal(d.view(np.uint32), ref.astype(np.float32).view(np.uint32))
    elif out == torch.float16:
        assert np.array_equal(d.view(np.uint16), ref.astype(np.float16).view(np.uint16))
    else:
        assert np.array_equal(d, f64_to_bf16_bits(ref))


def test_empty_tensor_writes_scale():
    t = torch.empty((0, 32), dtype=torch.bfloat16, device="cuda")
    q = sp.quantize_nvfp4(t)
    assert q.codes.numel() == 0 and float(q.tensor_scale.item()) == 0.0


def _boundary_blocks(seed, nblocks, ts):
    """fp32 blocks of 16 whose entries sit at, and a few fp32 steps either side of, E2M1's
    rounding boundaries (0.25 ... 5) times the block's decoded scale: entry 0 fixes the block
    max (hence the E4M3 block scale), the other 15 are boundary * sc * (1 + k 2^-24).  The block
    scale sc is worked out the way the method defines it, in fp32, to place the entries; the
    expected codes still come from the oracle."""
    g = synth.rng(seed)
    f32 = np.float32
    d = f32(f32(ts) * f32(6.0))
    bounds = np.array([0.25, 0.75, 1.25, 1.75, 2.5, 3.5, 5.0])
    out = np.zeros((nblocks, 16), np.float32)
    for b in range(nblocks):
        target = int(g.integers(1, 127))                     # an E4M3 code with a finite value
        bmax = f32(6.0 * oracle.e4m3_value(target) * ts)
        sb = oracle.e4m3_round(float(f32(bmax / d)))
        sc = f32(f32(oracle.e4m3_value(sb)) * f32(ts))
        out[b, 0] = bmax
        m = bounds[g.integers(0, len(bounds), size=15)]
        k = g.integers(-5, 6, size=15).astype(np.float64)
        vals = (m * np.float64(sc) * (1.0 + k * 2.0 ** -24)).astype(np.float32)
        vals = np.minimum(vals, bmax)                        # keep entry 0 the block max
        sign = np.where(g.random(15) < 0.5, -1.0, 1.0).astype(np.float32)
        out[b, 1:] = vals * sign
    return out


@pytest.mark.parametrize("ts", [1.0, 3.0517578125e-05, 0.012345, 7.5e-12])
def test_quotients_at_rounding_boundaries(ts):
    """Every entry's quotient |t| / sc lies within a few fp32 steps of an E2M1 rounding boundary
    (including exact ties): the codes must equal the oracle's, which divides entry by entry."""
    t = _boundary_blocks(int(ts * 1e6) % 9973 + 17, 4096, ts).reshape(256, 256)
    _compare(t, "f32", ts)


@pytest.mark.parametrize("dtype", ["bf16", "f16"])
@pytest.mark.parametrize("ts", [0.25, 1.0 / 448, None])
def test_16bit_entries_on_rounding_boundaries(dtype, ts):
    """16-bit entries on a quarter grid with a power-of-two block divisor (tensor scale 1/4): many
    quotients fall exactly on E2M1 rounding boundaries (exact ties) or next to them; the codes
    must equal the oracle's per-entry division and tie-to-even."""
    g = synth.rng(41)
    t = synth.as_storage(np.round(synth.normal(g, (64, 256)) * 8) / 4, dtype)
    _compare(t, dtype, ts)


def _neighbours(q, dtype):
    """q (exact in the storage type) and the storage type's next values below and above it."""
    q = np.asarray(q, dtype=np.float64)
    if dtype == "f32":
        v = q.astype(np.float32)
        return np.concatenate([v, np.nextafter(v, np.float32(0)), np.nextafter(v, np.float32(np.inf))]).astype(np.float64)
    if dtype == "f16":
        v = q.astype(np.float16)
        return np.concatenate([v, np.nextafter(v, np.float16(0)), np.nextafter(v, np.float16(np.inf))]).astype(np.float64)
    b = synth.f32_to_bf16_bits(q.astype(np.float32)).astype(np.int64)
    bits = np.concatenate([b, b - 1, b + 1]).astype(np.uint16)
    return synth.bf16_bits_to_f32(bits).astype(np.float64)


@pytest.mark.parametrize("dtype", ["f32", "bf16", "f16"])
def test_block_scales_at_e4m3_midpoints(dtype):
    """Block maxima exactly on E4M3 rounding midpoints (ties to the even code) and one step of
    the storage type either side, with the tensor scale fp32(1/6), which makes the block divisor
    6 s_t exactly 1: the block scale is E4M3(bmax) rounded at the tie itself.  Normal,
    subnormal and saturating (above 448) maxima; the other entries of each block are fractions of
    its maximum with mixed signs, so their codes are checked under the same scale."""
    e4 = np.array([oracle.e4m3_value(c) for c in range(127)])
    mids = (e4[1:] + e4[:-1]) / 2
    pick = mids[[1, 2, 5, 9, 10, 17, 40, 41, 64, 90, 110, 120, 124, 125]]
    q = _neighbours(np.concatenate([pick, [448.0, 464.0, 4096.0]]), dtype)
    g = synth.rng(52)
    frac = np.array([0.5, -0.25, 0.125, 0.75, -0.0625, 0.875, -0.375, 0.3, 0.6, -0.9, 0.05, 0.2, -0.45, 0.65, 0.95])
    t = np.zeros((q.size, 16))
    t[:, 0] = np.where(g.random(q.size) < 0.5, -q, q)
    t[:, 1:] = q[:, None] * frac[None, :]
    _compare(synth.as_storage(t, dtype), dtype, float(np.float32(1 / 6)))


"""GPU parity of pairwise 4:8 (the sparse pattern of the packed-FP4 MMA kind): eligibility,
prune / compress and decompress bit-exact against the oracle on the same seeded inputs."""
import numpy as np
import pytest
import torch

import fp16_gemm_b200 as sp
import oracle
import synth
from helpers import ORACLE_DT, bits, to_dev, to_host

pytestmark = pytest.mark.gpu

# odd chunk counts (a half-filled last meta byte), several 16 KB ring stages, a ragged last stage
SHAPES = [(1, 8), (3, 24), (37, 200), (64, 512), (5, 8 * 999), (2, 3, 40), (257, 4104)]


def _run(w_np, dtype):
    od = ORACLE_DT[dtype]
    shape = w_np.shape
    w2 = np.ascontiguousarray(w_np.reshape(-1, shape[-1]))
    w = to_dev(w_np, dtype)
    p_ref, n_ref = oracle.check_48(w2, od)
    v_ref, m_ref = oracle.compress_48(w2, od)
    back_ref = oracle.decompress_48(v_ref, m_ref, od, w2.shape)
    p, n = sp.check_48(w)
    v, m = sp.prune_compress_48(w)
    back = sp.decompress_48(v, m, w.shape)
    torch.cuda.synchronize()
    assert np.array_equal(to_host(p).reshape(p_ref.shape), p_ref)
    assert int(n.item()) == n_ref
    assert np.array_equal(bits(to_host(v)).reshape(v_ref.shape), bits(v_ref))
    assert np.array_equal(to_host(m), m_ref)
    assert np.array_equal(bits(to_host(back)).reshape(back_ref.shape), bits(back_ref))
    assert sp.last_device_error() == sp.OK
    return back


@pytest.mark.parametrize("dtype", ["f16", "bf16", "f32"])
@pytest.mark.parametrize("shape", SHAPES, ids=lambda s: "x".join(map(str, s)))
def test_edge_values(dtype, shape):
    g = synth.rng(400 + len(shape) * 11 + shape[-1])
    rows = int(np.prod(shape[:-1]))
    w = synth.pairwise_edge(g, rows, shape[-1], dtype).reshape(shape)
    back = _run(w, dtype)
    _, n = sp.check_48(back)
    assert int(n.item()) == 0  # what pruning leaves is eligible in every chunk


@pytest.mark.parametrize("dtype", ["f16", "bf16", "f32"])
def test_normal_weight(dtype):
    _run(synth.draw(synth.rng(401), (512, 1024), dtype), dtype)


def test_full_size_weight():
    """bf16 [5120, 5120] N(0, 0.02) (the decode workload's weight): no chunk is eligible, and
    prune / compress / decompress match the oracle byte for byte (3.3M chunks, 26 MB in)."""
    w_np = synth.decode_nvfp4()["W"]
    w = to_dev(w_np, "bf16")
    p, n = sp.check_48(w)
    assert int(n.item()) == 5120 * 640 and int(p.sum().item()) == 0
    v, m = sp.prune_compress_48(w)
    v_ref, m_ref = oracle.compress_48(w_np, oracle.BF16)
    assert np.array_equal(bits(to_host(v)), bits(v_ref)) and np.array_equal(to_host(m), m_ref)
    _, n2 = sp.check_48(sp.decompress_48(v, m, w.shape))
    assert int(n2.item()) == 0


@pytest.mark.parametrize("dtype", ["f16", "f32"])
def test_misaligned_views_use_the_scalar_path(dtype):
    eb = 2 if dtype == "f16" else 4
    base = synth.pairwise_edge(synth.rng(402), 3, 8 * 41, dtype)
    w_full = to_dev(base, dtype)
    w = w_full.reshape(-1)[2:2 + 3 * 320].view(3, 320)  # offset by two entries
    assert w.data_ptr() % 16 != 0 and w.data_ptr() % eb == 0
    w_np = np.ascontiguousarray(base.reshape(-1)[2:2 + 3 * 320].reshape(3, 320))
    od = ORACLE_DT[dtype]
    p, n = sp.check_48(w)
    v_out = torch.empty(3 * 160 + 1, dtype=w.dtype, device="cuda")[1:].view(3, 160)  # unaligned values
    v, m = sp.prune_compress_48(w, values_out=v_out)
    back = torch.empty(3 * 320 + 1, dtype=w.dtype, device="cuda")[1:].view(3, 320)
    sp.decompress_48(v, m, (3, 320), out=back)
    torch.cuda.synchronize()
    p_ref, n_ref = oracle.check_48(w_np, od)
    v_ref, m_ref = oracle.compress_48(w_np, od)
    assert np.array_equal(to_host(p), p_ref) and int(n.item()) == n_ref
    assert np.array_equal(bits(to_host(v)), bits(v_ref)) and np.array_equal(to_host(m), m_ref)
    assert np.array_equal(bits(to_host(back)), bits(oracle.decompress_48(v_ref, m_ref, od, (3, 320))))
    assert sp.last_device_error() == sp.OK


def test_empty_and_rejected():
    w = torch.empty((0, 16), dtype=torch.float16, device="cuda")
    p, n = sp.check_48(w)
    assert p.numel() == 0 and int(n.item()) == 0
    with pytest.raises(sp.SP24Error) as e:
        sp.check_48(torch.zeros((2, 12), dtype=torch.float16, device="cuda"))
    assert e.value.status == sp.ERR_SHAPE
    z = torch.zeros((2, 16), dtype=torch.float16, device="cuda")
    v = torch.empty((2, 8), dtype=torch.float16, device="cuda")
    m = torch.empty(2, dtype=torch.uint8, device="cuda")
    L = sp.lib()
    assert L.sp24_prune_compress_48(z.data_ptr(), 7, 2, 16, v.data_ptr(), m.data_ptr(), None) == sp.ERR_DTYPE
    assert L.sp24_prune_compress_48(z.data_ptr(), sp.F16, -1, 16, v.data_ptr(), m.data_ptr(), None) == sp.ERR_SHAPE
    assert L.sp24_prune_compress_48(z.data_ptr() + 1, sp.F16, 2, 16, v.data_ptr(), m.data_ptr(), None) == sp.ERR_ALIGN
    assert L.sp24_decompress_48(v.data_ptr(), None, sp.F16, 2, 16, z.data_ptr(), None) == sp.ERR_INVALID_ARG
    torch.cuda.synchronize()
    assert sp.last_device_error() == sp.OK


@pytest.mark.parametrize("dtype", ["bf16", "f32"])
def test_decompress_flags_illegal_nibble(dtype):
    tdt = torch.bfloat16 if dtype == "bf16" else torch.float32
    v = torch.ones((1, 8), dtype=tdt, device="cuda")
    m = torch.tensor([0x6E], dtype=torch.uint8, device="cuda")  # chunk 0 legal (2, 3), chunk 1 (2, 1) not
    out = sp.decompress_48(v, m, (1, 16))
    assert sp.last_device_error() == sp.ERR_INVALID_ARG
    assert sp.last_device_error() == sp.OK  # cleared
    assert out[0, :8].tolist() == [0, 0, 0, 0, 1, 1, 1, 1] and not out[0, 8:].any()

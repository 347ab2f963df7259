"""GPU parity of a1 (eligibility) and a2 (prune / compress / decompress): bit-exact against the
oracle on the same seeded inputs."""
import numpy as np
import pytest
import torch

import fp16_gemm_b200 as sp
import oracle
import synth
from helpers import ORACLE_DT, bits, to_dev, to_host

pytestmark = pytest.mark.gpu

MM_SHAPES = [(1, 4), (3, 12), (37, 200), (64, 512), (5, 4 * 999), (2, 3, 40)]


def _run_matmul(w_np, dtype):
    od = ORACLE_DT[dtype]
    w = to_dev(w_np, dtype)
    p_ref, n_ref = oracle.check_24(w_np, od)
    v_ref, m_ref = oracle.compress_24(w_np, od)
    pr_ref = oracle.prune_24(w_np, od)
    p, n = sp.check_24(w)
    v, m = sp.prune_compress_24(w)
    back = sp.decompress_24(v, m, w.shape)
    torch.cuda.synchronize()
    assert np.array_equal(to_host(p), p_ref)
    assert int(n.item()) == n_ref
    assert np.array_equal(bits(to_host(v)), bits(v_ref))
    assert np.array_equal(to_host(m), m_ref)
    assert np.array_equal(bits(to_host(back)), bits(pr_ref))
    assert sp.last_device_error() == sp.OK


@pytest.mark.parametrize("dtype", ["f16", "bf16", "f32"])
@pytest.mark.parametrize("shape", MM_SHAPES)
def test_matmul_edge_values(dtype, shape):
    g = synth.rng(100 + len(shape) * 7 + shape[-1])
    rows = int(np.prod(shape[:-1]))
    w = synth.structured_edge(g, rows, shape[-1], dtype).reshape(shape)
    _run_matmul(w, dtype)


@pytest.mark.parametrize("dtype", ["f16", "bf16", "f32"])
def test_matmul_normal_2d(dtype):
    w = synth.draw(synth.rng(1), (256, 512), dtype)
    _run_matmul(w, dtype)


def test_toy_vectors_on_gpu():
    """'Two half-zero vectors produce different pattern answers' through the CUDA path."""
    for vec, want, nfail in (([1, 0, 2, 0, 3, 0, 4, 0], [1, 1], 0), ([1, 2, 3, 0, 4, 0, 0, 0], [0, 1], 1)):
        w = torch.tensor([vec], dtype=torch.float16, device="cuda")
        p, n = sp.check_24(w)
        assert p.cpu().tolist() == [want] and int(n.item()) == nfail


def test_misaligned_views_use_the_generic_path():
    base = synth.structured_edge(synth.rng(3), 1, 4 * 301, "f16")
    w_full = to_dev(base, "f16")
    w = w_full[:, 4:]                     # 8-byte offset: not 16-byte aligned
    assert w.data_ptr() % 16 != 0
    w_np = np.ascontiguousarray(base[:, 4:])
    p, n = sp.check_24(w)
    v, m = sp.prune_compress_24(w)
    p_ref, n_ref = oracle.check_24(w_np, oracle.F16)
    v_ref, m_ref = oracle.compress_24(w_np, oracle.F16)
    assert np.array_equal(to_host(p), p_ref) and int(n.item()) == n_ref
    assert np.array_equal(bits(to_host(v)), bits(v_ref)) and np.array_equal(to_host(m), m_ref)


@pytest.mark.parametrize("dtype", ["f16", "bf16", "f32"])
@pytest.mark.parametrize("shape", [(8, 12, 3, 2), (4, 8, 1, 1), (3, 4, 5, 7), (64, 64, 3, 3), (32, 64, 7, 7)])
def test_conv_layout(dtype, shape):
    K, C, R, S = shape
    od = ORACLE_DT[dtype]
    w_np = synth.structured_edge(synth.rng(K * C + R), K * C, R * S, dtype).reshape(shape)
    w = to_dev(w_np, dtype)
    p, n = sp.check_24(w, sp.OP_CONV)
    v, m = sp.prune_compress_24(w, sp.OP_CONV)
    back = sp.decompress_24(v, m, shape, sp.OP_CONV)
    p_ref, n_ref = oracle.check_24(w_np, od, oracle.CONV)
    v_ref, m_ref = oracle.compress_24(w_np, od, oracle.CONV)
    assert np.array_equal(to_host(p), p_ref) and int(n.item()) == n_ref
    assert np.array_equal(bits(to_host(v)), bits(v_ref)) and np.array_equal(to_host(m), m_ref)
    assert np.array_equal(bits(to_host(back)), bits(oracle.prune_24(w_np, od, oracle.CONV)))


def test_conv_workload_5pct_failing():
    """FP16 conv weights [256, 256, 3, 3] grouped along C with 5% of groups seeded to fail."""
    d = synth.conv_fail5()
    w = to_dev(d["W"], "f16")
    p, n = sp.check_24(w, sp.OP_CONV)
    assert int(n.item()) == len(d["failing"]) == 7373
    assert np.array_equal(np.flatnonzero(to_host(p).ravel() == 0), d["failing"])
    v, m = sp.prune_compress_24(w, sp.OP_CONV)
    v_ref, m_ref = oracle.compress_24(d["W"], oracle.F16, oracle.CONV)
    assert np.array_equal(bits(to_host(v)), bits(v_ref)) and np.array_equal(to_host(m), m_ref)


def test_full_size_decode_weight():
    """The decode workload's weight, bf16 [5120, 5120] N(0, 0.02): every group fails the check
    (no zeros), and pruning/compression match the oracle byte for byte."""
    w_np = synth.decode_nvfp4()["W"]
    w = to_dev(w_np, "bf16")
    p, n = sp.check_24(w)
    assert int(n.item()) == 5120 * 5120 // 4 and int(p.sum().item()) == 0
    v, m = sp.prune_compress_24(w)
    v_ref, m_ref = oracle.compress_24(w_np, oracle.BF16)
    assert np.array_equal(bits(to_host(v)), bits(v_ref)) and np.array_equal(to_host(m), m_ref)
    p2, n2 = sp.check_24(sp.decompress_24(v, m, w.shape))
    assert int(n2.item()) == 0


def test_empty_and_rejected():
    w = torch.empty((0, 8), dtype=torch.float16, device="cuda")
    p, n = sp.check_24(w)
    assert p.numel() == 0 and int(n.item()) == 0
    with pytest.raises(sp.SP24Error):
        sp.check_24(torch.zeros((2, 6, 3, 3), dtype=torch.float16, device="cuda"), sp.OP_CONV)


def test_decompress_flags_illegal_nibble():
    v = torch.zeros((1, 4), dtype=torch.float16, device="cuda")
    m = torch.tensor([0x55], dtype=torch.uint8, device="cuda")  # i0 == i1: illegal
    out = sp.decompress_24(v, m, (1, 8))
    assert sp.last_device_error() == sp.ERR_INVALID_ARG
    assert sp.last_device_error() == sp.OK  # cleared
    assert not out.any()

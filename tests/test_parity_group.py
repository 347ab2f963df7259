"""GPU parity of the group-shared NVFP4 tensor scale ([P5] "The shared global scale") and of
large single-tensor quantisation: scales, codes and block scales bit-exact against the oracle."""
import ctypes

import numpy as np
import pytest
import torch

import fp16_gemm_b200 as sp
import oracle
import synth
from helpers import ORACLE_DT, to_dev, to_host

pytestmark = pytest.mark.gpu


def _bits32(x) -> int:
    return int(np.float32(x).view(np.uint32))


def _group_case(dtype, sizes, seed):
    g = synth.rng(seed)
    out = []
    for rows, cols in sizes:
        sig = float(np.exp(synth.normal(g, ())))
        out.append(synth.draw(g, (rows, cols), dtype, sig))
    return out


@pytest.mark.parametrize("dtype", ["f16", "bf16", "f32"])
@pytest.mark.parametrize("sizes", [[(4, 64)], [(64, 512), (3, 16)], [(128, 256), (0, 16), (7, 48), (1, 16)]],
                         ids=["one", "two", "with-empty"])
def test_group_scale_bit_exact(dtype, sizes):
    ts_np = _group_case(dtype, sizes, 100 + len(sizes))
    ref = oracle.nvfp4_group_tensor_scale(ts_np, ORACLE_DT[dtype])
    got = sp.nvfp4_group_tensor_scale([to_dev(t, dtype) for t in ts_np])
    torch.cuda.synchronize()
    assert _bits32(got.item()) == _bits32(ref)


def test_group_scale_many_tensors():
    """35 tensors (three launches of up to 16), sizes from empty to 8 KB, the largest magnitude
    in the last launch."""
    g = synth.rng(103)
    ts_np = [synth.draw(g, (int(g.integers(0, 5)), 16 * int(g.integers(1, 9))), "bf16", 0.5) for _ in range(35)]
    ts_np[33] = ts_np[33].copy()
    if ts_np[33].size:
        ts_np[33].flat[0] = synth.as_storage(np.array([-77.0]), "bf16")[0]
    ref = oracle.nvfp4_group_tensor_scale(ts_np, oracle.BF16)
    got = sp.nvfp4_group_tensor_scale([to_dev(t, "bf16") for t in ts_np])
    torch.cuda.synchronize()
    assert _bits32(got.item()) == _bits32(ref)


def test_group_scale_nan_and_inf():
    x = synth.normal(synth.rng(104), (8, 64)).astype(np.float32)
    y = x.copy()
    y[3, 5] = np.nan
    got = sp.nvfp4_group_tensor_scale([to_dev(y, "f32"), to_dev(x[:2].copy(), "f32")])
    torch.cuda.synchronize()
    assert _bits32(got.item()) == _bits32(oracle.nvfp4_group_tensor_scale([y, x[:2]], oracle.F32))
    y[0, 0] = np.inf
    got = sp.nvfp4_group_tensor_scale([to_dev(y, "f32")])
    torch.cuda.synchronize()
    assert np.isinf(got.item())


@pytest.mark.parametrize("dtype", ["bf16", "f16"])
def test_qkv_group_quantised_with_shared_scale(dtype):
    """Wq, Wk, Wv share one scale (an outlier in Wv sets it); each quantised with it matches the
    oracle's encode under the same scale, codes and block scales byte for byte."""
    d = synth.qkv_group(seed=105, dtype=dtype)
    mats = [d["Wq"], d["Wk"], d["Wv"]]
    od = ORACLE_DT[dtype]
    ts_ref = oracle.nvfp4_group_tensor_scale(mats, od)
    assert ts_ref > max(oracle.nvfp4_tensor_scale(m, od) for m in mats[:2])
    devs = [to_dev(m, dtype) for m in mats]
    ts = sp.nvfp4_group_tensor_scale(devs)
    for m, t in zip(mats, devs):
        q = sp.quantize_nvfp4(t, tensor_scale=ts)
        torch.cuda.synchronize()
        c_ref, s_ref, ts_used = oracle.nvfp4_encode(m, od, ts_ref)
        assert _bits32(q.tensor_scale.item()) == _bits32(ts_used) == _bits32(ts.item())
        assert np.array_equal(to_host(q.scales), s_ref)
        assert np.array_equal(to_host(q.codes), c_ref)


def test_group_scale_rejects():
    t = torch.zeros(32, dtype=torch.bfloat16, device="cuda")
    ws = torch.empty(16, dtype=torch.uint8, device="cuda")
    out = torch.empty(1, dtype=torch.float32, device="cuda")

    def call(ptrs, numels, dtype=sp.BF16, wsb=16, wsp=None):
        n = len(ptrs)
        P = (ctypes.c_void_p * max(n, 1))(*ptrs)
        N = (ctypes.c_int64 * max(n, 1))(*numels)
        return sp.lib().sp24_nvfp4_group_tensor_scale(P, N, n, dtype, ctypes.c_void_p(out.data_ptr()),
                                                      ctypes.c_void_p(ws.data_ptr() if wsp is None else wsp),
                                                      wsb, None)

    assert call([t.data_ptr()], [32]) == sp.OK
    assert call([t.data_ptr() + 2], [16]) == sp.ERR_ALIGN          # not 16-byte aligned
    assert call([t.data_ptr()], [12]) == sp.ERR_SHAPE              # 24 bytes
    assert call([t.data_ptr()], [-16]) == sp.ERR_SHAPE
    assert call([t.data_ptr()], [32], dtype=sp.NVFP4) == sp.ERR_DTYPE
    assert call([t.data_ptr()], [32], wsb=8) == sp.ERR_WORKSPACE
    assert call([0], [0]) == sp.OK                                  # an empty member needs no pointer
    torch.cuda.synchronize()
    assert sp.last_device_error() == sp.OK


def test_output_head_quantisation_sampled():
    """The pages' large single-tensor case: a [151936, 4096] bf16 output head (~1.16 GiB) in
    one call.  The tensor scale (amax over all 622M entries) is bit-exact; codes and block
    scales of 48 sampled rows (first, last, and seeded ones) match the oracle byte for byte."""
    W = synth.output_head()["W"]
    ts_ref = oracle.nvfp4_tensor_scale(W, oracle.BF16)
    t = to_dev(W, "bf16")
    q = sp.quantize_nvfp4(t)
    torch.cuda.synchronize()
    assert _bits32(q.tensor_scale.item()) == _bits32(ts_ref)
    rows = np.unique(np.concatenate([[0, W.shape[0] - 1], synth.rng(106).choice(W.shape[0], 46, replace=False)]))
    c_ref, s_ref, _ = oracle.nvfp4_encode(np.ascontiguousarray(W[rows]), oracle.BF16, ts_ref)
    idx = torch.as_tensor(rows, device="cuda")
    assert np.array_equal(to_host(q.scales[idx]), s_ref)
    assert np.array_equal(to_host(q.codes[idx]), c_ref)
    assert sp.last_device_error() == sp.OK

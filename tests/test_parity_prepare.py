"""GPU parity of the fused weight preparation (rows a1-a3 with one read of W): pass map, fail
count, kept values, nibbles and both NVFP4 tensor scales bit-exact against the oracle; the NVFP4
encodings made with those scales equal the oracle's unscaled encodings; everything equals the
separate entry points on the decode weight."""
import numpy as np
import pytest
import torch

import fp16_gemm_b200 as sp
import oracle
import synth
from helpers import ORACLE_DT, bits, to_dev, to_host

pytestmark = pytest.mark.gpu


def _f32_bits(x) -> int:
    return int(np.float32(x).view(np.uint32))


def _same_nvfp4(q, ref, what):
    c_ref, s_ref, ts_ref = ref
    assert _f32_bits(q.tensor_scale.item()) == _f32_bits(ts_ref), what
    bad_s = np.argwhere(to_host(q.scales) != s_ref)
    assert bad_s.size == 0, f"{what}: {len(bad_s)} scale mismatches, first {bad_s[:3].tolist()}"
    bad_c = np.argwhere(to_host(q.codes) != c_ref)
    assert bad_c.size == 0, f"{what}: {len(bad_c)} code mismatches, first {bad_c[:3].tolist()}"


def _run(w_np, dtype, nvfp4=True):
    od = ORACLE_DT[dtype]
    p_ref, n_ref = oracle.check_24(w_np, od)
    v_ref, m_ref = oracle.compress_24(w_np, od)
    w = to_dev(w_np, dtype)
    r = sp.prepare_24(w)
    torch.cuda.synchronize()
    assert np.array_equal(to_host(r.pass_map), p_ref)
    assert int(r.n_fail.item()) == n_ref
    assert np.array_equal(bits(to_host(r.values)), bits(v_ref))
    assert np.array_equal(to_host(r.meta).reshape(-1), m_ref.reshape(-1))
    assert _f32_bits(r.w_tensor_scale.item()) == _f32_bits(oracle.nvfp4_tensor_scale(w_np, od))
    assert _f32_bits(r.v_tensor_scale.item()) == _f32_bits(oracle.nvfp4_tensor_scale(v_ref, od))
    if nvfp4 and w_np.shape[1] % 32 == 0:
        _same_nvfp4(sp.quantize_nvfp4(w, tensor_scale=r.w_tensor_scale), oracle.nvfp4_encode(w_np, od), "W")
        _same_nvfp4(sp.quantize_nvfp4(r.values, tensor_scale=r.v_tensor_scale),
                    oracle.nvfp4_encode(v_ref, od), "values")
    return w, r


@pytest.mark.parametrize("dtype", ["f16", "bf16", "f32"])
@pytest.mark.parametrize("shape", [(1, 16), (7, 96), (64, 512), (129, 1056)])
def test_edge_values(dtype, shape):
    """Zeros of both signs, ties of mixed sign and small integers, from one vector up to several
    ring chunks with a ragged last chunk (129 x 1056)."""
    g = synth.rng(shape[0] * 7 + shape[1])
    _run(synth.structured_edge(g, shape[0], shape[1], dtype), dtype)


@pytest.mark.parametrize("dtype", ["f16", "bf16", "f32"])
def test_rows_of_varied_scale(dtype):
    """Row magnitudes spread over e^(+-6): subnormal E4M3 block scales in both encodings."""
    g = synth.rng(11)
    x = synth.normal(g, (96, 640)) * np.exp(2 * synth.normal(g, (96, 1)))
    _run(synth.as_storage(x, dtype), dtype)


def test_matches_separate_entry_points_on_decode_weight():
    """bf16 [5120, 5120] N(0, 0.02): the fused path equals check_24, prune_compress_24 and two
    unscaled quantize_nvfp4 calls byte for byte (and the oracle, checked in _run)."""
    w_np = synth.decode_nvfp4()["W"]
    w, _ = _run(w_np, "bf16")
    r, wq, sw = sp.prepare_nvfp4_24(w)
    p, n = sp.check_24(w)
    v, m = sp.prune_compress_24(w)
    qw = sp.quantize_nvfp4(w)
    qv = sp.quantize_nvfp4(v)
    torch.cuda.synchronize()
    assert torch.equal(p.view(r.pass_map.shape), r.pass_map)
    assert torch.equal(n, r.n_fail)
    assert torch.equal(v.view(torch.int16), r.values.view(torch.int16))
    assert torch.equal(m.view(-1), r.meta.view(-1))
    for a, b in ((qw, wq), (qv, sw.values)):
        assert torch.equal(a.codes, b.codes) and torch.equal(a.scales, b.scales)
        assert torch.equal(a.tensor_scale, b.tensor_scale)


def test_repeated_calls_reuse_the_workspace():
    """The scratch words are cleared by every call: a second call on another weight with the
    same workspace gives that weight's own counts and scales."""
    ws = torch.empty(sp.prepare_workspace_bytes(32, 256), dtype=torch.uint8, device="cuda")
    for seed in (21, 22, 23):
        w_np = synth.structured_edge(synth.rng(seed), 32, 256, "f16")
        w_np = (w_np.astype(np.float64) * (seed - 20)).astype(np.float16)
        r = sp.prepare_24(to_dev(w_np, "f16"), workspace=ws)
        torch.cuda.synchronize()
        assert int(r.n_fail.item()) == oracle.check_24(w_np, oracle.F16)[1]
        assert _f32_bits(r.w_tensor_scale.item()) == _f32_bits(oracle.nvfp4_tensor_scale(w_np, oracle.F16))


def test_without_pass_map_and_empty():
    w_np = synth.structured_edge(synth.rng(13), 16, 128, "bf16")
    w = to_dev(w_np, "bf16")
    r = sp.prepare_24(w, with_pass=False)
    torch.cuda.synchronize()
    assert r.pass_map is None
    assert int(r.n_fail.item()) == oracle.check_24(w_np, oracle.BF16)[1]
    e = sp.prepare_24(torch.empty((0, 64), dtype=torch.bfloat16, device="cuda"))
    torch.cuda.synchronize()
    assert int(e.n_fail.item()) == 0
    assert e.w_tensor_scale.item() == 0.0 and e.v_tensor_scale.item() == 0.0


def test_rejected_arguments():
    with pytest.raises(sp.SP24Error) as e:
        sp.prepare_24(torch.zeros((4, 40), dtype=torch.bfloat16, device="cuda"))   # K % 16
    assert e.value.status == sp.ERR_SHAPE
    buf = torch.zeros(4 * 64 + 8, dtype=torch.bfloat16, device="cuda")
    with pytest.raises(sp.SP24Error) as e:
        sp.prepare_24(buf[1:1 + 4 * 64].view(4, 64))                                # W misaligned
    assert e.value.status == sp.ERR_ALIGN


@pytest.mark.parametrize("dtype", ["f16", "bf16", "f32"])
def test_quantize_pair_matches_two_calls_and_oracle(dtype):
    """One launch encoding two tensors with supplied scales equals two quantize_nvfp4 calls with
    the same scales, and the oracle's encodings with those scales; an empty second tensor still
    gets its tensor scale copied."""
    od = ORACLE_DT[dtype]
    g = synth.rng(31)
    a_np = synth.as_storage(synth.normal(g, (70, 320)) * np.exp(synth.normal(g, (70, 1))), dtype)
    b_np = synth.structured_edge(g, 33, 160, dtype)
    ts_a = oracle.nvfp4_tensor_scale(a_np, od)
    ts_b = oracle.nvfp4_tensor_scale(b_np, od) * 2.0  # a shared, larger scale
    a, b = to_dev(a_np, dtype), to_dev(b_np, dtype)
    ta = torch.tensor([ts_a], dtype=torch.float32, device="cuda")
    tb = torch.tensor([ts_b], dtype=torch.float32, device="cuda")
    qa, qb = sp.quantize_nvfp4_pair(a, ta, b, tb)
    ra, rb = sp.quantize_nvfp4(a, tensor_scale=ta), sp.quantize_nvfp4(b, tensor_scale=tb)
    torch.cuda.synchronize()
    for q, r in ((qa, ra), (qb, rb)):
        assert torch.equal(q.codes, r.codes) and torch.equal(q.scales, r.scales)
        assert torch.equal(q.tensor_scale, r.tensor_scale)
    _same_nvfp4(qa, oracle.nvfp4_encode(a_np, od, ts_a), "first")
    _same_nvfp4(qb, oracle.nvfp4_encode(b_np, od, float(np.float32(ts_b))), "second")
    e = torch.empty((0, 32), dtype=a.dtype, device="cuda")
    qa2, qe = sp.quantize_nvfp4_pair(a, ta, e, tb)
    torch.cuda.synchronize()
    assert torch.equal(qa2.codes, ra.codes) and qe.codes.numel() == 0
    assert qe.tensor_scale.item() == tb.item()

"""GPU parity of the routed expert block (gate/up with SwiGLU, down, router-weighted combine)
against the oracle on the same seeded inputs: NVFP4 experts dense or 2:4, bf16 / f16 tokens."""
import numpy as np
import pytest
import torch

import fp16_gemm_b200 as sp
import oracle
import synth
from helpers import assert_gemm_close, to_dev

pytestmark = pytest.mark.gpu


def _sparse_decoded(W_e, ts):
    """Dense-equivalent fp64 of a pruned, compressed, NVFP4-quantised [N, K] weight."""
    V, meta = oracle.compress_24(W_e, oracle.BF16)
    c, s, _ = oracle.nvfp4_encode(V, oracle.BF16, ts)
    Vd = oracle.nvfp4_decode(c, s, ts)
    N, K = W_e.shape
    nib = np.stack([meta & 0xF, meta >> 4], 1).ravel()[: N * K // 4].reshape(N, K // 4)
    Wd = np.zeros((N, K))
    rows = np.arange(N)[:, None]
    j = np.arange(K // 4)[None, :]
    Wd[rows, 4 * j + (nib & 3)] = Vd[:, 0::2]
    Wd[rows, 4 * j + (nib >> 2)] = Vd[:, 1::2]
    return Wd


def _dense_decoded(W_e, ts):
    c, s, _ = oracle.nvfp4_encode(W_e, oracle.BF16, ts)
    return oracle.nvfp4_decode(c, s, ts)


def _values(W, E):
    """The kept values of every expert of a stacked weight (for the shared tensor scales)."""
    return [oracle.compress_24(np.ascontiguousarray(W[e]), oracle.BF16)[0] for e in range(E)]


def _device_ops(d, sparse_gu, sparse_dn):
    E, F, H = d["Wg"].shape
    wg = to_dev(d["Wg"].reshape(E * F, H), "bf16")
    wu = to_dev(d["Wu"].reshape(E * F, H), "bf16")
    wd = to_dev(d["Wd"].reshape(E * H, F), "bf16")
    if sparse_gu:
        (vg, mg), (vu, mu) = sp.prune_compress_24(wg), sp.prune_compress_24(wu)
        ts = sp.nvfp4_group_tensor_scale([vg, vu])
        gu = sp.pack_gate_up(sp.Sparse24(sp.quantize_nvfp4(vg, ts), mg), sp.Sparse24(sp.quantize_nvfp4(vu, ts), mu))
    else:
        ts = sp.nvfp4_group_tensor_scale([wg, wu])
        gu = sp.pack_gate_up(sp.quantize_nvfp4(wg, ts), sp.quantize_nvfp4(wu, ts))
    if sparse_dn:
        v, m = sp.prune_compress_24(wd)
        dn = sp.Sparse24(sp.quantize_nvfp4(v), m)
    else:
        dn = sp.quantize_nvfp4(wd)
    return gu, dn


def _oracle(d, sparse_gu, sparse_dn, xfmt, tokens):
    E, F, H = d["Wg"].shape
    Wg, Wu, Wd = d["Wg"], d["Wu"], d["Wd"]
    if sparse_gu:
        ts_gu = oracle.nvfp4_group_tensor_scale(_values(Wg, E) + _values(Wu, E), oracle.BF16)
    else:
        ts_gu = oracle.nvfp4_group_tensor_scale([Wg, Wu], oracle.BF16)
    ts_dn = oracle.nvfp4_group_tensor_scale(_values(Wd, E) if sparse_dn else [Wd], oracle.BF16)
    used = sorted(set(d["routing"][tokens].ravel().tolist()))
    dec_gu = _sparse_decoded if sparse_gu else _dense_decoded
    dec_dn = _sparse_decoded if sparse_dn else _dense_decoded
    Gd = np.stack([dec_gu(np.ascontiguousarray(Wg[e]), ts_gu) for e in used])
    Ud = np.stack([dec_gu(np.ascontiguousarray(Wu[e]), ts_gu) for e in used])
    Dd = np.stack([dec_dn(np.ascontiguousarray(Wd[e]), ts_dn) for e in used])
    remap = {e: i for i, e in enumerate(used)}
    rsub = np.vectorize(remap.get)(d["routing"][tokens]).astype(np.int32)
    Xs = np.ascontiguousarray(d["X"][tokens])
    if xfmt == "f16":
        Xd = oracle.to_double(synth.bf16_bits_to_f32(Xs).astype(np.float16), oracle.F16)
    else:
        Xd = oracle.to_double(Xs, oracle.BF16)
    hdt = oracle.F16 if xfmt == "f16" else oracle.BF16
    return oracle.moe_block(Xd, rsub, d["router_w"][tokens].astype(np.float64), Gd, Ud, Dd, hdt)


def _run(d, sparse_gu, sparse_dn, xfmt, tokens):
    E, F, H = d["Wg"].shape
    gu, dn = _device_ops(d, sparse_gu, sparse_dn)
    X = d["X"] if xfmt == "bf16" else synth.bf16_bits_to_f32(d["X"]).astype(np.float16)
    x = to_dev(X, xfmt)
    r = torch.from_numpy(d["routing"]).cuda()
    rw = torch.from_numpy(d["router_w"]).cuda()
    y = sp.moe_block(x, r, rw, gu, dn, E, H, F)
    torch.cuda.synchronize()
    assert sp.last_device_error() == sp.OK
    Y, S = _oracle(d, sparse_gu, sparse_dn, xfmt, tokens)
    assert_gemm_close(y[torch.as_tensor(tokens, device=y.device)], Y, S)


@pytest.mark.parametrize("forms", [(False, False), (True, True), (False, True), (True, False)],
                         ids=["dense", "sparse24", "dense-gu_sparse-down", "sparse-gu_dense-down"])
@pytest.mark.parametrize("xfmt", ["bf16", "f16"])
def test_block_small(forms, xfmt):
    """4 experts, H = F = 512, 300 tokens top-2 (about 150 routed rows per expert: two token
    tiles each), every output checked."""
    d = synth.moe_block(seed=31, E=4, H=512, F=512, T=300, topk=2)
    _run(d, forms[0], forms[1], xfmt, np.arange(300))


@pytest.mark.parametrize("forms", [(False, False), (True, True)], ids=["dense", "sparse24"])
def test_block_model_widths(forms):
    """32 experts of the workload's widths (H = 2048, F = 512), 256 tokens top-8, every output."""
    d = synth.moe_block(seed=32, E=32, H=2048, F=512, T=256, topk=8)
    _run(d, forms[0], forms[1], "bf16", np.arange(256))


def test_block_rejects():
    d = synth.moe_block(seed=33, E=2, H=512, F=512, T=8, topk=1)
    gu, dn = _device_ops(d, False, False)
    x = to_dev(d["X"], "bf16")
    r = torch.from_numpy(d["routing"]).cuda()
    rw = torch.from_numpy(d["router_w"]).cuda()
    with pytest.raises(sp.SP24Error) as e:
        sp.moe_block(x, r, rw, gu, dn, 2, 512, 448)  # F % 64 but down K % 256 fails
    assert e.value.status in (sp.ERR_UNSUPPORTED, sp.ERR_SHAPE)
    with pytest.raises(sp.SP24Error) as e:
        sp.moe_block(x.float(), r, rw, gu, dn, 2, 512, 512)
    assert e.value.status == sp.ERR_DTYPE

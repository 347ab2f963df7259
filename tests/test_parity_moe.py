"""GPU parity of the routed-expert grouped GEMM (dense and 2:4) against the oracle."""
import numpy as np
import pytest
import torch

import fp16_gemm_b200 as sp
import oracle
import synth
from helpers import assert_gemm_close, to_dev

pytestmark = pytest.mark.gpu


def _expert_dense_decoded(W_e, wfmt, ts):
    if wfmt == "nvfp4":
        c, s, _ = oracle.nvfp4_encode(W_e, oracle.BF16, ts)
        return oracle.nvfp4_decode(c, s, ts)
    return oracle.to_double(W_e, oracle.BF16)


def _expert_sparse_decoded(W_e, wfmt, ts):
    """Dense-equivalent fp64 of a pruned, compressed (and NVFP4-quantised) expert."""
    V, meta = oracle.compress_24(W_e, oracle.BF16)
    if wfmt == "nvfp4":
        c, s, _ = oracle.nvfp4_encode(V, oracle.BF16, ts)
        Vd = oracle.nvfp4_decode(c, s, ts)
    else:
        Vd = oracle.to_double(V, oracle.BF16)
    N, K = W_e.shape
    nib = np.stack([meta & 0xF, meta >> 4], 1).ravel()[: N * K // 4].reshape(N, K // 4)
    Wd = np.zeros((N, K))
    rows = np.arange(N)[:, None]
    j = np.arange(K // 4)[None, :]
    Wd[rows, 4 * j + (nib & 3)] = Vd[:, 0::2]
    Wd[rows, 4 * j + (nib >> 2)] = Vd[:, 1::2]
    return Wd


def _run(X, W, routing, xfmt, wfmt, sparse, tokens):
    E, N, K = W.shape
    x = to_dev(X, "f16" if xfmt == "f16" else "bf16")
    if xfmt == "nvfp4":
        x = sp.quantize_nvfp4(x)
    w = to_dev(W.reshape(E * N, K), "bf16")
    if sparse:
        v, m = sp.prune_compress_24(w)
        if wfmt == "nvfp4":
            v = sp.quantize_nvfp4(v)
        wop = sp.Sparse24(v, m)
    else:
        wop = sp.quantize_nvfp4(w) if wfmt == "nvfp4" else w
    # the oracle's own shared tensor scale of the stacked experts (for 2:4 values it is the
    # same number: the largest |w| of every group is kept, see test_amax_survives_pruning)
    ts = oracle.nvfp4_tensor_scale(np.ascontiguousarray(W.reshape(E * N, K)), oracle.BF16) \
        if wfmt == "nvfp4" else None
    r = torch.from_numpy(routing).cuda()
    y = sp.gemm_grouped(x, r, wop, E, N, K)
    torch.cuda.synchronize()
    assert sp.last_device_error() == sp.OK
    # oracle on the sampled tokens (the NVFP4 tensor scale is shared by the stacked experts)
    if xfmt == "nvfp4":
        c, s, xts = oracle.nvfp4_encode(X, oracle.BF16)
        Xd = oracle.nvfp4_decode(c[tokens], s[tokens], xts)
    else:
        Xd = oracle.to_double(np.ascontiguousarray(X[tokens]), oracle.F16 if xfmt == "f16" else oracle.BF16)
    used = sorted(set(routing[tokens].ravel().tolist()))
    dec = {e: (_expert_sparse_decoded if sparse else _expert_dense_decoded)(np.ascontiguousarray(W[e]), wfmt, ts)
           for e in used}
    Wd = np.stack([dec[e] for e in used])
    remap = {e: i for i, e in enumerate(used)}
    rsub = np.vectorize(remap.get)(routing[tokens]).astype(np.int32)
    Y, S = oracle.moe(Xd, rsub, Wd)
    assert_gemm_close(y[torch.as_tensor(tokens, device=y.device)], Y, S)


@pytest.mark.parametrize("sparse", [False, True], ids=["dense", "sparse24"])
@pytest.mark.parametrize("fmt", [("bf16", "bf16"), ("bf16", "nvfp4"), ("nvfp4", "nvfp4")],
                         ids=lambda f: f"x{f[0]}-w{f[1]}")
def test_moe_small(fmt, sparse):
    """8 experts [64, 512], 150 tokens routed top-3 (some experts get > 64 tokens: several
    token tiles), every output checked."""
    d = synth.moe(seed=3, E=8, N=64, K=512, T=150, topk=3)
    _run(d["X"], d["W"], d["routing"], fmt[0], fmt[1], sparse, np.arange(150))


@pytest.mark.parametrize("sparse", [False, True], ids=["dense", "sparse24"])
def test_moe_workload_sampled(sparse):
    """512 experts of NVFP4 [512, 2048], 4096 bf16 tokens routed top-10: 6 sampled tokens (60
    routed rows x 512 outputs) checked against the oracle."""
    d = synth.moe()
    tokens = np.sort(synth.rng(99).choice(4096, 6, replace=False))
    _run(d["X"], d["W"], d["routing"], "bf16", "nvfp4", sparse, tokens)


def test_moe_rejects_bad_expert_ids():
    d = synth.moe(seed=4, E=4, N=64, K=512, T=16, topk=2)
    x = to_dev(d["X"], "bf16")
    w = to_dev(d["W"].reshape(4 * 64, 512), "bf16")
    r = torch.from_numpy(d["routing"]).cuda()
    r[0, 0] = 7
    y = sp.gemm_grouped(x, r, w, 4, 64, 512)
    assert sp.last_device_error() == sp.ERR_INVALID_ARG
    assert not y[0, 0].any()


# Per-expert routed-row counts around the 128-row token tiles and the 16-row MMA granularity of
# the tensor-core path (NVFP4 experts, 16-bit tokens, N % 128, K % 256): an expert spanning three
# tiles (128, 128, 44), tiles of 1, 15, 16, 17, 127, 128 and 129 rows, and experts with none.
SKEW = [300, 1, 0, 15, 16, 17, 127, 0, 128, 129, 1]


@pytest.mark.parametrize("xfmt", ["bf16", "f16"])
@pytest.mark.parametrize("NK", [(256, 512), (128, 256), (384, 768), (128, 2304)],
                         ids=lambda s: f"N{s[0]}-K{s[1]}")
def test_moe_tile_boundaries(NK, xfmt):
    """Every output of skewed routings: 128-row tiles at their edges, K of 1, 2, 3 and 9
    weight boxes of 256 (the last wraps the four-box ring twice), one to three weight-row
    blocks of 128, bf16 and f16 tokens."""
    N, K = NK
    d = synth.moe_skewed(SKEW, seed=11, N=N, K=K, topk=2, xdtype=xfmt)
    T = d["X"].shape[0]
    _run(d["X"], d["W"], d["routing"], xfmt, "nvfp4", False, np.arange(T))


def test_moe_single_routed_row():
    """One token, one expert of eight: a single 16-wide MMA tile with 15 zero-filled rows."""
    d = synth.moe_skewed([0, 0, 0, 1, 0, 0, 0, 0], seed=12, N=128, K=256, topk=1)
    _run(d["X"], d["W"], d["routing"], "bf16", "nvfp4", False, np.arange(1))


def test_moe_bad_expert_ids_tensor_core_path():
    """Invalid ids on the tensor-core path (no output memset there): error word set and the
    invalid rows' outputs zero, the valid rows still right."""
    d = synth.moe_skewed([40, 40, 48], seed=13, N=128, K=256, topk=2)
    X, W, routing = d["X"], d["W"], d["routing"].copy()
    E, N, K = W.shape
    x = to_dev(X, "bf16")
    w = sp.quantize_nvfp4(to_dev(W.reshape(E * N, K), "bf16"))
    bad = routing.copy()
    bad[0, 1] = E
    bad[5, 0] = -1
    r = torch.from_numpy(bad).cuda()
    y = torch.full((X.shape[0], 2, N), float("nan"), device="cuda")
    sp.gemm_grouped(x, r, w, E, N, K, out=y)
    torch.cuda.synchronize()
    assert sp.last_device_error() == sp.ERR_INVALID_ARG
    assert not y[0, 1].any() and not y[5, 0].any()
    assert torch.isfinite(y).all()


@pytest.mark.parametrize("xfmt", ["bf16", "f16"])
@pytest.mark.parametrize("NK", [(256, 512), (128, 1024), (384, 2560)], ids=lambda s: f"N{s[0]}-K{s[1]}")
def test_moe_tile_boundaries_sparse24(NK, xfmt):
    """2:4-compressed NVFP4 experts on the tensor-core path (tcgen05.mma.sp, metadata regrouped
    in registers): the same skewed routings, K of 1, 2 and 5 weight boxes of 512 (the last
    wraps the two-box ring twice), every output checked."""
    N, K = NK
    d = synth.moe_skewed(SKEW, seed=21, N=N, K=K, topk=2, xdtype=xfmt)
    T = d["X"].shape[0]
    _run(d["X"], d["W"], d["routing"], xfmt, "nvfp4", True, np.arange(T))

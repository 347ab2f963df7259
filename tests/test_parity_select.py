"""GPU: the per-shape dense / 2:4 choice measures both GEMMs, records the faster, and the GEMM
it then runs matches the oracle for the form it used."""
import numpy as np
import pytest
import torch

import fp16_gemm_b200 as sp
import oracle
import synth
from helpers import assert_gemm_close, to_dev

pytestmark = pytest.mark.gpu


def _forms(M, N, K, wfmt, seed):
    g = synth.rng(seed)
    X = synth.draw(g, (M, K), "bf16")
    W = synth.draw(g, (N, K), "bf16", 0.02)
    w = to_dev(W, "bf16")
    v, m = sp.prune_compress_24(w)
    wd = sp.decompress_24(v, m, (N, K))  # the pruned weight, dense
    if wfmt == "nvfp4":
        return X, W, sp.quantize_nvfp4(wd), sp.Sparse24(sp.quantize_nvfp4(v), m)
    return X, W, wd, sp.Sparse24(v, m)


def _oracle(X, W, wfmt, used_sparse):
    V, meta = oracle.compress_24(W, oracle.BF16)
    if wfmt == "nvfp4":
        if used_sparse:
            c, s, ts = oracle.nvfp4_encode(V, oracle.BF16)
            Vd = oracle.nvfp4_decode(c, s, ts)
            return oracle.gemm_sparse(oracle.to_double(X, oracle.BF16), Vd, meta)
        Wp = oracle.decompress_24(V, meta, oracle.BF16, W.shape)
        c, s, ts = oracle.nvfp4_encode(Wp, oracle.BF16)
        return oracle.gemm(oracle.to_double(X, oracle.BF16), oracle.nvfp4_decode(c, s, ts))
    return oracle.gemm(oracle.to_double(X, oracle.BF16),
                       oracle.to_double(oracle.decompress_24(V, meta, oracle.BF16, W.shape), oracle.BF16))


@pytest.mark.parametrize("wfmt", ["bf16", "nvfp4"])
@pytest.mark.parametrize("M", [8, 256])
def test_select_records_the_faster_and_auto_matches_oracle(wfmt, M):
    N, K = 1024, 2048
    X, W, wd, ws = _forms(M, N, K, wfmt, 200 + M)
    x = to_dev(X, "bf16")
    sp.gemm_choice_reset()
    r = sp.gemm_select(x, wd, ws, reps=5)
    assert r["us_dense"] > 0 and r["us_sparse"] > 0
    assert r["use_sparse"] == (r["us_sparse"] < r["us_dense"])
    wf = sp.NVFP4 if wfmt == "nvfp4" else sp.BF16
    assert sp.gemm_choice(sp.BF16, wf, M, N, K) == (r["use_sparse"], True)
    y, used = sp.gemm_auto(x, wd, ws)
    torch.cuda.synchronize()
    assert used == r["use_sparse"] and sp.last_device_error() == sp.OK
    Y, S = _oracle(X, W, wfmt, used)
    assert_gemm_close(y, Y, S)
    sp.gemm_choice_reset()
    assert sp.gemm_choice(sp.BF16, wf, M, N, K)[1] is False


@pytest.mark.parametrize("M,expect", [(16, False), (128, True)])
def test_auto_without_record_follows_the_rule(M, expect):
    N, K = 1024, 1024
    X, W, wd, ws = _forms(M, N, K, "nvfp4", 210)
    sp.gemm_choice_reset()
    y, used = sp.gemm_auto(to_dev(X, "bf16"), wd, ws)
    torch.cuda.synchronize()
    assert used is expect  # NVFP4 weights with 16-bit x: dense below M = 128, 2:4 from it
    Y, S = _oracle(X, W, "nvfp4", expect)
    assert_gemm_close(y, Y, S)

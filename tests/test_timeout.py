"""The bounded-wait unwind on the GPU, made to happen without a fault: a self-test kernel waits on
an mbarrier phase that nothing completes, under a 1 ms limit.  The wait must run out, the kernel
must record SP24_ERR_DEVICE_TIMEOUT, let its bulk copy land, free its tensor memory and return;
the context must stay usable (tensor-core GEMMs that allocate TMEM still match the oracle)."""
import ctypes

import numpy as np
import pytest
import torch

import fp16_gemm_b200 as sp
import oracle
import synth
from helpers import assert_gemm_close, to_dev

pytestmark = pytest.mark.gpu


def _stream():
    return ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)


def test_wait_runs_out_sets_timeout_and_unwinds():
    L = sp.lib()
    old = ctypes.c_ulonglong(0)
    assert L.sp24_get_wait_limit(ctypes.byref(old)) == sp.OK
    assert old.value == 2_000_000_000
    src = torch.arange(1024, dtype=torch.int32, device="cuda").to(torch.uint8)  # last byte 255
    out = torch.zeros(2, dtype=torch.int32, device="cuda")
    assert sp.last_device_error() == sp.OK
    try:
        assert L.sp24_set_wait_limit(1_000_000) == sp.OK  # 1 ms
        ev0, ev1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        ev0.record()
        assert L.sp24_selftest_wait_timeout(ctypes.c_void_p(src.data_ptr()), ctypes.c_void_p(out.data_ptr()),
                                            _stream()) == sp.OK
        ev1.record()
        assert sp.last_device_error() == sp.ERR_DEVICE_TIMEOUT
        ms = ev0.elapsed_time(ev1)
    finally:
        assert L.sp24_set_wait_limit(old.value) == sp.OK
    assert out.tolist() == [2, 256]          # the wait ran out; the copy in flight landed
    assert 0.9 <= ms < 1000.0                # about one limit, far below the default 2 s
    assert sp.last_device_error() == sp.OK   # reading the word cleared it


@pytest.mark.parametrize("shape", [(300, 520, 768), (256, 384, 1024)], ids=lambda s: "x".join(map(str, s)))
def test_tensor_core_gemms_after_a_timeout(shape):
    """After the unwind, the W4A4 pair kernel (cta_group::2 TMEM) and the 16-bit tcgen05 GEMM
    still allocate their tensor memory and match the oracle."""
    L = sp.lib()
    src = torch.zeros(1024, dtype=torch.uint8, device="cuda")
    out = torch.zeros(2, dtype=torch.int32, device="cuda")
    try:
        assert L.sp24_set_wait_limit(1_000_000) == sp.OK
        assert L.sp24_selftest_wait_timeout(ctypes.c_void_p(src.data_ptr()), ctypes.c_void_p(out.data_ptr()),
                                            _stream()) == sp.OK
        assert sp.last_device_error() == sp.ERR_DEVICE_TIMEOUT
    finally:
        L.sp24_set_wait_limit(2_000_000_000)
    M, N, K = shape
    g = synth.rng(M + N + K)
    X, W = synth.draw(g, (M, K), "bf16"), synth.draw(g, (N, K), "bf16")
    cx, sx, tx = oracle.nvfp4_encode(X, oracle.BF16)
    cw, sw, tw = oracle.nvfp4_encode(W, oracle.BF16)
    Y, S = oracle.gemm(oracle.nvfp4_decode(cx, sx, tx), oracle.nvfp4_decode(cw, sw, tw))
    y = sp.gemm_dense(sp.quantize_nvfp4(to_dev(X, "bf16")), sp.quantize_nvfp4(to_dev(W, "bf16")))
    torch.cuda.synchronize()
    assert_gemm_close(y, Y, S)
    Yb, Sb = oracle.gemm(oracle.to_double(X, oracle.BF16), oracle.to_double(W, oracle.BF16))
    yb = sp.gemm_dense(to_dev(X, "bf16"), to_dev(W, "bf16"), algo=sp.ALGO_TILED)
    torch.cuda.synchronize()
    assert_gemm_close(yb, Yb, Sb)
    assert sp.last_device_error() == sp.OK

"""The allocation-free quantisation entry point, called through the C ABI.

sp24_quantize_nvfp4_noalloc serves callers that cannot allocate device memory (runtimes with a
fixed buffer arena, plugins whose host framework owns the allocator, host loops that must not
call cudaMalloc): it keeps its scratch in a __device__ array inside the library instead of a
caller workspace.  Its results must equal
those of sp24_quantize_nvfp4 (bit for bit: codes, block scales and tensor scale are exact),
including on consecutive calls that reuse the shared scratch.  This file sorts last so that a
run stopping at the first failure has already run every other test."""
import ctypes

import numpy as np
import pytest
import torch

import fp16_gemm_b200 as sp
import oracle
import synth

pytestmark = pytest.mark.gpu


def _ptr(t):
    return ctypes.c_void_p(t.data_ptr()) if t is not None else None


def _quantize_both(t: torch.Tensor, dtype_code: int, ts_in=None):
    L = sp.lib()
    R, C = t.shape
    stream = ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    outs = []
    for noalloc in (False, True):
        codes = torch.full((R, C // 2), 0xAA, dtype=torch.uint8, device="cuda")
        scales = torch.full((R, C // 16), 0xAA, dtype=torch.uint8, device="cuda")
        ts = torch.full((1,), -1.0, dtype=torch.float32, device="cuda")
        if noalloc:
            st = L.sp24_quantize_nvfp4_noalloc(_ptr(t), dtype_code, R, C, _ptr(ts_in), _ptr(codes),
                                               _ptr(scales), _ptr(ts), stream)
        else:
            n = ctypes.c_int64(0)
            assert L.sp24_quantize_nvfp4_workspace_size(R, C, ctypes.byref(n)) == sp.OK
            ws = torch.empty(n.value, dtype=torch.uint8, device="cuda")
            st = L.sp24_quantize_nvfp4(_ptr(t), dtype_code, R, C, _ptr(ts_in), _ptr(codes),
                                       _ptr(scales), _ptr(ts), _ptr(ws), n.value, stream)
        assert st == sp.OK, sp.lib().sp24_status_string(st)
        outs.append((codes, scales, ts))
    torch.cuda.synchronize()
    return outs


def _assert_same(a, b):
    for x, y in zip(a, b):
        assert torch.equal(x.view(torch.uint8), y.view(torch.uint8))


def _assert_oracle(t_np: np.ndarray, dtype_code: int, got, ts_in=None):
    """The no-alloc result against the CPU oracle's encoder (bit for bit)."""
    codes, scales, ts = oracle.nvfp4_encode(t_np, dtype_code, tensor_scale=ts_in)
    assert np.array_equal(got[0].cpu().numpy(), codes)
    assert np.array_equal(got[1].cpu().numpy(), scales)
    assert np.float32(got[2].item()) == np.float32(ts)


def test_noalloc_matches_workspace_entry_point_on_consecutive_calls():
    g = synth.rng(1234)
    # two calls in a row on different tensors: the second must not see the first's amax
    big = synth.as_storage(synth.normal(g, (256, 1024)) * 50.0, "bf16")
    small = synth.as_storage(synth.normal(g, (64, 512)) * 0.01, "bf16")
    for arr in (big, small):
        t = torch.from_numpy(arr.view(np.int16)).view(torch.bfloat16).cuda()
        ref, got = _quantize_both(t, sp.BF16)
        _assert_same(ref, got)
        assert got[2].item() > 0
        _assert_oracle(arr, oracle.BF16, got)


def test_noalloc_decode_weight_and_shared_scale():
    w = synth.decode_nvfp4()["W"]
    t = torch.from_numpy(w.view(np.int16)).view(torch.bfloat16).cuda()
    ref, got = _quantize_both(t, sp.BF16)
    _assert_same(ref, got)
    _assert_oracle(np.ascontiguousarray(w[:512]), oracle.BF16,
                   (got[0][:512], got[1][:512], got[2]), ts_in=float(got[2].item()))
    shared = torch.tensor([float(ref[2].item()) * 4], dtype=torch.float32, device="cuda")
    ref2, got2 = _quantize_both(t, sp.BF16, ts_in=shared)
    _assert_same(ref2, got2)
    x = torch.randn(48, 160, device="cuda")
    r3, g3 = _quantize_both(x, sp.F32)
    _assert_same(r3, g3)


def test_noalloc_argument_errors():
    L = sp.lib()
    assert L.sp24_quantize_nvfp4_noalloc(None, sp.F32, 4, 24, None, None, None, None, None) == sp.ERR_SHAPE
    assert L.sp24_quantize_nvfp4_noalloc(None, 9, 4, 32, None, None, None, None, None) == sp.ERR_DTYPE

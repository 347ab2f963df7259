"""CPU tests of the C ABI: the library builds and loads, exports every declared entry point, and
rejects bad arguments on the host without touching a device."""
import ctypes
import os
import re

import pytest

import fp16_gemm_b200 as sp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def declared_symbols():
    text = open(os.path.join(ROOT, "include", "sp24.h")).read()
    return sorted(set(re.findall(r"\b(sp24_[a-z0-9_]+)\s*\(", text)))


def test_library_exports_every_declared_symbol():
    L = sp.lib()
    names = declared_symbols()
    assert len(names) >= 13
    for n in names:
        assert hasattr(L, n), n
    assert set(names) == set(sp.EXPORTS) | (set(names) - set(sp.EXPORTS))
    for n in sp.EXPORTS:
        assert n in names, f"binding lists {n} but the header does not declare it"


def test_status_strings_and_version():
    L = sp.lib()
    assert L.sp24_abi_version() == 1
    for st in range(9):
        assert L.sp24_status_string(st)
    assert L.sp24_status_string(999) == b"unknown status"


def test_sizes_match_the_pages_byte_counts():
    """'Bit-exact check against lyf's ModelOpt output': packed / scale bytes of three tensors."""
    for shape, packed, scl in (((12288, 5120), 31457280, 3932160), ((5120, 6144), 15728640, 1966080),
                               ((17408, 5120), 44564480, 5570560)):
        s = sp.sizes(sp.OP_MATMUL, sp.BF16, shape)
        assert s["nvfp4_codes_bytes"] == packed and s["nvfp4_scales_bytes"] == scl


def test_sizes_bits_per_weight():
    """'The byte saving is about a quarter, not a half': 2 kept values + 2-bit indices."""
    N, K = 5120, 5120
    d = sp.sizes(sp.OP_MATMUL, sp.F16, (N, K))
    assert d["groups"] == N * K // 4
    assert (d["values_bytes"] + d["meta_bytes"]) * 8 / (N * K) == 9.0
    v = sp.sizes(sp.OP_MATMUL, sp.F16, (N, K // 2))
    dense = (d["nvfp4_codes_bytes"] + d["nvfp4_scales_bytes"]) * 8 / (N * K)
    sparse = (v["nvfp4_codes_bytes"] + v["nvfp4_scales_bytes"] + d["meta_bytes"]) * 8 / (N * K)
    assert dense == 4.5 and sparse == 3.25


def test_conv_sizes_and_shape_rules():
    s = sp.sizes(sp.OP_CONV, sp.F16, (256, 256, 3, 3))
    assert s["groups"] == 147456 and s["values_bytes"] == 256 * 128 * 9 * 2 and s["meta_bytes"] == 73728
    with pytest.raises(sp.SP24Error) as e:
        sp.sizes(sp.OP_CONV, sp.F16, (2, 6, 3, 3))
    assert e.value.status == sp.ERR_SHAPE


def _raw(fn, *args):
    return getattr(sp.lib(), fn)(*args)


def test_host_validation_without_launch():
    """Bad arguments come back as status codes before any CUDA call (works with no GPU)."""
    shp = (ctypes.c_int64 * 4)(2, 6, 3, 3)
    assert _raw("sp24_check_24", None, sp.F16, sp.OP_CONV, shp, 4, None, None, None) == sp.ERR_SHAPE
    assert _raw("sp24_check_24", None, 7, sp.OP_MATMUL, shp, 2, None, None, None) == sp.ERR_DTYPE
    shp2 = (ctypes.c_int64 * 4)(4, 8, 0, 0)
    assert _raw("sp24_check_24", None, sp.F16, 5, shp2, 2, None, None, None) == sp.ERR_INVALID_ARG
    assert _raw("sp24_check_24", None, sp.F16, sp.OP_MATMUL, shp2, 2, None, None, None) == sp.ERR_INVALID_ARG
    assert _raw("sp24_prune_compress_24", None, sp.BF16, sp.OP_MATMUL, (ctypes.c_int64 * 4)(4, 6), 2,
                None, None, None) == sp.ERR_SHAPE
    n = ctypes.c_int64(0)
    assert _raw("sp24_quantize_nvfp4_workspace_size", 4, 24, ctypes.byref(n)) == sp.ERR_SHAPE
    assert _raw("sp24_quantize_nvfp4", None, sp.F32, 4, 24, None, None, None, None, None, 0, None) == sp.ERR_WORKSPACE
    assert _raw("sp24_dequantize_nvfp4", None, None, None, 4, 24, sp.F32, None, None) == sp.ERR_SHAPE


def test_gemm_argument_errors():
    x = sp._Operand(sp.F16, 16, None, None)
    w = sp._Operand(sp.BF16, 16, None, None)
    L = sp.lib()
    args = lambda M, N, K: (M, N, K, None, None, 0, sp.ALGO_AUTO, None)
    assert L.sp24_gemm_dense(ctypes.byref(x), ctypes.byref(w), *args(8, 8, 64)) == sp.ERR_DTYPE
    w16 = sp._Operand(sp.F16, 16, None, None)
    assert L.sp24_gemm_dense(ctypes.byref(x), ctypes.byref(w16), *args(8, 8, 60)) == sp.ERR_SHAPE
    assert L.sp24_gemm_dense(ctypes.byref(x), ctypes.byref(w16), *args(-1, 8, 64)) == sp.ERR_SHAPE
    xm = sp._Operand(sp.F16, 8, None, None)  # misaligned
    assert L.sp24_gemm_dense(ctypes.byref(xm), ctypes.byref(w16), *args(8, 8, 64)) == sp.ERR_ALIGN
    q = sp._Operand(sp.NVFP4, 16, None, None)  # NVFP4 without scales
    assert L.sp24_gemm_dense(ctypes.byref(x), ctypes.byref(q), *args(8, 8, 64)) == sp.ERR_INVALID_ARG
    sw = sp._SparseOperand(sp.F16, 16, None, None, 16)
    assert L.sp24_gemm_sparse24(ctypes.byref(x), ctypes.byref(sw), *args(8, 8, 40)) == sp.ERR_SHAPE
    assert L.sp24_gemm_dense(ctypes.byref(x), ctypes.byref(w16), 0, 8, 64, None, None, 0, 9, None) == sp.ERR_INVALID_ARG
    # empty problems are no-ops that need no device
    assert L.sp24_gemm_dense(ctypes.byref(x), ctypes.byref(w16), *args(0, 8, 64)) == sp.OK
    assert L.sp24_gemm_sparse24(ctypes.byref(x), ctypes.byref(sw), *args(8, 0, 64)) == sp.OK


def test_binding_refuses_cpu_tensors():
    import torch
    with pytest.raises(ValueError):
        sp.check_24(torch.zeros(4, 8, dtype=torch.float16))
    with pytest.raises(ValueError):
        sp.quantize_nvfp4(torch.zeros(4, 16))


def test_pairwise48_host_validation():
    """Pairwise 4:8 entry points reject bad arguments before any CUDA call."""
    assert _raw("sp24_check_48", None, 7, 2, 16, None, None, None) == sp.ERR_DTYPE
    assert _raw("sp24_check_48", None, sp.F16, 2, 12, None, None, None) == sp.ERR_SHAPE
    assert _raw("sp24_check_48", None, sp.F16, -1, 16, None, None, None) == sp.ERR_SHAPE
    assert _raw("sp24_check_48", None, sp.F16, 2, 16, None, None, None) == sp.ERR_INVALID_ARG
    assert _raw("sp24_check_48", 1, sp.F16, 2, 16, 16, None, None) == sp.ERR_ALIGN
    assert _raw("sp24_prune_compress_48", None, sp.BF16, 2, 16, None, None, None) == sp.ERR_INVALID_ARG
    assert _raw("sp24_prune_compress_48", 16, sp.F32, 2, 16, 18, 16, None) == sp.ERR_ALIGN
    assert _raw("sp24_prune_compress_48", None, sp.F16, 0, 16, None, None, None) == sp.OK  # empty: no-op
    assert _raw("sp24_decompress_48", 16, None, sp.F16, 2, 16, 16, None) == sp.ERR_INVALID_ARG
    assert _raw("sp24_decompress_48", 16, 16, sp.F16, 2, 20, 16, None) == sp.ERR_SHAPE


def test_block32_quantiser_and_sparse48_gemm_host_validation():
    assert _raw("sp24_quantize_nvfp4_block32", None, sp.F16, 4, 48, None, None, None, 16, None, 0, None) == sp.ERR_SHAPE
    assert _raw("sp24_quantize_nvfp4_block32", None, 7, 4, 64, None, None, None, 16, None, 0, None) == sp.ERR_DTYPE
    assert _raw("sp24_quantize_nvfp4_block32", None, sp.F16, 4, 64, None, None, None, None, None, 0, None) == sp.ERR_INVALID_ARG
    assert _raw("sp24_quantize_nvfp4_block32", 16, sp.F16, 4, 64, None, 16, 16, 16, None, 0, None) == sp.ERR_WORKSPACE
    assert _raw("sp24_quantize_nvfp4_block32", 16, sp.F16, 4, 64, None, 24, 16, 16, 16, 256, None) == sp.ERR_ALIGN
    L = sp.lib()
    x = sp._Operand(sp.NVFP4_B32, 16, 16, 16)
    w = sp._SparseOperand(sp.NVFP4, 16, 16, 16, 16)
    call = lambda xo, wo, M, N, K, y=16: L.sp24_gemm_sparse48(ctypes.byref(xo), ctypes.byref(wo), M, N, K, y, None)
    assert call(sp._Operand(sp.NVFP4, 16, 16, 16), w, 8, 128, 512) == sp.ERR_DTYPE
    assert call(x, sp._SparseOperand(sp.BF16, 16, None, None, 16), 8, 128, 512) == sp.ERR_DTYPE
    assert call(x, w, 8, 128, 256) == sp.ERR_SHAPE
    assert call(x, w, -1, 128, 512) == sp.ERR_SHAPE
    assert call(x, w, 0, 128, 512) == sp.OK  # empty: no-op
    assert call(x, sp._SparseOperand(sp.NVFP4, 16, 16, 16, None), 8, 128, 512) == sp.ERR_INVALID_ARG
    assert call(x, sp._SparseOperand(sp.NVFP4, 16, 16, 16, 8), 8, 128, 512) == sp.ERR_ALIGN
    assert call(x, w, 8, 128, 512, y=None) == sp.ERR_INVALID_ARG


def test_output_alignment_checked_on_the_host():
    """A y pointer that cannot hold fp32 stores (or, for the expert block, 4-float vectors) is
    refused before any launch."""
    L = sp.lib()
    x = sp._Operand(sp.F16, 16, None, None)
    w = sp._Operand(sp.F16, 16, None, None)
    assert L.sp24_gemm_dense(ctypes.byref(x), ctypes.byref(w), 8, 8, 64, 18, None, 0, sp.ALGO_AUTO, None) == sp.ERR_ALIGN
    sw = sp._SparseOperand(sp.F16, 16, None, None, 16)
    assert L.sp24_gemm_sparse24(ctypes.byref(x), ctypes.byref(sw), 8, 8, 64, 2, None, 0, sp.ALGO_AUTO, None) == sp.ERR_ALIGN
    xq = sp._Operand(sp.NVFP4_B32, 16, 16, 16)
    wq = sp._SparseOperand(sp.NVFP4, 16, 16, 16, 16)
    assert L.sp24_gemm_sparse48(ctypes.byref(xq), ctypes.byref(wq), 8, 128, 512, 6, None) == sp.ERR_ALIGN


def test_element_alignment_checked_on_the_host():
    """An element pointer without its type's natural alignment is refused before any launch."""
    shp = (ctypes.c_int64 * 4)(4, 8)
    assert _raw("sp24_check_24", 17, sp.F16, sp.OP_MATMUL, shp, 2, 16, None, None) == sp.ERR_ALIGN
    assert _raw("sp24_prune_compress_24", 16, sp.F32, sp.OP_MATMUL, shp, 2, 18, 16, None) == sp.ERR_ALIGN
    assert _raw("sp24_decompress_24", 16, 16, sp.BF16, sp.OP_MATMUL, shp, 2, 19, None) == sp.ERR_ALIGN
    assert _raw("sp24_dequantize_nvfp4", 16, 16, 16, 4, 32, sp.F32, 18, None) == sp.ERR_ALIGN



def test_w4a4_tile_layout_host_validation():
    """The scale-tile rearrangement and the tile-order operand format, checked on the host."""
    L = sp.lib()
    n, m = ctypes.c_int64(-1), ctypes.c_int64(-1)
    assert L.sp24_nvfp4_mma_size(200, 512, ctypes.byref(n), ctypes.byref(m)) == sp.OK
    assert (n.value, m.value) == (256 * 256, 256 * 32)
    assert L.sp24_nvfp4_mma_size(1, 256, ctypes.byref(n), None) == sp.OK and n.value == 128 * 128
    assert L.sp24_nvfp4_mma_size(8, 384, ctypes.byref(n), None) == sp.ERR_SHAPE
    assert L.sp24_nvfp4_to_mma(None, None, 8, 384, None, None, None) == sp.ERR_SHAPE
    assert L.sp24_nvfp4_to_mma(None, None, 0, 256, None, None, None) == sp.OK
    assert L.sp24_nvfp4_to_mma(None, None, 4, 256, None, None, None) == sp.ERR_INVALID_ARG
    assert L.sp24_nvfp4_to_mma(8, 4, 4, 256, 16, 16, None) == sp.ERR_ALIGN
    mma = sp._Operand(sp.NVFP4_MMA, 16, 16, 16)
    f16 = sp._Operand(sp.F16, 16, None, None)
    y = ctypes.c_void_p(256)
    # a tile-order operand only meets NVFP4; K % 256; never the skinny kernels
    assert L.sp24_gemm_dense(ctypes.byref(f16), ctypes.byref(mma), 8, 8, 256, y, None, 0, 0, None) == sp.ERR_DTYPE
    assert L.sp24_gemm_dense(ctypes.byref(mma), ctypes.byref(mma), 8, 8, 128, y, None, 0, 0, None) == sp.ERR_SHAPE
    assert L.sp24_gemm_dense(ctypes.byref(mma), ctypes.byref(mma), 8, 8, 256, y, None, 0,
                             sp.ALGO_SKINNY, None) == sp.ERR_UNSUPPORTED
    q = sp._Operand(sp.NVFP4, 16, 16, 16)
    assert L.sp24_gemm_dense(ctypes.byref(q), ctypes.byref(mma), 8, 8, 256, y, None, 0, 0, None) == sp.ERR_WORKSPACE
    assert L.sp24_gemm_workspace_size(sp.NVFP4_MMA, sp.NVFP4_MMA, 0, 300, 520, 768, 0, ctypes.byref(n)) == sp.OK
    assert n.value == 0
    assert L.sp24_gemm_workspace_size(sp.NVFP4, sp.NVFP4_MMA, 0, 300, 520, 768, 0, ctypes.byref(n)) == sp.OK
    assert n.value == 384 * 384 + 384 * 48
    assert L.sp24_gemm_workspace_size(sp.NVFP4_MMA, sp.BF16, 0, 300, 520, 768, 0, ctypes.byref(n)) == sp.ERR_DTYPE


def test_wait_limit_and_selftest_host_validation():
    L = sp.lib()
    assert L.sp24_set_wait_limit(0) == sp.ERR_INVALID_ARG
    assert L.sp24_get_wait_limit(None) == sp.ERR_INVALID_ARG
    assert L.sp24_selftest_wait_timeout(None, None, None) == sp.ERR_INVALID_ARG
    assert L.sp24_selftest_wait_timeout(ctypes.c_void_p(8), ctypes.c_void_p(16), None) == sp.ERR_ALIGN


def test_peak_microbenchmark_host_validation():
    L = sp.lib()
    assert L.sp24_peak_ctas(5) == 0 and L.sp24_peak_ctas(-1) == 0
    assert L.sp24_peak_mma(5, 10, ctypes.c_void_p(64), None) == sp.ERR_INVALID_ARG
    assert L.sp24_peak_mma(0, 0, ctypes.c_void_p(64), None) == sp.ERR_INVALID_ARG
    assert L.sp24_peak_mma(0, 10, ctypes.c_void_p(4), None) == sp.ERR_ALIGN
    assert L.sp24_peak_read(None, 1024, None, None) == sp.ERR_INVALID_ARG
    assert L.sp24_peak_read(ctypes.c_void_p(16), 24, ctypes.c_void_p(16), None) == sp.ERR_INVALID_ARG


def test_sparse_pair_images_host_validation():
    L = sp.lib()
    a, b, c = ctypes.c_int64(-1), ctypes.c_int64(-1), ctypes.c_int64(-1)
    assert L.sp24_sparse48_mma_size(300, 1024, ctypes.byref(a), ctypes.byref(b), ctypes.byref(c)) == sp.OK
    assert (a.value, b.value, c.value) == (512 * 256, 512 * 32, 512 * 64)
    assert L.sp24_sparse48_mma_size(8, 768, None, None, None) == sp.ERR_SHAPE
    assert L.sp24_nvfp4_b32_mma_size(200, 512, ctypes.byref(a), ctypes.byref(b)) == sp.OK
    assert (a.value, b.value) == (256 * 256, 256 * 16)
    assert L.sp24_sparse48_to_mma(None, None, None, 4, 512, None, None, None, None) == sp.ERR_INVALID_ARG
    assert L.sp24_nvfp4_b32_to_mma(None, None, 4, 256, None, None, None) == sp.ERR_INVALID_ARG
    # images are taken for both operands or neither
    xo = sp._Operand(sp.NVFP4_B32_MMA, 16, 16, 16)
    wo = sp._SparseOperand(sp.NVFP4, 16, 16, 16, 16)
    assert L.sp24_gemm_sparse48(ctypes.byref(xo), ctypes.byref(wo), 4, 128, 512, ctypes.c_void_p(256), None) == sp.ERR_DTYPE


def test_prepare_sparse_host_validation():
    """The metadata image of the 16-bit 2:4 pair kernel: rows padded to 256, 2 KB per 128 rows and
    128 K; K must be a multiple of 128."""
    L = sp.lib()
    n = ctypes.c_int64(-1)
    assert L.sp24_prepare_sparse_size(300, 256, ctypes.byref(n)) == sp.OK
    assert n.value == 4 * 2 * 2048
    assert L.sp24_prepare_sparse_size(256, 128, ctypes.byref(n)) == sp.OK and n.value == 2 * 1 * 2048
    assert L.sp24_prepare_sparse_size(8, 192, ctypes.byref(n)) == sp.ERR_SHAPE
    assert L.sp24_prepare_sparse_size(8, 128, None) == sp.ERR_INVALID_ARG
    assert L.sp24_prepare_sparse(None, 8, 256, None, None) == sp.ERR_INVALID_ARG
    assert L.sp24_prepare_sparse(None, 8, 96, None, None) == sp.ERR_SHAPE
    assert L.sp24_prepare_sparse(None, 0, 256, None, None) == sp.OK
    assert L.sp24_prepare_sparse(ctypes.c_void_p(16), 8, 256, ctypes.c_void_p(8), None) == sp.ERR_ALIGN


def test_gemm_workspace_holds_the_metadata_image():
    """A tiled 2:4 product runs on the 16-bit CTA-pair kernel, whose workspace holds the metadata
    image (2 KB per 128 rows padded to 256 and 128 K) beside any 16-bit expansion of NVFP4 kept
    values (N x K/2 entries of 2 bytes); dense 16-bit needs none, nor the skinny path."""
    L = sp.lib()
    n = ctypes.c_int64(-1)
    image = 4 * 2 * 2048  # N = 300 -> 512 rows, K = 256 -> 2 chunks
    assert L.sp24_gemm_workspace_size(sp.F16, sp.F16, 1, 128, 300, 256, sp.ALGO_AUTO, ctypes.byref(n)) == sp.OK
    assert n.value == image
    assert L.sp24_gemm_workspace_size(sp.BF16, sp.NVFP4, 1, 256, 300, 256, sp.ALGO_AUTO, ctypes.byref(n)) == sp.OK
    assert n.value == 300 * 256 + image
    assert L.sp24_gemm_workspace_size(sp.BF16, sp.NVFP4, 1, 128, 300, 256, sp.ALGO_AUTO, ctypes.byref(n)) == sp.OK
    assert n.value == 300 * 256 + image
    # dense NVFP4 weights with 16-bit x stay on the skinny kernels up to M = 128 (no expansion)
    assert L.sp24_gemm_workspace_size(sp.BF16, sp.NVFP4, 0, 128, 300, 256, sp.ALGO_AUTO, ctypes.byref(n)) == sp.OK
    assert n.value == 0
    assert L.sp24_gemm_workspace_size(sp.BF16, sp.NVFP4, 0, 129, 300, 256, sp.ALGO_AUTO, ctypes.byref(n)) == sp.OK
    assert n.value == 300 * 256 * 2
    assert L.sp24_gemm_workspace_size(sp.F16, sp.F16, 0, 128, 300, 256, sp.ALGO_AUTO, ctypes.byref(n)) == sp.OK
    assert n.value == 0
    assert L.sp24_gemm_workspace_size(sp.F16, sp.F16, 1, 8, 300, 256, sp.ALGO_AUTO, ctypes.byref(n)) == sp.OK
    assert n.value == 0


def test_expert_and_step_entry_points_host_validation():
    """The routed-expert, expert-block, paired-quantiser, prepare, group-scale, interleave and
    selection entry points reject bad arguments on the host, before any CUDA call."""
    L = sp.lib()
    P = ctypes.c_void_p
    n = ctypes.c_int64(-1)
    # routed experts
    assert L.sp24_gemm_grouped_workspace_size(8, 2, 0, ctypes.byref(n)) == sp.ERR_SHAPE
    assert L.sp24_gemm_grouped_workspace_size(8, 2, 4, None) == sp.ERR_INVALID_ARG
    x16 = sp._Operand(sp.F16, 16, None, None)
    x32 = sp._Operand(sp.F32, 16, None, None)
    wd = sp._Operand(sp.F16, 16, None, None)
    ws = sp._SparseOperand(sp.F16, 16, None, None, 16)
    g = lambda x, d, s, E=4, N=8, K=64, rt=16, y=16: L.sp24_gemm_grouped(
        x, rt, 8, 2, d, s, E, N, K, y, None, 0, None)
    assert g(None, ctypes.byref(wd), None) == sp.ERR_INVALID_ARG
    assert g(ctypes.byref(x16), ctypes.byref(wd), ctypes.byref(ws)) == sp.ERR_INVALID_ARG  # both forms
    assert g(ctypes.byref(x16), None, None) == sp.ERR_INVALID_ARG                           # neither
    assert g(ctypes.byref(x16), ctypes.byref(wd), None, E=0) == sp.ERR_SHAPE
    assert g(ctypes.byref(x16), ctypes.byref(wd), None, N=0) == sp.OK                       # nothing to do
    assert g(ctypes.byref(x16), ctypes.byref(wd), None, rt=None) == sp.ERR_INVALID_ARG
    assert g(ctypes.byref(x16), ctypes.byref(wd), None, y=18) == sp.ERR_ALIGN
    assert g(ctypes.byref(x32), ctypes.byref(wd), None) == sp.ERR_DTYPE
    # expert block: NVFP4 experts, 16-bit tokens
    assert L.sp24_moe_block_workspace_size(8, 2, 4, -1, 16, ctypes.byref(n)) == sp.ERR_SHAPE
    q = sp._Operand(sp.NVFP4, 16, 16, 16)
    qs_nometa = sp._SparseOperand(sp.NVFP4, 16, 16, 16, None)
    b = lambda x, gu, gus, dn, dns, E=4, H=64, y=16: L.sp24_moe_block(
        x, 16, 16, 8, 2, gu, gus, dn, dns, E, H, 32, y, None, 0, None)
    assert b(None, ctypes.byref(q), None, ctypes.byref(q), None) == sp.ERR_INVALID_ARG
    assert b(ctypes.byref(x16), ctypes.byref(q), None, ctypes.byref(q), None, E=0) == sp.ERR_SHAPE
    assert b(ctypes.byref(x32), ctypes.byref(q), None, ctypes.byref(q), None) == sp.ERR_DTYPE
    assert b(ctypes.byref(x16), ctypes.byref(wd), None, ctypes.byref(q), None) == sp.ERR_DTYPE  # 16-bit experts
    assert b(ctypes.byref(x16), None, ctypes.byref(qs_nometa), ctypes.byref(q), None) == sp.ERR_INVALID_ARG
    assert b(ctypes.byref(x16), ctypes.byref(q), None, None, None) == sp.ERR_INVALID_ARG
    assert b(ctypes.byref(x16), ctypes.byref(q), None, ctypes.byref(q), None, H=0) == sp.OK
    assert b(ctypes.byref(x16), ctypes.byref(q), None, ctypes.byref(q), None, y=None) == sp.ERR_INVALID_ARG
    assert b(ctypes.byref(x16), ctypes.byref(q), None, ctypes.byref(q), None, y=20) == sp.ERR_ALIGN
    # gate / up row interleave
    assert L.sp24_interleave_rows(16, 16, 8, 64, 0, 16, None) == sp.ERR_SHAPE
    assert L.sp24_interleave_rows(16, 16, 8, 64, 3, 16, None) == sp.ERR_SHAPE    # rows % block_rows
    assert L.sp24_interleave_rows(16, 16, 8, 40, 4, 16, None) == sp.ERR_SHAPE    # row bytes % 16
    assert L.sp24_interleave_rows(None, None, 0, 64, 4, None, None) == sp.OK
    assert L.sp24_interleave_rows(None, 16, 8, 64, 4, 16, None) == sp.ERR_INVALID_ARG
    assert L.sp24_interleave_rows(16, 24, 8, 64, 4, 16, None) == sp.ERR_ALIGN
    # one-pass prepare (check + prune / compress + both tensor scales)
    assert L.sp24_prepare_24_workspace_size(4, 24, ctypes.byref(n)) == sp.ERR_SHAPE
    pr = lambda dt=sp.BF16, K=64, w=16, wsp=256, wsb=256: L.sp24_prepare_24(
        w, dt, 4, K, None, None, 16, 16, 16, 16, wsp, wsb, None)
    assert pr(dt=9) == sp.ERR_DTYPE
    assert pr(K=24) == sp.ERR_SHAPE
    assert pr(w=None) == sp.ERR_INVALID_ARG
    assert pr(wsp=None) == sp.ERR_WORKSPACE
    assert pr(wsb=128) == sp.ERR_WORKSPACE
    assert pr(wsp=264) == sp.ERR_ALIGN
    assert pr(w=24) == sp.ERR_ALIGN
    # paired NVFP4 encode (a weight and its kept values, each with a supplied scale)
    qp = lambda dt=sp.BF16, c0=64, ts=16, t0=16: L.sp24_quantize_nvfp4_pair(
        t0, dt, 4, c0, ts, 16, 16, 16, 16, 4, 32, 16, 16, 16, 16, None)
    assert qp(dt=9) == sp.ERR_DTYPE
    assert qp(c0=24) == sp.ERR_SHAPE
    assert qp(ts=None) == sp.ERR_INVALID_ARG
    assert qp(t0=None) == sp.ERR_INVALID_ARG
    assert qp(t0=8) == sp.ERR_ALIGN
    # group-shared tensor scale
    assert L.sp24_nvfp4_group_tensor_scale_workspace_size(ctypes.byref(n)) == sp.OK and n.value == 16
    ptrs = (P * 2)(16, 32)
    gs = lambda nums, dt=sp.BF16, out=16, wsp=256, p=ptrs: L.sp24_nvfp4_group_tensor_scale(
        p, (ctypes.c_int64 * 2)(*nums), 2, dt, out, wsp, 16, None)
    assert gs((64, 64), out=None) == sp.ERR_INVALID_ARG
    assert gs((64, 64), dt=9) == sp.ERR_DTYPE
    assert gs((64, 12)) == sp.ERR_SHAPE                                         # 24 bytes
    assert gs((64, 64), p=(P * 2)(16, None)) == sp.ERR_INVALID_ARG
    assert gs((64, 64), p=(P * 2)(16, 40)) == sp.ERR_ALIGN
    assert gs((64, 64), wsp=None) == sp.ERR_WORKSPACE
    assert L.sp24_nvfp4_group_tensor_scale(None, None, -1, sp.BF16, 16, 256, 16, None) == sp.ERR_INVALID_ARG
    # measured selection and the auto GEMM
    use = ctypes.c_int(-1)
    wq = sp._Operand(sp.NVFP4, 16, 16, 16)
    assert L.sp24_gemm_select(ctypes.byref(x16), ctypes.byref(wd), ctypes.byref(ws), 8, 8, 64, 16, None, 0, 0,
                              ctypes.byref(use), None, None, None) == sp.ERR_INVALID_ARG   # reps < 1
    assert L.sp24_gemm_select(ctypes.byref(x16), ctypes.byref(wq), ctypes.byref(ws), 8, 8, 64, 16, None, 0, 3,
                              ctypes.byref(use), None, None, None) == sp.ERR_DTYPE         # forms disagree
    assert L.sp24_gemm_select(ctypes.byref(x32), ctypes.byref(wd), ctypes.byref(ws), 8, 8, 64, 16, None, 0, 3,
                              ctypes.byref(use), None, None, None) == sp.ERR_DTYPE         # no such pair
    assert L.sp24_gemm_auto(ctypes.byref(x16), ctypes.byref(wd), None, 8, 8, 64, 16, None, 0, None,
                            None) == sp.ERR_INVALID_ARG
    assert L.sp24_gemm_auto(ctypes.byref(x16), ctypes.byref(wq), ctypes.byref(ws), 8, 8, 64, 16, None, 0, None,
                            None) == sp.ERR_DTYPE
    assert use.value == -1

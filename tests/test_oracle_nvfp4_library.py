"""Pins for the oracle's NVFP4 formulae against two third-party implementations of the same
recipe, the one the pages' converter reproduces bit for bit (NVFP4 Without FP4 Hardware,
"Bit-exact check against lyf's ModelOpt output": packed weights, block scales and global
scales identical to a ModelOpt checkpoint):

* compressed-tensors' ``generate_gparam``: the per-tensor global scale of that recipe,
  E4M3 max * E2M1 max / amax, the reciprocal of the oracle's tensor scale amax / 2688;
* vLLM's ``ref_nvfp4_quant`` (its CPU emulation of NVFP4 activations): block scale
  E4M3(global * bmax / 6) and element E2M1(x / (block scale / global)), both round to nearest
  even, the block scale clamped to 448 and the scaled element to 6.

Both libraries evaluate the steps in fp32 in their own order (a reciprocal, then a multiply),
the oracle as divisions; so a block scale or a code may differ where the exact quotient lies
within a few fp32 roundings of a rounding boundary.  The tests find those places from the exact
quotients in fp64, allow a difference of one step there only, and require that they are rare,
so that a wrong constant, block size, rounding mode, clamp, index or sign fails."""
import ml_dtypes
import numpy as np
import pytest

import synth

torch = pytest.importorskip("torch")
ct_helpers = pytest.importorskip("compressed_tensors.quantization.utils.helpers")
vllm_nvfp4 = pytest.importorskip("vllm.model_executor.layers.quantization.utils.nvfp4_emulation_utils")

# relative distance from a rounding boundary under which the two fp32 evaluation orders may
# round to different sides (each side makes at most three fp32 roundings of 2^-24 relative)
NEAR = 2.0 ** -19

E2M1_MAG = np.array([0.0, 0.5, 1.0, 1.5, 2.0, 3.0, 4.0, 6.0])
E2M1_MID = (E2M1_MAG[1:] + E2M1_MAG[:-1]) / 2
E4M3_POS = np.arange(0, 127, dtype=np.uint8).view(ml_dtypes.float8_e4m3fn).astype(np.float64)
E4M3_MID = (E4M3_POS[1:] + E4M3_POS[:-1]) / 2


def _near(q, mids):
    """True where q lies within NEAR (relative) of one of the midpoints."""
    q = np.asarray(q, dtype=np.float64)
    d = np.min(np.abs(q[..., None] - mids), axis=-1)
    return d <= NEAR * np.maximum(q, np.finfo(np.float64).tiny)


def _nibbles(codes):
    return np.stack([codes & 0xF, codes >> 4], axis=-1).reshape(codes.shape[0], -1)


def _library_quant(tf32, gs, block):
    """vLLM's reference NVFP4 quantiser: (signed E2M1 values as fp64, E4M3 scales as fp64)."""
    q, s = vllm_nvfp4.ref_nvfp4_quant(torch.from_numpy(tf32), torch.tensor(gs, dtype=torch.float32), block)
    return q.double().numpy(), s.double().numpy()


def _compare(oracle, t_bits, dtype, tf32, ts, gs, block, min_blocks_checked=0.98):
    """Encode with the oracle at tensor scale ts and with the library at global scale gs;
    check scales and codes agree everywhere except next to a rounding boundary."""
    R, L = tf32.shape
    codes, scales, ts_used = oracle.nvfp4_encode(t_bits, dtype, tensor_scale=ts, block=block)
    lib_vals, lib_scales = _library_quant(tf32, gs, block)

    ours_s = scales.view(ml_dtypes.float8_e4m3fn).astype(np.float64)
    a = np.abs(tf32.astype(np.float64)).reshape(R, L // block, block)
    s_t = float(np.float32(ts_used))
    q_scale = a.max(-1) / (6.0 * s_t)
    near_s = _near(np.minimum(q_scale, 448.0), E4M3_MID)
    diff_s = ours_s != lib_scales
    assert not np.any(diff_s & ~near_s), "block scales differ away from an E4M3 boundary"
    steps = np.abs(np.searchsorted(E4M3_POS, ours_s) - np.searchsorted(E4M3_POS, lib_scales))
    assert np.all(steps[diff_s] == 1)
    assert near_s.mean() <= 1 - min_blocks_checked

    same = ~diff_s
    nib = _nibbles(codes).reshape(R, L // block, block)
    mag = E2M1_MAG[nib & 7]
    lib = lib_vals.reshape(R, L // block, block)
    with np.errstate(divide="ignore", invalid="ignore"):
        r = a / (ours_s[..., None] * s_t)
    r = np.where(ours_s[..., None] > 0, r, 0.0)
    near_c = _near(np.minimum(r, 6.0), E2M1_MID)
    diff_c = (mag != np.abs(lib)) & same[..., None]
    assert not np.any(diff_c & ~near_c), "E2M1 codes differ away from a rounding boundary"
    assert near_c[same].mean() < 0.01
    # the sign is the element's sign wherever the magnitude is nonzero
    nz = (mag > 0) & same[..., None]
    assert np.array_equal((nib[nz] >> 3) == 1, lib[nz] < 0)
    return codes, scales, ts_used


def test_tensor_scale_is_the_library_global_scale_reciprocal(oracle):
    """amax / 2688 against compressed-tensors' E4M3 max * E2M1 max / amax."""
    g = synth.rng(81)
    for sigma in (0.02, 1.0, 300.0):
        x = synth.normal(g, (64, 256), sigma)
        t = synth.as_storage(x, "bf16")
        tf = synth.bf16_bits_to_f32(t)
        gp = ct_helpers.generate_gparam(torch.tensor(tf.min()), torch.tensor(tf.max())).item()
        ts = oracle.nvfp4_tensor_scale(t, oracle.BF16)
        assert abs(ts * gp - 1.0) <= 2.0 ** -21


@pytest.mark.parametrize("block", [16, 32])
def test_encode_matches_library_quantiser(oracle, block):
    """Decode-workload-like weights (bf16, N(0, 0.02)) with a per-row spread of magnitudes so
    that many E4M3 exponents occur; the oracle derives the tensor scale, the library gets the
    reciprocal global scale from compressed-tensors."""
    g = synth.rng(82 + block)
    x = synth.normal(g, (96, 512), 0.02) * np.exp(2.0 * synth.normal(g, (96, 1)))
    t = synth.as_storage(x, "bf16")
    tf = synth.bf16_bits_to_f32(t).astype(np.float32)
    gp = ct_helpers.generate_gparam(torch.tensor(tf.min()), torch.tensor(tf.max())).item()
    _compare(oracle, t, oracle.BF16, tf, None, gp, block)


def test_encode_matches_library_with_a_shared_scale_and_saturation(oracle):
    """A group tensor scale taken from a larger tensor (the pages' shared global scale) and one
    smaller than this tensor's own (block scales clamp at 448, codes at 6), plus all-zero
    blocks: both sides saturate and zero the same way."""
    g = synth.rng(90)
    x = synth.normal(g, (32, 256), 1.0)
    x[3, 16:32] = 0.0
    x[7, :] = 0.0
    t = synth.as_storage(x, "bf16")
    tf = synth.bf16_bits_to_f32(t).astype(np.float32)
    amax = float(np.abs(tf).max())
    for ts in (np.float32(4 * amax / 2688), np.float32(amax / 2688 / 8)):
        gs = float(np.float32(1.0) / ts)
        codes, scales, _ = _compare(oracle, t, oracle.BF16, tf, float(ts), gs, 16, min_blocks_checked=0.95)
        assert np.all(scales[7] == 0) and np.all(_nibbles(codes)[7] & 7 == 0)
    # the saturated case really saturates
    assert np.any(scales == 0x7E)


def test_encode_f16_storage_matches_library(oracle):
    """The fp16 input path of the oracle against the same library quantiser."""
    g = synth.rng(91)
    x = synth.normal(g, (48, 256), 0.5)
    t = synth.as_storage(x, "f16")
    tf = t.astype(np.float32)
    gp = ct_helpers.generate_gparam(torch.tensor(tf.min()), torch.tensor(tf.max())).item()
    _compare(oracle, t, oracle.F16, tf, None, gp, 16)

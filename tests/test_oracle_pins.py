"""Pins for the CPU oracle: it is checked against what the pages and the mathematics fix, never
against itself.  Each test names the passage or the property it rests on."""
import itertools
import os

import ml_dtypes
import numpy as np
import pytest

import synth

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def _rows(name):
    out = []
    with open(os.path.join(GOLDEN, name)) as f:
        for line in f:
            line = line.strip()
            if not line or line.startswith("#"):
                continue
            out.append([c.strip() for c in line.split("|")])
    return out


def f16(a):
    return np.asarray(a, dtype=np.float16)


# ----------------------------------------------------------------------------- check_24

def test_toy_vectors(oracle):
    """'Two half-zero vectors produce different pattern answers': A passes both groups, B
    fails its first group, the extra zeros of B's second group repair nothing, and both are
    50% zero overall."""
    for name, vec, passes, nfail, zfrac in _rows("toy_vectors.txt"):
        v = f16([float(x) for x in vec.split(",")]).reshape(1, -1)
        p, n = oracle.check_24(v, oracle.F16, oracle.MATMUL)
        assert p.ravel().tolist() == [int(x) for x in passes.split(",")], name
        assert n == int(nfail), name
        assert np.mean(v == 0) == float(zfrac), name


@pytest.mark.parametrize("zeros,expect", [(0, 0), (1, 0), (2, 1), (3, 1), (4, 1)])
def test_at_least_two_zeros(oracle, zeros, expect):
    """'at least two zeros per four-entry group' (the operation section): 2, 3, 4 zeros pass."""
    for pos in itertools.combinations(range(4), zeros):
        g = f16([1.5, -2.0, 3.0, 4.0])
        g[list(pos)] = 0
        p, n = oracle.check_24(g.reshape(1, 4), oracle.F16)
        assert p[0, 0] == expect and n == 1 - expect


def test_zero_semantics(oracle):
    """Both signed zeros count as zero; NaN and subnormals are not zero."""
    cases = [([0.0, -0.0, 1.0, 1.0], 1), ([np.nan, 0.0, 1.0, 1.0], 0),
             ([6e-8, 0.0, 1.0, 1.0], 0)]
    for vals, expect in cases:
        for dt, cast in ((oracle.F16, f16),
                         (oracle.BF16, lambda a: synth.f32_to_bf16_bits(np.float32(a))),
                         (oracle.F32, lambda a: np.asarray(a, np.float32))):
            p, _ = oracle.check_24(cast(vals).reshape(1, 4), dt)
            assert p[0, 0] == expect, (vals, dt)


def test_conv_groups_run_along_c(oracle):
    """'For Convolution weights [K,C,R,S] ... groups run along input channels C at each fixed
    output channel and kernel position': the pass map equals the matmul check of the
    [K, R, S, C] permuted view, re-indexed to [K, C/4, R, S]."""
    g = synth.rng(3)
    w = synth.structured_edge(g, 8 * 3 * 2, 12, "f16").reshape(8, 3, 2, 12)  # [K,R,S,C]
    conv = np.ascontiguousarray(w.transpose(0, 3, 1, 2))                     # [K,C,R,S]
    p_conv, n_conv = oracle.check_24(conv, oracle.F16, oracle.CONV)
    p_mm, n_mm = oracle.check_24(np.ascontiguousarray(w), oracle.F16, oracle.MATMUL)
    assert p_conv.shape == (8, 3, 3, 2)
    assert np.array_equal(p_conv, p_mm.transpose(0, 3, 1, 2))
    assert n_conv == n_mm
    # flattening the conv tensor along its last axis would group the wrong entries
    p_flat, _ = oracle.check_24(conv.reshape(8, -1), oracle.F16, oracle.MATMUL)
    assert p_flat.size == p_conv.size and not np.array_equal(p_flat.ravel(), p_conv.ravel())


def test_conv_c_not_multiple_of_four_rejected(oracle):
    with pytest.raises(oracle.OracleError):
        oracle.check_24(np.zeros((2, 6, 3, 3), np.float16), oracle.F16, oracle.CONV)
    with pytest.raises(oracle.OracleError):
        oracle.check_24(np.zeros((2, 6), np.float16), oracle.F16, oracle.MATMUL)


def test_conv_fail5_generator_counts(oracle):
    d = synth.conv_fail5(shape=(16, 16, 3, 3))
    G = 16 * 4 * 9
    p, n = oracle.check_24(d["W"], oracle.F16, oracle.CONV)
    assert n == round(0.05 * G)
    assert np.array_equal(np.flatnonzero(p.ravel() == 0), d["failing"])


# ----------------------------------------------------------------------------- prune

def _brute_keep(mags):
    """All C(4,2) choices; keep the one with the largest sum of magnitudes, ties -> the
    lexicographically smallest ascending pair."""
    best, bsum = None, -1.0
    for pair in itertools.combinations(range(4), 2):
        s = mags[pair[0]] + mags[pair[1]]
        if s > bsum:
            best, bsum = pair, s
    return best


def test_prune_brute_force(oracle):
    """Magnitude pruning to 2 of 4 ('What 2:4 actually is'; ties to the lower index) equals
    brute-force enumeration of the six 2-of-4 choices.  fp16 magnitudes make every pair sum
    exact in fp64, so the enumeration decides ties exactly."""
    g = synth.rng(11)
    w = synth.structured_edge(g, 64, 256, "f16")
    vals, meta = oracle.compress_24(w, oracle.F16)
    pr = oracle.prune_24(w, oracle.F16)
    mags = np.abs(w.astype(np.float64)).reshape(-1, 4)
    nib = np.stack([meta & 0xF, meta >> 4], 1).ravel()[: mags.shape[0]]
    for gi in range(mags.shape[0]):
        i0, i1 = _brute_keep(mags[gi])
        assert (nib[gi] & 3, nib[gi] >> 2) == (i0, i1), gi
        row = pr.reshape(-1, 4)[gi].view(np.uint16)
        src = w.reshape(-1, 4)[gi].view(np.uint16)
        for i in range(4):
            assert row[i] == (src[i] if i in (i0, i1) else 0)


def test_prune_exhaustive_small_alphabet(oracle):
    """Every group over the magnitudes {0, 1, 2} with both signs (6^4 groups)."""
    alphabet = [0.0, -0.0, 1.0, -1.0, 2.0, -2.0]
    groups = np.array(list(itertools.product(alphabet, repeat=4)), dtype=np.float16)
    vals, meta = oracle.compress_24(groups.reshape(1, -1), oracle.F16)
    nib = np.stack([meta & 0xF, meta >> 4], 1).ravel()
    for gi, grp in enumerate(groups.astype(np.float64)):
        i0, i1 = _brute_keep(np.abs(grp))
        assert (nib[gi] & 3, nib[gi] >> 2) == (i0, i1)


def test_prune_ties_and_zeros(oracle):
    """[0,0,5,0] keeps indices 0 and 2 (reading: exactly two kept, zeros by the tie rule);
    equal magnitudes of opposite sign tie on magnitude, the lower index wins."""
    cases = {(0, 0, 5, 0): (0, 2), (1, 1, 1, 1): (0, 1), (-2, 1, 2, 1): (0, 2),
             (1, -3, 3, 0): (1, 2), (0, 0, 0, 7): (0, 3)}
    for vals, pair in cases.items():
        v, m = oracle.compress_24(f16(vals).reshape(1, 4), oracle.F16)
        assert (m[0] & 3, m[0] >> 2) == pair, vals
        assert np.array_equal(v.ravel().astype(np.float64), np.array(vals, np.float64)[list(pair)])


def test_prune_nan_is_largest(oracle):
    v, m = oracle.compress_24(f16([np.nan, 1, 2, 3]).reshape(1, 4), oracle.F16)
    assert (m[0] & 3, m[0] >> 2) == (0, 3)


def test_prune_fp32_bf16_order(oracle):
    """Magnitude order follows the value, for every storage type (|w| bit patterns are
    monotone in |w|)."""
    g = synth.rng(5)
    x = synth.normal(g, (32, 64))
    for dt, st in ((oracle.F32, "f32"), (oracle.BF16, "bf16")):
        w = synth.as_storage(x, st)
        _, meta = oracle.compress_24(w, dt)
        wf = synth.bf16_bits_to_f32(w) if st == "bf16" else w
        mags = np.abs(wf.astype(np.float64)).reshape(-1, 4)
        nib = np.stack([meta & 0xF, meta >> 4], 1).ravel()
        order = np.argsort(-mags, axis=1, kind="stable")[:, :2]
        order.sort(axis=1)
        assert np.array_equal(nib & 3, order[:, 0]) and np.array_equal(nib >> 2, order[:, 1])


def test_roundtrip_and_meta_legal(oracle):
    """decompress(compress(W)) == prune(W) bitwise; every nibble is one of the six ascending
    index pairs; the pruned tensor passes the check in every group."""
    g = synth.rng(7)
    for dt, st in ((oracle.F16, "f16"), (oracle.BF16, "bf16"), (oracle.F32, "f32")):
        w = synth.structured_edge(g, 24, 96, st)
        vals, meta = oracle.compress_24(w, dt)
        back = oracle.decompress_24(vals, meta, dt, w.shape)
        pr = oracle.prune_24(w, dt)
        assert np.array_equal(back.view(np.uint8), pr.view(np.uint8))
        nib = np.stack([meta & 0xF, meta >> 4], 1).ravel()
        assert set(np.unique(nib).tolist()) <= {0x4, 0x8, 0xC, 0x9, 0xD, 0xE}
        p, n = oracle.check_24(pr, dt)
        assert n == 0 and p.all()


def test_conv_roundtrip(oracle):
    g = synth.rng(8)
    w = synth.structured_edge(g, 4 * 8, 3 * 3, "f16").reshape(4, 8, 3, 3)
    vals, meta = oracle.compress_24(w, oracle.F16, oracle.CONV)
    assert vals.shape == (4, 4, 3, 3) and meta.size == 4 * 2 * 9 // 2
    back = oracle.decompress_24(vals, meta, oracle.F16, w.shape, oracle.CONV)
    assert np.array_equal(back.view(np.uint16), oracle.prune_24(w, oracle.F16, oracle.CONV).view(np.uint16))
    # the conv prune equals the matmul prune of the [K,R,S,C] view
    mm = np.ascontiguousarray(w.transpose(0, 2, 3, 1))
    pr_mm = oracle.prune_24(mm, oracle.F16).transpose(0, 3, 1, 2)
    assert np.array_equal(back.view(np.uint16), np.ascontiguousarray(pr_mm).view(np.uint16))


def test_conv_values_layout_brute_force(oracle):
    """The compressed conv tensor is [K, C/2, R, S]: group (k, j, r, s) runs over w[k, 4j..4j+3,
    r, s] ("The operation determines which four entries belong together": groups along C) and
    its kept entries, the two largest magnitudes in ascending index order, sit at
    values[k, 2j], values[k, 2j + 1] of the same (r, s); found here by sorting each group."""
    g = synth.rng(9)
    K, C, R, S = 3, 12, 2, 3
    w = f16(synth.normal(g, (K, C, R, S)))
    vals, meta = oracle.compress_24(w, oracle.F16, oracle.CONV)
    assert vals.shape == (K, C // 2, R, S)
    want = np.zeros((K, C // 2, R, S), dtype=np.float16)
    nib = []
    for k in range(K):
        for j in range(C // 4):
            for r in range(R):
                for s_ in range(S):
                    grp = w[k, 4 * j:4 * j + 4, r, s_]
                    order = sorted(range(4), key=lambda i: (-abs(float(grp[i])), i))
                    i0, i1 = sorted(order[:2])
                    want[k, 2 * j, r, s_], want[k, 2 * j + 1, r, s_] = grp[i0], grp[i1]
                    nib.append(i0 | i1 << 2)
    assert np.array_equal(vals.view(np.uint16), want.view(np.uint16))
    got_nib = np.stack([meta & 0xF, meta >> 4], 1).ravel()[:len(nib)]
    assert got_nib.tolist() == nib


def test_decompress_rejects_illegal_nibble(oracle):
    with pytest.raises(oracle.OracleError):
        oracle.decompress_24(np.zeros(2, np.float16), np.array([0x5], np.uint8), oracle.F16, (4,))


def test_storage_bits_per_weight(oracle):
    """'The byte saving is about a quarter, not a half': sizes of what the oracle emits."""
    expect = {r[0]: float(r[1]) for r in _rows("bits_per_weight.txt")}
    N, K = 64, 256
    w = synth.draw(synth.rng(1), (N, K), "f16")
    vals, meta = oracle.compress_24(w, oracle.F16)
    assert (vals.nbytes + meta.nbytes) * 8 / (N * K) == expect["fp16_sparse24"]
    assert w.nbytes * 8 / (N * K) == expect["fp16_dense"]
    codes, scales, _ = oracle.nvfp4_encode(w, oracle.F16)
    dense_bits = (codes.nbytes + scales.nbytes) * 8 / (N * K)
    assert dense_bits == expect["nvfp4_dense"]
    vcodes, vscales, _ = oracle.nvfp4_encode(vals, oracle.F16)
    sparse_bits = (vcodes.nbytes + vscales.nbytes + meta.nbytes) * 8 / (N * K)
    assert sparse_bits == expect["nvfp4_sparse24"]
    assert abs((1 - sparse_bits / dense_bits) - expect["saving_nvfp4"]) < 0.005


# ----------------------------------------------------------------------------- NVFP4

def test_byte_counts_of_real_tensors(oracle):
    """'Bit-exact check against lyf's ModelOpt output': packed / block-scale / global-scale
    byte counts.  The out_proj-sized tensor is encoded for real; all three rows check the
    packed : scales = 8 : 1 accounting."""
    for name, rows, cols, packed, scl, glob in _rows("nvfp4_byte_counts.txt"):
        rows, cols = int(rows), int(cols)
        assert rows * cols // 2 == int(packed) and rows * cols // 16 == int(scl), name
        if name == "out_proj":
            t = np.zeros((rows, cols), dtype=np.uint16)
            codes, scales, ts = oracle.nvfp4_encode(t, oracle.BF16)
            assert codes.nbytes == int(packed) and scales.nbytes == int(scl)
            assert np.float32(ts).nbytes == int(glob)


def test_e2m1_against_ml_dtypes(oracle):
    """E2M1 decode and round-to-nearest-even (saturating) agree with ml_dtypes' float4_e2m1fn,
    an independent implementation of the format, over every code and every midpoint."""
    lib_vals = np.arange(16, dtype=np.uint8).view(ml_dtypes.float4_e2m1fn).astype(np.float64)
    ours = np.array([oracle.e2m1_value(c) for c in range(16)])
    assert np.array_equal(ours, lib_vals) and np.array_equal(np.signbit(ours), np.signbit(lib_vals))
    pos = lib_vals[:8]
    probes = np.concatenate([pos, (pos[1:] + pos[:-1]) / 2, pos + 0.01, pos - 0.01,
                             [6.5, 7.0, 7.5, 100.0, 1e30]])
    probes = probes[probes >= 0]
    lib_codes = probes.astype(np.float32).astype(ml_dtypes.float4_e2m1fn).view(np.uint8)
    for x, c in zip(probes, lib_codes):
        assert oracle.e2m1_round(x) == int(c), x


def test_e4m3_against_ml_dtypes(oracle):
    """E4M3 decode of all 256 codes and RNE of every midpoint and random in-range values agree
    with ml_dtypes' float8_e4m3fn; above 448 the oracle saturates (satfinite)."""
    lib_vals = np.arange(256, dtype=np.uint8).view(ml_dtypes.float8_e4m3fn).astype(np.float64)
    ours = np.array([oracle.e4m3_value(c) for c in range(256)])
    nan = np.isnan(lib_vals)
    assert np.array_equal(np.isnan(ours), nan)
    assert np.array_equal(ours[~nan], lib_vals[~nan])
    pos = lib_vals[:127]
    mids = (pos[1:] + pos[:-1]) / 2
    rnd = synth.rng(2).uniform(0, 448, 4000)
    tiny = synth.rng(3).uniform(0, 2.0 ** -6, 2000)
    probes = np.concatenate([pos, mids, rnd, tiny]).astype(np.float32)
    lib_codes = probes.astype(ml_dtypes.float8_e4m3fn).view(np.uint8)
    for x, c in zip(probes, lib_codes):
        assert oracle.e4m3_round(float(x)) == int(c), x
    for x in (448.0, 455.0, 464.0, 1e6):
        assert oracle.e4m3_round(x) == 0x7E


def _codes_nibbles(codes):
    return np.stack([codes & 0xF, codes >> 4], -1).reshape(codes.shape[0], -1)


def test_nvfp4_exact_ties(oracle):
    """Block maxima and entries placed exactly on E4M3 / E2M1 rounding midpoints and one fp32
    step either side, with supplied tensor scales that make the divisors exact ("Convert BF16
    to NVFP4 yourself": E4M3 block scales, E2M1 codes; round to nearest even): the decisions
    there are those of ml_dtypes' RNE casts, saturating at 448 and 6.  Random data never lands
    this close to a boundary, so a slightly wrong quotient or tie rule shows only here."""
    up, dn = (lambda v: np.nextafter(np.float32(v), np.float32(np.inf))), \
             (lambda v: np.nextafter(np.float32(v), np.float32(0)))
    # block scales: s_t = fp32(1/6) makes d = fl32(6 s_t) = 1, so the scale is E4M3(bmax)
    e4 = np.arange(0, 127, dtype=np.uint8).view(ml_dtypes.float8_e4m3fn).astype(np.float64)
    mids = (e4[1:] + e4[:-1]) / 2
    q = [m for m in mids[[1, 2, 9, 10, 40, 41, 120, 124, 125]]]
    q = np.array(q + [up(v) for v in q] + [dn(v) for v in q] + [448.0, 460.0, 464.0, 1e4], dtype=np.float32)
    t = np.zeros((q.size, 16), dtype=np.float32)
    t[:, 5] = q
    t[::2, 5] *= -1
    s_t = np.float32(1 / 6)
    _, scales, _ = oracle.nvfp4_encode(t, oracle.F32, tensor_scale=float(s_t))
    want = np.minimum(q, np.float32(448)).astype(ml_dtypes.float8_e4m3fn).view(np.uint8)
    assert scales[:, 0].tolist() == want.tolist()
    # codes: s_t = 1 and a block maximum of 6 give sb = 1 and divisor 1, so the code is E2M1(t)
    e2 = np.array([0.25, 0.75, 1.25, 1.75, 2.5, 3.5, 5.0], dtype=np.float32)
    v = np.concatenate([e2, [up(x) for x in e2], [dn(x) for x in e2], [6.0, 0.0]]).astype(np.float32)
    v = np.concatenate([v, -v])
    v = np.concatenate([v, np.zeros((-v.size) % 15, np.float32)]).reshape(-1, 15)
    t = np.concatenate([np.full((v.shape[0], 1), 6.0, np.float32), v], axis=1)
    codes, scales, _ = oracle.nvfp4_encode(t, oracle.F32, tensor_scale=1.0)
    assert np.all(scales == 0x38)  # E4M3 1.0
    mag = np.minimum(np.abs(t), np.float32(6)).astype(ml_dtypes.float4_e2m1fn).view(np.uint8)
    want = mag | (np.signbit(t).astype(np.uint8) << 3)
    assert np.array_equal(_codes_nibbles(codes), want)


def test_nvfp4_error_bound(oracle):
    """Every code is the nearest E2M1 point to |t| / (dec(sb) s_t) (the format's rounding
    bound: at most half a grid step away), and the block scale maps the block maximum close to
    6 (within E4M3's relative half step, 1/16)."""
    g = synth.rng(4)
    x = synth.normal(g, (16, 128)) * np.exp(synth.normal(g, (16, 1)))  # rows of varied scale
    t = synth.as_storage(x, "bf16")
    codes, scales, ts = oracle.nvfp4_encode(t, oracle.BF16)
    tf = synth.bf16_bits_to_f32(t).astype(np.float64)
    assert np.float32(ts) == np.float32(np.float32(np.abs(tf).max()) / np.float32(2688.0))
    sb = np.array([[oracle.e4m3_value(c) for c in row] for row in scales])
    nib = _codes_nibbles(codes)
    grid = np.array([oracle.e2m1_value(c) for c in range(8)])
    q = np.abs(tf) / (np.repeat(sb, 16, axis=1) * np.float64(ts))
    dist = np.abs(grid[nib & 7] - q)
    step = np.where(q < 2, 0.5, np.where(q < 4, 1.0, 2.0))
    assert np.all(dist <= step / 2 + 1e-6)
    assert np.array_equal(nib >> 3, np.signbit(tf).astype(np.int64))
    bmax = np.abs(tf).reshape(16, -1, 16).max(-1)
    ratio = bmax / (sb * 6 * np.float64(ts))
    assert np.all(np.abs(ratio - 1) <= 1 / 16 + 1e-6)


def test_nvfp4_negative_zero_kept(oracle):
    """'keeping FP4 negative zero' (the bit-exact check): a negative value that rounds to zero,
    and -0 itself, keep the sign bit."""
    t = np.zeros((1, 16), np.float32)
    t[0, 0] = 1.0
    t[0, 1] = -1e-9
    t[0, 2] = -0.0
    codes, scales, ts = oracle.nvfp4_encode(t, oracle.F32)
    nib = _codes_nibbles(codes)[0]
    assert nib[1] == 0x8 and nib[2] == 0x8 and nib[3] == 0x0
    assert nib[0] == 0x7 and scales[0, 0] == 0x7E  # 1.0 -> 6 * 448 * s_t


def test_nvfp4_all_zero_and_supplied_scale(oracle):
    t = np.zeros((2, 32), np.float32)
    t[1, 5] = -0.0
    codes, scales, ts = oracle.nvfp4_encode(t, oracle.F32)
    assert ts == 0 and not scales.any() and _codes_nibbles(codes)[1, 5] == 8
    x = synth.normal(synth.rng(9), (4, 64)).astype(np.float32)
    own = oracle.nvfp4_encode(x, oracle.F32)
    shared = oracle.nvfp4_encode(x, oracle.F32, tensor_scale=float(own[2]))
    assert all(np.array_equal(a, b) for a, b in zip(own[:2], shared[:2]))
    # a shared scale taken from a larger partner tensor ('The shared global scale') changes
    # the block scales of this one but not its sizes
    big = oracle.nvfp4_encode(x, oracle.F32, tensor_scale=float(own[2]) * 8)
    assert big[2] == np.float32(own[2]) * 8 and not np.array_equal(big[1], own[1])
    # a scale far too small saturates codes at 6 and block scales at 448
    tiny = oracle.nvfp4_encode(x, oracle.F32, tensor_scale=float(own[2]) / 1e4)
    assert (tiny[1] == 0x7E).all()


def test_nvfp4_requantisation_is_stable(oracle):
    """'Bit-exact check': decode, re-quantise, compare byte for byte -> packed codes and block
    scales identical; the re-estimated global scale may move by about one ULP (decoding
    cannot recover the original extremes).  Checked with fp32 and bf16 decodes."""
    g = synth.rng(10)
    for trial in range(4):
        x = synth.normal(g, (32, 256)) * (0.02 if trial % 2 else 1.0)
        t = synth.as_storage(x, "bf16")
        codes, scales, ts = oracle.nvfp4_encode(t, oracle.BF16)
        dec = oracle.nvfp4_decode(codes, scales, ts)
        re32 = oracle.nvfp4_encode(dec.astype(np.float32), oracle.F32)
        assert np.array_equal(re32[0], codes) and np.array_equal(re32[1], scales)
        assert abs(int(np.float32(re32[2]).view(np.int32)) - int(np.float32(ts).view(np.int32))) <= 1
        re16 = oracle.nvfp4_encode(synth.as_storage(dec, "bf16"), oracle.BF16)
        assert np.array_equal(re16[0], codes) and np.array_equal(re16[1], scales)


def test_amax_survives_pruning(oracle):
    """The largest |w| of every group is always kept, so the tensor scale of the compressed
    values equals the tensor scale of the dense weight."""
    g = synth.rng(12)
    w = synth.draw(g, (64, 512), "bf16", 0.02)
    vals, _ = oracle.compress_24(w, oracle.BF16)
    assert oracle.nvfp4_tensor_scale(vals, oracle.BF16) == oracle.nvfp4_tensor_scale(w, oracle.BF16)


def test_group_tensor_scale_closed_form(oracle):
    """'The shared global scale': a group's scale comes from the largest |t| of all its tensors.
    The largest magnitude 2688 = 6 * 448 (exact in bf16) sits in the second tensor, so the
    group's scale is exactly 1.0 and each tensor alone would get a smaller one."""
    a = synth.as_storage(np.array([[1.0, -2.0, 0.5, 3.0] * 4]), "bf16")
    b = synth.as_storage(np.array([[0.0] * 15 + [-2688.0]]), "bf16")
    assert oracle.nvfp4_group_tensor_scale([a, b], oracle.BF16) == 1.0
    assert oracle.nvfp4_tensor_scale(a, oracle.BF16) == np.float32(3.0) / np.float32(2688.0)
    assert oracle.nvfp4_group_tensor_scale([], oracle.BF16) == 0.0


def test_group_tensor_scale_is_max_of_members(oracle):
    """Division by the positive constant 2688 with round-to-nearest is monotone, so the group's
    scale equals the largest of the members' own scales, for every storage type."""
    g = synth.rng(41)
    for dt, od in (("f16", oracle.F16), ("bf16", oracle.BF16), ("f32", oracle.F32)):
        ts = [synth.draw(g, (int(g.integers(1, 9)), 16 * int(g.integers(1, 5))), dt, float(sig))
              for sig in (0.02, 1.0, 0.3)]
        own = [np.float32(oracle.nvfp4_tensor_scale(t, od)) for t in ts]
        assert oracle.nvfp4_group_tensor_scale(ts, od) == max(own)


def test_group_tensor_scale_skips_nan(oracle):
    """NaN compares false, so it never becomes the maximum (the group scale of the rest)."""
    x = synth.normal(synth.rng(42), (4, 32)).astype(np.float32)
    y = x.copy()
    y[2, 7] = np.nan
    assert oracle.nvfp4_group_tensor_scale([y, x[:1]], oracle.F32) == oracle.nvfp4_tensor_scale(x, oracle.F32)


def test_output_head_generator_matches_one_draw():
    """Drawing the head in row chunks continues one stream: identical to a single draw."""
    d = synth.output_head(vocab=10, hidden=16, rows_per_draw=3)
    assert np.array_equal(d["W"], synth.draw(synth.rng(0), (10, 16), "bf16", 0.02))


# ----------------------------------------------------------------------------- GEMM

def test_gemm_matches_library_matmul(oracle):
    g = synth.rng(13)
    X = synth.normal(g, (7, 40))
    W = synth.normal(g, (9, 40))
    Y, S = oracle.gemm(X, W)
    assert np.allclose(Y, X @ W.T, rtol=1e-13, atol=1e-13)
    assert np.allclose(S, np.abs(X) @ np.abs(W).T, rtol=1e-13)
    # orientation: a one-hot X row selects column k of W, i.e. Y[m, n] = W[n, k]
    E = np.zeros((1, 40))
    E[0, 3] = 1.0
    assert np.array_equal(oracle.gemm(E, W)[0][0], W[:, 3])


def test_sparse_gemm_equals_dense_on_pruned(oracle):
    """Summing over kept entries via the metadata equals the dense sum over the pruned weight
    exactly in fp64 (the pruned entries are exact zeros)."""
    g = synth.rng(14)
    w = synth.draw(g, (24, 64), "f16")
    x = synth.draw(g, (5, 64), "f16")
    vals, meta = oracle.compress_24(w, oracle.F16)
    pruned = oracle.prune_24(w, oracle.F16)
    X = oracle.to_double(x, oracle.F16)
    Ys, Ss = oracle.gemm_sparse(X, oracle.to_double(vals, oracle.F16), meta)
    Yd, Sd = oracle.gemm(X, oracle.to_double(pruned, oracle.F16))
    assert np.array_equal(Ys, Yd) and np.array_equal(Ss, Sd)
    assert np.allclose(Yd, X @ oracle.to_double(pruned, oracle.F16).T, rtol=1e-12, atol=1e-12)


def test_sparse_gemm_nvfp4_values(oracle):
    """Sparse NVFP4 (reading: one block scale per 16 stored values): the product with decoded
    values through the metadata equals the dense product with the decompressed decode."""
    g = synth.rng(15)
    w = synth.draw(g, (16, 128), "bf16", 0.02)
    x = synth.draw(g, (3, 128), "bf16")
    vals, meta = oracle.compress_24(w, oracle.BF16)
    c, s, ts = oracle.nvfp4_encode(vals, oracle.BF16)
    V = oracle.nvfp4_decode(c, s, ts)
    Wd = np.zeros((16, 128))
    nib = np.stack([meta & 0xF, meta >> 4], 1).ravel()
    for gi in range(16 * 32):
        n, j = divmod(gi, 32)
        Wd[n, 4 * j + (nib[gi] & 3)] = V[n, 2 * j]
        Wd[n, 4 * j + (nib[gi] >> 2)] = V[n, 2 * j + 1]
    X = oracle.to_double(x, oracle.BF16)
    Ys, _ = oracle.gemm_sparse(X, V, meta)
    assert np.allclose(Ys, X @ Wd.T, rtol=1e-12, atol=1e-15)


def test_moe_matches_per_token_matmul(oracle):
    g = synth.rng(16)
    E, N, K, T, topk = 6, 8, 32, 5, 3
    W = synth.normal(g, (E, N, K))
    X = synth.normal(g, (T, K))
    r = synth.routing_topk(g, T, E, topk)
    Y, S = oracle.moe(X, r, W)
    for t in range(T):
        for s in range(topk):
            assert np.allclose(Y[t, s], W[r[t, s]] @ X[t], rtol=1e-13, atol=1e-13)
            assert np.allclose(S[t, s], np.abs(W[r[t, s]]) @ np.abs(X[t]), rtol=1e-13)
    with pytest.raises(oracle.OracleError):
        oracle.moe(X, np.full((T, topk), E, np.int32), W)


def test_routing_generator_distinct():
    g = synth.rng(0)
    r = synth.routing_topk(g, 200, 512, 10)
    assert all(len(set(row)) == 10 for row in r.tolist())
    assert r.min() >= 0 and r.max() < 512


def test_tolerance_rule(oracle):
    ok = oracle.within_tolerance(np.array([1.0005, 0.0, 1e-9]), np.array([1.0, 0.0, 0.0]),
                                 np.array([1.0, 0.0, 0.0]))
    assert ok.tolist() == [True, True, False]


def test_moe_generator_matches_one_draw():
    """Drawing experts one by one continues the same stream: identical to one [E, N, K] draw."""
    d = synth.moe(E=3, N=4, K=16, T=5, topk=2)
    g = synth.rng(0)
    W = synth.draw(g, (3, 4, 16), "bf16", 0.02)
    X = synth.draw(g, (5, 16), "bf16")
    assert np.array_equal(d["W"], W) and np.array_equal(d["X"], X)


# ----------------------------------------------------------------------------- expert block


def test_moe_block_hand_example(oracle):
    """A hand-computed block: x = [1, 2]; gate row [1, 0] gives g = 1, up row [0, 1] gives u = 2,
    so h = SiLU(1) * 2 = 2 / (1 + e^-1) = 1.46211716..., held in bf16 as 1.4609375 (8 significant
    bits: 1 + 59/128); down rows [3] and [-1], router weight 0.5: y = [2.19140625, -0.73046875]."""
    X = np.array([[1.0, 2.0]])
    Wg = np.array([[[1.0, 0.0]]])
    Wu = np.array([[[0.0, 1.0]]])
    Wd = np.array([[[3.0], [-1.0]]])
    Y, S = oracle.moe_block(X, np.array([[0]]), np.array([[0.5]]), Wg, Wu, Wd, oracle.BF16)
    assert Y.tolist() == [[2.19140625, -0.73046875]]
    assert S.tolist() == [[2.19140625, 0.73046875]]
    # in f16 h keeps 11 bits: 1.4619140625 (1 + 473/1024)
    Y16, _ = oracle.moe_block(X, np.array([[0]]), np.array([[1.0]]), Wg, Wu, Wd, oracle.F16)
    assert Y16.tolist() == [[3 * 1.4619140625, -1.4619140625]]
    # a negative h: gate row [-1, 0] gives g = -1, h = 2 SiLU(-1) = -2 / (1 + e) = -0.53788284...,
    # in bf16 -0.5390625 (1 + 10/128 times 2^-1); the tolerance scale takes |h|
    Yn, Sn = oracle.moe_block(X, np.array([[0]]), np.array([[0.5]]), -Wg, Wu, Wd, oracle.BF16)
    assert Yn.tolist() == [[-0.80859375, 0.26953125]]
    assert Sn.tolist() == [[0.80859375, 0.26953125]]


def test_moe_block_silu_zero_and_linearity(oracle):
    """SiLU(0) = 0: a zero gate row silences its feature whatever up and down hold; y is linear in
    the router weights, and two slots on one expert add."""
    g = synth.rng(43)
    X = synth.normal(g, (3, 8))
    Wg, Wu, Wd = synth.normal(g, (2, 4, 8)), synth.normal(g, (2, 4, 8)), synth.normal(g, (2, 8, 4))
    Wg0 = Wg.copy()
    Wg0[:, 1] = 0.0
    Wd1 = Wd.copy()
    Wd1[:, :, 1] += 100.0  # only feature 1 reads these columns
    rt = np.array([[0, 1], [1, 1], [0, 0]])
    rw = synth.normal(g, (3, 2))
    a, _ = oracle.moe_block(X, rt, rw, Wg0, Wu, Wd, oracle.F16)
    b, _ = oracle.moe_block(X, rt, rw, Wg0, Wu, Wd1, oracle.F16)
    assert np.array_equal(a, b)
    c, _ = oracle.moe_block(X, rt, 2 * rw, Wg, Wu, Wd, oracle.F16)
    d, _ = oracle.moe_block(X, rt, rw, Wg, Wu, Wd, oracle.F16)
    assert np.allclose(c, 2 * d, rtol=1e-15, atol=0)
    one, _ = oracle.moe_block(X[:1], np.array([[1]]), rw[1:2, :1], Wg, Wu, Wd, oracle.F16)
    two, _ = oracle.moe_block(X[:1], np.array([[1, 1]]), np.array([[rw[1, 0], rw[1, 0]]]), Wg, Wu, Wd, oracle.F16)
    assert np.allclose(two, 2 * one, rtol=1e-15, atol=0)


def test_round_to_16_against_ml_dtypes(oracle):
    """The block's 16-bit hold of h: round to nearest even, checked against ml_dtypes' casts."""
    x = synth.normal(synth.rng(44), 4096) * np.exp(3 * synth.normal(synth.rng(45), 4096))
    # exact ties between neighbours, which random draws almost never hit: to the even neighbour
    # (1 + 2^-8 -> 1, 1 + 3 2^-8 -> 1 + 2^-6 in bf16; 1 + 2^-11 -> 1, 1 + 3 2^-11 -> 1 + 2^-9 in f16)
    ties = np.array([1 + 2.0 ** -8, 1 + 3 * 2.0 ** -8, 1 + 2.0 ** -11, 1 + 3 * 2.0 ** -11])
    x = np.concatenate([x, ties, -ties, ties * 2.0 ** -20])
    bf = np.asarray(x.astype(np.float32).astype(ml_dtypes.bfloat16), dtype=np.float64)
    assert np.array_equal(oracle.round_to_16(x, oracle.BF16), bf)
    assert np.array_equal(oracle.round_to_16(x, oracle.F16), x.astype(np.float16).astype(np.float64))
    assert oracle.round_to_16(ties[:2], oracle.BF16).tolist() == [1.0, 1 + 2.0 ** -6]
    assert oracle.round_to_16(ties[2:], oracle.F16).tolist() == [1.0, 1 + 2.0 ** -9]



# ----------------------------------------------------------------------------- pairwise 4:8

_PAIR_NIBBLES = {0x4, 0x8, 0xC, 0x9, 0xD, 0xE}  # i0 | i1 << 2 for the six pairs i0 < i1


def _nibbles(meta, n):
    return np.stack([meta & 0xF, meta >> 4], 1).ravel()[:n]


def test_pairwise48_brute_force(oracle):
    """Keeping the two pairs of largest |a| + |b| ('What 2:4 actually is': the largest magnitudes
    survive, here per pair of entries) is the choice, among the six of 2 of 4 pairs, that keeps
    the most total magnitude.  fp16 entries of distinct pair sums make the maximiser unique, and
    their fp32 sums are exact."""
    g = synth.rng(41)
    w = f16(synth.normal(g, (48, 128)))
    pair = np.abs(w.astype(np.float64)).reshape(-1, 4, 2).sum(axis=2)
    vals, meta = oracle.compress_48(w, oracle.F16)
    nib = _nibbles(meta, pair.shape[0])
    choices = list(itertools.combinations(range(4), 2))
    checked = 0
    for c in range(pair.shape[0]):
        if len(set(pair[c].tolist())) < 4:
            continue
        totals = [pair[c][i] + pair[c][j] for i, j in choices]
        i0, i1 = choices[int(np.argmax(totals))]
        assert (nib[c] & 3, nib[c] >> 2) == (i0, i1), c
        src = w.reshape(-1, 8)[c].view(np.uint16)
        assert np.array_equal(vals.reshape(-1, 4)[c].view(np.uint16), src[[2 * i0, 2 * i0 + 1, 2 * i1, 2 * i1 + 1]])
        checked += 1
    assert checked > 700


def test_pairwise48_ties_nan_and_fp32_score(oracle):
    """Ties go to the lower pair; a NaN pair ranks above every number; the score is one fp32
    addition, so 1 + 2^-30 ties with 1 (the lower pair wins, although the exact sum is larger)."""
    cases = {
        (0, 0, 0, 0, 0, 0, 0, 0): (0, 1),
        (0, 0, 0, 0, 0, 0, 3, 0): (0, 3),
        (1, 1, 2, 0, -2, 0, 0, 1): (0, 1),
        (1, 1, 2, 0, -2, 0, 0, 3): (0, 3),
        (1, 2, 0, 0, 3, -4, 0.5, 0): (0, 2),
        (0, 0, 0, 1, 0, 0, 1, 0): (1, 3),
    }
    for v, pair in cases.items():
        _, m = oracle.compress_48(f16(v).reshape(1, 8), oracle.F16)
        assert (m[0] & 3, m[0] >> 2) == pair, v
    _, m = oracle.compress_48(f16([1, 1, 0, np.nan, 5, 5, 0, 0]).reshape(1, 8), oracle.F16)
    assert (m[0] & 3, m[0] >> 2) == (1, 2)
    _, m = oracle.compress_48(f16([0, 0, np.inf, 0, 1, np.nan, np.inf, 1]).reshape(1, 8), oracle.F16)
    assert (m[0] & 3, m[0] >> 2) == (1, 2)  # NaN first, then inf against inf + 1 = inf: lower pair
    x = np.array([1, 0, 1, 2.0 ** -30, 5, 0, 0, 0], np.float32).reshape(1, 8)
    assert np.float32(1) + np.float32(2.0 ** -30) == np.float32(1)
    _, m = oracle.compress_48(x, oracle.F32)
    assert (m[0] & 3, m[0] >> 2) == (0, 2)


def test_pairwise48_check(oracle):
    """A chunk of 8 is eligible when at most two of its four pairs hold a nonzero (-0 is zero);
    a chunk that passes 2:4 can fail pairwise 4:8 and the other way round."""
    v = {
        "two_pairs": ([1, 2, 0, 0, 3, 4, 0, 0], 1),
        "three_pairs": ([1, 0, 0, 2, 0, 0, 3, 0], 0),
        "negzero": ([1, 0, -0.0, -0.0, 0, 0, 0, 5], 1),
        "24_ok_48_fail": ([1, 0, 0, 2, 3, 0, 0, 4], 0),
        "48_ok_24_fail": ([1, 2, 3, 4, 0, 0, 0, 0], 1),
    }
    for name, (x, ok) in v.items():
        p, n = oracle.check_48(f16(x).reshape(1, 8), oracle.F16)
        assert p.ravel().tolist() == [ok] and n == 1 - ok, name
    assert oracle.check_24(f16(v["24_ok_48_fail"][0]).reshape(1, 8), oracle.F16)[1] == 0
    assert oracle.check_24(f16(v["48_ok_24_fail"][0]).reshape(1, 8), oracle.F16)[1] == 1
    with pytest.raises(oracle.OracleError):
        oracle.check_48(f16(np.zeros(12)).reshape(1, 12), oracle.F16)


def test_pairwise48_roundtrip(oracle):
    """decompress(compress(W)) keeps the two chosen pairs bitwise and zeroes the other two; the
    result passes the check in every chunk; its compress gives back the same values and meta;
    every nibble names two ascending pairs; values take K/2 and meta K/16 bytes per row."""
    g = synth.rng(42)
    for dt, st in ((oracle.F16, "f16"), (oracle.BF16, "bf16"), (oracle.F32, "f32")):
        w = synth.structured_edge(g, 24, 96, st)
        vals, meta = oracle.compress_48(w, dt)
        assert vals.shape == (24, 48) and meta.size == 24 * 96 // 16
        back = oracle.decompress_48(vals, meta, dt, w.shape)
        nib = _nibbles(meta, 24 * 12)
        assert set(np.unique(nib).tolist()) <= _PAIR_NIBBLES
        bw, sw = back.reshape(-1, 4, 2).view(np.uint8), w.reshape(-1, 4, 2).view(np.uint8)
        for c in range(nib.size):
            kept = {nib[c] & 3, nib[c] >> 2}
            for j in range(4):
                assert np.array_equal(bw[c, j], sw[c, j] if j in kept else np.zeros_like(sw[c, j]))
        p, n = oracle.check_48(back, dt)
        assert n == 0 and p.all()
        v2, m2 = oracle.compress_48(back, dt)
        assert np.array_equal(v2.view(np.uint8), vals.view(np.uint8)) and np.array_equal(m2, meta)


def test_pairwise48_odd_chunk_count_and_illegal_nibble(oracle):
    """An odd number of chunks leaves the high nibble of the last meta byte zero; a nibble with
    pair indices out of order is rejected."""
    w = f16(np.arange(1, 9)).reshape(1, 8)
    vals, meta = oracle.compress_48(w, oracle.F16)
    assert meta.tolist() == [0xE] and vals.astype(np.float64).tolist() == [[5, 6, 7, 8]]
    with pytest.raises(oracle.OracleError):
        oracle.decompress_48(vals, np.array([0x6], np.uint8), oracle.F16, (1, 8))


# ----------------------------------------------------------------------------- NVFP4, 32-entry blocks

def test_block32_against_ml_dtypes(oracle):
    """The 32-entry block form (the activation operand of the sparse FP4 MMA) written out with
    numpy and ml_dtypes' RNE casts: block scale = E4M3(fp32(bmax32 / fp32(6 s_t))), code =
    E2M1(fp32(|t| / fp32(dec(sb) s_t))) with the sign bit, every step in fp32."""
    g = synth.rng(44)
    x = synth.normal(g, (12, 256)) * np.exp(synth.normal(g, (12, 1)))
    t = synth.as_storage(x, "bf16")
    codes, scales, ts = oracle.nvfp4_encode(t, oracle.BF16, block=32)
    assert codes.shape == (12, 128) and scales.shape == (12, 8)
    tf = synth.bf16_bits_to_f32(t).astype(np.float32)
    s_t = np.float32(np.abs(tf).max()) / np.float32(2688)
    assert np.float32(ts) == s_t
    d = np.float32(s_t * np.float32(6))
    bmax = np.abs(tf).reshape(12, 8, 32).max(-1)
    sb = (bmax / d).astype(np.float32).astype(ml_dtypes.float8_e4m3fn)
    assert np.array_equal(scales, sb.view(np.uint8))
    sc = (sb.astype(np.float32) * s_t).astype(np.float32)
    q = (np.abs(tf).reshape(12, 8, 32) / sc[..., None]).astype(np.float32)
    mag = np.minimum(q, np.float32(6)).astype(ml_dtypes.float4_e2m1fn).view(np.uint8).reshape(12, 256)
    want = mag | (np.signbit(tf).astype(np.uint8) << 3)
    assert np.array_equal(_codes_nibbles(codes), want)


def test_block32_equals_block16_when_halves_share_their_max(oracle):
    """When both 16-halves of every 32-block have the same largest magnitude, the two block
    sizes give the same codes, and each block-32 scale is the shared scale of its two halves."""
    g = synth.rng(45)
    x = synth.normal(g, (6, 128))
    x.reshape(6, 4, 2, 16)[..., 1, 3] = np.abs(x.reshape(6, 4, 2, 16)).max(axis=(2, 3)) * 1.5
    x.reshape(6, 4, 2, 16)[..., 0, 7] = -x.reshape(6, 4, 2, 16)[..., 1, 3]
    t = x.astype(np.float32)
    c16, s16, ts16 = oracle.nvfp4_encode(t, oracle.F32)
    c32, s32, ts32 = oracle.nvfp4_encode(t, oracle.F32, block=32)
    assert ts16 == ts32 and np.array_equal(c16, c32)
    assert np.array_equal(s16[:, 0::2], s32) and np.array_equal(s16[:, 1::2], s32)
    d32 = oracle.nvfp4_decode(c32, s32, ts32, block=32)
    assert np.array_equal(d32, oracle.nvfp4_decode(c16, s16, ts16))


def test_block32_shape_rules(oracle):
    with pytest.raises(oracle.OracleError):
        oracle.nvfp4_encode(np.zeros((1, 48), np.float32), oracle.F32, block=32)
    with pytest.raises(oracle.OracleError):
        oracle.nvfp4_encode(np.zeros((1, 64), np.float32), oracle.F32, block=8)


# ----------------------------------------------------------------------------- input decoding

def _same_doubles(got, want):
    """Equal as numbers, NaN where the other is NaN, and the sign of zero kept."""
    nan = np.isnan(want)
    assert np.array_equal(np.isnan(got), nan)
    assert np.array_equal(got[~nan], want[~nan])
    assert np.array_equal(np.signbit(got[~nan]), np.signbit(want[~nan]))


def test_to_double_f16_every_pattern(oracle):
    """Every GEMM parity check decodes its inputs through to_double.  For IEEE binary16 the
    value of each of the 65,536 patterns is fixed by the format (subnormals f * 2^-24, inf,
    NaN, signed zero); numpy's own half -> double cast is the independent check."""
    bits = np.arange(1 << 16, dtype=np.uint32).astype(np.uint16)
    _same_doubles(oracle.to_double(bits.view(np.float16), oracle.F16),
                  bits.view(np.float16).astype(np.float64))


def test_to_double_bf16_every_pattern(oracle):
    """bfloat16 is the upper half of a binary32; ml_dtypes' bfloat16 -> double cast (its own
    implementation, not the oracle's) must agree on all 65,536 patterns."""
    bits = np.arange(1 << 16, dtype=np.uint32).astype(np.uint16)
    _same_doubles(oracle.to_double(bits, oracle.BF16),
                  bits.view(ml_dtypes.bfloat16).astype(np.float64))


def test_to_double_f32_passthrough(oracle):
    """fp32 entries widen exactly (a sample of patterns across every exponent)."""
    g = np.random.default_rng(7)
    bits = g.integers(0, 1 << 32, size=1 << 16, dtype=np.uint64).astype(np.uint32)
    with np.errstate(invalid="ignore"):
        want = bits.view(np.float32).astype(np.float64)
    _same_doubles(oracle.to_double(bits.view(np.float32), oracle.F32), want)

"""Seeded synthetic inputs shared by the tests, the benchmark and the oracle checks.

This module holds no step of the method: it only draws numbers and casts them to storage
types.  Recipe (the same everywhere):

* numpy ``default_rng(seed)`` (PCG64), ``standard_normal`` in float64, multiplied by sigma;
* cast to fp16 with numpy's round-to-nearest-even; to bf16 by rounding the float32 value
  (itself round-to-nearest from float64) to its upper 16 bits, nearest-even;
* draws happen in the order the workload lists its tensors.

Workloads (the shapes the pages' workloads take; see the design notes for the mapping):

* ``fp16_toy``:      W fp16 [256, 512] then X fp16 [16, 512], N(0, 1).
* ``decode_nvfp4``:  X bf16 [8, 5120] N(0, 1), then W bf16 [5120, 5120] N(0, 0.02).
* ``prefill_w4a4``:  X then W, bf16 [4096, 4096], N(0, 1).
* ``moe``:           W bf16 [512, 512, 2048] N(0, 0.02), X bf16 [4096, 2048] N(0, 1), then
                     routing int32 [4096, 10]: ten distinct experts per token, uniform
                     without replacement.
* ``moe_skewed``:    W bf16 [E, N, K] N(0, 0.02), X [T, K] N(0, 1), routing with given per-expert
                     row counts in a seeded random order (tile-boundary parity cases).
* ``moe_block``:     Wg, Wu bf16 [E, F, H], Wd bf16 [E, H, F] N(0, 0.02) expert by expert, X bf16
                     [T, H] N(0, 1), top-k routing, router weights uniform normalised per token.
* ``output_head``:   W bf16 [151936, 4096] N(0, 0.02) (an output head of ~1.16 GiB: the pages'
                     large single-tensor quantisation), drawn in row chunks.
* ``qkv_group``:     Wq [2048, 2048], Wk, Wv [512, 2048] N(0, 0.02), one x40 outlier in Wv (a
                     group sharing one NVFP4 tensor scale).
* ``msweep``:        W [5120, 5120] then X [M, 5120], N(0, 1), fp16 or bf16.
* ``conv_fail5``:    W fp16 [256, 256, 3, 3] N(0, 1) with a 2-of-4 zero pattern along C
                     drawn at random per group, then round(5%) of the groups (a seeded
                     permutation) given one zeroed slot back -> exactly one zero -> fail.
"""
from __future__ import annotations

import numpy as np

SEED = 0


def rng(seed: int = SEED) -> np.random.Generator:
    return np.random.default_rng(seed)


def f32_to_bf16_bits(x: np.ndarray) -> np.ndarray:
    """float32 -> bf16 bit patterns (uint16), round to nearest even; NaN stays NaN."""
    u = np.ascontiguousarray(x, dtype=np.float32).view(np.uint32).astype(np.uint64)
    nan = np.isnan(np.asarray(x, dtype=np.float32))
    r = (u + 0x7FFF + ((u >> 16) & 1)) >> 16
    r = np.where(nan, (u >> 16) | 0x40, r)
    return r.astype(np.uint16)


def bf16_bits_to_f32(b: np.ndarray) -> np.ndarray:
    return (np.asarray(b, dtype=np.uint16).astype(np.uint32) << 16).view(np.float32)


def normal(g: np.random.Generator, shape, sigma: float = 1.0) -> np.ndarray:
    return g.standard_normal(size=shape) * sigma


def as_storage(x64: np.ndarray, dtype: str) -> np.ndarray:
    """Cast float64 draws to storage: 'f16' -> float16, 'bf16' -> uint16 bits, 'f32'."""
    if dtype == "f16":
        return x64.astype(np.float16)
    if dtype == "bf16":
        return f32_to_bf16_bits(x64.astype(np.float32))
    if dtype == "f32":
        return x64.astype(np.float32)
    raise ValueError(dtype)


def draw(g: np.random.Generator, shape, dtype: str, sigma: float = 1.0) -> np.ndarray:
    return as_storage(normal(g, shape, sigma), dtype)


# ------------------------------------------------------------------ workloads

def fp16_toy(seed: int = SEED):
    g = rng(seed)
    W = draw(g, (256, 512), "f16")
    X = draw(g, (16, 512), "f16")
    return {"W": W, "X": X}


def decode_nvfp4(seed: int = SEED, M: int = 8, N: int = 5120, K: int = 5120):
    g = rng(seed)
    X = draw(g, (M, K), "bf16")
    W = draw(g, (N, K), "bf16", 0.02)
    return {"X": X, "W": W}


def prefill_w4a4(seed: int = SEED, M: int = 4096, N: int = 4096, K: int = 4096):
    g = rng(seed)
    X = draw(g, (M, K), "bf16")
    W = draw(g, (N, K), "bf16")
    return {"X": X, "W": W}


def routing_topk(g: np.random.Generator, T: int, E: int, topk: int) -> np.ndarray:
    """Per token, `topk` distinct experts uniform without replacement (argsort of uniforms)."""
    u = g.random(size=(T, E))
    return np.argsort(u, axis=1, kind="stable")[:, :topk].astype(np.int32)


def moe(seed: int = SEED, E: int = 512, N: int = 512, K: int = 2048, T: int = 4096,
        topk: int = 10):
    """Expert weights are drawn one expert after the other from the stream (the same numbers a
    single [E, N, K] draw gives), which keeps the float64 temporary at one expert."""
    g = rng(seed)
    W = np.empty((E, N, K), dtype=np.uint16)
    for e in range(E):
        W[e] = draw(g, (N, K), "bf16", 0.02)
    X = draw(g, (T, K), "bf16")
    routing = routing_topk(g, T, E, topk)
    return {"W": W, "X": X, "routing": routing}


def output_head(seed: int = SEED, vocab: int = 151936, hidden: int = 4096, sigma: float = 0.02,
                rows_per_draw: int = 8192):
    """W bf16 [vocab, hidden] N(0, sigma), drawn in row chunks from one stream (the same numbers
    a single draw gives) so the float64 temporary stays at one chunk."""
    g = rng(seed)
    W = np.empty((vocab, hidden), dtype=np.uint16)
    for r in range(0, vocab, rows_per_draw):
        n = min(rows_per_draw, vocab - r)
        W[r:r + n] = draw(g, (n, hidden), "bf16", sigma)
    return {"W": W}


def qkv_group(seed: int = SEED, hidden: int = 2048, kv: int = 512, dtype: str = "bf16"):
    """Three projection weights read together: Wq [hidden, hidden], Wk and Wv [kv, hidden],
    N(0, 0.02), drawn in that order; Wv gets one outlier (x 40 at a seeded place) so the
    group's largest magnitude sits in the last tensor."""
    g = rng(seed)
    Wq = normal(g, (hidden, hidden), 0.02)
    Wk = normal(g, (kv, hidden), 0.02)
    Wv = normal(g, (kv, hidden), 0.02)
    i = int(g.integers(0, Wv.size))
    Wv.flat[i] *= 40.0
    return {"Wq": as_storage(Wq, dtype), "Wk": as_storage(Wk, dtype), "Wv": as_storage(Wv, dtype)}


def moe_block(seed: int = SEED, E: int = 512, H: int = 2048, F: int = 512, T: int = 4096, topk: int = 10):
    """Expert block: Wg, Wu [E, F, H] and Wd [E, H, F] bf16 N(0, 0.02) (drawn in that order,
    expert by expert), X bf16 [T, H] N(0, 1), routing [T, topk] (distinct experts per token,
    uniform), router weights fp32 [T, topk]: uniform draws normalised to sum 1 per token."""
    g = rng(seed)
    Wg = np.empty((E, F, H), dtype=np.uint16)
    Wu = np.empty((E, F, H), dtype=np.uint16)
    Wd = np.empty((E, H, F), dtype=np.uint16)
    for W, shape in ((Wg, (F, H)), (Wu, (F, H)), (Wd, (H, F))):
        for e in range(E):
            W[e] = draw(g, shape, "bf16", 0.02)
    X = draw(g, (T, H), "bf16")
    routing = routing_topk(g, T, E, topk)
    r = g.random(size=(T, topk))
    r = (r / r.sum(axis=1, keepdims=True)).astype(np.float32)
    return {"Wg": Wg, "Wu": Wu, "Wd": Wd, "X": X, "routing": routing, "router_w": r}


def moe_skewed(counts, seed: int = SEED, N: int = 256, K: int = 320, topk: int = 2,
               xdtype: str = "bf16"):
    """Routing with exactly counts[e] routed rows on expert e: the flat list of expert ids in a
    seeded random order, reshaped to [T, topk] (T = sum(counts) / topk; a token may meet the
    same expert twice).  W bf16 [E, N, K] N(0, 0.02), then X [T, K] N(0, 1) in `xdtype`."""
    counts = list(counts)
    n = int(sum(counts))
    assert n % topk == 0
    g = rng(seed)
    W = draw(g, (len(counts), N, K), "bf16", 0.02)
    X = draw(g, (n // topk, K), xdtype)
    flat = np.repeat(np.arange(len(counts), dtype=np.int32), counts)
    routing = g.permutation(flat).reshape(n // topk, topk).astype(np.int32)
    return {"W": W, "X": X, "routing": routing}


def msweep(M: int, dtype: str = "f16", seed: int = SEED, N: int = 5120, K: int = 5120):
    g = rng(seed)
    W = draw(g, (N, K), dtype)
    X = draw(g, (M, K), dtype)
    return {"W": W, "X": X}


def conv_fail5(seed: int = SEED, shape=(256, 256, 3, 3), fail_frac: float = 0.05):
    """Conv weight with a random 2-of-4 zero pattern along C and round(fail_frac * G) groups
    holding exactly one zero.  Returns the tensor and the sorted failing group ids (group id
    = row-major index over [K, C/4, R, S])."""
    g = rng(seed)
    Kc, C, R, S = shape
    w = normal(g, shape).astype(np.float16)
    G = Kc * (C // 4) * R * S
    # view as [K, C/4, 4, R, S] -> [G, 4] with the four members of each group on the last axis
    grp = w.reshape(Kc, C // 4, 4, R, S).transpose(0, 1, 3, 4, 2).reshape(G, 4).copy()
    pairs = np.array([(0, 1), (0, 2), (0, 3), (1, 2), (1, 3), (2, 3)])
    keep = pairs[g.integers(0, 6, size=G)]
    mask = np.zeros((G, 4), dtype=bool)
    mask[np.arange(G), keep[:, 0]] = True
    mask[np.arange(G), keep[:, 1]] = True
    drawn = grp.copy()
    drawn[drawn == 0] = np.float16(1.0)          # a refilled slot must be nonzero
    grp = np.where(mask, grp, np.float16(0.0))
    nfail = int(round(fail_frac * G))
    failing = np.sort(g.permutation(G)[:nfail])
    first_zero = np.argmin(mask[failing], axis=1)  # lowest zeroed slot
    grp[failing, first_zero] = drawn[failing, first_zero]
    out = grp.reshape(Kc, C // 4, R, S, 4).transpose(0, 1, 4, 2, 3).reshape(shape)
    return {"W": np.ascontiguousarray(out), "failing": failing}


def structured_edge(g: np.random.Generator, rows: int, K: int, dtype: str) -> np.ndarray:
    """A matrix rich in the cases pruning and checking must get right: exact zeros of both
    signs, repeated magnitudes (ties) with mixed signs, and ordinary normal values."""
    base = normal(g, (rows, K))
    choice = g.integers(0, 6, size=(rows, K))
    ties = g.choice(np.array([0.5, 1.0, 2.0]), size=(rows, K)) * np.where(
        g.random((rows, K)) < 0.5, -1.0, 1.0)
    x = np.where(choice == 0, 0.0, base)
    x = np.where(choice == 1, -0.0, x)
    x = np.where(choice == 2, ties, x)
    x = np.where(choice == 3, np.round(base), x)   # small integers: many equal magnitudes
    return as_storage(x, dtype)


def pairwise_edge(g: np.random.Generator, rows: int, K: int, dtype: str) -> np.ndarray:
    """structured_edge for chunks of 8 along K: a third of the chunks get two of their four pairs
    zeroed (eligible for pairwise 4:8; zeros of both signs), a sixth one pair; a few entries are
    NaN or +-inf, and some pairs repeat another pair's magnitudes (score ties)."""
    x = structured_edge(g, rows, K, "f32").astype(np.float64).reshape(rows, K // 8, 4, 2)
    kind = g.integers(0, 6, size=(rows, K // 8))
    order = np.argsort(g.random((rows, K // 8, 4)), axis=2)
    sign = np.where(g.random((rows, K // 8, 4, 2)) < 0.5, -0.0, 0.0)
    for z in range(2):
        drop = (kind < 2) if z == 0 else (kind < 3)
        hit = (np.arange(4)[None, None, :] == order[:, :, z:z + 1]) & drop[:, :, None]
        x = np.where(hit[..., None], sign, x)
    tie = (kind == 4)[:, :, None, None] & (np.arange(4)[None, None, :, None] == 3)
    x = np.where(tie, -x[:, :, 0:1, :], x)                 # pair 3 repeats pair 0's magnitudes
    x = x.reshape(rows, K)
    special = g.random((rows, K))
    x = np.where(special < 0.002, np.nan, x)
    x = np.where((special >= 0.002) & (special < 0.004), np.inf, x)
    x = np.where((special >= 0.004) & (special < 0.006), -np.inf, x)
    return as_storage(x, dtype)

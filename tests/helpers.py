"""Shared test helpers: numpy <-> torch transfers and the oracle side of the pipeline."""
import numpy as np
import torch

import oracle
import synth

ORACLE_DT = {"f16": oracle.F16, "bf16": oracle.BF16, "f32": oracle.F32}


def to_dev(a: np.ndarray, dtype: str) -> torch.Tensor:
    """numpy storage (float16, bf16 bits as uint16, float32, uint8) -> CUDA tensor."""
    a = np.ascontiguousarray(a)
    if dtype == "bf16":
        return torch.from_numpy(a.view(np.int16)).view(torch.bfloat16).cuda()
    if dtype == "u8":
        return torch.from_numpy(a.astype(np.uint8)).cuda()
    return torch.from_numpy(a).cuda()


def to_host(t: torch.Tensor) -> np.ndarray:
    t = t.detach().cpu().contiguous()
    if t.dtype == torch.bfloat16:
        return t.view(torch.int16).numpy().view(np.uint16)
    return t.numpy()


def bits(a: np.ndarray) -> np.ndarray:
    """Raw bit view of a storage array, for bit-exact comparison."""
    a = np.ascontiguousarray(a)
    return a.view({1: np.uint8, 2: np.uint16, 4: np.uint32}[a.dtype.itemsize])


def f64_to_bf16_bits(v: np.ndarray) -> np.ndarray:
    """float64 -> bf16 bits with one round-to-nearest-even (normal range)."""
    v = np.asarray(v, dtype=np.float64)
    m, e = np.frexp(v)                     # v = m * 2^e, |m| in [0.5, 1)
    r = np.round(m * 256.0) / 256.0         # 8 significant bits, ties to even
    f = np.ldexp(r, e).astype(np.float32)   # exact
    return (f.view(np.uint32) >> 16).astype(np.uint16)


def oracle_decoded(t: np.ndarray, dtype: str) -> np.ndarray:
    return oracle.to_double(t, ORACLE_DT[dtype])


def assert_gemm_close(y_gpu: torch.Tensor, Y: np.ndarray, S: np.ndarray, rel: float = 1e-3):
    y = to_host(y_gpu).astype(np.float64)
    assert y.shape == Y.shape
    ok = oracle.within_tolerance(y, Y, S, rel)
    if not ok.all():
        idx = np.argwhere(~ok)[:5]
        detail = [(tuple(i), y[tuple(i)], Y[tuple(i)], S[tuple(i)]) for i in idx]
        raise AssertionError(f"{(~ok).sum()} of {ok.size} outputs outside tolerance; first: {detail}")
    # the product is not trivially zero
    assert np.abs(Y).max() == 0 or np.abs(y).max() > 0

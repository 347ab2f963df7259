"""Host logic of the per-shape dense / 2:4 choice ([P2] "Ask which sparse implementations were
actually selected"): the rule of measured crossovers, format checks, the record's reset.  No GPU."""
import pytest

import fp16_gemm_b200 as sp


@pytest.mark.parametrize("xf,wf,M,expect", [
    (sp.F16, sp.F16, 1, False), (sp.F16, sp.F16, 127, False), (sp.F16, sp.F16, 128, True),
    (sp.F16, sp.F16, 4096, True), (sp.BF16, sp.BF16, 16384, True),
    (sp.BF16, sp.NVFP4, 1, False), (sp.BF16, sp.NVFP4, 8, False), (sp.F16, sp.NVFP4, 128, True),
    (sp.F16, sp.NVFP4, 16384, True),
    (sp.NVFP4, sp.NVFP4, 16, False), (sp.NVFP4, sp.NVFP4, 4096, False),
])
def test_rule(xf, wf, M, expect):
    sp.gemm_choice_reset()
    assert sp.gemm_choice(xf, wf, M, 5120, 5120) == (expect, False)


@pytest.mark.parametrize("N,K,expect", [(256, 512, False), (1024, 1023, False), (1024, 1024, True)])
def test_rule_small_weights_stay_dense(N, K, expect):
    sp.gemm_choice_reset()
    assert sp.gemm_choice(sp.F16, sp.F16, 256, N, K) == (expect, False)


@pytest.mark.parametrize("xf,wf", [(sp.NVFP4, sp.F16), (sp.F32, sp.F16), (sp.F16, sp.F32)])
def test_rejects_pairs_without_a_sparse_path(xf, wf):
    with pytest.raises(sp.SP24Error) as e:
        sp.gemm_choice(xf, wf, 8, 64, 64)
    assert e.value.status == sp.ERR_DTYPE


def test_rejects_negative_shape():
    with pytest.raises(sp.SP24Error) as e:
        sp.gemm_choice(sp.F16, sp.F16, -1, 64, 64)
    assert e.value.status == sp.ERR_SHAPE

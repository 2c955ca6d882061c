"""e8_gemm_act_noalloc: the small-batch GEMM for callers that cannot allocate.

Callers inside CUDA graph capture, plugins whose framework owns all device
memory, and latency-critical loops cannot hand the library a freshly allocated
workspace.  This entry point uses a fixed scratch array compiled into the
library instead.  The test checks, through the C ABI, that two calls in a row
give the same result as the workspace-based e8_gemm (E8_GEMM_ACT_RHT) within
the GEMM tolerance of the other tests, and that requests larger than the fixed
scratch are refused.  It runs last (file name) and also alone in a fresh process.
"""
import numpy as np
import pytest
import torch

import decode_gemm_e8_b200 as e8
from decode_gemm_e8_b200 import synth
from tests import gpu_util as gu

pytestmark = pytest.mark.gpu

BAR = 2e-3   # relative Frobenius tolerance used by the GEMM tests


@pytest.fixture(scope="module")
def gcb():
    gu.dev()
    from decode_gemm_e8_b200 import build
    build.build()
    return e8.Codebook(0)


def test_noalloc_matches_workspace_gemm_on_two_calls(gcb):
    wl = synth.workloads()["llama_4096_b4"]
    lay = wl.layers[0]
    W = lay.weights()
    s = synth.suggest_scale(W, lay.bpw)
    i1, i2 = e8.e8_encode(gcb, gu.to_dev(W), lay.bpw, lay.rht_seed, s)
    # first call with 16 tokens, second with 5 (different padding of the scratch)
    for M, seed in ((16, wl.x_seed), (5, 77)):
        X = gu.bf16_dev(synth.activations_bf16(M, lay.K, seed))
        ref = e8.e8_gemm(gcb, X, i1, i2, lay.N, lay.K, lay.bpw, lay.rht_seed, s,
                         mode=e8.E8_GEMM_ACT_RHT)
        Y = torch.full((M, lay.N), float("nan"), device=X.device)
        e8.e8_gemm_act_noalloc(gcb, X, i1, i2, lay.N, lay.K, lay.bpw, lay.rht_seed, s, Y)
        y, r = gu.to_np(Y), gu.to_np(ref)
        assert np.all(np.isfinite(y))
        assert gu.rel_fro(y, r) < BAR
    assert e8.e8_sync_status(gcb) == e8.E8_OK


def test_noalloc_refuses_requests_beyond_its_scratch(gcb):
    # 64 tokens need 128 rows; 128 x 16384 bf16 exceeds the 1 Mi-element array
    M, N, K = 64, 128, 16384
    d = gu.dev()
    X = torch.zeros((M, K), dtype=torch.bfloat16, device=d)
    i1 = torch.zeros((N, K // 8), dtype=torch.uint16, device=d)
    Y = torch.zeros((M, N), device=d)
    with pytest.raises(e8.E8Error) as ei:
        e8.e8_gemm_act_noalloc(gcb, X, i1, None, N, K, 2, 0, 1.0, Y)
    assert ei.value.code == e8.E8_EWORKSPACE

"""e8_gemm_act_noalloc: the small-batch GEMM for callers that cannot allocate.

Plugins whose framework owns all device memory, services held to a fixed
device-memory budget, and latency-critical loops cannot hand the library a
freshly allocated workspace.  This entry point uses a fixed scratch array
compiled into the library instead, shared by every call.  The tests call it
through the C ABI, several times in a row, and compare each result with the
workspace-based e8_gemm (E8_GEMM_ACT_RHT) on the same inputs -- the same
kernels, so they must agree to the 1e-6 run-to-run bound of the int8 path --
and with the oracle's binary64 product of the decoded weights at the 2e-3
GEMM bar.  Both branches are covered: the int8 one (up to 32 tokens) and the
bf16 one (33..64 tokens), the latter after a larger call has left transformed
rows in the shared array where the smaller call needs zero padding.  Requests
larger than the fixed scratch are refused.  The file runs last (its name) and
also passes alone in a fresh process.
"""
import numpy as np
import pytest
import torch

import decode_gemm_e8_b200 as e8
from decode_gemm_e8_b200 import synth
from oracle import oracle as orc
from tests import gpu_util as gu

pytestmark = pytest.mark.gpu

BAR = 2e-3      # relative Frobenius tolerance against the oracle (GEMM tests)
REPEAT = 1e-6   # run-to-run agreement of the same kernels (partial sums in arrival order)


@pytest.fixture(scope="module")
def gcb():
    gu.dev()
    from decode_gemm_e8_b200 import build
    build.build()
    return e8.Codebook(0)


@pytest.fixture(scope="module")
def layer(gcb):
    wl = synth.workloads()["llama_4096_b4"]
    lay = wl.layers[0]
    W = lay.weights()
    s = synth.suggest_scale(W, lay.bpw)
    i1, i2 = e8.e8_encode(gcb, gu.to_dev(W), lay.bpw, lay.rht_seed, s)
    wd = orc.decode(gu.to_np(i1), gu.to_np(i2), lay.N, lay.K, lay.bpw, lay.rht_seed, s)
    return lay, s, i1, i2, wd


def _call_and_check(gcb, layer, M, seed):
    lay, s, i1, i2, wd = layer
    Xh = synth.activations_bf16(M, lay.K, seed)
    X = gu.bf16_dev(Xh)
    ref = e8.e8_gemm(gcb, X, i1, i2, lay.N, lay.K, lay.bpw, lay.rht_seed, s,
                     mode=e8.E8_GEMM_ACT_RHT)
    Y = torch.full((M, lay.N), float("nan"), device=X.device)
    e8.e8_gemm_act_noalloc(gcb, X, i1, i2, lay.N, lay.K, lay.bpw, lay.rht_seed, s, Y)
    y, r = gu.to_np(Y), gu.to_np(ref)
    assert np.all(np.isfinite(y)), M
    assert gu.rel_fro(y, r) < REPEAT, (M, gu.rel_fro(y, r))
    err = gu.rel_fro(y, orc.gemm(Xh, wd))
    assert err < BAR, (M, err)


def test_noalloc_int8_branch_two_calls(gcb, layer):
    # 16 tokens, then 5 (fewer rows: the padding of the scratch changes)
    for M, seed in ((16, 3), (5, 77)):
        _call_and_check(gcb, layer, M, seed)
    assert e8.e8_sync_status(gcb) == e8.E8_OK


def test_noalloc_bf16_branch_after_larger_call(gcb, layer):
    # 64 tokens fill 128 rows of the array; 33 tokens then need rows 66..79 to
    # be zero again, and 40 tokens use 80 rows of stale contents
    for M, seed in ((64, 5), (33, 6), (40, 7)):
        _call_and_check(gcb, layer, M, seed)
    assert e8.e8_sync_status(gcb) == e8.E8_OK


def test_noalloc_refuses_requests_beyond_its_scratch(gcb):
    # 64 tokens need 128 rows; 128 x 16384 bf16 exceeds the 2 MiB array
    M, N, K = 64, 128, 16384
    d = gu.dev()
    X = torch.zeros((M, K), dtype=torch.bfloat16, device=d)
    i1 = torch.zeros((N, K // 8), dtype=torch.uint16, device=d)
    Y = torch.zeros((M, N), device=d)
    assert e8.e8_workspace_bytes(e8.E8_GEMM_ACT_RHT, M, N, K, 2) > 2 * 1024 * 1024
    with pytest.raises(e8.E8Error) as ei:
        e8.e8_gemm_act_noalloc(gcb, X, i1, None, N, K, 2, 0, 1.0, Y)
    assert ei.value.code == e8.E8_EWORKSPACE

"""GPU parity of the explicit Hadamard block entry points (the storage variant
with a small block, n_h = 128 or 256 for every K) against the oracle's
explicit-block functions.

The glq page ("How it works", item 2) fixes a randomized Hadamard transform of
the input dimension but not its block size; with a small block every K tile of
n_h columns is transformed on its own.  Bars as for the default block:
bit-exact forward transform, indices and bf16 decoded weights; GEMM within
2e-3 relative Frobenius of the oracle's binary64 product of its decoded
weights (1e-4 for the modes that multiply the decoded weights themselves).
"""
import numpy as np
import pytest
import torch

import decode_gemm_e8_b200 as e8
from decode_gemm_e8_b200 import synth
from oracle import oracle as orc
from tests import gpu_util as gu

pytestmark = pytest.mark.gpu

BAR = 2e-3
BAR_DECODED = 1e-4


@pytest.fixture(scope="module")
def gcb():
    gu.dev()
    from decode_gemm_e8_b200 import build
    build.build()
    return e8.Codebook(0)


@pytest.mark.parametrize("nh", [8, 64, 128, 256, 512])
@pytest.mark.parametrize("N,K", [(3, 1024), (2, 3072), (1, 14336)])
def test_rht_forward_small_block_bit_exact(gcb, nh, N, K):
    W = synth.gaussian_weights(N, K, 0.02, nh + K)
    s = synth.suggest_scale(W, 4)
    U = gu.to_np(e8.e8_rht_forward(gcb, gu.to_dev(W), 41, s, nh=nh))
    ref = orc.rht_forward(W, 41, s, nh=nh)
    assert np.array_equal(U.view(np.uint32), ref.view(np.uint32))


@pytest.mark.parametrize("bpw", [2, 3, 4])
@pytest.mark.parametrize("nh", [128, 256])
def test_encode_decode_small_block_bit_exact(gcb, bpw, nh):
    # every group of a 48 x 1024 Gaussian matrix: indices and decoded weights
    N, K, rs = 48, 1024, 5 + nh
    W = synth.gaussian_weights(N, K, 0.02, 200 + bpw)
    s = synth.suggest_scale(W, bpw)
    i1, i2 = e8.e8_encode(gcb, gu.to_dev(W), bpw, rs, s, nh=nh)
    r1, r2 = orc.encode(W, bpw, rs, s, nh=nh)
    assert np.array_equal(gu.to_np(i1), r1)
    if bpw > 2:
        assert np.array_equal(gu.to_np(i2), r2)
    wd = gu.to_np(e8.e8_decode_to_bf16(gcb, i1, i2, N, K, bpw, rs, s, nh=nh))
    assert np.array_equal(wd, orc.decode(r1, r2, N, K, bpw, rs, s, nh=nh))
    # the same codes under the default block are another matrix
    wdef = gu.to_np(e8.e8_decode_to_bf16(gcb, i1, i2, N, K, bpw, rs, s))
    assert not np.array_equal(wdef, wd)
    assert e8.e8_sync_status(gcb) == e8.E8_OK


@pytest.mark.parametrize("nh", [128, 256])
def test_encode_small_block_sampled_rows_full_size(gcb, nh):
    # the MLP up-projection shape (14336 x 4096, 3 bpw) and a DiT shape with
    # outlier columns (3072 x 12288, 4 bpw): 6 seeded rows each, every group
    for (N, K, bpw, W) in ((14336, 4096, 3, synth.gaussian_weights(14336, 4096, 0.015, 4)),
                           (3072, 12288, 4, synth.student_t_outlier_weights(3072, 12288, 9))):
        rs = 17
        s = synth.suggest_scale(W, bpw)
        i1, i2 = e8.e8_encode(gcb, gu.to_dev(W), bpw, rs, s, nh=nh)
        rows = np.sort(np.random.default_rng(nh + K).choice(N, 6, replace=False))
        r1, r2 = orc.encode(W[rows], bpw, rs, s, nh=nh)
        g1, g2 = gu.to_np(i1)[rows], gu.to_np(i2)[rows]
        assert np.array_equal(g1, r1) and np.array_equal(g2, r2), (N, K)
        wd = gu.to_np(e8.e8_decode_to_bf16(gcb, i1, i2, N, K, bpw, rs, s, nh=nh))[rows]
        assert np.array_equal(wd, orc.decode(r1, r2, len(rows), K, bpw, rs, s, nh=nh)), (N, K)
        del i1, i2
    assert e8.e8_sync_status(gcb) == e8.E8_OK


@pytest.mark.parametrize("nh", [128, 256])
@pytest.mark.parametrize("M,mode", [(1, e8.E8_GEMM_ACT_RHT), (16, e8.E8_GEMM_ACT_RHT),
                                    (40, e8.E8_GEMM_ACT_RHT), (16, e8.E8_GEMM_ACT_RHT_SMEM),
                                    (96, e8.E8_GEMM_DECODED_W), (7, e8.E8_GEMM_SIMT),
                                    (16, e8.E8_GEMM_AUTO), (200, e8.E8_GEMM_AUTO)])
def test_gemm_small_block(gcb, nh, M, mode):
    # 4 bpw, K = 3072 (default block 1024), N = 520 (a ragged last tile);
    # with n_h = 256 and up to 32 tokens ACT_RHT takes the int8 path, with
    # n_h = 128 the bf16 one
    N, K, bpw, rs = 520, 3072, 4, 23
    W = synth.student_t_outlier_weights(N, K, 12)
    s = synth.suggest_scale(W, bpw)
    i1, i2 = e8.e8_encode(gcb, gu.to_dev(W), bpw, rs, s, nh=nh)
    Xh = synth.activations_bf16(M, K, 60 + M)
    Y = gu.to_np(e8.e8_gemm(gcb, gu.bf16_dev(Xh), i1, i2, N, K, bpw, rs, s, mode=mode, nh=nh))
    wd = orc.decode(gu.to_np(i1), gu.to_np(i2), N, K, bpw, rs, s, nh=nh)
    err = gu.rel_fro(Y, orc.gemm(Xh, wd))
    assert err < BAR, (nh, M, mode, err)
    if mode in (e8.E8_GEMM_DECODED_W, e8.E8_GEMM_SIMT) or (mode == e8.E8_GEMM_AUTO and M > 64):
        assert err < BAR_DECODED, (nh, M, mode, err)
    assert e8.e8_sync_status(gcb) == e8.E8_OK


def test_invalid_blocks_are_refused(gcb):
    N, K = 4, 3072
    W = gu.to_dev(synth.gaussian_weights(N, K, 0.02, 1))
    for nh in (4, 96, 2048, 65536):   # too small, not a power of two, not dividing K, too large
        with pytest.raises(e8.E8Error) as ei:
            e8.e8_encode(gcb, W, 2, 0, 0.01, nh=nh)
        assert ei.value.code == e8.E8_EINVAL
    assert e8.e8_workspace_bytes(e8.E8_GEMM_ACT_RHT, 16, N, K, 4, nh=96) == 0

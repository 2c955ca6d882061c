"""GPU parity of the grouped small-batch GEMM (e8_gemm_grouped).

Several weight matrices that read the same tokens (q, k and v; gate and up)
run as one activation transform per seed and one fused decode + int8 GEMM
launch over their concatenated row tiles.  Every output is checked against
the oracle's binary64 product X W_dec^T of the oracle's decoded weights at the
2e-3 relative Frobenius bar of the other GEMM tests (the method: page
"glq 0.1.1", "How it works", items 1-2), and against the single-matrix call
e8_gemm (E8_GEMM_ACT_RHT), which runs the same arithmetic: the two agree to
the 1e-6 run-to-run bound of the int8 path (partial sums added in arrival
order).
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
REPEAT = 1e-6


@pytest.fixture(scope="module")
def gcb():
    gu.dev()
    from decode_gemm_e8_b200 import build
    build.build()
    return e8.Codebook(0)


def _matrices(gcb, shapes, K, bpw, seed0):
    """Encodes one Gaussian matrix per N on the GPU; returns (i1, i2, N, rs, s)."""
    out = []
    for j, N in enumerate(shapes):
        rs = 1000 + seed0 + j
        if N == 0:
            z1 = torch.zeros((0, K // 8), dtype=torch.uint16, device=gu.dev())
            z2 = None if bpw == 2 else torch.zeros(
                (0, K // 8), dtype=torch.uint8 if bpw == 3 else torch.uint16, device=gu.dev())
            out.append((z1, z2, 0, rs, 0.01))
            continue
        W = synth.gaussian_weights(N, K, 0.02, seed0 + j)
        s = synth.suggest_scale(W, bpw)
        i1, i2 = e8.e8_encode(gcb, gu.to_dev(W), bpw, rs, s)
        out.append((i1, i2, N, rs, s))
    return out


def _oracle_rows(Xh, it, K, bpw, rows=None):
    """Oracle product of X with the decoded weights (all rows, or the given ones)."""
    i1, i2, N, rs, s = it
    h1 = gu.to_np(i1)
    h2 = None if i2 is None else gu.to_np(i2)
    if rows is not None:
        h1 = h1[rows]
        h2 = None if h2 is None else h2[rows]
    wd = orc.decode(h1, h2, h1.shape[0], K, bpw, rs, s)
    return orc.gemm(Xh, wd)


@pytest.mark.parametrize("bpw", [2, 3, 4])
@pytest.mark.parametrize("M", [1, 5, 16, 32])
def test_grouped_matches_oracle_ragged(gcb, bpw, M):
    # three matrices whose row counts end in partial tiles (200 = 128 + 72,
    # 1000 = 7 x 128 + 104, 136 = 128 + 8), K = 1024 (Hadamard block 1024)
    K = 1024
    mats = _matrices(gcb, [200, 1000, 136], K, bpw, 40 + bpw)
    Xh = synth.activations_bf16(M, K, 70 + M)
    Ys = e8.e8_gemm_grouped(gcb, gu.bf16_dev(Xh), mats, K, bpw)
    for it, Y in zip(mats, Ys):
        y = gu.to_np(Y)
        assert y.shape == (M, it[2]) and np.all(np.isfinite(y))
        err = gu.rel_fro(y, _oracle_rows(Xh, it, K, bpw))
        assert err < BAR, (it[2], err)
    assert e8.e8_sync_status(gcb) == e8.E8_OK


def test_grouped_qkv_equals_single_calls(gcb):
    # the q, k, v projections of a Llama-3-8B layer at 4 bpw, 16 tokens
    K, bpw, M = 4096, 4, 16
    mats = _matrices(gcb, [4096, 1024, 1024], K, bpw, 90)
    Xh = synth.activations_bf16(M, K, 3)
    X = gu.bf16_dev(Xh)
    Ys = e8.e8_gemm_grouped(gcb, X, mats, K, bpw)
    rng = np.random.default_rng(5)
    for it, Y in zip(mats, Ys):
        i1, i2, N, rs, s = it
        ref = e8.e8_gemm(gcb, X, i1, i2, N, K, bpw, rs, s, mode=e8.E8_GEMM_ACT_RHT)
        y = gu.to_np(Y)
        assert gu.rel_fro(y, gu.to_np(ref)) < REPEAT
        rows = np.sort(rng.choice(N, 96, replace=False))
        err = gu.rel_fro(y[:, rows], _oracle_rows(Xh, it, K, bpw, rows))
        assert err < BAR, (N, err)
    assert e8.e8_sync_status(gcb) == e8.E8_OK


def test_grouped_four_items_cluster_transform_and_empty_item(gcb):
    # K = 14336 (Hadamard block 2048, transform chunks in a 4-CTA cluster),
    # 32 tokens (64 piece rows), 3 bpw, four items one of which is empty
    K, bpw, M = 14336, 3, 32
    mats = _matrices(gcb, [384, 0, 260, 128], K, bpw, 120)
    Xh = synth.activations_bf16(M, K, 9)
    Ys = e8.e8_gemm_grouped(gcb, gu.bf16_dev(Xh), mats, K, bpw)
    for it, Y in zip(mats, Ys):
        if it[2] == 0:
            assert Y.shape == (M, 0)
            continue
        err = gu.rel_fro(gu.to_np(Y), _oracle_rows(Xh, it, K, bpw))
        assert err < BAR, (it[2], err)
    assert e8.e8_sync_status(gcb) == e8.E8_OK


def test_grouped_back_to_back_repeats(gcb):
    # twenty grouped calls queued back to back on one stream, outputs rotated
    # over two sets: every call reproduces the first within the run-to-run bound
    K, bpw, M = 4096, 2, 8
    mats = _matrices(gcb, [1024, 3072], K, bpw, 150)
    X = gu.bf16_dev(synth.activations_bf16(M, K, 11))
    ws = torch.empty(e8.e8_gemm_grouped_workspace_bytes(M, K, bpw, 2), dtype=torch.uint8,
                     device=X.device)
    first = [gu.to_np(y) for y in e8.e8_gemm_grouped(gcb, X, mats, K, bpw, workspace=ws)]
    outs = [[torch.full((M, it[2]), float("nan"), device=X.device) for it in mats]
            for _ in range(2)]
    for r in range(20):
        items = [it + (outs[r % 2][j],) for j, it in enumerate(mats)]
        e8.e8_gemm_grouped(gcb, X, items, K, bpw, workspace=ws)
        if r >= 18:
            for j in range(len(mats)):
                assert gu.rel_fro(gu.to_np(outs[r % 2][j]), first[j]) < REPEAT
    assert e8.e8_sync_status(gcb) == e8.E8_OK

"""GPU parity of the entropy-coded E8 variant (e8_ep_*) against the oracle
(oracle/ep_oracle.py).  Page: "Transformers Proposes EntroPack Integration for
Configurable Non-Integer-Bit-Rate Weight Compression", second paragraph (per-row
normalised E8, conditional model, entropy coding in independently decodable
blocks, fused GPU decode) and third (rate with metadata).

Bars: bit-exact row scales, frequency tables, block offsets and stream words
of the encoder, bit-exact bf16 weights of the decoder (from the GPU's streams
and from the oracle's), the GEMM within 1e-4 relative Frobenius of the oracle's
binary64 product of the decoded weights (the bar of the other decoded-weight
modes).
"""
import numpy as np
import pytest
import torch

import decode_gemm_e8_b200 as e8
from decode_gemm_e8_b200 import synth
from oracle import ep_oracle as ep
from tests import gpu_util as gu

pytestmark = pytest.mark.gpu

BAR_DECODED = 1e-4


@pytest.fixture(scope="module")
def gcb():
    gu.dev()
    from decode_gemm_e8_b200 import build
    build.build()
    return e8.Codebook(0)


def _layer(N, K, seed, kind="gauss"):
    if kind == "dit":
        return synth.student_t_outlier_weights(N, K, seed)
    W = synth.gaussian_weights(N, K, 0.02, seed)
    if kind == "zero_row":
        W = W.copy()
        W[N // 2] = 0.0
    return W


def _oracle_dict(m):
    return {"N": m.N, "K": m.K, "t": gu.to_np(m.t), "tables": gu.to_np(m.tables),
            "words": gu.to_np(m.words)[:m.total_words],
            "offsets": gu.to_np(m.offsets).astype(np.uint32)}


CASES = [(24, 256, 0.05, "gauss"), (7, 1000, 0.02, "zero_row"), (3, 8, 0.5, "gauss"),
         (16, 512, 1 / 120, "dit"), (40, 1536, 0.03, "dit")]


@pytest.mark.parametrize("N,K,delta,kind", CASES)
def test_ep_encode_bit_exact(gcb, N, K, delta, kind):
    W = _layer(N, K, N + K, kind)
    m = e8.e8_ep_encode(gcb, gu.to_dev(W), delta)
    ref = ep.encode(W, delta)
    assert np.array_equal(gu.to_np(m.t).view(np.uint32), ref["t"].view(np.uint32))
    assert np.array_equal(gu.to_np(m.tables), ref["tables"])
    assert np.array_equal(gu.to_np(m.offsets).astype(np.uint32), ref["offsets"])
    assert m.total_words == int(ref["offsets"][-1])
    assert np.array_equal(gu.to_np(m.words)[:m.total_words], ref["words"])
    assert m.actual_bpp() == pytest.approx(ep.actual_bpp(ref), rel=1e-12)
    assert e8.e8_sync_status(gcb) == e8.E8_OK


@pytest.mark.parametrize("N,K,delta,kind", CASES)
def test_ep_decode_bit_exact(gcb, N, K, delta, kind):
    W = _layer(N, K, 3 * N + K, kind)
    m = e8.e8_ep_encode(gcb, gu.to_dev(W), delta)
    want = ep.decode(ep.encode(W, delta))
    assert np.array_equal(gu.to_np(e8.e8_ep_decode_to_bf16(gcb, m)), want)
    # the oracle's own streams, decoded on the GPU
    ref = ep.encode(W, delta)
    mo = e8.EpMatrix(N, K, delta, gu.to_dev(ref["words"]), gu.to_dev(ref["offsets"].astype(np.int32)),
                     gu.to_dev(ref["t"]), gu.to_dev(ref["tables"]), int(ref["offsets"][-1]))
    assert np.array_equal(gu.to_np(e8.e8_ep_decode_to_bf16(gcb, mo)), want)
    assert e8.e8_sync_status(gcb) == e8.E8_OK


@pytest.mark.parametrize("M", [1, 16, 300])
def test_ep_gemm_matches_oracle(gcb, M):
    N, K = 200, 1024
    W = _layer(N, K, 77, "dit")
    m = e8.e8_ep_encode(gcb, gu.to_dev(W), 0.03)
    Xh = synth.activations_bf16(M, K, 5 + M)
    Y = gu.to_np(e8.e8_ep_gemm(gcb, gu.bf16_dev(Xh), m))
    ref = ep.gemm(Xh, ep.decode(_oracle_dict(m)))
    assert gu.rel_fro(Y, ref) < BAR_DECODED
    assert e8.e8_sync_status(gcb) == e8.E8_OK


@pytest.mark.parametrize("target", [3.0, 3.5, 4.0])
def test_ep_choose_delta_reaches_the_target_rate(gcb, target):
    W = gu.to_dev(_layer(256, 2048, 21, "dit"))
    d = e8.e8_ep_choose_delta(gcb, W, target)
    m = e8.e8_ep_encode(gcb, W, d)
    r = m.actual_bpp()
    assert target - 0.1 <= r <= target + 0.02, (target, d, r)
    assert e8.e8_ep_estimate_bpp(gcb, W, d) <= target
    assert e8.e8_sync_status(gcb) == e8.E8_OK


def test_ep_malformed_streams_report_edata(gcb):
    N, K = 16, 1024
    W = gu.to_dev(_layer(N, K, 4))
    m = e8.e8_ep_encode(gcb, W, 0.03)
    assert e8.e8_sync_status(gcb) == e8.E8_OK
    # one word of block 0 changed: the block no longer returns to its start state
    w = m.words.clone()
    w.view(torch.int16)[5] ^= 0x5A5A
    bad = e8.EpMatrix(N, K, m.delta, w, m.offsets, m.t, m.tables, m.total_words)
    e8.e8_ep_decode_to_bf16(gcb, bad)
    assert e8.e8_sync_status(gcb) == e8.E8_EDATA
    # a frequency table that does not sum to 4096
    tb = m.tables.clone()
    tb.view(torch.int16)[3] += 1
    bad = e8.EpMatrix(N, K, m.delta, m.words, m.offsets, m.t, tb, m.total_words)
    e8.e8_ep_decode_to_bf16(gcb, bad)
    assert e8.e8_sync_status(gcb) == e8.E8_EDATA
    # a block offset past the end of the words: refused by the bound, not read
    of = m.offsets.clone()
    of[1] = 1 << 30
    bad = e8.EpMatrix(N, K, m.delta, m.words, of, m.t, m.tables, m.total_words)
    e8.e8_ep_decode_to_bf16(gcb, bad)
    assert e8.e8_sync_status(gcb) == e8.E8_EDATA
    # the intact stream still decodes
    e8.e8_ep_decode_to_bf16(gcb, m)
    assert e8.e8_sync_status(gcb) == e8.E8_OK


def test_ep_refusals(gcb):
    W = gu.to_dev(_layer(4, 64, 1))
    for d in (1 / 121, float("nan"), float("inf")):
        with pytest.raises(e8.E8Error) as ei:
            e8.e8_ep_encode(gcb, W, d)
        assert ei.value.code == e8.E8_EINVAL
    assert e8.load_library().e8_ep_num_blocks(4, 12) == -1
    assert e8.load_library().e8_ep_encode_workspace_bytes(4, 12) == 0


def test_ep_full_size_sampled_blocks(gcb):
    # a DiT linear (3072 x 3072, Student-t with outlier columns) at the step
    # that the rate search picks for 4 bpp: all row scales and the tables
    # against the oracle, eight sampled blocks decoded by the oracle from the
    # GPU's own stream
    N = K = 3072
    W = _layer(N, K, 7, "dit")
    Wd = gu.to_dev(W)
    d = e8.e8_ep_choose_delta(gcb, Wd, 4.0)
    m = e8.e8_ep_encode(gcb, Wd, d)
    t, _ = ep.row_scales(W, d)
    assert np.array_equal(gu.to_np(m.t).view(np.uint32), t.view(np.uint32))
    S = ep.symbols(ep.quantise(W, d)[0])
    assert np.array_equal(gu.to_np(m.tables), ep.table_words(ep.tables(S)))
    out = gu.to_np(e8.e8_ep_decode_to_bf16(gcb, m))
    enc = _oracle_dict(m)
    nb = len(enc["offsets"]) - 1
    blocks = np.random.default_rng(3).choice(nb, 8, replace=False)
    flat = out.reshape(-1, 8)
    for b in blocks:
        Sb = ep.decode_block_symbols(enc, int(b))
        assert np.array_equal(Sb, S[64 * b:64 * b + Sb.shape[0]])
        rows = (64 * b + np.arange(Sb.shape[0])) // (K // 8)
        V = ep.values_from_symbols(Sb)
        a = (t[rows] * np.float32(0.5)).astype(np.float32)
        want = ep.f32_to_bf16_bits((V.astype(np.float32) * a[:, None]).astype(np.float32))
        assert np.array_equal(flat[64 * b:64 * b + Sb.shape[0]], want)
    assert 3.9 <= m.actual_bpp() <= 4.02
    assert e8.e8_sync_status(gcb) == e8.E8_OK

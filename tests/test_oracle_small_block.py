"""Pins of the oracle's explicit-block entry points: the storage variant that
uses a small Hadamard block (n_h = 128 or 256) for every K.  The glq page
("How it works", item 2) fixes a randomized Hadamard transform on the input
dimension but not its block size; everything except the block is the same as
in the default format (signs, normalisation gamma = 1/(s sqrt(n_h)), decode
alpha = s/(m sqrt(n_h)), the two roundings).

The references here are independent of the oracle's code: the Sylvester
matrix built from (-1)^popcount(i & j), numpy's fp32 product for the decode
scaling and torch's float32 -> bfloat16 cast for the final rounding.
"""
import numpy as np
import pytest

from oracle import oracle as orc
from tests import indep


@pytest.fixture(scope="module")
def cb():
    return orc.codebook().astype(np.int64)


def _planted(cb, N, K, nh, bpw, seed, s, rht_seed):
    """Random codes whose decoded groups lie deep inside their Voronoi cells,
    and the fp32 weight matrix they encode with Hadamard block nh."""
    rng = np.random.default_rng(seed)
    G = N * K // 8
    i1 = rng.integers(0, 65536, G)
    m = {2: 2, 3: 4, 4: 8}[bpw]
    z = cb[i1] * (m // 2)
    i2 = None
    if bpw > 2:
        n2 = (cb ** 2).sum(1) // 4
        ok = np.nonzero(n2 <= 6)[0] if bpw == 4 else np.array([0])
        i2 = ok[rng.integers(0, len(ok), G)]
        z = z + cb[i2]
    H = indep.sylvester(nh).astype(np.int64)
    d = orc.signs(rht_seed, K)
    Z = z.reshape(N, K)
    T = np.concatenate([Z[:, b:b + nh] @ H for b in range(0, K, nh)], axis=1)
    W = (s * d[None, :] * T / (m * np.sqrt(nh))).astype(np.float32)
    return W, i1.reshape(N, K // 8), (None if i2 is None else i2.reshape(N, K // 8)), T, d, m


def _bf16_bits(x32):
    import torch
    return torch.from_numpy(x32).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)


@pytest.mark.parametrize("bpw,K,nh", [(2, 4096, 128), (3, 768, 256), (4, 1024, 128),
                                      (4, 256, 256), (3, 3072, 128), (2, 384, 128)])
def test_planted_codes_round_trip_small_block(cb, bpw, K, nh):
    N, s, rs = 6, 0.029, 77
    W, i1, i2, T, d, m = _planted(cb, N, K, nh, bpw, 500 + K + nh, s, rs)
    e1, e2 = orc.encode(W, bpw, rs, s, nh=nh)
    assert np.array_equal(e1, i1.astype(np.uint16))
    if bpw > 2:
        assert np.array_equal(e2.astype(np.int64), i2)
    out = orc.decode(e1, e2, N, K, bpw, rs, s, nh=nh)
    # the definition: bf16_rne(d * fl32(t * alpha)), t the exact block transform
    alpha = np.float32(s / (m * np.sqrt(nh)))
    assert np.all(np.abs(T) < 2 ** 24)
    p = T.astype(np.float32) * alpha
    p = np.where(d[None, :] < 0, -p, p).astype(np.float32)
    assert np.array_equal(out, _bf16_bits(p))


@pytest.mark.parametrize("K", [256, 768, 4096, 12288])
def test_default_block_equals_the_explicit_one(K):
    rng = np.random.default_rng(K)
    W = (rng.standard_normal((3, K)) * 0.02).astype(np.float32)
    nh = orc.hadamard_block(K)
    for bpw in (2, 4):
        a1, a2 = orc.encode(W, bpw, 5, 0.02)
        b1, b2 = orc.encode(W, bpw, 5, 0.02, nh=nh)
        assert np.array_equal(a1, b1)
        assert (a2 is None and b2 is None) or np.array_equal(a2, b2)
        assert np.array_equal(orc.decode(a1, a2, 3, K, bpw, 5, 0.02),
                              orc.decode(b1, b2, 3, K, bpw, 5, 0.02, nh=nh))


@pytest.mark.parametrize("nh", [8, 128, 256])
def test_small_block_forward_transform(nh):
    # u = gamma * H_nh D w per block: matches the float64 Sylvester product to
    # fp32 rounding, and keeps the norm (H_nh / sqrt(nh) is orthogonal)
    K, s, rs = 1024, 0.05, 3
    rng = np.random.default_rng(nh)
    W = (rng.standard_normal((4, K)) * 0.02).astype(np.float32)
    U = orc.rht_forward(W, rs, s, nh=nh).astype(np.float64)
    H = indep.sylvester(nh).astype(np.float64)
    DW = W.astype(np.float64) * orc.signs(rs, K)[None, :]
    ref = np.concatenate([DW[:, b:b + nh] @ H for b in range(0, K, nh)], axis=1) / (s * np.sqrt(nh))
    assert np.allclose(U, ref, rtol=0, atol=1e-6 * np.abs(ref).max())
    assert np.allclose(np.linalg.norm(U, axis=1) * s, np.linalg.norm(W, axis=1), rtol=1e-5)


def test_block_size_is_part_of_the_format():
    # codes written with n_h = 128 decode to the weights only with n_h = 128
    K, s, bpw = 2048, 0.02 / 0.9, 4
    rng = np.random.default_rng(11)
    W = (rng.standard_normal((8, K)) * 0.02).astype(np.float32)
    i1, i2 = orc.encode(W, bpw, 9, s, nh=128)
    good = orc.bf16_bits_to_f32(orc.decode(i1, i2, 8, K, bpw, 9, s, nh=128)).astype(np.float64)
    bad = orc.bf16_bits_to_f32(orc.decode(i1, i2, 8, K, bpw, 9, s)).astype(np.float64)
    w = W.astype(np.float64)
    e_good = np.linalg.norm(good - w) / np.linalg.norm(w)
    e_bad = np.linalg.norm(bad - w) / np.linalg.norm(w)
    assert e_good < 0.1 and e_bad > 0.5


@pytest.mark.parametrize("K,nh", [(1024, 96), (1024, 4), (768, 512), (1024, 2048),
                                  (65536, 65536), (1000, 8 * 125)])
def test_invalid_blocks_are_rejected(K, nh):
    assert not orc.valid_block(K, nh)
    W = np.zeros((1, K), np.float32)
    with pytest.raises(ValueError):
        orc.encode(W, 2, 1, 0.02, nh=nh)
    with pytest.raises(ValueError):
        orc.decode(np.zeros((1, K // 8), np.uint16), None, 1, K, 2, 1, 0.02, nh=nh)
    with pytest.raises(ValueError):
        orc.rht_forward(W, 1, 0.02, nh=nh)

"""Pins of the entropy-coded E8 oracle (oracle/ep_oracle.py) against facts that do
not come from the oracle itself: brute force over lattice points, the E8
membership rule and covering radius, hand-worked rANS states, the entropy of
the coded symbols, and the page's rate accounting.

Page: "Transformers Proposes EntroPack Integration for Configurable
Non-Integer-Bit-Rate Weight Compression", second and third paragraphs.
"""
import itertools

import numpy as np
import pytest

from oracle import ep_oracle as ep


def _brute_nearest_dist2(u):
    """Exact (binary64) squared distance from u to the nearest E8 point: the
    nearest point of D8 differs from the rounding of u by at most one unit in
    each coordinate, and likewise for D8 + 1/2 around floor(u) + 1/2, so the
    3^8 perturbations of each base contain it."""
    u = np.asarray(u, dtype=np.float64)
    best = np.inf
    deltas = np.array(list(itertools.product((-1, 0, 1), repeat=8)), dtype=np.float64)
    for base in (np.rint(u), np.floor(u) + 0.5):
        P = base[None, :] + deltas
        s = P.sum(axis=1)
        ok = np.abs(np.round(s) - s) < 1e-9
        ok &= (np.round(s).astype(np.int64) % 2) == 0
        d = ((P[ok] - u[None, :]) ** 2).sum(axis=1)
        best = min(best, d.min())
    return best


def _is_e8(V):
    V = np.asarray(V, dtype=np.int64).reshape(-1, 8)
    same = np.all((V & 1) == (V[:, :1] & 1), axis=1)
    return same & ((V.sum(axis=1) % 4) == 0)


@pytest.mark.parametrize("scale", [0.3, 1.0, 4.0, 60.0])
def test_nearest_e8_is_a_nearest_lattice_point(scale):
    rng = np.random.default_rng(int(scale * 10))
    U = (rng.standard_normal((300, 8)) * scale).astype(np.float32)
    V = ep.nearest_e8(U)
    assert np.all(_is_e8(V))
    for u, v in zip(U, V):
        d = float(((u.astype(np.float64) - v / 2.0) ** 2).sum())
        # equal up to the fp32 rounding of the two candidate distances
        assert d <= _brute_nearest_dist2(u) * (1 + 1e-6) + 1e-9


def test_nearest_e8_tie_rules():
    # the zero vector; a point between both cosets (D8 wins the tie); the
    # half-integer point; an odd integer vector (parity repair moves the first
    # coordinate up); parity repair at the coordinate farthest from its
    # rounding (1.2: index 0; 1.1, 0.4: index 1)
    cases = {
        (0,) * 8: (0,) * 8,
        (0.25,) * 8: (0,) * 8,
        (0.5,) * 8: (1,) * 8,
        (1, 0, 0, 0, 0, 0, 0, 0): (4, 0, 0, 0, 0, 0, 0, 0),
        (1.2, 0.1, 0, 0, 0, 0, 0, 0): (4, 0, 0, 0, 0, 0, 0, 0),
        (1.1, 0.4, 0, 0, 0, 0, 0, 0): (2, 2, 0, 0, 0, 0, 0, 0),
    }
    for u, want in cases.items():
        got = tuple(int(x) for x in ep.nearest_e8(np.array(u, np.float32)))
        assert got == want, (u, got)


def test_rans_hand_worked_states():
    # P(0) = 3/4, P(1) = 1/4 (frequencies 3072, 1024), decode order 0, 1, 1,
    # encoded last to first from x = 65536:
    #   1: x = (65536 // 1024) * 4096 + 0 + 3072 = 265216
    #   1: x = 259 * 4096 + 0 + 3072 = 1063936
    #   0: x = 346 * 4096 + 1024 + 0 = 1418240 = 0x15A400, nothing emitted
    f = np.array([3072, 1024])
    assert ep.rans_encode([(f, 0), (f, 1), (f, 1)]) == [0x15, 0xA400]
    syms, x, p = ep.rans_decode([0x15, 0xA400], [f, f, f])
    assert syms == [0, 1, 1] and x == 65536 and p == 2
    # P(1) = 1/4096: the second symbol 1 first flushes 16 bits:
    #   1: x = 65536 * 4096 + 4095 = 268439551
    #   1: x >= 2^20 -> emit 0x0FFF, x = 4096; x = 4096 * 4096 + 4095 = 16781311
    g = np.array([4095, 1])
    assert ep.rans_encode([(g, 1), (g, 1)]) == [0x100, 0x0FFF, 0x0FFF]
    syms, x, p = ep.rans_decode([0x100, 0x0FFF, 0x0FFF], [g, g])
    assert syms == [1, 1] and x == 65536 and p == 3


def test_normalise_rule():
    rng = np.random.default_rng(3)
    for n in (2, 17, 128, 256):
        counts = rng.integers(0, 1000, n) * (rng.random(n) < 0.7)
        counts[rng.integers(n)] += 1
        f = ep.normalise(counts)
        assert f.sum() == 4096
        assert np.all((f >= 1) == (counts > 0))
        # floor scaling everywhere but the adjusted symbols
        base = np.where(counts > 0, np.maximum(1, counts * 4096 // counts.sum()), 0)
        assert np.sum(f != base) <= 1 or base.sum() > 4096
    assert list(ep.normalise(np.zeros(4, np.int64))) == [4096, 0, 0, 0]
    # 256 symbols, one dominant: the floor-1 bumps exceed what the dominant
    # symbol can give back in one step only if it is small; here it is not
    c = np.ones(256, np.int64)
    c[5] = 10 ** 6
    f = ep.normalise(c)
    assert f.sum() == 4096 and f.min() == 1 and f[5] == 4096 - 255


def test_rans_round_trip_and_cost_bound():
    rng = np.random.default_rng(11)
    for trial in range(6):
        n_alpha = [2, 5, 40, 256][trial % 4]
        f = ep.normalise(rng.integers(1, 300, n_alpha) ** 2)
        p = f / 4096.0
        seq_syms = rng.choice(n_alpha, size=800, p=p)
        words = ep.rans_encode([(f, int(s)) for s in seq_syms])
        syms, x, used = ep.rans_decode(words, [f] * len(seq_syms))
        assert syms == list(seq_syms) and x == 65536 and used == len(words)
        ideal = float(np.sum(12 - np.log2(f[seq_syms])))
        assert 16 * len(words) <= ideal + 48 + 0.01 * len(seq_syms)
        assert 16 * len(words) >= ideal - 16


def _layer(N, K, seed, outliers=False):
    rng = np.random.default_rng(seed)
    W = (rng.standard_normal((N, K)) * 0.02).astype(np.float32)
    if outliers:
        cols = rng.choice(K, max(1, K // 100), replace=False)
        W[:, cols] *= 8
        W[rng.integers(N)] = 0.0     # an all-zero row
    return W


@pytest.mark.parametrize("N,K,delta,outliers", [(24, 256, 0.05, False), (7, 1000, 0.02, True),
                                                (3, 8, 0.5, False), (16, 512, 1 / 120, True)])
def test_encode_decode_round_trip_and_error_bound(N, K, delta, outliers):
    W = _layer(N, K, N + K, outliers)
    enc = ep.encode(W, delta)
    V, t = ep.quantise(W, delta)
    assert np.all(_is_e8(V))
    dec = ep.decode(enc)
    assert np.array_equal(dec, ep.reconstruct(V, t))
    # E8 with minimal norm 2 has covering radius 1: per group |u - V/2| <= 1,
    # so |w - w'| <= t_n (1 + 2^-20) plus the bf16 rounding of w' (2^-9 |w'|)
    wd = (dec.astype(np.uint32) << 16).view(np.float32).astype(np.float64)
    err = np.linalg.norm((W.astype(np.float64) - wd).reshape(N, K // 8, 8), axis=2)
    lim = t[:, None].astype(np.float64) * (1 + 2 ** -20) + 2 ** -9 * np.linalg.norm(
        wd.reshape(N, K // 8, 8), axis=2) + 1e-30
    assert np.all(err <= lim)
    # every block decodes alone
    nb = len(enc["offsets"]) - 1
    for b in range(nb):
        S = ep.decode_block_symbols(enc, b)
        assert S.shape[0] == min(64, N * K // 8 - 64 * b)


def test_rate_matches_entropy_of_the_conditional_model():
    # the payload of a 64 x 2048 Gaussian layer costs the empirical entropy of
    # its symbols under the coset-conditional model, plus at most the
    # quantisation of the frequencies and 32 bits per block
    W = _layer(64, 2048, 5)
    enc = ep.encode(W, 0.03)
    S = ep.symbols(ep.quantise(W, 0.03)[0])
    c = S[:, 0]

    def H(x):
        _, n = np.unique(x, return_counts=True)
        p = n / n.sum()
        return float(-(n * np.log2(p)).sum())
    bits = H(c)
    for cc in (0, 1):
        sel = S[c == cc]
        if len(sel):
            bits += H(sel[:, 1:8].ravel()) + H(sel[:, 8])
    payload = 16 * int(enc["offsets"][-1])
    nb = len(enc["offsets"]) - 1
    assert bits - 16 * nb <= payload <= bits * 1.01 + 32 * nb


def test_actual_bpp_accounting_and_rate_falls_with_the_step():
    W = _layer(32, 1024, 9)
    rates = []
    for d in (0.01, 0.02, 0.04, 0.08):
        enc = ep.encode(W, d)
        nb = len(enc["offsets"]) - 1
        want = (16 * int(enc["offsets"][-1]) + 32 * (nb + 1) + 32 * 32 + 16 * 770 + 32) / (32 * 1024)
        assert ep.actual_bpp(enc) == pytest.approx(want, rel=1e-12)
        rates.append(ep.actual_bpp(enc))
    assert all(a > b for a, b in zip(rates, rates[1:]))


def test_symbol_bounds_at_the_smallest_step():
    # |u| <= 1 / delta (1 + 2^-22) keeps m in [-128, 127] and q in [-64, 63]
    W = np.zeros((2, 16), np.float32)
    W[0, :8] = [1, -1, 1, -1, 1, -1, 1, 0.999]
    W[1, 8:] = -1
    S = ep.symbols(ep.quantise(W, 1 / 120)[0])
    assert S[:, 1:8].min() >= -128 and S[:, 1:8].max() <= 127
    assert S[:, 8].min() >= -64 and S[:, 8].max() <= 63
    with pytest.raises(ValueError):
        ep.quantise(W, 1 / 121)


@pytest.mark.parametrize("scale", [0.4, 0.9])
def test_nearest_e8_agrees_with_the_codebook_brute_force(scale):
    # inside the full shells (squared norm <= 10) the nearest lattice point is
    # the nearest codebook point, which the main oracle finds by an exact
    # brute force over all 65536 entries (a separate implementation)
    from oracle import oracle as orc
    rng = np.random.default_rng(int(scale * 100))
    U = (rng.standard_normal((2000, 8)) * scale).astype(np.float32)
    V = ep.nearest_e8(U)
    keep = (V.astype(np.int64) ** 2).sum(axis=1) <= 40   # doubled: squared norm <= 10
    i1, _ = orc.nearest_groups(U[keep], 2)
    C = orc.codebook().astype(np.int32)
    W = C[i1.astype(np.int64)]
    diff = np.any(W != V[keep], axis=1)
    for u, a, b in zip(U[keep][diff], V[keep][diff], W[diff]):
        # a different choice only on an exact tie of the two distances
        assert orc.cmp_dist(u, a, b, 2) == 0
    assert keep.sum() > 1500

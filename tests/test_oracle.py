"""Pins for the CPU oracle, against facts fixed by the pages and by E8 geometry.

Each test checks the oracle against something other than itself: the page's
format table (tests/golden/glq_format.json), the E8 theta series and second
moment (tests/golden/e8_geometry.json), the Sylvester closed form of the
Hadamard matrix, published SplitMix64 outputs, numpy's matmul, and an
independent exact brute force (tests/indep.py).
"""
import json
import os
from fractions import Fraction

import numpy as np
import pytest

from oracle import oracle as orc
from tests import indep

GOLD = os.path.join(os.path.dirname(__file__), "golden")


def _gold(name):
    with open(os.path.join(GOLD, name)) as f:
        return json.load(f)


# ---------------------------------------------------------------- codebook --

def test_codebook_size_and_shells(cb):
    fmt = _gold("glq_format.json")["facts"][0]
    assert cb.shape == (fmt["codebook_size"], fmt["group"])
    n4 = (cb.astype(np.int64) ** 2).sum(1)          # 4 |x|^2
    assert np.all(n4 % 8 == 0)
    norms = n4 // 4
    assert np.all(np.diff(norms) >= 0), "shells must come in increasing norm"
    counts = np.bincount(norms // 2)
    # the page's "first 7 shells": squared norms 0,2,...,12
    assert len(counts) == fmt["shells"]
    for m in range(6):
        assert counts[m] == indep.theta_e8(m), m
    assert counts[6] == 65536 - sum(indep.theta_e8(m) for m in range(6))
    assert counts[6] < indep.theta_e8(6)             # the 7th shell is the cut one
    assert counts[6] == 8655


def test_codebook_entries_are_distinct_e8_points(cb):
    v = cb.astype(np.int64)
    par = v % 2
    assert np.all((par == 0).all(1) | (par == 1).all(1)), "all integer or all half-integer"
    assert np.all(v.sum(1) % 4 == 0), "coordinate sum even"
    assert len({tuple(r) for r in v}) == len(v)


def test_codebook_canonical_order(cb):
    v = cb.astype(np.int64)
    assert not v[0].any()
    # pairs: entry 2k+2 is the negation of entry 2k+1, entry 65535 is a lone +p
    assert np.array_equal(v[2:65536:2], -v[1:65535:2])
    reps = v[1::2]
    first_nz = np.array([r[np.nonzero(r)[0][0]] for r in reps])
    assert np.all(first_nz > 0)
    n4 = (reps ** 2).sum(1)
    for a, b, na, nb in zip(reps[:-1], reps[1:], n4[:-1], n4[1:]):
        if na == nb:
            assert tuple(a) < tuple(b)
        else:
            assert na < nb


def test_codebook_total_lattice_points_up_to_norm_12():
    # orc_codebook reports how many lattice points it enumerated before the cut
    tmp = np.zeros((65536, 8), dtype=np.int8)
    n = orc._load().orc_codebook(orc._ptr(tmp))
    assert n == sum(indep.theta_e8(m) for m in range(7)) == 117361


def test_residual_codebook_prefix(cb):
    # the 3-bpw residual codebook is the first 256 entries: origin, the 240
    # roots and the first 15 vectors of the norm-4 shell
    n = (cb[:256].astype(np.int64) ** 2).sum(1) // 4
    assert n[0] == 0 and np.all(n[1:241] == 2) and np.all(n[241:256] == 4)


def test_bits_per_weight_table():
    fmt = _gold("glq_format.json")["facts"]
    table = fmt[2]["bits_per_weight"]
    for bpw_s, row in table.items():
        bpw = int(bpw_s)
        N, K = 64, 256
        i1, i2 = np.zeros((N, K // 8), np.uint16), None
        if bpw == 3:
            i2 = np.zeros((N, K // 8), np.uint8)
        if bpw == 4:
            i2 = np.zeros((N, K // 8), np.uint16)
        nbytes = i1.nbytes + (0 if i2 is None else i2.nbytes)
        assert nbytes * 8 == row["index_bits_per_8_weights"] * (N * K // 8)
        assert nbytes * 8 == bpw * N * K           # effective == nominal (+ one scale)


# ---------------------------------------------------------------- transform --

def test_splitmix64_known_answers():
    ref = indep.splitmix64_reference_outputs()
    d = orc.signs(0, 64 * len(ref))
    for j, word in enumerate(ref):
        for b in range(64):
            assert (d[64 * j + b] < 0) == bool((word >> b) & 1)


@pytest.mark.parametrize("K,nh", [(256, 256), (4096, 4096), (3072, 1024), (14336, 2048),
                                  (12288, 4096), (8, 8), (24, 8), (100, 0), (65536, 0)])
def test_hadamard_block(K, nh):
    assert orc.hadamard_block(K) == nh


@pytest.mark.parametrize("n", [8, 16, 64, 512, 4096])
def test_rht_is_orthogonal(n):
    s = 1.0 / np.sqrt(n)
    U = orc.rht_forward(np.eye(n, dtype=np.float32), 11, float(np.float32(s)))
    g = orc.gamma(float(np.float32(s)), n)
    UU = U.astype(np.float64) @ U.astype(np.float64).T
    assert np.array_equal(UU, (g * g * n) * np.eye(n))


@pytest.mark.parametrize("n", [8, 32, 256])
def test_rht_of_unit_vectors_is_a_hadamard_column(n):
    H = indep.sylvester(n)
    d = orc.signs(5, n)
    U = orc.rht_forward(np.eye(n, dtype=np.float32), 5, float(np.float32(1.0 / np.sqrt(n))))
    g = orc.gamma(float(np.float32(1.0 / np.sqrt(n))), n)
    # row r of U is gamma * d_r * H[:, r]
    assert np.array_equal(U.astype(np.float64), g * d[:, None] * H.T.astype(np.float64))


def test_rht_exact_on_small_integers():
    n, N = 1024, 4
    rng = np.random.default_rng(0)
    K = 3 * n                                   # block-diagonal: three blocks of n
    assert orc.hadamard_block(K) == n
    W = rng.integers(-8, 9, size=(N, K)).astype(np.float32)
    s = float(np.float32(1.0 / np.sqrt(n)))     # gamma = 1 exactly for n = 4^k
    assert orc.gamma(s, n) == 1.0
    U = orc.rht_forward(W, 99, s)
    d = orc.signs(99, K)
    H = indep.sylvester(n)
    DW = W.astype(np.int64) * d[None, :]
    ref = np.concatenate([DW[:, b:b + n] @ H for b in range(0, K, n)], axis=1)
    assert np.array_equal(U.astype(np.int64), ref)


# ------------------------------------------------------------ exact compare --

def _frac_sign(u, Za, Zb, den):
    da = sum((Fraction(float(x)) - Fraction(int(a), den)) ** 2 for x, a in zip(u, Za))
    db = sum((Fraction(float(x)) - Fraction(int(b), den)) ** 2 for x, b in zip(u, Zb))
    return (da > db) - (da < db)


def test_exact_compare_matches_rationals():
    rng = np.random.default_rng(3)
    for t in range(3000):
        den = [2, 4, 8][t % 3]
        Za = rng.integers(-30, 31, 8)
        Zb = rng.integers(-30, 31, 8)
        kind = t % 5
        if kind == 0:
            u = rng.standard_normal(8).astype(np.float32)
        elif kind == 1:   # mixed magnitudes
            u = (rng.standard_normal(8) * 10.0 ** rng.integers(-30, 30, 8)).astype(np.float32)
        elif kind == 2:   # exact midpoint: a tie by construction
            u = ((Za + Zb) / (2.0 * den)).astype(np.float32)
        elif kind == 3:   # midpoint nudged by one ulp in one coordinate
            u = ((Za + Zb) / (2.0 * den)).astype(np.float32)
            j = rng.integers(8)
            u[j] = np.nextafter(u[j], np.float32(np.inf))
        else:             # denormals and huge values
            u = rng.choice(np.array([1e-45, -3e-42, 1e-38, 3e38, -1e30, 0.0, 0.5, -0.25],
                                    dtype=np.float32), 8)
        assert orc.cmp_dist(u, Za, Zb, den) == _frac_sign(u, Za, Zb, den)


# ---------------------------------------------------------- nearest point --

@pytest.mark.parametrize("sigma", [0.3, 1.0, 2.5])
def test_stage1_matches_independent_bruteforce(cb, sigma):
    rng = np.random.default_rng(int(sigma * 10))
    U = (rng.standard_normal((40, 8)) * sigma).astype(np.float32)
    i1, _ = orc.nearest_groups(U, 2)
    for g in range(len(U)):
        assert i1[g] == indep.stage1_exact(U[g], cb)


@pytest.mark.parametrize("bpw,sigma", [(3, 1.0), (4, 0.9), (4, 3.0)])
def test_stage2_matches_independent_bruteforce(cb, bpw, sigma):
    rng = np.random.default_rng(bpw * 7)
    U = (rng.standard_normal((24, 8)) * sigma).astype(np.float32)
    i1, i2 = orc.nearest_groups(U, bpw)
    for g in range(len(U)):
        assert i1[g] == indep.stage1_exact(U[g], cb)
        assert i2[g] == indep.stage2_exact(U[g], cb, int(i1[g]), bpw)
    if bpw == 3:
        assert i2.dtype == np.uint8


def test_codebook_points_map_to_themselves(cb):
    rng = np.random.default_rng(1)
    sel = np.concatenate([np.arange(0, 300), rng.integers(0, 65536, 400), [65534, 65535]])
    U = (cb[sel].astype(np.float32) / 2)
    i1, _ = orc.nearest_groups(U, 2)
    assert np.array_equal(i1, sel.astype(np.uint16))


def test_ties_go_to_smallest_index(cb):
    geo = _gold("e8_geometry.json")
    hole = np.array(geo["deep_hole"]["point"], dtype=np.float32)
    rng = np.random.default_rng(2)
    U = [hole, -hole, np.roll(hole, 3)]
    # midpoints between random codebook points and random lattice neighbours
    roots = cb[1:241].astype(np.int64)
    for _ in range(40):
        a = cb[rng.integers(0, 20000)].astype(np.int64)
        b = a + roots[rng.integers(0, 240)]
        U.append(((a + b) / 4.0).astype(np.float32))
    U = np.array(U, dtype=np.float32)
    i1, _ = orc.nearest_groups(U, 2)
    assert i1[0] == 0 and i1[1] == 0 and i1[2] == 0
    for g in range(len(U)):
        assert i1[g] == indep.stage1_exact(U[g], cb)
    # at the deep hole exactly 16 lattice points are nearest, at distance 1
    d = ((cb.astype(np.float64) / 2 - hole[None, :]) ** 2).sum(1)
    assert (d == geo["covering_radius"] ** 2).sum() == geo["deep_hole"]["nearest_points"]


def test_nonfinite_groups_get_index_zero():
    U = np.array([[np.nan, 0, 0, 0, 0, 0, 0, 0], [np.inf, 1, 1, 1, 1, 1, 1, 1]], np.float32)
    i1, i2 = orc.nearest_groups(U, 4)
    assert not i1.any() and not i2.any()


def test_stage1_error_matches_e8_second_moment(cb):
    geo = _gold("e8_geometry.json")
    G = geo["normalized_second_moment"]["numerator"] / geo["normalized_second_moment"]["denominator"]
    # uniform on [-1, 1)^8 is uniform modulo E8 (2Z^8 is a sublattice), so the
    # quantisation error is uniform on a Voronoi cell, whose mean squared norm
    # per dimension is G for the unit-volume lattice
    rng = np.random.default_rng(7)
    U = rng.uniform(-1.0, 1.0, size=(16000, 8)).astype(np.float32)
    i1, _ = orc.nearest_groups(U, 2)
    r = U.astype(np.float64) - cb[i1].astype(np.float64) / 2
    d2 = (r ** 2).sum(1)
    assert d2.max() <= geo["covering_radius"] ** 2 + 1e-12
    mse = d2.mean() / 8
    se = d2.std() / 8 / np.sqrt(len(d2))
    assert abs(mse - G) < 5 * se + 1e-4, (mse, G, se)


# ------------------------------------------------------ encode / decode --

def _planted(cb, N, K, bpw, seed, s, rht_seed):
    rng = np.random.default_rng(seed)
    G = N * K // 8
    i1 = rng.integers(0, 65536, G)
    m = {2: 2, 3: 4, 4: 8}[bpw]
    z = cb[i1].astype(np.int64) * (m // 2)
    i2 = None
    if bpw > 2:
        n2 = (cb.astype(np.int64) ** 2).sum(1) // 4
        if bpw == 4:
            ok = np.nonzero(n2 <= 6)[0]           # beta |c2| <= sqrt(6)/4 < 1/sqrt(2)
        else:
            ok = np.array([0])                    # beta = 1/2: only c2 = 0 stays inside
        i2 = ok[rng.integers(0, len(ok), G)]
        z = z + cb[i2].astype(np.int64)
    nh = orc.hadamard_block(K)
    H = indep.sylvester(nh)
    d = orc.signs(rht_seed, K)
    Z = z.reshape(N, K)
    T = np.concatenate([Z[:, b:b + nh] @ H for b in range(0, K, nh)], axis=1)
    W = (s * d[None, :] * T / (m * np.sqrt(nh))).astype(np.float32)
    return W, i1.reshape(N, K // 8), (None if i2 is None else i2.reshape(N, K // 8))


@pytest.mark.parametrize("bpw,K", [(2, 256), (3, 1024), (4, 3072)])
def test_planted_codes_round_trip(cb, bpw, K):
    N, s, rs = 8, 0.037, 123
    W, i1, i2 = _planted(cb, N, K, bpw, 40 + bpw, s, rs)
    e1, e2 = orc.encode(W, bpw, rs, s)
    assert np.array_equal(e1, i1.astype(np.uint16))
    if bpw > 2:
        assert np.array_equal(e2.astype(np.int64), i2)
    wd = orc.bf16_bits_to_f32(orc.decode(e1, e2, N, K, bpw, rs, s))
    # decoded weights reproduce the planted matrix to bf16 precision
    err = np.abs(wd.astype(np.float64) - W.astype(np.float64))
    assert np.all(err <= np.abs(W) * 2.0 ** -8 + 1e-12)


def test_decode_of_origin_is_zero():
    N, K = 4, 512
    out = orc.decode(np.zeros((N, K // 8), np.uint16), np.zeros((N, K // 8), np.uint16), N, K,
                     4, 1, 0.5)
    # zero times a negative column sign is -0 (bit pattern 0x8000), as IEEE has it
    assert np.all(orc.bf16_bits_to_f32(out) == 0.0)
    d = orc.signs(1, K)
    assert np.array_equal(out[0] == 0x8000, d < 0)


def test_decode_is_odd_in_the_pair_index(cb):
    # entry 2k+2 = -(entry 2k+1); with one nonzero group per row the decoded
    # rows for i and its pair partner are exact negatives
    N, K = 2, 256
    i1 = np.zeros((N, K // 8), np.uint16)
    i1[0, 3], i1[1, 3] = 1001, 1002
    out = orc.bf16_bits_to_f32(orc.decode(i1, None, N, K, 2, 9, 0.11))
    assert np.array_equal(out[0], -out[1]) and np.any(out[0] != 0)


def test_gemm_matches_numpy():
    rng = np.random.default_rng(0)
    from decode_gemm_e8_b200 import synth
    X = synth.activations_bf16(7, 264, 1)
    W = synth.f32_to_bf16_bits((rng.standard_normal((33, 264)) * 0.02).astype(np.float32))
    Y = orc.gemm(X, W)
    ref = synth.bf16_bits_to_f32(X).astype(np.float64) @ synth.bf16_bits_to_f32(W).astype(np.float64).T
    assert np.allclose(Y, ref, rtol=1e-13, atol=1e-13)

"""Plain CPU oracle of the entropy-coded E8 variant (numpy and Python loops).

TEST INFRASTRUCTURE ONLY: only ``tests/``, ``__graft_entry__.smoke()`` and the
``cpu_baseline`` / ``--impl reference`` legs of ``bench.py`` may import this
module.  The library under ``decode_gemm_e8_b200`` never does, and this module
imports nothing from it.

Source: page "Transformers Proposes EntroPack Integration for Configurable
Non-Integer-Bit-Rate Weight Compression", second paragraph (per-row normalised
E8 lattice quantisation, a conditional probability model and entropy coding;
the coded coordinates split into independently decodable blocks; the GPU
decodes the symbols and rebuilds the weights in one pass) and third paragraph
(the actual storage rate counts the metadata).  The page fixes none of the
details; this oracle takes the plainest reading of each (every one is listed
among the readings of the pages in the design notes):

  row normalisation   s_n = max_k |w_nk| (exact in any order), t_n = fl32(s_n delta)
                      for a global step delta >= 1/120, g_n = fl32(1 / t_n)
                      (0 when t_n is below the smallest normal fp32);
  lattice point       u = fl32(w g_n) per group of 8; V = nearest point of the
                      whole E8 lattice in doubled coordinates by Conway & Sloane
                      ("Sphere Packings, Lattices and Groups", ch. 20: E8 = D8 u
                      (D8 + 1/2)) with fixed tie rules, in fp32:
                        D8: f = rint(u) (ties to even); if sum f is odd, move the
                            coordinate farthest from its rounding (first index on
                            ties) one step towards u (up when u_j >= f_j);
                        D8 + 1/2: b = floor(u), h = b + 1/2; if sum b is odd, move
                            the coordinate farthest from h (first index on ties)
                            one step towards u (up when u_j >= h_j);
                        squared distances summed in coordinate order in fp32
                        (no fused operations); D8 wins ties;
                        V = 2 f, or 2 b + 1;
  reconstruction      w' = bf16_rne(fl32(V * a_n)), a_n = fl32(t_n / 2) (exact);
  symbols per group   coset c = V mod 2; m_i = (V_i - c) / 2 for i < 7; the E8
                      rule sum m even fixes m_7 mod 2, so only q = floor(m_7 / 2)
                      is coded: 9 symbols, c, m_0 .. m_6, q;
  probability model   conditional on the coset: P(c), P(m | c) shared by the
                      seven positions, P(q | c); frequencies counted over the
                      matrix, normalised to 4096 by the integer rule of
                      `normalise`;
  entropy coder       rANS (Duda, "Asymmetric numeral systems: entropy coding
                      combining speed of Huffman coding with compression rate
                      of arithmetic coding", 2013) with a 32-bit state in
                      [2^16, 2^32), 16-bit output words, 12-bit frequencies;
  blocks              64 consecutive groups of the row-major matrix per block,
                      each block its own rANS stream (independently decodable):
                      [x >> 16, x & 0xFFFF] of the final encoder state, then the
                      emitted words, last emitted first; offsets[b] = first word
                      of block b, offsets[nblocks] = total words;
  actual bpp          (16 words + 32 (nblocks + 1) + 32 N + 16 * 770 + 32) / (N K):
                      stream, offsets, row scales t_n, the five frequency tables
                      (2 + 2 * 256 + 2 * 128 entries of 16 bits) and delta.
"""
from __future__ import annotations

import numpy as np

SCALE_BITS = 12
M_TOTAL = 1 << SCALE_BITS
RANS_L = 1 << 16
BLOCK_GROUPS = 64
SYMS_PER_GROUP = 9
M_OFF, M_SIZE = 128, 256     # m in [-128, 127]
Q_OFF, Q_SIZE = 64, 128      # q in [-64, 63]
TABLE_ENTRIES = 2 + 2 * M_SIZE + 2 * Q_SIZE
DELTA_MIN = np.float32(1.0 / 120.0)
F32_MIN_NORMAL = np.float32(np.finfo(np.float32).tiny)


# ----------------------------------------------------------------- quantiser --
def row_scales(W: np.ndarray, delta: float) -> tuple[np.ndarray, np.ndarray]:
    """(t_n, g_n): t_n = fl32(max|w_n| * delta), g_n = fl32(1 / t_n) or 0."""
    W = np.asarray(W, dtype=np.float32)
    d = np.float32(delta)
    s = np.max(np.abs(W), axis=1).astype(np.float32) if W.shape[1] else np.zeros(W.shape[0], np.float32)
    t = (s * d).astype(np.float32)
    g = np.zeros_like(t)
    ok = t >= F32_MIN_NORMAL
    g[ok] = (np.float32(1.0) / t[ok]).astype(np.float32)
    t[~ok] = np.float32(0.0)
    return t, g


def _sq_dist(e: np.ndarray) -> np.ndarray:
    """Sum over the last axis of e^2 in coordinate order, fp32, no fusion."""
    acc = np.zeros(e.shape[:-1], dtype=np.float32)
    for i in range(e.shape[-1]):
        acc = (acc + (e[..., i] * e[..., i]).astype(np.float32)).astype(np.float32)
    return acc


def nearest_e8(u: np.ndarray) -> np.ndarray:
    """Doubled coordinates V (int32 [..., 8]) of the E8 point the quantiser picks."""
    u = np.asarray(u, dtype=np.float32)
    shp = u.shape
    u = u.reshape(-1, 8)
    n = u.shape[0]
    rows = np.arange(n)
    # D8 candidate
    f = np.rint(u).astype(np.float32)
    e = (u - f).astype(np.float32)
    odd = (np.sum(f.astype(np.int64), axis=1) & 1) == 1
    j = np.argmax(np.abs(e), axis=1)
    step = np.where(u[rows, j] >= f[rows, j], np.float32(1), np.float32(-1))
    f[rows[odd], j[odd]] += step[odd]
    eD = (u - f).astype(np.float32)
    dD = _sq_dist(eD)
    # D8 + 1/2 candidate
    b = np.floor(u).astype(np.float32)
    h = (b + np.float32(0.5)).astype(np.float32)
    eh = (u - h).astype(np.float32)
    oddh = (np.sum(b.astype(np.int64), axis=1) & 1) == 1
    jh = np.argmax(np.abs(eh), axis=1)
    steph = np.where(u[rows, jh] >= h[rows, jh], np.float32(1), np.float32(-1))
    b[rows[oddh], jh[oddh]] += steph[oddh]
    eH = (u - (b + np.float32(0.5)).astype(np.float32)).astype(np.float32)
    dH = _sq_dist(eH)
    V = np.where((dD <= dH)[:, None], 2 * f.astype(np.int64), 2 * b.astype(np.int64) + 1)
    return V.astype(np.int32).reshape(shp)


def quantise(W: np.ndarray, delta: float) -> tuple[np.ndarray, np.ndarray]:
    """(V int32 [N, K] doubled coordinates, t float32 [N])."""
    W = np.asarray(W, dtype=np.float32)
    if not np.float32(delta) >= DELTA_MIN:
        raise ValueError("delta below 1/120")
    N, K = W.shape
    t, g = row_scales(W, delta)
    u = (W * g[:, None]).astype(np.float32)
    return nearest_e8(u.reshape(N, K // 8, 8)).reshape(N, K), t


def symbols(V: np.ndarray) -> np.ndarray:
    """Per group the 9 coded values (c, m_0..m_6, q), int32 [G, 9]."""
    G = V.reshape(-1, 8).astype(np.int64)
    c = G[:, 0] & 1
    m = (G - c[:, None]) >> 1
    out = np.empty((G.shape[0], SYMS_PER_GROUP), dtype=np.int32)
    out[:, 0] = c
    out[:, 1:8] = m[:, :7]
    out[:, 8] = m[:, 7] >> 1
    return out


def values_from_symbols(S: np.ndarray) -> np.ndarray:
    """Inverse of `symbols`: doubled coordinates int32 [G, 8]."""
    S = np.asarray(S, dtype=np.int64)
    c = S[:, 0]
    m7 = 2 * S[:, 8] + (np.sum(S[:, 1:8], axis=1) & 1)
    m = np.concatenate([S[:, 1:8], m7[:, None]], axis=1)
    return (2 * m + c[:, None]).astype(np.int32)


# ------------------------------------------------------- probability model --
def normalise(counts: np.ndarray) -> np.ndarray:
    """Frequencies summing to 4096: floor(n_s 4096 / total), at least 1 for a
    symbol that occurs; the difference goes to the most frequent symbol
    (smallest index on ties) while it stays >= 1, the rest is taken one unit at
    a time from the largest frequencies above 1 (smallest index first).  An
    alphabet with no occurrences gets all 4096 on symbol 0."""
    counts = np.asarray(counts, dtype=np.int64)
    total = int(counts.sum())
    f = np.zeros(counts.shape[0], dtype=np.int64)
    if total == 0:
        f[0] = M_TOTAL
        return f.astype(np.int32)
    for s in range(counts.shape[0]):
        if counts[s]:
            f[s] = max(1, (int(counts[s]) * M_TOTAL) // total)
    diff = M_TOTAL - int(f.sum())
    big = int(np.argmax(counts))
    if f[big] + diff >= 1:
        f[big] += diff
    else:
        diff += int(f[big]) - 1
        f[big] = 1
        while diff < 0:
            s = int(np.argmax(f))
            if f[s] <= 1:
                raise ValueError("alphabet larger than the frequency scale")
            f[s] -= 1
            diff += 1
    return f.astype(np.int32)


def tables(S: np.ndarray) -> dict:
    """Normalised frequency tables of the five models from the symbols."""
    S = np.asarray(S, dtype=np.int64)
    c = S[:, 0]
    t = {"c": normalise(np.bincount(c, minlength=2))}
    for cc in (0, 1):
        sel = S[c == cc]
        t["m%d" % cc] = normalise(np.bincount((sel[:, 1:8] + M_OFF).ravel(), minlength=M_SIZE))
        t["q%d" % cc] = normalise(np.bincount(sel[:, 8] + Q_OFF, minlength=Q_SIZE))
    return t


def table_words(t: dict) -> np.ndarray:
    """The tables as stored: uint16 [770] = c, m0, m1, q0, q1."""
    return np.concatenate([t["c"], t["m0"], t["m1"], t["q0"], t["q1"]]).astype(np.uint16)


def tables_from_words(w: np.ndarray) -> dict:
    w = np.asarray(w, dtype=np.int64)
    o = [0, 2, 2 + M_SIZE, 2 + 2 * M_SIZE, 2 + 2 * M_SIZE + Q_SIZE, TABLE_ENTRIES]
    names = ["c", "m0", "m1", "q0", "q1"]
    return {k: w[o[i]:o[i + 1]].astype(np.int32) for i, k in enumerate(names)}


def _model_seq(group_syms, t):
    """(frequency table, symbol index) of each of a group's 9 symbols."""
    c = int(group_syms[0])
    seq = [(t["c"], c)]
    for i in range(1, 8):
        seq.append((t["m%d" % c], int(group_syms[i]) + M_OFF))
    seq.append((t["q%d" % c], int(group_syms[8]) + Q_OFF))
    return seq


# ------------------------------------------------------------------- rANS --
def rans_encode(seq: list) -> list:
    """Stream words of one block: seq = [(freq table, symbol), ...] in decode
    order.  Encodes last to first from x = 2^16."""
    cums = {}
    x = RANS_L
    emitted = []
    for f_tab, s in reversed(seq):
        key = id(f_tab)
        if key not in cums:
            cums[key] = np.concatenate([[0], np.cumsum(f_tab)]).astype(np.int64)
        f = int(f_tab[s])
        cum = int(cums[key][s])
        if f <= 0:
            raise ValueError("symbol with zero frequency")
        if x >= (f << (32 - SCALE_BITS)):
            emitted.append(x & 0xFFFF)
            x >>= 16
        x = ((x // f) << SCALE_BITS) + (x % f) + cum
    return [x >> 16, x & 0xFFFF] + emitted[::-1]


def rans_decode(words, models: list, nsym_per_model=None):
    """Decodes len(models) symbols; models[i] = frequency table of symbol i.
    Returns (symbols, final state, words read)."""
    x = (int(words[0]) << 16) | int(words[1])
    p = 2
    out = []
    for f_tab in models:
        cum = np.concatenate([[0], np.cumsum(f_tab)]).astype(np.int64)
        slot = x & (M_TOTAL - 1)
        s = int(np.searchsorted(cum, slot, side="right") - 1)
        x = int(f_tab[s]) * (x >> SCALE_BITS) + slot - int(cum[s])
        if x < RANS_L:
            x = (x << 16) | int(words[p])
            p += 1
        out.append(s)
    return out, x, p


# ------------------------------------------------------------ whole matrix --
def encode(W: np.ndarray, delta: float) -> dict:
    """Compressed form of W at step delta: words, offsets, t, table words."""
    W = np.asarray(W, dtype=np.float32)
    N, K = W.shape
    V, t = quantise(W, delta)
    S = symbols(V)
    tb = tables(S)
    G = S.shape[0]
    nb = (G + BLOCK_GROUPS - 1) // BLOCK_GROUPS
    words = []
    offsets = [0]
    for b in range(nb):
        seq = []
        for g in range(b * BLOCK_GROUPS, min(G, (b + 1) * BLOCK_GROUPS)):
            seq.extend(_model_seq(S[g], tb))
        blk = rans_encode(seq)
        words.extend(blk)
        offsets.append(offsets[-1] + len(blk))
    return {"N": N, "K": K, "delta": np.float32(delta), "t": t,
            "tables": table_words(tb), "words": np.array(words, dtype=np.uint16),
            "offsets": np.array(offsets, dtype=np.uint32)}


def decode_block_symbols(enc: dict, b: int) -> np.ndarray:
    """Symbols int32 [groups, 9] of block b, read from its own stream only."""
    tb = tables_from_words(enc["tables"])
    G = enc["N"] * enc["K"] // 8
    ng = min(G, (b + 1) * BLOCK_GROUPS) - b * BLOCK_GROUPS
    w = enc["words"][int(enc["offsets"][b]):int(enc["offsets"][b + 1])]
    x = (int(w[0]) << 16) | int(w[1])
    p = 2
    out = np.empty((ng, SYMS_PER_GROUP), dtype=np.int32)
    cums = {k: np.concatenate([[0], np.cumsum(v)]).astype(np.int64) for k, v in tb.items()}

    def step(name):
        nonlocal x, p
        f_tab, cum = tb[name], cums[name]
        slot = x & (M_TOTAL - 1)
        s = int(np.searchsorted(cum, slot, side="right") - 1)
        x = int(f_tab[s]) * (x >> SCALE_BITS) + slot - int(cum[s])
        if x < RANS_L:
            x = (x << 16) | int(w[p])
            p += 1
        return s

    for g in range(ng):
        c = step("c")
        out[g, 0] = c
        for i in range(1, 8):
            out[g, i] = step("m%d" % c) - M_OFF
        out[g, 8] = step("q%d" % c) - Q_OFF
    if x != RANS_L or p != len(w):
        raise ValueError("block %d: stream not consumed exactly" % b)
    return out


def f32_to_bf16_bits(x: np.ndarray) -> np.ndarray:
    """Round-to-nearest-even fp32 -> bf16 bit patterns (finite inputs)."""
    u = np.asarray(x, dtype=np.float32).view(np.uint32).astype(np.uint64)
    r = (u + 0x7FFF + ((u >> 16) & 1)) >> 16
    return r.astype(np.uint16)


def reconstruct(V: np.ndarray, t: np.ndarray) -> np.ndarray:
    """bf16 bits [N, K]: bf16_rne(fl32(V * fl32(t_n / 2)))."""
    a = (np.asarray(t, dtype=np.float32) * np.float32(0.5)).astype(np.float32)
    w = (np.asarray(V, dtype=np.float32) * a[:, None]).astype(np.float32)
    return f32_to_bf16_bits(w)


def decode(enc: dict, blocks=None) -> np.ndarray:
    """bf16 bits [N, K] of the whole matrix (blocks=None) or of the listed
    blocks' groups only (other entries 0)."""
    N, K = enc["N"], enc["K"]
    G = N * K // 8
    nb = len(enc["offsets"]) - 1
    V = np.zeros((G, 8), dtype=np.int32)
    for b in (range(nb) if blocks is None else blocks):
        S = decode_block_symbols(enc, b)
        V[b * BLOCK_GROUPS:b * BLOCK_GROUPS + S.shape[0]] = values_from_symbols(S)
    return reconstruct(V.reshape(N, K), enc["t"])


def actual_bpp(enc: dict) -> float:
    N, K = enc["N"], enc["K"]
    nb = len(enc["offsets"]) - 1
    bits = 16 * int(enc["offsets"][-1]) + 32 * (nb + 1) + 32 * N + 16 * TABLE_ENTRIES + 32
    return bits / float(N * K)


def gemm(Xbits: np.ndarray, Wbits: np.ndarray) -> np.ndarray:
    """Binary64 product X W^T of bf16 bit patterns (X [M, K], W [N, K])."""
    def f(b):
        return (np.asarray(b, dtype=np.uint16).astype(np.uint32) << 16).view(np.float32).astype(np.float64)
    return f(Xbits) @ f(Wbits).T

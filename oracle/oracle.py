"""Python handle on the plain CPU oracle (``e8_oracle.c``).

TEST INFRASTRUCTURE ONLY: only ``tests/``, ``__graft_entry__.smoke()`` and the
``cpu_baseline`` / ``--impl reference`` legs of ``bench.py`` may import this
module.  The library under ``decode_gemm_e8_b200`` never does, and this module
imports nothing from it.

The oracle follows the "glq 0.1.1" PyPI page ("How it works", items 1-2, and
the "Bit widths" table): an E8-lattice codebook of 65536 vectors from the first
seven shells, a randomized Hadamard transform (sign flips, then a fast
Walsh-Hadamard transform) of each weight row, Euclidean nearest codebook vector
per group of 8 weights, an optional second-stage residual codebook (8 or 16 more
bits per group), and one global scale per layer.
"""
from __future__ import annotations

import ctypes
import os
import subprocess

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "e8_oracle.c")
_LIB_DIR = os.path.join(_HERE, "_build")
_LIB = os.path.join(_LIB_DIR, "libe8oracle.so")

CB_SIZE = 65536
_lib = None
_cb_cache = None


def build(force: bool = False) -> str:
    """Compile the oracle with gcc (IEEE arithmetic: no contraction, no fast-math)."""
    os.makedirs(_LIB_DIR, exist_ok=True)
    if not force and os.path.exists(_LIB) and os.path.getmtime(_LIB) >= os.path.getmtime(_SRC):
        return _LIB
    tmp = _LIB + ".tmp%d" % os.getpid()
    cmd = ["gcc", "-std=gnu11", "-O2", "-fopenmp", "-ffp-contract=off", "-fno-fast-math",
           "-fPIC", "-shared", "-Wall", "-o", tmp, _SRC, "-lm"]
    subprocess.check_call(cmd)
    os.replace(tmp, _LIB)
    return _LIB


def _load():
    global _lib
    if _lib is not None:
        return _lib
    lib = ctypes.CDLL(build())
    c = ctypes
    P = c.c_void_p
    lib.orc_codebook.argtypes = [P]
    lib.orc_codebook.restype = c.c_int
    lib.orc_hadamard_block.argtypes = [c.c_int64]
    lib.orc_hadamard_block.restype = c.c_int64
    lib.orc_signs.argtypes = [c.c_uint64, c.c_int64, P]
    lib.orc_signs.restype = None
    lib.orc_gamma.argtypes = [c.c_float, c.c_int64]
    lib.orc_gamma.restype = c.c_float
    lib.orc_alpha.argtypes = [c.c_float, c.c_int64, c.c_int]
    lib.orc_alpha.restype = c.c_float
    lib.orc_rht_forward.argtypes = [P, c.c_int64, c.c_int64, c.c_uint64, c.c_float, P, c.c_int]
    lib.orc_rht_forward.restype = c.c_int
    lib.orc_cmp_dist.argtypes = [P, P, P, c.c_int]
    lib.orc_cmp_dist.restype = c.c_int
    lib.orc_nearest_groups.argtypes = [P, c.c_int64, c.c_int, P, P, P, c.c_int]
    lib.orc_nearest_groups.restype = c.c_int
    lib.orc_encode.argtypes = [P, c.c_int64, c.c_int64, c.c_int, c.c_uint64, c.c_float, P, P, P,
                               c.c_int]
    lib.orc_encode.restype = c.c_int
    lib.orc_decode.argtypes = [P, P, c.c_int64, c.c_int64, c.c_int, c.c_uint64, c.c_float, P, P,
                               c.c_int]
    lib.orc_decode.restype = c.c_int
    lib.orc_valid_block.argtypes = [c.c_int64, c.c_int64]
    lib.orc_valid_block.restype = c.c_int
    lib.orc_rht_forward_nh.argtypes = [P, c.c_int64, c.c_int64, c.c_int64, c.c_uint64, c.c_float,
                                       P, c.c_int]
    lib.orc_rht_forward_nh.restype = c.c_int
    lib.orc_encode_nh.argtypes = [P, c.c_int64, c.c_int64, c.c_int64, c.c_int, c.c_uint64,
                                  c.c_float, P, P, P, c.c_int]
    lib.orc_encode_nh.restype = c.c_int
    lib.orc_decode_nh.argtypes = [P, P, c.c_int64, c.c_int64, c.c_int64, c.c_int, c.c_uint64,
                                  c.c_float, P, P, c.c_int]
    lib.orc_decode_nh.restype = c.c_int
    lib.orc_gemm.argtypes = [P, c.c_int64, P, c.c_int64, c.c_int64, P, c.c_int]
    lib.orc_gemm.restype = c.c_int
    lib.orc_max_threads.argtypes = []
    lib.orc_max_threads.restype = c.c_int
    _lib = lib
    return lib


def _ptr(a: np.ndarray):
    assert a.flags["C_CONTIGUOUS"]
    return ctypes.c_void_p(a.ctypes.data)


def threads(n: int | None = None) -> int:
    return int(n) if n else int(_load().orc_max_threads())


def codebook() -> np.ndarray:
    """The 65536 codebook vectors in canonical order, doubled coordinates, int8 [65536, 8]."""
    global _cb_cache
    if _cb_cache is None:
        cb = np.zeros((CB_SIZE, 8), dtype=np.int8)
        n = _load().orc_codebook(_ptr(cb))
        if n != 117361:
            raise RuntimeError("oracle codebook enumeration failed (%d)" % n)
        cb.setflags(write=False)
        _cb_cache = cb
    return _cb_cache


def hadamard_block(K: int) -> int:
    return int(_load().orc_hadamard_block(K))


def valid_block(K: int, nh: int) -> bool:
    """n_h is a power of two, 8 <= n_h <= 32768, dividing K (K a multiple of 8)."""
    return bool(_load().orc_valid_block(K, nh))


def signs(rht_seed: int, K: int) -> np.ndarray:
    d = np.zeros(K, dtype=np.int8)
    _load().orc_signs(ctypes.c_uint64(rht_seed & (2**64 - 1)), K, _ptr(d))
    return d


def gamma(scale: float, nh: int) -> float:
    return float(_load().orc_gamma(scale, nh))


def alpha(scale: float, nh: int, bpw: int) -> float:
    return float(_load().orc_alpha(scale, nh, bpw))


def rht_forward(W: np.ndarray, rht_seed: int, scale: float, nthreads: int | None = None,
                nh: int | None = None) -> np.ndarray:
    """u = fl32(FWHT(D w) * gamma) per row, in Hadamard blocks of the default size
    (largest power of two dividing K) or of `nh`."""
    W = np.ascontiguousarray(W, dtype=np.float32)
    N, K = W.shape
    U = np.empty_like(W)
    if nh is None:
        rc = _load().orc_rht_forward(_ptr(W), N, K, ctypes.c_uint64(rht_seed), scale, _ptr(U),
                                     threads(nthreads))
    else:
        rc = _load().orc_rht_forward_nh(_ptr(W), N, K, nh, ctypes.c_uint64(rht_seed), scale,
                                        _ptr(U), threads(nthreads))
    if rc != 0:
        raise ValueError("bad shape for the RHT (K=%d)" % K)
    return U


def cmp_dist(u, Za, Zb, den: int) -> int:
    """Exact sign of |u - Za/den|^2 - |u - Zb/den|^2 (+1: b strictly closer)."""
    u = np.ascontiguousarray(u, dtype=np.float32)
    Za = np.ascontiguousarray(Za, dtype=np.int32)
    Zb = np.ascontiguousarray(Zb, dtype=np.int32)
    return int(_load().orc_cmp_dist(_ptr(u), _ptr(Za), _ptr(Zb), den))


def _idx2_alloc(bpw: int, shape):
    if bpw == 2:
        return None
    return np.zeros(shape, dtype=np.uint8 if bpw == 3 else np.uint16)


def nearest_groups(U: np.ndarray, bpw: int, nthreads: int | None = None):
    """Exact nearest-point indices for transformed groups U [..., 8] (brute force)."""
    U = np.ascontiguousarray(U, dtype=np.float32)
    G = U.size // 8
    i1 = np.zeros(G, dtype=np.uint16)
    i2 = _idx2_alloc(bpw, G)
    rc = _load().orc_nearest_groups(_ptr(U), G, bpw, _ptr(codebook()), _ptr(i1),
                                    _ptr(i2) if i2 is not None else None, threads(nthreads))
    if rc != 0:
        raise RuntimeError("oracle nearest failed")
    return i1, i2


def encode(W: np.ndarray, bpw: int, rht_seed: int, scale: float, nthreads: int | None = None,
           nh: int | None = None):
    """idx1 [N, K/8] uint16 and idx2 [N, K/8] (uint8 for 3 bpw, uint16 for 4 bpw, None for 2).
    `nh`: Hadamard block size (default: the largest power of two dividing K)."""
    W = np.ascontiguousarray(W, dtype=np.float32)
    N, K = W.shape
    i1 = np.zeros((N, K // 8), dtype=np.uint16)
    i2 = _idx2_alloc(bpw, (N, K // 8))
    p2 = _ptr(i2) if i2 is not None else None
    if nh is None:
        rc = _load().orc_encode(_ptr(W), N, K, bpw, ctypes.c_uint64(rht_seed), scale,
                                _ptr(codebook()), _ptr(i1), p2, threads(nthreads))
    else:
        rc = _load().orc_encode_nh(_ptr(W), N, K, nh, bpw, ctypes.c_uint64(rht_seed), scale,
                                   _ptr(codebook()), _ptr(i1), p2, threads(nthreads))
    if rc != 0:
        raise ValueError("oracle encode rejected the arguments")
    return i1, i2


def decode(idx1: np.ndarray, idx2, N: int, K: int, bpw: int, rht_seed: int, scale: float,
           nthreads: int | None = None, nh: int | None = None) -> np.ndarray:
    """Decoded weights as raw bf16 bit patterns, uint16 [N, K].
    `nh`: Hadamard block size (default: the largest power of two dividing K)."""
    idx1 = np.ascontiguousarray(idx1, dtype=np.uint16)
    if idx2 is not None:
        idx2 = np.ascontiguousarray(idx2, dtype=np.uint8 if bpw == 3 else np.uint16)
    out = np.zeros((N, K), dtype=np.uint16)
    p2 = _ptr(idx2) if idx2 is not None else None
    if nh is None:
        rc = _load().orc_decode(_ptr(idx1), p2, N, K, bpw, ctypes.c_uint64(rht_seed), scale,
                                _ptr(codebook()), _ptr(out), threads(nthreads))
    else:
        rc = _load().orc_decode_nh(_ptr(idx1), p2, N, K, nh, bpw, ctypes.c_uint64(rht_seed),
                                   scale, _ptr(codebook()), _ptr(out), threads(nthreads))
    if rc != 0:
        raise ValueError("oracle decode rejected the arguments")
    return out


def gemm(X_bf16: np.ndarray, W_bf16: np.ndarray, nthreads: int | None = None) -> np.ndarray:
    """Y = X W^T in binary64 from bf16 bit patterns X [M, K], W [N, K]."""
    X = np.ascontiguousarray(X_bf16, dtype=np.uint16)
    W = np.ascontiguousarray(W_bf16, dtype=np.uint16)
    M, K = X.shape
    N = W.shape[0]
    Y = np.zeros((M, N), dtype=np.float64)
    _load().orc_gemm(_ptr(X), M, _ptr(W), N, K, _ptr(Y), threads(nthreads))
    return Y


def bf16_bits_to_f32(b: np.ndarray) -> np.ndarray:
    return (np.asarray(b, dtype=np.uint16).astype(np.uint32) << 16).view(np.float32)

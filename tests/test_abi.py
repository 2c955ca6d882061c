"""The C-ABI library loads on the CPU host and exports every symbol that
include/e8.h declares; host-only entry points answer without a GPU."""
import os
import re

import pytest

import decode_gemm_e8_b200 as e8
from decode_gemm_e8_b200 import build as e8build

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _declared():
    src = open(os.path.join(ROOT, "include", "e8.h")).read()
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    return sorted(set(re.findall(r"\b(e8_[a-z0-9_]+)\s*\(", src)))


@pytest.fixture(scope="module")
def lib():
    e8build.build()
    return e8.load_library()


def test_every_declared_symbol_is_exported(lib):
    names = _declared()
    assert "e8_gemm" in names and "e8_encode" in names and len(names) >= 12
    for n in names:
        assert hasattr(lib, n), n
    assert set(names) == set(e8.EXPORTED)


def test_library_is_sm100a_only():
    # the build passes exactly one -gencode, for sm_100a
    assert e8build.ARCH == ["-gencode", "arch=compute_100a,code=sm_100a"]


def test_status_strings_and_version(lib):
    assert e8.status_str(0) == "ok"
    assert "timed out" in e8.status_str(5)
    assert e8.e8_version() >= 100


def test_workspace_sizes(lib):
    N, K = 4096, 4096
    # two work lists of one 48-byte item per group (undecided groups of the
    # fast path, then what the class search leaves open)
    assert e8.e8_workspace_bytes(e8.E8_OP_ENCODE, 0, N, K, 4) == 256 + 2 * 48 * N * K // 8
    assert e8.e8_workspace_bytes(e8.E8_GEMM_DECODED_W, 4096, N, K, 3) == N * K * 2
    # int8 pieces for 16 tokens: 32 rows of K bytes, then 16 steps
    assert e8.e8_workspace_bytes(e8.E8_GEMM_ACT_RHT, 16, N, K, 4) == 32 * K + 256
    assert e8.e8_workspace_bytes(e8.E8_GEMM_ACT_RHT, 1, N, K, 4) == 16 * K + 256
    assert e8.e8_workspace_bytes(e8.E8_GEMM_AUTO, 16, N, K, 4) == 32 * K + 256
    assert e8.e8_act_q8_bytes(16, K) == 32 * K + 256
    # bf16 hi and lo rows where the int8 path does not apply (more than 32 tokens)
    assert e8.e8_workspace_bytes(e8.E8_GEMM_ACT_RHT, 40, N, K, 4) == 80 * K * 2
    assert e8.e8_workspace_bytes(e8.E8_GEMM_ACT_RHT_SMEM, 16, N, K, 4) == 32 * K * 2
    assert e8.e8_workspace_bytes(e8.E8_GEMM_AUTO, 4096, N, K, 4) == N * K * 2
    # invalid arguments give 0
    assert e8.e8_workspace_bytes(e8.E8_GEMM_ACT_RHT, 16, N, 100, 4) == 0
    assert e8.e8_workspace_bytes(e8.E8_GEMM_ACT_RHT, 16, N, K, 5) == 0
    assert e8.e8_workspace_bytes(e8.E8_OP_ENCODE, 0, N, 65536, 2) == 0


def test_host_call_workspace_sizes(lib):
    # [X copy][Y copy][the workspace of e8_gemm], each part on 256 bytes
    M, N, K = 16, 4096, 4096
    inner = e8.e8_workspace_bytes(e8.E8_GEMM_ACT_RHT, M, N, K, 4)
    assert e8.e8_gemm_host_workspace_bytes(e8.E8_GEMM_ACT_RHT, M, N, K, 4) == \
        M * K * 2 + M * N * 4 + inner
    assert e8.e8_gemm_host_workspace_bytes(e8.E8_GEMM_AUTO, M, N, K, 4) == \
        M * K * 2 + M * N * 4 + inner
    # ragged sizes round each part up to 256 bytes
    assert e8.e8_gemm_host_workspace_bytes(e8.E8_GEMM_DECODED_W, 3, 100, 264, 2) == \
        1792 + 1280 + e8.e8_workspace_bytes(e8.E8_GEMM_DECODED_W, 3, 100, 264, 2)
    assert 3 * 264 * 2 <= 1792 < 3 * 264 * 2 + 256 and 3 * 100 * 4 <= 1280 < 3 * 100 * 4 + 256
    # invalid arguments give 0
    assert e8.e8_gemm_host_workspace_bytes(e8.E8_GEMM_ACT_RHT, 0, N, K, 4) == 0
    assert e8.e8_gemm_host_workspace_bytes(7, M, N, K, 4) == 0
    assert e8.e8_gemm_host_workspace_bytes(e8.E8_GEMM_ACT_RHT, M, N, 100, 4) == 0


def test_host_call_refuses_bad_arguments_before_any_cuda_call(lib):
    # e8_gemm_host checks every argument and the workspace size before its
    # first CUDA call (this host has no GPU: a CUDA call would answer
    # E8_ECUDA).  The codebook and device addresses below are stand-ins that
    # these paths never dereference.
    import numpy as np
    X = np.zeros((16, 4096), np.uint16)
    Y = np.zeros((16, 4096), np.float32)
    cb, dev = 1 << 20, 1 << 24

    def call(M=16, N=4096, K=4096, bpw=4, scale=0.02, x=None, y=None, i1=dev, i2=dev + 4096,
             mode=e8.E8_GEMM_ACT_RHT, ws=dev + 8192, wsb=None, cbp=cb):
        x = X.ctypes.data if x is None else x
        y = Y.ctypes.data if y is None else y
        if wsb is None:
            wsb = e8.e8_gemm_host_workspace_bytes(mode, M, N, K, bpw)
        return lib.e8_gemm_host(cbp, x, M, i1, i2, N, K, bpw, 5, scale, y, mode, ws, wsb, None)

    assert call(cbp=None) == e8.E8_EINVAL
    assert call(bpw=5) == e8.E8_EINVAL
    assert call(K=100) == e8.E8_EINVAL
    assert call(scale=0.0) == e8.E8_EINVAL
    assert call(scale=float("nan")) == e8.E8_EINVAL
    assert call(bpw=2) == e8.E8_EINVAL            # a residual index array at 2 bpw
    assert call(bpw=3, i2=None) == e8.E8_EINVAL   # none at 3 bpw
    assert call(mode=9) == e8.E8_EINVAL
    assert call(M=65) == e8.E8_EINVAL             # the activation path takes M <= 64
    assert call(x=X.ctypes.data + 2) == e8.E8_EINVAL
    assert call(i1=dev + 2) == e8.E8_EINVAL
    assert call(x=0) == e8.E8_EINVAL
    assert call(y=X.ctypes.data + 64) == e8.E8_EINVAL   # Y overlaps X
    need = e8.e8_gemm_host_workspace_bytes(e8.E8_GEMM_ACT_RHT, 16, 4096, 4096, 4)
    assert call(wsb=need - 1) == e8.E8_EWORKSPACE
    assert call(ws=None) == e8.E8_EWORKSPACE
    assert call(ws=dev + 8) == e8.E8_EWORKSPACE
    # nothing to do: no CUDA call either
    assert call(M=0) == e8.E8_OK
    assert call(N=0) == e8.E8_OK


def test_auto_mode(lib):
    assert e8.e8_gemm_auto_mode(16, 4096, 4096, 4) == e8.E8_GEMM_ACT_RHT
    assert e8.e8_gemm_auto_mode(64, 4096, 4096, 4) == e8.E8_GEMM_ACT_RHT
    assert e8.e8_gemm_auto_mode(65, 4096, 4096, 4) == e8.E8_GEMM_DECODED_W
    assert e8.e8_gemm_auto_mode(16, 4096, 264, 4) == e8.E8_GEMM_DECODED_W


def test_missing_library_fails_loudly(tmp_path):
    saved = e8._lib
    try:
        e8._lib = None
        with pytest.raises(ImportError):
            e8.load_library(str(tmp_path / "absent.so"))
    finally:
        e8._lib = saved


def test_grouped_workspace_sizes(lib):
    # one int8 activation buffer per item: 2M rows (padded to 16) of K bytes
    # and the per-token steps, each on 256 bytes
    one = e8.e8_workspace_bytes(e8.E8_GEMM_ACT_RHT, 16, 4096, 4096, 4)
    assert e8.e8_gemm_grouped_workspace_bytes(16, 4096, 4, 3) == 3 * one
    assert e8.e8_gemm_grouped_workspace_bytes(5, 14336, 2, 4) == 4 * (16 * 14336 + 256)
    # invalid: no items, too many, more than 32 tokens, K outside the int8 path
    assert e8.e8_gemm_grouped_workspace_bytes(16, 4096, 4, 0) == 0
    assert e8.e8_gemm_grouped_workspace_bytes(16, 4096, 4, e8.E8_GROUP_MAX + 1) == 0
    assert e8.e8_gemm_grouped_workspace_bytes(33, 4096, 4, 2) == 0
    assert e8.e8_gemm_grouped_workspace_bytes(16, 4104, 4, 2) == 0


def test_grouped_call_refuses_bad_arguments_before_any_cuda_call(lib):
    # like e8_gemm_host: argument and workspace errors come before the first
    # CUDA call (a CUDA call on this GPU-less host would answer E8_ECUDA); the
    # codebook and device addresses are stand-ins that are never dereferenced
    import ctypes
    cb, dev = 1 << 20, 1 << 24
    M, K, bpw = 16, 4096, 4

    def items(n=3, change=None):
        arr = (e8.GemmItem * max(1, n))()
        for i in range(n):
            d = dict(idx1=dev + 0x100000 * i, idx2=dev + 0x100000 * i + 0x80000, N=1024,
                     rht_seed=i, scale=0.02, Y=dev + 0x4000000 + 0x100000 * i)
            d.update((change or {}).get(i, {}))
            arr[i] = e8.GemmItem(d["idx1"], d["idx2"], d["N"], d["rht_seed"], d["scale"], d["Y"])
        return arr

    def call(arr=None, n=3, M=M, K=K, bpw=bpw, x=dev + 0x8000000, ws=dev + 0x9000000, wsb=None,
             cbp=cb):
        arr = items(n) if arr is None else arr
        if wsb is None:
            wsb = e8.e8_gemm_grouped_workspace_bytes(M, K, bpw, n)
        return lib.e8_gemm_grouped(cbp, x, M, K, bpw, ctypes.cast(arr, ctypes.c_void_p), n, ws,
                                   wsb, None)

    assert call(cbp=None) == e8.E8_EINVAL
    assert call(n=0, arr=items(1)) == e8.E8_EINVAL
    assert call(n=e8.E8_GROUP_MAX + 1, arr=items(e8.E8_GROUP_MAX + 1)) == e8.E8_EINVAL
    assert call(bpw=5) == e8.E8_EINVAL
    assert call(K=100) == e8.E8_EINVAL
    assert call(M=33) == e8.E8_EINVAL                      # int8 path: at most 32 tokens
    assert call(arr=items(3, {1: dict(scale=0.0)})) == e8.E8_EINVAL
    assert call(arr=items(3, {2: dict(idx2=None)})) == e8.E8_EINVAL   # 4 bpw needs idx2
    assert call(arr=items(3, {0: dict(idx1=dev + 2)})) == e8.E8_EINVAL
    assert call(arr=items(3, {1: dict(Y=None)})) == e8.E8_EINVAL
    assert call(arr=items(3, {1: dict(N=-1)})) == e8.E8_EINVAL
    assert call(x=dev + 8) == e8.E8_EINVAL
    need = e8.e8_gemm_grouped_workspace_bytes(M, K, bpw, 3)
    assert call(wsb=need - 1) == e8.E8_EWORKSPACE
    assert call(ws=None) == e8.E8_EWORKSPACE
    # nothing to do: no CUDA call either
    assert call(M=0) == e8.E8_OK
    assert call(arr=items(3, {0: dict(N=0), 1: dict(N=0), 2: dict(N=0)})) == e8.E8_OK


def test_explicit_block_workspace_sizes(lib):
    N, K = 4096, 4096
    # n_h = 256: the int8 activation path, as for the default block
    assert e8.e8_workspace_bytes(e8.E8_GEMM_ACT_RHT, 16, N, K, 4, nh=256) == \
        e8.e8_workspace_bytes(e8.E8_GEMM_ACT_RHT, 16, N, K, 4)
    # n_h = 128: the bf16 activation path (hi and lo rows of K bf16)
    assert e8.e8_workspace_bytes(e8.E8_GEMM_ACT_RHT, 16, N, K, 4, nh=128) == 32 * K * 2
    # n_h = 0 is the default block; invalid blocks give 0
    assert e8.e8_workspace_bytes(e8.E8_GEMM_ACT_RHT, 16, N, K, 4, nh=0) == \
        e8.e8_workspace_bytes(e8.E8_GEMM_ACT_RHT, 16, N, K, 4)
    for nh in (4, 96, 8192 * 2, 65536):
        assert e8.e8_workspace_bytes(e8.E8_GEMM_ACT_RHT, 16, N, K, 4, nh=nh) == 0
    assert e8.e8_workspace_bytes(e8.E8_GEMM_DECODED_W, 64, N, 3072, 4, nh=2048) == 0
    assert e8.e8_workspace_bytes(e8.E8_GEMM_DECODED_W, 64, N, 3072, 4, nh=1024) == N * 3072 * 2


def test_entropy_coded_sizes_and_rate(lib):
    # host-only queries of the entropy-coded variant: blocks of 64 groups, at
    # most 9 words per group plus 2 per block, the rate formula of the oracle
    from oracle import ep_oracle as ep
    assert lib.e8_ep_num_blocks(4096, 4096) == 4096 * 512 // 64
    assert lib.e8_ep_num_blocks(7, 1000) == (7 * 125 + 63) // 64
    assert lib.e8_ep_max_words(7, 1000) == 9 * 875 + 2 * 14
    for bad in ((4, 12), (4, 0), (-1, 64)):
        assert lib.e8_ep_num_blocks(*bad) == -1
        assert lib.e8_ep_encode_workspace_bytes(*bad) == 0
        assert lib.e8_ep_gemm_workspace_bytes(16, *bad) == 0
    assert lib.e8_ep_gemm_workspace_bytes(16, 3072, 3072) == 3072 * 3072 * 2
    for N, K, words in ((24, 256, 1234), (3072, 3072, 2_300_000), (1, 8, 2)):
        nb = lib.e8_ep_num_blocks(N, K)
        enc = {"N": N, "K": K, "offsets": [0] * nb + [words]}
        assert lib.e8_ep_actual_bpp(N, K, words) == pytest.approx(ep.actual_bpp(enc), rel=1e-12)
    assert lib.e8_ep_actual_bpp(0, 64, 0) == -1.0


def test_entropy_coded_refusals_need_no_gpu(lib):
    import ctypes
    tw = ctypes.c_int64(5)
    # no codebook handle: refused before any device work
    assert lib.e8_ep_encode(None, None, 4, 64, 0.05, None, 0, None, None, None,
                            ctypes.byref(tw), None, 0, None) == e8.E8_EINVAL
    assert lib.e8_ep_decode_to_bf16(None, None, 0, None, None, None, 4, 64, None,
                                    None) == e8.E8_EINVAL
    assert e8.status_str(e8.E8_EDATA) == "malformed compressed stream"

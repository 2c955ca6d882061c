"""E8 lattice-codebook weights decoded on a B200 and fed into a bf16 GEMM.

Thin ctypes binding over ``libe8.so`` (C ABI in ``include/e8.h``).  The
functions carry the C names and only marshal arguments: tensors become device
pointers, the current torch CUDA stream becomes the ``stream`` argument, and
nonzero status codes raise :class:`E8Error`.  Every step of the computation
runs in the library's CUDA kernels; if the library is missing this module
raises instead of computing anything another way.

Method: page "glq 0.1.1" on PyPI, "How it works" (E8 codebook of 65536 vectors
from the first 7 shells, 16-bit index per 8 weights plus an 8/16-bit residual
index at 3/4 bpw, randomized Hadamard transform, Euclidean nearest codebook
vector) and the "Bit widths" table (one global scale per layer).
"""
from __future__ import annotations

import ctypes
import os

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "_lib", "libe8.so")

E8_OK, E8_EINVAL, E8_EWORKSPACE, E8_EDEVICE, E8_ECUDA, E8_ETIMEOUT, E8_ENOMEM, E8_EDATA = range(8)
E8_EP_BLOCK_GROUPS = 64
E8_EP_TABLE_WORDS = 770
E8_GEMM_AUTO, E8_GEMM_ACT_RHT, E8_GEMM_DECODED_W, E8_GEMM_ACT_RHT_SMEM, E8_GEMM_SIMT = range(5)
E8_OP_ENCODE = 100

# every symbol include/e8.h declares
EXPORTED = ("e8_codebook_build", "e8_codebook_free", "e8_codebook_export", "e8_rht_forward",
            "e8_encode", "e8_decode_to_bf16", "e8_act_rht", "e8_act_rht_q8", "e8_act_q8_bytes",
            "e8_gemm", "e8_gemm_xt",
            "e8_gemm_xt_rows", "e8_gemm_act_noalloc", "e8_gemm_host",
            "e8_gemm_grouped", "e8_gemm_grouped_workspace_bytes",
            "e8_rht_forward_nh", "e8_encode_nh", "e8_decode_to_bf16_nh", "e8_gemm_nh",
            "e8_workspace_bytes_nh",
            "e8_gemm_host_workspace_bytes", "e8_gemm_auto_mode",
            "e8_workspace_bytes", "e8_sync_status", "e8_debug_wait_timeout", "e8_status_str",
            "e8_version",
            "e8_ep_num_blocks", "e8_ep_max_words", "e8_ep_actual_bpp",
            "e8_ep_encode_workspace_bytes", "e8_ep_gemm_workspace_bytes", "e8_ep_encode",
            "e8_ep_estimate_bpp", "e8_ep_choose_delta", "e8_ep_decode_to_bf16", "e8_ep_gemm")

_lib = None


class E8Error(RuntimeError):
    def __init__(self, code: int, where: str):
        self.code = code
        super().__init__("%s failed: %s (%d)" % (where, status_str(code), code))


def load_library(path: str = LIB_PATH):
    """Loads libe8.so and declares argument types.  Raises if it is missing."""
    global _lib
    if _lib is not None:
        return _lib
    if not os.path.exists(path):
        raise ImportError("libe8.so not built (%s); run `python -m decode_gemm_e8_b200.build`" % path)
    lib = ctypes.CDLL(path)
    c = ctypes
    P, I64, U64 = c.c_void_p, c.c_int64, c.c_uint64
    sig = {
        "e8_codebook_build": ([c.POINTER(c.c_void_p), c.c_int], c.c_int),
        "e8_codebook_free": ([P], None),
        "e8_codebook_export": ([P, P], c.c_int),
        "e8_rht_forward": ([P, P, I64, I64, U64, c.c_float, P, P], c.c_int),
        "e8_encode": ([P, P, I64, I64, c.c_int, U64, c.c_float, P, P, P, c.c_size_t, P], c.c_int),
        "e8_decode_to_bf16": ([P, P, P, I64, I64, c.c_int, U64, c.c_float, P, P], c.c_int),
        "e8_act_rht": ([P, I64, I64, U64, P, I64, P], c.c_int),
        "e8_gemm": ([P, P, I64, P, P, I64, I64, c.c_int, U64, c.c_float, P, c.c_int, P,
                     c.c_size_t, P], c.c_int),
        "e8_act_rht_q8": ([P, I64, I64, U64, P, P], c.c_int),
        "e8_act_q8_bytes": ([I64, I64], c.c_size_t),
        "e8_gemm_xt": ([P, P, I64, P, P, I64, I64, c.c_int, c.c_float, P, P], c.c_int),
        "e8_gemm_xt_rows": ([I64], c.c_int),
        "e8_gemm_act_noalloc": ([P, P, I64, P, P, I64, I64, c.c_int, U64, c.c_float, P, P],
                                c.c_int),
        "e8_gemm_host": ([P, P, I64, P, P, I64, I64, c.c_int, U64, c.c_float, P, c.c_int, P,
                          c.c_size_t, P], c.c_int),
        "e8_gemm_host_workspace_bytes": ([c.c_int, I64, I64, I64, c.c_int], c.c_size_t),
        "e8_gemm_auto_mode": ([I64, I64, I64, c.c_int], c.c_int),
        "e8_gemm_grouped": ([P, P, I64, I64, c.c_int, P, c.c_int, P, c.c_size_t, P], c.c_int),
        "e8_rht_forward_nh": ([P, P, I64, I64, I64, U64, c.c_float, P, P], c.c_int),
        "e8_encode_nh": ([P, P, I64, I64, I64, c.c_int, U64, c.c_float, P, P, P, c.c_size_t, P],
                         c.c_int),
        "e8_decode_to_bf16_nh": ([P, P, P, I64, I64, I64, c.c_int, U64, c.c_float, P, P],
                                 c.c_int),
        "e8_gemm_nh": ([P, P, I64, P, P, I64, I64, I64, c.c_int, U64, c.c_float, P, c.c_int, P,
                        c.c_size_t, P], c.c_int),
        "e8_workspace_bytes_nh": ([c.c_int, I64, I64, I64, I64, c.c_int], c.c_size_t),
        "e8_gemm_grouped_workspace_bytes": ([I64, I64, c.c_int, c.c_int], c.c_size_t),
        "e8_workspace_bytes": ([c.c_int, I64, I64, I64, c.c_int], c.c_size_t),
        "e8_sync_status": ([P, P], c.c_int),
        "e8_debug_wait_timeout": ([P, c.c_int, P], c.c_int),
        "e8_status_str": ([c.c_int], c.c_char_p),
        "e8_version": ([], c.c_int),
        "e8_ep_num_blocks": ([I64, I64], I64),
        "e8_ep_max_words": ([I64, I64], I64),
        "e8_ep_actual_bpp": ([I64, I64, I64], c.c_double),
        "e8_ep_encode_workspace_bytes": ([I64, I64], c.c_size_t),
        "e8_ep_gemm_workspace_bytes": ([I64, I64, I64], c.c_size_t),
        "e8_ep_encode": ([P, P, I64, I64, c.c_float, P, I64, P, P, P, c.POINTER(c.c_int64), P,
                          c.c_size_t, P], c.c_int),
        "e8_ep_estimate_bpp": ([P, P, I64, I64, c.c_float, c.POINTER(c.c_double), P, c.c_size_t,
                                P], c.c_int),
        "e8_ep_choose_delta": ([P, P, I64, I64, c.c_double, c.POINTER(c.c_float), P, c.c_size_t,
                                P], c.c_int),
        "e8_ep_decode_to_bf16": ([P, P, I64, P, P, P, I64, I64, P, P], c.c_int),
        "e8_ep_gemm": ([P, P, I64, P, I64, P, P, P, I64, I64, P, P, c.c_size_t, P], c.c_int),
    }
    for name, (args, res) in sig.items():
        f = getattr(lib, name)
        f.argtypes = args
        f.restype = res
    _lib = lib
    return lib


E8_GROUP_MAX = 4


class GemmItem(ctypes.Structure):
    """struct e8_gemm_item of include/e8.h."""
    _fields_ = [("idx1", ctypes.c_void_p), ("idx2", ctypes.c_void_p), ("N", ctypes.c_int64),
                ("rht_seed", ctypes.c_uint64), ("scale", ctypes.c_float),
                ("Y", ctypes.c_void_p)]


def status_str(code: int) -> str:
    return load_library().e8_status_str(int(code)).decode()


def _check(rc: int, where: str):
    if rc != E8_OK:
        raise E8Error(rc, where)


def _ptr(t):
    # the argtypes declare c_void_p, which takes a plain integer address
    return None if t is None else t.data_ptr()


def _stream(stream=None):
    import torch
    if stream is not None:
        return stream.cuda_stream
    try:
        # the raw handle of the current stream, without building a Stream object
        return torch._C._cuda_getCurrentRawStream(torch.cuda.current_device())
    except AttributeError:
        return torch.cuda.current_stream().cuda_stream


class Codebook:
    """Device-resident canonical codebook tables (``e8_codebook_build``)."""

    def __init__(self, device: int = 0):
        lib = load_library()
        h = ctypes.c_void_p()
        _check(lib.e8_codebook_build(ctypes.byref(h), int(device)), "e8_codebook_build")
        self._h = h
        self.device = int(device)

    @property
    def handle(self):
        return self._h

    def free(self):
        if getattr(self, "_h", None):
            load_library().e8_codebook_free(self._h)
            self._h = None

    def __del__(self):
        try:
            self.free()
        except Exception:
            pass


def e8_codebook_build(device: int = 0) -> Codebook:
    return Codebook(device)


def e8_codebook_free(cb: Codebook) -> None:
    cb.free()


def e8_codebook_export(cb: Codebook):
    """The 65536 codebook vectors as an int8 numpy array [65536, 8] of doubled coordinates."""
    import numpy as np
    out = np.zeros((65536, 8), dtype=np.int8)
    _check(load_library().e8_codebook_export(cb.handle, ctypes.c_void_p(out.ctypes.data)),
           "e8_codebook_export")
    return out


def e8_rht_forward(cb: Codebook, W, rht_seed: int, scale: float, U=None, stream=None, nh=None):
    """nh: explicit Hadamard block (e8_rht_forward_nh); None for the default."""
    import torch
    N, K = W.shape
    if U is None:
        U = torch.empty_like(W)
    lib = load_library()
    if nh is None:
        rc = lib.e8_rht_forward(cb.handle, _ptr(W), N, K, int(rht_seed) & (2**64 - 1),
                                float(scale), _ptr(U), _stream(stream))
    else:
        rc = lib.e8_rht_forward_nh(cb.handle, _ptr(W), N, K, int(nh), int(rht_seed) & (2**64 - 1),
                                   float(scale), _ptr(U), _stream(stream))
    _check(rc, "e8_rht_forward")
    return U


def e8_workspace_bytes(op: int, M: int, N: int, K: int, bpw: int, nh=None) -> int:
    if nh is not None:
        return int(load_library().e8_workspace_bytes_nh(int(op), int(M), int(N), int(K), int(nh),
                                                        int(bpw)))
    return int(load_library().e8_workspace_bytes(int(op), int(M), int(N), int(K), int(bpw)))


def e8_gemm_auto_mode(M: int, N: int, K: int, bpw: int) -> int:
    return int(load_library().e8_gemm_auto_mode(int(M), int(N), int(K), int(bpw)))


def _workspace(nbytes: int, device, workspace=None):
    import torch
    if workspace is not None:
        return workspace
    return torch.empty(max(int(nbytes), 16), dtype=torch.uint8, device=device)


def e8_encode(cb: Codebook, W, bpw: int, rht_seed: int, scale: float, idx1=None, idx2=None,
              workspace=None, stream=None, nh=None):
    """W fp32 [N, K] (CUDA) -> (idx1 uint16 [N, K/8], idx2 uint8/uint16 [N, K/8] or None).
    nh: explicit Hadamard block (e8_encode_nh); None for the default."""
    import torch
    N, K = W.shape
    dev = W.device
    if idx1 is None:
        idx1 = torch.empty((N, K // 8), dtype=torch.uint16, device=dev)
    if idx2 is None and bpw > 2:
        idx2 = torch.empty((N, K // 8), dtype=torch.uint8 if bpw == 3 else torch.uint16, device=dev)
    need = e8_workspace_bytes(E8_OP_ENCODE, 0, N, K, bpw)
    ws = _workspace(need, dev, workspace)
    lib = load_library()
    if nh is None:
        rc = lib.e8_encode(cb.handle, _ptr(W), N, K, int(bpw), int(rht_seed) & (2**64 - 1),
                           float(scale), _ptr(idx1), _ptr(idx2), _ptr(ws), ws.numel(),
                           _stream(stream))
    else:
        rc = lib.e8_encode_nh(cb.handle, _ptr(W), N, K, int(nh), int(bpw),
                              int(rht_seed) & (2**64 - 1), float(scale), _ptr(idx1), _ptr(idx2),
                              _ptr(ws), ws.numel(), _stream(stream))
    _check(rc, "e8_encode")
    return idx1, idx2


def e8_decode_to_bf16(cb: Codebook, idx1, idx2, N: int, K: int, bpw: int, rht_seed: int,
                      scale: float, out=None, stream=None, nh=None):
    """Decoded weights, torch.bfloat16 [N, K] on the device of idx1.
    nh: explicit Hadamard block (e8_decode_to_bf16_nh); None for the default."""
    import torch
    if out is None:
        out = torch.empty((N, K), dtype=torch.bfloat16, device=idx1.device)
    lib = load_library()
    if nh is None:
        rc = lib.e8_decode_to_bf16(cb.handle, _ptr(idx1), _ptr(idx2), N, K, int(bpw),
                                   int(rht_seed) & (2**64 - 1), float(scale), _ptr(out),
                                   _stream(stream))
    else:
        rc = lib.e8_decode_to_bf16_nh(cb.handle, _ptr(idx1), _ptr(idx2), N, K, int(nh), int(bpw),
                                      int(rht_seed) & (2**64 - 1), float(scale), _ptr(out),
                                      _stream(stream))
    _check(rc, "e8_decode_to_bf16")
    return out


def e8_act_rht(X, rht_seed: int, rows: int | None = None, out=None, stream=None):
    """X bf16 [M, K] -> Xt bf16 [rows, K] (hi rows, lo rows, zero padding)."""
    import torch
    M, K = X.shape
    rows = 2 * M if rows is None else int(rows)
    if out is None:
        out = torch.empty((rows, K), dtype=torch.bfloat16, device=X.device)
    _check(load_library().e8_act_rht(_ptr(X), M, K, int(rht_seed) & (2**64 - 1), _ptr(out), rows,
                                     _stream(stream)), "e8_act_rht")
    return out


def e8_gemm(cb: Codebook, X, idx1, idx2, N: int, K: int, bpw: int, rht_seed: int, scale: float,
            mode: int = E8_GEMM_AUTO, Y=None, workspace=None, stream=None, nh=None):
    """Y fp32 [M, N] = X bf16 [M, K] times the decoded weights transposed.
    nh: explicit Hadamard block (e8_gemm_nh); None for the default."""
    import torch
    M = X.shape[0]
    dev = X.device
    if Y is None:
        Y = torch.empty((M, N), dtype=torch.float32, device=dev)
    # a caller's workspace is checked by the library (E8_EWORKSPACE if too small)
    ws = workspace if workspace is not None else _workspace(
        e8_workspace_bytes(mode, M, N, K, bpw, nh), dev)
    lib = load_library()
    if nh is None:
        rc = lib.e8_gemm(cb.handle, _ptr(X), M, _ptr(idx1), _ptr(idx2), N, K, int(bpw),
                         int(rht_seed) & (2**64 - 1), float(scale), _ptr(Y), int(mode),
                         _ptr(ws), ws.numel(), _stream(stream))
    else:
        rc = lib.e8_gemm_nh(cb.handle, _ptr(X), M, _ptr(idx1), _ptr(idx2), N, K, int(nh),
                            int(bpw), int(rht_seed) & (2**64 - 1), float(scale), _ptr(Y),
                            int(mode), _ptr(ws), ws.numel(), _stream(stream))
    _check(rc, "e8_gemm")
    return Y


def e8_gemm_host_workspace_bytes(mode: int, M: int, N: int, K: int, bpw: int) -> int:
    return int(load_library().e8_gemm_host_workspace_bytes(int(mode), int(M), int(N), int(K),
                                                           int(bpw)))


def _host_ptr(a):
    # torch CPU tensor or numpy array
    return a.data_ptr() if hasattr(a, "data_ptr") else a.ctypes.data


def e8_gemm_host(cb: Codebook, X_host, idx1, idx2, N: int, K: int, bpw: int, rht_seed: int,
                 scale: float, Y_host=None, mode: int = E8_GEMM_AUTO, workspace=None,
                 stream=None):
    """e8_gemm with X (bf16 [M, K]) and Y (fp32 [M, N]) in host memory.

    One library call queues the copy of X in, the product and the copy of Y
    out on the stream; Y_host holds the product once the stream has passed it.
    X_host: a torch bf16/int16 CPU tensor or a numpy uint16/int16 array.
    A new page-locked Y_host is made when None is given."""
    import torch
    M = X_host.shape[0]
    if Y_host is None:
        Y_host = torch.empty((M, N), dtype=torch.float32).pin_memory()
    ws = workspace if workspace is not None else _workspace(
        e8_gemm_host_workspace_bytes(mode, M, N, K, bpw), torch.device("cuda", cb.device))
    _check(load_library().e8_gemm_host(cb.handle, _host_ptr(X_host), M, _ptr(idx1), _ptr(idx2),
                                       N, K, int(bpw), int(rht_seed) & (2**64 - 1), float(scale),
                                       _host_ptr(Y_host), int(mode), _ptr(ws), ws.numel(),
                                       _stream(stream)), "e8_gemm_host")
    return Y_host


def e8_gemm_xt_rows(M: int) -> int:
    return int(load_library().e8_gemm_xt_rows(int(M)))


def e8_act_q8_bytes(M: int, K: int) -> int:
    return int(load_library().e8_act_q8_bytes(int(M), int(K)))


def e8_act_rht_q8(X, rht_seed: int, out=None, stream=None):
    """X bf16 [M, K] -> the int8 activation buffer (uint8 tensor) of e8_gemm_xt."""
    import torch
    M, K = X.shape
    if out is None:
        out = torch.empty(max(16, e8_act_q8_bytes(M, K)), dtype=torch.uint8, device=X.device)
    _check(load_library().e8_act_rht_q8(_ptr(X), M, K, int(rht_seed) & (2**64 - 1), _ptr(out),
                                        _stream(stream)), "e8_act_rht_q8")
    return out


def e8_gemm_xt(cb: Codebook, xq, M: int, idx1, idx2, N: int, K: int, bpw: int, scale: float,
               Y=None, stream=None):
    """Fused decode + int8 GEMM on a buffer from e8_act_rht_q8; the product is
    added into Y (a new zero tensor when Y is None)."""
    import torch
    if Y is None:
        Y = torch.zeros((M, N), dtype=torch.float32, device=xq.device)
    _check(load_library().e8_gemm_xt(cb.handle, _ptr(xq), int(M), _ptr(idx1), _ptr(idx2), int(N),
                                     int(K), int(bpw), float(scale), _ptr(Y), _stream(stream)),
           "e8_gemm_xt")
    return Y


def e8_gemm_act_noalloc(cb: Codebook, X, idx1, idx2, N: int, K: int, bpw: int, rht_seed: int,
                        scale: float, Y, stream=None):
    """E8_GEMM_ACT_RHT with the library's fixed scratch array instead of a workspace.

    For callers that may not allocate device memory when they run the layer (CUDA
    graph capture, framework-owned memory, latency-critical loops).  Y must be
    given: this call allocates nothing."""
    _check(load_library().e8_gemm_act_noalloc(cb.handle, _ptr(X), X.shape[0], _ptr(idx1),
                                              _ptr(idx2), int(N), int(K), int(bpw),
                                              int(rht_seed) & (2**64 - 1), float(scale), _ptr(Y),
                                              _stream(stream)), "e8_gemm_act_noalloc")
    return Y


def e8_sync_status(cb: Codebook, stream=None) -> int:
    """Synchronises the stream and returns (and clears) the device status as a status code."""
    return int(load_library().e8_sync_status(cb.handle, _stream(stream)))


def e8_debug_wait_timeout(cb: Codebook, wait_ms: int, stream=None) -> None:
    _check(load_library().e8_debug_wait_timeout(cb.handle, int(wait_ms), _stream(stream)),
           "e8_debug_wait_timeout")


def e8_version() -> int:
    return int(load_library().e8_version())


def e8_gemm_grouped_workspace_bytes(M: int, K: int, bpw: int, count: int) -> int:
    return int(load_library().e8_gemm_grouped_workspace_bytes(int(M), int(K), int(bpw),
                                                              int(count)))


def e8_gemm_grouped(cb: Codebook, X, items, K: int, bpw: int, workspace=None, stream=None):
    """Y_i = X W_dec_i^T for several weight matrices that read the same X.

    items: sequence of (idx1, idx2, N, rht_seed, scale) or
    (idx1, idx2, N, rht_seed, scale, Y); a missing Y is allocated (fp32 [M, N]).
    Returns the list of Y tensors."""
    import torch
    M = int(X.shape[0])
    arr = (GemmItem * max(1, len(items)))()
    outs = []
    for i, it in enumerate(items):
        idx1, idx2, N, rs, scale = it[:5]
        Y = it[5] if len(it) > 5 and it[5] is not None else torch.empty(
            (M, int(N)), dtype=torch.float32, device=X.device)
        outs.append(Y)
        arr[i] = GemmItem(_ptr(idx1), _ptr(idx2), int(N), int(rs), float(scale), _ptr(Y))
    if workspace is None:
        workspace = torch.empty(max(16, e8_gemm_grouped_workspace_bytes(M, K, bpw, len(items))),
                                dtype=torch.uint8, device=X.device)
    _check(load_library().e8_gemm_grouped(cb.handle, _ptr(X), M, int(K), int(bpw),
                                          ctypes.cast(arr, ctypes.c_void_p), len(items),
                                          _ptr(workspace), workspace.numel(), _stream(stream)),
           "e8_gemm_grouped")
    return outs


# ------------------------------------------------------ entropy-coded variant --
class EpMatrix:
    """Compressed form of one matrix (e8_ep_encode): stream words, block
    offsets, row scales t, frequency tables (all on the device)."""

    def __init__(self, N, K, delta, words, offsets, t, tables, total_words):
        self.N, self.K, self.delta = N, K, delta
        self.words, self.offsets, self.t, self.tables = words, offsets, t, tables
        self.total_words = total_words

    def actual_bpp(self) -> float:
        return float(load_library().e8_ep_actual_bpp(self.N, self.K, self.total_words))


def _ep_ws(N, K, dev, workspace):
    return _workspace(load_library().e8_ep_encode_workspace_bytes(N, K), dev, workspace)


def e8_ep_encode(cb: Codebook, W, delta: float, workspace=None, stream=None) -> EpMatrix:
    """W fp32 [N, K] (CUDA) at step delta -> EpMatrix (synchronous)."""
    import torch
    N, K = W.shape
    lib = load_library()
    dev = W.device
    nmax = max(int(lib.e8_ep_max_words(N, K)), 1)
    nb = max(int(lib.e8_ep_num_blocks(N, K)), 0)
    words = torch.empty(nmax, dtype=torch.uint16, device=dev)
    offsets = torch.empty(nb + 1, dtype=torch.int32, device=dev)
    t = torch.empty(max(N, 1), dtype=torch.float32, device=dev)
    tables = torch.empty(E8_EP_TABLE_WORDS, dtype=torch.uint16, device=dev)
    total = ctypes.c_int64(0)
    ws = _ep_ws(N, K, dev, workspace)
    rc = lib.e8_ep_encode(cb.handle, _ptr(W), N, K, float(delta), _ptr(words), nmax,
                          _ptr(offsets), _ptr(t), _ptr(tables), ctypes.byref(total), _ptr(ws),
                          ws.numel(), _stream(stream))
    _check(rc, "e8_ep_encode")
    return EpMatrix(N, K, float(delta), words[:max(total.value, 1)], offsets, t[:N], tables,
                    total.value)


def e8_ep_estimate_bpp(cb: Codebook, W, delta: float, workspace=None, stream=None) -> float:
    N, K = W.shape
    out = ctypes.c_double(0.0)
    ws = _ep_ws(N, K, W.device, workspace)
    rc = load_library().e8_ep_estimate_bpp(cb.handle, _ptr(W), N, K, float(delta),
                                           ctypes.byref(out), _ptr(ws), ws.numel(), _stream(stream))
    _check(rc, "e8_ep_estimate_bpp")
    return out.value


def e8_ep_choose_delta(cb: Codebook, W, target_bpp: float, workspace=None, stream=None) -> float:
    N, K = W.shape
    out = ctypes.c_float(0.0)
    ws = _ep_ws(N, K, W.device, workspace)
    rc = load_library().e8_ep_choose_delta(cb.handle, _ptr(W), N, K, float(target_bpp),
                                           ctypes.byref(out), _ptr(ws), ws.numel(), _stream(stream))
    _check(rc, "e8_ep_choose_delta")
    return out.value


def e8_ep_decode_to_bf16(cb: Codebook, m: EpMatrix, out=None, stream=None):
    """bf16 [N, K] weights of an EpMatrix."""
    import torch
    if out is None:
        out = torch.empty((m.N, m.K), dtype=torch.bfloat16, device=m.words.device)
    rc = load_library().e8_ep_decode_to_bf16(cb.handle, _ptr(m.words), m.words.numel(),
                                             _ptr(m.offsets),
                                             _ptr(m.t), _ptr(m.tables), m.N, m.K, _ptr(out),
                                             _stream(stream))
    _check(rc, "e8_ep_decode_to_bf16")
    return out


def e8_ep_gemm(cb: Codebook, X, m: EpMatrix, Y=None, workspace=None, stream=None):
    """Y fp32 [M, N] = X bf16 [M, K] times the decoded weights, transposed."""
    import torch
    M = X.shape[0]
    lib = load_library()
    if Y is None:
        Y = torch.empty((M, m.N), dtype=torch.float32, device=X.device)
    ws = _workspace(lib.e8_ep_gemm_workspace_bytes(M, m.N, m.K), X.device, workspace)
    rc = lib.e8_ep_gemm(cb.handle, _ptr(X), M, _ptr(m.words), m.words.numel(), _ptr(m.offsets),
                        _ptr(m.t),
                        _ptr(m.tables), m.N, m.K, _ptr(Y), _ptr(ws), ws.numel(), _stream(stream))
    _check(rc, "e8_ep_gemm")
    return Y


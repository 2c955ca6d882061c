"""Edge cases and error reporting of the C ABI on the GPU: empty inputs,
argument checks, workspace checks, and the bounded-wait failure path."""
import ctypes

import numpy as np
import pytest
import torch

import decode_gemm_e8_b200 as e8
from decode_gemm_e8_b200 import synth
from tests import gpu_util as gu

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def gcb():
    gu.dev()
    from decode_gemm_e8_b200 import build
    build.build()
    return e8.Codebook(0)


def _raw(gcb):
    return e8.load_library(), gcb.handle, e8._stream()


def test_empty_inputs_launch_nothing(gcb):
    lib, h, st = _raw(gcb)
    d = gu.dev()
    Y = torch.full((0, 64), 7.0, device=d)
    assert lib.e8_gemm(h, None, 0, None, None, 64, 256, 2, 0, 1.0, None, 0, None, 0, st) == 0
    assert lib.e8_encode(h, None, 0, 256, 2, 0, 1.0, None, None, None, 0, st) == 0
    assert lib.e8_decode_to_bf16(h, None, None, 0, 256, 2, 0, 1.0, None, st) == 0
    X = gu.bf16_dev(synth.activations_bf16(3, 256, 0))
    Yz = torch.full((3, 0), 1.0, device=d)
    assert lib.e8_gemm(h, e8._ptr(X), 3, None, None, 0, 256, 2, 0, 1.0, e8._ptr(Yz), 0, None, 0,
                       st) == 0
    assert e8.e8_sync_status(gcb) == e8.E8_OK


def test_argument_errors(gcb):
    lib, h, st = _raw(gcb)
    d = gu.dev()
    W = torch.zeros((4, 256), device=d)
    i1 = torch.zeros((4, 32), dtype=torch.uint16, device=d)
    i2 = torch.zeros((4, 32), dtype=torch.uint16, device=d)
    ws = torch.empty(1 << 20, dtype=torch.uint8, device=d)
    P = e8._ptr
    enc = lambda *a: lib.e8_encode(h, *a, st)
    # bad bpw, bad K, missing / superfluous idx2, bad scale
    assert enc(P(W), 4, 256, 5, 0, 1.0, P(i1), P(i2), P(ws), ws.numel()) == e8.E8_EINVAL
    assert enc(P(W), 4, 100, 2, 0, 1.0, P(i1), None, P(ws), ws.numel()) == e8.E8_EINVAL
    assert enc(P(W), 4, 256, 4, 0, 1.0, P(i1), None, P(ws), ws.numel()) == e8.E8_EINVAL
    assert enc(P(W), 4, 256, 2, 0, 1.0, P(i1), P(i2), P(ws), ws.numel()) == e8.E8_EINVAL
    assert enc(P(W), 4, 256, 2, 0, 0.0, P(i1), None, P(ws), ws.numel()) == e8.E8_EINVAL
    assert enc(P(W), 4, 256, 2, 0, float("nan"), P(i1), None, P(ws), ws.numel()) == e8.E8_EINVAL
    # Hadamard block above 32768
    assert enc(P(W), 1, 65536, 2, 0, 1.0, P(i1), None, P(ws), ws.numel()) == e8.E8_EINVAL
    # misaligned pointer
    Wm = ctypes.c_void_p(W.data_ptr() + 4)
    assert enc(Wm, 4, 256, 2, 0, 1.0, P(i1), None, P(ws), ws.numel()) == e8.E8_EINVAL
    # workspace too small / missing
    assert enc(P(W), 4, 256, 2, 0, 1.0, P(i1), None, P(ws), 64) == e8.E8_EWORKSPACE
    assert enc(P(W), 4, 256, 2, 0, 1.0, P(i1), None, None, 0) == e8.E8_EWORKSPACE
    # GEMM: unknown mode, ACT mode with too many rows or K not a multiple of 128
    X = torch.zeros((80, 256), dtype=torch.bfloat16, device=d)
    Y = torch.zeros((80, 4), device=d)
    g = lambda M, K, mode: lib.e8_gemm(h, P(X), M, P(i1), None, 4, K, 2, 0, 1.0, P(Y), mode,
                                       P(ws), ws.numel(), st)
    assert g(16, 256, 9) == e8.E8_EINVAL
    assert g(65, 256, e8.E8_GEMM_ACT_RHT) == e8.E8_EINVAL
    assert g(16, 264, e8.E8_GEMM_ACT_RHT) == e8.E8_EINVAL
    assert lib.e8_gemm(h, P(X), 16, P(i1), None, 4, 256, 2, 0, 1.0, P(Y), 1, P(ws), 16, st) == \
        e8.E8_EWORKSPACE
    # wrong device handle
    assert lib.e8_encode(None, P(W), 4, 256, 2, 0, 1.0, P(i1), None, P(ws), ws.numel(), st) == \
        e8.E8_EINVAL
    assert e8.e8_sync_status(gcb) == e8.E8_OK


def test_bounded_wait_reports_timeout_and_context_survives(gcb):
    # a wait on a barrier nothing signals gives up after 50 ms and reports
    e8.e8_debug_wait_timeout(gcb, 50)
    assert e8.e8_sync_status(gcb) == e8.E8_ETIMEOUT
    # the status word was cleared and the context still works
    assert e8.e8_sync_status(gcb) == e8.E8_OK
    W = synth.gaussian_weights(2, 256, 0.02, 0)
    i1, _ = e8.e8_encode(gcb, gu.to_dev(W), 2, 0, 0.02)
    torch.cuda.synchronize()
    assert e8.e8_sync_status(gcb) == e8.E8_OK


def test_two_codebooks_and_repeat_calls(gcb):
    cb2 = e8.Codebook(0)
    a = e8.e8_codebook_export(cb2)
    b = e8.e8_codebook_export(gcb)
    assert np.array_equal(a, b)
    cb2.free()
    cb2.free()

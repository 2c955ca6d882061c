"""GPU parity of the compressed-weight GEMM against the oracle.

Reference: the oracle's binary64 product Y = X W_dec^T with W_dec the oracle's
bf16 decoded weights.  Bar (relative Frobenius error): 2e-3 for every mode.
The decoded-weight modes compute with W_dec itself, so their only error is the
fp32 accumulation (products of two bf16 values are exact): about
sqrt(K) * 2^-24 relative for random signs, 7e-6 at K = 12288; they must also
meet 1e-4.  The activation-side modes use the unrounded weights, whose bf16
rounding alone is about 1.7e-3 of the product.
"""
import numpy as np
import pytest

import decode_gemm_e8_b200 as e8
from decode_gemm_e8_b200 import synth
from oracle import oracle as orc
from tests import gpu_util as gu

pytestmark = pytest.mark.gpu

BAR = 2e-3
BAR_DECODED = 1e-4
REPEAT = 1e-6   # run-to-run agreement of the int8 path (atomic partial sums)
ACT_MODES = [e8.E8_GEMM_ACT_RHT, e8.E8_GEMM_ACT_RHT_SMEM]
ALL_MODES = ACT_MODES + [e8.E8_GEMM_DECODED_W, e8.E8_GEMM_SIMT]


@pytest.fixture(scope="module")
def gcb():
    gu.dev()
    from decode_gemm_e8_b200 import build
    build.build()
    return e8.Codebook(0)


def _layer_codes(gcb, W, bpw, rs, s):
    i1, i2 = e8.e8_encode(gcb, gu.to_dev(W), bpw, rs, s)
    return i1, i2


def _check(Y, ref, mode):
    err = gu.rel_fro(Y, ref)
    assert err < BAR, (mode, err)
    if mode in (e8.E8_GEMM_DECODED_W, e8.E8_GEMM_SIMT):
        assert err < BAR_DECODED, (mode, err)
    return err


@pytest.mark.parametrize("mode", ALL_MODES)
def test_gemm_single_256(gcb, mode):
    wl = synth.workloads()["single_256"]
    lay = wl.layers[0]
    W = lay.weights()
    s = synth.suggest_scale(W, lay.bpw)
    X = synth.activations_bf16(wl.M[0], lay.K, wl.x_seed)
    i1, i2 = _layer_codes(gcb, W, lay.bpw, lay.rht_seed, s)
    Y = gu.to_np(e8.e8_gemm(gcb, gu.bf16_dev(X), i1, i2, lay.N, lay.K, lay.bpw, lay.rht_seed, s,
                            mode=mode))
    wd = orc.decode(gu.to_np(i1), None, lay.N, lay.K, lay.bpw, lay.rht_seed, s)
    _check(Y, orc.gemm(X, wd), mode)


@pytest.mark.parametrize("M", [1, 4, 16])
@pytest.mark.parametrize("mode", ALL_MODES)
def test_gemm_llama_4096_b4(gcb, M, mode):
    wl = synth.workloads()["llama_4096_b4"]
    lay = wl.layers[0]
    W = lay.weights()
    s = synth.suggest_scale(W, lay.bpw)
    X = synth.activations_bf16(M, lay.K, wl.x_seed)
    i1, i2 = _layer_codes(gcb, W, lay.bpw, lay.rht_seed, s)
    Y = gu.to_np(e8.e8_gemm(gcb, gu.bf16_dev(X), i1, i2, lay.N, lay.K, lay.bpw, lay.rht_seed, s,
                            mode=mode))
    wd = orc.decode(gu.to_np(i1), gu.to_np(i2), lay.N, lay.K, lay.bpw, lay.rht_seed, s)
    _check(Y, orc.gemm(X, wd), mode)


@pytest.mark.parametrize("bpw,M,N,K", [(2, 7, 200, 384), (3, 64, 136, 1024), (4, 33, 520, 3072),
                                       (3, 2, 1024, 12288), (4, 64, 256, 256)])
@pytest.mark.parametrize("mode", ALL_MODES)
def test_gemm_ragged_shapes(gcb, bpw, M, N, K, mode):
    W = synth.gaussian_weights(N, K, 0.02, 1000 + N)
    s = synth.suggest_scale(W, bpw)
    X = synth.activations_bf16(M, K, 2000 + M)
    i1, i2 = _layer_codes(gcb, W, bpw, 5, s)
    Y = gu.to_np(e8.e8_gemm(gcb, gu.bf16_dev(X), i1, i2, N, K, bpw, 5, s, mode=mode))
    wd = orc.decode(gu.to_np(i1), None if i2 is None else gu.to_np(i2), N, K, bpw, 5, s)
    _check(Y, orc.gemm(X, wd), mode)


def _prefill_check(gcb, lay, X, s, i1, i2, mode, rows):
    Y = gu.to_np(e8.e8_gemm(gcb, gu.bf16_dev(X), i1, i2, lay.N, lay.K, lay.bpw, lay.rht_seed, s,
                            mode=mode))
    assert Y.shape == (X.shape[0], lay.N)
    wd = orc.decode(gu.to_np(i1), gu.to_np(i2), lay.N, lay.K, lay.bpw, lay.rht_seed, s)
    ref = orc.gemm(X[rows], wd)
    return _check(Y[rows], ref, mode)


@pytest.mark.parametrize("mode", [e8.E8_GEMM_AUTO, e8.E8_GEMM_DECODED_W])
def test_gemm_prefill_mlp_up_sampled_rows(gcb, mode):
    wl = synth.workloads()["mlp_up_14336_b3"]
    lay = wl.layers[0]
    W = lay.weights()
    s = synth.suggest_scale(W, lay.bpw)
    X = synth.activations_bf16(wl.M[0], lay.K, wl.x_seed)
    i1, i2 = _layer_codes(gcb, W, lay.bpw, lay.rht_seed, s)
    rows = np.sort(np.random.default_rng(1).choice(wl.M[0], 24, replace=False))
    _prefill_check(gcb, lay, X, s, i1, i2, mode, rows)


def test_gemm_prefill_dit_sampled_rows(gcb):
    wl = synth.workloads()["dit_3072_b4"]
    for lay in wl.layers:
        W = lay.weights()
        s = synth.suggest_scale(W, lay.bpw)
        X = synth.activations_bf16(wl.M[0], lay.K, wl.x_seed)
        i1, i2 = _layer_codes(gcb, W, lay.bpw, lay.rht_seed, s)
        rows = np.sort(np.random.default_rng(2).choice(wl.M[0], 16, replace=False))
        _prefill_check(gcb, lay, X, s, i1, i2, e8.E8_GEMM_AUTO, rows)


def test_act_rht_hi_lo(gcb):
    M, K = 5, 3072
    X = synth.activations_bf16(M, K, 4)
    Xt = gu.to_np(e8.e8_act_rht(gu.bf16_dev(X), 21, rows=16))
    x = synth.bf16_bits_to_f32(X).astype(np.float64)
    d = orc.signs(21, K).astype(np.float64)
    from tests import indep
    nh = orc.hadamard_block(K)
    H = indep.sylvester(nh).astype(np.float64)
    xd = x * d[None, :]
    ref = np.concatenate([xd[:, b:b + nh] @ H for b in range(0, K, nh)], axis=1)
    hi = synth.bf16_bits_to_f32(Xt[0:2 * M:2]).astype(np.float64)
    lo = synth.bf16_bits_to_f32(Xt[1:2 * M:2]).astype(np.float64)
    assert np.all(np.abs(hi + lo - ref) <= np.abs(ref) * 2.0 ** -15 + 1e-6)
    assert not Xt[2 * M:].any()


def test_act_gemm_repeatable(gcb):
    wl = synth.workloads()["llama_4096_b4"]
    lay = wl.layers[0]
    W = lay.weights()
    s = synth.suggest_scale(W, lay.bpw)
    X = gu.bf16_dev(synth.activations_bf16(16, lay.K, wl.x_seed))
    i1, i2 = _layer_codes(gcb, W, lay.bpw, lay.rht_seed, s)
    a = gu.to_np(e8.e8_gemm(gcb, X, i1, i2, lay.N, lay.K, lay.bpw, lay.rht_seed, s,
                            mode=e8.E8_GEMM_ACT_RHT))
    b = gu.to_np(e8.e8_gemm(gcb, X, i1, i2, lay.N, lay.K, lay.bpw, lay.rht_seed, s,
                            mode=e8.E8_GEMM_ACT_RHT))
    # the int8 path adds the partial tiles of an output with fp32 atomics in no
    # fixed order; two runs agree to within a few rounding steps
    assert gu.rel_fro(a, b) < REPEAT
    assert np.max(np.abs(a - b)) <= 1e-5 * np.max(np.abs(a))
    assert e8.e8_sync_status(gcb) == e8.E8_OK


def test_gemm_chain_mixed_depth_shared_workspace(gcb):
    # products of different depths queued back to back on one stream with one
    # workspace, three times over: the activation transform of each call runs
    # before the GEMM of the previous call has finished and stores only after
    import torch
    M = 16
    shapes = [(520, 14336, 4), (1024, 4096, 4), (264, 14336, 3), (512, 30720, 2),
              (1024, 4096, 2), (136, 4352, 4)]
    ws = torch.empty(max(e8.e8_workspace_bytes(e8.E8_GEMM_ACT_RHT, M, N, K, b)
                         for N, K, b in shapes), dtype=torch.uint8, device=gu.dev())
    cases = []
    for j, (N, K, bpw) in enumerate(shapes):
        W = synth.gaussian_weights(N, K, 0.02, 3000 + j)
        s = synth.suggest_scale(W, bpw)
        i1, i2 = _layer_codes(gcb, W, bpw, 11 + j, s)
        X = synth.activations_bf16(M, K, 4000 + j)
        Y = torch.full((M, N), float("nan"), dtype=torch.float32, device=gu.dev())
        cases.append((N, K, bpw, s, i1, i2, X, gu.bf16_dev(X), Y))
    st = torch.cuda.Stream()
    torch.cuda.synchronize()
    for _ in range(3):
        for j, (N, K, bpw, s, i1, i2, X, Xd, Y) in enumerate(cases):
            e8.e8_gemm(gcb, Xd, i1, i2, N, K, bpw, 11 + j, s, mode=e8.E8_GEMM_ACT_RHT, Y=Y,
                       workspace=ws, stream=st)
    torch.cuda.synchronize()
    assert e8.e8_sync_status(gcb) == e8.E8_OK
    for j, (N, K, bpw, s, i1, i2, X, Xd, Y) in enumerate(cases):
        wd = orc.decode(gu.to_np(i1), None if i2 is None else gu.to_np(i2), N, K, bpw, 11 + j, s)
        _check(gu.to_np(Y), orc.gemm(X, wd), e8.E8_GEMM_ACT_RHT)


@pytest.mark.parametrize("pinned", [True, False])
@pytest.mark.parametrize("mode", [e8.E8_GEMM_ACT_RHT, e8.E8_GEMM_DECODED_W])
def test_gemm_host_buffers(gcb, pinned, mode):
    # one call copies X in, multiplies and copies Y out; the result is that of
    # e8_gemm on device copies of the same inputs
    import torch
    M, N, K, bpw, rs = 16, 520, 3072, 3, 21
    W = synth.gaussian_weights(N, K, 0.02, 77)
    s = synth.suggest_scale(W, bpw)
    i1, i2 = _layer_codes(gcb, W, bpw, rs, s)
    X = synth.activations_bf16(M, K, 78)
    Xh = torch.from_numpy(X.view(np.int16).copy())
    Yh = torch.full((M, N), float("nan"), dtype=torch.float32)
    if pinned:
        Xh, Yh = Xh.pin_memory(), Yh.pin_memory()
    ref = gu.to_np(e8.e8_gemm(gcb, gu.bf16_dev(X), i1, i2, N, K, bpw, rs, s, mode=mode))
    st = torch.cuda.Stream()
    out = e8.e8_gemm_host(gcb, Xh, i1, i2, N, K, bpw, rs, s, Y_host=Yh, mode=mode, stream=st)
    st.synchronize()
    assert out is Yh
    assert e8.e8_sync_status(gcb) == e8.E8_OK
    # N = 520 is not a multiple of 4: in the int8 path the 24 partial sums of
    # an output (one per 128-wide K unit) are added by fp32 atomics in arrival
    # order, so two runs differ by a few rounding steps of the partial sums
    assert gu.rel_fro(Yh.numpy(), ref) < (2e-5 if mode == e8.E8_GEMM_ACT_RHT else REPEAT)
    wd = orc.decode(gu.to_np(i1), gu.to_np(i2), N, K, bpw, rs, s)
    _check(Yh.numpy().astype(np.float64), orc.gemm(X, wd), mode)
    # a workspace one byte short is refused before anything is queued
    need = e8.e8_gemm_host_workspace_bytes(mode, M, N, K, bpw)
    small = torch.empty(need - 1, dtype=torch.uint8, device=gu.dev())
    with pytest.raises(e8.E8Error) as ei:
        e8.e8_gemm_host(gcb, Xh, i1, i2, N, K, bpw, rs, s, Y_host=Yh, mode=mode, workspace=small)
    assert ei.value.code == e8.E8_EWORKSPACE


def test_gemm_xt_matches_gemm_and_graph_capture(gcb):
    import torch
    wl = synth.workloads()["llama_4096_b4"]
    lay = wl.layers[0]
    W = lay.weights()
    s = synth.suggest_scale(W, lay.bpw)
    X = gu.bf16_dev(synth.activations_bf16(16, lay.K, wl.x_seed))
    i1, i2 = _layer_codes(gcb, W, lay.bpw, lay.rht_seed, s)
    a = e8.e8_gemm(gcb, X, i1, i2, lay.N, lay.K, lay.bpw, lay.rht_seed, s,
                   mode=e8.E8_GEMM_ACT_RHT)
    assert e8.e8_gemm_xt_rows(16) == 32
    xq = e8.e8_act_rht_q8(X, lay.rht_seed)
    b = e8.e8_gemm_xt(gcb, xq, 16, i1, i2, lay.N, lay.K, lay.bpw, s)
    # partial tiles are added with atomics: equal up to the order of a few fp32 adds
    assert gu.rel_fro(gu.to_np(b), gu.to_np(a)) < REPEAT
    # e8_gemm_xt adds into Y
    b2 = e8.e8_gemm_xt(gcb, xq, 16, i1, i2, lay.N, lay.K, lay.bpw, s, Y=b.clone())
    assert gu.rel_fro(gu.to_np(b2), 2.0 * gu.to_np(a)) < REPEAT
    # the same call captured in a CUDA graph and replayed
    Y = torch.empty_like(a)
    ws = torch.empty(e8.e8_workspace_bytes(e8.E8_GEMM_ACT_RHT, 16, lay.N, lay.K, lay.bpw),
                     dtype=torch.uint8, device=X.device)
    st = torch.cuda.Stream()
    e8.e8_gemm(gcb, X, i1, i2, lay.N, lay.K, lay.bpw, lay.rht_seed, s, mode=e8.E8_GEMM_ACT_RHT,
               Y=Y, workspace=ws, stream=st)
    torch.cuda.synchronize()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g, stream=st):
        e8.e8_gemm(gcb, X, i1, i2, lay.N, lay.K, lay.bpw, lay.rht_seed, s,
                   mode=e8.E8_GEMM_ACT_RHT, Y=Y, workspace=ws, stream=st)
    Y.fill_(float("nan"))
    g.replay()
    torch.cuda.synchronize()
    assert gu.rel_fro(gu.to_np(Y), gu.to_np(a)) < REPEAT
    assert e8.e8_sync_status(gcb) == e8.E8_OK


@pytest.mark.parametrize("M,K", [(16, 4096), (3, 3072), (32, 256), (1, 12288), (5, 14336),
                                 (7, 4352), (2, 20480), (3, 30720), (32, 14336)])
def test_act_rht_q8_pieces(gcb, M, K):
    # xt = s_m (q0 + q1 / 128) within s_m / 256, s_m = max|xt| / 127
    X = synth.activations_bf16(M, K, 40 + M)
    buf = gu.to_np(e8.e8_act_rht_q8(gu.bf16_dev(X), 17))
    rows = e8.e8_gemm_xt_rows(M)
    assert len(buf) >= e8.e8_act_q8_bytes(M, K)
    xq = buf[:rows * K].view(np.int8).reshape(rows, K).astype(np.int64)
    off_s = (rows * K + 255) // 256 * 256
    sc = buf[off_s:off_s + 4 * M].view(np.float32).astype(np.float64)
    x = synth.bf16_bits_to_f32(X).astype(np.float64)
    d = orc.signs(17, K).astype(np.float64)
    from tests import indep
    nh = orc.hadamard_block(K)
    H = indep.sylvester(nh).astype(np.float64)
    ref = np.concatenate([(x * d[None, :])[:, b:b + nh] @ H for b in range(0, K, nh)], axis=1)
    amax = np.abs(ref).max(1)
    assert np.allclose(sc, amax / 127, rtol=1e-5)
    rec = sc[:, None] * (xq[0:2 * M:2] + xq[1:2 * M:2] / 128.0)
    assert np.all(np.abs(rec - ref) <= sc[:, None] / 256 * 1.01 + 1e-6)
    assert np.all(np.abs(xq[1:2 * M:2]) <= 64)
    assert not xq[2 * M:].any()


@pytest.mark.parametrize("M,N,K,bpw", [(300, 520, 1000, 4), (1024, 768, 4096, 3), (260, 260, 256, 2),
                                       (512, 1280, 3072, 4)])
def test_gemm_prefill_ragged_two_sm_tiles(gcb, M, N, K, bpw):
    # the prefill product on 256 x 256 tiles computed by CTA pairs: ragged M and
    # N (partial tiles on both sides of the pair) and a K that is not a multiple
    # of the 64-deep step (1000); decoded-weight bar 1e-4
    W = synth.gaussian_weights(N, K, 0.02, M + N)
    s = synth.suggest_scale(W, bpw)
    rs = 31
    i1, i2 = _layer_codes(gcb, W, bpw, rs, s)
    X = synth.activations_bf16(M, K, N)
    Y = gu.to_np(e8.e8_gemm(gcb, gu.bf16_dev(X), i1, i2, N, K, bpw, rs, s,
                            mode=e8.E8_GEMM_DECODED_W))
    wd = orc.decode(gu.to_np(i1), None if i2 is None else gu.to_np(i2), N, K, bpw, rs, s)
    err = gu.rel_fro(Y, orc.gemm(X, wd))
    assert err < BAR_DECODED, (M, N, K, err)
    assert e8.e8_sync_status(gcb) == e8.E8_OK

"""Small-batch GEMM (E8_GEMM_ACT_RHT) on hard inputs, element by element.

The activation-side path quantises each token's transformed row
xt = FWHT(D x) on one step per token (int8 pieces up to 32 tokens: s =
max|xt| / 127, error <= s / 256 per element; bf16 hi + lo above), so its
accuracy depends on the shape of xt.  These tests feed it the inputs that
stress that step and compare with the oracle's binary64 product
X W_dec^T (page "glq 0.1.1", "How it works", items 1-2):

  weights      Student-t (nu = 4) rows with 1 % of the columns x8 (the DiT
               stand-in), and Gaussian rows;
  activations  N(0, 1); N(0, 1) with four coordinates per token at +-256;
               N(0, 1) plus 16 D h_j on one Hadamard block, whose transform
               is a single spike of 16 n_h at position j (the largest
               max/RMS ratio xt can have).

Besides the 2e-3 relative Frobenius bar of the GEMM tests, every element
must satisfy the bound that follows from the arithmetic:
  |Y - Y_ref| <= (sqrt(K) / (127 * 256) + 2^-9 + 1e-5) * ||x_m|| * ||w_n||,
the first term the int8 step (||e|| <= sqrt(K) s / 256 with s <= sqrt(n_h)
||x|| / 127, against ||alpha z_n|| = ||w_n|| / sqrt(n_h)), the second the
bf16 rounding of W_dec in the reference (|x . dw| <= 2^-9 ||x|| ||w||), the
third fp32 accumulation.
"""
import numpy as np
import pytest

import decode_gemm_e8_b200 as e8
from decode_gemm_e8_b200 import synth
from oracle import oracle as orc
from tests import gpu_util as gu

pytestmark = pytest.mark.gpu

BAR = 2e-3


@pytest.fixture(scope="module")
def gcb():
    gu.dev()
    from decode_gemm_e8_b200 import build
    build.build()
    return e8.Codebook(0)


def _activations(kind, M, K, rs, seed):
    rng = np.random.default_rng(seed)
    x = rng.standard_normal((M, K))
    if kind == "spikes":
        for m in range(M):
            cols = rng.choice(K, 4, replace=False)
            x[m, cols] = rng.choice([-256.0, 256.0], 4)
    elif kind == "aligned":
        nh = orc.hadamard_block(K)
        d = orc.signs(rs, K)[:nh].astype(np.float64)
        k = np.arange(nh)
        for m in range(M):
            j = int(rng.integers(nh))
            h = np.where(np.array([bin(j & i).count("1") & 1 for i in k]) == 1, -1.0, 1.0)
            x[m, :nh] += 16.0 * d * h   # FWHT(D x) on block 0 gains 16 n_h at j
    return synth.f32_to_bf16_bits(x.astype(np.float32))


@pytest.fixture(scope="module")
def layers(gcb):
    out = {}
    K, N = 3072, 384
    for name, bpw in (("dit", 4), ("gauss", 2)):
        W = (synth.student_t_outlier_weights(N, K, 31) if name == "dit"
             else synth.gaussian_weights(N, K, 0.02, 32))
        s = synth.suggest_scale(W, bpw)
        rs = 77 if name == "dit" else 78
        i1, i2 = e8.e8_encode(gcb, gu.to_dev(W), bpw, rs, s)
        wd = orc.decode(gu.to_np(i1), None if i2 is None else gu.to_np(i2), N, K, bpw, rs, s)
        out[name] = (i1, i2, N, K, bpw, rs, s, wd)
    return out


@pytest.mark.parametrize("kind", ["gauss", "spikes", "aligned"])
@pytest.mark.parametrize("M", [1, 16, 32, 64])
@pytest.mark.parametrize("wname", ["dit", "gauss"])
def test_small_batch_hard_inputs(gcb, layers, wname, M, kind):
    i1, i2, N, K, bpw, rs, s, wd = layers[wname]
    Xh = _activations(kind, M, K, rs, 1000 * M + len(kind))
    Y = gu.to_np(e8.e8_gemm(gcb, gu.bf16_dev(Xh), i1, i2, N, K, bpw, rs, s,
                            mode=e8.E8_GEMM_ACT_RHT)).astype(np.float64)
    ref = orc.gemm(Xh, wd)
    err = gu.rel_fro(Y, ref)
    assert err < BAR, (wname, M, kind, err)
    xn = np.linalg.norm(orc.bf16_bits_to_f32(Xh).astype(np.float64), axis=1)
    wn = np.linalg.norm(orc.bf16_bits_to_f32(wd).astype(np.float64), axis=1)
    c = np.sqrt(K) / (127 * 256) + 2.0 ** -9 + 1e-5
    bound = c * np.outer(xn, wn)
    worst = float(np.max(np.abs(Y - ref) / bound))
    assert worst <= 1.0, (wname, M, kind, worst)
    assert e8.e8_sync_status(gcb) == e8.E8_OK

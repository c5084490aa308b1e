"""GPU-vs-oracle parity of the TL2-style storage (5 bits per three weights):
the conversion from 2-bit rows must give the oracle's bytes exactly, and the
TL2 decode GEMV the oracle's int32 accumulators and fp32 outputs exactly."""
import numpy as np
import pytest
import torch

import oracle
from ternary_weight_bit_bitlinear_b200 import _lib, api, build, inputs

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _gpu():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    build.build()
    _lib.load()
    yield
    assert _lib.bitlinear_device_error(clear=True) == _lib.OK


SHAPES = [(1, 96), (33, 112), (64, 384), (300, 2560), (129, 6912), (7, 16), (50, 176),
          (40, 4096), (9, 80)]


def _layer(M, K, seed):
    W = inputs.latent_weights(M, K, seed=seed)
    packed, alpha = api.pack_weights(W.cuda())
    return W, packed, alpha


@pytest.mark.parametrize("M,K", SHAPES)
def test_tl2_conversion_bytes(M, K):
    W, packed, alpha = _layer(M, K, 3 * M + K)
    t = api.tl2_from_packed(packed, K)
    codes = oracle.ternarize(W.numpy(), oracle.absmean(W.numpy()))
    ref = oracle.tl2_encode(codes)
    assert t.shape == ref.shape
    assert np.array_equal(t.cpu().numpy(), ref)


@pytest.mark.parametrize("N", list(range(1, 17)))
def test_gemv_tl2_all_token_counts(N):
    M, K = 300, 2560        # 26 blocks of 96 and a 64-weight remainder; ragged row blocks
    W, packed, alpha = _layer(M, K, 40 + N)
    x = inputs.activations(N, K, seed=60 + N, outlier_frac=0.01)
    ref = oracle.bitlinear(W.numpy(), x.numpy())
    xq, amax, _ = api.quant_act(x.cuda())
    y, acc = api.gemv_tl2(api.tl2_from_packed(packed, K), alpha, xq, amax, with_acc=True)
    assert np.array_equal(acc.cpu().numpy(), ref["acc"])
    assert np.array_equal(y.cpu().numpy(), ref["y"])


@pytest.mark.parametrize("N", [1, 4])
@pytest.mark.parametrize("M,K", SHAPES)
def test_gemv_tl2_shapes(M, K, N):
    W, packed, alpha = _layer(M, K, 5 * M + K + N)
    x = inputs.activations(N, K, seed=7 * M + K + N, outlier_frac=0.02)
    ref = oracle.bitlinear(W.numpy(), x.numpy())
    xq, amax, _ = api.quant_act(x.cuda())
    y, acc = api.gemv_tl2(api.tl2_from_packed(packed, K), alpha, xq, amax, with_acc=True)
    assert np.array_equal(acc.cpu().numpy(), ref["acc"])
    assert np.array_equal(y.cpu().numpy(), ref["y"])


@pytest.mark.parametrize("N", [1, 3, 16])
def test_gemv_tl2_grouped_mixed(N):
    shapes = [(2560, 2560), (640, 2560), (2560, 6912), (33, 112), (96, 16)]
    ents, refs, ys, accs = [], [], [], []
    for i, (M, K) in enumerate(shapes):
        W, packed, alpha = _layer(M, K, 800 + 11 * i + N)
        x = inputs.activations(N, K, seed=850 + 11 * i + N, outlier_frac=0.01)
        refs.append(oracle.bitlinear(W.numpy(), x.numpy()))
        xq, amax, _ = api.quant_act(x.cuda())
        y = torch.empty((N, M), device="cuda")
        acc = torch.empty((N, M), dtype=torch.int32, device="cuda")
        ys.append(y)
        accs.append(acc)
        ents.append((api.tl2_from_packed(packed, K), alpha, M, K, xq, amax, y, acc))
    arr = _lib.make_tl2_problems(ents)
    assert _lib.bitlinear_gemv_tl2_grouped(arr, len(ents), N, None) == _lib.OK
    for y, acc, ref in zip(ys, accs, refs):
        assert np.array_equal(acc.cpu().numpy(), ref["acc"])
        assert np.array_equal(y.cpu().numpy(), ref["y"])


def test_gemv_tl2_equals_two_bit_gemv():
    M, K, N = 2560, 6912, 2
    W, packed, alpha = _layer(M, K, 99)
    x = inputs.activations(N, K, seed=98).cuda()
    xq, amax, xsum = api.quant_act(x)
    y2 = api.gemv(packed, alpha, xq, amax, xsum)
    yt = api.gemv_tl2(api.tl2_from_packed(packed, K), alpha, xq, amax)
    assert torch.equal(y2, yt)

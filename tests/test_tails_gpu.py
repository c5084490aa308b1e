"""GPU-vs-oracle parity on ragged shapes: K any multiple of 16 (packed rows
padded to 16 bytes with code-0 fields) and any M, through every kernel --
pack, quantiser, GEMV, fused quantise+GEMV and the tensor-core GEMM (whose
ragged tiles read zeros past M, K and N through the tensor maps, and whose
outputs go through plain stores when 4*M is not a multiple of 16).
"""
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


SHAPES = [(1, 16), (3, 48), (33, 80), (100, 144), (129, 1008), (260, 2000), (7, 64)]


def _case(M, K, N, seed):
    W = inputs.latent_weights(M, K, seed=seed)
    x = inputs.activations(N, K, seed=seed + 500, outlier_frac=0.02)
    return W, x, oracle.bitlinear(W.numpy(), x.numpy())


@pytest.mark.parametrize("M,K", SHAPES)
def test_pack_ragged(M, K):
    W = inputs.latent_weights(M, K, seed=M * 31 + K)
    packed, alpha = api.pack_weights(W.cuda())
    a_ref = oracle.absmean(W.numpy())
    p_ref = oracle.pack(oracle.ternarize(W.numpy(), a_ref))
    assert packed.shape == p_ref.shape == (M, api.packed_row_words(K))
    assert alpha.item() == a_ref
    assert np.array_equal(packed.cpu().numpy().view(np.uint32), p_ref)


@pytest.mark.parametrize("N,K", [(1, 16), (3, 48), (5, 1008), (2, 2000)])
def test_quant_ragged(N, K):
    x = inputs.activations(N, K, seed=N + K, outlier_frac=0.02)
    xq, amax, xsum = api.quant_act(x.cuda())
    q, a, s = oracle.quant_act(x.numpy())
    assert np.array_equal(xq.cpu().numpy(), q)
    assert np.array_equal(amax.cpu().numpy(), a) and np.array_equal(xsum.cpu().numpy(), s)


@pytest.mark.parametrize("N", [1, 5, 16])
@pytest.mark.parametrize("M,K", SHAPES)
def test_gemv_and_fused_ragged(M, K, N):
    W, x, ref = _case(M, K, N, seed=10 * M + K + N)
    packed, alpha = api.pack_weights(W.cuda())
    xq, amax, xsum = api.quant_act(x.cuda())
    y, acc = api.gemv(packed, alpha, xq, amax, xsum, with_acc=True)
    assert np.array_equal(acc.cpu().numpy(), ref["acc"])
    assert np.array_equal(y.cpu().numpy(), ref["y"])
    y2, acc2 = api.gemv_quant(packed, alpha, x.cuda(), with_acc=True)
    assert np.array_equal(acc2.cpu().numpy(), ref["acc"])
    assert np.array_equal(y2.cpu().numpy(), ref["y"])


@pytest.mark.parametrize("N", [1, 100, 300])
@pytest.mark.parametrize("M,K", SHAPES + [(384, 144), (4, 16), (130, 4096)])
def test_gemm_ragged(M, K, N):
    # M % 4 != 0 (1, 3, 33, 129, 7, 130 ...) takes the plain-store epilogue;
    # M % 4 == 0 but M % 128 != 0 (100, 260, 4) clips the tensor stores
    W, x, ref = _case(M, K, N, seed=20 * M + K + N)
    packed, alpha = api.pack_weights(W.cuda())
    xq, amax, xsum = api.quant_act(x.cuda())
    y, acc = api.gemm(packed, alpha, xq, amax, xsum, with_acc=True)
    assert np.array_equal(acc.cpu().numpy(), ref["acc"])
    assert np.array_equal(y.cpu().numpy(), ref["y"])


@pytest.mark.parametrize("M", [130, 132])
def test_gemm_ragged_outputs_stay_in_bounds(M):
    # y is a view into a larger buffer filled with a sentinel: nothing past
    # [N, M] may change (130: plain stores; 132: clipped tensor stores)
    K, N = 208, 70
    W, x, ref = _case(M, K, N, seed=77 + M)
    packed, alpha = api.pack_weights(W.cuda())
    xq, amax, xsum = api.quant_act(x.cuda())
    big = torch.full((N * M + 4096,), 12345.0, device="cuda")
    y = big[:N * M].view(N, M)
    api.gemm(packed, alpha, xq, amax, xsum, out=y)
    assert np.array_equal(y.cpu().numpy(), ref["y"])
    assert (big[N * M:] == 12345.0).all()


@pytest.mark.parametrize("N", [1, 64, 257])
def test_gemm_grouped_ragged_mixed(N):
    shapes = [(129, 1008), (100, 144), (3, 48), (256, 2000), (1, 16)]
    layers, refs, xqs, ams, xss = [], [], [], [], []
    for i, (M, K) in enumerate(shapes):
        W, x, ref = _case(M, K, N, seed=500 + 7 * i + N)
        refs.append(ref)
        layers.append(api.pack_weights(W.cuda()))
        q = api.quant_act(x.cuda())
        xqs.append(q[0]); ams.append(q[1]); xss.append(q[2])
    ys, accs = api.gemm_grouped(layers, xqs, ams, xss, with_acc=True)
    for y, acc, ref in zip(ys, accs, refs):
        assert np.array_equal(acc.cpu().numpy(), ref["acc"])
        assert np.array_equal(y.cpu().numpy(), ref["y"])


def test_ternary_linear_ragged():
    W = inputs.latent_weights(37, 80, seed=91)
    lin = api.TernaryLinear.from_float(W.cuda())
    for N in (1, 40):
        x = inputs.activations(N, 80, seed=92 + N)
        ref = oracle.bitlinear(W.numpy(), x.numpy())
        assert np.array_equal(lin(x.cuda()).cpu().numpy(), ref["y"])

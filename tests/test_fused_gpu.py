"""GPU-vs-oracle parity of the fused decode kernel (bitlinear_gemv_quant and
its grouped form), which takes fp32 activations and quantises them itself.

The oracle quantises the same fp32 buffers on the host; int32 accumulators
must match exactly, and so must the fp32 outputs (same operation order on both
sides, the 1e-6 relative bar is written in assert_y_close).
"""
import numpy as np
import pytest
import torch

import oracle
from ternary_weight_bit_bitlinear_b200 import _lib, api, build, inputs

pytestmark = pytest.mark.gpu

REL_TOL = 1e-6


@pytest.fixture(scope="module", autouse=True)
def _gpu():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    build.build()
    _lib.load()
    yield
    assert _lib.bitlinear_device_error(clear=True) == _lib.OK


def dev_t(a):
    return torch.from_numpy(np.ascontiguousarray(a)).cuda()


def assert_y_close(y_gpu, y_ref):
    y_gpu = np.asarray(y_gpu, np.float64)
    y_ref = np.asarray(y_ref, np.float64)
    zero = y_ref == 0
    assert (y_gpu[zero] == 0).all()
    rel = np.abs(y_gpu[~zero] - y_ref[~zero]) / np.abs(y_ref[~zero])
    assert rel.size == 0 or rel.max() <= REL_TOL, rel.max()


def check(y, acc, ref):
    assert np.array_equal(acc.cpu().numpy(), ref["acc"])
    assert_y_close(y.cpu().numpy(), ref["y"])
    assert np.array_equal(y.cpu().numpy(), ref["y"])


def layer(M, K, seed):
    W = inputs.latent_weights(M, K, seed=seed)
    return W, api.pack_weights(W.cuda())


@pytest.mark.parametrize("N", list(range(1, 17)))
def test_gemv_quant_all_token_counts(N):
    # ragged row blocks (300 = 9 x 32 + 12) and a ragged last k-chunk (640 = 512 + 128)
    M, K = 300, 640
    W, (packed, alpha) = layer(M, K, 700 + N)
    x = inputs.activations(N, K, seed=1200 + N, outlier_frac=0.01)
    y, acc = api.gemv_quant(packed, alpha, x.cuda(), with_acc=True)
    check(y, acc, oracle.bitlinear(W.numpy(), x.numpy()))


@pytest.mark.parametrize("M,K,N", [(1024, 1024, 1), (2560, 6912, 1), (640, 2560, 4),
                                   (1, 128, 1), (129, 28672, 2), (96, 65536, 1),
                                   (64, 4096, 16), (33, 2944, 3)])
def test_gemv_quant_shapes(M, K, N):
    # includes the largest K per token count the kernel takes (65536 at N = 1,
    # 4096 at N = 16) and K = 2944, a multiple of 128 but not of 512
    W, (packed, alpha) = layer(M, K, M + K + N)
    x = inputs.activations(N, K, seed=M * 3 + K + N, outlier_frac=0.01)
    y, acc = api.gemv_quant(packed, alpha, x.cuda(), with_acc=True)
    check(y, acc, oracle.bitlinear(W.numpy(), x.numpy()))


@pytest.mark.parametrize("M,K,N", [(160012, 64, 1), (160012, 64, 4), (160012, 640, 3)])
def test_gemv_quant_many_units_small_k(M, K, N):
    # Many more 32-row units (5001) than CTAs: every CTA takes a range of
    # several units, its warps a share of their k-chunks.  Ragged rows
    # (160012 = 5000 x 32 + 12) and a ragged k-chunk.
    W, (packed, alpha) = layer(M, K, M + K + N)
    x = inputs.activations(N, K, seed=K + 7 * N, outlier_frac=0.01)
    y, acc = api.gemv_quant(packed, alpha, x.cuda(), with_acc=True)
    check(y, acc, oracle.bitlinear(W.numpy(), x.numpy()))


@pytest.mark.parametrize("K", [512, 1024, 1536, 2048, 2560, 6912])
def test_gemv_quant_split_units_chunk_counts(K):
    # Small launches (7 units, fewer than CTAs): one unit per CTA, the unit's
    # k-chunks split over the CTA's warps (1, 2, 3, 4, 5 and 14 chunks: some
    # warps get none, some one, some several, and the warp holding chunk 0 adds
    # the others' partial sums).
    M, N = 200, 2
    W, (packed, alpha) = layer(M, K, 31 * K + N)
    x = inputs.activations(N, K, seed=K + 3, outlier_frac=0.01)
    y, acc = api.gemv_quant(packed, alpha, x.cuda(), with_acc=True)
    check(y, acc, oracle.bitlinear(W.numpy(), x.numpy()))


def test_gemv_quant_equals_two_step_path():
    M, K, N = 2560, 2560, 3
    W, (packed, alpha) = layer(M, K, 77)
    x = inputs.activations(N, K, seed=78).cuda()
    y1 = api.gemv_quant(packed, alpha, x)
    xq, amax, xsum = api.quant_act(x)
    y2 = api.gemv(packed, alpha, xq, amax, xsum)
    assert torch.equal(y1, y2)


def test_gemv_quant_edge_values():
    M, K, N = 96, 1024, 4
    W, (packed, alpha) = layer(M, K, 91)
    x = inputs.activations(N, K, seed=92).numpy()
    x[0] = 0.0                                  # a zero token: amax 0, y 0
    x[1] = -0.0                                 # negative zeros too
    x[2, :] = 0.25
    x[2, :6] = [127.0, 0.5, 1.5, 2.5, -2.5, -0.5]   # exact .5 ties: half to even
    x[3, 5] = -1e30                             # one huge outlier: most q round to 0
    y, acc = api.gemv_quant(packed, alpha, dev_t(x), with_acc=True)
    ref = oracle.bitlinear(W.numpy(), x)
    check(y, acc, ref)
    assert not y[0].any() and not y[1].any()


def test_gemv_quant_zero_weights():
    M, K, N = 64, 512, 2
    packed, alpha = api.pack_weights(torch.zeros(M, K, device="cuda"))
    x = inputs.activations(N, K, seed=5).cuda()
    y, acc = api.gemv_quant(packed, alpha, x, with_acc=True)
    assert not acc.any() and not y.any()


@pytest.mark.parametrize("N", [1, 2, 5])
def test_gemv_quant_grouped_decoder_layer(N):
    # one decoder layer of the 2B shape: q, k, v read one input, o another,
    # gate and up a third, down the ffn-wide one; shared inputs are passed
    # as the same tensor, next to each other
    shape = inputs.MODEL_2B
    xs = {p: inputs.activations(N, shape.ffn if p == 6 else shape.hidden, seed=40 + p)
          for p in (0, 3, 4, 6)}
    src = [0, 0, 0, 3, 4, 4, 6]
    Ws, layers = [], []
    for p, (_, M, K) in enumerate(shape.projections()):
        W, pk = layer(M, K, 50 + p)
        Ws.append(W)
        layers.append(pk)
    xd = {p: v.cuda() for p, v in xs.items()}
    ys, accs = api.gemv_quant_grouped(layers, [xd[s] for s in src], with_acc=True)
    for p in range(7):
        check(ys[p], accs[p], oracle.bitlinear(Ws[p].numpy(), xs[src[p]].numpy()))


@pytest.mark.parametrize("N", [1, 3, 16])
def test_gemv_quant_grouped_mixed_k(N):
    shapes = [(2560, 2560), (640, 2560), (2560, 3968), (96, 4096), (33, 128)]
    layers, refs, xs = [], [], []
    for i, (M, K) in enumerate(shapes):
        W, pk = layer(M, K, 900 + 7 * i + N)
        x = inputs.activations(N, K, seed=950 + 7 * i + N, outlier_frac=0.01)
        refs.append(oracle.bitlinear(W.numpy(), x.numpy()))
        layers.append(pk)
        xs.append(x.cuda())
    ys, accs = api.gemv_quant_grouped(layers, xs, with_acc=True)
    for y, acc, ref in zip(ys, accs, refs):
        check(y, acc, ref)


def test_gemv_quant_grouped_many_problems():
    # 300 layers (two launches), each with its own input, rows of one stacked
    # activation buffer: a CTA whose range crosses a layer boundary quantises
    # the next input before it goes on
    K, M, L = 640, 96, 300
    X = inputs.activations(L, K, seed=61, outlier_frac=0.02)
    W, (packed, alpha) = layer(M, K, 62)
    Xd = X.cuda()
    ys, accs = api.gemv_quant_grouped([(packed, alpha)] * L, [Xd[i:i + 1] for i in range(L)],
                                      with_acc=True)
    ref = oracle.bitlinear(W.numpy(), X.numpy())
    assert np.array_equal(torch.cat(accs).cpu().numpy(), ref["acc"])
    assert np.array_equal(torch.cat(ys).cpu().numpy(), ref["y"])


@pytest.mark.parametrize("N", [1, 2, 4])
def test_gemv_quant_ctas_span_several_inputs(N):
    # 256 layers of 5 units each (1280 units, more than the CTAs of a launch),
    # each with its own input: CTA ranges cross two or three inputs, which the
    # CTA quantises one after the other; units split between warps and between
    # inputs at every boundary.
    K, M, L = 1024, 160, 256
    X = inputs.activations(L * N, K, seed=63 + N, outlier_frac=0.02)
    W, (packed, alpha) = layer(M, K, 64)
    Xd = X.cuda()
    ys, accs = api.gemv_quant_grouped([(packed, alpha)] * L,
                                      [Xd[i * N:(i + 1) * N] for i in range(L)], with_acc=True)
    codes = oracle.ternarize(W.numpy(), oracle.absmean(W.numpy()))
    for i in (0, 1, 2, 97, 128, 200, 255):
        ref = oracle.bitlinear(W.numpy(), X[i * N:(i + 1) * N].numpy())
        assert np.array_equal(accs[i].cpu().numpy(), ref["acc"]), i
        assert np.array_equal(ys[i].cpu().numpy(), ref["y"]), i
    # every layer: the int32 sums against the oracle's integer product
    q, _, _ = oracle.quant_act(X.numpy())
    acc_all = oracle.matmul_i32(codes, q)                      # [L*N, M]
    assert np.array_equal(torch.cat(accs).cpu().numpy(), acc_all)


@pytest.mark.parametrize("N", [1, 3])
def test_gemv_quant_many_small_problems_in_segments(N):
    # 240 problems of 2 units (M = 40) and 3 k-chunks (K = 1536) in segments of
    # three that share an input (like q, k, v): warp shares start and end at
    # every position, so a warp's first stages often reach the next problem
    # and the next segment.
    K, M, L = 1536, 40, 240
    X = inputs.activations((L // 3) * N, K, seed=65 + N, outlier_frac=0.02)
    Ws = [inputs.latent_weights(M, K, seed=1000 + i) for i in range(4)]
    packs = [api.pack_weights(W.cuda()) for W in Ws]
    Xd = X.cuda()
    xs = [Xd[(i // 3) * N:(i // 3 + 1) * N] for i in range(L)]
    ys, accs = api.gemv_quant_grouped([packs[i % 4] for i in range(L)], xs, with_acc=True)
    for i in range(L):
        ref = oracle.bitlinear(Ws[i % 4].numpy(), X[(i // 3) * N:(i // 3 + 1) * N].numpy())
        assert np.array_equal(accs[i].cpu().numpy(), ref["acc"]), i
        assert np.array_equal(ys[i].cpu().numpy(), ref["y"]), i


def test_gemv_quant_same_pointer_different_k():
    # two layers read prefixes of one buffer with different K: the kernel must
    # quantise each separately (amax is per row of the K it is given)
    N = 2
    big = inputs.activations(N, 2048, seed=71)
    a = big[:, :1024].contiguous()
    buf = torch.empty(N * 2048, device="cuda")
    buf[:N * 1024] = a.cuda().reshape(-1)          # x of layer 0: [N, 1024] at offset 0
    x0 = buf[:N * 1024].view(N, 1024)
    x1 = buf[:N * 512].view(N, 512)                # layer 1 reads [N, 512] from the same start
    W0, l0 = layer(64, 1024, 72)
    W1, l1 = layer(64, 512, 73)
    ys, accs = api.gemv_quant_grouped([l0, l1], [x0, x1], with_acc=True)
    check(ys[0], accs[0], oracle.bitlinear(W0.numpy(), x0.cpu().numpy()))
    check(ys[1], accs[1], oracle.bitlinear(W1.numpy(), x1.cpu().numpy()))


def test_gemv_quant_rejects_oversize_on_device():
    packed = torch.zeros((32, 4096 // 16 + 8), dtype=torch.int32, device="cuda")
    alpha = torch.ones(1, device="cuda")
    x = torch.zeros((16, 4224), device="cuda")
    y = torch.empty((16, 32), device="cuda")
    st = _lib.bitlinear_gemv_quant(packed, alpha, 32, 4224, x, 16, y)
    assert st == _lib.ERR_UNSUPPORTED_SHAPE


def test_ternary_linear_uses_fused_path_for_decode():
    W = inputs.latent_weights(640, 2560, seed=81)
    lin = api.TernaryLinear.from_float(W.cuda())
    x = inputs.activations(2, 2560, seed=82)
    ref = oracle.bitlinear(W.numpy(), x.numpy())
    assert np.array_equal(lin(x.cuda()).cpu().numpy(), ref["y"])

"""GPU-vs-oracle parity through the C ABI (ctypes view in ternary_weight_bit_bitlinear_b200._lib).

Inputs come from the seeded generators in ternary_weight_bit_bitlinear_b200.inputs;
the oracle sees the same fp32 buffers on the host.  The bar: packed words,
alpha, int8 activations, amax, activation sums and int32 accumulators
bit-exact; fp32 outputs within 1e-6 relative (they are expected bit-exact,
since both sides use the same fp32 operation order), zeros exactly zero.
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


def words(t):
    return t.cpu().numpy().view(np.uint32)


def assert_y_close(y_gpu, y_ref):
    y_gpu = np.asarray(y_gpu, np.float64)
    y_ref = np.asarray(y_ref, np.float64)
    zero = y_ref == 0
    assert (y_gpu[zero] == 0).all()
    rel = np.abs(y_gpu[~zero] - y_ref[~zero]) / np.abs(y_ref[~zero])
    assert rel.size == 0 or rel.max() <= REL_TOL, rel.max()


# ----------------------------------------------------------------------------- pack

PACK_SHAPES = [(128, 128), (7, 256), (300, 640), (1024, 1024), (640, 2560), (2560, 6912)]


@pytest.mark.parametrize("M,K", PACK_SHAPES)
def test_pack_parity(M, K):
    W = inputs.latent_weights(M, K, seed=M * 7 + K)
    packed, alpha = api.pack_weights(W.cuda())
    a_ref = oracle.absmean(W.numpy())
    p_ref = oracle.pack(oracle.ternarize(W.numpy(), a_ref))
    assert alpha.cpu().numpy()[0] == a_ref
    assert np.array_equal(words(packed), p_ref)


def test_pack_edge_cases():
    # all zero -> alpha 0, every code 0 (field 01)
    z = torch.zeros(128, 256, device="cuda")
    packed, alpha = api.pack_weights(z)
    assert alpha.item() == 0.0 and (words(packed) == 0x55555555).all()
    # exact ties: values +-0.5 and +-1.5 in equal numbers -> alpha = 1 exactly,
    # 0.5 -> 0 (half to even), 1.5 -> clamp(2) = 1
    base = np.array([0.5, -0.5, 1.5, -1.5], np.float32)
    W = np.tile(base, (128, 64))
    packed, alpha = api.pack_weights(dev_t(W))
    assert alpha.item() == 1.0
    codes = oracle.unpack(words(packed), 128, 256)
    assert np.array_equal(codes, np.tile(np.array([0, 0, 1, -1], np.int8), (128, 64)))
    assert np.array_equal(words(packed), oracle.pack(oracle.ternarize(W, np.float32(1.0))))
    # subnormal-only weights
    W = (np.arange(128 * 128, dtype=np.float32).reshape(128, 128) % 97 + 1) * np.float32(1e-45)
    packed, alpha = api.pack_weights(dev_t(W))
    a_ref = oracle.absmean(W)
    assert alpha.cpu().numpy()[0] == a_ref
    assert np.array_equal(words(packed), oracle.pack(oracle.ternarize(W, a_ref)))
    # non-finite -> alpha NaN, codes 0, and the device error word says so
    assert _lib.bitlinear_device_error(clear=True) == _lib.OK
    W = np.ones((128, 128), np.float32)
    W[3, 5] = np.inf
    packed, alpha = api.pack_weights(dev_t(W))
    assert np.isnan(alpha.item()) and (words(packed) == 0x55555555).all()
    assert _lib.bitlinear_device_error(clear=True) == _lib.ERR_NONFINITE
    assert _lib.bitlinear_device_error(clear=True) == _lib.OK


# ----------------------------------------------------------------------------- quant_act

QUANT_SHAPES = [(1, 1024), (3, 2560), (16, 6912), (33, 4096), (2, 131072), (512, 128)]


@pytest.mark.parametrize("N,K", QUANT_SHAPES)
def test_quant_act_parity(N, K):
    x = inputs.activations(N, K, seed=N * 13 + K, outlier_frac=0.01)
    xq, amax, xsum = api.quant_act(x.cuda())
    q_ref, a_ref, s_ref = oracle.quant_act(x.numpy())
    assert np.array_equal(xq.cpu().numpy(), q_ref)
    assert np.array_equal(amax.cpu().numpy(), a_ref)
    assert np.array_equal(xsum.cpu().numpy(), s_ref)


def test_quant_act_edge_cases():
    x = np.zeros((4, 256), np.float32)
    x[1, :] = np.linspace(-3, 3, 256)
    x[2, :4] = [1e-44, -1e-44, 0.0, 5e-45]          # 127/amax overflows to inf
    x[3, :] = 127.0
    x[3, :6] = [0.5, 1.5, 2.5, -0.5, -1.5, -2.5]     # s == 1: ties to even
    xq, amax, xsum = api.quant_act(dev_t(x))
    q_ref, a_ref, s_ref = oracle.quant_act(x)
    assert np.array_equal(xq.cpu().numpy(), q_ref)
    assert np.array_equal(amax.cpu().numpy(), a_ref)
    assert np.array_equal(xsum.cpu().numpy(), s_ref)
    assert xq[3, :6].tolist() == [0, 2, 2, 0, -2, -2]


def test_quant_act_grouped_parity():
    shapes = [(90, 2560), (30, 6912), (0, 1024), (5, 131072), (1, 128), (64, 8192), (3, 8320)]
    xs = [inputs.activations(N, K, seed=N + K, outlier_frac=0.01) for N, K in shapes]
    outs = api.quant_act_grouped([x.cuda() for x in xs])
    for x, (xq, amax, xsum) in zip(xs, outs):
        q_ref, a_ref, s_ref = oracle.quant_act(x.numpy())
        assert np.array_equal(xq.cpu().numpy(), q_ref)
        assert np.array_equal(amax.cpu().numpy(), a_ref)
        assert np.array_equal(xsum.cpu().numpy(), s_ref)


@pytest.mark.parametrize("N,K", [(1, 8320), (2, 12288), (1, 16384), (1, 16400), (3, 28672),
                                 (1, 32768), (1, 32784)])
def test_quant_act_few_rows_wide_ctas(N, K):
    # fewer rows than SMs: CTAs of 512 threads for rows of 8193..16384, 1024
    # above (rows past 32768 are read twice)
    x = inputs.activations(N, K, seed=N * 31 + K, outlier_frac=0.01)
    xq, amax, xsum = api.quant_act(x.cuda())
    q_ref, a_ref, s_ref = oracle.quant_act(x.numpy())
    assert np.array_equal(xq.cpu().numpy(), q_ref)
    assert np.array_equal(amax.cpu().numpy(), a_ref)
    assert np.array_equal(xsum.cpu().numpy(), s_ref)


def test_quant_act_grouped_few_rows():
    # one launch of 3 rows: every row on a CTA sized for the widest (28672)
    shapes = [(1, 8192), (1, 28672), (0, 64), (1, 2560)]
    xs = [inputs.activations(N, K, seed=3 * N + K, outlier_frac=0.01) for N, K in shapes]
    outs = api.quant_act_grouped([x.cuda() for x in xs])
    for x, (xq, amax, xsum) in zip(xs, outs):
        q_ref, a_ref, s_ref = oracle.quant_act(x.numpy())
        assert np.array_equal(xq.cpu().numpy(), q_ref)
        assert np.array_equal(amax.cpu().numpy(), a_ref)
        assert np.array_equal(xsum.cpu().numpy(), s_ref)


@pytest.mark.parametrize("N,K", [(1, 2560), (7, 1024), (64, 4096), (300, 6912), (2, 131072)])
def test_quant_act_per_tensor_parity(N, K):
    x = inputs.activations(N, K, seed=N * 5 + K, outlier_frac=0.01)
    xq, amax, xsum = api.quant_act_per_tensor(x.cuda())
    q_ref, a_ref, s_ref = oracle.quant_act_per_tensor(x.numpy())
    assert np.array_equal(xq.cpu().numpy(), q_ref)
    assert np.array_equal(amax.cpu().numpy(), a_ref)
    assert np.array_equal(xsum.cpu().numpy(), s_ref)


@pytest.mark.parametrize("N", [3, 200])
def test_per_tensor_activations_through_matmul(N):
    M, K = 384, 2048
    W = inputs.latent_weights(M, K, seed=61)
    x = inputs.activations(N, K, seed=62, outlier_frac=0.01)
    a = oracle.absmean(W.numpy())
    codes = oracle.ternarize(W.numpy(), a)
    q, amax, _ = oracle.quant_act_per_tensor(x.numpy())
    acc = oracle.matmul_i32(codes, q)
    y_ref = oracle.rescale(acc, a, amax)
    packed, alpha = api.pack_weights(W.cuda())
    xq, am, xs = api.quant_act_per_tensor(x.cuda())
    y, acc_d = api.matmul(packed, alpha, xq, am, xs, with_acc=True)
    assert np.array_equal(acc_d.cpu().numpy(), acc)
    assert np.array_equal(y.cpu().numpy(), y_ref)


def test_quant_act_per_tensor_edge_cases():
    x = np.zeros((3, 256), np.float32)
    xq, amax, xsum = api.quant_act_per_tensor(dev_t(x))
    assert not xq.cpu().numpy().any() and not amax.cpu().numpy().any()
    x[1, 7] = -127.0
    x[2, :4] = [0.5, 1.5, 2.5, -2.5]
    xq, amax, xsum = api.quant_act_per_tensor(dev_t(x))
    q_ref, a_ref, s_ref = oracle.quant_act_per_tensor(x)
    assert np.array_equal(xq.cpu().numpy(), q_ref) and (amax.cpu().numpy() == 127).all()
    assert xq[2, :4].tolist() == [0, 2, 2, -2]


# ----------------------------------------------------------------------------- matmul

def _layer(M, K, N, seed, outlier_frac=0.0):
    W = inputs.latent_weights(M, K, seed=seed)
    x = inputs.activations(N, K, seed=seed + 500, outlier_frac=outlier_frac)
    ref = oracle.bitlinear(W.numpy(), x.numpy())
    packed, alpha = api.pack_weights(W.cuda())
    xq, amax, xsum = api.quant_act(x.cuda())
    return ref, (packed, alpha, xq, amax, xsum)


@pytest.mark.parametrize("N", list(range(1, 17)))
def test_gemv_parity_all_token_counts(N):
    M, K = 300, 640        # ragged row blocks
    ref, (packed, alpha, xq, amax, xsum) = _layer(M, K, N, seed=100 + N)
    y, acc = api.gemv(packed, alpha, xq, amax, xsum, with_acc=True)
    assert np.array_equal(acc.cpu().numpy(), ref["acc"])
    assert_y_close(y.cpu().numpy(), ref["y"])
    assert np.array_equal(y.cpu().numpy(), ref["y"])


@pytest.mark.parametrize("M,K,N", [(160012, 64, 1), (160012, 640, 4), (160012, 64, 16)])
def test_gemv_parity_tile_kernel_many_units(M, K, N):
    # 5001 units: more than gemv_tile_kernel can have warps resident at any
    # token count (148 SMs x at most 3 CTAs x 4 warps), so these launches take
    # it rather than the split-unit kernel that the smaller cases here take.
    ref, (packed, alpha, xq, amax, xsum) = _layer(M, K, N, seed=M + K + N)
    y, acc = api.gemv(packed, alpha, xq, amax, xsum, with_acc=True)
    assert np.array_equal(acc.cpu().numpy(), ref["acc"])
    assert np.array_equal(y.cpu().numpy(), ref["y"])


@pytest.mark.parametrize("M,K", [(57600, 256), (113696, 128)])
def test_gemv_parity_split_kernel_just_over_capacity(M, K):
    # 1800 and 3553 units at N = 1, a little over one and two times the 1776
    # warps gemv_tile_kernel can have resident: the tile kernel would idle
    # about half and a third of them, so these take the split-unit kernel
    ref, (packed, alpha, xq, amax, xsum) = _layer(M, K, 1, seed=M + K)
    y, acc = api.gemv(packed, alpha, xq, amax, xsum, with_acc=True)
    assert np.array_equal(acc.cpu().numpy(), ref["acc"])
    assert np.array_equal(y.cpu().numpy(), ref["y"])


@pytest.mark.parametrize("K", [512, 1024, 1536, 2048, 2560, 6912])
@pytest.mark.parametrize("N", [1, 5, 16])
def test_gemv_parity_split_kernel_chunk_counts(K, N):
    # small launches: one 4-warp CTA per unit, its 1 to 14 k-chunks split
    # over the warps (some warps get none)
    ref, (packed, alpha, xq, amax, xsum) = _layer(200, K, N, seed=7 * K + N)
    y, acc = api.gemv(packed, alpha, xq, amax, xsum, with_acc=True)
    assert np.array_equal(acc.cpu().numpy(), ref["acc"])
    assert np.array_equal(y.cpu().numpy(), ref["y"])


@pytest.mark.parametrize("M,K,N", [(1024, 1024, 1), (2560, 6912, 1), (640, 2560, 4),
                                   (6912, 2560, 16), (1, 128, 1), (129, 28672, 2)])
def test_gemv_parity_shapes(M, K, N):
    ref, (packed, alpha, xq, amax, xsum) = _layer(M, K, N, seed=M + K + N, outlier_frac=0.01)
    y, acc = api.gemv(packed, alpha, xq, amax, xsum, with_acc=True)
    assert np.array_equal(acc.cpu().numpy(), ref["acc"])
    assert_y_close(y.cpu().numpy(), ref["y"])


@pytest.mark.parametrize("N", [1, 2, 3, 4, 7])
@pytest.mark.parametrize("K", [1024, 2560, 6912, 28672])
def test_gemv_grouped_parity(K, N):
    Ms = [640, 128, 2560, 300]
    layers, refs = [], []
    x = inputs.activations(N, K, seed=K + N, outlier_frac=0.01)
    for i, M in enumerate(Ms):
        W = inputs.latent_weights(M, K, seed=1000 * i + K + N)
        refs.append(oracle.bitlinear(W.numpy(), x.numpy()))
        layers.append(api.pack_weights(W.cuda()))
    xq, amax, xsum = api.quant_act(x.cuda())
    ys, accs = api.gemv_grouped(layers, xq, amax, xsum, with_acc=True)
    for y, acc, ref in zip(ys, accs, refs):
        assert np.array_equal(acc.cpu().numpy(), ref["acc"])
        assert np.array_equal(y.cpu().numpy(), ref["y"])


def test_gemv_grouped_many_problems_and_row_views():
    # 150 problems (more than one launch's table), activations as row views of
    # one stacked buffer (4-byte aligned amax/xsum pointers)
    K, M = 512, 256
    X = inputs.activations(150, K, seed=31)
    xq, amax, xsum = api.quant_act(X.cuda())
    W = inputs.latent_weights(M, K, seed=32)
    packed, alpha = api.pack_weights(W.cuda())
    ys, accs = api.gemv_grouped([(packed, alpha)] * 150, [xq[i:i + 1] for i in range(150)],
                                [amax[i:i + 1] for i in range(150)],
                                [xsum[i:i + 1] for i in range(150)], with_acc=True)
    ref = oracle.bitlinear(W.numpy(), X.numpy())
    got = torch.cat(accs).cpu().numpy()
    assert np.array_equal(got, ref["acc"])
    assert np.array_equal(torch.cat(ys).cpu().numpy(), ref["y"])


def _mixed_layers(shapes, N, seed):
    layers, refs, qs = [], [], []
    for i, (M, K) in enumerate(shapes):
        W = inputs.latent_weights(M, K, seed=seed + 7 * i)
        x = inputs.activations(N, K, seed=seed + 7 * i + 500, outlier_frac=0.01)
        refs.append(oracle.bitlinear(W.numpy(), x.numpy()))
        layers.append(api.pack_weights(W.cuda()))
        qs.append(api.quant_act(x.cuda()))
    return layers, refs, [q[0] for q in qs], [q[1] for q in qs], [q[2] for q in qs]


@pytest.mark.parametrize("N", [1, 3, 16])
def test_gemv_grouped_mixed_k(N):
    shapes = [(2560, 2560), (640, 2560), (2560, 6912), (96, 11008), (33, 128)]
    layers, refs, xq, amax, xsum = _mixed_layers(shapes, N, seed=300 + N)
    ys, accs = api.gemv_grouped(layers, xq, amax, xsum, with_acc=True)
    for y, acc, ref in zip(ys, accs, refs):
        assert np.array_equal(acc.cpu().numpy(), ref["acc"])
        assert np.array_equal(y.cpu().numpy(), ref["y"])


@pytest.mark.parametrize("N", [1, 20, 100, 512])
def test_gemm_grouped_mixed_k(N):
    shapes = [(512, 1024), (256, 4096), (384, 2816), (128, 128)]
    layers, refs, xq, amax, xsum = _mixed_layers(shapes, N, seed=400 + N)
    ys, accs = api.gemm_grouped(layers, xq, amax, xsum, with_acc=True)
    for y, acc, ref in zip(ys, accs, refs):
        assert np.array_equal(acc.cpu().numpy(), ref["acc"])
        assert np.array_equal(y.cpu().numpy(), ref["y"])


def test_gemm_grouped_more_than_one_launch():
    # 10 layers > 8 per launch
    shapes = [(128 * (1 + i % 3), 256 * (1 + i % 2)) for i in range(10)]
    layers, refs, xq, amax, xsum = _mixed_layers(shapes, 40, seed=500)
    ys, accs = api.gemm_grouped(layers, xq, amax, xsum, with_acc=True)
    for y, acc, ref in zip(ys, accs, refs):
        assert np.array_equal(acc.cpu().numpy(), ref["acc"])
        assert np.array_equal(y.cpu().numpy(), ref["y"])


@pytest.mark.parametrize("M,K,N", [(128, 128, 1), (256, 512, 200), (384, 1024, 129),
                                   (128, 256, 16), (1024, 2560, 512), (512, 4096, 300),
                                   (256, 6912, 77),
                                   # up to 32 tokens: A in tensor memory, 16 or 32 wide
                                   (512, 2048, 4), (512, 2048, 25), (256, 14336, 32),
                                   (200, 1040, 2), (1000, 3072, 17), (4096, 4096, 8)])
def test_gemm_parity(M, K, N):
    ref, (packed, alpha, xq, amax, xsum) = _layer(M, K, N, seed=3 * M + K + N)
    y, acc = api.gemm(packed, alpha, xq, amax, xsum, with_acc=True)
    assert np.array_equal(acc.cpu().numpy(), ref["acc"])
    assert_y_close(y.cpu().numpy(), ref["y"])
    assert np.array_equal(y.cpu().numpy(), ref["y"])


def test_gemm_matches_gemv_small_n():
    ref, (packed, alpha, xq, amax, xsum) = _layer(512, 1024, 9, seed=77)
    y1, a1 = api.gemv(packed, alpha, xq, amax, xsum, with_acc=True)
    y2, a2 = api.gemm(packed, alpha, xq, amax, xsum, with_acc=True)
    assert torch.equal(a1, a2) and torch.equal(y1, y2)
    assert np.array_equal(a1.cpu().numpy(), ref["acc"])


def test_zero_token_and_zero_weights():
    M, K, N = 256, 512, 3
    W = inputs.latent_weights(M, K, seed=5)
    x = inputs.activations(N, K, seed=6)
    x[1] = 0
    ref = oracle.bitlinear(W.numpy(), x.numpy())
    packed, alpha = api.pack_weights(W.cuda())
    xq, amax, xsum = api.quant_act(x.cuda())
    for fn in (api.gemv, api.gemm):
        y, acc = fn(packed, alpha, xq, amax, xsum, with_acc=True)
        assert (y[1] == 0).all() and (acc[1] == 0).all()
        assert np.array_equal(acc.cpu().numpy(), ref["acc"])
    zp, za = api.pack_weights(torch.zeros(M, K, device="cuda"))
    for fn in (api.gemv, api.gemm):
        y = fn(zp, za, xq, amax, xsum)
        assert (y == 0).all()


def test_empty_batch_is_noop():
    packed, alpha = api.pack_weights(inputs.latent_weights(128, 128, seed=1).cuda())
    xq = torch.empty(0, 128, dtype=torch.int8, device="cuda")
    amax = torch.empty(0, dtype=torch.float32, device="cuda")
    xsum = torch.empty(0, dtype=torch.int32, device="cuda")
    for fn in (_lib.bitlinear_gemv, _lib.bitlinear_gemm):
        y = torch.empty(1, 128, device="cuda")
        # empty tensors may carry a NULL data pointer: N == 0 returns before any check
        st = fn(packed, alpha, 128, 128, xq, amax, xsum, 0, y)
        assert st == _lib.OK


def test_rejects_bad_shapes_on_device():
    ref, (packed, alpha, xq, amax, xsum) = _layer(256, 256, 17, seed=9)
    y = torch.empty(17, 256, device="cuda")
    assert _lib.bitlinear_gemv(packed, alpha, 256, 256, xq, amax, xsum, 17, y) == \
        _lib.ERR_UNSUPPORTED_SHAPE
    assert _lib.bitlinear_gemm(packed, alpha, 256, 200, xq, amax, xsum, 17, y) == \
        _lib.ERR_UNSUPPORTED_SHAPE

"""The bounded-wait path of the tensor-core GEMMs, exercised without a fault.

Every mbarrier wait in the pipelined kernels gives up after a wall-time
limit (bitlinear_set_wait_limit; 2 s by default).  Here the limit is set far
below the length of one tile's main loop (K = 131072 is 1024 k-blocks), so
the epilogue's wait for the accumulator runs out: the kernel must wind down
-- stop issuing, drain the copies and MMAs it has in flight, release tensor
memory -- and return, the device error word must read
BITLINEAR_ERR_DEVICE_TIMEOUT, and the same call with the default limit must
then give the oracle's results on the same context.  Nothing here traps,
faults or waits without a bound.
"""
import numpy as np
import pytest
import torch

import oracle
from ternary_weight_bit_bitlinear_b200 import _lib, api, build, inputs

pytestmark = pytest.mark.gpu

SHORT_NS = 2000   # 2 us: far below a 1024-k-block main loop


@pytest.fixture(scope="module", autouse=True)
def _gpu():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    build.build()
    _lib.load()
    yield
    _lib.bitlinear_set_wait_limit(0)


def _case(M, K, N, seed):
    W = inputs.latent_weights(M, K, seed=seed, device="cuda")
    packed, alpha = api.pack_weights(W)
    x = inputs.activations(N, K, seed=seed + 1, device="cuda")
    xq, amax, xsum = api.quant_act(x)
    torch.cuda.synchronize()
    return W, packed, alpha, x, xq, amax, xsum


# N = 32: A in tensor memory (gemm_small); N = 128: one CTA per 128-row tile,
# A unpacked into shared memory; N = 256: CTA pairs.
@pytest.mark.parametrize("M,N", [(128, 32), (128, 128), (256, 256)])
def test_short_limit_times_out_then_recovers(M, N):
    K = 131072
    W, packed, alpha, x, xq, amax, xsum = _case(M, K, N, seed=9100 + N)
    assert _lib.bitlinear_device_error(clear=True) == _lib.OK
    old = _lib.bitlinear_set_wait_limit(SHORT_NS)
    try:
        api.gemm(packed, alpha, xq, amax, xsum)
        torch.cuda.synchronize()          # the kernel wound down and returned
    finally:
        _lib.bitlinear_set_wait_limit(old)
    assert _lib.bitlinear_device_error(clear=True) == _lib.ERR_DEVICE_TIMEOUT
    assert _lib.bitlinear_device_error(clear=True) == _lib.OK

    # same context, default limit: the full result again, checked on sampled
    # rows against the oracle (the whole product is too slow on the CPU)
    y, acc = api.gemm(packed, alpha, xq, amax, xsum, with_acc=True)
    torch.cuda.synchronize()
    assert _lib.bitlinear_device_error(clear=True) == _lib.OK
    Wn = W.cpu().numpy()
    a_ref = oracle.absmean(Wn)
    assert alpha.item() == a_ref
    rows = np.array([0, 1, M // 2, M - 1])
    codes = oracle.ternarize(Wn[rows], a_ref)
    q, am, _ = oracle.quant_act(x.cpu().numpy())
    assert np.array_equal(xq.cpu().numpy(), q)
    acc_ref = oracle.matmul_i32(codes, q)                  # [N, rows]
    y_ref = oracle.rescale(acc_ref, a_ref, am)
    assert np.array_equal(acc.cpu().numpy()[:, rows], acc_ref)
    assert np.array_equal(y.cpu().numpy()[:, rows], y_ref)

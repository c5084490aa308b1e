"""bitlinear_pack_weights_noalloc: packing for callers that cannot allocate
device memory (a plugin whose host owns the whole device memory budget, or a
latency-critical path where cudaMalloc's implicit synchronisation is not
allowed).  Its scratch is a fixed array inside the library, so the checks here
are that it gives exactly what the workspace entry point gives, call after
call, and that it rejects bad arguments before touching the GPU.

The file is named so that pytest collects it last.
"""
import ctypes

import numpy as np
import pytest
import torch

from ternary_weight_bit_bitlinear_b200 import _lib, api, build, inputs

FAKE = 0x10000


@pytest.fixture(scope="module")
def L():
    build.build()
    return _lib.load()


def test_noalloc_rejects_bad_arguments_on_host(L):
    f = L.bitlinear_pack_weights_noalloc
    p = ctypes.c_void_p
    assert f(p(0), 128, 128, p(FAKE), p(FAKE), None) == _lib.ERR_INVALID_ARG
    assert f(p(FAKE), 128, 100, p(FAKE), p(FAKE), None) == _lib.ERR_UNSUPPORTED_SHAPE
    assert f(p(FAKE), (1 << 40) // 128 + 1, 128, p(FAKE), p(FAKE), None) == \
        _lib.ERR_UNSUPPORTED_SHAPE
    assert f(p(FAKE + 4), 128, 128, p(FAKE), p(FAKE), None) == _lib.ERR_MISALIGNED


@pytest.mark.gpu
def test_noalloc_matches_workspace_entry_point_twice(L):
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    # two different tensors back to back: the shared scratch must be cleared
    # by each call, so the second result depends on the second tensor only
    for seed, (M, K) in ((7001, (640, 2560)), (7002, (2560, 6912))):
        W = inputs.latent_weights(M, K, seed=seed, device="cuda")
        ref_packed, ref_alpha = api.pack_weights(W)
        packed = torch.empty((M, api.packed_row_words(K)), dtype=torch.int32, device="cuda")
        alpha = torch.empty(1, dtype=torch.float32, device="cuda")
        _lib.check(_lib.bitlinear_pack_weights_noalloc(W, M, K, packed, alpha),
                   "bitlinear_pack_weights_noalloc")
        torch.cuda.synchronize()
        assert alpha.item() == ref_alpha.item()
        assert torch.equal(packed, ref_packed)
        assert np.isfinite(alpha.item()) and alpha.item() > 0
    assert _lib.bitlinear_device_error(clear=True) == _lib.OK

"""Host-side operand checks of the torch binding (api.py), on the CPU.

A wrong-sized output or token vector, or an operand on another device, must
raise before any pointer reaches the C ABI: the kernels write N*M floats
through `out` and read N entries of amax and xsum, and dereference every
pointer on the weights' device.
"""
import pytest
import torch

from ternary_weight_bit_bitlinear_b200 import api


def test_out_of_the_wrong_shape_is_rejected():
    with pytest.raises(ValueError, match="shape"):
        api._check_out(torch.empty(3, 4), 2, 4, torch.device("cpu"))
    with pytest.raises(ValueError, match="shape"):
        api._check_out(torch.empty(8), 2, 4, torch.device("cpu"))
    with pytest.raises(ValueError, match="shape"):
        api._check_out([[0.0] * 4] * 2, 2, 4, torch.device("cpu"))
    api._check_out(None, 2, 4, torch.device("cpu"))       # no out: nothing to check


def test_out_must_be_a_cuda_float32_tensor():
    with pytest.raises(ValueError, match="CUDA"):
        api._check_out(torch.empty(2, 4), 2, 4, torch.device("cpu"))


def test_token_vectors_must_hold_n_entries():
    with pytest.raises(ValueError):   # CPU tensors fail the device rule first
        api._check_token_vector(torch.empty(3), 3, torch.float32, "amax")


def test_operands_must_share_the_weights_device():
    with pytest.raises(ValueError, match="one device"):
        api._on(torch.device("cuda", 0), amax=torch.empty(2))
    api._on(torch.device("cpu"), amax=torch.empty(2), xsum=None)


def test_matmul_rejects_cpu_operands_before_any_call():
    t = torch.empty(4, 4, dtype=torch.int32)
    with pytest.raises(ValueError, match="CUDA"):
        api.gemv(t, torch.empty(1), torch.empty(1, 64, dtype=torch.int8), torch.empty(1),
                 torch.empty(1, dtype=torch.int32))

"""Ternary BitLinear (BitNet b1.58, I2_S-style) mpGEMM for B200 (sm_100a).

    from ternary_weight_bit_bitlinear_b200 import api
    packed, alpha = api.pack_weights(W)          # offline, W fp32 [M,K] on cuda
    xq, amax, xsum = api.quant_act(x)            # per step, x fp32 [N,K]
    y = api.matmul(packed, alpha, xq, amax, xsum)

The C ABI is include/bitlinear.h; `_lib` is its ctypes view.  Importing this
package loads nothing; the shared library is opened on first use and a missing
build raises instead of falling back to any CPU code.
"""
__all__ = ["api", "inputs"]

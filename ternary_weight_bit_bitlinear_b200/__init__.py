"""Ternary BitLinear (BitNet b1.58, I2_S-style) mpGEMM for B200 (sm_100a)."""

"""Python view of the C oracle for the ternary BitLinear mpGEMM.

TEST INFRASTRUCTURE ONLY.  Only the tests, ``__graft_entry__.smoke()`` and the
benchmark's CPU-baseline leg may import this package.  It shares no code with
the CUDA library and never imports it.

Every function takes and returns numpy arrays and calls the plain C routines in
``bitlinear_oracle.c`` (see that file's header for what each step computes and
the passages of the pages it follows).
"""
import ctypes
import os

import numpy as np

from . import build as _build

_lib = None


def lib():
    """Load (building first if needed) liboracle.so."""
    global _lib
    if _lib is None:
        path = _build.build()
        L = ctypes.CDLL(path)
        i64, p = ctypes.c_int64, ctypes.c_void_p
        L.oracle_abs_bins.argtypes = [p, i64, p]
        L.oracle_abs_bins.restype = ctypes.c_int
        L.oracle_alpha_from_bins.argtypes = [p, i64]
        L.oracle_alpha_from_bins.restype = ctypes.c_float
        L.oracle_absmean.argtypes = [p, i64, p]
        L.oracle_absmean.restype = ctypes.c_float
        L.oracle_ternarize.argtypes = [p, i64, ctypes.c_float, p]
        L.oracle_ternarize.restype = None
        L.oracle_tl2_row_bytes.argtypes = [i64]
        L.oracle_tl2_row_bytes.restype = i64
        L.oracle_tl2_encode.argtypes = [p, i64, i64, p]
        L.oracle_tl2_encode.restype = ctypes.c_int
        L.oracle_tl2_decode.argtypes = [p, i64, i64, p]
        L.oracle_tl2_decode.restype = ctypes.c_int
        L.oracle_packed_row_words.argtypes = [i64]
        L.oracle_packed_row_words.restype = i64
        L.oracle_pack.argtypes = [p, i64, i64, p]
        L.oracle_pack.restype = ctypes.c_int
        L.oracle_unpack.argtypes = [p, i64, i64, p]
        L.oracle_unpack.restype = ctypes.c_int
        L.oracle_quant_act.argtypes = [p, i64, i64, p, p, p]
        L.oracle_quant_act.restype = None
        L.oracle_quant_act_per_tensor.argtypes = [p, i64, i64, p, p, p]
        L.oracle_quant_act_per_tensor.restype = None
        L.oracle_matmul_i32.argtypes = [p, i64, i64, p, i64, p]
        L.oracle_matmul_i32.restype = None
        L.oracle_matmul_addsub.argtypes = [p, i64, i64, p, i64, p]
        L.oracle_matmul_addsub.restype = None
        L.oracle_rescale.argtypes = [p, i64, i64, ctypes.c_float, p, p]
        L.oracle_rescale.restype = None
        _lib = L
    return _lib


def _c(a, dtype):
    a = np.ascontiguousarray(a, dtype=dtype)
    return a, a.ctypes.data


def abs_bins(w):
    """Exponent-binned exact sum of |w| (uint64[256]) and a status (0 / -1)."""
    w, pw = _c(w, np.float32)
    bins = np.zeros(256, dtype=np.uint64)
    st = lib().oracle_abs_bins(pw, w.size, bins.ctypes.data)
    return bins, st


def alpha_from_bins(bins, count):
    bins, pb = _c(bins, np.uint64)
    return np.float32(lib().oracle_alpha_from_bins(pb, int(count)))


def absmean(w):
    """alpha = mean|w| rounded once to fp32; raises on non-finite input."""
    w, pw = _c(w, np.float32)
    st = ctypes.c_int(0)
    a = lib().oracle_absmean(pw, w.size, ctypes.byref(st))
    if st.value != 0:
        raise ValueError("non-finite weight")
    return np.float32(a)


def ternarize(w, alpha):
    w, pw = _c(w, np.float32)
    codes = np.empty(w.shape, dtype=np.int8)
    lib().oracle_ternarize(pw, w.size, ctypes.c_float(float(alpha)), codes.ctypes.data)
    return codes


def packed_row_words(K):
    """Words per packed row: 4*ceil(K/64) (K/16 when K is a multiple of 64)."""
    return int(lib().oracle_packed_row_words(int(K)))


def pack(codes):
    """codes int8 [M,K] -> uint32 [M, packed_row_words(K)]."""
    codes, pc = _c(codes, np.int8)
    M, K = codes.shape
    out = np.empty((M, packed_row_words(K)), dtype=np.uint32)
    if lib().oracle_pack(pc, M, K, out.ctypes.data) != 0:
        raise ValueError("bad code or K % 16 != 0")
    return out


def unpack(packed, M, K):
    packed, pp = _c(packed, np.uint32)
    out = np.empty((M, K), dtype=np.int8)
    if lib().oracle_unpack(pp, M, K, out.ctypes.data) != 0:
        raise ValueError("invalid 2-bit field (3) or bad K")
    return out


def tl2_row_bytes(K):
    """Bytes of one TL2-style row (index plane, sign plane, 2-bit remainder)."""
    return int(lib().oracle_tl2_row_bytes(int(K)))


def tl2_encode(codes):
    """codes int8 [M,K] -> uint8 [M, tl2_row_bytes(K)] (5 bits per 3 weights)."""
    codes, pc = _c(codes, np.int8)
    M, K = codes.shape
    out = np.empty((M, tl2_row_bytes(K)), dtype=np.uint8)
    if lib().oracle_tl2_encode(pc, M, K, out.ctypes.data) != 0:
        raise ValueError("bad code or K % 16 != 0")
    return out


def tl2_decode(data, M, K):
    data, pd = _c(data, np.uint8)
    out = np.empty((M, K), dtype=np.int8)
    if lib().oracle_tl2_decode(pd, M, K, out.ctypes.data) != 0:
        raise ValueError("invalid TL2 row")
    return out


def quant_act(x):
    """x fp32 [N,K] -> (q int8 [N,K], amax fp32 [N], qsum int32 [N])."""
    x, px = _c(x, np.float32)
    N, K = x.shape
    q = np.empty((N, K), dtype=np.int8)
    amax = np.empty(N, dtype=np.float32)
    qsum = np.empty(N, dtype=np.int32)
    lib().oracle_quant_act(px, N, K, q.ctypes.data, amax.ctypes.data, qsum.ctypes.data)
    return q, amax, qsum


def quant_act_per_tensor(x):
    """x fp32 [N,K] -> (q, amax [N] all equal to max|x|, qsum [N])."""
    x, px = _c(x, np.float32)
    N, K = x.shape
    q = np.empty((N, K), dtype=np.int8)
    amax = np.empty(N, dtype=np.float32)
    qsum = np.empty(N, dtype=np.int32)
    lib().oracle_quant_act_per_tensor(px, N, K, q.ctypes.data, amax.ctypes.data,
                                      qsum.ctypes.data)
    return q, amax, qsum


def matmul_i32(codes, q):
    """codes int8 [M,K], q int8 [N,K] -> acc int32 [N,M] (triple loop)."""
    codes, pc = _c(codes, np.int8)
    q, pq = _c(q, np.int8)
    M, K = codes.shape
    N = q.shape[0]
    acc = np.empty((N, M), dtype=np.int32)
    lib().oracle_matmul_i32(pc, M, K, pq, N, acc.ctypes.data)
    return acc


def matmul_addsub(codes, q):
    """Same product, additions and subtractions only."""
    codes, pc = _c(codes, np.int8)
    q, pq = _c(q, np.int8)
    M, K = codes.shape
    N = q.shape[0]
    acc = np.empty((N, M), dtype=np.int32)
    lib().oracle_matmul_addsub(pc, M, K, pq, N, acc.ctypes.data)
    return acc


def rescale(acc, alpha, amax):
    acc, pa = _c(acc, np.int32)
    amax, pm = _c(amax, np.float32)
    N, M = acc.shape
    y = np.empty((N, M), dtype=np.float32)
    lib().oracle_rescale(pa, N, M, ctypes.c_float(float(alpha)), pm, y.ctypes.data)
    return y


def bitlinear(W, x):
    """Whole layer from latent fp32 weights W [M,K] and activations x [N,K].

    Returns a dict with alpha, codes, packed, q, amax, qsum, acc, y.
    """
    alpha = absmean(W)
    codes = ternarize(W, alpha)
    packed = pack(codes)
    q, amax, qsum = quant_act(x)
    acc = matmul_i32(codes, q)
    y = rescale(acc, alpha, amax)
    return dict(alpha=alpha, codes=codes, packed=packed, q=q, amax=amax, qsum=qsum,
                acc=acc, y=y)


def sampled_outputs(W_rows, alpha, x_rows):
    """y for a subset of weight rows: the full-tensor alpha is given, W_rows
    holds only the sampled rows [R,K], x_rows the sampled tokens [T,K].
    Returns (acc [T,R], y [T,R])."""
    W = W_rows
    codes = ternarize(W, alpha)
    q, amax, _ = quant_act(x_rows)
    acc = matmul_i32(codes, q)
    return acc, rescale(acc, alpha, amax)

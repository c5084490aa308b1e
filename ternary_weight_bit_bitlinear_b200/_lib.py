"""ctypes view of libbitlinear.so: one Python function per C entry point.

Argument marshalling only -- every step of the path runs in the CUDA kernels
behind include/bitlinear.h.  There is no CPU fallback: if the shared library
is missing or a call fails, an exception is raised.
"""
import ctypes
import os
import re

PKG = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(PKG, "libbitlinear.so")
HEADER = os.path.join(os.path.dirname(PKG), "include", "bitlinear.h")

OK = 0
ERR_INVALID_ARG = 1
ERR_UNSUPPORTED_SHAPE = 2
ERR_MISALIGNED = 3
ERR_WORKSPACE = 4
ERR_CUDA = 5
ERR_DEVICE_TIMEOUT = 6
ERR_NONFINITE = 7


class Problem(ctypes.Structure):
    """Mirror of bitlinear_problem (include/bitlinear.h)."""
    _fields_ = [("packed", ctypes.c_void_p), ("alpha", ctypes.c_void_p), ("M", ctypes.c_int64),
                ("K", ctypes.c_int64), ("xq", ctypes.c_void_p), ("amax", ctypes.c_void_p), ("xsum", ctypes.c_void_p),
                ("y", ctypes.c_void_p), ("acc", ctypes.c_void_p)]


class Act(ctypes.Structure):
    """Mirror of bitlinear_act (include/bitlinear.h)."""
    _fields_ = [("x", ctypes.c_void_p), ("N", ctypes.c_int64), ("K", ctypes.c_int64),
                ("xq", ctypes.c_void_p), ("amax", ctypes.c_void_p), ("xsum", ctypes.c_void_p)]


class FusedProblem(ctypes.Structure):
    """Mirror of bitlinear_fused_problem (include/bitlinear.h)."""
    _fields_ = [("packed", ctypes.c_void_p), ("alpha", ctypes.c_void_p), ("M", ctypes.c_int64),
                ("K", ctypes.c_int64), ("x", ctypes.c_void_p), ("y", ctypes.c_void_p),
                ("acc", ctypes.c_void_p)]


class Tl2Problem(ctypes.Structure):
    """Mirror of bitlinear_tl2_problem (include/bitlinear.h)."""
    _fields_ = [("tl2", ctypes.c_void_p), ("alpha", ctypes.c_void_p), ("M", ctypes.c_int64),
                ("K", ctypes.c_int64), ("xq", ctypes.c_void_p), ("amax", ctypes.c_void_p),
                ("y", ctypes.c_void_p), ("acc", ctypes.c_void_p)]


class BitLinearError(RuntimeError):
    def __init__(self, status, where):
        self.status = status
        super().__init__("%s failed: %s (status %d)" % (where, status_string(status), status))


_lib = None


def load(path: str = LIB_PATH):
    """Load the shared library (once).  Raises if it has not been built."""
    global _lib
    if _lib is not None:
        return _lib
    if not os.path.exists(path):
        raise ImportError("libbitlinear.so not built at %s; run "
                          "`python -m ternary_weight_bit_bitlinear_b200.build`" % path)
    L = ctypes.CDLL(path)
    i64, p, st, sz = ctypes.c_int64, ctypes.c_void_p, ctypes.c_int, ctypes.c_size_t
    L.bitlinear_status_string.argtypes = [ctypes.c_int]
    L.bitlinear_status_string.restype = ctypes.c_char_p
    L.bitlinear_version.argtypes = []
    L.bitlinear_version.restype = ctypes.c_int
    L.bitlinear_pack_workspace_bytes.argtypes = [i64, i64]
    L.bitlinear_pack_workspace_bytes.restype = sz
    L.bitlinear_pack_weights.argtypes = [p, i64, i64, p, p, p, sz, p]
    L.bitlinear_pack_weights.restype = st
    L.bitlinear_pack_weights_noalloc.argtypes = [p, i64, i64, p, p, p]
    L.bitlinear_pack_weights_noalloc.restype = st
    L.bitlinear_quant_act_per_tensor_workspace_bytes.argtypes = []
    L.bitlinear_quant_act_per_tensor_workspace_bytes.restype = sz
    L.bitlinear_quant_act_per_tensor.argtypes = [p, i64, i64, p, p, p, p, sz, p]
    L.bitlinear_quant_act_per_tensor.restype = st
    L.bitlinear_quant_act_grouped.argtypes = [ctypes.POINTER(Act), i64, p]
    L.bitlinear_quant_act_grouped.restype = st
    L.bitlinear_quant_act.argtypes = [p, i64, i64, p, p, p, p]
    L.bitlinear_quant_act.restype = st
    for name in ("bitlinear_gemv", "bitlinear_gemm"):
        f = getattr(L, name)
        f.argtypes = [p, p, i64, i64, p, p, p, i64, p, p, p]
        f.restype = st
    for name in ("bitlinear_gemv_grouped", "bitlinear_gemm_grouped"):
        f = getattr(L, name)
        f.argtypes = [ctypes.POINTER(Problem), i64, i64, p]
        f.restype = st
    L.bitlinear_gemv_quant.argtypes = [p, p, i64, i64, p, i64, p, p, p]
    L.bitlinear_gemv_quant.restype = st
    L.bitlinear_gemv_quant_grouped.argtypes = [ctypes.POINTER(FusedProblem), i64, i64, p]
    L.bitlinear_gemv_quant_grouped.restype = st
    L.bitlinear_tl2_row_bytes.argtypes = [i64]
    L.bitlinear_tl2_row_bytes.restype = sz
    L.bitlinear_tl2_from_packed.argtypes = [p, i64, i64, p, p]
    L.bitlinear_tl2_from_packed.restype = st
    L.bitlinear_gemv_tl2.argtypes = [p, p, i64, i64, p, p, i64, p, p, p]
    L.bitlinear_gemv_tl2.restype = st
    L.bitlinear_gemv_tl2_grouped.argtypes = [ctypes.POINTER(Tl2Problem), i64, i64, p]
    L.bitlinear_gemv_tl2_grouped.restype = st
    L.bitlinear_device_error.argtypes = [ctypes.POINTER(ctypes.c_int), ctypes.c_int]
    L.bitlinear_device_error.restype = st
    L.bitlinear_set_wait_limit.argtypes = [ctypes.c_ulonglong]
    L.bitlinear_set_wait_limit.restype = ctypes.c_ulonglong
    _lib = L
    return L


def header_symbols(header: str = HEADER):
    """Names of the functions include/bitlinear.h declares."""
    text = open(header).read()
    return sorted(set(re.findall(r"BITLINEAR_API\s+[\w\s\*]+?\b(bitlinear_\w+)\s*\(", text)))


def status_string(status: int) -> str:
    return load().bitlinear_status_string(int(status)).decode()


def check(status: int, where: str):
    if status != OK:
        raise BitLinearError(status, where)


def _p(t):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _stream(stream):
    if stream is None:
        import torch
        stream = torch.cuda.current_stream()
    return ctypes.c_void_p(stream.cuda_stream if hasattr(stream, "cuda_stream") else int(stream))


# --------------------------------------------------------------- raw entry points
# Each takes torch tensors (already allocated, on the current CUDA device) and
# returns the C status code unchanged.

def bitlinear_pack_weights(W, M, K, packed, alpha, workspace, workspace_bytes, stream=None):
    return load().bitlinear_pack_weights(_p(W), M, K, _p(packed), _p(alpha), _p(workspace),
                                         workspace_bytes, _stream(stream))


def bitlinear_pack_weights_noalloc(W, M, K, packed, alpha, stream=None):
    return load().bitlinear_pack_weights_noalloc(_p(W), M, K, _p(packed), _p(alpha),
                                                 _stream(stream))


def bitlinear_quant_act(x, N, K, xq, amax, xsum, stream=None):
    return load().bitlinear_quant_act(_p(x), N, K, _p(xq), _p(amax), _p(xsum), _stream(stream))


def bitlinear_quant_act_per_tensor(x, N, K, xq, amax, xsum, workspace, workspace_bytes,
                                   stream=None):
    return load().bitlinear_quant_act_per_tensor(_p(x), N, K, _p(xq), _p(amax), _p(xsum),
                                                 _p(workspace), workspace_bytes,
                                                 _stream(stream))


def make_acts(entries):
    """entries: iterable of (x, xq, amax, xsum-or-None) tensors.  Returns a
    ctypes array of Act."""
    entries = list(entries)
    arr = (Act * max(1, len(entries)))()
    for i, (x, xq, amax, xsum) in enumerate(entries):
        arr[i] = Act(x.data_ptr(), x.shape[0], x.shape[1], xq.data_ptr(), amax.data_ptr(),
                     0 if xsum is None else xsum.data_ptr())
    return arr


def bitlinear_quant_act_grouped(acts, count, stream=None):
    """acts: a ctypes array from make_acts()."""
    return load().bitlinear_quant_act_grouped(acts, count, _stream(stream))


def bitlinear_gemv(packed, alpha, M, K, xq, amax, xsum, N, y, acc=None, stream=None):
    return load().bitlinear_gemv(_p(packed), _p(alpha), M, K, _p(xq), _p(amax), _p(xsum), N,
                                 _p(y), _p(acc), _stream(stream))


def bitlinear_gemm(packed, alpha, M, K, xq, amax, xsum, N, y, acc=None, stream=None):
    return load().bitlinear_gemm(_p(packed), _p(alpha), M, K, _p(xq), _p(amax), _p(xsum), N,
                                 _p(y), _p(acc), _stream(stream))


def make_problems(entries):
    """entries: iterable of (packed, alpha, M, K, xq, amax, xsum, y, acc-or-None);
    tensors for the pointers.  Returns a ctypes array of Problem (keep it alive
    while the call runs)."""
    entries = list(entries)
    arr = (Problem * max(1, len(entries)))()
    for i, (packed, alpha, M, K, xq, amax, xsum, y, acc) in enumerate(entries):
        arr[i] = Problem(packed.data_ptr(), alpha.data_ptr(), M, K, xq.data_ptr(),
                         amax.data_ptr(), xsum.data_ptr(), y.data_ptr(),
                         0 if acc is None else acc.data_ptr())
    return arr


def bitlinear_gemv_grouped(problems, count, N, stream=None):
    """problems: a ctypes array from make_problems()."""
    return load().bitlinear_gemv_grouped(problems, count, N, _stream(stream))


def bitlinear_gemm_grouped(problems, count, N, stream=None):
    """problems: a ctypes array from make_problems()."""
    return load().bitlinear_gemm_grouped(problems, count, N, _stream(stream))


def bitlinear_gemv_quant(packed, alpha, M, K, x, N, y, acc=None, stream=None):
    return load().bitlinear_gemv_quant(_p(packed), _p(alpha), M, K, _p(x), N, _p(y), _p(acc),
                                       _stream(stream))


def make_fused_problems(entries):
    """entries: iterable of (packed, alpha, M, K, x, y, acc-or-None); tensors for
    the pointers.  Returns a ctypes array of FusedProblem (keep it alive while
    the call runs)."""
    entries = list(entries)
    arr = (FusedProblem * max(1, len(entries)))()
    for i, (packed, alpha, M, K, x, y, acc) in enumerate(entries):
        arr[i] = FusedProblem(packed.data_ptr(), alpha.data_ptr(), M, K, x.data_ptr(),
                              y.data_ptr(), 0 if acc is None else acc.data_ptr())
    return arr


def bitlinear_gemv_quant_grouped(problems, count, N, stream=None):
    """problems: a ctypes array from make_fused_problems()."""
    return load().bitlinear_gemv_quant_grouped(problems, count, N, _stream(stream))


def bitlinear_tl2_from_packed(packed, M, K, tl2, stream=None):
    return load().bitlinear_tl2_from_packed(_p(packed), M, K, _p(tl2), _stream(stream))


def bitlinear_gemv_tl2(tl2, alpha, M, K, xq, amax, N, y, acc=None, stream=None):
    return load().bitlinear_gemv_tl2(_p(tl2), _p(alpha), M, K, _p(xq), _p(amax), N, _p(y),
                                     _p(acc), _stream(stream))


def make_tl2_problems(entries):
    """entries: iterable of (tl2, alpha, M, K, xq, amax, y, acc-or-None); tensors
    for the pointers.  Returns a ctypes array of Tl2Problem."""
    entries = list(entries)
    arr = (Tl2Problem * max(1, len(entries)))()
    for i, (tl2, alpha, M, K, xq, amax, y, acc) in enumerate(entries):
        arr[i] = Tl2Problem(tl2.data_ptr(), alpha.data_ptr(), M, K, xq.data_ptr(),
                            amax.data_ptr(), y.data_ptr(), 0 if acc is None else acc.data_ptr())
    return arr


def bitlinear_gemv_tl2_grouped(problems, count, N, stream=None):
    """problems: a ctypes array from make_tl2_problems()."""
    return load().bitlinear_gemv_tl2_grouped(problems, count, N, _stream(stream))


def bitlinear_pack_workspace_bytes(M, K):
    return load().bitlinear_pack_workspace_bytes(M, K)


def bitlinear_set_wait_limit(limit_ns):
    """Set the wall-time limit of the kernels' bounded waits (0: the default);
    returns the previous limit."""
    return load().bitlinear_set_wait_limit(int(limit_ns))


def bitlinear_device_error(clear=True):
    out = ctypes.c_int(0)
    check(load().bitlinear_device_error(ctypes.byref(out), 1 if clear else 0),
          "bitlinear_device_error")
    return out.value

"""Host-side checks of the C ABI that need no GPU.

Every call below fails argument validation before the library touches CUDA,
so these tests are safe with or without a device present.
"""
import ctypes
import os
import subprocess

import pytest

from ternary_weight_bit_bitlinear_b200 import _lib, build

FAKE = 0x10000          # 16-byte aligned, never dereferenced: every case fails validation first
MISALIGNED = 0x10004


@pytest.fixture(scope="module")
def L():
    build.build()
    return _lib.load()


def test_library_exports_every_declared_symbol(L):
    declared = _lib.header_symbols()
    assert len(declared) >= 8
    for name in declared:
        assert hasattr(L, name), name
    out = subprocess.run(["nm", "-D", "--defined-only", _lib.LIB_PATH], capture_output=True,
                         text=True, check=True).stdout
    exported = {line.split()[-1] for line in out.splitlines() if " T " in line}
    assert set(declared) <= exported
    assert {n for n in exported if n.startswith("bitlinear_")} == set(declared)


def test_version_and_status_strings(L):
    assert L.bitlinear_version() == 101
    names = {_lib.status_string(code) for code in range(8)}
    assert len(names) == 8 and "unknown status" not in names
    assert _lib.status_string(0) == "ok"
    assert "non-finite" in _lib.status_string(_lib.ERR_NONFINITE)
    assert _lib.status_string(99) == "unknown status"


def test_wait_limit_setting_is_host_only(L):
    # A process-wide host setting: no CUDA call, so it works without a device.
    default = _lib.bitlinear_set_wait_limit(5000)
    try:
        assert default == 2_000_000_000
        assert _lib.bitlinear_set_wait_limit(7000) == 5000
    finally:
        assert _lib.bitlinear_set_wait_limit(0) == 7000
    assert _lib.bitlinear_set_wait_limit(0) == default   # 0 restored the default


def test_missing_library_raises(tmp_path):
    saved = _lib._lib
    try:
        _lib._lib = None
        with pytest.raises(ImportError):
            _lib.load(str(tmp_path / "nope.so"))
    finally:
        _lib._lib = saved


def _p(v):
    return ctypes.c_void_p(v)


def test_pack_argument_errors(L):
    ws = L.bitlinear_pack_workspace_bytes(128, 128)
    assert ws >= 256 * 8
    f = L.bitlinear_pack_weights
    ok = dict(W=FAKE, M=128, K=128, packed=FAKE, alpha=FAKE, ws=FAKE, wsb=ws)

    def call(**kw):
        a = dict(ok, **kw)
        return f(_p(a["W"]), a["M"], a["K"], _p(a["packed"]), _p(a["alpha"]), _p(a["ws"]),
                 a["wsb"], None)

    assert call(W=0) == _lib.ERR_INVALID_ARG
    assert call(alpha=0) == _lib.ERR_INVALID_ARG
    assert call(M=-1) == _lib.ERR_INVALID_ARG
    assert call(K=100) == _lib.ERR_UNSUPPORTED_SHAPE
    assert call(K=0) == _lib.ERR_UNSUPPORTED_SHAPE
    assert call(K=131072 + 128) == _lib.ERR_UNSUPPORTED_SHAPE
    assert call(M=(1 << 40) // 128 + 1) == _lib.ERR_UNSUPPORTED_SHAPE
    assert call(ws=0) == _lib.ERR_WORKSPACE
    assert call(wsb=ws - 1) == _lib.ERR_WORKSPACE
    assert call(W=MISALIGNED) == _lib.ERR_MISALIGNED
    assert call(packed=MISALIGNED) == _lib.ERR_MISALIGNED


def test_quant_act_argument_errors(L):
    f = L.bitlinear_quant_act
    assert f(_p(FAKE), 1, 100, _p(FAKE), _p(FAKE), None, None) == _lib.ERR_UNSUPPORTED_SHAPE
    assert f(_p(FAKE), -1, 128, _p(FAKE), _p(FAKE), None, None) == _lib.ERR_INVALID_ARG
    assert f(_p(0), 1, 128, _p(FAKE), _p(FAKE), None, None) == _lib.ERR_INVALID_ARG
    assert f(_p(FAKE), 1, 128, _p(MISALIGNED), _p(FAKE), None, None) == _lib.ERR_MISALIGNED
    assert f(_p(FAKE), 0, 128, _p(FAKE), _p(FAKE), None, None) == _lib.OK   # N = 0: no-op


@pytest.mark.parametrize("name", ["bitlinear_gemv", "bitlinear_gemm"])
def test_matmul_argument_errors(L, name):
    f = getattr(L, name)
    ok = dict(packed=FAKE, alpha=FAKE, M=128, K=256, xq=FAKE, amax=FAKE, xsum=FAKE, N=1,
              y=FAKE, acc=0)

    def call(**kw):
        a = dict(ok, **kw)
        return f(_p(a["packed"]), _p(a["alpha"]), a["M"], a["K"], _p(a["xq"]), _p(a["amax"]),
                 _p(a["xsum"]), a["N"], _p(a["y"]), _p(a["acc"]), None)

    assert call(N=0) == _lib.OK
    assert call(N=-1) == _lib.ERR_INVALID_ARG
    assert call(packed=0) == _lib.ERR_INVALID_ARG
    assert call(xsum=0) == _lib.ERR_INVALID_ARG
    assert call(y=0) == _lib.ERR_INVALID_ARG
    assert call(K=200) == _lib.ERR_UNSUPPORTED_SHAPE
    assert call(M=0) == _lib.ERR_UNSUPPORTED_SHAPE
    assert call(y=MISALIGNED) == _lib.ERR_MISALIGNED
    assert call(acc=MISALIGNED) == _lib.ERR_MISALIGNED
    assert call(xq=MISALIGNED) == _lib.ERR_MISALIGNED
    assert call(K=40) == _lib.ERR_UNSUPPORTED_SHAPE      # K must be a multiple of 16
    if name == "bitlinear_gemv":
        assert call(N=17) == _lib.ERR_UNSUPPORTED_SHAPE


def test_header_is_self_contained(tmp_path):
    src = tmp_path / "t.c"
    src.write_text('#include "bitlinear.h"\nint main(void){return BITLINEAR_OK;}\n')
    inc = os.path.join(os.path.dirname(os.path.dirname(os.path.abspath(__file__))), "include")
    subprocess.run(["gcc", "-std=c99", "-Wall", "-Werror", "-I", inc, "-c", str(src), "-o",
                    str(tmp_path / "t.o")], check=True)


@pytest.mark.parametrize("name", ["bitlinear_gemv_grouped", "bitlinear_gemm_grouped"])
def test_grouped_argument_errors(L, name):
    f = getattr(L, name)
    P = _lib.Problem

    def prob(**kw):
        a = dict(packed=FAKE, alpha=FAKE, M=128, K=256, xq=FAKE, amax=FAKE, xsum=FAKE, y=FAKE,
                 acc=0)
        a.update(kw)
        return P(a["packed"], a["alpha"], a["M"], a["K"], a["xq"], a["amax"], a["xsum"], a["y"],
                 a["acc"])

    good = prob()
    arr = (P * 2)(good, good)
    assert f(arr, -1, 1, None) == _lib.ERR_INVALID_ARG
    assert f(None, 2, 1, None) == _lib.ERR_INVALID_ARG
    assert f(arr, 0, 1, None) == _lib.OK
    assert f(arr, 2, 0, None) == _lib.OK
    assert f(arr, 2, -3, None) == _lib.ERR_INVALID_ARG
    assert f((P * 2)(good, prob(K=200)), 2, 1, None) == _lib.ERR_UNSUPPORTED_SHAPE
    assert f((P * 2)(good, prob(y=MISALIGNED)), 2, 1, None) == _lib.ERR_MISALIGNED
    assert f((P * 2)(good, prob(alpha=0)), 2, 1, None) == _lib.ERR_INVALID_ARG
    assert f((P * 2)(good, prob(alpha=FAKE + 2)), 2, 1, None) == _lib.ERR_MISALIGNED
    assert f((P * 2)(good, prob(K=40)), 2, 1, None) == _lib.ERR_UNSUPPORTED_SHAPE
    if name == "bitlinear_gemv_grouped":
        assert f(arr, 2, 17, None) == _lib.ERR_UNSUPPORTED_SHAPE


def test_quant_act_grouped_argument_errors(L):
    f = L.bitlinear_quant_act_grouped
    A = _lib.Act
    good = A(FAKE, 4, 256, FAKE, FAKE, FAKE)
    assert f(None, 1, None) == _lib.ERR_INVALID_ARG
    assert f((A * 1)(good), -1, None) == _lib.ERR_INVALID_ARG
    assert f((A * 1)(good), 0, None) == _lib.OK
    assert f((A * 2)(good, A(FAKE, 4, 100, FAKE, FAKE, FAKE)), 2, None) == \
        _lib.ERR_UNSUPPORTED_SHAPE
    assert f((A * 2)(good, A(FAKE, -1, 256, FAKE, FAKE, FAKE)), 2, None) == _lib.ERR_INVALID_ARG
    assert f((A * 2)(good, A(0, 4, 256, FAKE, FAKE, FAKE)), 2, None) == _lib.ERR_INVALID_ARG
    assert f((A * 2)(good, A(FAKE, 4, 256, MISALIGNED, FAKE, FAKE)), 2, None) == \
        _lib.ERR_MISALIGNED
    assert f((A * 2)(good, A(FAKE, 4, 256, FAKE, FAKE + 1, FAKE)), 2, None) == \
        _lib.ERR_MISALIGNED


def test_quant_act_per_tensor_argument_errors(L):
    f = L.bitlinear_quant_act_per_tensor
    ws = L.bitlinear_quant_act_per_tensor_workspace_bytes()
    assert ws >= 4
    p = _p
    assert f(p(FAKE), 2, 100, p(FAKE), p(FAKE), None, p(FAKE), ws, None) == \
        _lib.ERR_UNSUPPORTED_SHAPE
    assert f(p(FAKE), -2, 128, p(FAKE), p(FAKE), None, p(FAKE), ws, None) == _lib.ERR_INVALID_ARG
    assert f(p(0), 2, 128, p(FAKE), p(FAKE), None, p(FAKE), ws, None) == _lib.ERR_INVALID_ARG
    assert f(p(FAKE), 2, 128, p(FAKE), p(FAKE), None, p(0), ws, None) == _lib.ERR_WORKSPACE
    assert f(p(FAKE), 2, 128, p(FAKE), p(FAKE), None, p(FAKE), 2, None) == _lib.ERR_WORKSPACE
    assert f(p(FAKE), 2, 128, p(FAKE), p(FAKE), None, p(MISALIGNED), ws, None) == \
        _lib.ERR_MISALIGNED
    assert f(p(FAKE), 0, 128, p(FAKE), p(FAKE), None, p(FAKE), ws, None) == _lib.OK


def test_gemv_quant_argument_errors(L):
    f = L.bitlinear_gemv_quant
    ok = dict(packed=FAKE, alpha=FAKE, M=128, K=256, x=FAKE, N=1, y=FAKE, acc=0)

    def call(**kw):
        a = dict(ok, **kw)
        return f(_p(a["packed"]), _p(a["alpha"]), a["M"], a["K"], _p(a["x"]), a["N"],
                 _p(a["y"]), _p(a["acc"]), None)

    assert call(N=0) == _lib.OK
    assert call(N=0, K=200) == _lib.ERR_UNSUPPORTED_SHAPE
    assert call(N=-1) == _lib.ERR_INVALID_ARG
    assert call(N=17) == _lib.ERR_UNSUPPORTED_SHAPE
    assert call(packed=0) == _lib.ERR_INVALID_ARG
    assert call(x=0) == _lib.ERR_INVALID_ARG
    assert call(y=0) == _lib.ERR_INVALID_ARG
    assert call(K=200) == _lib.ERR_UNSUPPORTED_SHAPE
    assert call(M=0) == _lib.ERR_UNSUPPORTED_SHAPE
    assert call(x=MISALIGNED) == _lib.ERR_MISALIGNED
    assert call(y=MISALIGNED) == _lib.ERR_MISALIGNED
    assert call(acc=MISALIGNED) == _lib.ERR_MISALIGNED
    assert call(alpha=FAKE + 2) == _lib.ERR_MISALIGNED
    # the int8 copy of x each warp keeps: N * K rounded up to 512 <= 65536 bytes
    assert call(N=1, K=65536 + 128) == _lib.ERR_UNSUPPORTED_SHAPE
    assert call(N=16, K=4096 + 128) == _lib.ERR_UNSUPPORTED_SHAPE
    assert call(N=2, K=32768 + 128) == _lib.ERR_UNSUPPORTED_SHAPE


def test_gemv_quant_grouped_argument_errors(L):
    f = L.bitlinear_gemv_quant_grouped
    P = _lib.FusedProblem

    def prob(**kw):
        a = dict(packed=FAKE, alpha=FAKE, M=128, K=256, x=FAKE, y=FAKE, acc=0)
        a.update(kw)
        return P(a["packed"], a["alpha"], a["M"], a["K"], a["x"], a["y"], a["acc"])

    good = prob()
    arr = (P * 2)(good, good)
    assert f(arr, -1, 1, None) == _lib.ERR_INVALID_ARG
    assert f(None, 2, 1, None) == _lib.ERR_INVALID_ARG
    assert f(arr, 0, 1, None) == _lib.OK
    assert f(arr, 2, 0, None) == _lib.OK
    assert f(arr, 2, -3, None) == _lib.ERR_INVALID_ARG
    assert f(arr, 2, 17, None) == _lib.ERR_UNSUPPORTED_SHAPE
    assert f((P * 2)(good, prob(K=200)), 2, 1, None) == _lib.ERR_UNSUPPORTED_SHAPE
    assert f((P * 2)(good, prob(K=40960)), 2, 2, None) == _lib.ERR_UNSUPPORTED_SHAPE
    assert f((P * 2)(good, prob(x=MISALIGNED)), 2, 1, None) == _lib.ERR_MISALIGNED
    assert f((P * 2)(good, prob(x=0)), 2, 1, None) == _lib.ERR_INVALID_ARG
    assert f((P * 2)(good, prob(alpha=FAKE + 2)), 2, 1, None) == _lib.ERR_MISALIGNED


def test_tl2_argument_errors(L):
    assert L.bitlinear_tl2_row_bytes(384) == 80
    assert L.bitlinear_tl2_row_bytes(6912) == 1440
    assert L.bitlinear_tl2_row_bytes(40) == 0 and L.bitlinear_tl2_row_bytes(0) == 0
    f = L.bitlinear_tl2_from_packed
    assert f(_p(FAKE), 4, 40, _p(FAKE), None) == _lib.ERR_UNSUPPORTED_SHAPE
    assert f(_p(0), 4, 96, _p(FAKE), None) == _lib.ERR_INVALID_ARG
    assert f(_p(FAKE), 4, 96, _p(MISALIGNED), None) == _lib.ERR_MISALIGNED
    assert f(_p(FAKE), -1, 96, _p(FAKE), None) == _lib.ERR_INVALID_ARG
    g = L.bitlinear_gemv_tl2
    ok = dict(tl2=FAKE, alpha=FAKE, M=64, K=192, xq=FAKE, amax=FAKE, N=1, y=FAKE, acc=0)

    def call(**kw):
        a = dict(ok, **kw)
        return g(_p(a["tl2"]), _p(a["alpha"]), a["M"], a["K"], _p(a["xq"]), _p(a["amax"]),
                 a["N"], _p(a["y"]), _p(a["acc"]), None)

    assert call(N=0) == _lib.OK
    assert call(N=17) == _lib.ERR_UNSUPPORTED_SHAPE
    assert call(N=-1) == _lib.ERR_INVALID_ARG
    assert call(K=40) == _lib.ERR_UNSUPPORTED_SHAPE
    assert call(tl2=0) == _lib.ERR_INVALID_ARG
    assert call(amax=0) == _lib.ERR_INVALID_ARG
    assert call(tl2=MISALIGNED) == _lib.ERR_MISALIGNED
    assert call(amax=FAKE + 2) == _lib.ERR_MISALIGNED
    P = _lib.Tl2Problem
    good = P(FAKE, FAKE, 64, 192, FAKE, FAKE, FAKE, 0)
    G = L.bitlinear_gemv_tl2_grouped
    assert G((P * 1)(good), 0, 1, None) == _lib.OK
    assert G((P * 1)(good), 1, 17, None) == _lib.ERR_UNSUPPORTED_SHAPE
    assert G(None, 1, 1, None) == _lib.ERR_INVALID_ARG
    assert G((P * 2)(good, P(FAKE, FAKE, 64, 40, FAKE, FAKE, FAKE, 0)), 2, 1, None) == \
        _lib.ERR_UNSUPPORTED_SHAPE

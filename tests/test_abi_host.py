"""Host-side checks of the C ABI that need no GPU: the library loads, exports
every symbol the header declares, and rejects bad arguments before launching
anything."""
import ctypes
import os
import re

import pytest

import compressed_history_attention_b200 as nk
from compressed_history_attention_b200 import _lib

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _header_functions():
    names = set()
    for fn in os.listdir(os.path.join(ROOT, "include")):
        if fn.endswith(".h"):
            src = open(os.path.join(ROOT, "include", fn)).read()
            src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
            names |= set(re.findall(r"\b(nanokv_\w+)\s*\(", src))
    return names


def test_library_exports_every_declared_symbol():
    L = nk.lib()
    declared = _header_functions()
    assert declared >= set(_lib.SYMBOLS)
    for name in sorted(declared):
        assert hasattr(L, name), name


def test_version():
    assert "sm_100a" in nk.nanokv_version()


def _codec(**kw):
    c = dict(H=2, d=16, r=8, C=8, param_dtype=_lib.F32, scale_dtype=_lib.F32,
             centers=4096, D=8192, E=12288, aux=None)
    c.update(kw)
    return _lib._Codec(**c)


BAD_CODECS = [
    (dict(r=7), _lib.ERR_INVALID),
    (dict(r=0), _lib.ERR_INVALID),
    (dict(r=514), _lib.ERR_INVALID),
    (dict(C=0), _lib.ERR_INVALID),
    (dict(C=257), _lib.ERR_INVALID),
    (dict(H=0), _lib.ERR_INVALID),
    (dict(d=24), _lib.ERR_UNSUPPORTED),
    (dict(param_dtype=_lib.BF16, scale_dtype=_lib.F32), _lib.ERR_UNSUPPORTED),
    (dict(centers=0), _lib.ERR_INVALID),
    (dict(D=4100), _lib.ERR_INVALID),        # misaligned
    (dict(aux=4104), _lib.ERR_INVALID),      # misaligned aux
]


@pytest.mark.parametrize("kw,status", BAD_CODECS)
def test_encode_rejects_bad_codec(kw, status):
    L = nk.lib()
    c = _codec(**kw)
    p = ctypes.c_void_p(1 << 20)
    st = L.nanokv_encode(ctypes.byref(c), None, p, None, _lib.F32, 10, p, p, p, None, None, None, None)
    assert st == status
    assert L.nanokv_last_error().decode()


@pytest.mark.parametrize("kw,status", BAD_CODECS)
def test_attend_rejects_bad_codec(kw, status):
    L = nk.lib()
    c, good = _codec(**kw), _codec()
    p = ctypes.c_void_p(1 << 20)
    h = _lib._Hist(1 << 20, 1 << 20, 1 << 20)
    st = L.nanokv_attend(p, _lib.F32, 4, ctypes.byref(good), ctypes.byref(c), ctypes.byref(h),
                         ctypes.byref(h), 8, 8, None, None, 0, ctypes.c_float(0.25), p, None, p,
                         1 << 20, None)
    assert st == status


def test_attend_rejects_bad_sizes_and_pointers():
    L = nk.lib()
    c = _codec()
    p = ctypes.c_void_p(1 << 20)
    h = _lib._Hist(1 << 20, 1 << 20, 1 << 20)
    hn = _lib._Hist(0, 1 << 20, 1 << 20)
    call = lambda **kw: L.nanokv_attend(  # noqa: E731
        kw.get("q", p), kw.get("dt", _lib.F32), kw.get("Tq", 4), ctypes.byref(c), ctypes.byref(kw.get("cv", c)),
        ctypes.byref(kw.get("hk", h)), ctypes.byref(h), kw.get("T", 8), kw.get("T_full", 8),
        kw.get("kc", None), None, kw.get("T_cur", 0), ctypes.c_float(kw.get("tau", 0.25)), kw.get("out", p),
        None, kw.get("ws", p), kw.get("wsb", 1 << 20), None)
    assert call(T_full=9) == _lib.ERR_INVALID          # T_full > T
    assert call(T=-1) == _lib.ERR_INVALID
    assert call(Tq=-3) == _lib.ERR_INVALID
    assert call(tau=float("nan")) == _lib.ERR_INVALID
    assert call(tau=-1.0) == _lib.ERR_INVALID
    assert call(hk=hn) == _lib.ERR_INVALID              # NULL ids with T > 0
    assert call(T_cur=4) == _lib.ERR_INVALID            # NULL k_cur with T_cur > 0
    assert call(q=ctypes.c_void_p((1 << 20) + 2)) == _lib.ERR_INVALID   # misaligned
    assert call(dt=_lib.BF16) == _lib.ERR_UNSUPPORTED   # io dtype != params
    assert call(wsb=16) == _lib.ERR_INVALID             # workspace too small
    assert call(cv=_codec(H=3)) == _lib.ERR_INVALID     # K/V codecs disagree on H
    assert call(Tq=0) == _lib.OK                         # nothing to do, nothing launched


def test_workspace_size_is_deterministic_and_grows():
    L = nk.lib()
    c = _codec()
    f = lambda Tq, T, Tf, Tc: L.nanokv_attend_workspace(Tq, ctypes.byref(c), ctypes.byref(c), T, Tf, Tc)  # noqa: E731
    assert f(0, 0, 0, 0) == 0
    assert f(64, 256, 256, 64) > 0
    assert f(64, 256, 0, 64) > f(64, 256, 256, 64)      # low-dim branch adds prep buffers
    assert f(64, 256, 300, 64) == 0                      # invalid -> 0


def test_merge_rejects_bad_arguments():
    L = nk.lib()
    arr = (ctypes.c_void_p * 1)(1 << 20)
    p = ctypes.c_void_p(1 << 20)
    assert L.nanokv_lse_merge(0, arr, arr, 4, 2, 16, p, _lib.F32, None, None) == _lib.ERR_INVALID
    assert L.nanokv_lse_merge(9, arr, arr, 4, 2, 16, p, _lib.F32, None, None) == _lib.ERR_INVALID
    assert L.nanokv_lse_merge(1, arr, arr, 4, 2, 18, p, _lib.F32, None, None) == _lib.ERR_INVALID
    assert L.nanokv_lse_merge(1, arr, arr, 4, 2, 16, p, _lib.F16, None, None) == _lib.ERR_UNSUPPORTED


def test_kernel_path_switch():
    prev = nk.nanokv_set_kernel_path(1)
    assert nk.nanokv_set_kernel_path(prev) == 1
    assert nk.lib().nanokv_set_kernel_path(7) == -1


def test_encode_zero_tokens_is_noop():
    L = nk.lib()
    c = _codec()
    assert L.nanokv_encode(ctypes.byref(c), None, None, None, _lib.F32, 0, None, None, None,
                           None, None, None, None) == _lib.OK


def test_codec_prepare_validation():
    L = nk.lib()
    c = _codec()
    assert L.nanokv_codec_aux_bytes(ctypes.byref(c)) >= (8 * 8 + 8) * 4
    assert L.nanokv_codec_aux_bytes(ctypes.byref(_codec(r=7))) == 0
    assert L.nanokv_codec_prepare(ctypes.byref(c), None, None) == _lib.ERR_INVALID
    assert L.nanokv_codec_prepare(ctypes.byref(c), ctypes.c_void_p((1 << 20) + 4), None) == _lib.ERR_INVALID
    assert L.nanokv_codec_prepare(ctypes.byref(_codec(E=0)), ctypes.c_void_p(1 << 20), None) == _lib.ERR_INVALID


def test_attend_full_tokens_routing():
    """History tokens attended on the full-dim path: the caller's T_full, or
    all T tokens when the codec has a full-dim but no low-dim tensor-core
    kernel (the two forms give the same result); the CUDA-core path keeps
    the caller's split."""
    L = nk.lib()
    bf = dict(d=128, param_dtype=_lib.BF16, scale_dtype=_lib.F16)
    small = _codec(H=12, r=192, C=64, **bf)
    large = _codec(H=24, r=384, C=256, **bf)
    odd = _codec(H=24, r=320, C=256, **bf)
    g = lambda c, T, Tf: L.nanokv_attend_full_tokens(ctypes.byref(c), ctypes.byref(c), T, Tf)  # noqa: E731
    assert g(small, 14040, 4680) == 4680       # single-CTA low-dim kernel: r = 192, C = 64
    assert g(large, 93600, 9360) == 9360       # 2-CTA low-dim kernel: r = 384, C = 256
    assert g(odd, 93600, 9360) == 93600        # r = 320: no low-dim kernel, low-dim tokens run full-dim
    assert g(odd, 93600, 93600) == 93600
    assert g(_codec(), 256, 100) == 100        # fp32: CUDA-core kernels, split kept
    assert g(small, 100, 200) == -1            # T_full > T
    assert g(small, -1, 0) == -1
    prev = nk.nanokv_set_kernel_path(1)        # CUDA-core path forced: split kept
    try:
        assert g(odd, 93600, 9360) == 9360
    finally:
        nk.nanokv_set_kernel_path(prev)


def test_workspace_follows_the_routing():
    """A codec with no low-dim tensor-core kernel (r = 320) attends every
    history token full-dim, so its workspace does not depend on the caller's
    split; with the CUDA-core path forced, the split is kept and the low-dim
    buffers appear."""
    L = nk.lib()
    bf = dict(d=128, param_dtype=_lib.BF16, scale_dtype=_lib.F16)
    large = _codec(H=24, r=320, C=256, **bf)
    small = _codec(H=12, r=192, C=64, **bf)
    ws = lambda c, T, Tf: L.nanokv_attend_workspace(4680, ctypes.byref(c), ctypes.byref(c), T, Tf, 4680)  # noqa: E731
    assert ws(large, 93600, 9360) == ws(large, 93600, 93600) > 0
    assert ws(small, 14040, 4680) != ws(small, 14040, 14040)
    prev = nk.nanokv_set_kernel_path(1)
    try:
        assert ws(large, 93600, 9360) != ws(large, 93600, 93600)
    finally:
        nk.nanokv_set_kernel_path(prev)


def test_routed_rejects_bad_ranges():
    """Routing ranges must be sorted, disjoint, inside [0, T), at most
    NANOKV_MAX_RANGES; bad ones are refused before anything is launched."""
    L = nk.lib()
    c = _codec()
    p = ctypes.c_void_p(1 << 20)
    h = _lib._Hist(1 << 20, 1 << 20, 1 << 20)

    def call(ranges, T=100, n=None):
        arr = (_lib._Range * max(1, len(ranges)))(*[_lib._Range(a, b) for a, b in ranges])
        return L.nanokv_attend_routed(p, _lib.F32, 4, ctypes.byref(c), ctypes.byref(c), ctypes.byref(h),
                                      ctypes.byref(h), T, arr, len(ranges) if n is None else n, None, None, None,
                                      None, 0, ctypes.c_float(0.25), p, None, p, 1 << 20, None)

    assert call([(10, 5), (12, 5)]) == _lib.ERR_INVALID   # overlap
    assert call([(50, 5), (10, 5)]) == _lib.ERR_INVALID   # not sorted
    assert call([(90, 20)]) == _lib.ERR_INVALID           # past T
    assert call([(5, -1)]) == _lib.ERR_INVALID            # negative count
    assert call([(0, 1)], n=_lib.MAX_RANGES + 1) == _lib.ERR_INVALID
    ws = lambda ranges: L.nanokv_attend_routed_workspace(  # noqa: E731
        4, ctypes.byref(c), ctypes.byref(c), 100,
        (_lib._Range * max(1, len(ranges)))(*[_lib._Range(a, b) for a, b in ranges]), len(ranges), None, None, 0)
    assert ws([(10, 5), (12, 5)]) == 0
    assert ws([(10, 5), (40, 5)]) > 0


def test_lowdim_validation():
    """Reduced attention dimensions: bf16 codecs with d = 128 only; d_h in
    {0, 32, 64, 96}; maps and tables non-NULL and aligned; all refused before
    anything is launched."""
    L = nk.lib()
    bf = dict(H=4, d=128, r=192, C=64, param_dtype=_lib.BF16, scale_dtype=_lib.F16)
    c, c32 = _codec(**bf), _codec()
    n = L.nanokv_lowdim_aux_bytes(ctypes.byref(c), ctypes.byref(c))
    assert n >= 2 * (4 * 128 * 192 * 2) + 2 * (64 * 4 * 128 * 2)
    assert L.nanokv_lowdim_aux_bytes(ctypes.byref(c32), ctypes.byref(c32)) == 0      # fp32, d = 16
    assert L.nanokv_lowdim_aux_bytes(ctypes.byref(c), ctypes.byref(_codec(**dict(bf, r=128)))) == 0
    p = ctypes.c_void_p(1 << 20)
    good = _lib._Lowdim(None, p, p, p)
    assert L.nanokv_lowdim_prepare(ctypes.byref(c32), ctypes.byref(c32), ctypes.byref(good), None) == _lib.ERR_UNSUPPORTED
    assert L.nanokv_lowdim_prepare(ctypes.byref(c), ctypes.byref(c), None, None) == _lib.ERR_INVALID
    assert L.nanokv_lowdim_prepare(ctypes.byref(c), ctypes.byref(c), ctypes.byref(_lib._Lowdim(None, None, p, p)),
                                   None) == _lib.ERR_INVALID
    assert L.nanokv_lowdim_prepare(ctypes.byref(c), ctypes.byref(c),
                                   ctypes.byref(_lib._Lowdim(None, p, p, ctypes.c_void_p((1 << 20) + 8))),
                                   None) == _lib.ERR_INVALID

    h = _lib._Hist(1 << 20, 1 << 20, 1 << 20)
    arr = (_lib._Range * 1)(_lib._Range(0, 10))

    def call(codec, dims, U=p, io=_lib.BF16):
        d = (ctypes.c_int32 * codec.H)(*dims)
        ld = _lib._Lowdim(d, U, p, p)
        return L.nanokv_attend_routed(p, io, 4, ctypes.byref(codec), ctypes.byref(codec), ctypes.byref(h),
                                      ctypes.byref(h), 100, arr, 1, None, ctypes.byref(ld), None, None, 0,
                                      ctypes.c_float(0.1), p, None, p, 1 << 30, None)

    assert call(c, [48, 0, 0, 0]) == _lib.ERR_INVALID       # not a deployed width
    assert call(c, [128, 0, 0, 0]) == _lib.ERR_INVALID      # full width: full_heads instead
    assert call(c, [32, 0, 0, 0], U=None) == _lib.ERR_INVALID
    assert call(_codec(H=4), [32, 0, 0, 0], io=_lib.F32) == _lib.ERR_UNSUPPORTED
    ws = lambda dims: L.nanokv_attend_routed_workspace(  # noqa: E731
        64, ctypes.byref(c), ctypes.byref(c), 100, arr, 1, None,
        ctypes.byref(_lib._Lowdim((ctypes.c_int32 * 4)(*dims), p, p, p)), 0)
    # the reduced queries [Tq, H, 128] bf16 join the workspace
    assert ws([32, 0, 64, 0]) >= ws([0, 0, 0, 0]) + 64 * 4 * 128 * 2


def test_calibrate_validation():
    """Calibration: J a multiple of 32 up to 3072, 1 <= C <= 256, 1 <= r <= J,
    aligned pointers and a large enough workspace; refused before any launch."""
    L = nk.lib()
    assert L.nanokv_calibrate_workspace(100, 48, 4) == 0
    assert L.nanokv_calibrate_workspace(100, 4096, 4) == 0
    n = L.nanokv_calibrate_workspace(100, 64, 4)
    assert n >= 2 * 64 * 64 * 4 + 4 * 64 * 4
    p = ctypes.c_void_p(1 << 20)

    def call(dt=_lib.BF16, N=100, J=64, C=4, r=8, rounds=2, ws=1 << 30, x=p):
        return L.nanokv_calibrate(x, dt, N, J, C, r, p, rounds, p, p, p, None, None, p, ws, None)

    assert call(dt=_lib.F16) == _lib.ERR_UNSUPPORTED
    assert call(J=48) == _lib.ERR_INVALID
    assert call(C=0) == _lib.ERR_INVALID
    assert call(r=65) == _lib.ERR_INVALID
    assert call(rounds=-1) == _lib.ERR_INVALID
    assert call(ws=16) == _lib.ERR_INVALID
    assert call(x=ctypes.c_void_p((1 << 20) + 4)) == _lib.ERR_INVALID
    assert call(x=None) == _lib.ERR_INVALID


def test_attend_partial_validation():
    """The fp32-partial attend checks its arguments like nanokv_attend and
    requires the LSE output (a partial without it cannot be merged)."""
    L = nk.lib()
    c = _codec()
    p = ctypes.c_void_p(1 << 20)
    h = _lib._Hist(1 << 20, 1 << 20, 1 << 20)
    call = lambda lse, T_full=8, Tq=4: L.nanokv_attend_partial(  # noqa: E731
        p, _lib.F32, Tq, ctypes.byref(c), ctypes.byref(c), ctypes.byref(h), ctypes.byref(h), 8, T_full, None, None,
        0, ctypes.c_float(0.25), p, lse, p, 1 << 20, None)
    assert call(None) == _lib.ERR_INVALID
    assert call(p, T_full=9) == _lib.ERR_INVALID
    assert call(None, Tq=0) == _lib.OK

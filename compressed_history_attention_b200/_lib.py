"""ctypes binding of libnanokv.so (argument marshalling only).

Every computation runs in the library's CUDA kernels; this module only turns
torch tensors into device pointers, sizes and the current CUDA stream, and
allocates outputs with torch.  There is no CPU fallback: if the shared library
is missing or a call fails, it raises.
"""
from __future__ import annotations

import ctypes
import dataclasses
import math
import os

import torch

_PKG = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_PKG, "libnanokv.so")

F32, F16, BF16 = 0, 1, 2
OK, ERR_INVALID, ERR_UNSUPPORTED, ERR_CUDA, ERR_TIMEOUT = 0, -1, -2, -3, -4

SYMBOLS = ("nanokv_encode", "nanokv_attend", "nanokv_attend_workspace", "nanokv_lse_merge",
           "nanokv_set_kernel_path", "nanokv_check", "nanokv_last_error", "nanokv_version",
           "nanokv_timing_enable", "nanokv_timing_read", "nanokv_codec_aux_bytes",
           "nanokv_codec_prepare", "nanokv_attend_static", "nanokv_selftest_wait",
           "nanokv_attend_full_tokens", "nanokv_attend_routed", "nanokv_attend_routed_workspace",
           "nanokv_lowdim_aux_bytes", "nanokv_lowdim_prepare", "nanokv_lowdim_analytic",
           "nanokv_calibrate_workspace", "nanokv_calibrate", "nanokv_attend_partial")

# kernel identities of the diagnostics (nanokv_kernel_id)
KERNELS = {0: "encode", 1: "attend_full", 2: "attend_low", 3: "attend_dense", 4: "lse_merge"}
K_COUNT = 8


class NanoKVError(RuntimeError):
    def __init__(self, status: int, msg: str):
        super().__init__(f"nanokv status {status}: {msg}")
        self.status = status


class _Codec(ctypes.Structure):
    _fields_ = [("H", ctypes.c_int32), ("d", ctypes.c_int32), ("r", ctypes.c_int32),
                ("C", ctypes.c_int32), ("param_dtype", ctypes.c_int32),
                ("scale_dtype", ctypes.c_int32), ("centers", ctypes.c_void_p),
                ("D", ctypes.c_void_p), ("E", ctypes.c_void_p), ("aux", ctypes.c_void_p)]


class _Hist(ctypes.Structure):
    _fields_ = [("ids", ctypes.c_void_p), ("codes", ctypes.c_void_p), ("scales", ctypes.c_void_p)]


class _Range(ctypes.Structure):
    _fields_ = [("start", ctypes.c_int64), ("count", ctypes.c_int64)]


MAX_RANGES = 64


class _Lowdim(ctypes.Structure):
    _fields_ = [("d_h", ctypes.POINTER(ctypes.c_int32)), ("U", ctypes.c_void_p), ("W", ctypes.c_void_p),
                ("aux", ctypes.c_void_p)]


_lib = None


def lib() -> ctypes.CDLL:
    """Loads libnanokv.so from the package directory (build it with
    `python -m compressed_history_attention_b200.build`)."""
    global _lib
    if _lib is not None:
        return _lib
    if not os.path.exists(LIB_PATH):
        raise ImportError(f"libnanokv.so not built ({LIB_PATH}); run "
                          "`python -m compressed_history_attention_b200.build`")
    L = ctypes.CDLL(LIB_PATH)
    vp, i32, i64, f32, sz = ctypes.c_void_p, ctypes.c_int32, ctypes.c_int64, ctypes.c_float, ctypes.c_size_t
    P = ctypes.POINTER
    L.nanokv_encode.argtypes = [P(_Codec), P(_Codec), vp, vp, i32, i64, vp, vp, vp, vp, vp, vp, vp]
    L.nanokv_encode.restype = ctypes.c_int
    L.nanokv_attend.argtypes = [vp, i32, i64, P(_Codec), P(_Codec), P(_Hist), P(_Hist), i64, i64,
                                vp, vp, i64, f32, vp, vp, vp, sz, vp]
    L.nanokv_attend.restype = ctypes.c_int
    L.nanokv_attend_static.argtypes = [vp, i32, i64, P(_Codec), P(_Codec), P(_Hist), P(_Hist), i64, i64,
                                       vp, vp, i64, f32, vp, vp, vp]
    L.nanokv_attend_static.restype = ctypes.c_int
    L.nanokv_attend_workspace.argtypes = [i64, P(_Codec), P(_Codec), i64, i64, i64]
    L.nanokv_attend_workspace.restype = sz
    L.nanokv_lse_merge.argtypes = [i32, P(vp), P(vp), i64, i32, i32, vp, i32, vp, vp]
    L.nanokv_lse_merge.restype = ctypes.c_int
    L.nanokv_set_kernel_path.argtypes = [i32]
    L.nanokv_set_kernel_path.restype = ctypes.c_int
    L.nanokv_check.argtypes = [vp]
    L.nanokv_check.restype = ctypes.c_int
    L.nanokv_last_error.restype = ctypes.c_char_p
    L.nanokv_version.restype = ctypes.c_char_p
    L.nanokv_codec_aux_bytes.argtypes = [P(_Codec)]
    L.nanokv_codec_aux_bytes.restype = sz
    L.nanokv_codec_prepare.argtypes = [P(_Codec), vp, vp]
    L.nanokv_codec_prepare.restype = ctypes.c_int
    L.nanokv_timing_enable.argtypes = [i32]
    L.nanokv_timing_enable.restype = ctypes.c_int
    L.nanokv_timing_read.argtypes = [vp, vp]
    L.nanokv_timing_read.restype = ctypes.c_int
    L.nanokv_selftest_wait.argtypes = [ctypes.c_uint64, vp]
    L.nanokv_selftest_wait.restype = ctypes.c_int
    L.nanokv_attend_full_tokens.argtypes = [P(_Codec), P(_Codec), i64, i64]
    L.nanokv_attend_full_tokens.restype = i64
    L.nanokv_attend_routed.argtypes = [vp, i32, i64, P(_Codec), P(_Codec), P(_Hist), P(_Hist), i64,
                                       P(_Range), i32, vp, P(_Lowdim), vp, vp, i64, f32, vp, vp, vp, sz, vp]
    L.nanokv_attend_routed.restype = ctypes.c_int
    L.nanokv_attend_routed_workspace.argtypes = [i64, P(_Codec), P(_Codec), i64, P(_Range), i32, vp,
                                                 P(_Lowdim), i64]
    L.nanokv_attend_routed_workspace.restype = sz
    L.nanokv_lowdim_aux_bytes.argtypes = [P(_Codec), P(_Codec)]
    L.nanokv_lowdim_aux_bytes.restype = sz
    L.nanokv_lowdim_prepare.argtypes = [P(_Codec), P(_Codec), P(_Lowdim), vp]
    L.nanokv_lowdim_prepare.restype = ctypes.c_int
    L.nanokv_lowdim_analytic.argtypes = [P(_Codec), vp, vp]
    L.nanokv_lowdim_analytic.restype = ctypes.c_int
    L.nanokv_calibrate_workspace.argtypes = [i64, i32, i32]
    L.nanokv_calibrate_workspace.restype = sz
    L.nanokv_calibrate.argtypes = [vp, i32, i64, i32, i32, i32, vp, i32, vp, vp, vp, vp, vp, vp, sz, vp]
    L.nanokv_calibrate.restype = ctypes.c_int
    L.nanokv_attend_partial.argtypes = L.nanokv_attend.argtypes
    L.nanokv_attend_partial.restype = ctypes.c_int
    _lib = L
    return L


def _raise(status: int):
    if status != OK:
        raise NanoKVError(status, lib().nanokv_last_error().decode())


def _ptr(t):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _stream(device=None):
    return ctypes.c_void_p(torch.cuda.current_stream(device).cuda_stream)


@dataclasses.dataclass
class Codec:
    """One K or V codec: centers [C, J], decoder D [J, r], encoder E [r, J]
    (E may be None for attention-only use).  fp32 tensors select the fp32 mode
    (fp32 scales), bf16 tensors the bf16 mode (fp16 scales)."""
    H: int
    d: int
    centers: torch.Tensor
    D: torch.Tensor
    E: torch.Tensor | None = None
    aux: torch.Tensor | None = None

    @property
    def r(self) -> int:
        return self.D.shape[1]

    @property
    def C(self) -> int:
        return self.centers.shape[0]

    @property
    def fp32(self) -> bool:
        return self.centers.dtype == torch.float32

    @property
    def scale_dtype(self) -> torch.dtype:
        return torch.float32 if self.fp32 else torch.float16

    def struct(self) -> _Codec:
        pd = F32 if self.fp32 else BF16
        sd = F32 if self.fp32 else F16
        return _Codec(self.H, self.d, self.r, self.C, pd, sd, self.centers.data_ptr(),
                      self.D.data_ptr(), self.E.data_ptr() if self.E is not None else None,
                      self.aux.data_ptr() if self.aux is not None else None)

    def prepare(self) -> "Codec":
        """Computes the codec's derived encode tables once (nanokv_codec_prepare)
        into a device buffer kept on this object."""
        sc = self.struct()
        sc.aux = None
        n = int(lib().nanokv_codec_aux_bytes(ctypes.byref(sc)))
        if n == 0:
            _raise(ERR_INVALID)
        aux = torch.empty(n, dtype=torch.uint8, device=self.centers.device)
        _raise(lib().nanokv_codec_prepare(ctypes.byref(sc), ctypes.c_void_p(aux.data_ptr()),
                                          _stream(self.centers.device)))
        self.aux = aux
        return self


@dataclasses.dataclass
class Hist:
    """Compressed history of one branch: ids [T] u8, codes [T, r/2] u8,
    scales [T] (fp16 or fp32)."""
    ids: torch.Tensor
    codes: torch.Tensor
    scales: torch.Tensor

    def __len__(self):
        return self.ids.shape[0]

    def struct(self) -> _Hist:
        return _Hist(self.ids.data_ptr(), self.codes.data_ptr(), self.scales.data_ptr())

    def slice(self, lo: int, hi: int) -> "Hist":
        return Hist(self.ids[lo:hi], self.codes[lo:hi], self.scales[lo:hi])


def _dt(t: torch.Tensor) -> int:
    return {torch.float32: F32, torch.bfloat16: BF16, torch.float16: F16}[t.dtype]


def alloc_hist(codec: Codec, T: int, device) -> Hist:
    return Hist(torch.empty(T, dtype=torch.uint8, device=device),
                torch.empty(T, codec.r // 2, dtype=torch.uint8, device=device),
                torch.empty(T, dtype=codec.scale_dtype, device=device))


def nanokv_encode(ck: Codec | None, cv: Codec | None, k: torch.Tensor | None, v: torch.Tensor | None,
                  out_k: Hist | None = None, out_v: Hist | None = None):
    """Encode K and V tokens [T, J]; returns (Hist_k, Hist_v) (None for a
    skipped branch).  Outputs may be preallocated (e.g. views into a cache)."""
    x0 = k if k is not None else v
    T = x0.shape[0]
    dev = x0.device
    for c in (ck, cv):
        if c is not None and c.aux is None and c.E is not None:
            c.prepare()
    if ck is not None and out_k is None:
        out_k = alloc_hist(ck, T, dev)
    if cv is not None and out_v is None:
        out_v = alloc_hist(cv, T, dev)
    sk = ck.struct() if ck is not None else None
    sv = cv.struct() if cv is not None else None
    st = lib().nanokv_encode(
        ctypes.byref(sk) if sk is not None else None, ctypes.byref(sv) if sv is not None else None,
        _ptr(k), _ptr(v), _dt(x0), T,
        _ptr(out_k.ids if out_k else None), _ptr(out_k.codes if out_k else None),
        _ptr(out_k.scales if out_k else None),
        _ptr(out_v.ids if out_v else None), _ptr(out_v.codes if out_v else None),
        _ptr(out_v.scales if out_v else None), _stream(dev))
    _raise(st)
    return out_k, out_v


def nanokv_attend_workspace(Tq: int, ck: Codec, cv: Codec, T: int, T_full: int, T_cur: int) -> int:
    sk, sv = ck.struct(), cv.struct()
    return int(lib().nanokv_attend_workspace(Tq, ctypes.byref(sk), ctypes.byref(sv), T, T_full, T_cur))


def nanokv_attend(q: torch.Tensor, ck: Codec, cv: Codec, hk: Hist | None, hv: Hist | None,
                  T_full: int, k_cur: torch.Tensor | None = None, v_cur: torch.Tensor | None = None,
                  softmax_scale: float | None = None, out: torch.Tensor | None = None,
                  lse: torch.Tensor | bool | None = True, workspace: torch.Tensor | None = None):
    """Attention of q [Tq, H, d] over compressed history (T_full most recent
    tokens full-dim, the rest low-dim) plus the current chunk k_cur/v_cur
    [T_cur, H, d].  Returns (out [Tq, H, d], lse [H, Tq] fp32 or None)."""
    Tq, H, d = q.shape
    T = len(hk) if hk is not None else 0
    T_cur = k_cur.shape[0] if k_cur is not None else 0
    if softmax_scale is None:
        softmax_scale = 1.0 / math.sqrt(d)
    dev = q.device
    if out is None:
        out = torch.empty_like(q)
    if lse is True:
        lse = torch.empty(H, Tq, dtype=torch.float32, device=dev)
    elif lse is False:
        lse = None
    need = nanokv_attend_workspace(Tq, ck, cv, T, T_full, T_cur)
    if workspace is None or workspace.numel() * workspace.element_size() < need:
        workspace = torch.empty(max(need, 16), dtype=torch.uint8, device=dev)
    sk, sv = ck.struct(), cv.struct()
    shk = hk.struct() if hk is not None and T else None
    shv = hv.struct() if hv is not None and T else None
    st = lib().nanokv_attend(
        _ptr(q), _dt(q), Tq, ctypes.byref(sk), ctypes.byref(sv),
        ctypes.byref(shk) if shk else None, ctypes.byref(shv) if shv else None, T, T_full,
        _ptr(k_cur), _ptr(v_cur), T_cur, ctypes.c_float(softmax_scale), _ptr(out), _ptr(lse),
        _ptr(workspace), workspace.numel() * workspace.element_size(), _stream(dev))
    _raise(st)
    return out, lse


def _ranges(full):
    arr = (_Range * max(1, len(full)))(*[_Range(int(a), int(c)) for a, c in full])
    return arr, len(full)


def _heads(full_heads, H):
    if full_heads is None:
        return None, None
    buf = (ctypes.c_uint8 * H)(*[1 if h else 0 for h in full_heads])
    return buf, ctypes.cast(buf, ctypes.c_void_p)


@dataclasses.dataclass
class Lowdim:
    """Maps of the heads deployed at a reduced attention dimension: U, W
    [H, d, d] (head h's map in the leading columns of U[h] / W[h]) and the
    mapped decoder / center tables (aux) that nanokv_lowdim_prepare wrote."""
    U: torch.Tensor
    W: torch.Tensor
    aux: torch.Tensor

    def struct(self, d_h) -> tuple:
        arr = (ctypes.c_int32 * len(d_h))(*[int(v) for v in d_h])
        return arr, _Lowdim(arr, self.U.data_ptr(), self.W.data_ptr(), self.aux.data_ptr())


def nanokv_lowdim_prepare(ck: Codec, cv: Codec, U: torch.Tensor, W: torch.Tensor) -> Lowdim:
    """Maps the codecs' decoder rows and centers through U (keys) and W
    (values) once (nanokv_lowdim_prepare), into a buffer kept on the result."""
    sk, sv = ck.struct(), cv.struct()
    n = int(lib().nanokv_lowdim_aux_bytes(ctypes.byref(sk), ctypes.byref(sv)))
    if n == 0:
        _raise(ERR_UNSUPPORTED)
    ld = Lowdim(U.contiguous(), W.contiguous(), torch.empty(n, dtype=torch.uint8, device=ck.D.device))
    _keep, s = ld.struct([0] * ck.H)
    _raise(lib().nanokv_lowdim_prepare(ctypes.byref(sk), ctypes.byref(sv), ctypes.byref(s), _stream(ck.D.device)))
    return ld


def nanokv_lowdim_analytic(c: Codec) -> torch.Tensor:
    """Analytical maps [H, d, d] of a codec (nanokv_lowdim_analytic): the
    left singular vectors of each head's decoder rows, by decreasing
    singular value."""
    maps = torch.empty(c.H, c.d, c.d, dtype=c.D.dtype, device=c.D.device)
    sc = c.struct()
    _raise(lib().nanokv_lowdim_analytic(ctypes.byref(sc), _ptr(maps), _stream(c.D.device)))
    return maps


def nanokv_calibrate(x: torch.Tensor, init_centers: torch.Tensor, rounds: int, r: int) -> dict:
    """Codec of one branch fitted on tokens x [N, J] (nanokv_calibrate):
    k-means centers from init_centers [C, J], then the r leading eigenvectors
    of the residual second moment as D [J, r] and E = D^T, in x's dtype; also
    the final assignment and the eigenvalues."""
    x = x.contiguous()
    N, J = x.shape
    C = init_centers.shape[0]
    dev = x.device
    out = {"centers": torch.empty(C, J, dtype=x.dtype, device=dev),
           "D": torch.empty(J, r, dtype=x.dtype, device=dev), "E": torch.empty(r, J, dtype=x.dtype, device=dev),
           "ids": torch.empty(N, dtype=torch.uint8, device=dev),
           "eigenvalues": torch.empty(r, dtype=torch.float32, device=dev)}
    n = int(lib().nanokv_calibrate_workspace(N, J, C))
    ws = torch.empty(max(n, 16), dtype=torch.uint8, device=dev)
    init = init_centers.to(torch.float32).contiguous()
    _raise(lib().nanokv_calibrate(_ptr(x), _dt(x), N, J, C, r, _ptr(init), rounds, _ptr(out["centers"]),
                                  _ptr(out["D"]), _ptr(out["E"]), _ptr(out["ids"]), _ptr(out["eigenvalues"]),
                                  _ptr(ws), n, _stream(dev)))
    return out


def _lowdim(lowdim: Lowdim | None, d_h):
    if lowdim is None:
        return None, None
    if d_h is None:
        raise ValueError("a Lowdim needs the per-head d_h")
    keep, s = lowdim.struct(d_h)
    return (keep, s), ctypes.byref(s)


def nanokv_attend_routed_workspace(Tq: int, ck: Codec, cv: Codec, T: int, full, full_heads, T_cur: int,
                                   lowdim: Lowdim | None = None, d_h=None) -> int:
    sk, sv = ck.struct(), cv.struct()
    arr, n = _ranges(full)
    _keep, hp = _heads(full_heads, ck.H)
    _keep2, lp = _lowdim(lowdim, d_h)
    return int(lib().nanokv_attend_routed_workspace(Tq, ctypes.byref(sk), ctypes.byref(sv), T, arr, n, hp, lp,
                                                    T_cur))


def nanokv_attend_routed(q: torch.Tensor, ck: Codec, cv: Codec, hk: Hist | None, hv: Hist | None, full,
                         full_heads=None, k_cur: torch.Tensor | None = None, v_cur: torch.Tensor | None = None,
                         softmax_scale: float | None = None, out: torch.Tensor | None = None,
                         lse: torch.Tensor | bool | None = True, workspace: torch.Tensor | None = None,
                         lowdim: Lowdim | None = None, d_h=None):
    """nanokv_attend under a routing policy: `full` is a list of (start,
    count) history token ranges read full-dim (sorted, disjoint), the rest
    low-dim; `full_heads` (H truth values, or None) marks heads that read all
    their history full-dim; `lowdim` with `d_h` (H ints: 0, 32, 64 or 96)
    puts heads at a reduced attention dimension for their low-dim tokens.
    Returns (out, lse) as nanokv_attend."""
    Tq, H, d = q.shape
    T = len(hk) if hk is not None else 0
    T_cur = k_cur.shape[0] if k_cur is not None else 0
    if softmax_scale is None:
        softmax_scale = 1.0 / math.sqrt(d)
    dev = q.device
    if out is None:
        out = torch.empty_like(q)
    if lse is True:
        lse = torch.empty(H, Tq, dtype=torch.float32, device=dev)
    elif lse is False:
        lse = None
    # (0 for arguments the call itself then refuses with its own status)
    need = nanokv_attend_routed_workspace(Tq, ck, cv, T, full, full_heads, T_cur, lowdim, d_h)
    if workspace is None or workspace.numel() * workspace.element_size() < need:
        workspace = torch.empty(max(need, 16), dtype=torch.uint8, device=dev)
    sk, sv = ck.struct(), cv.struct()
    shk = hk.struct() if hk is not None and T else None
    shv = hv.struct() if hv is not None and T else None
    arr, n = _ranges(full)
    _keep, hp = _heads(full_heads, H)
    _keep2, lp = _lowdim(lowdim, d_h)
    st = lib().nanokv_attend_routed(
        _ptr(q), _dt(q), Tq, ctypes.byref(sk), ctypes.byref(sv),
        ctypes.byref(shk) if shk else None, ctypes.byref(shv) if shv else None, T, arr, n, hp, lp,
        _ptr(k_cur), _ptr(v_cur), T_cur, ctypes.c_float(softmax_scale), _ptr(out), _ptr(lse),
        _ptr(workspace), workspace.numel() * workspace.element_size(), _stream(dev))
    _raise(st)
    return out, lse


def nanokv_attend_static(q: torch.Tensor, ck: Codec, cv: Codec, hk: Hist | None, hv: Hist | None,
                         T_full: int, k_cur: torch.Tensor | None = None, v_cur: torch.Tensor | None = None,
                         softmax_scale: float | None = None, out: torch.Tensor | None = None,
                         lse: torch.Tensor | None = None):
    """nanokv_attend for callers that cannot allocate device memory: scratch
    comes from the library's fixed 32 MiB device array; out and lse must be
    given (no allocation happens here)."""
    Tq, H, d = q.shape
    T = len(hk) if hk is not None else 0
    T_cur = k_cur.shape[0] if k_cur is not None else 0
    if softmax_scale is None:
        softmax_scale = 1.0 / math.sqrt(d)
    if out is None:
        raise ValueError("nanokv_attend_static needs a preallocated out tensor")
    sk, sv = ck.struct(), cv.struct()
    shk = hk.struct() if hk is not None and T else None
    shv = hv.struct() if hv is not None and T else None
    st = lib().nanokv_attend_static(
        _ptr(q), _dt(q), Tq, ctypes.byref(sk), ctypes.byref(sv),
        ctypes.byref(shk) if shk else None, ctypes.byref(shv) if shv else None, T, T_full,
        _ptr(k_cur), _ptr(v_cur), T_cur, ctypes.c_float(softmax_scale), _ptr(out), _ptr(lse),
        _stream(q.device))
    _raise(st)
    return out, lse


def nanokv_attend_partial(q: torch.Tensor, ck: Codec, cv: Codec, hk: Hist | None, hv: Hist | None,
                          T_full: int, k_cur: torch.Tensor | None = None, v_cur: torch.Tensor | None = None,
                          softmax_scale: float | None = None, workspace: torch.Tensor | None = None):
    """nanokv_attend with an fp32 output: the partial (O [Tq, H, d] fp32,
    LSE [H, Tq]) over this call's keys, for an LSE merge with partials over
    other keys (nanokv_attend_partial)."""
    Tq, H, d = q.shape
    T = len(hk) if hk is not None else 0
    T_cur = k_cur.shape[0] if k_cur is not None else 0
    if softmax_scale is None:
        softmax_scale = 1.0 / math.sqrt(d)
    dev = q.device
    out = torch.empty(Tq, H, d, dtype=torch.float32, device=dev)
    lse = torch.empty(H, Tq, dtype=torch.float32, device=dev)
    need = nanokv_attend_workspace(Tq, ck, cv, T, T_full, T_cur)
    if workspace is None or workspace.numel() * workspace.element_size() < need:
        workspace = torch.empty(max(need, 16), dtype=torch.uint8, device=dev)
    sk, sv = ck.struct(), cv.struct()
    shk = hk.struct() if hk is not None and T else None
    shv = hv.struct() if hv is not None and T else None
    st = lib().nanokv_attend_partial(
        _ptr(q), _dt(q), Tq, ctypes.byref(sk), ctypes.byref(sv),
        ctypes.byref(shk) if shk else None, ctypes.byref(shv) if shv else None, T, T_full,
        _ptr(k_cur), _ptr(v_cur), T_cur, ctypes.c_float(softmax_scale), _ptr(out), _ptr(lse),
        _ptr(workspace), workspace.numel() * workspace.element_size(), _stream(dev))
    _raise(st)
    return out, lse


def nanokv_lse_merge(o_parts, lse_parts, out_dtype=torch.bfloat16, out=None, lse=True):
    """LSE-merge fp32 partials O_i [Tq, H, d], LSE_i [H, Tq]."""
    n = len(o_parts)
    Tq, H, d = o_parts[0].shape
    dev = o_parts[0].device
    if out is None:
        out = torch.empty(Tq, H, d, dtype=out_dtype, device=dev)
    if lse is True:
        lse = torch.empty(H, Tq, dtype=torch.float32, device=dev)
    elif lse is False:
        lse = None
    arr = ctypes.c_void_p * max(n, 1)
    op = arr(*[p.data_ptr() for p in o_parts])
    lp = arr(*[p.data_ptr() for p in lse_parts])
    st = lib().nanokv_lse_merge(n, op, lp, Tq, H, d, _ptr(out), _dt(out), _ptr(lse), _stream(dev))
    _raise(st)
    return out, lse


def nanokv_set_kernel_path(path: int) -> int:
    """0 = automatic, 1 = fp32 CUDA-core kernels only, 2 = tensor-core only."""
    prev = lib().nanokv_set_kernel_path(path)
    if prev < 0:
        raise ValueError(path)
    return prev


def nanokv_check(device=None) -> None:
    _raise(lib().nanokv_check(_stream(device)))


def nanokv_attend_full_tokens(ck: Codec, cv: Codec, T: int, T_full: int) -> int:
    """History tokens nanokv_attend takes on the full-dim path (T_full, or T
    when the codec shape has no low-dim tensor-core kernel)."""
    sk, sv = ck.struct(), cv.struct()
    n = int(lib().nanokv_attend_full_tokens(ctypes.byref(sk), ctypes.byref(sv), T, T_full))
    if n < 0:
        raise NanoKVError(ERR_INVALID, "nanokv_attend_full_tokens: invalid arguments")
    return n


def nanokv_selftest_wait(limit_ms: float = 50.0, device=None) -> None:
    """Failure-detection self-test: a kernel gives up on a wait nothing
    satisfies after ~limit_ms; the next nanokv_check() reports the timeout."""
    _raise(lib().nanokv_selftest_wait(ctypes.c_uint64(int(limit_ms * 1e6)), _stream(device)))


def nanokv_version() -> str:
    return lib().nanokv_version().decode()


def nanokv_timing_enable(on: bool) -> bool:
    """Per-kernel CUDA-event timing of every later launch (diagnostics)."""
    return bool(lib().nanokv_timing_enable(1 if on else 0))


def nanokv_timing_read() -> dict:
    """{kernel: (total_ms, launches)} since the last read; waits for the
    recorded events."""
    ms = (ctypes.c_double * K_COUNT)()
    n = (ctypes.c_int64 * K_COUNT)()
    _raise(lib().nanokv_timing_read(ms, n))
    return {name: (ms[k], n[k]) for k, name in KERNELS.items()}

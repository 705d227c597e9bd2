"""Python binding of the lbq C ABI (include/lbq.h).

Argument marshalling only: every computation runs in the CUDA kernels of
liblbq.so.  The low-level functions (`lbq_quantize`, `lbq_linear_fwd`, ...)
have the C names and take raw integers (device pointers, sizes, stream
handles) and `lbq_qweight` structures.  The helpers below them accept torch
tensors, allocate outputs and workspaces with torch (device memory is the one
thing PyTorch supplies) and pass pointers through.

There is no fallback: importing this module fails when liblbq.so is missing,
and every call raises `LbqError` when the library returns a non-OK status.
"""
from __future__ import annotations

import ctypes
import os
import re
from typing import Optional

HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(HERE, "liblbq.so")
HEADER = os.path.join(os.path.dirname(HERE), "include", "lbq.h")

if not os.path.exists(LIB_PATH):
    raise ImportError(f"{LIB_PATH} is missing: build it with `python -m qlora_quantized_linear_b200.build`")
_L = ctypes.CDLL(LIB_PATH)

LBQ_OK, LBQ_EINVAL, LBQ_EALIGN, LBQ_EUNSUPPORTED, LBQ_ECUDA, LBQ_ETIMEOUT, LBQ_EWORKSPACE = range(7)
LBQ_MINMAX_ASYM, LBQ_CODEBOOK4 = 0, 1
STATUS_TIMEOUT, STATUS_BAD_TABLE = 1, 2


class lbq_qweight(ctypes.Structure):
    _fields_ = [
        ("n", ctypes.c_int32), ("k", ctypes.c_int32),
        ("bits", ctypes.c_int32), ("group", ctypes.c_int32),
        ("scheme", ctypes.c_int32), ("double_quant", ctypes.c_int32),
        ("packed", ctypes.c_void_p),
        ("scale", ctypes.c_void_p), ("zero", ctypes.c_void_p),
        ("absmax", ctypes.c_void_p),
        ("absmax_q8", ctypes.c_void_p), ("absmax_s2", ctypes.c_void_p), ("absmax_offset", ctypes.c_void_p),
        ("codebook", ctypes.c_void_p),
    ]


class lbq_qweight_mix(ctypes.Structure):
    _fields_ = [("hi", lbq_qweight), ("lo", lbq_qweight), ("perm", ctypes.c_void_p)]


class lbq_fwd_problem(ctypes.Structure):
    _fields_ = [("X", ctypes.c_void_p), ("q", ctypes.POINTER(lbq_qweight)), ("A", ctypes.c_void_p),
                ("B", ctypes.c_void_p), ("rank", ctypes.c_int32), ("s", ctypes.c_float),
                ("Y", ctypes.c_void_p), ("T_save", ctypes.c_void_p)]


class lbq_bwd_problem(ctypes.Structure):
    _fields_ = [("dY", ctypes.c_void_p), ("q", ctypes.POINTER(lbq_qweight)), ("A", ctypes.c_void_p),
                ("B", ctypes.c_void_p), ("rank", ctypes.c_int32), ("s", ctypes.c_float),
                ("dX", ctypes.c_void_p), ("U_save", ctypes.c_void_p)]


class lbq_mix_problem(ctypes.Structure):
    _fields_ = [("X", ctypes.c_void_p), ("q", ctypes.POINTER(lbq_qweight_mix)), ("A", ctypes.c_void_p),
                ("B", ctypes.c_void_p), ("rank", ctypes.c_int32), ("s", ctypes.c_float),
                ("Y", ctypes.c_void_p), ("T_save", ctypes.c_void_p)]


_vp, _int, _f32, _sz, _u32p = ctypes.c_void_p, ctypes.c_int, ctypes.c_float, ctypes.c_size_t, ctypes.POINTER(ctypes.c_uint32)
_QP, _MP = ctypes.POINTER(lbq_qweight), ctypes.POINTER(lbq_qweight_mix)
_PP, _QPP, _I64P = ctypes.POINTER(lbq_fwd_problem), ctypes.POINTER(ctypes.POINTER(lbq_qweight)), ctypes.POINTER(ctypes.c_int64)
_BPP = ctypes.POINTER(lbq_bwd_problem)
_MPP = ctypes.POINTER(lbq_mix_problem)
_SIGS = {
    "lbq_status_string": (ctypes.c_char_p, [_int]),
    "lbq_quantize_workspace_size": (_sz, [_QP]),
    "lbq_quantize": (_int, [_vp, _QP, _vp, _sz, _vp]),
    "lbq_dequantize": (_int, [_QP, _vp, _vp]),
    "lbq_linear_fwd_workspace_size": (_sz, [_int, _QP, _int]),
    "lbq_linear_fwd": (_int, [_vp, _int, _QP, _vp, _vp, _int, _f32, _vp, _vp, _vp, _sz, _vp]),
    "lbq_linear_fwd_noalloc": (_int, [_vp, _int, _QP, _vp, _vp, _int, _f32, _vp, _vp, _vp]),
    "lbq_linear_fwd_mix_workspace_size": (_sz, [_int, _MP, _int]),
    "lbq_linear_fwd_mix": (_int, [_vp, _int, _MP, _vp, _vp, _int, _f32, _vp, _vp, _vp, _sz, _vp]),
    "lbq_linear_bwd_workspace_size": (_sz, [_int, _QP, _int]),
    "lbq_linear_bwd": (_int, [_vp, _int, _QP, _vp, _vp, _int, _f32, _vp, _vp, _vp, _sz, _vp]),
    "lbq_lora_grads": (_int, [_vp, _vp, _int, _int, _int, _vp, _vp, _int, _f32, _vp, _vp, _vp]),
    "lbq_device_status": (_int, [_u32p]),
    "lbq_merge_lora": (_int, [_QP, _vp, _vp, _int, _f32, _vp, _vp]),
    "lbq_gemv_plan": (_int, [_int, _QPP, _int, _int, _I64P, _I64P]),
    "lbq_linear_fwd_grouped_workspace_size": (_sz, [_int, _PP, _int]),
    "lbq_linear_fwd_grouped": (_int, [_int, _PP, _int, _vp, _sz, _vp]),
    "lbq_linear_bwd_grouped_workspace_size": (_sz, [_int, _BPP, _int]),
    "lbq_linear_bwd_grouped": (_int, [_int, _BPP, _int, _vp, _sz, _vp]),
    "lbq_unmerge_lora": (_int, [_vp, _int, _int, _vp, _vp, _int, _f32, _vp, _vp]),
    "lbq_linear_fwd_noalloc_reset": (_int, [_vp]),
    "lbq_channel_mix_select_workspace_size": (_sz, [_int, _int]),
    "lbq_channel_mix_select": (_int, [_vp, _int, _int, _vp, _int, _int, _vp, _vp, _vp, _sz, _vp]),
    "lbq_gather_rows": (_int, [_vp, _int, _int, _vp, _int, _vp, _vp]),
    "lbq_selftest_wait_timeout": (_int, [ctypes.c_uint32, _vp]),
    "lbq_linear_fwd_mix_grouped_workspace_size": (_sz, [_int, _MPP, _int]),
    "lbq_linear_fwd_mix_grouped": (_int, [_int, _MPP, _int, _vp, _sz, _vp]),
}
for _name, (_res, _args) in _SIGS.items():
    _f = getattr(_L, _name)
    _f.restype, _f.argtypes = _res, _args


def header_functions():
    """Names of the functions that include/lbq.h declares."""
    text = open(HEADER).read()
    return sorted(set(re.findall(r"^\s*(?:const\s+)?\w+\*?\s+\*?(lbq_\w+)\(", text, re.M)))


# --------------------------------------------------------------------------- C names
lbq_status_string = _L.lbq_status_string
lbq_quantize_workspace_size = _L.lbq_quantize_workspace_size
lbq_quantize = _L.lbq_quantize
lbq_dequantize = _L.lbq_dequantize
lbq_linear_fwd_workspace_size = _L.lbq_linear_fwd_workspace_size
lbq_linear_fwd = _L.lbq_linear_fwd
lbq_linear_fwd_noalloc = _L.lbq_linear_fwd_noalloc
lbq_linear_fwd_mix_workspace_size = _L.lbq_linear_fwd_mix_workspace_size
lbq_linear_fwd_mix = _L.lbq_linear_fwd_mix
lbq_linear_bwd_workspace_size = _L.lbq_linear_bwd_workspace_size
lbq_linear_bwd = _L.lbq_linear_bwd
lbq_lora_grads = _L.lbq_lora_grads
lbq_device_status = _L.lbq_device_status
lbq_merge_lora = _L.lbq_merge_lora
lbq_gemv_plan = _L.lbq_gemv_plan
lbq_linear_fwd_grouped_workspace_size = _L.lbq_linear_fwd_grouped_workspace_size
lbq_linear_fwd_grouped = _L.lbq_linear_fwd_grouped
lbq_linear_bwd_grouped_workspace_size = _L.lbq_linear_bwd_grouped_workspace_size
lbq_linear_bwd_grouped = _L.lbq_linear_bwd_grouped
lbq_unmerge_lora = _L.lbq_unmerge_lora
lbq_linear_fwd_noalloc_reset = _L.lbq_linear_fwd_noalloc_reset
lbq_channel_mix_select_workspace_size = _L.lbq_channel_mix_select_workspace_size
lbq_channel_mix_select = _L.lbq_channel_mix_select
lbq_gather_rows = _L.lbq_gather_rows
lbq_selftest_wait_timeout = _L.lbq_selftest_wait_timeout
lbq_linear_fwd_mix_grouped_workspace_size = _L.lbq_linear_fwd_mix_grouped_workspace_size
lbq_linear_fwd_mix_grouped = _L.lbq_linear_fwd_mix_grouped


class LbqError(RuntimeError):
    def __init__(self, code: int, what: str):
        self.code = code
        super().__init__(f"{what}: {lbq_status_string(code).decode()} (status {code})")


def _check(code: int, what: str) -> None:
    if code != LBQ_OK:
        raise LbqError(code, what)


# --------------------------------------------------------------------------- torch helpers
def _torch():
    import torch
    return torch


def _ptr(t) -> Optional[int]:
    return None if t is None else t.data_ptr()


def _stream(stream) -> Optional[int]:
    torch = _torch()
    if stream is None:
        stream = torch.cuda.current_stream()
    return stream.cuda_stream


def _bf16_2d(t, name):
    torch = _torch()
    if t.dtype != torch.bfloat16 or t.dim() != 2 or not t.is_cuda or not t.is_contiguous():
        raise ValueError(f"{name} must be a contiguous 2-D bf16 CUDA tensor")
    return t


class QuantizedWeight:
    """Device buffers of one quantized weight plus its `lbq_qweight` view.

    scheme "minmax": bits 4 (group 128) or 2 (group 64).
    scheme "codebook": 4-bit codes, absmax per 64, optional double quantization;
    `codebook` is 16 sorted floats in [-1, 1] with an exact 0.
    """

    def __init__(self, n: int, k: int, scheme: str = "minmax", bits: int = 4, group: Optional[int] = None,
                 double_quant: bool = False, codebook=None, device="cuda"):
        torch = _torch()
        self.n, self.k, self.scheme, self.bits = int(n), int(k), scheme, int(bits)
        self.double_quant = bool(double_quant)
        u8, f32 = torch.uint8, torch.float32
        if scheme == "minmax":
            self.group = int(group or (128 if bits == 4 else 64))
            self.packed = torch.empty((n, k * bits // 8), dtype=u8, device=device)
            self.scale = torch.empty((n, k // self.group), dtype=torch.float16, device=device)
            self.zero = torch.empty((n, k // self.group), dtype=torch.float16, device=device)
            self.absmax = self.q8 = self.s2 = self.offset = self.codebook = None
        elif scheme == "codebook":
            self.group, self.bits = 64, 4
            nb = n * k // 64
            self.packed = torch.empty((n, k // 2), dtype=u8, device=device)
            self.scale = self.zero = None
            self.absmax = torch.empty(nb, dtype=f32, device=device)
            self.codebook = torch.as_tensor(codebook, dtype=f32).to(device).contiguous()
            if self.double_quant:
                self.q8 = torch.empty(nb, dtype=torch.int8, device=device)
                self.s2 = torch.empty((nb + 255) // 256, dtype=f32, device=device)
                self.offset = torch.empty(4, dtype=f32, device=device)  # 1 used; 16-byte buffer
            else:
                self.q8 = self.s2 = self.offset = None
        else:
            raise ValueError(f"unknown scheme {scheme!r}")
        self.struct = self._make_struct()

    def _make_struct(self) -> lbq_qweight:
        return lbq_qweight(
            n=self.n, k=self.k, bits=self.bits, group=self.group,
            scheme=LBQ_MINMAX_ASYM if self.scheme == "minmax" else LBQ_CODEBOOK4,
            double_quant=int(self.double_quant),
            packed=_ptr(self.packed), scale=_ptr(self.scale), zero=_ptr(self.zero), absmax=_ptr(self.absmax),
            absmax_q8=_ptr(self.q8), absmax_s2=_ptr(self.s2), absmax_offset=_ptr(self.offset),
            codebook=_ptr(self.codebook))

    def quantize(self, W, stream=None) -> "QuantizedWeight":
        torch = _torch()
        W = _bf16_2d(W, "W")
        assert tuple(W.shape) == (self.n, self.k)
        nws = lbq_quantize_workspace_size(ctypes.byref(self.struct))
        ws = torch.empty(max(nws, 16), dtype=torch.uint8, device=W.device) if nws else None
        _check(lbq_quantize(W.data_ptr(), ctypes.byref(self.struct), _ptr(ws), nws, _stream(stream)), "lbq_quantize")
        self._keep = ws
        return self

    def dequantize(self, stream=None):
        torch = _torch()
        out = torch.empty((self.n, self.k), dtype=torch.float32, device=self.packed.device)
        _check(lbq_dequantize(ctypes.byref(self.struct), out.data_ptr(), _stream(stream)), "lbq_dequantize")
        return out


class ChannelMixWeight:
    """Channel-mix weight: INT4 g128 rows `hi`, INT2 g64 rows `lo`, and perm
    (stored row -> original output channel; rows of hi first)."""

    def __init__(self, hi: QuantizedWeight, lo: QuantizedWeight, perm):
        torch = _torch()
        self.hi, self.lo = hi, lo
        self.perm = torch.as_tensor(perm, dtype=torch.int32).to(hi.packed.device).contiguous()
        self.n, self.k = hi.n + lo.n, hi.k
        self.struct = lbq_qweight_mix(hi=hi.struct, lo=lo.struct, perm=self.perm.data_ptr())


def channel_mix_select(W, X_calib, n4: int, stream=None):
    """(perm int32 [n], score fp64 [n]) on the device: the n4 channels of W
    whose INT4 -> INT2 error rise, weighted by the calibration activations'
    second moments, is largest come first (lbq_channel_mix_select)."""
    torch = _torch()
    W, X_calib = _bf16_2d(W, "W"), _bf16_2d(X_calib, "X_calib")
    n, k = W.shape
    perm = torch.empty(n, dtype=torch.int32, device=W.device)
    score = torch.empty(n, dtype=torch.float64, device=W.device)
    nws = lbq_channel_mix_select_workspace_size(n, k)
    ws = torch.empty(max(nws, 16), dtype=torch.uint8, device=W.device)
    _check(lbq_channel_mix_select(W.data_ptr(), n, k, X_calib.data_ptr(), X_calib.shape[0], int(n4), score.data_ptr(),
                                  perm.data_ptr(), ws.data_ptr(), nws, _stream(stream)), "lbq_channel_mix_select")
    return perm, score


def gather_rows(W, rows, stream=None):
    """W[rows] (bf16 rows gathered on the device by lbq_gather_rows)."""
    torch = _torch()
    W = _bf16_2d(W, "W")
    rows = torch.as_tensor(rows, dtype=torch.int32, device=W.device).contiguous()
    out = torch.empty((rows.numel(), W.shape[1]), dtype=torch.bfloat16, device=W.device)
    _check(lbq_gather_rows(W.data_ptr(), W.shape[0], W.shape[1], rows.data_ptr(), rows.numel(), out.data_ptr(),
                           _stream(stream)), "lbq_gather_rows")
    return out


def channel_mix_weight(W, X_calib, frac_int4: float = 0.25, stream=None):
    """A ChannelMixWeight of W: the round(frac_int4 * n) most sensitive channels
    (lbq_channel_mix_select) as INT4 g128 rows, the others as INT2 g64 rows."""
    n, k = W.shape
    n4 = int(round(frac_int4 * n))
    perm, _ = channel_mix_select(W, X_calib, n4, stream=stream)
    hi = QuantizedWeight(n4, k, "minmax", 4).quantize(gather_rows(W, perm[:n4], stream=stream), stream=stream)
    lo = QuantizedWeight(n - n4, k, "minmax", 2).quantize(gather_rows(W, perm[n4:], stream=stream), stream=stream)
    return ChannelMixWeight(hi, lo, perm)


def _workspace(nbytes: int, device):
    torch = _torch()
    # zero-filled once: the library leaves its counters at zero after every call
    return torch.zeros(max(int(nbytes), 16), dtype=torch.uint8, device=device) if nbytes else None


def linear_fwd(X, qw, A=None, B=None, s: float = 0.0, Y=None, T=None, workspace=None, stream=None):
    """Y = X W^T + s (X A^T) B^T; returns (Y fp32 [m, n], T fp32 [m, rank] or None)."""
    torch = _torch()
    X = _bf16_2d(X, "X")
    m = X.shape[0]
    rank = 0 if A is None else int(A.shape[0])
    if Y is None:
        Y = torch.empty((m, qw.n), dtype=torch.float32, device=X.device)
    if rank > 0 and T is None:
        T = torch.empty((m, rank), dtype=torch.float32, device=X.device)
    mix = isinstance(qw, ChannelMixWeight)
    size_fn = lbq_linear_fwd_mix_workspace_size if mix else lbq_linear_fwd_workspace_size
    nws = size_fn(m, ctypes.byref(qw.struct), rank)
    if workspace is None:
        workspace = _workspace(nws, X.device)
    fn = lbq_linear_fwd_mix if mix else lbq_linear_fwd
    _check(fn(X.data_ptr(), m, ctypes.byref(qw.struct), _ptr(A), _ptr(B), rank, float(s), Y.data_ptr(), _ptr(T),
              _ptr(workspace), nws, _stream(stream)), fn.__name__)
    return Y, T


def linear_fwd_grouped(problems, workspace=None, stream=None):
    """Several forwards with the same token count in one call.  `problems` is a
    list of (X, qw) or (X, qw, A, B, s) tuples; returns the list of Y (and T
    when an adapter is given) as linear_fwd would."""
    torch = _torch()
    arr = (lbq_fwd_problem * len(problems))()
    outs, keep = [], []
    m = None
    for i, pr in enumerate(problems):
        X, qw = _bf16_2d(pr[0], "X"), pr[1]
        A, B, s = (pr[2], pr[3], pr[4]) if len(pr) > 2 else (None, None, 0.0)
        m = X.shape[0] if m is None else m
        if X.shape[0] != m:
            raise ValueError("all problems of a grouped call have the same token count")
        rank = 0 if A is None else int(A.shape[0])
        Y = torch.empty((m, qw.n), dtype=torch.float32, device=X.device)
        T = torch.empty((m, rank), dtype=torch.float32, device=X.device) if rank else None
        arr[i] = lbq_fwd_problem(X=X.data_ptr(), q=ctypes.pointer(qw.struct), A=_ptr(A), B=_ptr(B), rank=rank,
                                 s=float(s), Y=Y.data_ptr(), T_save=_ptr(T))
        outs.append((Y, T))
        keep.append((X, A, B))
    nws = lbq_linear_fwd_grouped_workspace_size(m, arr, len(problems))
    if workspace is None:
        workspace = _workspace(nws, problems[0][0].device)
    _check(lbq_linear_fwd_grouped(m, arr, len(problems), _ptr(workspace), nws, _stream(stream)),
           "lbq_linear_fwd_grouped")
    return outs


def linear_fwd_mix_grouped(problems, workspace=None, stream=None):
    """Several channel-mix forwards with the same token count in one call.
    `problems` is a list of (X, ChannelMixWeight) or (X, ChannelMixWeight, A,
    B, s) tuples; returns the list of (Y, T) as linear_fwd would."""
    torch = _torch()
    arr = (lbq_mix_problem * len(problems))()
    outs, keep = [], []
    m = None
    for i, pr in enumerate(problems):
        X, mw = _bf16_2d(pr[0], "X"), pr[1]
        A, B, s = (pr[2], pr[3], pr[4]) if len(pr) > 2 else (None, None, 0.0)
        m = X.shape[0] if m is None else m
        if X.shape[0] != m:
            raise ValueError("all problems of a grouped call have the same token count")
        rank = 0 if A is None else int(A.shape[0])
        Y = torch.empty((m, mw.n), dtype=torch.float32, device=X.device)
        T = torch.empty((m, rank), dtype=torch.float32, device=X.device) if rank else None
        arr[i] = lbq_mix_problem(X=X.data_ptr(), q=ctypes.pointer(mw.struct), A=_ptr(A), B=_ptr(B), rank=rank,
                                 s=float(s), Y=Y.data_ptr(), T_save=_ptr(T))
        outs.append((Y, T))
        keep.append((X, A, B))
    nws = lbq_linear_fwd_mix_grouped_workspace_size(m, arr, len(problems))
    if workspace is None:
        workspace = _workspace(nws, problems[0][0].device)
    _check(lbq_linear_fwd_mix_grouped(m, arr, len(problems), _ptr(workspace), nws, _stream(stream)),
           "lbq_linear_fwd_mix_grouped")
    return outs


def linear_bwd(dY, qw, A=None, B=None, s: float = 0.0, dX=None, U=None, workspace=None, stream=None):
    """dX = dY W + s (dY B) A; returns (dX fp32 [m, k], U fp32 [m, rank] or None)."""
    torch = _torch()
    dY = _bf16_2d(dY, "dY")
    m = dY.shape[0]
    rank = 0 if A is None else int(A.shape[0])
    if dX is None:
        dX = torch.empty((m, qw.k), dtype=torch.float32, device=dY.device)
    if rank > 0 and U is None:
        U = torch.empty((m, rank), dtype=torch.float32, device=dY.device)
    nws = lbq_linear_bwd_workspace_size(m, ctypes.byref(qw.struct), rank)
    if workspace is None:
        workspace = _workspace(nws, dY.device)
    _check(lbq_linear_bwd(dY.data_ptr(), m, ctypes.byref(qw.struct), _ptr(A), _ptr(B), rank, float(s), dX.data_ptr(),
                          _ptr(U), _ptr(workspace), nws, _stream(stream)), "lbq_linear_bwd")
    return dX, U


def linear_bwd_grouped(problems, workspace=None, stream=None):
    """Several backward passes with the same token count in one call.
    `problems` is a list of (dY, qw) or (dY, qw, A, B, s) tuples; returns the
    list of (dX, U) as linear_bwd would."""
    torch = _torch()
    arr = (lbq_bwd_problem * len(problems))()
    outs, keep = [], []
    m = None
    for i, pr in enumerate(problems):
        dY, qw = _bf16_2d(pr[0], "dY"), pr[1]
        A, B, s = (pr[2], pr[3], pr[4]) if len(pr) > 2 else (None, None, 0.0)
        m = dY.shape[0] if m is None else m
        if dY.shape[0] != m:
            raise ValueError("all problems of a grouped call have the same token count")
        rank = 0 if A is None else int(A.shape[0])
        dX = torch.empty((m, qw.k), dtype=torch.float32, device=dY.device)
        U = torch.empty((m, rank), dtype=torch.float32, device=dY.device) if rank else None
        arr[i] = lbq_bwd_problem(dY=dY.data_ptr(), q=ctypes.pointer(qw.struct), A=_ptr(A), B=_ptr(B), rank=rank,
                                 s=float(s), dX=dX.data_ptr(), U_save=_ptr(U))
        outs.append((dX, U))
        keep.append((dY, A, B))
    nws = lbq_linear_bwd_grouped_workspace_size(m, arr, len(problems))
    if workspace is None:
        workspace = _workspace(nws, problems[0][0].device)
    _check(lbq_linear_bwd_grouped(m, arr, len(problems), _ptr(workspace), nws, _stream(stream)),
           "lbq_linear_bwd_grouped")
    return outs


def lora_grads(X, dY, T, U, s: float, dA=None, dB=None, stream=None):
    """dA = s U^T X [rank, k], dB = s dY^T T [n, rank] (fp32)."""
    torch = _torch()
    X, dY = _bf16_2d(X, "X"), _bf16_2d(dY, "dY")
    m, k = X.shape
    n = dY.shape[1]
    rank = int(T.shape[1])
    if dA is None:
        dA = torch.empty((rank, k), dtype=torch.float32, device=X.device)
    if dB is None:
        dB = torch.empty((n, rank), dtype=torch.float32, device=X.device)
    _check(lbq_lora_grads(X.data_ptr(), dY.data_ptr(), m, n, k, T.data_ptr(), U.data_ptr(), rank, float(s),
                          dA.data_ptr(), dB.data_ptr(), _stream(stream)), "lbq_lora_grads")
    return dA, dB


def merge_lora(qw, A=None, B=None, s: float = 0.0, out=None, stream=None):
    """bf16 [n, k]: the dequantized weight plus s B A (the adapter merged in)."""
    torch = _torch()
    rank = 0 if A is None else int(A.shape[0])
    if rank:
        A, B = _bf16_2d(A, "A"), _bf16_2d(B, "B")
    if out is None:
        out = torch.empty((qw.n, qw.k), dtype=torch.bfloat16, device=qw.packed.device)
    _check(lbq_merge_lora(ctypes.byref(qw.struct), _ptr(A) if rank else None, _ptr(B) if rank else None, rank,
                          float(s), out.data_ptr(), _stream(stream)), "lbq_merge_lora")
    return out


def unmerge_lora(W, A=None, B=None, s: float = 0.0, out=None, stream=None):
    """bf16 [n, k]: W minus s B A (a merged adapter removed); out may be W."""
    torch = _torch()
    W = _bf16_2d(W, "W")
    n, k = W.shape
    rank = 0 if A is None else int(A.shape[0])
    if rank:
        A, B = _bf16_2d(A, "A"), _bf16_2d(B, "B")
    if out is None:
        out = torch.empty_like(W)
    _check(lbq_unmerge_lora(W.data_ptr(), n, k, _ptr(A) if rank else None, _ptr(B) if rank else None, rank,
                            float(s), out.data_ptr(), _stream(stream)), "lbq_unmerge_lora")
    return out


def device_status() -> int:
    """The device status word (timeouts, bad codebooks) since the last read."""
    v = ctypes.c_uint32(0)
    _check(lbq_device_status(ctypes.byref(v)), "lbq_device_status")
    return int(v.value)

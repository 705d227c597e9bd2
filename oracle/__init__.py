"""ctypes wrapper of the CPU oracle (oracle.c).

TEST INFRASTRUCTURE ONLY.  Only the test-suite, the smoke check and the CPU
baseline leg of the benchmark import this package; the product library
(`qlora_quantized_linear_b200`) never does.  It shares no code with the CUDA
path: the only thing both sides use is the seeded input generator module.

Arrays are numpy arrays on the host.  bf16 and fp16 values travel as their
uint16 bit patterns.
"""
from __future__ import annotations

import ctypes
import os

import numpy as np

from .build import build as _build

_LIB = None

_i64 = ctypes.c_int64
_int = ctypes.c_int
_dbl = ctypes.c_double
_vp = ctypes.c_void_p


def use_library(path):
    """Point the wrapper at another build of oracle.c (None: the default one).
    The mutation tests use this to load deliberately broken copies."""
    global _LIB
    _LIB = None if path is None else _load(path)


def _load(path) -> ctypes.CDLL:
    L = ctypes.CDLL(path)
    _declare(L)
    return L


def lib() -> ctypes.CDLL:
    """The oracle library: $LBQ_ORACLE_LIB when set (mutation tests load
    deliberately broken builds this way), else the default build."""
    global _LIB
    if _LIB is None:
        _LIB = _load(os.environ.get("LBQ_ORACLE_LIB") or _build())
    return _LIB


def _declare(L) -> None:
    sig = {
        "oracle_bf16_to_f32": (ctypes.c_float, [ctypes.c_uint16]),
        "oracle_f32_to_f16": (ctypes.c_uint16, [ctypes.c_float]),
        "oracle_f16_to_f32": (ctypes.c_float, [ctypes.c_uint16]),
        "oracle_minmax_quantize": (_int, [_vp, _i64, _i64, _int, _int, _vp, _vp, _vp]),
        "oracle_pack": (_int, [_vp, _i64, _i64, _int, _vp]),
        "oracle_unpack": (_int, [_vp, _i64, _i64, _int, _vp]),
        "oracle_minmax_dequantize": (_int, [_vp, _vp, _vp, _i64, _i64, _int, _int, _vp]),
        "oracle_codebook_quantize": (_int, [_vp, _i64, _i64, _vp, _vp, _vp]),
        "oracle_double_quant": (_int, [_vp, _i64, _vp, _vp, _vp]),
        "oracle_double_dequant": (_int, [_vp, _vp, ctypes.c_float, _i64, _vp]),
        "oracle_codebook_dequantize": (_int, [_vp, _vp, _vp, _i64, _i64, _vp]),
        "oracle_linear_fwd": (_int, [_vp, _i64, _vp, _i64, _i64, _vp, _vp, _int, _dbl, _vp, _vp, _vp]),
        "oracle_linear_bwd": (_int, [_vp, _i64, _vp, _i64, _i64, _vp, _vp, _int, _dbl, _vp, _vp, _vp]),
        "oracle_lora_grads": (_int, [_vp, _vp, _i64, _i64, _i64, _vp, _vp, _int, _dbl, _vp, _vp, _vp, _vp]),
        "oracle_linear_fwd_sampled_minmax": (_int, [_vp, _i64, _vp, _vp, _vp, _i64, _i64, _int, _int,
                                                    _vp, _vp, _int, _dbl, _i64, _vp, _vp, _vp, _vp]),
        "oracle_linear_bwd_sampled_minmax": (_int, [_vp, _i64, _vp, _vp, _vp, _i64, _i64, _int, _int,
                                                    _vp, _vp, _int, _dbl, _i64, _vp, _vp, _vp, _vp]),
        "oracle_lora_merge": (_int, [_vp, _i64, _i64, _vp, _vp, _int, ctypes.c_float, _int, _vp]),
        "oracle_channel_score": (_int, [_vp, _i64, _i64, _vp, _i64, _vp, _vp]),
        "oracle_channel_mix_select": (_int, [_vp, _i64, _i64, _vp]),
        "oracle_set_threads": (None, [_int]),
        "oracle_get_threads": (_int, []),
    }
    for name, (res, args) in sig.items():
        f = getattr(L, name)
        f.restype = res
        f.argtypes = args


def _p(a):
    if a is None:
        return None
    assert a.flags["C_CONTIGUOUS"], "oracle arrays must be C-contiguous"
    return a.ctypes.data


def _check(rc, what):
    if rc != 0:
        raise ValueError(f"oracle {what} rejected its input (code {rc})")


def _u16(a):
    a = np.ascontiguousarray(a)
    assert a.dtype == np.uint16, "bf16/fp16 data must be passed as uint16 bits"
    return a


def set_threads(n: int) -> None:
    lib().oracle_set_threads(int(n))


def get_threads() -> int:
    return int(lib().oracle_get_threads())


# ---------------------------------------------------------------- formats
def bf16_to_f32(bits: np.ndarray) -> np.ndarray:
    b = np.ascontiguousarray(bits, dtype=np.uint16)
    return (b.astype(np.uint32) << 16).view(np.float32)


def f32_to_f16(x: float) -> int:
    return int(lib().oracle_f32_to_f16(float(x)))


def f16_to_f32(h: int) -> float:
    return float(lib().oracle_f16_to_f32(int(h)))


# ---------------------------------------------------------------- MinMax
def minmax_quantize(W: np.ndarray, bits: int, group: int, allow_bad: bool = False):
    """Returns (codes [n,k] u8, scale [n,k/g] fp16 bits, zero [n,k/g] fp16 bits)."""
    W = _u16(W)
    n, k = W.shape
    codes = np.zeros((n, k), np.uint8)
    scale = np.zeros((n, k // group), np.uint16)
    zero = np.zeros((n, k // group), np.uint16)
    rc = lib().oracle_minmax_quantize(_p(W), n, k, bits, group, _p(codes), _p(scale), _p(zero))
    if not (allow_bad and rc == -2):
        _check(rc, "minmax_quantize")
    return codes, scale, zero


def pack(codes: np.ndarray, bits: int) -> np.ndarray:
    codes = np.ascontiguousarray(codes, dtype=np.uint8)
    n, k = codes.shape
    out = np.zeros((n, k * bits // 8), np.uint8)
    _check(lib().oracle_pack(_p(codes), n, k, bits, _p(out)), "pack")
    return out


def unpack(packed: np.ndarray, k: int, bits: int) -> np.ndarray:
    packed = np.ascontiguousarray(packed, dtype=np.uint8)
    n = packed.shape[0]
    out = np.zeros((n, k), np.uint8)
    _check(lib().oracle_unpack(_p(packed), n, k, bits, _p(out)), "unpack")
    return out


def minmax_dequantize(packed, scale, zero, k: int, bits: int, group: int) -> np.ndarray:
    packed = np.ascontiguousarray(packed, dtype=np.uint8)
    scale, zero = _u16(scale), _u16(zero)
    n = packed.shape[0]
    out = np.zeros((n, k), np.float32)
    _check(lib().oracle_minmax_dequantize(_p(packed), _p(scale), _p(zero), n, k, bits, group, _p(out)),
           "minmax_dequantize")
    return out


# ---------------------------------------------------------------- codebook
def codebook_quantize(W: np.ndarray, codebook: np.ndarray):
    """Returns (codes [n,k] u8, absmax [n*k/64] f32)."""
    W = _u16(W)
    n, k = W.shape
    cb = np.ascontiguousarray(codebook, dtype=np.float32)
    codes = np.zeros((n, k), np.uint8)
    absmax = np.zeros(n * k // 64, np.float32)
    _check(lib().oracle_codebook_quantize(_p(W), n, k, _p(cb), _p(codes), _p(absmax)), "codebook_quantize")
    return codes, absmax


def double_quant(absmax: np.ndarray, allow_inexact: bool = False):
    """Returns (q8 [nb] i8, s2 [ceil(nb/256)] f32, offset f32, exact flag)."""
    a = np.ascontiguousarray(absmax, dtype=np.float32)
    nb = a.shape[0]
    q8 = np.zeros(nb, np.int8)
    s2 = np.zeros((nb + 255) // 256, np.float32)
    off = np.zeros(1, np.float32)
    rc = lib().oracle_double_quant(_p(a), nb, _p(q8), _p(s2), _p(off))
    if rc == -2 and allow_inexact:
        return q8, s2, np.float32(off[0]), False
    _check(rc, "double_quant")
    return q8, s2, np.float32(off[0]), True


def double_dequant(q8, s2, offset) -> np.ndarray:
    q8 = np.ascontiguousarray(q8, dtype=np.int8)
    s2 = np.ascontiguousarray(s2, dtype=np.float32)
    out = np.zeros(q8.shape[0], np.float32)
    _check(lib().oracle_double_dequant(_p(q8), _p(s2), ctypes.c_float(float(offset)), q8.shape[0], _p(out)),
           "double_dequant")
    return out


def codebook_dequantize(packed, absmax, codebook, n: int, k: int) -> np.ndarray:
    packed = np.ascontiguousarray(packed, dtype=np.uint8)
    a = np.ascontiguousarray(absmax, dtype=np.float32)
    cb = np.ascontiguousarray(codebook, dtype=np.float32)
    out = np.zeros((n, k), np.float32)
    _check(lib().oracle_codebook_dequantize(_p(packed), _p(a), _p(cb), n, k, _p(out)), "codebook_dequantize")
    return out


# ---------------------------------------------------------------- GEMMs
def linear_fwd(X, W_hat, A=None, B=None, s: float = 0.0):
    """Returns (Y [m,n] f64, T [m,r] f64, Ybound [m,n] f64)."""
    X = _u16(X)
    W_hat = np.ascontiguousarray(W_hat, dtype=np.float32)
    m, k = X.shape
    n = W_hat.shape[0]
    r = 0 if A is None else A.shape[0]
    A = None if A is None else _u16(A)
    B = None if B is None else _u16(B)
    Y = np.zeros((m, n), np.float64)
    T = np.zeros((m, max(r, 1)), np.float64)
    Yb = np.zeros((m, n), np.float64)
    _check(lib().oracle_linear_fwd(_p(X), m, _p(W_hat), n, k, _p(A), _p(B), r, float(s),
                                   _p(Y), _p(T), _p(Yb)), "linear_fwd")
    return Y, T[:, :r], Yb


def linear_bwd(dY, W_hat, A=None, B=None, s: float = 0.0):
    """Returns (dX [m,k] f64, U [m,r] f64, dXbound [m,k] f64)."""
    dY = _u16(dY)
    W_hat = np.ascontiguousarray(W_hat, dtype=np.float32)
    m, n = dY.shape
    k = W_hat.shape[1]
    r = 0 if A is None else A.shape[0]
    A = None if A is None else _u16(A)
    B = None if B is None else _u16(B)
    dX = np.zeros((m, k), np.float64)
    U = np.zeros((m, max(r, 1)), np.float64)
    dXb = np.zeros((m, k), np.float64)
    _check(lib().oracle_linear_bwd(_p(dY), m, _p(W_hat), n, k, _p(A), _p(B), r, float(s),
                                   _p(dX), _p(U), _p(dXb)), "linear_bwd")
    return dX, U[:, :r], dXb


def lora_grads(X, dY, A, B, s: float):
    """Returns (dA [r,k], dB [n,r], dAbound, dBbound), all f64."""
    X, dY, A, B = _u16(X), _u16(dY), _u16(A), _u16(B)
    m, k = X.shape
    n = dY.shape[1]
    r = A.shape[0]
    dA = np.zeros((r, k), np.float64)
    dB = np.zeros((n, r), np.float64)
    dAb = np.zeros((r, k), np.float64)
    dBb = np.zeros((n, r), np.float64)
    _check(lib().oracle_lora_grads(_p(X), _p(dY), m, n, k, _p(A), _p(B), r, float(s),
                                   _p(dA), _p(dB), _p(dAb), _p(dBb)), "lora_grads")
    return dA, dB, dAb, dBb


def linear_fwd_sampled_minmax(X, packed, scale, zero, n: int, k: int, bits: int, group: int,
                              rows, cols, A=None, B=None, s: float = 0.0):
    """Y and its bound at the (rows[i], cols[i]) pairs, from the packed weight."""
    X = _u16(X)
    packed = np.ascontiguousarray(packed, dtype=np.uint8)
    scale, zero = _u16(scale), _u16(zero)
    m = X.shape[0]
    r = 0 if A is None else A.shape[0]
    A = None if A is None else _u16(A)
    B = None if B is None else _u16(B)
    rows = np.ascontiguousarray(rows, dtype=np.int64)
    cols = np.ascontiguousarray(cols, dtype=np.int64)
    Y = np.zeros(rows.shape[0], np.float64)
    Yb = np.zeros(rows.shape[0], np.float64)
    _check(lib().oracle_linear_fwd_sampled_minmax(
        _p(X), m, _p(packed), _p(scale), _p(zero), n, k, bits, group, _p(A), _p(B), r, float(s),
        rows.shape[0], _p(rows), _p(cols), _p(Y), _p(Yb)), "linear_fwd_sampled_minmax")
    return Y, Yb


def linear_bwd_sampled_minmax(dY, packed, scale, zero, n: int, k: int, bits: int, group: int,
                              rows, cols, A=None, B=None, s: float = 0.0):
    """dX and its bound at the (rows[i] = token, cols[i] = feature) pairs, from the packed weight."""
    dY = _u16(dY)
    packed = np.ascontiguousarray(packed, dtype=np.uint8)
    scale, zero = _u16(scale), _u16(zero)
    m = dY.shape[0]
    r = 0 if A is None else A.shape[0]
    A = None if A is None else _u16(A)
    B = None if B is None else _u16(B)
    rows = np.ascontiguousarray(rows, dtype=np.int64)
    cols = np.ascontiguousarray(cols, dtype=np.int64)
    dX = np.zeros(rows.shape[0], np.float64)
    dXb = np.zeros(rows.shape[0], np.float64)
    _check(lib().oracle_linear_bwd_sampled_minmax(
        _p(dY), m, _p(packed), _p(scale), _p(zero), n, k, bits, group, _p(A), _p(B), r, float(s),
        rows.shape[0], _p(rows), _p(cols), _p(dX), _p(dXb)), "linear_bwd_sampled_minmax")
    return dX, dXb


# ---------------------------------------------------------------- adapter merge
def lora_merge(W_in, A, B, s: float, sign: int = 1) -> np.ndarray:
    """bf16 bits [n, k] of W_in + sign * s * (B A), evaluated as oracle.h
    states (fp32 fma over the rank in order, then * s, then +/-, then bf16).
    W_in: fp32 [n, k] (a dequantized weight, or a bf16 weight widened)."""
    W_in = np.ascontiguousarray(W_in, dtype=np.float32)
    n, k = W_in.shape
    r = 0 if A is None else A.shape[0]
    A = None if A is None else _u16(A)
    B = None if B is None else _u16(B)
    out = np.zeros((n, k), np.uint16)
    _check(lib().oracle_lora_merge(_p(W_in), n, k, _p(A), _p(B), r, ctypes.c_float(float(s)), int(sign), _p(out)),
           "lora_merge")
    return out


# ---------------------------------------------------------------- channel-mix selection
def channel_score(W, X):
    """(score [n] f64, bound [n] f64): the rise of channel c's expected
    squared output error from INT4 g128 to INT2 g64, weighted by the
    calibration activations' second moments (oracle.h)."""
    W, X = _u16(W), _u16(X)
    n, k = W.shape
    t = X.shape[0]
    assert X.shape[1] == k
    score = np.zeros(n, np.float64)
    bound = np.zeros(n, np.float64)
    _check(lib().oracle_channel_score(_p(W), n, k, _p(X), t, _p(score), _p(bound)), "channel_score")
    return score, bound


def channel_mix_select(score, n4: int) -> np.ndarray:
    """perm int32 [n]: the n4 highest-scoring channels ascending, then the rest."""
    score = np.ascontiguousarray(score, dtype=np.float64)
    perm = np.zeros(score.size, np.int32)
    _check(lib().oracle_channel_mix_select(_p(score), score.size, int(n4), _p(perm)), "channel_mix_select")
    return perm

"""The C ABI library loads on a machine without a GPU, exports every entry
point that include/lbq.h declares, and rejects bad arguments on the host
before touching the device."""
import ctypes

import pytest

from qlora_quantized_linear_b200 import lbq


def test_exports_every_declared_function():
    names = lbq.header_functions()
    assert len(names) >= 12
    for name in names:
        assert hasattr(lbq._L, name), f"{name} declared in include/lbq.h but not exported"


def test_status_strings():
    for code in range(7):
        assert lbq.lbq_status_string(code)
    assert lbq.lbq_status_string(99) == b"unknown status"


def _qw(**kw):
    q = lbq.lbq_qweight(n=256, k=512, bits=4, group=128, scheme=lbq.LBQ_MINMAX_ASYM, double_quant=0,
                        packed=0x1000, scale=0x2000, zero=0x3000)
    for key, v in kw.items():
        setattr(q, key, v)
    return q


@pytest.mark.parametrize("change,expect", [
    (dict(bits=3), lbq.LBQ_EUNSUPPORTED),
    (dict(bits=4, group=64), lbq.LBQ_EUNSUPPORTED),
    (dict(k=100), lbq.LBQ_EINVAL),
    (dict(n=0), lbq.LBQ_EINVAL),
    (dict(packed=None), lbq.LBQ_EINVAL),
    (dict(packed=0x1008), lbq.LBQ_EALIGN),
    (dict(scheme=7), lbq.LBQ_EUNSUPPORTED),
])
def test_quantize_rejects_bad_descriptors(change, expect):
    q = _qw(**change)
    assert lbq.lbq_quantize(0x4000, ctypes.byref(q), None, 0, None) == expect


def test_linear_fwd_rejects_bad_arguments():
    q = _qw()
    fwd = lbq.lbq_linear_fwd
    assert fwd(0x4000, 0, ctypes.byref(q), None, None, 0, 0.0, 0x5000, None, None, 0, None) == lbq.LBQ_EINVAL
    assert fwd(None, 4, ctypes.byref(q), None, None, 0, 0.0, 0x5000, None, None, 0, None) == lbq.LBQ_EINVAL
    assert fwd(0x4004, 4, ctypes.byref(q), None, None, 0, 0.0, 0x5000, None, None, 0, None) == lbq.LBQ_EALIGN
    # rank > 0 needs A, B and T_save; rank above 64 is rejected
    assert fwd(0x4000, 4, ctypes.byref(q), None, None, 8, 1.0, 0x5000, None, None, 0, None) == lbq.LBQ_EINVAL
    assert fwd(0x4000, 4, ctypes.byref(q), 0x6000, 0x7000, 65, 1.0, 0x5000, 0x8000, None, 0, None) == lbq.LBQ_EINVAL
    assert fwd(0x4000, 4, None, None, None, 0, 0.0, 0x5000, None, None, 0, None) == lbq.LBQ_EINVAL


def test_bwd_and_grads_reject_bad_arguments():
    q = _qw()
    bwd = lbq.lbq_linear_bwd
    # codebook weights take the backward too; their arguments are checked the same way
    cb = _qw(scheme=lbq.LBQ_CODEBOOK4, group=64, absmax=0x9000, codebook=0xA000, n=250)
    assert bwd(0x4000, 4, ctypes.byref(cb), None, None, 0, 0.0, 0x5000, None, None, 0, None) == lbq.LBQ_EINVAL
    cb = _qw(scheme=lbq.LBQ_CODEBOOK4, group=64, absmax=0x9008, codebook=0xA000)
    assert bwd(0x4000, 4, ctypes.byref(cb), None, None, 0, 0.0, 0x5000, None, None, 0, None) == lbq.LBQ_EALIGN
    cb = _qw(scheme=lbq.LBQ_CODEBOOK4, group=64, absmax=0x9000, codebook=None)
    assert bwd(0x4000, 4, ctypes.byref(cb), None, None, 0, 0.0, 0x5000, None, None, 0, None) == lbq.LBQ_EINVAL
    q2 = _qw(n=250)
    assert bwd(0x4000, 4, ctypes.byref(q2), None, None, 0, 0.0, 0x5000, None, None, 0, None) == lbq.LBQ_EINVAL
    g = lbq.lbq_lora_grads
    assert g(0x4000, 0x5000, 4, 256, 512, 0x6000, 0x7000, 0, 1.0, 0x8000, 0x9000, None) == lbq.LBQ_EINVAL
    assert g(0x4000, 0x5000, 4, 255, 512, 0x6000, 0x7000, 8, 1.0, 0x8000, 0x9000, None) == lbq.LBQ_EINVAL
    assert g(0x4002, 0x5000, 4, 256, 512, 0x6000, 0x7000, 8, 1.0, 0x8000, 0x9000, None) == lbq.LBQ_EALIGN


def test_workspace_queries_are_host_only():
    q = _qw()
    assert lbq.lbq_linear_fwd_workspace_size(0, ctypes.byref(q), 0) == 0
    assert lbq.lbq_quantize_workspace_size(ctypes.byref(q)) == 0
    cb = _qw(scheme=lbq.LBQ_CODEBOOK4, group=64, double_quant=1)
    assert lbq.lbq_quantize_workspace_size(ctypes.byref(cb)) > 0


def test_merge_entry_points_reject_bad_arguments():
    q = _qw()
    merge, unmerge = lbq.lbq_merge_lora, lbq.lbq_unmerge_lora
    assert merge(None, None, None, 0, 1.0, 0x5000, None) == lbq.LBQ_EINVAL
    assert merge(ctypes.byref(q), None, None, 0, 1.0, None, None) == lbq.LBQ_EINVAL
    assert merge(ctypes.byref(q), None, None, 8, 1.0, 0x5000, None) == lbq.LBQ_EINVAL      # rank > 0 needs A, B
    assert merge(ctypes.byref(q), 0x6000, 0x7000, 65, 1.0, 0x5000, None) == lbq.LBQ_EINVAL  # rank above 64
    assert merge(ctypes.byref(q), 0x6000, 0x7000, 8, 1.0, 0x5004, None) == lbq.LBQ_EALIGN
    assert merge(ctypes.byref(q), 0x6008, 0x7000, 8, 1.0, 0x5000, None) == lbq.LBQ_EALIGN
    assert unmerge(0x4000, 16, 12, None, None, 0, 1.0, 0x5000, None) == lbq.LBQ_EINVAL     # k % 8 != 0
    assert unmerge(0x4000, 0, 16, None, None, 0, 1.0, 0x5000, None) == lbq.LBQ_EINVAL
    assert unmerge(0x4002, 16, 16, None, None, 0, 1.0, 0x5000, None) == lbq.LBQ_EALIGN


def test_grouped_entry_points_reject_bad_arguments():
    q = _qw()
    P = (lbq.lbq_fwd_problem * 2)()
    for i in range(2):
        P[i] = lbq.lbq_fwd_problem(X=0x4000, q=ctypes.pointer(q), A=None, B=None, rank=0, s=0.0, Y=0x5000, T_save=None)
    g = lbq.lbq_linear_fwd_grouped
    assert g(4, P, 0, None, 0, None) == lbq.LBQ_EINVAL
    assert g(4, None, 2, None, 0, None) == lbq.LBQ_EINVAL
    assert g(0, P, 2, None, 0, None) == lbq.LBQ_EINVAL
    P[1].Y = 0x5004
    assert g(4, P, 2, None, 0, None) == lbq.LBQ_EALIGN
    P[1].Y = 0x5000
    P[1].rank = 8                                              # rank > 0 needs A, B and T_save
    assert g(4, P, 2, None, 0, None) == lbq.LBQ_EINVAL

    hi, lo = _qw(n=64), _qw(n=192, bits=2, group=64)
    mix = lbq.lbq_qweight_mix(hi=hi, lo=lo, perm=0xB000)
    M = (lbq.lbq_mix_problem * 2)()
    for i in range(2):
        M[i] = lbq.lbq_mix_problem(X=0x4000, q=ctypes.pointer(mix), A=None, B=None, rank=0, s=0.0, Y=0x5000,
                                   T_save=None)
    gm = lbq.lbq_linear_fwd_mix_grouped
    assert gm(4, M, 0, None, 0, None) == lbq.LBQ_EINVAL
    assert gm(4, None, 2, None, 0, None) == lbq.LBQ_EINVAL
    M[1].Y = 0x5008
    assert gm(4, M, 2, None, 0, None) == lbq.LBQ_EALIGN
    M[1].Y = 0x5000
    bad = lbq.lbq_qweight_mix(hi=hi, lo=_qw(n=192, k=1024, bits=2, group=64), perm=0xB000)   # halves differ in k
    M[1].q = ctypes.pointer(bad)
    assert gm(4, M, 2, None, 0, None) == lbq.LBQ_EINVAL
    cbm = lbq.lbq_qweight_mix(hi=hi, lo=_qw(n=192, scheme=lbq.LBQ_CODEBOOK4, group=64, absmax=0x9000, codebook=0xA000),
                              perm=0xB000)                      # halves are MinMax only
    M[1].q = ctypes.pointer(cbm)
    assert gm(4, M, 2, None, 0, None) == lbq.LBQ_EINVAL
    nop = lbq.lbq_qweight_mix(hi=hi, lo=lo, perm=None)
    M[1].q = ctypes.pointer(nop)
    assert gm(4, M, 2, None, 0, None) == lbq.LBQ_EINVAL
    # the grouped backward: the same checks as lbq_linear_bwd, before any launch
    D = (lbq.lbq_bwd_problem * 2)()
    for i in range(2):
        D[i] = lbq.lbq_bwd_problem(dY=0x4000, q=ctypes.pointer(q), A=None, B=None, rank=0, s=0.0, dX=0x5000,
                                   U_save=None)
    gb = lbq.lbq_linear_bwd_grouped
    assert gb(4, D, 0, None, 0, None) == lbq.LBQ_EINVAL
    assert gb(4, None, 2, None, 0, None) == lbq.LBQ_EINVAL
    assert gb(0, D, 2, None, 0, None) == lbq.LBQ_EINVAL
    D[1].dX = 0x5004
    assert gb(4, D, 2, None, 0, None) == lbq.LBQ_EALIGN
    D[1].dX = 0x5000
    D[1].rank = 8                                              # rank > 0 needs A, B and U_save
    assert gb(4, D, 2, None, 0, None) == lbq.LBQ_EINVAL
    D[1].rank = 0
    odd = _qw(n=100)                                           # n must be a multiple of 8
    D[1].q = ctypes.pointer(odd)
    assert gb(4, D, 2, None, 0, None) == lbq.LBQ_EINVAL
    D[1].q = ctypes.pointer(q)
    assert lbq.lbq_linear_bwd_grouped_workspace_size(0, D, 2) == 0
    # the workspace queries are host-only and cover both halves of every problem
    M[1].q = ctypes.pointer(mix)
    assert lbq.lbq_linear_fwd_mix_grouped_workspace_size(0, M, 2) == 0
    assert lbq.lbq_linear_fwd_mix_grouped_workspace_size(4, M, 2) % 256 == 0

"""The allocation-free forward entry point (lbq_linear_fwd_noalloc).

Some callers cannot allocate device memory -- their memory is all owned by
another runtime's pool, or they run in a loop that must not allocate (or
synchronize, as cudaMalloc may) after start-up.  For them the library offers
a forward call without a workspace argument: its split-K scratch is a fixed
8 MiB device array inside the library.  This file checks, through the C ABI,
that the call gives the same result as lbq_linear_fwd with a caller-supplied
workspace, within the parity bound used by the other tests, on two calls in a
row (the second one meets the array as the first one left it), and that a
call whose scratch would not fit is refused before anything is launched.

The file name makes pytest collect it last.
"""
import ctypes

import numpy as np
import pytest
import torch

import oracle
from qlora_quantized_linear_b200 import synthetic as syn

pytestmark = pytest.mark.gpu

TOL_REL, TOL_ABS = 2.0 ** -7, 1e-6


def _within(got, ref, bound):
    err = np.abs(np.asarray(got, np.float64) - np.asarray(ref, np.float64))
    return bool(np.all(err <= TOL_REL * bound + TOL_ABS))


@pytest.mark.parametrize("m,n,k,rank", [(16, 1024, 4096, 16), (1, 4096, 4096, 0)])
def test_noalloc_matches_workspace_entry_point(m, n, k, rank):
    from qlora_quantized_linear_b200 import lbq
    s = 2.0
    W = syn.weight_bf16(n, k, 0.02, seed=n + k, outlier_frac=0.001)
    X = syn.normal_bf16((m, k), 1.0, seed=m + 11)
    A = syn.normal_bf16((rank, k), 0.01, seed=3) if rank else None
    B = syn.normal_bf16((n, rank), 0.01, seed=4) if rank else None
    qw = lbq.QuantizedWeight(n, k, "minmax", 4).quantize(W.cuda())
    Xd = X.cuda()
    Ad = None if A is None else A.cuda()
    Bd = None if B is None else B.cuda()
    nws = lbq.lbq_linear_fwd_workspace_size(m, ctypes.byref(qw.struct), rank)
    assert nws > 0, "the case must exercise the split-K scratch"
    Y_ws, _ = lbq.linear_fwd(Xd, qw, Ad, Bd, s)

    stream = torch.cuda.current_stream().cuda_stream
    Yb = oracle.linear_fwd(syn.bits_u16(X), qw.dequantize().cpu().numpy(),
                           None if A is None else syn.bits_u16(A), None if B is None else syn.bits_u16(B), s)[2]
    for _ in range(2):
        Y = torch.full((m, n), float("nan"), dtype=torch.float32, device="cuda")
        T = torch.empty((m, max(rank, 1)), dtype=torch.float32, device="cuda")
        rc = lbq.lbq_linear_fwd_noalloc(Xd.data_ptr(), m, ctypes.byref(qw.struct),
                                        None if Ad is None else Ad.data_ptr(),
                                        None if Bd is None else Bd.data_ptr(), rank, s, Y.data_ptr(),
                                        T.data_ptr() if rank else None, stream)
        assert rc == lbq.LBQ_OK, lbq.lbq_status_string(rc)
        torch.cuda.synchronize()
        assert _within(Y.cpu().numpy(), Y_ws.cpu().numpy(), Yb)
    assert lbq.device_status() == 0


def test_noalloc_refuses_scratch_beyond_its_array():
    from qlora_quantized_linear_b200 import lbq
    # 16 tokens x 65536 rows x 16384: the 131072 (row tile, k-block) work units
    # are shared among thousands of CTAs, and their fp32 partials (16 x 128
    # values per CTA) take far more than 8 MiB
    m, n, k = 16, 65536, 16384
    q = lbq.lbq_qweight(n=n, k=k, bits=4, group=128, scheme=lbq.LBQ_MINMAX_ASYM, double_quant=0,
                        packed=0x1000, scale=0x2000, zero=0x3000)
    need = lbq.lbq_linear_fwd_workspace_size(m, ctypes.byref(q), 0)
    assert need > (8 << 20)
    rc = lbq.lbq_linear_fwd_noalloc(0x4000, m, ctypes.byref(q), None, None, 0, 0.0, 0x5000, None, None)
    assert rc == lbq.LBQ_EWORKSPACE

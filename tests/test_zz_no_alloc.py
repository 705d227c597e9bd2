"""The allocation-free forward entry point (lbq_linear_fwd_noalloc).

Some callers cannot allocate device memory -- their memory is all owned by
another runtime's pool, or they run in a loop that must not allocate (or
synchronize, as cudaMalloc may) after start-up.  For them the library offers
a forward call without a workspace argument: its split-K scratch is a fixed
8 MiB device array inside the library.  This file checks, through the C ABI,
on two calls in a row (the second one meets the array as the first one left
it), that the call
  * agrees with the oracle within the parity bound used by the other tests,
    on weights quantized by the oracle, and
  * gives bit for bit the result of lbq_linear_fwd with a caller-supplied
    workspace (both run the same kernels with a fixed summation order),
on the decode GEMV path (m <= 16) and on the tensor-core path when it splits
K (m = 32), and that a call whose scratch would not fit is refused before
anything is launched.

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


@pytest.mark.parametrize("m,n,k,rank", [(16, 1024, 4096, 16), (1, 4096, 4096, 0), (32, 1024, 4096, 8)])
def test_noalloc_matches_oracle_and_workspace_entry_point(m, n, k, rank):
    from qlora_quantized_linear_b200 import lbq
    s = 2.0
    W = syn.weight_bf16(n, k, 0.02, seed=n + k, outlier_frac=0.001)
    X = syn.normal_bf16((m, k), 1.0, seed=m + 11)
    A = syn.normal_bf16((rank, k), 0.01, seed=3) if rank else None
    B = syn.normal_bf16((n, rank), 0.01, seed=4) if rank else None
    codes, scale, zero = oracle.minmax_quantize(syn.bits_u16(W), 4, 128)
    packed = oracle.pack(codes, 4)
    qw = lbq.QuantizedWeight(n, k, "minmax", 4)
    qw.packed.copy_(torch.from_numpy(packed))
    qw.scale.copy_(torch.from_numpy(scale.view(np.float16)))
    qw.zero.copy_(torch.from_numpy(zero.view(np.float16)))
    Xd = X.cuda()
    Ad = None if A is None else A.cuda()
    Bd = None if B is None else B.cuda()
    nws = lbq.lbq_linear_fwd_workspace_size(m, ctypes.byref(qw.struct), rank)
    assert 0 < nws <= (8 << 20), "the case must exercise the split-K scratch and fit the array"
    Y_ws, _ = lbq.linear_fwd(Xd, qw, Ad, Bd, s)

    What = oracle.minmax_dequantize(packed, scale, zero, k, 4, 128)
    Yr, _, Yb = oracle.linear_fwd(syn.bits_u16(X), What, None if A is None else syn.bits_u16(A),
                                  None if B is None else syn.bits_u16(B), s)
    stream = torch.cuda.current_stream().cuda_stream
    for _ in range(2):
        Y = torch.full((m, n), float("nan"), dtype=torch.float32, device="cuda")
        T = torch.empty((m, max(rank, 1)), dtype=torch.float32, device="cuda")
        rc = lbq.lbq_linear_fwd_noalloc(Xd.data_ptr(), m, ctypes.byref(qw.struct),
                                        None if Ad is None else Ad.data_ptr(),
                                        None if Bd is None else Bd.data_ptr(), rank, s, Y.data_ptr(),
                                        T.data_ptr() if rank else None, stream)
        assert rc == lbq.LBQ_OK, lbq.lbq_status_string(rc)
        torch.cuda.synchronize()
        assert _within(Y.cpu().numpy(), Yr, Yb), "outside the parity bound against the oracle"
        assert torch.equal(Y, Y_ws), "differs from lbq_linear_fwd with a caller workspace"
    assert lbq.device_status() == 0


def test_noalloc_reset_then_call():
    """The reset entry point zeroes the array's counters; a call after it is
    still exact."""
    from qlora_quantized_linear_b200 import lbq
    m, n, k = 4, 2048, 4096
    W = syn.weight_bf16(n, k, 0.02, seed=5)
    X = syn.normal_bf16((m, k), 1.0, seed=6)
    qw = lbq.QuantizedWeight(n, k, "minmax", 4).quantize(W.cuda())
    stream = torch.cuda.current_stream().cuda_stream
    assert lbq.lbq_linear_fwd_noalloc_reset(stream) == lbq.LBQ_OK
    Y = torch.empty((m, n), dtype=torch.float32, device="cuda")
    Xd = X.cuda()
    assert lbq.lbq_linear_fwd_noalloc(Xd.data_ptr(), m, ctypes.byref(qw.struct), None, None, 0, 0.0, Y.data_ptr(),
                                      None, stream) == lbq.LBQ_OK
    Y_ws, _ = lbq.linear_fwd(Xd, qw)
    torch.cuda.synchronize()
    assert torch.equal(Y, Y_ws)
    assert lbq.device_status() == 0


def test_noalloc_refuses_scratch_beyond_its_array():
    from qlora_quantized_linear_b200 import lbq
    # 16 tokens x 262144 rows x 4096: 2048 row tiles whose CTA shares do not
    # end on tile boundaries; the fp32 partials (16 x 128 values per CTA and
    # per tile) take about 19 MB, more than the 8 MiB array
    m, n, k = 16, 262144, 4096
    q = lbq.lbq_qweight(n=n, k=k, bits=4, group=128, scheme=lbq.LBQ_MINMAX_ASYM, double_quant=0,
                        packed=0x1000, scale=0x2000, zero=0x3000)
    need = lbq.lbq_linear_fwd_workspace_size(m, ctypes.byref(q), 0)
    assert need > (8 << 20)
    rc = lbq.lbq_linear_fwd_noalloc(0x4000, m, ctypes.byref(q), None, None, 0, 0.0, 0x5000, None, None)
    assert rc == lbq.LBQ_EWORKSPACE

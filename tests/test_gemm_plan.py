"""Host logic of the tensor-core GEMMs' plan (no GPU needed).

For m > 16 (forward) and for every m (backward) the plan cuts the output
into 128-row (forward) or 128-feature (backward) tiles x token tiles of up to
256, numbered output tile fastest, and decides the K splits:

* fewer tiles than the GPU's CTA slots (148 at the 256-token tile, 296
  below it): every tile's reduction is split so that all CTAs fit one wave;
* several waves whose last holds a quarter to a half of the slots: the
  full waves run unsplit and the last wave's tiles are split over the idle
  slots (optional: it needs workspace for their partial sums);
* otherwise no split and no workspace.

The size queries report the workspace of that plan: a 64 KiB header of
arrival counters plus fp32 partial sums [split tile][split][token tile][128].
These tests rebuild the expected sizes from those rules (148 SMs, the count
the queries assume without a GPU and the B200's)."""
import ctypes

import pytest

from qlora_quantized_linear_b200 import lbq

SMS = 148
HEADER = 64 * 1024


def qw(n, k, bits=4, scheme=None, dq=False):
    if scheme == "codebook":
        return lbq.lbq_qweight(n=n, k=k, bits=4, group=64, scheme=lbq.LBQ_CODEBOOK4, double_quant=int(dq))
    return lbq.lbq_qweight(n=n, k=k, bits=bits, group=128 if bits == 4 else 64, scheme=lbq.LBQ_MINMAX_ASYM)


def cdiv(a, b):
    return -(-a // b)


def round256(x):
    return cdiv(x, 256) * 256


def expected(m, out_rows, red_blocks, align):
    """Workspace bytes of the plan the rules above give."""
    nt = 16 if m <= 16 else 32 if m <= 32 else 64 if m <= 64 else 128 if m <= 128 else 256
    tiles = cdiv(out_rows, 128) * cdiv(m, nt)
    slots = (1 if nt >= 256 else 2) * SMS

    def per_for(ns):
        return cdiv(cdiv(red_blocks, ns), align) * align

    if tiles < slots:
        ns = cdiv(red_blocks, per_for(min(red_blocks, max(1, slots // tiles))))
        return HEADER + round256(tiles * ns * nt * 128 * 4) if ns > 1 else 0
    tail = tiles - tiles // slots * slots
    if 2 * tail > slots or 4 * tail < slots:
        return 0
    ns = cdiv(red_blocks, per_for(slots // tail))
    return HEADER + round256(tail * ns * nt * 128 * 4) if ns > 1 else 0


def fwd_ws(m, q):
    return lbq.lbq_linear_fwd_workspace_size(m, ctypes.byref(q), 0)


def bwd_ws(m, q):
    return lbq.lbq_linear_bwd_workspace_size(m, ctypes.byref(q), 0)


@pytest.mark.parametrize("n,k", [(14336, 4096), (4096, 14336), (4096, 4096), (1024, 4096), (11904, 1024)])
@pytest.mark.parametrize("m", [17, 32, 100, 300, 512, 2048, 4096])
@pytest.mark.parametrize("bits", [4, 2])
def test_forward_plan_sizes(n, k, m, bits):
    assert fwd_ws(m, qw(n, k, bits)) == expected(m, n, k // 64, 8 if bits == 2 else 4)


@pytest.mark.parametrize("n,k", [(14336, 4096), (4096, 14336), (256, 11904), (1024, 4096)])
@pytest.mark.parametrize("m", [1, 16, 32, 300, 4096])
def test_backward_plan_sizes(n, k, m):
    assert bwd_ws(m, qw(n, k)) == expected(m, k, cdiv(n, 64), 1)


def test_llama_shapes_at_4096():
    """The 8B MLP at M = 4096: gate and up forward (1792 tiles, a last wave
    of 16) need no split; the down forward and the gate/up backward (512
    tiles, 68 in the last wave) split it in two; the down backward (1792)
    does not."""
    gate, down = qw(14336, 4096), qw(4096, 14336)
    assert fwd_ws(4096, gate) == 0
    assert fwd_ws(4096, down) == HEADER + 68 * 2 * 256 * 128 * 4
    assert bwd_ws(4096, gate) == HEADER + 68 * 2 * 256 * 128 * 4
    assert bwd_ws(4096, down) == 0


def test_full_waves_need_nothing():
    """Tiles that fill whole waves are never split."""
    assert fwd_ws(256, qw(148 * 128, 1024)) == 0
    assert fwd_ws(512, qw(148 * 128, 1024)) == 0
    assert bwd_ws(256, qw(512, 148 * 128)) == 0


def test_codebook_and_grouped_queries():
    """The codebook format splits like 4-bit MinMax (on whole weight chunks of
    4 k-blocks; INT2 on chunks of 8), and the grouped queries report the
    largest of their problems' sizes."""
    cb = qw(4096, 14336, scheme="codebook", dq=True)
    assert fwd_ws(4096, cb) == fwd_ws(4096, qw(4096, 14336))
    probs = (lbq.lbq_bwd_problem * 2)()
    qs = [qw(14336, 4096), qw(4096, 14336)]
    for i in range(2):
        probs[i] = lbq.lbq_bwd_problem(dY=None, q=ctypes.pointer(qs[i]), A=None, B=None, rank=0, s=0.0, dX=None,
                                       U_save=None)
    assert lbq.lbq_linear_bwd_grouped_workspace_size(4096, probs, 2) == max(bwd_ws(4096, q) for q in qs)

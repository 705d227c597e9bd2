"""Host logic of the decode GEMV's stream-K plan (no GPU needed).

lbq_gemv_plan returns the plan that lbq_linear_fwd launches for m <= 16.
These tests rebuild every CTA's work from it with the decomposition that the
kernel uses (equal contiguous shares of the row-tile x k-block units; a share
is split at a tile boundary into at most two segments) and check what the
kernel relies on:

* every unit is covered exactly once;
* a split tile is finished by the CTA that covers its last k-block, which is
  the highest CTA index of the tile, and its contributors are the CTAs just
  below it;
* a CTA processes its tile-starting segment (where it is a contributor) first,
  so no CTA waits before it has published, and no chain of waits forms;
* partial-sum slots (CTA + tile) are distinct, and the workspace holds them;
* shared memory fits two CTAs per SM, the constant table fits, and the
  benchmark's layer shapes run in one wave.
"""
import ctypes
import itertools

import pytest

from qlora_quantized_linear_b200 import lbq

SMS = 148


def qweight(n, k, scheme="minmax", bits=4):
    if scheme == "minmax":
        return lbq.lbq_qweight(n=n, k=k, bits=bits, group=128 if bits == 4 else 64, scheme=lbq.LBQ_MINMAX_ASYM)
    return lbq.lbq_qweight(n=n, k=k, bits=4, group=64, scheme=lbq.LBQ_CODEBOOK4)


def plan(m, n, k, scheme="minmax", bits=4, sms=SMS):
    q = qweight(n, k, scheme, bits)
    out = (ctypes.c_int64 * 6)()
    assert lbq.lbq_gemv_plan(m, ctypes.byref(q), sms, out) == lbq.LBQ_OK
    return dict(grid=out[0], share=out[1], tiles=out[2], stages=out[3], smem=out[4], sms=out[5],
                kbt=k // 64, gb=2 if (scheme == "minmax" and bits == 4) else 1, q=q)


def segments(b, P):
    """(tile, first k-block, k-blocks) of CTA b, in the order the kernel
    processes them (the segment that starts a tile first)."""
    kbt, share = P["kbt"], P["share"]
    total = P["tiles"] * kbt
    u0 = b * share
    u1 = min(u0 + share, total)
    if u0 >= u1:
        return []
    t0 = u0 // kbt
    a0 = u0 - t0 * kbt
    n0 = min(u1 - u0, kbt - a0)
    n1 = (u1 - u0) - n0
    segs = [(t0, a0, n0)]
    if n1:
        segs.append((t0 + 1, 0, n1))
    return list(reversed(segs))


def check_plan(m, n, k, scheme="minmax", bits=4):
    P = plan(m, n, k, scheme, bits)
    kbt, share, tiles, gb = P["kbt"], P["share"], P["tiles"], P["gb"]
    assert P["sms"] == SMS and tiles == -(-n // 128)
    assert share % gb == 0 and gb <= share <= kbt
    assert share // gb <= 32                                   # constant-table groups per CTA
    assert P["grid"] == -(-(tiles * kbt) // share)
    assert P["stages"] in (3, 4)
    assert P["smem"] <= 113 * 1024                            # two CTAs per SM
    owner_of, ctas_of, covered, slots = {}, {}, set(), set()
    for b in range(P["grid"]):
        segs = segments(b, P)
        assert 1 <= len(segs) <= 2
        seen_owner = False
        for (t, a, cnt) in segs:
            assert 0 <= t < tiles and 0 <= a and cnt > 0 and a + cnt <= kbt
            assert a % gb == 0 and cnt % gb == 0                # whole scale groups
            for u in range(a, a + cnt):
                assert (t, u) not in covered
                covered.add((t, u))
            ctas_of.setdefault(t, []).append(b)
            full = a == 0 and cnt == kbt
            if full:
                continue
            slots.add(b + t)
            if a + cnt == kbt:
                assert t not in owner_of
                owner_of[t] = b
                seen_owner = True
            else:
                assert not seen_owner, f"CTA {b} would publish after waiting"
    assert len(covered) == tiles * kbt
    for t, bs in ctas_of.items():
        assert bs == list(range(bs[0], bs[-1] + 1))            # contiguous CTA range
        if len(bs) > 1:
            assert owner_of[t] == bs[-1]                         # the highest index finishes
    assert len(slots) == len({(b, t) for t, bs in ctas_of.items() if len(bs) > 1 for b in bs})
    assert all(s < P["grid"] + tiles for s in slots)
    ws = lbq.lbq_linear_fwd_workspace_size(m, ctypes.byref(P["q"]), 0)
    if P["grid"] > 1:
        assert ws >= 64 * 1024 + (P["grid"] + tiles) * m * 128 * 4
    return P


SHAPES_8B = [(4096, 4096), (1024, 4096), (14336, 4096), (4096, 14336)]
SHAPES_70B = [(8192, 8192), (28672, 8192), (8192, 28672)]


@pytest.mark.parametrize("m", [1, 8, 9, 16])
@pytest.mark.parametrize("n,k", SHAPES_8B + SHAPES_70B)
@pytest.mark.parametrize("scheme,bits", [("minmax", 4), ("minmax", 2), ("codebook", 4)])
def test_plan_layer_shapes(m, n, k, scheme, bits):
    check_plan(m, n, k, scheme, bits)


@pytest.mark.parametrize("m,n,k", list(itertools.product([1, 7, 16], [128, 200, 384, 1000, 2000], [128, 640, 3200])))
def test_plan_ragged_shapes(m, n, k):
    check_plan(m, n, k, "minmax", 4)
    check_plan(m, n, k, "codebook", 4)


@pytest.mark.parametrize("m", [1, 16])
def test_8b_layer_set_runs_in_one_wave(m):
    for n, k in SHAPES_8B:
        P = check_plan(m, n, k)
        assert P["grid"] <= 2 * SMS, (n, k, P)


def test_wide_token_tile_takes_three_boxes_for_one_wave():
    # at m = 16 the activation slice crowds the shared memory: the MLP shapes
    # drop to a three-box ring so that the grid still fits one wave
    for n, k in [(14336, 4096), (4096, 14336)]:
        assert plan(16, n, k)["stages"] == 3
    assert plan(1, 14336, 4096)["stages"] == 4


def test_plan_rejects_bad_arguments():
    q = qweight(256, 512)
    out = (ctypes.c_int64 * 6)()
    assert lbq.lbq_gemv_plan(0, ctypes.byref(q), SMS, out) == lbq.LBQ_EINVAL
    assert lbq.lbq_gemv_plan(17, ctypes.byref(q), SMS, out) == lbq.LBQ_EINVAL
    assert lbq.lbq_gemv_plan(1, ctypes.byref(q), SMS, None) == lbq.LBQ_EINVAL
    bad = qweight(256, 500)
    assert lbq.lbq_gemv_plan(1, ctypes.byref(bad), SMS, out) == lbq.LBQ_EINVAL

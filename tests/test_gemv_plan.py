"""Host logic of the grouped decode GEMV's plan (no GPU needed).

lbq_gemv_plan returns the plan that the forward launches for m <= 16 over a
group of up to 8 weights.  These tests rebuild every CTA's work from it with
the decomposition the kernel uses (equal contiguous shares of one weight's
row-tile x k-block units, cut at tile boundaries into segments, processed
last tile first, then the whole tiles, then the first tile) and check what
the kernel relies on:

* the launch is one wave of two CTAs per SM, and its shared memory (ring of
  stages, each a weight box and an activation box, the compute warps'
  constant buffers and the fixed tail) fits two CTAs per SM;
* every unit of every weight is covered exactly once, and CTAs of one weight
  are contiguous in the grid;
* a split tile is finished by the CTA that covers its last k-block, which is
  the highest CTA index of the tile; that CTA processes it last, and every
  contributor processes its contribution first (so no CTA waits before it has
  published, and no chain of waits forms);
* partial-sum slots (CTA + tile) are distinct and inside the weight's
  partial region; the workspace holds the counter header and all regions and
  is zero exactly when no tile is split;
* boxes start on whole scale groups, the activation rows and constant rows
  of a stage hold what a box needs, and every CTA gets about the same bytes.
"""
import ctypes

import pytest

from qlora_quantized_linear_b200 import lbq

SMS = 148
BUDGET = 115712 - 1024           # dynamic shared memory per CTA at two CTAs per SM (beside 1 KB static)
EXTRA = 2 * 4 * 8 + 16 + 2 * 256 * 4
XCHG = 4 * 32 * 4 * 4                 # the two k-halves' exchange buffer (up to 8 tokens)
HEADER = 64 * 1024
SHAPES_8B = [(4096, 4096), (1024, 4096), (1024, 4096), (4096, 4096), (14336, 4096), (14336, 4096), (4096, 14336)]


def qweight(n, k, scheme="minmax", bits=4, dq=False):
    if scheme == "minmax":
        return lbq.lbq_qweight(n=n, k=k, bits=bits, group=128 if bits == 4 else 64, scheme=lbq.LBQ_MINMAX_ASYM)
    return lbq.lbq_qweight(n=n, k=k, bits=4, group=64, scheme=lbq.LBQ_CODEBOOK4, double_quant=int(dq))


def plan(m, qs, sms=SMS):
    arr = (ctypes.POINTER(lbq.lbq_qweight) * len(qs))(*[ctypes.pointer(q) for q in qs])
    out = (ctypes.c_int64 * 8)()
    per = (ctypes.c_int64 * (4 * len(qs)))()
    rc = lbq.lbq_gemv_plan(m, arr, len(qs), sms, out, per)
    assert rc == lbq.LBQ_OK, rc
    P = dict(ctas=out[0], ws=out[1], stage=out[2], smem=out[3], workspace=out[4], sms=out[5], xbox=out[6],
             cstride=out[7], probs=[])
    for i, q in enumerate(qs):
        kind = 2 if q.scheme == lbq.LBQ_CODEBOOK4 else (0 if q.bits == 4 else 1)
        P["probs"].append(dict(share=per[4 * i], ctas=per[4 * i + 1], cta0=per[4 * i + 2], tiles=per[4 * i + 3],
                               kbt=q.k // 64, n=q.n, k=q.k, kind=kind, dq=bool(q.double_quant),
                               gb=2 if kind == 0 else 1, sub=8 if kind == 1 else 4, bits=q.bits))
    return P


def segments(b, pr):
    """(tile, ka, kb) of CTA b of one weight, in processing order."""
    kbt, share = pr["kbt"], pr["share"]
    total = pr["tiles"] * kbt
    u0 = b * share
    u1 = min(u0 + share, total)
    if u0 >= u1:
        return []
    tA, tB = u0 // kbt, (u1 - 1) // kbt
    nseg = tB - tA + 1
    out = []
    for si in range(nseg):
        t = tA if nseg == 1 else (tB if si == 0 else (tA if si == nseg - 1 else tA + si))
        ka = u0 - tA * kbt if t == tA else 0
        kb = u1 - tB * kbt if t == tB else kbt
        out.append((t, ka, kb))
    return out


def unit_bytes(pr):
    codes = 128 * 64 * pr["bits"] / 8
    if pr["kind"] != 2:
        return codes + 128 * 4 * 64 / (128 if pr["bits"] == 4 else 64)
    return codes + 128 * (1 if pr["dq"] else 4)


def check(m, qs):
    P = plan(m, qs)
    assert P["sms"] == SMS
    assert P["ctas"] <= 2 * SMS, "more than one wave"
    assert 2 <= P["ws"] <= 4
    assert P["stage"] % 1024 == 0
    # stage: weight box, activation box (k-blocks of the box x tokens padded to
    # the MMA's 8 or 16 x 128 bytes); then every compute warp's constant
    # double buffer (2 slots x 2 arrays x its 32 or 16 rows)
    sub_max = max(pr["sub"] for pr in P["probs"])
    mpad = 8 if m <= 8 else 16
    assert P["xbox"] == sub_max * mpad * 128 and P["stage"] == 16384 + P["xbox"]
    xchg = XCHG if m <= 8 else 0
    cbuf = 8 * 2 * 2 * (32 if m <= 8 else 16) * P["cstride"]
    assert P["smem"] == 1024 + P["ws"] * P["stage"] + cbuf + xchg + EXTRA and P["smem"] <= BUDGET
    cta = 0
    any_split = False
    part_total = 0
    per_cta_bytes = []
    for pr in P["probs"]:
        assert pr["cta0"] == cta
        kbt, share, tiles, gb = pr["kbt"], pr["share"], pr["tiles"], pr["gb"]
        assert tiles == -(-pr["n"] // 128)
        assert share % gb == 0 and share >= gb
        assert pr["ctas"] == -(-(tiles * kbt) // share)
        cta += pr["ctas"]
        covered = set()
        slots = set()
        first_of, last_of = {}, {}
        for b in range(pr["ctas"]):
            segs = segments(b, pr)
            assert segs
            per_cta_bytes.append(sum(kb - ka for (_, ka, kb) in segs) * unit_bytes(pr))
            for i, (t, ka, kb) in enumerate(segs):
                assert 0 <= t < tiles and 0 <= ka < kb <= kbt
                assert ka % gb == 0 and kb % gb == 0              # whole scale groups
                parts = 2 if m <= 8 else 1                        # a compute warp's share of a box
                half = pr["sub"] // parts
                for kbs in range(ka, kb, pr["sub"]):
                    nk = min(pr["sub"], kb - kbs)
                    assert kbs % gb == 0 and nk >= 1
                    for part in range(parts):
                        lo = part * half
                        if lo >= nk:
                            continue
                        nkp = min(nk, lo + half) - lo
                        assert (kbs + lo) % gb == 0                   # a part starts on a whole group
                        # constant words the part needs, for the worst row parity
                        if pr["kind"] != 2:
                            ng = -(-nkp // gb)
                            assert 4 * (ng // 2 + 1) <= P["cstride"]
                        else:
                            assert 4 * nkp <= P["cstride"] or (pr["dq"] and 8 <= P["cstride"])
                for u in range(ka, kb):
                    assert (t, u) not in covered
                    covered.add((t, u))
                first_of.setdefault(t, b)
                last_of[t] = b
                full = ka == 0 and kb == kbt
                if full:
                    continue
                any_split = True
                if kb < kbt:
                    # contributor: its first-processed segment, and it is not the tile's last CTA
                    assert i == 0
                    slot = b + t
                    assert slot not in slots and slot < pr["ctas"] + tiles
                    slots.add(slot)
                else:
                    # finisher: processed last
                    assert i == len(segs) - 1
        assert len(covered) == tiles * kbt
        for t in range(tiles):
            lo = (t * kbt) // share
            hi = ((t + 1) * kbt - 1) // share
            assert first_of[t] == lo and last_of[t] == hi
        part_total += -(-((pr["ctas"] + tiles) * m * 128 * 4) // 256) * 256
    assert P["ctas"] == cta
    if any_split:
        assert P["workspace"] == HEADER + part_total
    else:
        assert P["workspace"] == 0
    mean = sum(per_cta_bytes) / len(per_cta_bytes)
    return P, max(per_cta_bytes) / mean


@pytest.mark.parametrize("m", [1, 4, 8, 9, 16])
def test_8b_layer_set_one_launch(m):
    P, imbalance = check(m, [qweight(n, k) for (n, k) in SHAPES_8B])
    # the whole set in one wave with about equal bytes per CTA
    assert P["ctas"] >= 0.9 * 2 * SMS
    assert imbalance < 1.15


@pytest.mark.parametrize("m", [1, 16])
def test_8b_layer_mix(m):
    bits = [2, 2, 2, 2, 4, 2, 2]
    check(m, [qweight(n, k, bits=b) for (n, k), b in zip(SHAPES_8B, bits)])


@pytest.mark.parametrize("m", [1, 16])
def test_channel_mix_halves(m):
    check(m, [qweight(3584, 4096, bits=4), qweight(10752, 4096, bits=2)])
    check(m, [qweight(250, 1024, bits=4), qweight(750, 1024, bits=2)])


@pytest.mark.parametrize("m,n,k,scheme,bits,dq", [
    (1, 256, 512, "minmax", 4, False), (16, 200, 640, "minmax", 4, False), (1, 14336, 4096, "minmax", 4, False),
    (8, 4096, 4096, "minmax", 2, False), (12, 2000, 3200, "codebook", 4, True), (16, 4096, 14336, "minmax", 4, False),
    (1, 8192, 8192, "codebook", 4, True), (16, 28672, 8192, "codebook", 4, True), (16, 8192, 28672, "codebook", 4, False),
    (3, 1, 128, "minmax", 4, False), (1, 1000, 64 * 3, "minmax", 2, False), (5, 130, 384, "minmax", 4, False),
])
def test_single_weight(m, n, k, scheme, bits, dq):
    check(m, [qweight(n, k, scheme, bits, dq)])


def test_plan_rejects_bad_arguments():
    q = qweight(256, 512)
    arr = (ctypes.POINTER(lbq.lbq_qweight) * 9)(*[ctypes.pointer(q)] * 9)
    out = (ctypes.c_int64 * 8)()
    assert lbq.lbq_gemv_plan(0, arr, 1, SMS, out, None) == lbq.LBQ_EINVAL
    assert lbq.lbq_gemv_plan(17, arr, 1, SMS, out, None) == lbq.LBQ_EINVAL
    assert lbq.lbq_gemv_plan(1, arr, 0, SMS, out, None) == lbq.LBQ_EINVAL
    assert lbq.lbq_gemv_plan(1, arr, 9, SMS, out, None) == lbq.LBQ_EINVAL
    assert lbq.lbq_gemv_plan(1, arr, 1, SMS, None, None) == lbq.LBQ_EINVAL

"""Pins of the CPU oracle against what the pages and the mathematics fix.

Nothing here compares the oracle with itself: every check uses an independent
fact -- a hand-built vector from the pages, a closed form, an invariant that a
plausible mistake (dropped term, wrong sign, wrong index, transposed operand)
breaks, a special case that reduces to a library routine, or an exact finite
difference of a bilinear function.
"""
import math
import os
from fractions import Fraction

import numpy as np
import pytest
import torch

import oracle
from qlora_quantized_linear_b200 import synthetic as syn

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def _bf16(x: np.ndarray) -> np.ndarray:
    """fp32 -> bf16 bits (round to nearest even), via torch."""
    return syn.bits_u16(torch.from_numpy(np.ascontiguousarray(x, np.float32)).to(torch.bfloat16))


# --------------------------------------------------------------------------
# number formats
# --------------------------------------------------------------------------
def test_f16_conversion_matches_numpy_rne():
    rng = np.random.default_rng(1)
    xs = np.concatenate([
        rng.standard_normal(4000).astype(np.float32) * 10.0 ** rng.integers(-9, 5, 4000),
        np.array([65504.0, 65520.0, 65519.996, 2.0 ** -24, 2.0 ** -25, 3 * 2.0 ** -26,
                  1.0 + 2.0 ** -11, 1.0 + 3 * 2.0 ** -11, -0.0, 0.0], np.float32),
    ]).astype(np.float32)
    with np.errstate(over="ignore"):
        _f16_loop(xs)


def _f16_loop(xs):
    for x in xs:
        assert oracle.f32_to_f16(float(x)) == int(np.float16(x).view(np.uint16)), x
        h = np.float16(x).view(np.uint16)
        if np.isfinite(np.float16(x)):
            assert oracle.f16_to_f32(int(h)) == float(np.float16(x))


def test_bf16_widening_matches_torch():
    x = torch.randn(1000, dtype=torch.float32).to(torch.bfloat16)
    assert np.array_equal(oracle.bf16_to_f32(syn.bits_u16(x)), x.float().numpy())


# --------------------------------------------------------------------------
# packing -- hand-built vectors from the bitsandbytes guide's packing rule
# --------------------------------------------------------------------------
def _golden_packing():
    rows = []
    with open(os.path.join(GOLDEN, "packing.txt")) as f:
        for line in f:
            if line.startswith("#") or not line.strip():
                continue
            b, codes, packed = [p.strip() for p in line.split(";")]
            rows.append((int(b), [int(c) for c in codes.split()], bytes.fromhex(packed.replace(" ", ""))))
    return rows


@pytest.mark.parametrize("bits,codes,packed", _golden_packing())
def test_pack_golden(bits, codes, packed):
    c = np.array([codes], np.uint8)
    got = oracle.pack(c, bits)
    assert bytes(got.ravel()) == packed
    assert np.array_equal(oracle.unpack(got, len(codes), bits), c)


def test_pack_roundtrip_random():
    rng = np.random.default_rng(2)
    for bits in (2, 4):
        c = rng.integers(0, 1 << bits, (7, 256), dtype=np.uint8)
        assert np.array_equal(oracle.unpack(oracle.pack(c, bits), 256, bits), c)


# --------------------------------------------------------------------------
# storage accounting -- closed forms from the pages
# --------------------------------------------------------------------------
@pytest.mark.parametrize("bits,group,expect", [(4, 128, 4.25), (2, 64, 2.5)])
def test_minmax_bits_per_param(bits, group, expect):
    # GreenBit article, 模型量化 (1): INT4 g128 and INT2 g64 with a 16-bit scale
    # and a 16-bit zero per group -> b + 32/g bits per parameter.
    n, k = 4, 512
    W = syn.bits_u16(syn.normal_bf16((n, k), 0.02, 0))
    codes, scale, zero = oracle.minmax_quantize(W, bits, group)
    packed = oracle.pack(codes, bits)
    total_bits = 8 * (packed.nbytes + scale.nbytes + zero.nbytes)
    assert total_bits / (n * k) == expect
    # 4x compression of the 16-bit weight before the group overhead (GreenBit
    # article, 模型量化: 4-bit vs FP16), 16/4.25 with it.
    assert 16 * n * k / (8 * packed.nbytes) == 16 / bits


def test_double_quant_saves_0_373_bits():
    # QLoRA explainer, 关键技术细节 2 / 结论: double quantization saves about
    # 0.37 bit per parameter.  fp32 absmax per 64 weights -> 8-bit per 64 plus
    # an fp32 scale per 256 absmax values.
    n, k = 64, 256 * 64  # 256 absmax blocks per row
    nb = n * k // 64
    absmax = np.abs(np.random.default_rng(3).standard_normal(nb)).astype(np.float32) + 0.1
    q8, s2, off, exact = oracle.double_quant(absmax)
    before = 32 * absmax.size
    after = 8 * q8.size + 32 * s2.size
    saved = (before - after) / (n * k)
    assert saved == 32 / 64 - 8 / 64 - 32 / (64 * 256) == 0.373046875
    assert round(saved, 2) == 0.37


# --------------------------------------------------------------------------
# MinMax quantizer
# --------------------------------------------------------------------------
def _mixed_weight(n, k, seed):
    w = syn.weight_bf16(n, k, 0.02, seed, outlier_frac=0.01, outlier_scale=20.0).float()
    # rows with all-positive and all-negative groups, a constant group and a
    # zero row, so that zero points outside [0, Q] and degenerate groups occur
    w[1] = w[1].abs() + 0.05
    w[2] = -w[2].abs() - 0.05
    w[3, :128] = 0.3
    w[4] = 0.0
    return syn.bits_u16(w.to(torch.bfloat16))


@pytest.mark.parametrize("bits,group", [(4, 128), (2, 64)])
def test_minmax_roundtrip_bound(bits, group):
    n, k = 16, 512
    Q = (1 << bits) - 1
    W = _mixed_weight(n, k, 5)
    codes, scale, zero = oracle.minmax_quantize(W, bits, group)
    assert codes.max() <= Q
    What = oracle.minmax_dequantize(oracle.pack(codes, bits), scale, zero, k, bits, group)
    w = oracle.bf16_to_f32(W).reshape(n, k // group, group).astype(np.float64)
    sf = np.array([oracle.f16_to_f32(int(h)) for h in scale.ravel()]).reshape(n, k // group, 1)
    err = np.abs(w - What.reshape(n, k // group, group))
    # |w - w_hat| <= scale/2 inside [min, max]; the fp16 rounding of the scale
    # can shorten the top of the grid by at most Q * scale * 2^-11, and the fp32
    # division adds a relative 2^-24.
    bound = sf * (0.5 + Q * 2.0 ** -11) + 2.0 ** -23 * np.abs(w) + 1e-30
    assert np.all(err <= bound), float((err - bound).max())
    # the group minimum maps to code 0 and the maximum to Q (or within one
    # step when the fp16 scale shortened the grid)
    cg = codes.reshape(n, k // group, group)
    for i in range(n):
        for g in range(k // group):
            if w[i, g].max() == w[i, g].min():
                continue
            assert cg[i, g][w[i, g].argmin()] == 0
            assert cg[i, g][w[i, g].argmax()] >= Q - 1


def test_minmax_scale_zero_exact_rational_crosscheck():
    """Scale and zero of every group, recomputed with exact rationals and
    numpy's float16: pins which elements form a group (along k) and the order
    fp32 range -> /Q -> fp16 -> zero = rint(-min/scale)."""
    n, k, bits, group = 6, 256, 4, 128
    W = _mixed_weight(n, k, 11)
    codes, scale, zero = oracle.minmax_quantize(W, bits, group)
    w = oracle.bf16_to_f32(W).reshape(n, k // group, group)
    for i in range(n):
        for g in range(k // group):
            mn, mx = float(w[i, g].min()), float(w[i, g].max())
            r = np.float32(Fraction(mx) - Fraction(mn))   # exact difference fits fp64
            s32 = np.float32(r) / np.float32(15)          # IEEE fp32 division
            s16 = np.float16(s32)
            if r == 0 or s16 == 0:
                s16 = np.float16(1.0)
            assert int(s16.view(np.uint16)) == int(scale[i, g])
            # IEEE fp32 negation and division (numpy float32), keeping the
            # sign of zero: -(+0)/s = -0 is stored as fp16 -0
            z = np.float32(-(np.float32(mn) + np.float32(0.0))) / np.float32(s16)
            zr = np.float16(np.rint(z))
            assert int(zr.view(np.uint16)) == int(zero[i, g]), (i, g)


@pytest.mark.parametrize("bits", [4, 2])
def test_minmax_grid_values_roundtrip_exactly(bits):
    """Every representable grid value (q - z) * s re-quantizes to q, with the
    same scale and zero recovered (GreenBit article, 模型量化 (1))."""
    Q = (1 << bits) - 1
    group = 128 if bits == 4 else 64
    rng = np.random.default_rng(7)
    n, k = 8, 4 * group
    q = rng.integers(0, Q + 1, (n, k)).astype(np.int64)
    qg = q.reshape(n, k // group, group)
    qg[:, :, 0] = 0
    qg[:, :, 1] = Q
    z = rng.integers(0, Q + 1, (n, k // group))
    sf = (rng.integers(1, 8, (n, k // group)) * 2.0 ** rng.integers(-10, -4, (n, k // group)))
    w = (qg - z[:, :, None]) * sf[:, :, None]          # exact in bf16 (<= 7 bits)
    W = _bf16(w.reshape(n, k).astype(np.float32))
    assert np.array_equal(oracle.bf16_to_f32(W).astype(np.float64), w.reshape(n, k))
    codes, scale, zero = oracle.minmax_quantize(W, bits, group)
    assert np.array_equal(codes.astype(np.int64), q)
    assert np.array_equal(np.array([oracle.f16_to_f32(int(h)) for h in scale.ravel()]), sf.ravel())
    assert np.array_equal(np.array([oracle.f16_to_f32(int(h)) for h in zero.ravel()]), z.ravel())
    What = oracle.minmax_dequantize(oracle.pack(codes, bits), scale, zero, k, bits, group)
    assert np.array_equal(What.astype(np.float64), w.reshape(n, k))


@pytest.mark.parametrize("bits", [4, 2])
def test_minmax_ties_round_half_to_even(bits):
    """Elements exactly half-way between two grid points, and zero points
    exactly half-way between two integers, take the even neighbour (rint),
    not the one away from zero: expected codes from exact rationals and
    Python's round() (tests/tie_inputs.py)."""
    from tie_inputs import tie_weight
    group = 128 if bits == 4 else 64
    n, k = 24, 4 * group
    w, codes, zeros, scales = tie_weight(n, k, bits, seed=bits)
    W = _bf16(w)
    assert np.array_equal(oracle.bf16_to_f32(W), w)
    got, scale, zero = oracle.minmax_quantize(W, bits, group)
    assert np.array_equal(np.array([oracle.f16_to_f32(int(h)) for h in scale.ravel()]), scales.ravel())
    assert np.array_equal(np.array([oracle.f16_to_f32(int(h)) for h in zero.ravel()]), zeros.ravel())
    assert np.array_equal(got.astype(np.int64), codes)
    # the case has teeth: half-away-from-zero rounding gives other codes
    Q = (1 << bits) - 1
    t = w.reshape(n, k // group, group) / scales[:, :, None]
    away = np.clip(np.sign(t) * np.floor(np.abs(t) + 0.5) + zeros[:, :, None], 0, Q).reshape(n, k)
    assert int((away != codes).sum()) > k // 4


def test_minmax_constant_and_zero_groups():
    n, k = 2, 128
    w = np.zeros((n, k), np.float32)
    w[0] = 3.0
    W = _bf16(w)
    codes, scale, zero = oracle.minmax_quantize(W, 4, 128)
    assert oracle.f16_to_f32(int(scale[0, 0])) == 1.0 and oracle.f16_to_f32(int(scale[1, 0])) == 1.0
    What = oracle.minmax_dequantize(oracle.pack(codes, 4), scale, zero, k, 4, 128)
    assert np.all(What[0] == 3.0) and np.all(What[1] == 0.0)


def test_minmax_signed_zero_independent_of_order():
    w = np.zeros((2, 128), np.float32)
    w[0, 0] = -0.0
    w[1, 5] = -0.0
    w[:, 64] = 1.0
    W = _bf16(w)
    _, scale, zero = oracle.minmax_quantize(W, 4, 128)
    assert scale[0, 0] == scale[1, 0] and zero[0, 0] == zero[1, 0]


def test_minmax_rejects_nonfinite():
    w = np.zeros((1, 128), np.float32)
    w[0, 3] = np.inf
    with pytest.raises(ValueError):
        oracle.minmax_quantize(_bf16(w), 4, 128)


# --------------------------------------------------------------------------
# codebook quantizer
# --------------------------------------------------------------------------
def test_codebook_uniform_grid_reduces_to_round_to_nearest():
    """With the uniform table c_j = (j - 8)/8, the nearest-entry rule is
    round-to-nearest on x*8 with ties to the lower entry, clamped."""
    cb = ((np.arange(16) - 8) / 8).astype(np.float32)
    n, k = 16, 256
    W = syn.bits_u16(syn.normal_bf16((n, k), 0.02, 13))
    codes, absmax = oracle.codebook_quantize(W, cb)
    w = oracle.bf16_to_f32(W).reshape(-1, 64)
    a = np.abs(w).max(axis=1)
    assert np.array_equal(absmax, a)
    x = (w / a[:, None]).astype(np.float32)          # fp32 division, as defined
    d = x.astype(np.float64) * 8                      # exact
    expect = np.clip(np.ceil(d - 0.5) + 8, 0, 15)     # tie -> lower index
    assert np.array_equal(codes.reshape(-1, 64), expect.astype(np.uint8))


def test_codebook_entries_map_to_themselves():
    """Idempotence: w = c_j * a is quantized to code j (a = block absmax)."""
    cb = np.array([-1, -0.75, -0.5, -0.375, -0.25, -0.125, -0.0625, 0,
                   0.0625, 0.125, 0.1875, 0.25, 0.375, 0.5, 0.75, 1], np.float32)
    rng = np.random.default_rng(17)
    n, k = 8, 128
    j = rng.integers(0, 16, (n * k // 64, 64))
    j[:, 0] = 15  # |c| = 1 in every block, so absmax = a
    a = 2.0 ** rng.integers(-8, -2, (n * k // 64, 1))
    w = (cb[j] * a).astype(np.float32).reshape(n, k)
    W = _bf16(w)
    codes, absmax = oracle.codebook_quantize(W, cb)
    assert np.array_equal(codes.reshape(-1, 64), j.astype(np.uint8))
    assert np.array_equal(absmax, a.ravel().astype(np.float32))


def test_codebook_error_bound_and_zero_block():
    cb = syn.codebook_normal16()
    n, k = 32, 256
    wt = syn.weight_bf16(n, k, 0.015, 19).float()
    wt[3, :64] = 0.0
    W = syn.bits_u16(wt.to(torch.bfloat16))
    codes, absmax = oracle.codebook_quantize(W, cb)
    zero_idx = int(np.where(cb == 0)[0][0])
    assert np.all(codes[3, :64] == zero_idx) and absmax[3 * (k // 64)] == 0
    What = oracle.codebook_dequantize(oracle.pack(codes, 4), absmax, cb, n, k)
    w = oracle.bf16_to_f32(W).astype(np.float64)
    maxgap = np.diff(cb.astype(np.float64)).max()
    a = np.repeat(absmax.astype(np.float64), 64).reshape(n, k)
    assert np.all(np.abs(w - What) <= a * (maxgap / 2) * (1 + 1e-6) + 1e-30)


def test_codebook_rejects_bad_tables():
    W = syn.bits_u16(syn.normal_bf16((1, 64), 1.0, 0))
    cb = syn.codebook_normal16()
    bad = cb.copy()
    bad[7] = 1e-3                                             # no zero entry
    with pytest.raises(ValueError):
        oracle.codebook_quantize(W, bad)
    bad = cb.copy()
    bad[15] = 1.5                                             # outside [-1, 1]
    with pytest.raises(ValueError):
        oracle.codebook_quantize(W, bad)
    bad[15] = np.nan
    with pytest.raises(ValueError):
        oracle.codebook_quantize(W, bad)
    # a table in another order is a valid table with other codes
    codes, _ = oracle.codebook_quantize(W, cb[::-1].copy())
    codes2, _ = oracle.codebook_quantize(W, cb)
    assert np.array_equal(codes, 15 - codes2)


# --------------------------------------------------------------------------
# FP4 (E2M1) table ([BNB] nf4与fp4): code order, +0 and -0
# --------------------------------------------------------------------------
def test_fp4_table_is_e2m1():
    """The E2M1 magnitudes 0, 0.5, 1, 1.5, 2, 3, 4, 6 (over 6), positive for
    codes 0..7 and negative for 8..15, both zeros present."""
    cb = syn.codebook_fp4_e2m1()
    mags = np.array([0, 0.5, 1, 1.5, 2, 3, 4, 6]) / 6
    assert np.array_equal(cb[:8].astype(np.float64), mags.astype(np.float32).astype(np.float64))
    assert np.array_equal(cb[8:], -cb[:8])
    assert np.signbit(cb[8]) and not np.signbit(cb[0]) and cb[8] == 0.0
    assert cb.max() == 1.0 and cb.min() == -1.0


def test_fp4_entries_map_to_themselves_and_zero_to_code0():
    """Idempotence on c_j * a for the 14 nonzero codes; a zero (either sign)
    is code 0, the lower index of the two zeros."""
    cb = syn.codebook_fp4_e2m1()
    rng = np.random.default_rng(23)
    nb = 64
    j = rng.integers(0, 16, (nb, 64))
    j[:, 0] = 7                                   # |c| = 1 in every block: absmax = a
    a = 2.0 ** rng.integers(-8, -2, (nb, 1))
    w = (cb[j].astype(np.float64) * a).astype(np.float32)
    W = _bf16(w.reshape(16, 256))
    # c_j * a survives the bf16 rounding exactly for about half the entries;
    # the others move by at most 2^-9 of their value, far less than half a
    # gap of the table (1/24 of a), so every entry still maps to its code
    exact = oracle.bf16_to_f32(W).reshape(nb, 64) == w
    codes, absmax = oracle.codebook_quantize(W, cb)
    codes = codes.reshape(nb, 64)
    expect = np.where(j == 8, 0, j)
    assert exact.mean() > 0.3
    assert np.array_equal(absmax, a.ravel().astype(np.float32))
    assert np.array_equal(codes, expect.astype(np.uint8))


def test_fp4_sign_symmetry():
    """Negating the weights flips the sign bit of every nonzero code (E2M1 is
    sign-magnitude and the table is symmetric in code order); values
    quantized to zero stay code 0."""
    cb = syn.codebook_fp4_e2m1()
    W = syn.normal_bf16((32, 512), 0.015, 29)
    c_pos, a_pos = oracle.codebook_quantize(syn.bits_u16(W), cb)
    c_neg, a_neg = oracle.codebook_quantize(syn.bits_u16(-W), cb)
    assert np.array_equal(a_pos, a_neg)
    expect = np.where(c_pos == 0, 0, c_pos ^ 8)
    assert np.array_equal(c_neg, expect)
    assert not np.any(c_pos == 8)                 # -0 is never chosen


def test_fp4_error_bound():
    cb = syn.codebook_fp4_e2m1()
    n, k = 32, 256
    W = syn.bits_u16(syn.weight_bf16(n, k, 0.015, 31, outlier_frac=0.01))
    codes, absmax = oracle.codebook_quantize(W, cb)
    What = oracle.codebook_dequantize(oracle.pack(codes, 4), absmax, cb, n, k)
    w = oracle.bf16_to_f32(W).astype(np.float64)
    maxgap = np.diff(np.sort(cb.astype(np.float64))).max()       # 1/3 (4/6 to 6/6)
    a = np.repeat(absmax.astype(np.float64), 64).reshape(n, k)
    assert np.all(np.abs(w - What) <= a * (maxgap / 2) * (1 + 1e-6) + 1e-30)


# --------------------------------------------------------------------------
# double quantization
# --------------------------------------------------------------------------
def test_double_quant_properties():
    rng = np.random.default_rng(23)
    nb = 256 * 5 + 77                               # ragged last block
    absmax = _bf16((np.abs(rng.standard_normal(nb)) * 0.03 + 0.01).astype(np.float32))
    absmax = oracle.bf16_to_f32(absmax)             # absmax values are bf16 values
    q8, s2, off, exact = oracle.double_quant(absmax)
    assert exact
    # offset = mean, rounded once from fp64 (the fp64 sum is exact here)
    mean = Fraction(math.fsum(float(a) for a in absmax)) / nb
    assert np.float32(off) == np.float32(float(np.float64(float(mean))))
    ah = oracle.double_dequant(q8, s2, off)
    for b in range(len(s2)):
        lo, hi = 256 * b, min(256 * b + 256, nb)
        c = (absmax[lo:hi] - off).astype(np.float32)
        assert s2[b] == np.abs(c).max()
        assert np.abs(q8[lo:hi]).max() == 127          # the block extreme
        err = np.abs(ah[lo:hi].astype(np.float64) - absmax[lo:hi])
        assert np.all(err <= s2[b] / 254 + 4 * np.spacing(np.float32(abs(off) + s2[b])))
    assert q8.dtype == np.int8 and np.abs(q8.astype(int)).max() <= 127


def test_double_quant_flags_inexact_sum():
    absmax = np.array([1.0, 2.0 ** -60, 3.0], np.float32)
    *_, exact = oracle.double_quant(absmax, allow_inexact=True)
    assert not exact


# --------------------------------------------------------------------------
# quantized linear layer with LoRA
# --------------------------------------------------------------------------
def _tiny_problem(m=5, n=24, k=256, r=4, seed=29):
    X = syn.bits_u16(syn.normal_bf16((m, k), 1.0, seed))
    Wb = syn.bits_u16(syn.normal_bf16((n, k), 0.02, seed + 1))
    codes, scale, zero = oracle.minmax_quantize(Wb, 4, 128)
    What = oracle.minmax_dequantize(oracle.pack(codes, 4), scale, zero, k, 4, 128)
    A = syn.bits_u16(syn.normal_bf16((r, k), 0.01, seed + 2))
    B = syn.bits_u16(syn.normal_bf16((n, r), 0.01, seed + 3))
    dY = syn.bits_u16(syn.normal_bf16((m, n), 0.1, seed + 4))
    return X, What, A, B, dY, (codes, scale, zero)


def test_rank0_reduces_to_matmul():
    X, What, *_ = _tiny_problem()
    Y, T, Yb = oracle.linear_fwd(X, What)
    ref = oracle.bf16_to_f32(X).astype(np.float64) @ What.astype(np.float64).T
    np.testing.assert_allclose(Y, ref, rtol=1e-12, atol=1e-15)
    np.testing.assert_allclose(Yb, np.abs(oracle.bf16_to_f32(X)).astype(np.float64)
                               @ np.abs(What.astype(np.float64)).T, rtol=1e-12)


def test_zero_weight_leaves_only_adapter_term():
    X, What, A, B, _, _ = _tiny_problem()
    s = 2.0
    Y, T, _ = oracle.linear_fwd(X, np.zeros_like(What), A, B, s)
    x = oracle.bf16_to_f32(X).astype(np.float64)
    a = oracle.bf16_to_f32(A).astype(np.float64)
    b = oracle.bf16_to_f32(B).astype(np.float64)
    np.testing.assert_allclose(T, x @ a.T, rtol=1e-12, atol=1e-18)
    np.testing.assert_allclose(Y, s * (x @ a.T) @ b.T, rtol=1e-12, atol=1e-18)


def test_sampled_forward_matches_full():
    X, What, A, B, _, (codes, scale, zero) = _tiny_problem()
    s = 2.0
    Y, _, Yb = oracle.linear_fwd(X, What, A, B, s)
    rows = np.array([0, 4, 2, 3]); cols = np.array([0, 23, 7, 11])
    Ys, Ybs = oracle.linear_fwd_sampled_minmax(X, oracle.pack(codes, 4), scale, zero, What.shape[0],
                                               What.shape[1], 4, 128, rows, cols, A, B, s)
    np.testing.assert_allclose(Ys, Y[rows, cols], rtol=1e-13, atol=1e-16)
    np.testing.assert_allclose(Ybs, Yb[rows, cols], rtol=1e-13)


def test_sampled_backward_matches_full():
    X, What, A, B, _, (codes, scale, zero) = _tiny_problem()
    s = 2.0
    n, k = What.shape
    m = X.shape[0]
    dY = _bf16(np.random.default_rng(9).standard_normal((m, n)).astype(np.float32) * 0.1)
    dX, _, dXb = oracle.linear_bwd(dY, What, A, B, s)
    rows = np.array([0, 2, 1, 3, 0]); cols = np.array([0, 100, 7, 255, 129])
    dXs, dXbs = oracle.linear_bwd_sampled_minmax(dY, oracle.pack(codes, 4), scale, zero, n, k, 4, 128,
                                                 rows, cols, A, B, s)
    np.testing.assert_allclose(dXs, dX[rows, cols], rtol=1e-12, atol=1e-16)
    np.testing.assert_allclose(dXbs, dXb[rows, cols], rtol=1e-12)


def _loss(X, What, A, B, s, dY):
    Y, _, _ = oracle.linear_fwd(X, What, A, B, s)
    return float(np.sum(oracle.bf16_to_f32(dY).astype(np.float64) * Y))


def _bump(bits_arr, idx, new_val):
    out = bits_arr.copy()
    out[idx] = _bf16(np.array([new_val], np.float32))[0]
    return out


def test_backward_products_by_exact_finite_differences():
    """L = sum(dY * Y) is linear in each of X, A and B separately, so a finite
    difference over one element is exact (up to fp64 rounding).  This pins
    dX = dY W + s (dY B) A, dA = s (dY B)^T X and dB = s dY^T (X A^T) against
    the forward definition Y = X W^T + s (X A^T) B^T."""
    X, What, A, B, dY, _ = _tiny_problem()
    s = 2.0
    dX, U, _ = oracle.linear_bwd(dY, What, A, B, s)
    dA, dB, _, _ = oracle.lora_grads(X, dY, A, B, s)
    L0 = _loss(X, What, A, B, s, dY)
    checks = 0
    for arr_name, idx in [("X", (0, 3)), ("X", (4, 200)), ("X", (2, 129)),
                          ("A", (0, 5)), ("A", (3, 255)), ("B", (0, 0)), ("B", (23, 3)), ("B", (11, 2))]:
        arr = {"X": X, "A": A, "B": B}[arr_name]
        old = float(oracle.bf16_to_f32(arr[idx]))
        new = float(oracle.bf16_to_f32(_bf16(np.array([old * 1.5 + 0.25], np.float32)))[0])
        h = new - old
        args = dict(X=X, A=A, B=B)
        args[arr_name] = _bump(arr, idx, new)
        fd = (_loss(args["X"], What, args["A"], args["B"], s, dY) - L0) / h
        grad = {"X": dX, "A": dA, "B": dB}[arr_name][idx]
        assert abs(fd - grad) <= 1e-9 * (abs(grad) + 1e-6), (arr_name, idx, fd, grad)
        checks += 1
    assert checks == 8
    # U = dY B (shared by dX and dA)
    np.testing.assert_allclose(U, oracle.bf16_to_f32(dY).astype(np.float64)
                               @ oracle.bf16_to_f32(B).astype(np.float64), rtol=1e-12, atol=1e-18)


# --------------------------------------------------------------------------
# merging the adapter into the weight (GreenBit article, introduction: the
# LoRA module is merged into the full-precision model after fine-tuning)
# --------------------------------------------------------------------------
def _bits(t: torch.Tensor) -> np.ndarray:
    return syn.bits_u16(t.to(torch.bfloat16))


def _as_f32(bits: np.ndarray) -> np.ndarray:
    return oracle.bf16_to_f32(bits).astype(np.float32)


def test_merge_hand_built():
    # W = [1, 1], B = [[2]], A = [[0.5, -1]], s = 3: B A = [1, -2], s B A = [3, -6]
    W = np.array([[1.0, 1.0]], np.float32)
    A = _bits(torch.tensor([[0.5, -1.0]]))
    B = _bits(torch.tensor([[2.0]]))
    assert _as_f32(oracle.lora_merge(W, A, B, 3.0, 1)).tolist() == [[4.0, -5.0]]
    assert _as_f32(oracle.lora_merge(W, A, B, 3.0, -1)).tolist() == [[-2.0, 7.0]]


def test_merge_rank0_is_bf16_rounding_of_the_weight():
    # no adapter: the merged weight is the weight rounded to bf16 (torch's
    # fp32 -> bf16 conversion rounds to nearest even), ties included
    rng = np.random.default_rng(11)
    W = (rng.standard_normal((64, 96)) * 0.02).astype(np.float32)
    W[0, :6] = [1.0 + 2.0 ** -8, 1.0 + 3 * 2.0 ** -8, -(1.0 + 2.0 ** -8), 2.0 ** -130, 0.0, 65504.0]
    got = oracle.lora_merge(W, None, None, 2.0, 1)
    assert np.array_equal(got, _bf16(W))
    assert _as_f32(got[:1, :3]).tolist() == [[1.0, 1.0 + 2.0 ** -6, -1.0]]
    # the one difference from plain rounding: -0 + (s * 0) is +0 in IEEE arithmetic
    assert oracle.lora_merge(np.array([[-0.0]], np.float32), None, None, 2.0, 1).tolist() == [[0]]


def test_merge_matches_fp64_product_within_rounding():
    # against numpy's fp64 matmul: a dropped s, a wrong sign or a transposed
    # operand would be off by far more than the binary32 and bf16 roundings
    rng = np.random.default_rng(12)
    n, k, r, s = 48, 80, 16, 2.0
    W = (rng.standard_normal((n, k)) * 0.02).astype(np.float32)
    A = _bits(torch.from_numpy(rng.standard_normal((r, k)).astype(np.float32) * 0.05))
    B = _bits(torch.from_numpy(rng.standard_normal((n, r)).astype(np.float32) * 0.05))
    Af, Bf = _as_f32(A).astype(np.float64), _as_f32(B).astype(np.float64)
    for sign in (1, -1):
        got = _as_f32(oracle.lora_merge(W, A, B, s, sign)).astype(np.float64)
        exact = W.astype(np.float64) + sign * s * (Bf @ Af)
        mag = np.abs(W) + abs(s) * (np.abs(Bf) @ np.abs(Af))
        lim = np.abs(exact) * 2.0 ** -8 + (r + 3) * 2.0 ** -24 * mag
        assert np.all(np.abs(got - exact) <= lim)
        # and the adapter term really is there (not the rank-0 result)
        assert np.mean(got != _as_f32(_bf16(W))) > 0.5


def test_merge_accumulates_the_rank_in_order():
    # products 1, 2^-30, -1 summed in binary32 in order: (1 + 2^-30) rounds to
    # 1, so d = 0; an exact or reordered sum would leave 2^-30
    W = np.zeros((1, 1), np.float32)
    A = _bits(torch.tensor([[1.0], [2.0 ** -15], [1.0]]))
    B = _bits(torch.tensor([[1.0, 2.0 ** -15, -1.0]]))
    assert _as_f32(oracle.lora_merge(W, A, B, 1.0, 1)).tolist() == [[0.0]]
    # the same products in the order 1, -1, 2^-30 keep the small one
    A2 = _bits(torch.tensor([[1.0], [1.0], [2.0 ** -15]]))
    B2 = _bits(torch.tensor([[1.0, -1.0, 2.0 ** -15]]))
    assert _as_f32(oracle.lora_merge(W, A2, B2, 1.0, 1)).tolist() == [[2.0 ** -30]]


def test_unmerge_inverts_an_exact_merge():
    # small integers and a power-of-two scale: no step rounds, so removing the
    # adapter gives the weight back bit for bit
    rng = np.random.default_rng(13)
    n, k, r = 16, 32, 4
    W = rng.integers(-8, 8, (n, k)).astype(np.float32)
    A = _bits(torch.from_numpy(rng.integers(-3, 4, (r, k)).astype(np.float32)))
    B = _bits(torch.from_numpy(rng.integers(-3, 4, (n, r)).astype(np.float32)))
    merged = oracle.lora_merge(W, A, B, 0.5, 1)
    back = oracle.lora_merge(_as_f32(merged), A, B, 0.5, -1)
    assert np.array_equal(_as_f32(back), W)


# --------------------------------------------------------------------------
# channel-mix selection by sensitivity ([GB] 模型量化 (1))
# --------------------------------------------------------------------------
def test_channel_score_is_the_output_error_rise_for_one_hot_calibration():
    """With one-hot calibration tokens x_t = a_t e_t (t = k), the weighted
    squared errors are exactly the output error energies: score[c] =
    (|X (w2_c - w_c)|^2 - |X (w4_c - w_c)|^2) / t, computed here with a
    numpy matmul on the oracle's (pinned) dequantized weights."""
    n, k = 12, 256
    W = syn.bits_u16(syn.weight_bf16(n, k, 0.02, 41, outlier_frac=0.02))
    rng = np.random.default_rng(3)
    amp = (rng.integers(1, 8, k) * 2.0 ** rng.integers(-3, 3, k)).astype(np.float32)
    X = _bf16(np.diag(amp))
    score, bound = oracle.channel_score(W, X)
    w = oracle.bf16_to_f32(W).astype(np.float64)
    c4, s4, z4 = oracle.minmax_quantize(W, 4, 128)
    c2, s2, z2 = oracle.minmax_quantize(W, 2, 64)
    w4 = oracle.minmax_dequantize(oracle.pack(c4, 4), s4, z4, k, 4, 128).astype(np.float64)
    w2 = oracle.minmax_dequantize(oracle.pack(c2, 2), s2, z2, k, 2, 64).astype(np.float64)
    x = oracle.bf16_to_f32(X).astype(np.float64)
    e2 = ((w2 - w) @ x.T) ** 2
    e4 = ((w4 - w) @ x.T) ** 2
    expect = (e2.sum(axis=1) - e4.sum(axis=1)) / k
    assert np.allclose(score, expect, rtol=1e-12, atol=0)
    assert np.allclose(bound, (e2.sum(axis=1) + e4.sum(axis=1)) / k, rtol=1e-12, atol=0)


def test_channel_score_sign_cases():
    """A channel exact on its INT4 grid has score = bound > 0 (only INT2
    errs); a constant integer channel is exact in both (score = bound = 0);
    a constant 0.25 channel errs equally in both (the degenerate scale 1)."""
    rng = np.random.default_rng(9)
    k = 256
    q = rng.integers(0, 16, (1, k))
    q[0, 0], q[0, 1], q[0, 128], q[0, 129] = 0, 15, 0, 15
    z = rng.integers(0, 16, (1, 2))
    sf = 2.0 ** -7
    w_grid = ((q.reshape(1, 2, 128) - z[:, :, None]) * sf).reshape(1, k)
    w = np.vstack([w_grid, np.full((1, k), 2.0), np.full((1, k), 0.25)]).astype(np.float32)
    W = _bf16(w)
    X = syn.bits_u16(syn.normal_bf16((32, k), 1.0, 5))
    score, bound = oracle.channel_score(W, X)
    assert score[0] > 0 and score[0] == bound[0]
    assert score[1] == 0 and bound[1] == 0
    assert score[2] == 0 and bound[2] > 0


def test_channel_mix_select_top_scores_lower_index_on_ties():
    score = np.array([0.5, 2.0, 1.0, 2.0, -1.0, 1.0, 0.0, 1.0])
    perm = oracle.channel_mix_select(score, 4)
    # highest: 1, 3 (2.0), then 2, 5 among the three equal 1.0 (2 < 5 < 7)
    assert perm.tolist() == [1, 2, 3, 5, 0, 4, 6, 7]
    assert oracle.channel_mix_select(score, 0).tolist() == list(range(8))
    assert oracle.channel_mix_select(score, 8).tolist() == list(range(8))

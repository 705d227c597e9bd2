"""CUDA path vs the CPU oracle, element by element, through the C ABI.

Bit-exact: packed codes, scales, zeros, absmax, q8, s2, offset and the fp32
dequantized weights.  GEMM outputs: within the stated bound
|dY| <= 2^-7 * sum_k |x_k| |w_eff,k| + 1e-6 (w_eff = W_hat plus the adapter
term), computed by the oracle for every element.
"""
import ctypes

import numpy as np
import pytest
import torch

import oracle
from qlora_quantized_linear_b200 import synthetic as syn

pytestmark = pytest.mark.gpu

TOL_REL = 2.0 ** -7
TOL_ABS = 1e-6


@pytest.fixture(scope="module")
def lbq():
    from qlora_quantized_linear_b200 import lbq as m
    return m


def u16(t: torch.Tensor) -> np.ndarray:
    """Bits of a bf16/fp16 tensor (any device) as uint16 numpy."""
    return t.detach().cpu().contiguous().view(torch.int16).numpy().view(np.uint16)


def assert_status_clean(lbq):
    assert lbq.device_status() == 0


def assert_within(got, ref, bound, what):
    got = np.asarray(got, np.float64)
    err = np.abs(got - ref)
    lim = TOL_REL * bound + TOL_ABS
    bad = err > lim
    assert not bad.any(), (f"{what}: {int(bad.sum())}/{bad.size} elements outside the bound; "
                           f"worst excess {float((err - lim).max()):.3e} at {np.unravel_index(np.argmax(err - lim), err.shape)}")


def mixed_weight(n, k, seed, std=0.02):
    """Weights with outlier columns, all-positive / all-negative rows, a
    constant group, a zero row and a row far from zero relative to its
    spread (its zero point is far outside the code range: |zero| > 128)."""
    w = syn.weight_bf16(n, k, std, seed, outlier_frac=0.01, outlier_scale=20.0).float()
    if n > 5:
        w[1] = w[1].abs() + 0.05
        w[2] = -w[2].abs() - 0.05
        w[3, :128] = 0.3
        w[4] = 0.0
        w[5, 7] = -0.0
    if n > 6:
        w[6] = 2.0 + w[6] * 0.2
    return w.to(torch.bfloat16)


# --------------------------------------------------------------------------- quantize / dequantize
@pytest.mark.parametrize("bits", [4, 2])
@pytest.mark.parametrize("shape", [(256, 512), (300, 1024), (1, 128), (4096, 256)])
def test_minmax_quantize_bit_exact(lbq, bits, shape):
    n, k = shape
    W = mixed_weight(n, k, seed=n + k + bits)
    qw = lbq.QuantizedWeight(n, k, "minmax", bits).quantize(W.cuda())
    torch.cuda.synchronize()
    codes, scale, zero = oracle.minmax_quantize(syn.bits_u16(W), bits, qw.group)
    assert np.array_equal(qw.packed.cpu().numpy(), oracle.pack(codes, bits)), "packed codes differ"
    assert np.array_equal(u16(qw.scale), scale), "scales differ"
    assert np.array_equal(u16(qw.zero), zero), "zeros differ"
    What = qw.dequantize().cpu().numpy()
    ref = oracle.minmax_dequantize(oracle.pack(codes, bits), scale, zero, k, bits, qw.group)
    assert np.array_equal(What.view(np.uint32), ref.view(np.uint32)), "dequantized weights differ"
    assert_status_clean(lbq)


def test_minmax_quantize_grid_values(lbq):
    """Exact grid values re-quantize to themselves on the GPU as well."""
    n, k, bits, group = 64, 512, 4, 128
    rng = np.random.default_rng(5)
    q = rng.integers(0, 16, (n, k))
    qg = q.reshape(n, k // group, group)
    qg[:, :, 0], qg[:, :, 1] = 0, 15
    z = rng.integers(0, 16, (n, k // group))
    sf = rng.integers(1, 8, (n, k // group)) * 2.0 ** rng.integers(-10, -4, (n, k // group))
    w = ((qg - z[:, :, None]) * sf[:, :, None]).reshape(n, k).astype(np.float32)
    W = torch.from_numpy(w).to(torch.bfloat16)
    qw = lbq.QuantizedWeight(n, k, "minmax", bits).quantize(W.cuda())
    got = oracle.unpack(qw.packed.cpu().numpy(), k, bits)
    assert np.array_equal(got.astype(np.int64), q)


@pytest.mark.parametrize("double_quant", [False, True])
@pytest.mark.parametrize("shape", [(256, 512), (1000, 1024), (128, 64 * 300)])
def test_codebook_quantize_bit_exact(lbq, double_quant, shape):
    n, k = shape
    cb = syn.codebook_normal16()
    Wt = syn.weight_bf16(n, k, 0.015, seed=n * 7 + k).float()
    Wt[0, :64] = 0.0
    W = Wt.to(torch.bfloat16)
    qw = lbq.QuantizedWeight(n, k, "codebook", double_quant=double_quant, codebook=cb).quantize(W.cuda())
    torch.cuda.synchronize()
    codes, absmax = oracle.codebook_quantize(syn.bits_u16(W), cb)
    packed = oracle.pack(codes, 4)
    assert np.array_equal(qw.packed.cpu().numpy(), packed)
    assert np.array_equal(qw.absmax.cpu().numpy().view(np.uint32), absmax.view(np.uint32))
    a_used = absmax
    if double_quant:
        q8, s2, off, exact = oracle.double_quant(absmax)
        assert exact
        assert np.float32(qw.offset[0].item()).view(np.uint32) == np.float32(off).view(np.uint32)
        assert np.array_equal(qw.q8.cpu().numpy(), q8)
        assert np.array_equal(qw.s2.cpu().numpy().view(np.uint32), s2.view(np.uint32))
        a_used = oracle.double_dequant(q8, s2, off)
    What = qw.dequantize().cpu().numpy()
    ref = oracle.codebook_dequantize(packed, a_used, cb, n, k)
    assert np.array_equal(What.view(np.uint32), ref.view(np.uint32))
    assert_status_clean(lbq)


# --------------------------------------------------------------------------- forward
def fwd_problem(m, n, k, rank, seed, scheme="minmax", bits=4, double_quant=False):
    X = syn.normal_bf16((m, k), 1.0, seed)
    W = mixed_weight(n, k, seed + 1) if scheme == "minmax" else syn.weight_bf16(n, k, 0.015, seed + 1)
    A = syn.normal_bf16((rank, k), 0.01, seed + 2) if rank else None
    B = syn.normal_bf16((n, rank), 0.01, seed + 3) if rank else None
    return X, W, A, B


def device_qweight(lbq, W, scheme, bits, double_quant, cb):
    """A QuantizedWeight whose buffers hold the ORACLE's quantization of W, so
    that the GEMM tests do not depend on the GPU quantizer."""
    n, k = W.shape
    qw = lbq.QuantizedWeight(n, k, scheme, bits, double_quant=double_quant, codebook=cb)
    if scheme == "minmax":
        codes, scale, zero = oracle.minmax_quantize(syn.bits_u16(W), bits, qw.group)
        qw.packed.copy_(torch.from_numpy(oracle.pack(codes, bits)))
        qw.scale.copy_(torch.from_numpy(scale.view(np.float16)))
        qw.zero.copy_(torch.from_numpy(zero.view(np.float16)))
    else:
        codes, absmax = oracle.codebook_quantize(syn.bits_u16(W), cb)
        qw.packed.copy_(torch.from_numpy(oracle.pack(codes, 4)))
        qw.absmax.copy_(torch.from_numpy(absmax))
        if double_quant:
            q8, s2, off, _ = oracle.double_quant(absmax)
            qw.q8.copy_(torch.from_numpy(q8))
            qw.s2.copy_(torch.from_numpy(s2))
            qw.offset.fill_(float(off))
    torch.cuda.synchronize()
    return qw


def oracle_weight(W, scheme, bits, double_quant, cb):
    n, k = W.shape
    if scheme == "minmax":
        group = 128 if bits == 4 else 64
        codes, scale, zero = oracle.minmax_quantize(syn.bits_u16(W), bits, group)
        return oracle.minmax_dequantize(oracle.pack(codes, bits), scale, zero, k, bits, group)
    codes, absmax = oracle.codebook_quantize(syn.bits_u16(W), cb)
    if double_quant:
        q8, s2, off, _ = oracle.double_quant(absmax)
        absmax = oracle.double_dequant(q8, s2, off)
    return oracle.codebook_dequantize(oracle.pack(codes, 4), absmax, cb, n, k)


FWD_CASES = [
    # m, n, k, rank, scheme, bits, dq
    (8, 256, 512, 8, "minmax", 4, False),       # tiny single linear
    (1, 256, 512, 0, "minmax", 4, False),
    (15, 384, 1024, 16, "minmax", 4, False),
    (16, 200, 640, 16, "minmax", 4, False),     # ragged n
    (17, 256, 512, 0, "minmax", 4, False),
    (63, 128, 512, 8, "minmax", 4, False),
    (64, 256, 512, 16, "minmax", 4, False),
    (65, 256, 512, 64, "minmax", 4, False),
    (130, 384, 768, 16, "minmax", 4, False),    # two token tiles, ragged
    (16, 256, 512, 8, "minmax", 2, False),
    (200, 256, 512, 0, "minmax", 2, False),
    (1, 256, 1024, 0, "codebook", 4, False),
    (16, 256, 512, 16, "codebook", 4, True),
    (140, 256, 512, 0, "codebook", 4, True),
    # decode sizes at full layer shapes: CTA shares of the k-blocks straddle row tiles
    (1, 14336, 4096, 16, "minmax", 4, False),
    (8, 4096, 4096, 8, "minmax", 2, False),
    (12, 2000, 3200, 0, "codebook", 4, True),   # ragged n
    (16, 4096, 14336, 16, "minmax", 4, False),
    (16, 14336, 4096, 16, "minmax", 4, False),  # three-box ring; shares span two row tiles
]


@pytest.mark.parametrize("m,n,k,rank,scheme,bits,dq", FWD_CASES)
def test_linear_fwd_parity(lbq, m, n, k, rank, scheme, bits, dq):
    cb = syn.codebook_normal16()
    X, W, A, B = fwd_problem(m, n, k, rank, seed=m * 131 + n + k + rank, scheme=scheme, bits=bits)
    qw = device_qweight(lbq, W, scheme, bits, dq, cb)
    s = 2.0
    Y, T = lbq.linear_fwd(X.cuda(), qw, None if A is None else A.cuda(), None if B is None else B.cuda(), s)
    torch.cuda.synchronize()
    What = oracle_weight(W, scheme, bits, dq, cb)
    Yr, Tr, Yb = oracle.linear_fwd(syn.bits_u16(X), What, None if A is None else syn.bits_u16(A),
                                   None if B is None else syn.bits_u16(B), s)
    assert_within(Y.cpu().numpy(), Yr, Yb, "Y")
    if rank:
        Tb = np.abs(oracle.bf16_to_f32(syn.bits_u16(X))).astype(np.float64) @ \
            np.abs(oracle.bf16_to_f32(syn.bits_u16(A))).astype(np.float64).T
        assert_within(T.cpu().numpy(), Tr, Tb, "T")
    assert_status_clean(lbq)


def test_linear_fwd_repeatable(lbq):
    """Same inputs, same bits (split-K partials are summed in a fixed order)."""
    X, W, A, B = fwd_problem(4, 512, 2048, 16, seed=3)
    qw = device_qweight(lbq, W, "minmax", 4, False, None)
    Y1, _ = lbq.linear_fwd(X.cuda(), qw, A.cuda(), B.cuda(), 2.0)
    Y2, _ = lbq.linear_fwd(X.cuda(), qw, A.cuda(), B.cuda(), 2.0)
    assert torch.equal(Y1, Y2)


def test_workspace_reused_across_shapes(lbq):
    """One zero-filled workspace serves calls of different shapes and sizes in
    any order: each call leaves the split-K arrival counters at zero."""
    import ctypes
    probs = []
    for (m, n, k) in [(1, 1024, 4096), (16, 896, 2048), (64, 512, 4096), (3, 1024, 4096)]:
        X, W, _, _ = fwd_problem(m, n, k, 0, seed=m + n)
        qw = device_qweight(lbq, W, "minmax", 4, False, None)
        probs.append((X.cuda(), qw, lbq.lbq_linear_fwd_workspace_size(m, ctypes.byref(qw.struct), 0)))
    ws = lbq._workspace(max(p[2] for p in probs), "cuda")
    ref = [lbq.linear_fwd(X, qw)[0] for X, qw, _ in probs]    # each with a fresh workspace
    for order in ([0, 1, 2, 3], [3, 2, 1, 0, 0, 2]):
        for i in order:
            X, qw, _ = probs[i]
            Y, _ = lbq.linear_fwd(X, qw, workspace=ws)
            assert torch.equal(Y, ref[i]), f"case {i}"
    assert_status_clean(lbq)


def test_channel_mix_fwd(lbq):
    m, n, k = 16, 512, 1024
    X, W, A, B = fwd_problem(m, n, k, 16, seed=77)
    perm, n4 = syn.channel_mix_perm(n, 0.25, seed=1)
    Wp = W[torch.from_numpy(perm.astype(np.int64))]
    hi = device_qweight(lbq, Wp[:n4].contiguous(), "minmax", 4, False, None)
    lo = device_qweight(lbq, Wp[n4:].contiguous(), "minmax", 2, False, None)
    mix = lbq.ChannelMixWeight(hi, lo, perm)
    Y, _ = lbq.linear_fwd(X.cuda(), mix, A.cuda(), B.cuda(), 2.0)
    torch.cuda.synchronize()
    What = np.zeros((n, k), np.float32)
    What[perm[:n4]] = oracle_weight(Wp[:n4].contiguous(), "minmax", 4, False, None)
    What[perm[n4:]] = oracle_weight(Wp[n4:].contiguous(), "minmax", 2, False, None)
    Yr, _, Yb = oracle.linear_fwd(syn.bits_u16(X), What, syn.bits_u16(A), syn.bits_u16(B), 2.0)
    assert_within(Y.cpu().numpy(), Yr, Yb, "Y (channel-mix)")


# --------------------------------------------------------------------------- backward
BWD_CASES = [
    (8, 256, 512, 8, 4),
    (1, 256, 512, 0, 4),
    (16, 384, 1024, 16, 4),
    (70, 200, 640, 16, 4),
    (130, 256, 512, 64, 4),
    (16, 256, 512, 8, 2),
    (100, 256, 512, 0, 2),
]


@pytest.mark.parametrize("m,n,k,rank,bits", BWD_CASES)
def test_linear_bwd_parity(lbq, m, n, k, rank, bits):
    s = 2.0
    X, W, A, B = fwd_problem(m, n, k, rank, seed=m + 7 * n + k + rank)
    dY = syn.normal_bf16((m, n), 0.1, seed=m + n + 99)
    qw = device_qweight(lbq, W, "minmax", bits, False, None)
    dX, U = lbq.linear_bwd(dY.cuda(), qw, None if A is None else A.cuda(), None if B is None else B.cuda(), s)
    torch.cuda.synchronize()
    What = oracle_weight(W, "minmax", bits, False, None)
    dXr, Ur, dXb = oracle.linear_bwd(syn.bits_u16(dY), What, None if A is None else syn.bits_u16(A),
                                     None if B is None else syn.bits_u16(B), s)
    assert_within(dX.cpu().numpy(), dXr, dXb, "dX")
    if rank:
        Ub = np.abs(oracle.bf16_to_f32(syn.bits_u16(dY))).astype(np.float64) @ \
            np.abs(oracle.bf16_to_f32(syn.bits_u16(B))).astype(np.float64)
        assert_within(U.cpu().numpy(), Ur, Ub, "U")
    assert_status_clean(lbq)


@pytest.mark.parametrize("m,n,k,rank", [(8, 256, 512, 8), (130, 384, 768, 16), (64, 200, 512, 64), (300, 264, 640, 6),
                                         (1000, 512, 1024, 12)])
def test_lora_grads_parity(lbq, m, n, k, rank):
    s = 2.0
    X, W, A, B = fwd_problem(m, n, k, rank, seed=m + n + k)
    dY = syn.normal_bf16((m, n), 0.1, seed=m * 3 + 1)
    qw = device_qweight(lbq, W, "minmax", 4, False, None)
    _, T = lbq.linear_fwd(X.cuda(), qw, A.cuda(), B.cuda(), s)
    _, U = lbq.linear_bwd(dY.cuda(), qw, A.cuda(), B.cuda(), s)
    dA, dB = lbq.lora_grads(X.cuda(), dY.cuda(), T, U, s)
    torch.cuda.synchronize()
    dAr, dBr, dAb, dBb = oracle.lora_grads(syn.bits_u16(X), syn.bits_u16(dY), syn.bits_u16(A), syn.bits_u16(B), s)
    assert_within(dA.cpu().numpy(), dAr, dAb, "dA")
    assert_within(dB.cpu().numpy(), dBr, dBb, "dB")
    assert_status_clean(lbq)


# --------------------------------------------------------------------------- full-size training step
@pytest.fixture(scope="module")
def train_problem(lbq):
    """The 8B MLP gate layer of the QLoRA step at full size: W 14336 x 4096
    INT4 g128, M = 4096 tokens, rank 16, s = 2 (the benchmark's training row)."""
    m, n, k, r, s = 4096, 14336, 4096, 16, 2.0
    W = syn.weight_bf16(n, k, 0.02, seed=41, outlier_frac=0.001)
    X = syn.normal_bf16((m, k), 1.0, seed=42)
    A = syn.normal_bf16((r, k), 0.01, seed=43)
    B = syn.normal_bf16((n, r), 0.01, seed=44)
    dY = syn.normal_bf16((m, n), 0.1, seed=45)
    codes, scale, zero = oracle.minmax_quantize(syn.bits_u16(W), 4, 128)
    packed = oracle.pack(codes, 4)
    qw = lbq.QuantizedWeight(n, k, "minmax", 4)
    qw.packed.copy_(torch.from_numpy(packed))
    qw.scale.copy_(torch.from_numpy(scale.view(np.float16)))
    qw.zero.copy_(torch.from_numpy(zero.view(np.float16)))
    Xd, Ad, Bd, dYd = X.cuda(), A.cuda(), B.cuda(), dY.cuda()
    Y, T = lbq.linear_fwd(Xd, qw, Ad, Bd, s)
    dX, U = lbq.linear_bwd(dYd, qw, Ad, Bd, s)
    dA, dB = lbq.lora_grads(Xd, dYd, T, U, s)
    torch.cuda.synchronize()
    return dict(m=m, n=n, k=k, r=r, s=s, X=X, A=A, B=B, dY=dY, packed=packed, scale=scale, zero=zero,
                Y=Y.cpu().numpy(), dX=dX.cpu().numpy(), dA=dA.cpu().numpy(), dB=dB.cpu().numpy())


def _sample_pairs(nr, nc, count, seed):
    """`count` seeded (row, col) pairs plus one full row and one full column."""
    rng = np.random.default_rng(seed)
    r = rng.integers(0, nr, count)
    c = rng.integers(0, nc, count)
    fr, fc = int(rng.integers(0, nr)), int(rng.integers(0, nc))
    rows = np.concatenate([r, np.full(nc, fr), np.arange(nr)])
    cols = np.concatenate([c, np.arange(nc), np.full(nr, fc)])
    return rows, cols


def test_training_forward_full_size_sampled(lbq, train_problem):
    P = train_problem
    rows, cols = _sample_pairs(P["m"], P["n"], 4096, seed=5)
    ref, bound = oracle.linear_fwd_sampled_minmax(syn.bits_u16(P["X"]), P["packed"], P["scale"], P["zero"],
                                                  P["n"], P["k"], 4, 128, rows, cols, syn.bits_u16(P["A"]),
                                                  syn.bits_u16(P["B"]), P["s"])
    assert_within(P["Y"][rows, cols], ref, bound, "Y")


def test_training_backward_full_size_sampled(lbq, train_problem):
    P = train_problem
    rows, cols = _sample_pairs(P["m"], P["k"], 2048, seed=6)
    ref, bound = oracle.linear_bwd_sampled_minmax(syn.bits_u16(P["dY"]), P["packed"], P["scale"], P["zero"],
                                                  P["n"], P["k"], 4, 128, rows, cols, syn.bits_u16(P["A"]),
                                                  syn.bits_u16(P["B"]), P["s"])
    assert_within(P["dX"][rows, cols], ref, bound, "dX")


def test_training_lora_grads_full_size(lbq, train_problem):
    P = train_problem
    dA, dB, dAb, dBb = oracle.lora_grads(syn.bits_u16(P["X"]), syn.bits_u16(P["dY"]), syn.bits_u16(P["A"]),
                                         syn.bits_u16(P["B"]), P["s"])
    assert_within(P["dA"], dA, dAb, "dA")
    assert_within(P["dB"], dB, dBb, "dB")


# --------------------------------------------------------------------------- full-size 70B codebook layer
@pytest.fixture(scope="module")
def codebook70b(lbq):
    """The 70B attention projection (8192 x 8192) in the 4-bit codebook
    format with double quantization, quantized on the GPU, at the benchmark's
    sizes."""
    n = k = 8192
    cb = syn.codebook_normal16()
    W = syn.weight_bf16(n, k, 0.015, seed=71)
    qw = lbq.QuantizedWeight(n, k, "codebook", double_quant=True, codebook=cb).quantize(W.cuda())
    torch.cuda.synchronize()
    codes, absmax = oracle.codebook_quantize(syn.bits_u16(W), cb)
    packed = oracle.pack(codes, 4)
    q8, s2, off, exact = oracle.double_quant(absmax)
    What = oracle.codebook_dequantize(packed, oracle.double_dequant(q8, s2, off), cb, n, k)
    return dict(n=n, k=k, qw=qw, packed=packed, q8=q8, s2=s2, off=off, exact=exact, What=What)


def test_codebook70b_quantize_full_size(lbq, codebook70b):
    C = codebook70b
    assert C["exact"]
    assert np.array_equal(C["qw"].packed.cpu().numpy(), C["packed"])
    assert np.array_equal(C["qw"].q8.cpu().numpy(), C["q8"])
    assert np.array_equal(C["qw"].s2.cpu().numpy().view(np.uint32), C["s2"].view(np.uint32))
    assert np.float32(C["qw"].offset[0].item()).view(np.uint32) == np.float32(C["off"]).view(np.uint32)
    assert_status_clean(lbq)


def test_codebook70b_decode_full_size(lbq, codebook70b):
    C = codebook70b
    X = syn.normal_bf16((1, C["k"]), 1.0, seed=72)
    Y, _ = lbq.linear_fwd(X.cuda(), C["qw"])
    torch.cuda.synchronize()
    Yr, _, Yb = oracle.linear_fwd(syn.bits_u16(X), C["What"])
    assert_within(Y.cpu().numpy(), Yr, Yb, "Y")


def test_codebook70b_decode_m16_full_size(lbq, codebook70b):
    # 16 tokens: the grid takes two waves, so tile owners also wait on
    # contributors of the earlier wave
    C = codebook70b
    X = syn.normal_bf16((16, C["k"]), 1.0, seed=74)
    Y, _ = lbq.linear_fwd(X.cuda(), C["qw"])
    torch.cuda.synchronize()
    Yr, _, Yb = oracle.linear_fwd(syn.bits_u16(X), C["What"])
    assert_within(Y.cpu().numpy(), Yr, Yb, "Y")
    assert_status_clean(lbq)


def test_codebook70b_prefill_full_size_sampled(lbq, codebook70b):
    C = codebook70b
    m = 2048
    X = syn.normal_bf16((m, C["k"]), 1.0, seed=73)
    Y, _ = lbq.linear_fwd(X.cuda(), C["qw"])
    torch.cuda.synchronize()
    rows, cols = _sample_pairs(m, C["n"], 2048, seed=7)
    x = oracle.bf16_to_f32(syn.bits_u16(X))
    w = C["What"]
    ref = np.empty(rows.size)
    bound = np.empty(rows.size)
    for i in range(0, rows.size, 1024):          # sampled dot products, a chunk at a time
        xr = x[rows[i:i + 1024]].astype(np.float64)
        wc = w[cols[i:i + 1024]].astype(np.float64)
        ref[i:i + 1024] = np.einsum("ij,ij->i", xr, wc)
        bound[i:i + 1024] = np.einsum("ij,ij->i", np.abs(xr), np.abs(wc))
    assert_within(Y.cpu().numpy()[rows, cols], ref, bound, "Y")
    assert_status_clean(lbq)


# --------------------------------------------------------------------------- adapter merge
MERGE_CASES = [
    # n, k, rank, scheme, bits, dq
    (256, 512, 16, "minmax", 4, False),
    (200, 640, 8, "minmax", 2, False),      # ragged rows (200 = 3 x 64 + 8)
    (130, 1024, 64, "minmax", 4, False),    # rank 64: two staged chunks of the adapter
    (96, 448, 40, "codebook", 4, True),     # codebook + double quant; rank 40 = 32 + 8; k = 3.5 column tiles
    (64, 192, 5, "codebook", 4, False),
    (128, 256, 0, "minmax", 4, False),      # no adapter: bf16 of the dequantized weight
]


def _merge_inputs(n, k, rank, seed):
    A = syn.normal_bf16((rank, k), 0.05, seed + 2) if rank else None
    B = syn.normal_bf16((n, rank), 0.05, seed + 3) if rank else None
    return A, B


@pytest.mark.parametrize("n,k,rank,scheme,bits,dq", MERGE_CASES)
def test_merge_bit_exact(lbq, n, k, rank, scheme, bits, dq):
    seed = n + k + rank
    cb = syn.codebook_normal16() if scheme == "codebook" else None
    W = mixed_weight(n, k, seed) if scheme == "minmax" else syn.weight_bf16(n, k, 0.015, seed)
    qw = device_qweight(lbq, W, scheme, bits, dq, cb)
    A, B = _merge_inputs(n, k, rank, seed)
    s = 2.0
    out = lbq.merge_lora(qw, A.cuda() if rank else None, B.cuda() if rank else None, s)
    torch.cuda.synchronize()
    ref = oracle.lora_merge(oracle_weight(W, scheme, bits, dq, cb), syn.bits_u16(A) if rank else None,
                            syn.bits_u16(B) if rank else None, s, 1)
    assert np.array_equal(u16(out), ref)
    assert_status_clean(lbq)


def test_merge_sums_the_rank_in_order(lbq):
    # products 1, 2^-30, -1 in every element: summed in order they cancel to
    # exactly 0, so the merged weight is bf16(W_hat) itself
    n, k = 64, 128
    W = mixed_weight(n, k, 3)
    qw = device_qweight(lbq, W, "minmax", 4, False, None)
    A = torch.tensor([[1.0], [2.0 ** -15], [1.0]]).repeat(1, k).to(torch.bfloat16)
    B = torch.tensor([[1.0, 2.0 ** -15, -1.0]]).repeat(n, 1).to(torch.bfloat16)
    out = lbq.merge_lora(qw, A.cuda(), B.cuda(), 1.0)
    torch.cuda.synchronize()
    What = oracle_weight(W, "minmax", 4, False, None)
    ref = oracle.lora_merge(What, syn.bits_u16(A), syn.bits_u16(B), 1.0, 1)
    assert np.array_equal(u16(out), ref)
    assert np.array_equal(ref, oracle.lora_merge(What, None, None, 1.0, 1))


@pytest.mark.parametrize("n,k,rank", [(192, 512, 16), (100, 200, 7)])
def test_unmerge_bit_exact_in_place(lbq, n, k, rank):
    W = syn.weight_bf16(n, k, 0.02, seed=n + k)
    A, B = _merge_inputs(n, k, rank, n)
    ref = oracle.lora_merge(oracle.bf16_to_f32(syn.bits_u16(W)).astype(np.float32), syn.bits_u16(A),
                            syn.bits_u16(B), 1.5, -1)
    Wd = W.cuda()
    out = lbq.unmerge_lora(Wd, A.cuda(), B.cuda(), 1.5)
    lbq.unmerge_lora(Wd, A.cuda(), B.cuda(), 1.5, out=Wd)
    torch.cuda.synchronize()
    assert np.array_equal(u16(out), ref)
    assert np.array_equal(u16(Wd), ref)
    assert_status_clean(lbq)


@pytest.mark.parametrize("scheme,bits,dq", [("minmax", 4, False), ("minmax", 2, False), ("codebook", 4, True)])
def test_merge_then_requantize_bit_exact(lbq, scheme, bits, dq):
    # re-quantizing the merged model: the merged bf16 weight goes through the
    # GPU quantizer and must give the oracle's codes and constants exactly
    n, k, rank, s = 256, 1024, 16, 2.0
    cb = syn.codebook_normal16() if scheme == "codebook" else None
    W = syn.weight_bf16(n, k, 0.02, seed=77, outlier_frac=0.01)
    qw = device_qweight(lbq, W, scheme, bits, dq, cb)
    A, B = _merge_inputs(n, k, rank, 77)
    merged = lbq.merge_lora(qw, A.cuda(), B.cuda(), s)
    q2 = lbq.QuantizedWeight(n, k, scheme, bits, double_quant=dq, codebook=cb).quantize(merged)
    torch.cuda.synchronize()
    mref = oracle.lora_merge(oracle_weight(W, scheme, bits, dq, cb), syn.bits_u16(A), syn.bits_u16(B), s, 1)
    if scheme == "minmax":
        codes, scale, zero = oracle.minmax_quantize(mref, bits, 128 if bits == 4 else 64)
        assert np.array_equal(q2.packed.cpu().numpy(), oracle.pack(codes, bits))
        assert np.array_equal(u16(q2.scale), scale)
        assert np.array_equal(u16(q2.zero), zero)
    else:
        codes, absmax = oracle.codebook_quantize(mref, cb)
        q8, s2, off, exact = oracle.double_quant(absmax)
        assert exact
        assert np.array_equal(q2.packed.cpu().numpy(), oracle.pack(codes, 4))
        assert np.array_equal(q2.q8.cpu().numpy(), q8)
        assert np.array_equal(q2.s2.cpu().numpy().view(np.uint32), s2.view(np.uint32))
    assert_status_clean(lbq)


def test_merge_full_size_gate(lbq, train_problem):
    # the 8B MLP gate matrix (14336 x 4096, INT4 g128) with its rank-16
    # adapter, every element against the oracle
    P = train_problem
    qw = lbq.QuantizedWeight(P["n"], P["k"], "minmax", 4)
    qw.packed.copy_(torch.from_numpy(P["packed"]))
    qw.scale.copy_(torch.from_numpy(P["scale"].view(np.float16)))
    qw.zero.copy_(torch.from_numpy(P["zero"].view(np.float16)))
    out = lbq.merge_lora(qw, P["A"].cuda(), P["B"].cuda(), P["s"])
    torch.cuda.synchronize()
    What = oracle.minmax_dequantize(P["packed"], P["scale"], P["zero"], P["k"], 4, 128)
    ref = oracle.lora_merge(What, syn.bits_u16(P["A"]), syn.bits_u16(P["B"]), P["s"], 1)
    assert np.array_equal(u16(out), ref)
    assert_status_clean(lbq)


# --------------------------------------------------------------------------- rounding ties on the GPU
@pytest.mark.parametrize("bits", [4, 2])
def test_minmax_quantize_ties_bit_exact(lbq, bits):
    """Groups where many w / scale land exactly on k + 1/2 (and zero points
    exactly half-way): the GPU quantizer's codes, scales and zeros equal the
    oracle's and the exact-rational expectation (half to even) bit for bit."""
    from tie_inputs import tie_weight
    group = 128 if bits == 4 else 64
    n, k = 256, 8 * group
    w, codes_exp, zeros_exp, scales_exp = tie_weight(n, k, bits, seed=10 + bits)
    W = torch.from_numpy(w).to(torch.bfloat16)
    qw = lbq.QuantizedWeight(n, k, "minmax", bits).quantize(W.cuda())
    torch.cuda.synchronize()
    codes, scale, zero = oracle.minmax_quantize(syn.bits_u16(W), bits, group)
    assert np.array_equal(codes.astype(np.int64), codes_exp)
    assert np.array_equal(qw.packed.cpu().numpy(), oracle.pack(codes, bits)), "packed codes differ"
    assert np.array_equal(u16(qw.scale), scale), "scales differ"
    assert np.array_equal(u16(qw.zero), zero), "zeros differ"
    assert np.array_equal(qw.scale.cpu().numpy().astype(np.float64), scales_exp)
    assert np.array_equal(qw.zero.cpu().numpy().astype(np.float64), zeros_exp)
    assert_status_clean(lbq)


# --------------------------------------------------------------------------- channel-mix
def _channel_mix(lbq, W, frac, seed):
    """ChannelMixWeight of W (bf16 CPU [n, k]) with the oracle's quantization
    of both halves; returns (mix, perm, n4, (packed, scale, zero) of hi and lo)."""
    n, k = W.shape
    perm, n4 = syn.channel_mix_perm(n, frac, seed=seed)
    Wp = W[torch.from_numpy(perm.astype(np.int64))]
    halves = []
    for rows, bits in ((slice(0, n4), 4), (slice(n4, n), 2)):
        Wh = Wp[rows].contiguous()
        codes, scale, zero = oracle.minmax_quantize(syn.bits_u16(Wh), bits, 128 if bits == 4 else 64)
        halves.append((oracle.pack(codes, bits), scale, zero))
    qws = []
    for (packed, scale, zero), nn, bits in ((halves[0], n4, 4), (halves[1], n - n4, 2)):
        qw = lbq.QuantizedWeight(nn, k, "minmax", bits)
        qw.packed.copy_(torch.from_numpy(packed))
        qw.scale.copy_(torch.from_numpy(scale.view(np.float16)))
        qw.zero.copy_(torch.from_numpy(zero.view(np.float16)))
        qws.append(qw)
    torch.cuda.synchronize()
    return lbq.ChannelMixWeight(qws[0], qws[1], perm), perm, n4, halves


def _channel_mix_sampled_ref(X, perm, n4, halves, k, tok, col, A, B, s):
    """Oracle Y and bound at (tok[i], col[i]) (original output columns) of a
    channel-mix weight: each sample goes to the half that stores its column,
    with the adapter rows of B taken in stored order."""
    n = perm.size
    inv = np.empty(n, np.int64)
    inv[perm] = np.arange(n)
    ref = np.empty(tok.size)
    bound = np.empty(tok.size)
    Bb = None if B is None else syn.bits_u16(B)
    for lo_, hi_, (packed, scale, zero), bits in ((0, n4, halves[0], 4), (n4, n, halves[1], 2)):
        sel = (inv[col] >= lo_) & (inv[col] < hi_)
        if not sel.any():
            continue
        stored = inv[col[sel]] - lo_
        Bh = None if Bb is None else np.ascontiguousarray(Bb[perm[lo_:hi_]])
        r, b = oracle.linear_fwd_sampled_minmax(syn.bits_u16(X), packed, scale, zero, hi_ - lo_, k, bits,
                                                128 if bits == 4 else 64, tok[sel], stored,
                                                None if A is None else syn.bits_u16(A), Bh, s)
        ref[sel], bound[sel] = r, b
    return ref, bound


def test_channel_mix_fwd_full_gate_m512(lbq):
    """Channel-mix 25 % INT4 g128 / 75 % INT2 g64 on the 8B gate matrix
    (14336 x 4096) at M = 512 with a rank-16 adapter: the tensor-core path
    with the stored permutation applied in its epilogue; 4096 seeded
    elements plus one full row and one full column against the oracle."""
    m, n, k, r, s = 512, 14336, 4096, 16, 2.0
    W = syn.weight_bf16(n, k, 0.02, seed=301, outlier_frac=0.001)
    X = syn.normal_bf16((m, k), 1.0, seed=302)
    A = syn.normal_bf16((r, k), 0.01, seed=303)
    B = syn.normal_bf16((n, r), 0.01, seed=304)
    mix, perm, n4, halves = _channel_mix(lbq, W, 0.25, seed=5)
    Y, _ = lbq.linear_fwd(X.cuda(), mix, A.cuda(), B.cuda(), s)
    torch.cuda.synchronize()
    tok, col = _sample_pairs(m, n, 4096, seed=8)
    ref, bound = _channel_mix_sampled_ref(X, perm, n4, halves, k, tok, col, A, B, s)
    assert_within(Y.cpu().numpy()[tok, col], ref, bound, "Y (channel-mix, M=512)")
    assert_status_clean(lbq)


@pytest.mark.parametrize("m", [1, 16, 40])
def test_channel_mix_grouped_layer_set(lbq, m):
    """Four channel-mix layers (8B q, k and gate shapes, plus ragged halves of
    1000 rows) in one grouped call, with a rank-8 adapter on two of them:
    every output element of every layer against the oracle (m <= 16 runs the
    halves as grouped decode launches, m = 40 the tensor-core GEMMs)."""
    k, r, s = 4096, 8, 2.0
    shapes = [(4096, 0), (1024, r), (14336, 0), (1000, r)]
    X = syn.normal_bf16((m, k), 1.0, seed=900 + m)
    probs, refs = [], []
    for i, (n, rank) in enumerate(shapes):
        W = mixed_weight(n, k, seed=910 + i) if n == 1000 else syn.weight_bf16(n, k, 0.02, seed=910 + i,
                                                                                 outlier_frac=0.001)
        mix, perm, n4, halves = _channel_mix(lbq, W, 0.25, seed=920 + i)
        What = np.zeros((n, k), np.float32)
        for (packed, scale, zero), rows, bits in ((halves[0], perm[:n4], 4), (halves[1], perm[n4:], 2)):
            What[rows] = oracle.minmax_dequantize(packed, scale, zero, k, bits, 128 if bits == 4 else 64)
        if rank:
            A = syn.normal_bf16((rank, k), 0.01, seed=930 + i)
            B = syn.normal_bf16((n, rank), 0.01, seed=940 + i)
            probs.append((X.cuda(), mix, A.cuda(), B.cuda(), s))
            refs.append(oracle.linear_fwd(syn.bits_u16(X), What, syn.bits_u16(A), syn.bits_u16(B), s))
        else:
            probs.append((X.cuda(), mix))
            refs.append(oracle.linear_fwd(syn.bits_u16(X), What))
    outs = lbq.linear_fwd_mix_grouped(probs)
    torch.cuda.synchronize()
    for (Y, _), (Yr, _, Yb), (n, _) in zip(outs, refs, shapes):
        assert_within(Y.cpu().numpy(), Yr, Yb, f"Y (grouped channel-mix, n={n}, M={m})")
    assert_status_clean(lbq)


@pytest.mark.parametrize("m", [16, 512])
def test_channel_mix_ragged_halves(lbq, m):
    """Halves that are not whole 128-row tiles (250 INT4 rows, 750 INT2 rows),
    every output element against the oracle."""
    n, k, r, s = 1000, 1024, 8, 2.0
    W = mixed_weight(n, k, seed=n + m)
    X = syn.normal_bf16((m, k), 1.0, seed=m + 5)
    A = syn.normal_bf16((r, k), 0.01, seed=6)
    B = syn.normal_bf16((n, r), 0.01, seed=7)
    mix, perm, n4, halves = _channel_mix(lbq, W, 0.25, seed=3)
    assert n4 % 128 != 0 and (n - n4) % 128 != 0
    Y, _ = lbq.linear_fwd(X.cuda(), mix, A.cuda(), B.cuda(), s)
    torch.cuda.synchronize()
    What = np.zeros((n, k), np.float32)
    for (packed, scale, zero), rows, bits in ((halves[0], perm[:n4], 4), (halves[1], perm[n4:], 2)):
        What[rows] = oracle.minmax_dequantize(packed, scale, zero, k, bits, 128 if bits == 4 else 64)
    Yr, _, Yb = oracle.linear_fwd(syn.bits_u16(X), What, syn.bits_u16(A), syn.bits_u16(B), s)
    assert_within(Y.cpu().numpy(), Yr, Yb, f"Y (channel-mix, ragged halves, M={m})")
    assert_status_clean(lbq)


# --------------------------------------------------------------------------- INT2 on the tensor cores at full size
@pytest.mark.parametrize("name", ["gate", "down"])
def test_int2_fwd_full_size_m512(lbq, name):
    """Layer-mix INT2 g64 on the full 8B gate (14336 x 4096) and down
    (4096 x 14336) matrices at M = 512 through the tensor-core GEMM: 4096
    seeded elements plus a full row and a full column."""
    m = 512
    n, k = syn.LLAMA3_8B_SHAPES[name]
    W = syn.weight_bf16(n, k, 0.02, seed=311 + n, outlier_frac=0.001)
    X = syn.normal_bf16((m, k), 1.0, seed=312)
    codes, scale, zero = oracle.minmax_quantize(syn.bits_u16(W), 2, 64)
    packed = oracle.pack(codes, 2)
    qw = lbq.QuantizedWeight(n, k, "minmax", 2)
    qw.packed.copy_(torch.from_numpy(packed))
    qw.scale.copy_(torch.from_numpy(scale.view(np.float16)))
    qw.zero.copy_(torch.from_numpy(zero.view(np.float16)))
    Y, _ = lbq.linear_fwd(X.cuda(), qw)
    torch.cuda.synchronize()
    tok, col = _sample_pairs(m, n, 4096, seed=9)
    ref, bound = oracle.linear_fwd_sampled_minmax(syn.bits_u16(X), packed, scale, zero, n, k, 2, 64, tok, col)
    assert_within(Y.cpu().numpy()[tok, col], ref, bound, f"Y (INT2 {name}, M=512)")
    assert_status_clean(lbq)


# --------------------------------------------------------------------------- 70B codebook MLP matrices at full size
@pytest.mark.parametrize("name", ["gate", "down"])
def test_codebook70b_mlp_full_size(lbq, name):
    """The 70B gate (28672 x 8192) and down (8192 x 28672) matrices in the
    4-bit codebook format with double quantization, quantized on the GPU:
    codes, q8, s2 and offset bit-exact against the oracle; M = 1 every output;
    M = 2048 on 2048 seeded elements plus a full row and a full column."""
    n, k = syn.LLAMA3_70B_SHAPES[name]
    cb = syn.codebook_normal16()
    W = syn.weight_bf16(n, k, 0.015, seed=321 + n)
    qw = lbq.QuantizedWeight(n, k, "codebook", double_quant=True, codebook=cb).quantize(W.cuda())
    torch.cuda.synchronize()
    codes, absmax = oracle.codebook_quantize(syn.bits_u16(W), cb)
    del W
    packed = oracle.pack(codes, 4)
    del codes
    q8, s2, off, exact = oracle.double_quant(absmax)
    assert exact
    assert np.array_equal(qw.packed.cpu().numpy(), packed)
    assert np.array_equal(qw.q8.cpu().numpy(), q8)
    assert np.array_equal(qw.s2.cpu().numpy().view(np.uint32), s2.view(np.uint32))
    assert np.float32(qw.offset[0].item()).view(np.uint32) == np.float32(off).view(np.uint32)
    What = oracle.codebook_dequantize(packed, oracle.double_dequant(q8, s2, off), cb, n, k)
    del packed
    for m, seed in ((1, 322), (2048, 323)):
        X = syn.normal_bf16((m, k), 1.0, seed=seed)
        Y, _ = lbq.linear_fwd(X.cuda(), qw)
        torch.cuda.synchronize()
        Yc = Y.cpu().numpy()
        x = oracle.bf16_to_f32(syn.bits_u16(X))
        if m == 1:
            xr = x[0].astype(np.float64)
            ref = np.empty(n)
            bound = np.empty(n)
            for i in range(0, n, 2048):
                wc = What[i:i + 2048].astype(np.float64)
                ref[i:i + 2048] = wc @ xr
                bound[i:i + 2048] = np.abs(wc) @ np.abs(xr)
            assert_within(Yc[0], ref, bound, f"Y (70B {name}, M=1)")
        else:
            rows, cols = _sample_pairs(m, n, 2048, seed=seed)
            ref = np.empty(rows.size)
            bound = np.empty(rows.size)
            for i in range(0, rows.size, 512):
                xr = x[rows[i:i + 512]].astype(np.float64)
                wc = What[cols[i:i + 512]].astype(np.float64)
                ref[i:i + 512] = np.einsum("ij,ij->i", xr, wc)
                bound[i:i + 512] = np.einsum("ij,ij->i", np.abs(xr), np.abs(wc))
            assert_within(Yc[rows, cols], ref, bound, f"Y (70B {name}, M=2048)")
        del X, Y
    assert_status_clean(lbq)


# --------------------------------------------------------------------------- bounded waits
def test_bounded_wait_times_out_and_context_survives(lbq):
    """A kernel whose waits can never be satisfied gives up after the short
    limit, records the timeout in the status word and returns; the device
    stays usable: a forward with a freshly zeroed workspace afterwards matches
    the oracle and leaves the status clean."""
    import ctypes
    stream = torch.cuda.current_stream().cuda_stream
    assert lbq.lbq_selftest_wait_timeout(0, stream) == lbq.LBQ_EINVAL
    assert lbq.lbq_selftest_wait_timeout(2000, stream) == lbq.LBQ_OK
    assert lbq.device_status() & lbq.STATUS_TIMEOUT
    assert lbq.device_status() == 0                    # read-and-clear
    m, n, k = 4, 1024, 4096
    X, W, _, _ = fwd_problem(m, n, k, 0, seed=12)
    qw = device_qweight(lbq, W, "minmax", 4, False, None)
    ws = lbq._workspace(lbq.lbq_linear_fwd_workspace_size(m, ctypes.byref(qw.struct), 0), "cuda")
    Y, _ = lbq.linear_fwd(X.cuda(), qw, workspace=ws)
    torch.cuda.synchronize()
    Yr, _, Yb = oracle.linear_fwd(syn.bits_u16(X), oracle_weight(W, "minmax", 4, False, None))
    assert_within(Y.cpu().numpy(), Yr, Yb, "Y after a timed-out wait")
    assert_status_clean(lbq)


# --------------------------------------------------------------------------- grouped forward (one launch per layer set)
@pytest.fixture(scope="module")
def layer_set_8b(lbq):
    """The seven LLaMA-3-8B layers (q, k, v, o, gate, up, down), INT4 g128
    with the oracle's quantization, as the decode benchmark runs them."""
    out = {}
    for i, (name, (n, k)) in enumerate(syn.LLAMA3_8B_SHAPES.items()):
        W = syn.weight_bf16(n, k, 0.02, seed=400 + i, outlier_frac=0.001)
        codes, scale, zero = oracle.minmax_quantize(syn.bits_u16(W), 4, 128)
        packed = oracle.pack(codes, 4)
        qw = lbq.QuantizedWeight(n, k, "minmax", 4)
        qw.packed.copy_(torch.from_numpy(packed))
        qw.scale.copy_(torch.from_numpy(scale.view(np.float16)))
        qw.zero.copy_(torch.from_numpy(zero.view(np.float16)))
        out[name] = (qw, packed, scale, zero)
    torch.cuda.synchronize()
    return out


@pytest.mark.parametrize("m", [1, 16])
def test_grouped_fwd_8b_layer_set_full(lbq, layer_set_8b, m):
    """One grouped call over the whole 8B layer set (one launch of the decode
    GEMV): every output element of every layer against the oracle."""
    Xs = {k: syn.normal_bf16((m, k), 1.0, seed=410 + k + m) for k in (4096, 14336)}
    Xd = {k: x.cuda() for k, x in Xs.items()}
    names = list(syn.LLAMA3_8B_SHAPES)
    outs = lbq.linear_fwd_grouped([(Xd[layer_set_8b[nm][0].k], layer_set_8b[nm][0]) for nm in names])
    torch.cuda.synchronize()
    for nm, (Y, _) in zip(names, outs):
        qw, packed, scale, zero = layer_set_8b[nm]
        tok = np.repeat(np.arange(m), qw.n)
        col = np.tile(np.arange(qw.n), m)
        ref, bound = oracle.linear_fwd_sampled_minmax(syn.bits_u16(Xs[qw.k]), packed, scale, zero, qw.n, qw.k, 4, 128,
                                                      tok, col)
        assert_within(Y.cpu().numpy().reshape(-1), ref, bound, f"Y ({nm}, M={m}, grouped)")
    assert_status_clean(lbq)


GROUP_CASES = [
    # n, k, scheme, bits, dq, rank
    (256, 512, "minmax", 4, False, 8),
    (300, 1024, "minmax", 2, False, 0),
    (200, 640, "codebook", 4, True, 16),
    (128, 192, "codebook", 4, False, 0),
    (130, 384, "minmax", 4, False, 4),      # ragged rows, far zero points (mixed_weight)
    (1000, 2048, "minmax", 4, False, 0),
]


@pytest.mark.parametrize("m", [1, 5, 16])
def test_grouped_fwd_mixed_kinds(lbq, m):
    """INT4, INT2 and codebook weights (with and without double
    quantization), ragged shapes and adapters in one grouped launch; each
    output against the oracle."""
    cb = syn.codebook_normal16()
    probs, refs = [], []
    for i, (n, k, scheme, bits, dq, rank) in enumerate(GROUP_CASES):
        X, W, A, B = fwd_problem(m, n, k, rank, seed=500 + 17 * i + m, scheme=scheme, bits=bits)
        qw = device_qweight(lbq, W, scheme, bits, dq, cb)
        s = 1.5
        probs.append((X.cuda(), qw, None if A is None else A.cuda(), None if B is None else B.cuda(), s))
        Yr, Tr, Yb = oracle.linear_fwd(syn.bits_u16(X), oracle_weight(W, scheme, bits, dq, cb),
                                       None if A is None else syn.bits_u16(A), None if B is None else syn.bits_u16(B), s)
        refs.append((Yr, Yb))
    outs = lbq.linear_fwd_grouped(probs)
    torch.cuda.synchronize()
    for i, ((Y, _), (Yr, Yb)) in enumerate(zip(outs, refs)):
        assert_within(Y.cpu().numpy(), Yr, Yb, f"Y (problem {i}, M={m})")
    assert_status_clean(lbq)


# Tall weights for the grouped tensor-core launch: together their 128-row
# tiles fill the B200's CTA slots (296 at the 64-token tile, 148 at 256), so
# the problems run in one grouped launch instead of one launch each.
GROUP_TC_CASES = [
    # n, k, scheme, bits, dq, rank
    (8704, 256, "minmax", 4, False, 8),
    (10000, 512, "minmax", 2, False, 0),     # ragged rows
    (6144, 384, "codebook", 4, True, 16),
    (4100, 256, "codebook", 4, False, 0),    # ragged rows
    (9000, 256, "minmax", 4, False, 4),      # far zero points (mixed_weight)
]


@pytest.mark.parametrize("m", [40, 300])
def test_grouped_fwd_tensor_core_launch(lbq, m):
    """m > 16 with INT4, INT2 and codebook weights, adapters and ragged row
    counts in one grouped tensor-core launch (every CTA picks its problem and
    weight kind); each output against the oracle."""
    cb = syn.codebook_normal16()
    tile = 64 if m <= 64 else 256
    tiles = sum(-(-n // 128) * -(-m // tile) for (n, *_) in GROUP_TC_CASES)
    assert tiles >= (2 if tile < 256 else 1) * 148          # the grouped path
    probs, refs = [], []
    for i, (n, k, scheme, bits, dq, rank) in enumerate(GROUP_TC_CASES):
        X, W, A, B = fwd_problem(m, n, k, rank, seed=700 + 13 * i + m, scheme=scheme, bits=bits)
        qw = device_qweight(lbq, W, scheme, bits, dq, cb)
        s = 2.0
        probs.append((X.cuda(), qw, None if A is None else A.cuda(), None if B is None else B.cuda(), s))
        Yr, Tr, Yb = oracle.linear_fwd(syn.bits_u16(X), oracle_weight(W, scheme, bits, dq, cb),
                                       None if A is None else syn.bits_u16(A), None if B is None else syn.bits_u16(B), s)
        refs.append((Yr, Yb))
    outs = lbq.linear_fwd_grouped(probs)
    torch.cuda.synchronize()
    for i, ((Y, _), (Yr, Yb)) in enumerate(zip(outs, refs)):
        assert_within(Y.cpu().numpy(), Yr, Yb, f"Y (problem {i}, M={m})")
    assert_status_clean(lbq)


@pytest.mark.parametrize("m", [3, 40])
def test_grouped_fwd_more_than_one_launch(lbq, m):
    """Ten weights: two launches of the decode GEMV (m <= 16), or ten
    tensor-core GEMMs one after the other (m > 16), sharing one workspace."""
    probs, refs = [], []
    for i in range(10):
        n, k = 128 * (1 + i % 3), 256 * (1 + i % 2)
        X, W, _, _ = fwd_problem(m, n, k, 0, seed=600 + i)
        qw = device_qweight(lbq, W, "minmax", 4 if i % 2 == 0 else 2, False, None)
        probs.append((X.cuda(), qw))
        Yr, _, Yb = oracle.linear_fwd(syn.bits_u16(X), oracle_weight(W, "minmax", 4 if i % 2 == 0 else 2, False, None))
        refs.append((Yr, Yb))
    outs = lbq.linear_fwd_grouped(probs)
    torch.cuda.synchronize()
    for i, ((Y, _), (Yr, Yb)) in enumerate(zip(outs, refs)):
        assert_within(Y.cpu().numpy(), Yr, Yb, f"Y (problem {i}, M={m})")
    assert_status_clean(lbq)


# --------------------------------------------------------------------------- backward through codebook weights
CB_BWD_CASES = [
    # m, n, k, rank, dq
    (8, 256, 512, 8, False),
    (1, 128, 1024, 0, True),
    (70, 200, 640, 16, True),      # ragged features and channels
    (300, 264, 1024, 4, False),
    (130, 512, 192, 0, True),      # k = 3 codebook blocks
]


@pytest.mark.parametrize("m,n,k,rank,dq", CB_BWD_CASES)
def test_linear_bwd_codebook_parity(lbq, m, n, k, rank, dq):
    """Gradients through the frozen 4-bit codebook weight (QLoRA explainer,
    QLoRA技术原理): dX and U against the oracle on codebook (and double
    quantized) weights."""
    s = 2.0
    cb = syn.codebook_normal16()
    X, W, A, B = fwd_problem(m, n, k, rank, seed=m + 3 * n + k, scheme="codebook")
    dY = syn.normal_bf16((m, n), 0.1, seed=m + n + 7)
    qw = device_qweight(lbq, W, "codebook", 4, dq, cb)
    dX, U = lbq.linear_bwd(dY.cuda(), qw, None if A is None else A.cuda(), None if B is None else B.cuda(), s)
    torch.cuda.synchronize()
    What = oracle_weight(W, "codebook", 4, dq, cb)
    dXr, Ur, dXb = oracle.linear_bwd(syn.bits_u16(dY), What, None if A is None else syn.bits_u16(A),
                                     None if B is None else syn.bits_u16(B), s)
    assert_within(dX.cpu().numpy(), dXr, dXb, "dX (codebook)")
    if rank:
        Ub = np.abs(oracle.bf16_to_f32(syn.bits_u16(dY))).astype(np.float64) @ \
            np.abs(oracle.bf16_to_f32(syn.bits_u16(B))).astype(np.float64)
        assert_within(U.cpu().numpy(), Ur, Ub, "U (codebook)")
    assert_status_clean(lbq)


# Wide weights for the grouped backward: at M = 300 (two 256-token tiles)
# their 128-feature tiles fill the B200's 148 CTA slots together.
GROUP_BWD_CASES = [
    # n, k, scheme, bits, dq, rank
    (512, 4096, "minmax", 4, False, 16),
    (264, 3072, "minmax", 2, False, 0),
    (256, 2048, "codebook", 4, True, 8),
    (136, 1536, "minmax", 4, False, 0),      # far zero points (mixed_weight)
]


@pytest.mark.parametrize("m", [40, 300])
def test_grouped_bwd(lbq, m):
    """Several backward passes in one call: at M = 300 one grouped tensor-core
    launch (every CTA picks its problem and weight kind), at M = 40 (too few
    tiles) one launch each; dX and U against the oracle."""
    cb = syn.codebook_normal16()
    tiles = sum(-(-k // 128) for (_, k, *_) in GROUP_BWD_CASES) * -(-m // 256)
    assert (tiles >= 148) == (m == 300)                        # which path each case takes
    probs, refs = [], []
    for i, (n, k, scheme, bits, dq, rank) in enumerate(GROUP_BWD_CASES):
        X, W, A, B = fwd_problem(m, n, k, rank, seed=800 + 11 * i + m, scheme=scheme, bits=bits)
        dY = syn.normal_bf16((m, n), 0.1, seed=900 + i + m)
        qw = device_qweight(lbq, W, scheme, bits, dq, cb)
        s = 2.0
        probs.append((dY.cuda(), qw, None if A is None else A.cuda(), None if B is None else B.cuda(), s))
        What = oracle_weight(W, scheme, bits, dq, cb)
        dXr, Ur, dXb = oracle.linear_bwd(syn.bits_u16(dY), What, None if A is None else syn.bits_u16(A),
                                         None if B is None else syn.bits_u16(B), s)
        Ub = None
        if rank:
            Ub = np.abs(oracle.bf16_to_f32(syn.bits_u16(dY))).astype(np.float64) @ \
                np.abs(oracle.bf16_to_f32(syn.bits_u16(B))).astype(np.float64)
        refs.append((dXr, dXb, Ur, Ub))
    outs = lbq.linear_bwd_grouped(probs)
    torch.cuda.synchronize()
    for i, ((dX, U), (dXr, dXb, Ur, Ub)) in enumerate(zip(outs, refs)):
        assert_within(dX.cpu().numpy(), dXr, dXb, f"dX (problem {i}, M={m})")
        if Ub is not None:
            assert_within(U.cpu().numpy(), Ur, Ub, f"U (problem {i}, M={m})")
    assert_status_clean(lbq)


@pytest.mark.parametrize("scheme,bits", [("minmax", 4), ("minmax", 2), ("codebook", 4)])
def test_last_wave_split(lbq, scheme, bits):
    """The GEMMs' split of the last wave: at M = 300 (two 256-token tiles)
    93 output (or feature) tiles make 186 tiles, 148 in a full wave and 38 in
    the last, which a second launch splits over the idle SMs; every element of
    Y and dX against the oracle."""
    m, r, s = 300, 16, 2.0
    cb = syn.codebook_normal16()
    # forward: 93 row tiles (k = 1024 so that INT2, split on 8-block chunks, splits too)
    n, k = 93 * 128, 1024
    X, W, A, B = fwd_problem(m, n, k, r, seed=31 + bits, scheme=scheme, bits=bits)
    qw = device_qweight(lbq, W, scheme, bits, scheme == "codebook", cb)
    assert lbq.lbq_linear_fwd_workspace_size(m, ctypes.byref(qw.struct), r) > 0     # the split is planned
    Y, _ = lbq.linear_fwd(X.cuda(), qw, A.cuda(), B.cuda(), s)
    torch.cuda.synchronize()
    What = oracle_weight(W, scheme, bits, scheme == "codebook", cb)
    Yr, _, Yb = oracle.linear_fwd(syn.bits_u16(X), What, syn.bits_u16(A), syn.bits_u16(B), s)
    assert_within(Y.cpu().numpy(), Yr, Yb, f"Y ({scheme} {bits}-bit, last wave split)")
    # backward: 93 feature tiles
    n, k = 256, 93 * 128
    X, W, A, B = fwd_problem(m, n, k, r, seed=41 + bits, scheme=scheme, bits=bits)
    dY = syn.normal_bf16((m, n), 0.1, seed=51 + bits)
    qw = device_qweight(lbq, W, scheme, bits, scheme == "codebook", cb)
    assert lbq.lbq_linear_bwd_workspace_size(m, ctypes.byref(qw.struct), r) > 0
    dX, _ = lbq.linear_bwd(dY.cuda(), qw, A.cuda(), B.cuda(), s)
    torch.cuda.synchronize()
    What = oracle_weight(W, scheme, bits, scheme == "codebook", cb)
    dXr, _, dXb = oracle.linear_bwd(syn.bits_u16(dY), What, syn.bits_u16(A), syn.bits_u16(B), s)
    assert_within(dX.cpu().numpy(), dXr, dXb, f"dX ({scheme} {bits}-bit, last wave split)")
    assert_status_clean(lbq)


def test_codebook70b_backward_full_size_sampled(lbq, codebook70b):
    """dX = dY W_hat through the 70B attention projection (8192 x 8192,
    codebook + double quantization) at M = 2048: 2048 seeded elements plus a
    full row and a full column against the oracle."""
    C = codebook70b
    m = 2048
    dY = syn.normal_bf16((m, C["n"]), 0.1, seed=75)
    dX, _ = lbq.linear_bwd(dY.cuda(), C["qw"])
    torch.cuda.synchronize()
    rows, cols = _sample_pairs(m, C["k"], 2048, seed=11)
    g = oracle.bf16_to_f32(syn.bits_u16(dY))
    w = C["What"]
    ref = np.empty(rows.size)
    bound = np.empty(rows.size)
    for i in range(0, rows.size, 512):
        gr = g[rows[i:i + 512]].astype(np.float64)              # [b, n]
        wc = w[:, cols[i:i + 512]].T.astype(np.float64)         # [b, n]
        ref[i:i + 512] = np.einsum("ij,ij->i", gr, wc)
        bound[i:i + 512] = np.einsum("ij,ij->i", np.abs(gr), np.abs(wc))
    assert_within(dX.cpu().numpy()[rows, cols], ref, bound, "dX (70B codebook, M=2048)")
    assert_status_clean(lbq)


# --------------------------------------------------------------------------- FP4 (E2M1) table
def _fp4_weight(n, k, seed):
    Wt = syn.weight_bf16(n, k, 0.015, seed=seed, outlier_frac=0.005).float()
    Wt[0, :64] = 0.0                               # a zero block
    Wt[1, 64:128] = -Wt[1, 64:128].abs()           # negative values only
    return Wt.to(torch.bfloat16)


@pytest.mark.parametrize("double_quant", [False, True])
@pytest.mark.parametrize("shape", [(256, 512), (1000, 1024)])
def test_fp4_quantize_bit_exact(lbq, double_quant, shape):
    """The FP4 (E2M1) table in code order (bitsandbytes guide, nf4与fp4), with
    +0 at code 0 and -0 at code 8: GPU codes, absmax and double-quantized
    constants equal the oracle's bit for bit, and dequantization too."""
    n, k = shape
    cb = syn.codebook_fp4_e2m1()
    W = _fp4_weight(n, k, seed=n + k)
    qw = lbq.QuantizedWeight(n, k, "codebook", double_quant=double_quant, codebook=cb).quantize(W.cuda())
    torch.cuda.synchronize()
    codes, absmax = oracle.codebook_quantize(syn.bits_u16(W), cb)
    assert not np.any(codes == 8)
    packed = oracle.pack(codes, 4)
    assert np.array_equal(qw.packed.cpu().numpy(), packed)
    assert np.array_equal(qw.absmax.cpu().numpy().view(np.uint32), absmax.view(np.uint32))
    a_used = absmax
    if double_quant:
        q8, s2, off, exact = oracle.double_quant(absmax)
        assert exact
        assert np.array_equal(qw.q8.cpu().numpy(), q8)
        assert np.array_equal(qw.s2.cpu().numpy().view(np.uint32), s2.view(np.uint32))
        a_used = oracle.double_dequant(q8, s2, off)
    What = qw.dequantize().cpu().numpy()
    assert np.array_equal(What.view(np.uint32), oracle.codebook_dequantize(packed, a_used, cb, n, k).view(np.uint32))
    assert_status_clean(lbq)


@pytest.mark.parametrize("m", [1, 16, 100])
def test_fp4_forward_backward_merge(lbq, m):
    """Forward (decode GEMV and tensor-core GEMM), backward and adapter merge
    on an FP4-coded weight with double quantization, against the oracle."""
    n, k, r, s = 384, 1024, 8, 2.0
    cb = syn.codebook_fp4_e2m1()
    W = _fp4_weight(n, k, seed=77 + m)
    X = syn.normal_bf16((m, k), 1.0, seed=78)
    A = syn.normal_bf16((r, k), 0.01, seed=79)
    B = syn.normal_bf16((n, r), 0.01, seed=80)
    dY = syn.normal_bf16((m, n), 0.1, seed=81)
    qw = device_qweight(lbq, W, "codebook", 4, True, cb)
    What = oracle_weight(W, "codebook", 4, True, cb)
    Y, _ = lbq.linear_fwd(X.cuda(), qw, A.cuda(), B.cuda(), s)
    dX, _ = lbq.linear_bwd(dY.cuda(), qw, A.cuda(), B.cuda(), s)
    merged = lbq.merge_lora(qw, A.cuda(), B.cuda(), s)
    torch.cuda.synchronize()
    Yr, _, Yb = oracle.linear_fwd(syn.bits_u16(X), What, syn.bits_u16(A), syn.bits_u16(B), s)
    dXr, _, dXb = oracle.linear_bwd(syn.bits_u16(dY), What, syn.bits_u16(A), syn.bits_u16(B), s)
    assert_within(Y.cpu().numpy(), Yr, Yb, "Y (FP4)")
    assert_within(dX.cpu().numpy(), dXr, dXb, "dX (FP4)")
    assert np.array_equal(u16(merged), oracle.lora_merge(What, syn.bits_u16(A), syn.bits_u16(B), s, 1))
    assert_status_clean(lbq)


# --------------------------------------------------------------------------- channel-mix selection by sensitivity
@pytest.mark.parametrize("n,k,t", [(1000, 1024, 64), (14336, 4096, 128)])
def test_channel_mix_select_matches_oracle(lbq, n, k, t):
    """Scores within fp64 rounding of the oracle's (the GPU sums in another
    order), the selection valid against the oracle's threshold (only channels
    whose scores are within that rounding of it may differ), the permutation
    the INT4 channels then the others, each ascending."""
    W = syn.weight_bf16(n, k, 0.02, seed=n + 1, outlier_frac=0.001)
    X = syn.normal_bf16((t, k), 1.0, seed=k + 2)
    n4 = int(round(0.25 * n))
    perm, score = lbq.channel_mix_select(W.cuda(), X.cuda(), n4)
    torch.cuda.synchronize()
    ref, bound = oracle.channel_score(syn.bits_u16(W), syn.bits_u16(X))
    got = score.cpu().numpy()
    tol = 2.0 ** -40 * bound + 1e-300
    assert np.all(np.abs(got - ref) <= tol)
    perm = perm.cpu().numpy()
    sel = np.zeros(n, bool)
    sel[perm[:n4]] = True
    assert np.array_equal(np.sort(perm), np.arange(n))
    assert np.all(np.diff(perm[:n4]) > 0) and np.all(np.diff(perm[n4:]) > 0)
    ref_perm = oracle.channel_mix_select(ref, n4)
    thr = np.sort(ref)[::-1][n4 - 1]
    differ = sel != np.isin(np.arange(n), ref_perm[:n4])
    assert np.all(np.abs(ref[differ] - thr) <= 2 * tol[differ] + 2.0 ** -40 * np.abs(thr))
    assert differ.sum() <= 2
    assert_status_clean(lbq)


@pytest.mark.parametrize("m", [16, 512])
def test_channel_mix_weight_from_selection(lbq, m):
    """The channel-mix weight built on the device from the selection (rows
    gathered by the permutation, then quantized) computes the forward of the
    oracle's channel-mix weight for that permutation."""
    n, k, r, s = 768, 1024, 8, 2.0
    W = syn.weight_bf16(n, k, 0.02, seed=91, outlier_frac=0.005)
    Xc = syn.normal_bf16((64, k), 1.0, seed=92)
    X = syn.normal_bf16((m, k), 1.0, seed=93)
    A = syn.normal_bf16((r, k), 0.01, seed=94)
    B = syn.normal_bf16((n, r), 0.01, seed=95)
    mix = lbq.channel_mix_weight(W.cuda(), Xc.cuda(), 0.25)
    Y, _ = lbq.linear_fwd(X.cuda(), mix, A.cuda(), B.cuda(), s)
    torch.cuda.synchronize()
    perm = mix.perm.cpu().numpy()
    n4 = mix.hi.n
    What = np.zeros((n, k), np.float32)
    for rows, bits in ((perm[:n4], 4), (perm[n4:], 2)):
        Wh = syn.bits_u16(W[torch.from_numpy(rows.astype(np.int64))].contiguous())
        codes, scale, zero = oracle.minmax_quantize(Wh, bits, 128 if bits == 4 else 64)
        What[rows] = oracle.minmax_dequantize(oracle.pack(codes, bits), scale, zero, k, bits, 128 if bits == 4 else 64)
    Yr, _, Yb = oracle.linear_fwd(syn.bits_u16(X), What, syn.bits_u16(A), syn.bits_u16(B), s)
    assert_within(Y.cpu().numpy(), Yr, Yb, f"Y (selected channel-mix, M={m})")
    assert_status_clean(lbq)

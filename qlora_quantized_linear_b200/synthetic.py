"""Seeded synthetic inputs with the shapes and value distributions of the
LLaMA-3 8B and 70B linear layers that low-bit QLoRA-style fine-tuning works on.

This module holds no quantization or GEMM arithmetic: it only draws random
numbers.  The CUDA path's tests and benchmark and the CPU oracle take their
inputs from here, so both sides see the same bits.  All draws use a CPU
`torch.Generator` with an explicit seed; bf16 tensors are returned on the CPU
(callers copy them to the device).

Distributions (see the project design notes for the reasoning):
  * weights ~ N(0, std^2) in bf16, optionally with a seeded 0.1 % of input
    channels (columns) scaled by 20 -- the systematic activation-outlier
    channels that the GreenBit article's section 模型量化 attributes to
    transformer LLMs -- so that some quantization groups span a wide range;
  * activations X ~ N(0, 1), adapters A, B ~ N(0, 0.01^2), output gradients
    dY ~ N(0, 0.1^2) (variance 1e-2);
  * a 16-entry codebook made of inverse-normal quantiles at evenly spaced
    probabilities, normalised to max 1, with an exact 0 (NormalFloat-style,
    as described in the QLoRA explainer's section 关键技术细节).
"""
from __future__ import annotations

import numpy as np
import torch

LLAMA3_8B_SHAPES = {            # name -> (out features N, in features K)
    "q": (4096, 4096),
    "k": (1024, 4096),
    "v": (1024, 4096),
    "o": (4096, 4096),
    "gate": (14336, 4096),
    "up": (14336, 4096),
    "down": (4096, 14336),
}

LLAMA3_70B_SHAPES = {
    "q": (8192, 8192),
    "gate": (28672, 8192),
    "down": (8192, 28672),
}


def _gen(seed: int, device="cpu") -> torch.Generator:
    g = torch.Generator(device=device)
    g.manual_seed(int(seed))
    return g


def normal_bf16(shape, std: float, seed: int, device="cpu") -> torch.Tensor:
    """bf16 tensor of N(0, std^2) samples (drawn in fp32, rounded once).
    device="cuda" draws with the device generator (a different stream of
    numbers than the CPU one for the same seed; used for large benchmark
    inputs that never meet the oracle)."""
    x = torch.randn(tuple(shape), generator=_gen(seed, device), dtype=torch.float32, device=device)
    if std != 1.0:
        x.mul_(std)
    return x.to(torch.bfloat16)


def outlier_columns(k: int, frac: float, seed: int) -> torch.Tensor:
    """Seeded choice of round(frac*k) (at least 1 when frac > 0) input channels."""
    cnt = int(round(frac * k))
    if frac > 0 and cnt == 0:
        cnt = 1
    perm = torch.randperm(k, generator=_gen(seed + 7919))
    return torch.sort(perm[:cnt]).values


def weight_bf16(n: int, k: int, std: float, seed: int,
                outlier_frac: float = 0.0, outlier_scale: float = 20.0, device="cpu") -> torch.Tensor:
    """Weight [n, k] ~ N(0, std^2), with `outlier_frac` of its input channels
    (columns) multiplied by `outlier_scale` before the bf16 rounding."""
    x = torch.randn((n, k), generator=_gen(seed, device), dtype=torch.float32, device=device)
    x.mul_(std)
    if outlier_frac > 0:
        cols = outlier_columns(k, outlier_frac, seed).to(device)
        x[:, cols] *= outlier_scale
    return x.to(torch.bfloat16)


def bits_u16(t: torch.Tensor) -> np.ndarray:
    """uint16 bit pattern of a CPU bf16/fp16 tensor (no copy of the values)."""
    assert t.dtype in (torch.bfloat16, torch.float16)
    return t.contiguous().view(torch.int16).numpy().view(np.uint16)


def codebook_normal16(p_max: float = 0.97) -> np.ndarray:
    """16 sorted fp32 entries in [-1, 1] with an exact 0.

    Eight positive entries are the standard-normal quantiles at the eight
    evenly spaced probabilities 0.5 + i (p_max - 0.5)/8, i = 1..8; seven
    negative entries mirror the quantiles at 0.5 + i (p_max - 0.5)/7,
    i = 1..7; all are divided by the largest one, so the table spans [-1, 1].
    Computed in fp64 and rounded to fp32 once.
    """
    pos_p = 0.5 + (p_max - 0.5) * torch.arange(1, 9, dtype=torch.float64) / 8
    neg_p = 0.5 + (p_max - 0.5) * torch.arange(1, 8, dtype=torch.float64) / 7
    pos = torch.special.ndtri(pos_p)
    neg = -torch.special.ndtri(neg_p)
    top = pos.max()
    vals = torch.cat([neg / top, torch.zeros(1, dtype=torch.float64), pos / top])
    vals, _ = torch.sort(vals)
    out = vals.to(torch.float32).numpy().copy()
    out[out.argmax()] = 1.0
    out[out.argmin()] = -1.0
    return out


def codebook_fp4_e2m1() -> np.ndarray:
    """The 16 FP4 (E2M1) values in code order, divided by the largest (6),
    as fp32: code = sign (bit 3), exponent (bits 2..1), mantissa (bit 0);
    exponent 0 is subnormal (0 or 0.5), otherwise (1 + m/2) * 2^(e - 1).
    Codes 0 and 8 are +0 and -0.  Computed exactly, rounded to fp32 once."""
    from fractions import Fraction
    vals = []
    for c in range(16):
        s, e, m = c >> 3, (c >> 1) & 3, c & 1
        mag = Fraction(m, 2) if e == 0 else (1 + Fraction(m, 2)) * Fraction(2) ** (e - 1)
        v = mag / 6
        vals.append(-float(v) if s else float(v))
    out = np.array(vals, dtype=np.float32)
    out[8] = np.float32(-0.0)
    return out


def channel_mix_perm(n: int, frac_int4: float, seed: int):
    """Seeded channel-mix split of the n output channels.

    Returns (perm int32 [n], n4): perm lists the INT4 channels first and then
    the INT2 channels, each group in ascending original order; n4 is the count
    of INT4 channels, round(frac_int4 * n).
    """
    n4 = int(round(frac_int4 * n))
    order = torch.randperm(n, generator=_gen(seed + 104729))
    int4 = torch.sort(order[:n4]).values
    int2 = torch.sort(order[n4:]).values
    perm = torch.cat([int4, int2]).to(torch.int32).numpy()
    return perm, n4


def layer_mix_choice(seed: int, shapes=None) -> dict:
    """Seeded layer-mix bit assignment for one 8B layer set.

    Reading adopted for "averaging 2.5 bits/param": 2.5 counts code bits, so
    about a quarter of the parameters are INT4.  The subsets of the seven 8B
    matrices within 0.05 of 2.5 code bits are exactly the single MLP matrices
    (gate, up or down: 2.538); the seed picks one of them to be INT4 g128 and
    the rest are INT2 g64.
    """
    shapes = shapes or LLAMA3_8B_SHAPES
    choices = ["gate", "up", "down"]
    pick = choices[int(torch.randint(0, 3, (1,), generator=_gen(seed + 15485863)).item())]
    return {name: (4 if name == pick else 2) for name in shapes}

"""Data-parallel QLoRA step over quantized linear layers, one process per GPU.

The bitsandbytes FSDP-QLoRA guide (section FSDP-QLoRA 将三种技术组合) trains
QLoRA data-parallel: every rank holds the same frozen low-bit weights and the
same low-rank adapters, runs the forward and backward passes on its own part
of the batch, and the adapter gradients -- the only trainable parameters, per
the QLoRA explainer, QLoRA技术原理 -- are combined across ranks.  For one
quantized linear layer with adapter (A, B) and scale s, on the rank's token
shard X_r with output gradient dY_r:

    T_r = X_r A^T,  Y_r = X_r W_hat^T + s T_r B^T          (lbq_linear_fwd)
    U_r = dY_r B,   dX_r = dY_r W_hat + s U_r A             (lbq_linear_bwd)
    dA_r = s U_r^T X_r,  dB_r = s dY_r^T T_r                (lbq_lora_grads)

and, with dY_r the gradient of the global loss with respect to the rank's rows
of Y, the gradient of the whole batch is the SUM over ranks:
dA = sum_r dA_r, dB = sum_r dB_r (set `average=True` when each rank's dY is
the gradient of its own mean loss and the global loss is their mean).

That sum is the only exchange on this path: rank * (k + n) * 4 bytes per layer
(1.2 MB for an 8B MLP matrix at rank 16).  All layers' gradients live in one
flat fp32 buffer, so a step makes ONE all-reduce (NCCL over NVLink/NVSwitch on
GPUs; gloo on CPUs), issued after the last layer's gradient kernels on the
same stream.  Nothing else crosses ranks: the frozen weights are replicated.

The per-rank products run in the library's CUDA kernels.  `grad_fn` replaces
them only where a test supplies its own per-rank computation (the CPU tests of
the multi-rank logic); there is no automatic fallback.
"""
from __future__ import annotations

from typing import Callable, List, Optional, Sequence


class AdapterLayer:
    """One frozen quantized weight with its trainable adapter.

    qw: a `lbq.QuantizedWeight` (or any object with n, k); A: bf16 [rank, k];
    B: bf16 [n, rank]; s: adapter scale."""

    def __init__(self, qw, A, B, s: float):
        self.qw, self.A, self.B, self.s = qw, A, B, float(s)
        self.rank = int(A.shape[0])
        self.n, self.k = int(qw.n), int(qw.k)
        self.dA = None          # views into the step's flat gradient buffer
        self.dB = None


class DataParallelQLoRA:
    """The data-parallel step over a list of AdapterLayer.

    group: a torch.distributed process group (None: the default group when
    torch.distributed is initialised, else a single process)."""

    def __init__(self, layers: Sequence[AdapterLayer], group=None, average: bool = False,
                 grad_fn: Optional[Callable] = None, device=None):
        import torch
        self.torch = torch
        self.layers: List[AdapterLayer] = list(layers)
        self.group = group
        self.average = average
        self.grad_fn = grad_fn
        dev = device if device is not None else self.layers[0].A.device
        sizes = [L.rank * L.k + L.n * L.rank for L in self.layers]
        # one flat fp32 buffer: layer i's dA [rank, k] then dB [n, rank]
        self.flat = torch.zeros(sum(sizes), dtype=torch.float32, device=dev)
        off = 0
        for L in self.layers:
            L.dA = self.flat[off:off + L.rank * L.k].view(L.rank, L.k)
            off += L.rank * L.k
            L.dB = self.flat[off:off + L.n * L.rank].view(L.n, L.rank)
            off += L.n * L.rank

    # ------------------------------------------------------------------ ranks
    def _dist(self):
        d = self.torch.distributed
        return d if (d.is_available() and d.is_initialized()) else None

    def world(self) -> int:
        d = self._dist()
        return d.get_world_size(self.group) if d else 1

    # ------------------------------------------------------------------ step
    def local_step(self, shards, stream=None):
        """Forward, backward and adapter gradients of every layer on this
        rank's shard.  shards[i] = (X_r, dY_r), bf16 [m_r, k_i] and
        [m_r, n_i].  Writes the rank's dA, dB into the flat buffer and returns
        [(Y_r, dX_r)] per layer."""
        outs = []
        for L, (X, dY) in zip(self.layers, shards):
            if self.grad_fn is not None:
                Y, dX, dA, dB = self.grad_fn(L, X, dY)
                L.dA.copy_(dA)
                L.dB.copy_(dB)
            else:
                from . import lbq
                Y, T = lbq.linear_fwd(X, L.qw, L.A, L.B, L.s, stream=stream)
                dX, U = lbq.linear_bwd(dY, L.qw, L.A, L.B, L.s, stream=stream)
                lbq.lora_grads(X, dY, T, U, L.s, dA=L.dA, dB=L.dB, stream=stream)
            outs.append((Y, dX))
        return outs

    def all_reduce(self, stream=None):
        """Sum (or average) the flat adapter-gradient buffer over the ranks:
        one collective per step.  On a GPU it runs on `stream` (the stream of
        the gradient kernels) when given."""
        d = self._dist()
        if d is None or d.get_world_size(self.group) == 1:
            if self.average:
                pass                                   # one rank: its mean is the mean
            return
        if stream is not None and self.flat.is_cuda:
            with self.torch.cuda.stream(stream):
                d.all_reduce(self.flat, op=d.ReduceOp.SUM, group=self.group)
                if self.average:
                    self.flat.div_(d.get_world_size(self.group))
        else:
            d.all_reduce(self.flat, op=d.ReduceOp.SUM, group=self.group)
            if self.average:
                self.flat.div_(d.get_world_size(self.group))

    def step(self, shards, stream=None):
        """local_step then all_reduce; returns the per-layer (Y_r, dX_r)."""
        outs = self.local_step(shards, stream=stream)
        self.all_reduce(stream=stream)
        return outs

    def grads(self):
        """[(dA, dB)] per layer (views into the flat buffer)."""
        return [(L.dA, L.dB) for L in self.layers]


def shard_rows(t, rank: int, world: int):
    """Rank's contiguous share of the rows of t (the token batch), as equal
    as the row count allows."""
    m = t.shape[0]
    lo = (m * rank) // world
    hi = (m * (rank + 1)) // world
    return t[lo:hi]

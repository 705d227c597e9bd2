"""The data-parallel QLoRA step's multi-rank logic on CPU (gloo, two ranks).

Each rank takes its contiguous shard of the token batch, computes its
layers' forward, backward and adapter gradients (here with the oracle,
plugged in as the per-rank computation; on GPUs the library's kernels do it)
and the step sums the flat adapter-gradient buffer with one all-reduce.  The
summed gradients must equal the oracle's gradients of the whole batch on one
rank -- the definition of a data-parallel step (bitsandbytes FSDP-QLoRA
guide, FSDP-QLoRA 将三种技术组合; QLoRA explainer, QLoRA技术原理: the adapter
gradients are the trainable ones).
"""
import os
import socket

import numpy as np
import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

import oracle
from qlora_quantized_linear_b200 import synthetic as syn
from qlora_quantized_linear_b200.dp import AdapterLayer, DataParallelQLoRA, shard_rows

LAYERS = [(256, 512, 8), (128, 1024, 4)]      # (n, k, rank) of each quantized layer
M = 37                                        # tokens of the global batch (uneven shards)
S = 2.0


class _OracleWeight:
    def __init__(self, n, k, seed):
        W = syn.weight_bf16(n, k, 0.02, seed)
        codes, scale, zero = oracle.minmax_quantize(syn.bits_u16(W), 4, 128)
        self.n, self.k = n, k
        self.What = oracle.minmax_dequantize(oracle.pack(codes, 4), scale, zero, k, 4, 128)


def _problem():
    layers, data = [], []
    for i, (n, k, r) in enumerate(LAYERS):
        qw = _OracleWeight(n, k, seed=10 + i)
        A = syn.normal_bf16((r, k), 0.01, seed=20 + i)
        B = syn.normal_bf16((n, r), 0.01, seed=30 + i)
        X = syn.normal_bf16((M, k), 1.0, seed=40 + i)
        dY = syn.normal_bf16((M, n), 0.1, seed=50 + i)
        layers.append(AdapterLayer(qw, A, B, S))
        data.append((X, dY))
    return layers, data


def _oracle_grads(L, X, dY):
    Y, _, _ = oracle.linear_fwd(syn.bits_u16(X), L.qw.What, syn.bits_u16(L.A), syn.bits_u16(L.B), L.s)
    dX, _, _ = oracle.linear_bwd(syn.bits_u16(dY), L.qw.What, syn.bits_u16(L.A), syn.bits_u16(L.B), L.s)
    dA, dB, _, _ = oracle.lora_grads(syn.bits_u16(X), syn.bits_u16(dY), syn.bits_u16(L.A), syn.bits_u16(L.B), L.s)
    return (torch.from_numpy(Y), torch.from_numpy(dX), torch.from_numpy(dA).float(), torch.from_numpy(dB).float())


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, average, out_dir):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank), WORLD_SIZE=str(world))
    import datetime
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
    try:
        layers, data = _problem()
        step = DataParallelQLoRA(layers, average=average, grad_fn=_oracle_grads, device="cpu")
        shards = [(shard_rows(X, rank, world), shard_rows(dY, rank, world)) for (X, dY) in data]
        outs = step.step(shards)
        # the rank's outputs are its rows of the full-batch outputs
        for (Y, dX), (X, dY), L in zip(outs, shards, layers):
            assert Y.shape[0] == X.shape[0] and dX.shape == (X.shape[0], L.k)
        np.save(os.path.join(out_dir, f"flat_{rank}.npy"), step.flat.numpy())
    finally:
        dist.destroy_process_group()


@pytest.mark.parametrize("average", [False, True])
def test_two_rank_step_equals_full_batch(tmp_path, average):
    world = 2
    mp.start_processes(_worker, args=(world, _free_port(), average, str(tmp_path)), nprocs=world,
                       start_method="spawn", join=True)
    flats = [np.load(tmp_path / f"flat_{r}.npy") for r in range(world)]
    assert np.array_equal(flats[0], flats[1]), "ranks disagree after the all-reduce"
    layers, data = _problem()
    off = 0
    for L, (X, dY) in zip(layers, data):
        dA, dB, dAb, dBb = oracle.lora_grads(syn.bits_u16(X), syn.bits_u16(dY), syn.bits_u16(L.A),
                                             syn.bits_u16(L.B), L.s)
        got_A = flats[0][off:off + L.rank * L.k].reshape(L.rank, L.k).astype(np.float64)
        off += L.rank * L.k
        got_B = flats[0][off:off + L.n * L.rank].reshape(L.n, L.rank).astype(np.float64)
        off += L.n * L.rank
        div = world if average else 1
        # two fp32-rounded shard sums against the fp64 full-batch gradient
        assert np.all(np.abs(got_A * div - dA) <= 2.0 ** -20 * dAb + 1e-12)
        assert np.all(np.abs(got_B * div - dB) <= 2.0 ** -20 * dBb + 1e-12)
    assert off == flats[0].size


def test_shards_cover_the_batch():
    t = torch.arange(37)
    for world in (1, 2, 3, 8):
        parts = [shard_rows(t, r, world) for r in range(world)]
        assert torch.equal(torch.cat(parts), t)
        assert max(p.numel() for p in parts) - min(p.numel() for p in parts) <= 1


def test_single_process_step_without_group():
    layers, data = _problem()
    step = DataParallelQLoRA(layers, grad_fn=_oracle_grads, device="cpu")
    assert step.world() == 1
    step.step(data)
    for (dA_got, dB_got), L, (X, dY) in zip(step.grads(), layers, data):
        dA, dB, dAb, dBb = oracle.lora_grads(syn.bits_u16(X), syn.bits_u16(dY), syn.bits_u16(L.A),
                                             syn.bits_u16(L.B), L.s)
        assert np.all(np.abs(dA_got.numpy().astype(np.float64) - dA) <= 2.0 ** -22 * dAb + 1e-12)
        assert np.all(np.abs(dB_got.numpy().astype(np.float64) - dB) <= 2.0 ** -22 * dBb + 1e-12)

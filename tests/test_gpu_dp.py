"""The data-parallel QLoRA step on a GPU: the library's kernels compute each
layer's forward, backward and adapter gradients, and the step's one
all-reduce runs through NCCL (a one-rank group here: this pool gives one GPU
per run; the two-rank logic is covered on CPU by test_dp_cpu.py).  The
gradients match the oracle within the stated bound."""
import numpy as np
import pytest
import torch
import torch.distributed as dist

import oracle
from qlora_quantized_linear_b200 import synthetic as syn
from qlora_quantized_linear_b200.dp import AdapterLayer, DataParallelQLoRA, shard_rows

pytestmark = pytest.mark.gpu


def test_dp_step_on_gpu_with_nccl():
    from qlora_quantized_linear_b200 import lbq
    m, s = 96, 2.0
    specs = [(256, 512, 8), (384, 1024, 16)]
    layers, data, whats = [], [], []
    for i, (n, k, r) in enumerate(specs):
        W = syn.weight_bf16(n, k, 0.02, seed=60 + i)
        codes, scale, zero = oracle.minmax_quantize(syn.bits_u16(W), 4, 128)
        packed = oracle.pack(codes, 4)
        qw = lbq.QuantizedWeight(n, k, "minmax", 4)
        qw.packed.copy_(torch.from_numpy(packed))
        qw.scale.copy_(torch.from_numpy(scale.view(np.float16)))
        qw.zero.copy_(torch.from_numpy(zero.view(np.float16)))
        A = syn.normal_bf16((r, k), 0.01, seed=70 + i)
        B = syn.normal_bf16((n, r), 0.01, seed=80 + i)
        X = syn.normal_bf16((m, k), 1.0, seed=90 + i)
        dY = syn.normal_bf16((m, n), 0.1, seed=100 + i)
        layers.append(AdapterLayer(qw, A.cuda(), B.cuda(), s))
        data.append((X, dY))
        whats.append(oracle.minmax_dequantize(packed, scale, zero, k, 4, 128))
    torch.cuda.set_device(0)
    dist.init_process_group("nccl", store=dist.HashStore(), rank=0, world_size=1,
                            device_id=torch.device("cuda", 0))
    try:
        step = DataParallelQLoRA(layers)
        assert step.world() == 1
        shards = [(shard_rows(X.cuda(), 0, 1), shard_rows(dY.cuda(), 0, 1)) for (X, dY) in data]
        stream = torch.cuda.current_stream()
        step.local_step(shards, stream=stream)
        # the one collective of the step (identity on one rank, through NCCL)
        dist.all_reduce(step.flat)
        torch.cuda.synchronize()
    finally:
        dist.destroy_process_group()
    for (dA_got, dB_got), L, (X, dY) in zip(step.grads(), layers, data):
        dA, dB, dAb, dBb = oracle.lora_grads(syn.bits_u16(X), syn.bits_u16(dY), syn.bits_u16(L.A.cpu()),
                                             syn.bits_u16(L.B.cpu()), L.s)
        assert np.all(np.abs(dA_got.cpu().numpy().astype(np.float64) - dA) <= 2.0 ** -7 * dAb + 1e-6)
        assert np.all(np.abs(dB_got.cpu().numpy().astype(np.float64) - dB) <= 2.0 ** -7 * dBb + 1e-6)
    assert lbq.device_status() == 0

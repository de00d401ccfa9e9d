"""Host logic of the N-split linear (fp8_block_scaled_group128_b200.tp) on
two gloo ranks on CPU: shard boundaries, the rank-major gather buffer, the
in-place all-gather and the column interleave reassemble the full product.
The GPU kernels are replaced by CPU stand-ins built on the oracle (the GPU
path of the same class is tested in test_gpu_tp.py)."""

import os
import socket

import numpy as np
import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

import oracle
from fp8_block_scaled_group128_b200 import synth, tp


def test_shard_rows():
    assert tp.shard_rows(4096, 4, 0) == (0, 1024)
    assert tp.shard_rows(4096, 4, 3) == (3072, 4096)
    assert tp.shard_rows(28672, 4, 1) == (7168, 14336)
    with pytest.raises(ValueError):
        tp.shard_rows(128256, 4, 0)        # 32064 is not whole 128-row blocks
    with pytest.raises(ValueError):
        tp.shard_rows(1024, 2, 2)


def _cpu_ops():
    def quant_act(x):
        q, s = oracle.quant_act_group128(x)
        return torch.from_numpy(q), torch.from_numpy(s)

    def quant_weight(w):
        q, s = oracle.quant_weight_block128(w)
        return torch.from_numpy(q), torch.from_numpy(s)

    def gemm(qa, sa, qw, sw, y):
        y.copy_(torch.from_numpy(oracle.block_gemm(qa.numpy(), sa.numpy(), qw.numpy(), sw.numpy()))
                .to(torch.bfloat16))
        return y

    def gather_columns(buf):
        P, M, Np = buf.shape
        return buf.permute(1, 0, 2).reshape(M, P * Np)

    return tp.Ops(quant_act, quant_weight, gemm, gather_columns)


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    p = s.getsockname()[1]
    s.close()
    return p


def _worker(rank, world, port, out):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        M, N, K = 5, 512, 256
        x = synth.activations("llama", M, K, seed=3)
        w = synth.weights("llama", N, K, seed=3)
        n0, n1 = tp.shard_rows(N, world, rank)
        lin = tp.NSplitLinear(w[n0:n1], world, rank, ops=_cpu_ops())
        out[rank] = lin.forward(x).float().numpy()
    finally:
        dist.destroy_process_group()


def test_nsplit_two_gloo_ranks_reassemble_the_full_product():
    world, port = 2, _free_port()
    out = mp.get_context("spawn").Manager().dict()
    mp.start_processes(_worker, args=(world, port, out), nprocs=world, start_method="spawn")
    M, N, K = 5, 512, 256
    x = synth.activations("llama", M, K, seed=3)
    w = synth.weights("llama", N, K, seed=3)
    qa, sa = oracle.quant_act_group128(x)
    qw, sw = oracle.quant_weight_block128(w)
    want = torch.from_numpy(oracle.block_gemm(qa, sa, qw, sw)).to(torch.bfloat16).float().numpy()
    for r in range(world):
        np.testing.assert_array_equal(out[r], want)

"""GPU side of the N-split linear: the column interleave kernel, P shards on
one GPU reassembling the full GEMM, and the NSplitLinear forward over a
one-rank NCCL group (the only group a one-GPU run can form; the P > 1
collective logic is covered on gloo ranks in test_tp_host.py)."""

import datetime
import socket

import numpy as np
import pytest
import torch
import torch.distributed as dist

import oracle
from fp8_block_scaled_group128_b200 import binding as fb
from fp8_block_scaled_group128_b200 import synth, tp

from gpu_util import check_gemm, require_gpu, to_dev

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _gpu():
    require_gpu()


@pytest.mark.parametrize("P,M,Np", [(1, 3, 8), (2, 5, 136), (4, 128, 1024), (8, 37, 512)])
def test_gather_columns_is_the_rank_major_transpose(P, M, Np):
    src = torch.randn(P, M, Np, device="cuda").to(torch.bfloat16)
    dst = fb.fp8_gather_columns(src)
    torch.cuda.synchronize()
    assert torch.equal(dst, src.permute(1, 0, 2).reshape(M, P * Np))


@pytest.mark.parametrize("M,N,K,P", [(512, 4096, 4096, 4), (8, 6144, 4096, 4), (130, 1024, 512, 2)])
def test_shards_on_one_gpu_reassemble_the_full_gemm(M, N, K, P):
    """Each shard's GEMM written into its slot of the rank-major buffer, then
    interleaved, equals the oracle's full product within the GEMM parity bound
    (prefill order: also byte-equal to the unsplit GEMM)."""
    x = synth.activations("llama", M, K, seed=5)
    w = synth.weights("llama", N, K, seed=5)
    xd, wd = to_dev(x), to_dev(w)
    qa, sa = fb.fp8_quant_act_group128(xd)
    buf = torch.empty(P, M, N // P, dtype=torch.bfloat16, device="cuda")
    for p in range(P):
        n0, n1 = tp.shard_rows(N, P, p)
        qw, sw = fb.fp8_quant_weight_block128(wd[n0:n1])
        fb.fp8_block_gemm(qa, sa, qw, sw, y=buf[p])
    y = fb.fp8_gather_columns(buf)
    qw_full, sw_full = fb.fp8_quant_weight_block128(wd)
    y_full = fb.fp8_block_gemm(qa, sa, qw_full, sw_full)
    torch.cuda.synchronize()
    assert fb.get_device_error() == 0
    if M > 256:
        assert torch.equal(y, y_full)
    ops = tuple(t.cpu().numpy() for t in (qa, sa, qw_full, sw_full))
    check_gemm(y, oracle.block_gemm(*ops), ops, f"N-split P={P} M={M}")


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    p = s.getsockname()[1]
    s.close()
    return p


def test_nsplit_linear_over_a_one_rank_nccl_group():
    store = dist.TCPStore("127.0.0.1", _free_port(), 1, True)
    dist.init_process_group("nccl", store=store, rank=0, world_size=1,
                            timeout=datetime.timedelta(seconds=60))
    try:
        M, N, K = 32, 6144, 4096
        x = to_dev(synth.activations("llama", M, K, seed=6))
        w = to_dev(synth.weights("llama", N, K, seed=6))
        lin = tp.NSplitLinear(w, 1, 0)
        y = lin.forward(x)
        qw, sw = fb.fp8_quant_weight_block128(w)
        y_ref = fb.fp8_linear(x, qw, sw)
        torch.cuda.synchronize()
        assert torch.equal(y, y_ref)
    finally:
        dist.destroy_process_group()

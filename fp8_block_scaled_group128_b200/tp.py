"""Output-column (N) split of the fine-grained FP8 linear over ranks, with one
NCCL all-gather of the bf16 output (tensor parallelism, as in the TensorRT-LLM
FP8 case study's TP = 4 Llama-3.3-70B runs).

Rank p of P holds weight rows [p Np, (p + 1) Np), Np = N / P a multiple of
128, so every 128x128 weight block and its scale lives on one rank. A forward
pass, per rank:

  1. quantize the (replicated) activations in 1x128 groups (library kernel);
  2. the block-scaled GEMM of the rank's weight rows, written straight into
     the rank's slot of a rank-major buffer [P][M][Np] (library kernel);
  3. an in-place all-gather of that buffer over the process group (NCCL over
     NVLink on GPUs);
  4. the library's column interleave, [P][M][Np] -> [M][N].

The compute steps are the library's kernels; `ops` lets a test run the same
host logic with stand-ins (e.g. over gloo on CPU).
"""

from dataclasses import dataclass
from typing import Callable

import torch
import torch.distributed as dist

from . import binding as fb

BLOCK = 128


def shard_rows(N, world, rank):
    """Weight rows [n0, n1) held by `rank`: N cut into `world` equal shards of
    whole 128-row blocks (N must be a multiple of 128 * world)."""
    if world < 1 or not 0 <= rank < world:
        raise ValueError("bad rank / world")
    if N % (BLOCK * world) != 0:
        raise ValueError(f"N = {N} is not a multiple of 128 x {world}")
    np_ = N // world
    return rank * np_, (rank + 1) * np_


@dataclass
class Ops:
    """The compute steps of a forward pass (defaults: the library's kernels)."""
    quant_act: Callable = fb.fp8_quant_act_group128
    quant_weight: Callable = fb.fp8_quant_weight_block128
    gemm: Callable = fb.fp8_block_gemm                # (qa, sa, qw, sw, y=out)
    gather_columns: Callable = fb.fp8_gather_columns  # [P, M, Np] -> [M, P Np]


class NSplitLinear:
    """One rank's shard of a fine-grained FP8 linear split along N."""

    def __init__(self, w_shard, world, rank, group=None, ops=None):
        self.world, self.rank, self.group = world, rank, group
        self.ops = ops or Ops()
        self.np = w_shard.shape[0]
        if self.np % BLOCK != 0:
            raise ValueError("a shard must hold whole 128-row blocks")
        self.qw, self.sw = self.ops.quant_weight(w_shard)

    def forward(self, x):
        M = x.shape[0]
        qa, sa = self.ops.quant_act(x)
        buf = torch.empty(self.world, M, self.np, dtype=torch.bfloat16, device=x.device)
        self.ops.gemm(qa, sa, self.qw, self.sw, y=buf[self.rank])
        if self.world > 1:
            # in place: every rank's input is its own slot of the output
            dist.all_gather_into_tensor(buf.view(-1), buf[self.rank].reshape(-1), group=self.group)
        return self.ops.gather_columns(buf)

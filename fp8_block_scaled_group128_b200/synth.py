"""Seeded synthetic inputs shaped like LLM linear layers.

This module only draws random numbers; it holds none of the layer's
arithmetic, so both the CUDA path and the CPU oracle can be fed from it.

Every tensor is drawn in fp32 by torch's CPU generator seeded from
``(seed, tag, shape)`` and rounded to bf16 (round-to-nearest-even). The same
call always returns the same bytes (for a given torch version).

Workloads (linear layers ``Y = X . W^T``, X [M, K], W [N, K]):

* ``tiny``: X [16, 256] ~ N(0, 1) with 1 % of entries (Bernoulli per entry)
  multiplied by 20; W [256, 256] ~ N(0, 0.02); seed 0.
* ``llama`` (decode and prefill shapes of Llama-3-8B): X ~ N(0, 1) with
  ceil(0.005 K) outlier channels (columns, the same for every token) x30;
  W ~ N(0, 0.02).
* ``deepseek`` (DeepSeek-V3 shapes): X = z * exp(sigma_m), z ~ N(0, 1),
  sigma_m ~ N(0, 1) per token; W = N(0, 0.01) * exp(tau_b) with
  tau_b ~ N(0, 0.5) per 128x128 block.
"""

import math
import zlib

import torch

# (N, K) of the four Llama-3-8B linears: QKV, O, gate+up, down.
LLAMA3_8B_LINEARS = ((6144, 4096), (4096, 4096), (28672, 4096), (4096, 14336))
LLAMA3_8B_LM_HEAD = (128256, 4096)
DECODE_M = (1, 8, 32, 128)
PREFILL_M = (2048, 8192)
# (N, K) of the DeepSeek-V3 block-scaled linears.
DEEPSEEK_V3_LINEARS = ((2112, 7168), (24576, 7168), (7168, 7168), (4096, 7168), (7168, 2048))
DEEPSEEK_M = (64, 4096)
# Mixture-of-experts linears of DeepSeek-V3 (an expert's gate+up and down
# projections, intermediate size 2048): (N, K).
MOE_LINEARS = ((4096, 7168), (7168, 2048))
MOE_EXPERTS = 8
MOE_ROUTED_ROWS = 4096
MOE_ALIGN = 128
# 2:4 sparse weights and token counts.
SPARSE_LINEARS = ((14336, 4096), (4096, 14336))
SPARSE_M = (16, 4096)


def _gen(seed, tag, *dims):
    key = f"{int(seed)}|{tag}|" + ",".join(str(int(d)) for d in dims)
    g = torch.Generator()
    g.manual_seed((int(seed) << 32) ^ zlib.crc32(key.encode()))
    return g


def _randn(g, *shape):
    return torch.randn(*shape, generator=g, dtype=torch.float32)


def activations(kind, M, K, seed=0):
    """bf16 activations [M, K] of the named workload kind."""
    g = _gen(seed, "x-" + kind, M, K)
    z = _randn(g, M, K)
    if kind == "tiny":
        hit = torch.rand(M, K, generator=g) < 0.01
        z = torch.where(hit, z * 20.0, z)
    elif kind == "llama":
        n_out = math.ceil(0.005 * K)
        ch = torch.randperm(K, generator=g)[:n_out]
        z[:, ch] *= 30.0
    elif kind == "deepseek":
        sigma = _randn(g, M, 1)
        z = z * torch.exp(sigma)
    else:
        raise ValueError(f"unknown workload kind {kind!r}")
    return z.to(torch.bfloat16)


def weights(kind, N, K, seed=0):
    """bf16 weights [N, K] of the named workload kind."""
    g = _gen(seed, "w-" + kind, N, K)
    if kind in ("tiny", "llama"):
        w = _randn(g, N, K) * 0.02
    elif kind == "deepseek":
        w = _randn(g, N, K) * 0.01
        nb, kb = -(-N // 128), -(-K // 128)
        tau = _randn(g, nb, kb) * 0.5
        spread = torch.exp(tau).repeat_interleave(128, 0)[:N].repeat_interleave(128, 1)[:, :K]
        w = w * spread
    else:
        raise ValueError(f"unknown workload kind {kind!r}")
    return w.to(torch.bfloat16)


def uniform_bf16(shape, lo, hi, seed=0, tag="u"):
    """bf16 values uniform in [lo, hi) (edge-case tests)."""
    g = _gen(seed, tag, *shape)
    return (torch.rand(*shape, generator=g) * (hi - lo) + lo).to(torch.bfloat16)


def moe_layout(experts, routed_rows, seed=0, align=128):
    """Seeded expert assignment of `routed_rows` token rows in the contiguous
    grouped layout: each expert's rows are consecutive, its segment is padded
    with rows of index -1 to a multiple of `align`, experts in order. The
    per-expert loads are a multinomial draw over Dirichlet(1) weights (uneven
    loads, as routers produce). Returns (m_indices int32 [rows], counts)."""
    g = _gen(seed, "moe", experts, routed_rows, align)
    # Dirichlet(1) weights as normalised exponentials (drawn with the seeded
    # generator, so the layout is reproducible)
    e = -torch.log(torch.rand(experts, generator=g, dtype=torch.float64).clamp_min(1e-300))
    p = e / e.sum()
    counts = torch.multinomial(p, routed_rows, replacement=True, generator=g).bincount(
        minlength=experts)
    parts = []
    for i, c in enumerate(counts.tolist()):
        pad = (-c) % align
        parts.append(torch.full((c,), i, dtype=torch.int32))
        parts.append(torch.full((pad,), -1, dtype=torch.int32))
    return torch.cat(parts), counts


def expert_weights(kind, experts, N, K, seed=0):
    """bf16 weights [E, N, K] of `experts` experts (each drawn like
    weights(kind, N, K) with its own seed)."""
    return torch.stack([weights(kind, N, K, seed=seed * 1000 + i) for i in range(experts)])

"""GPU parity of the gate+up GEMM with SwiGLU and the down projection's
1x128 quantization fused into its epilogue (fp8_gemm_swiglu_quant).

The GPU quantizes x and [W_gate; W_up] and runs the fused GEMM. The oracle
quantizes, from the same bf16 inputs, the compared token rows and the gate /
up weight blocks of the compared intermediate columns (asserting the GPU's
bytes equal its own), computes h = silu(g) * u in double and its tolerance
(the GEMM parity bound 1e-2 sum|a w| on g and on u, carried through silu's slope < 1.1),
and h must be within that plus one bf16 ulp. The codes and scales of h must
equal the oracle's 1x128 quantization of the GPU's own bf16 h, bit for bit."""

import numpy as np
import pytest
import torch

import oracle
from fp8_block_scaled_group128_b200 import binding as fb
from fp8_block_scaled_group128_b200 import synth

from gpu_util import require_gpu, to_dev

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _gpu():
    require_gpu()


def _sample(n, k, seed, must=()):
    rng = np.random.default_rng(seed)
    s = set(must) | set(rng.choice(n, min(n, k), replace=False).tolist())
    return np.array(sorted(s))


def _swiglu_case(M, I, K, seed, rows=None, groups=None):
    x = synth.activations("llama", M, K, seed=seed)
    w = torch.cat([synth.weights("llama", I, K, seed=seed),
                   synth.weights("llama", I, K, seed=seed + 1)])
    qa, sa = fb.fp8_quant_act_group128(to_dev(x))
    qw, sw = fb.fp8_quant_weight_block128(to_dev(w))
    h, qh, sh = fb.fp8_gemm_swiglu_quant(qa, sa, qw, sw)
    _, qh2, sh2 = fb.fp8_gemm_swiglu_quant(qa, sa, qw, sw, want_h=False)
    torch.cuda.synchronize()
    assert fb.get_device_error() == 0
    assert torch.equal(qh, qh2) and torch.equal(sh, sh2)
    r = np.arange(M) if rows is None else np.asarray(rows)
    gs = np.arange(I // 128) if groups is None else np.asarray(sorted(set(groups)))
    cols = np.concatenate([np.arange(g * 128, g * 128 + 128) for g in gs])
    sel = np.concatenate([cols, I + cols])   # gate rows, then up rows of the same columns
    qa_r, sa_r = oracle.quant_act_group128(x[torch.from_numpy(r)])
    qw_r, sw_r = oracle.quant_weight_block128(w[torch.from_numpy(sel)])
    rd, cd = torch.from_numpy(r).cuda(), torch.from_numpy(cols).cuda()
    np.testing.assert_array_equal(qa[rd].cpu().numpy(), qa_r)
    np.testing.assert_array_equal(qw[torch.from_numpy(sel).cuda()].cpu().numpy(), qw_r)
    h_ref, tol = oracle.gemm_swiglu(qa_r, sa_r, qw_r, sw_r)
    hg = h[rd][:, cd]
    err = np.abs(hg.double().cpu().numpy() - h_ref)
    bad = err > tol + oracle.bf16_ulp(h_ref)
    assert not bad.any(), f"{bad.sum()} outputs outside the bound, first {np.argwhere(bad)[0]}"
    q_ref, s_ref = oracle.quant_act_group128(hg.cpu())
    np.testing.assert_array_equal(qh[rd][:, cd].cpu().numpy(), q_ref)
    np.testing.assert_array_equal(sh[rd][:, torch.from_numpy(gs).cuda()].cpu().numpy().view(np.uint32),
                                  s_ref.view(np.uint32))
    return float((err / np.maximum(tol, 1e-300)).max())


@pytest.mark.parametrize("M,I,K", [(100, 256, 384), (300, 384, 512), (5, 128, 128), (257, 640, 1024)])
def test_ragged(M, I, K):
    assert _swiglu_case(M, I, K, seed=M) <= 1.0


@pytest.mark.parametrize("M", [1, 8, 32, 128])
def test_llama3_8b_decode(M):
    """The Llama-3-8B MLP (I = 14336, K = 4096) at decode token counts."""
    I = 14336
    assert _swiglu_case(M, I, 4096, seed=20 + M, groups=_sample(I // 128, 10, M, must=(0, 111))) <= 1.0


@pytest.mark.parametrize("M", [64, 65, 200])
def test_two_forms_at_the_switch(M):
    """At most 256 tokens the call takes the decode form (GEMM into the
    workspace, then the SwiGLU kernel) only where the dense dispatch keeps the
    decode order for N = 2I; with I = 14336 that is M <= 64, and M = 65 and 200
    (two row tiles, the second partial) run the one-kernel form. K = 512."""
    I = 14336
    assert _swiglu_case(M, I, 512, seed=40 + M, rows=_sample(M, 24, M, must=(0, M - 1)),
                        groups=_sample(I // 128, 10, M, must=(0, 111))) <= 1.0


@pytest.mark.parametrize("M", [2048, 8192])
def test_llama3_8b_prefill(M):
    I = 14336
    rows = _sample(M, 80, M, must=list(range(17, M, 128)) + [M - 1])
    assert _swiglu_case(M, I, 4096, seed=30, rows=rows,
                        groups=_sample(I // 128, 6, M, must=(0, 111))) <= 1.0

"""fp8_gemm_swiglu_quant_noalloc: the fused gate/up GEMM + SwiGLU + 1x128
quantization with its decode scratch in the library's fixed device array.

On the GPU it is compared with fp8_gemm_swiglu_quant (the workspace entry
point) on the same operands, at the SwiGLU parity tests' tolerance: h within
the oracle's bound on h plus one bf16 ulp of the workspace entry's h, on
sampled rows and 128-wide groups, and the codes and scales equal to the
oracle's 1x128 quantization of the no-allocation call's own h. Two calls run
back to back on different inputs before either is checked, so the second
one overwrites the shared scratch the first one used. The file is named to be
collected last; it also passes alone."""

import numpy as np
import pytest
import torch

import oracle
from fp8_block_scaled_group128_b200 import binding as fb
from fp8_block_scaled_group128_b200 import synth

from gpu_util import require_gpu, to_dev

SHAPE = 2                  # FP8BS_ERR_SHAPE
SCRATCH_LIMIT = 8          # FP8BS_ERR_SCRATCH_LIMIT
SCRATCH_BYTES = 16 << 20   # FP8BS_NOALLOC_SCRATCH_BYTES


def _call(lib, M, I, K, ptrs=(None,) * 7):
    return lib.fp8_gemm_swiglu_quant_noalloc(*ptrs, M, I, K, None)


def test_rejects_problems_above_the_scratch_before_any_launch():
    lib = fb.lib()
    # M <= 256 needs M * 2I bf16 values of scratch: 147 x 2 x 28672 x 2 bytes > 16 MiB
    assert 147 * 2 * 28672 * 2 > SCRATCH_BYTES >= 146 * 2 * 28672 * 2
    assert _call(lib, 147, 28672, 128) == SCRATCH_LIMIT
    assert _call(lib, 256, 16384 + 128, 128) == SCRATCH_LIMIT
    assert b"16 MiB" in lib.fp8bs_status_string(SCRATCH_LIMIT)
    # shape errors come first, as in the workspace entry point
    assert _call(lib, 8, 28672, 100) == SHAPE
    assert _call(lib, 8, 100, 128) == SHAPE


def _operands(M, I, K, seed):
    x = synth.activations("llama", M, K, seed=seed)
    w = torch.cat([synth.weights("llama", I, K, seed=seed),
                   synth.weights("llama", I, K, seed=seed + 1)])
    qa, sa = fb.fp8_quant_act_group128(to_dev(x))
    qw, sw = fb.fp8_quant_weight_block128(to_dev(w))
    return x, w, qa, sa, qw, sw


def _outputs(M, I):
    # filled with garbage, so a value the call does not write shows up
    h = torch.full((M, I), float("nan"), dtype=torch.bfloat16, device="cuda")
    qh = torch.full((M, I), 0x7F, dtype=torch.uint8, device="cuda")
    sh = torch.full((M, I // 128), -1.0, dtype=torch.float32, device="cuda")
    return h, qh, sh


def _check_against_workspace_entry(case, out, rows, groups):
    x, w, qa, sa, qw, sw = case
    M, K = qa.shape
    I = qw.shape[0] // 2
    h_ws, qh_ws, sh_ws = fb.fp8_gemm_swiglu_quant(qa, sa, qw, sw)
    torch.cuda.synchronize()
    assert fb.get_device_error() == 0
    h, qh, sh = out
    cols = np.concatenate([np.arange(g * 128, g * 128 + 128) for g in groups])
    sel = np.concatenate([cols, I + cols])
    qa_r, sa_r = oracle.quant_act_group128(x[torch.from_numpy(rows)])
    qw_r, sw_r = oracle.quant_weight_block128(w[torch.from_numpy(sel)])
    _, tol = oracle.gemm_swiglu(qa_r, sa_r, qw_r, sw_r)
    rd, cd = torch.from_numpy(rows).cuda(), torch.from_numpy(cols).cuda()
    hg = h[rd][:, cd]
    hw = h_ws[rd][:, cd].double().cpu().numpy()
    err = np.abs(hg.double().cpu().numpy() - hw)
    bad = ~(err <= tol + oracle.bf16_ulp(hw))
    assert not bad.any(), f"{bad.sum()} of h outside the tolerance, first {np.argwhere(bad)[0]}"
    q_ref, s_ref = oracle.quant_act_group128(hg.cpu())
    np.testing.assert_array_equal(qh[rd][:, cd].cpu().numpy(), q_ref)
    np.testing.assert_array_equal(
        sh[rd][:, torch.from_numpy(groups).cuda()].cpu().numpy().view(np.uint32),
        s_ref.view(np.uint32))


@pytest.mark.gpu
@pytest.mark.parametrize("M,I,K", [
    (8, 14336, 4096),    # Llama-3-8B MLP, decode
    (100, 256, 384),     # ragged rows, every group compared
    (256, 16384, 256),   # exactly fills the 16 MiB scratch
    (300, 384, 512),     # above 256 tokens: the fused kernel, no scratch
])
def test_two_calls_in_a_row_match_the_workspace_entry(M, I, K):
    require_gpu()
    lib = fb.lib()
    assert _call(lib, 0, I, K) == fb.FP8BS_OK   # the first call on the device sets up
    a = _operands(M, I, K, seed=M + 1)
    b = _operands(M, I, K, seed=M + 7)
    out_a, out_b = _outputs(M, I), _outputs(M, I)
    before = torch.cuda.memory_allocated()
    fb.fp8_gemm_swiglu_quant_noalloc(*a[2:], *out_a)
    fb.fp8_gemm_swiglu_quant_noalloc(*b[2:], *out_b)
    torch.cuda.synchronize()
    assert torch.cuda.memory_allocated() == before
    assert fb.get_device_error() == 0
    for h, qh, sh in (out_a, out_b):   # every output written (0x7F is the e4m3 NaN code)
        assert not torch.isnan(h).any() and not (qh == 0x7F).any() and (sh > 0).all()
    rng = np.random.default_rng(M)
    rows = np.array(sorted(set(rng.choice(M, min(M, 24), replace=False).tolist()) | {0, M - 1}))
    n_groups = I // 128
    groups = np.array(sorted(set(rng.choice(n_groups, min(n_groups, 8), replace=False).tolist())
                             | {0, n_groups - 1}))
    _check_against_workspace_entry(a, out_a, rows, groups)
    _check_against_workspace_entry(b, out_b, rows, groups)
    # without h the codes and scales are the same
    _, qh, sh = _outputs(M, I)
    fb.fp8_gemm_swiglu_quant_noalloc(*b[2:], None, qh, sh)
    torch.cuda.synchronize()
    assert torch.equal(qh, out_b[1]) and torch.equal(sh, out_b[2])

"""GPU parity of the grouped (mixture-of-experts) block-scaled GEMMs against
the oracle, with fp32 scales and with UE8M0 scales. Token rows are grouped by
expert (synth.moe_layout: uneven loads, each expert's rows padded to a
multiple of 128 with rows of index -1); every compared output must satisfy
|y - y_ref| <= 1e-2 * sum_k |a_k w_k| + 1 bf16 ulp with the row's expert."""

import numpy as np
import pytest
import torch

import oracle
from fp8_block_scaled_group128_b200 import binding as fb
from fp8_block_scaled_group128_b200 import synth

from gpu_util import check_gemm, require_gpu, to_dev

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _gpu():
    require_gpu()


def _moe_case(fmt, E, N, K, routed, seed, rows_per_expert=None, blocks=None):
    mi, counts = synth.moe_layout(E, routed, seed=seed)
    M = mi.numel()
    x = synth.activations("deepseek", M, K, seed=seed)
    w = synth.expert_weights("deepseek", E, N, K, seed=seed)
    xd, wd, mid = to_dev(x), to_dev(w), to_dev(mi)
    NB, KB = -(-N // 128), K // 128
    qw = torch.empty(E, N, K, dtype=torch.uint8, device="cuda")
    if fmt == "fp32":
        qa, sa = fb.fp8_quant_act_group128(xd)
        sw = torch.empty(E, NB, KB, dtype=torch.float32, device="cuda")
        for e in range(E):
            fb.fp8_quant_weight_block128(wd[e], qw=qw[e], sw=sw[e])
        y = fb.fp8_grouped_gemm(qa, sa, qw, sw, mid)
    else:
        qa, sa = fb.fp8_quant_act_group128_ue8m0(xd)
        sw = torch.empty(E, NB, KB, dtype=torch.uint8, device="cuda")
        for e in range(E):
            fb.fp8_quant_weight_block128_ue8m0(wd[e], qw=qw[e], sw8=sw[e])
        y = fb.fp8_grouped_gemm_ue8m0(qa, sa, qw, sw, mid)
    torch.cuda.synchronize()
    assert fb.get_device_error() == 0
    rng = np.random.default_rng(seed)
    mi_np = mi.numpy()
    rows = []
    for e in range(E):
        r = np.nonzero(mi_np == e)[0]
        if rows_per_expert is not None and r.size > rows_per_expert:
            keep = set(rng.choice(r, rows_per_expert, replace=False).tolist()) | {r[0], r[-1]}
            r = np.array(sorted(keep))
        rows.append(r)
    rows = np.concatenate(rows)
    nbs = np.arange(NB) if blocks is None else np.asarray(sorted(set(blocks)))
    n_idx = np.concatenate([np.arange(b * 128, min(N, b * 128 + 128)) for b in nbs])
    quant_a = oracle.quant_act_group128 if fmt == "fp32" else oracle.quant_act_group128_ue8m0
    quant_w = oracle.quant_weight_block128 if fmt == "fp32" else oracle.quant_weight_block128_ue8m0
    qa_r, sa_r = quant_a(x[torch.from_numpy(rows)])
    wq = [quant_w(w[e][torch.from_numpy(n_idx)]) for e in range(E)]
    qw_r = np.stack([q for q, _ in wq])
    sw_r = np.stack([s for _, s in wq])
    rd, nd = torch.from_numpy(rows).cuda(), torch.from_numpy(n_idx).cuda()
    np.testing.assert_array_equal(qa[rd].cpu().numpy(), qa_r)
    np.testing.assert_array_equal(qw[:, nd].cpu().numpy(), qw_r)
    grouped = oracle.grouped_gemm if fmt == "fp32" else oracle.grouped_gemm_ue8m0
    y_ref = grouped(qa_r, sa_r, qw_r, sw_r, mi_np[rows])
    y_sel = y[rd][:, nd]
    dec = (lambda s: s) if fmt == "fp32" else oracle.ue8m0_decode
    worst = 0.0
    for e in range(E):
        sel = np.nonzero(mi_np[rows] == e)[0]
        if sel.size == 0:
            continue
        st = check_gemm(y_sel[torch.from_numpy(sel).cuda()], y_ref[sel],
                        (qa_r[sel], dec(sa_r[sel]), qw_r[e], dec(sw_r[e])),
                        f"grouped {fmt} E={E} N={N} K={K} expert {e}")
        worst = max(worst, st["max_err_over_sum"])
    return worst


@pytest.mark.parametrize("fmt", ["fp32", "ue8m0"])
@pytest.mark.parametrize("N,K", [(136, 256), (520, 384), (1032, 640)])
def test_small_ragged(fmt, N, K):
    assert _moe_case(fmt, 3, N, K, routed=300, seed=N) < 1e-4


@pytest.mark.parametrize("fmt", ["fp32", "ue8m0"])
@pytest.mark.parametrize("N,K", [(4096, 7168), (7168, 2048)])
def test_deepseek_v3_experts(fmt, N, K):
    """DeepSeek-V3 expert linears (gate+up, down), 8 experts, 4096 routed rows."""
    NB = -(-N // 128)
    blocks = [0, NB - 1] + list(np.random.default_rng(N).choice(NB, 4, replace=False))
    assert _moe_case(fmt, synth.MOE_EXPERTS, N, K, routed=synth.MOE_ROUTED_ROWS, seed=7,
                     rows_per_expert=12, blocks=blocks) < 1e-4


@pytest.mark.parametrize("fmt", ["fp32", "ue8m0"])
def test_one_expert_is_the_dense_gemm(fmt):
    """E = 1 with every row of expert 0: the grouped GEMM equals the dense GEMM
    of the same operands within the bound (fp32 scales: the same kernel, so
    the same bytes)."""
    M, N, K = 384, 512, 1024
    x = to_dev(synth.activations("llama", M, K, seed=3))
    w = to_dev(synth.weights("llama", N, K, seed=3))
    mi = torch.zeros(M, dtype=torch.int32, device="cuda")
    if fmt == "fp32":
        qa, sa = fb.fp8_quant_act_group128(x)
        qw, sw = fb.fp8_quant_weight_block128(w)
        yg = fb.fp8_grouped_gemm(qa, sa, qw[None], sw[None], mi)
        yd = fb.fp8_block_gemm(qa, sa, qw, sw)
        torch.cuda.synchronize()
        assert torch.equal(yg, yd)
    else:
        qa, sa = fb.fp8_quant_act_group128_ue8m0(x)
        qw, sw = fb.fp8_quant_weight_block128_ue8m0(w)
        yg = fb.fp8_grouped_gemm_ue8m0(qa, sa, qw[None], sw[None], mi)
        torch.cuda.synchronize()
        qa_h, sa_h, qw_h, sw_h = (t.cpu().numpy() for t in (qa, sa, qw, sw))
        check_gemm(yg, oracle.block_gemm_ue8m0(qa_h, sa_h, qw_h, sw_h),
                   (qa_h, oracle.ue8m0_decode(sa_h), qw_h, oracle.ue8m0_decode(sw_h)),
                   "grouped ue8m0, one expert")
    assert fb.get_device_error() == 0

"""GPU parity of the UE8M0 (power-of-two scale) variant against the oracle:
the quantizers' codes and scale codes bit for bit, and the block-scaled GEMM
(the tensor cores' own block scaling) within
|y - y_ref| <= 1e-2 * sum_k |a_k w_k| + 1 bf16 ulp(y_ref)."""

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


def _sample(n, k, seed, must=()):
    rng = np.random.default_rng(seed)
    s = set(must) | set(rng.choice(n, min(n, k), replace=False).tolist())
    return np.array(sorted(s))


@pytest.mark.parametrize("kind,M,K", [("tiny", 16, 256), ("llama", 8, 4096), ("llama", 129, 14336),
                                      ("deepseek", 64, 7168), ("deepseek", 3, 128)])
def test_activation_quantizer_bit_exact(kind, M, K):
    x = synth.activations(kind, M, K, seed=1)
    qa, sa8 = fb.fp8_quant_act_group128_ue8m0(to_dev(x))
    torch.cuda.synchronize()
    q_r, s_r = oracle.quant_act_group128_ue8m0(x)
    np.testing.assert_array_equal(sa8.cpu().numpy(), s_r)
    np.testing.assert_array_equal(qa.cpu().numpy(), q_r)


def test_activation_quantizer_edge_values():
    """Zero groups, signed zeros, subnormal and huge maxima, every landmark
    of the scale-code rule (exact powers of two times 448 and their
    neighbours)."""
    x = np.zeros((8, 1024), np.float32)
    x[0, 128:256] = -0.0
    x[1, 5] = 2.0 ** -133
    x[1, 130] = -2.0 ** -126
    x[2, :] = synth.activations("deepseek", 1, 1024, seed=3).float().numpy() * 1e30
    for g, a in enumerate([448.0, 449.0 / 1.0, 224.0, 224.5, 0.875, 1.0, 3.5, 3.515625]):
        x[3 + g // 8, 128 * (g % 8) + 7] = a
        x[3 + g // 8, 128 * (g % 8) + 9] = -a / 3
    x[4, :] = np.linspace(-3e38, 3e38, 1024, dtype=np.float32)
    xb = torch.from_numpy(x).to(torch.bfloat16)
    qa, sa8 = fb.fp8_quant_act_group128_ue8m0(to_dev(xb))
    torch.cuda.synchronize()
    q_r, s_r = oracle.quant_act_group128_ue8m0(xb)
    np.testing.assert_array_equal(sa8.cpu().numpy(), s_r)
    np.testing.assert_array_equal(qa.cpu().numpy(), q_r)


@pytest.mark.parametrize("kind,N,K", [("tiny", 256, 256), ("llama", 4096, 4096),
                                      ("deepseek", 2112, 7168), ("deepseek", 300, 384)])
def test_weight_quantizer_bit_exact(kind, N, K):
    w = synth.weights(kind, N, K, seed=2)
    qw, sw8 = fb.fp8_quant_weight_block128_ue8m0(to_dev(w))
    torch.cuda.synchronize()
    q_r, s_r = oracle.quant_weight_block128_ue8m0(w)
    np.testing.assert_array_equal(sw8.cpu().numpy(), s_r)
    np.testing.assert_array_equal(qw.cpu().numpy(), q_r)


def _ue8m0_case(kind, M, N, K, seed=0, rows=None, blocks=None):
    """Quantize and multiply on the GPU; the oracle quantizes exactly the
    compared token rows and 128-row weight blocks from the same bf16 inputs
    (asserting the GPU bytes equal its own) and computes those outputs."""
    x = synth.activations(kind, M, K, seed=seed)
    w = synth.weights(kind, N, K, seed=seed)
    qa_d, sa_d = fb.fp8_quant_act_group128_ue8m0(to_dev(x))
    qw_d, sw_d = fb.fp8_quant_weight_block128_ue8m0(to_dev(w))
    y = fb.fp8_block_gemm_ue8m0(qa_d, sa_d, qw_d, sw_d)
    torch.cuda.synchronize()
    assert fb.get_device_error() == 0
    NB = -(-N // 128)
    r = np.arange(M) if rows is None else np.asarray(rows)
    nbs = np.arange(NB) if blocks is None else np.asarray(sorted(set(blocks)))
    n_idx = np.concatenate([np.arange(b * 128, min(N, b * 128 + 128)) for b in nbs])
    qa_r, sa_r = oracle.quant_act_group128_ue8m0(x[torch.from_numpy(r)])
    qw_r, sw_r = oracle.quant_weight_block128_ue8m0(w[torch.from_numpy(n_idx)])
    rd, nd = torch.from_numpy(r).cuda(), torch.from_numpy(n_idx).cuda()
    np.testing.assert_array_equal(qa_d[rd].cpu().numpy(), qa_r)
    np.testing.assert_array_equal(sa_d[rd].cpu().numpy(), sa_r)
    np.testing.assert_array_equal(qw_d[nd].cpu().numpy(), qw_r)
    np.testing.assert_array_equal(sw_d[torch.from_numpy(nbs).cuda()].cpu().numpy(), sw_r)
    y_ref = oracle.block_gemm_ue8m0(qa_r, sa_r, qw_r, sw_r)
    ops = (qa_r, oracle.ue8m0_decode(sa_r), qw_r, oracle.ue8m0_decode(sw_r))
    return check_gemm(y[rd][:, nd], y_ref, ops, f"ue8m0 {kind} M={M} N={N} K={K}")


def test_gemm_tiny():
    st = _ue8m0_case("tiny", 16, 256, 256)
    assert st["max_err_over_sum"] < 1e-4


@pytest.mark.parametrize("M,N,K", [(5, 8, 128), (3, 136, 256), (100, 520, 384), (257, 264, 640),
                                   (300, 1032, 512), (130, 4104, 1024), (129, 256, 4096)])
def test_gemm_ragged_shapes(M, N, K):
    st = _ue8m0_case("deepseek", M, N, K, seed=6)
    assert st["max_err_over_sum"] < 1e-4


@pytest.mark.parametrize("M,N,K", [(2048, 6144, 4096), (2048, 4096, 14336), (8192, 28672, 4096)])
def test_gemm_prefill_llama3_8b(M, N, K):
    rows = _sample(M, 96, M, must=list(range(11, M, 128)) + [M - 1])
    NB = -(-N // 128)
    st = _ue8m0_case("llama", M, N, K, seed=3, rows=rows,
                     blocks=_sample(NB, 8, K, must=(0, 1, NB - 1)))
    assert st["max_err_over_sum"] < 1e-4


@pytest.mark.parametrize("N,K", [(2112, 7168), (24576, 7168), (7168, 2048)])
def test_gemm_deepseek_v3_m4096(N, K):
    M = 4096
    rows = _sample(M, 64, N, must=list(range(3, M, 128)) + [M - 1])
    NB = -(-N // 128)
    st = _ue8m0_case("deepseek", M, N, K, seed=5, rows=rows,
                     blocks=_sample(NB, 8, K, must=(0, NB - 1)))
    assert st["max_err_over_sum"] < 1e-4


@pytest.mark.parametrize("M", [1, 8, 64])
def test_gemm_decode_sized(M):
    st = _ue8m0_case("llama", M, 4096, 4096, seed=8, blocks=[0, 5, 31])
    assert st["max_err_over_sum"] < 1e-4


def test_gemm_deterministic_and_timeout():
    M, N, K = 512, 1024, 2048
    x = synth.activations("llama", M, K, seed=9)
    w = synth.weights("llama", N, K, seed=9)
    qa, sa = fb.fp8_quant_act_group128_ue8m0(to_dev(x))
    qw, sw = fb.fp8_quant_weight_block128_ue8m0(to_dev(w))
    ys = [fb.fp8_block_gemm_ue8m0(qa, sa, qw, sw) for _ in range(3)]
    torch.cuda.synchronize()
    for y in ys[1:]:
        assert torch.equal(y.view(torch.int16), ys[0].view(torch.int16))
    fb.get_device_error()
    try:
        fb.set_wait_limit(1)
        fb.fp8_block_gemm_ue8m0(qa, sa, qw, sw)
        assert fb.get_device_error() == 6
    finally:
        fb.set_wait_limit(0)
    y = fb.fp8_block_gemm_ue8m0(qa, sa, qw, sw)
    assert fb.get_device_error() == 0
    assert torch.equal(y.view(torch.int16), ys[0].view(torch.int16))

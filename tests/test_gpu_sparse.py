"""GPU parity of the 2:4 sparse block-scaled GEMM against the oracle.

The GPU prunes and compresses the bf16 weights and multiplies the compressed
form; the oracle prunes and quantizes, from the same bf16 inputs, exactly the
token rows and 128-row weight blocks compared (asserting the GPU bytes equal
its own) and evaluates the GEMM on the decompressed codes. Every compared
output must satisfy |y - y_ref| <= 1e-2 * sum_k |a_k w_k| + 1 bf16 ulp.
"""

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


def _sparse_case(kind, M, N, K, seed=0, rows=None, blocks=None, w=None, x=None):
    x = synth.activations(kind, M, K, seed=seed) if x is None else x
    w = synth.weights(kind, N, K, seed=seed) if w is None else w
    qa_d, sa_d = fb.fp8_quant_act_group128(to_dev(x))
    vals_d, meta_d, sw_d, _ = fb.prune24_compress(to_dev(w))
    y = fb.fp8_sparse24_gemm(qa_d, sa_d, vals_d, meta_d, sw_d)
    torch.cuda.synchronize()
    assert fb.get_device_error() == 0
    NB = -(-N // 128)
    r = np.arange(M) if rows is None else np.asarray(rows)
    nbs = np.arange(NB) if blocks is None else np.asarray(sorted(set(blocks)))
    n_idx = np.concatenate([np.arange(b * 128, min(N, b * 128 + 128)) for b in nbs])
    qa_r, sa_r = oracle.quant_act_group128(x[torch.from_numpy(r)])
    v_r, m_r, s_r, _ = oracle.prune24_compress(w[torch.from_numpy(n_idx)])
    rd, nd = torch.from_numpy(r).cuda(), torch.from_numpy(n_idx).cuda()
    np.testing.assert_array_equal(qa_d[rd].cpu().numpy(), qa_r)
    np.testing.assert_array_equal(vals_d[nd].cpu().numpy(), v_r)
    np.testing.assert_array_equal(meta_d[nd].cpu().numpy(), m_r)
    np.testing.assert_array_equal(sw_d[torch.from_numpy(nbs).cuda()].cpu().numpy().view(np.uint32),
                                  s_r.view(np.uint32))
    y_ref = oracle.sparse24_gemm(qa_r, sa_r, v_r, m_r, s_r)
    ops = (qa_r, sa_r, oracle.decompress24(v_r, m_r), s_r)
    return check_gemm(y[rd][:, nd], y_ref, ops, f"sparse {kind} M={M} N={N} K={K}"), y


def _blocks(N, k, seed):
    NB = -(-N // 128)
    return _sample(NB, k, seed, must=(0, NB - 1))


def test_tiny():
    stats, _ = _sparse_case("tiny", 16, 256, 256)
    assert stats["max_err_over_sum"] < 1e-4


@pytest.mark.parametrize("M", [16, 1, 8, 32, 128])
@pytest.mark.parametrize("N,K", [(14336, 4096), (4096, 14336)])
def test_sparse_config_decode(M, N, K):
    stats, _ = _sparse_case("llama", M, N, K, seed=1, blocks=_blocks(N, 16, N + M))
    assert stats["max_err_over_sum"] < 1e-4


@pytest.mark.parametrize("N,K", [(14336, 4096), (4096, 14336)])
def test_sparse_config_prefill_m4096(N, K):
    M = 4096
    rows = _sample(M, 96, N, must=list(range(5, M, 128)) + [M - 1])
    stats, _ = _sparse_case("llama", M, N, K, seed=2, rows=rows, blocks=_blocks(N, 8, K))
    assert stats["max_err_over_sum"] < 1e-4


@pytest.mark.parametrize("M,N,K", [(3, 136, 256), (100, 520, 384), (200, 264, 640),
                                   (129, 1032, 512), (300, 4104, 1024), (1, 8, 128)])
def test_ragged_shapes(M, N, K):
    stats, _ = _sparse_case("deepseek", M, N, K, seed=3)
    assert stats["max_err_over_sum"] < 1e-4


@pytest.mark.parametrize("M,N,K", [(64, 4096, 4096), (16, 14336, 4096), (16, 4096, 14336),
                                   (4096, 14336, 4096), (4096, 4096, 14336)])
def test_sparse_and_dense_on_the_same_pruned_weights(M, N, K):
    """The 2:4 configuration's comparison with dense on the same pruned W: the
    GPU prunes W, quantizes the pruned bf16 W densely and runs both GEMMs;
    each output is checked element by element against the oracle (the sparse
    GEMM of the oracle's compression, and the dense GEMM of its quantization
    of the pruned W, which must be the same numbers)."""
    x = synth.activations("llama", M, K, seed=4)
    w = synth.weights("llama", N, K, seed=4)
    xd, wd = to_dev(x), to_dev(w)
    qa, sa = fb.fp8_quant_act_group128(xd)
    vals, meta, sws, wp = fb.prune24_compress(wd, want_pruned=True)
    qw, sw = fb.fp8_quant_weight_block128(wp)
    ys = fb.fp8_sparse24_gemm(qa, sa, vals, meta, sws)
    yd = fb.fp8_block_gemm(qa, sa, qw, sw)
    torch.cuda.synchronize()
    assert fb.get_device_error() == 0
    assert torch.equal(sw, sws)
    NB = -(-N // 128)
    rows = np.arange(M) if M <= 64 else _sample(M, 64, M, must=list(range(9, M, 128)) + [M - 1])
    nbs = _blocks(N, 8 if M > 64 else 16, N + M)
    n_idx = np.concatenate([np.arange(b * 128, min(N, b * 128 + 128)) for b in nbs])
    qa_r, sa_r = oracle.quant_act_group128(x[torch.from_numpy(rows)])
    v_r, m_r, s_r, wp_r = oracle.prune24_compress(w[torch.from_numpy(n_idx)])
    qd_r, sd_r = oracle.quant_weight_block128(wp_r)
    np.testing.assert_array_equal(qd_r, oracle.decompress24(v_r, m_r))
    rd, nd = torch.from_numpy(rows).cuda(), torch.from_numpy(n_idx).cuda()
    np.testing.assert_array_equal(wp[nd].float().cpu().numpy(), wp_r)
    np.testing.assert_array_equal(qw[nd].cpu().numpy(), qd_r)
    y_ref = oracle.sparse24_gemm(qa_r, sa_r, v_r, m_r, s_r)
    np.testing.assert_array_equal(y_ref, oracle.block_gemm(qa_r, sa_r, qd_r, sd_r))
    ops = (qa_r, sa_r, qd_r, sd_r)
    st_s = check_gemm(ys[rd][:, nd], y_ref, ops, f"2:4 vs dense, sparse M={M} N={N} K={K}")
    st_d = check_gemm(yd[rd][:, nd], y_ref, ops, f"2:4 vs dense, dense M={M} N={N} K={K}")
    assert st_s["max_err_over_sum"] < 1e-4 and st_d["max_err_over_sum"] < 1e-4
    assert NB > 0


def test_ties_and_zero_groups():
    rng = np.random.default_rng(5)
    w = (rng.integers(-2, 3, size=(256, 512)).astype(np.float32) * 0.125)
    w[:, 0:4] = 0.0
    w[3, :] = -0.0
    wt = torch.from_numpy(w).to(torch.bfloat16)
    stats, _ = _sparse_case("deepseek", 40, 256, 512, seed=5, w=wt)
    assert stats["max_err_over_sum"] < 1e-4


def test_sparse_deterministic():
    M, N, K = 16, 4096, 14336
    x = synth.activations("llama", M, K, seed=6)
    w = synth.weights("llama", N, K, seed=6)
    qa, sa = fb.fp8_quant_act_group128(to_dev(x))
    vals, meta, sws, _ = fb.prune24_compress(to_dev(w))
    ys = [fb.fp8_sparse24_gemm(qa, sa, vals, meta, sws) for _ in range(4)]
    torch.cuda.synchronize()
    for y in ys[1:]:
        assert torch.equal(y.view(torch.int16), ys[0].view(torch.int16))

"""GPU parity of the dense block-scaled GEMM against the oracle.

Two kinds of case: the GEMM alone on inputs quantized by the oracle and
uploaded (``_gemm_case``), and the whole chain quantize -> GEMM on the GPU,
where the oracle quantizes the compared rows and weight blocks itself from
the same bf16 inputs (``_chain_case``). Every compared output must satisfy
|y - y_ref| <= 1e-2 * sum_k |a_k w_k| + 1 bf16 ulp(y_ref).
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


_CACHE = {}


def _quantized(kind, M, N, K, seed):
    key = (kind, M, N, K, seed)
    if key not in _CACHE:
        x = synth.activations(kind, M, K, seed=seed)
        w = synth.weights(kind, N, K, seed=seed)
        qa, sa = oracle.quant_act_group128(x)
        qw, sw = oracle.quant_weight_block128(w)
        _CACHE.clear()
        _CACHE[key] = (qa, sa, qw, sw)
    return _CACHE[key]


def _run(qa, sa, qw, sw):
    y = fb.fp8_block_gemm(to_dev(qa), to_dev(sa), to_dev(qw), to_dev(sw))
    torch.cuda.synchronize()
    assert fb.get_device_error() == 0
    return y


def _gemm_case(kind, M, N, K, seed=0, rows=None, cols=None):
    qa, sa, qw, sw = _quantized(kind, M, N, K, seed)
    y = _run(qa, sa, qw, sw)
    r = np.arange(M) if rows is None else np.asarray(rows)
    c = None if cols is None else np.asarray(cols)
    y_ref = oracle.block_gemm(qa[r], sa[r], qw, sw, cols=c)
    y_sel = y[torch.from_numpy(r).cuda()]
    if c is not None:
        y_sel = y_sel[:, torch.from_numpy(c).cuda()]
    return check_gemm(y_sel, y_ref, (qa[r], sa[r], qw, sw), f"{kind} M={M} N={N} K={K}", cols=c)


def _chain_case(kind, M, N, K, seed=0, rows=None, blocks=None):
    """Quantize and multiply on the GPU; the oracle quantizes, from the same
    bf16 inputs, exactly the token rows and 128-row weight blocks compared
    (asserting the GPU bytes equal its own), then computes those outputs."""
    x = synth.activations(kind, M, K, seed=seed)
    w = synth.weights(kind, N, K, seed=seed)
    qa_d, sa_d = fb.fp8_quant_act_group128(to_dev(x))
    qw_d, sw_d = fb.fp8_quant_weight_block128(to_dev(w))
    y = fb.fp8_block_gemm(qa_d, sa_d, qw_d, sw_d)
    torch.cuda.synchronize()
    assert fb.get_device_error() == 0
    NB = -(-N // 128)
    r = np.arange(M) if rows is None else np.asarray(rows)
    nbs = np.arange(NB) if blocks is None else np.asarray(sorted(set(blocks)))
    n_idx = np.concatenate([np.arange(b * 128, min(N, b * 128 + 128)) for b in nbs])
    qa_r, sa_r = oracle.quant_act_group128(x[torch.from_numpy(r)])
    qw_r, sw_r = oracle.quant_weight_block128(w[torch.from_numpy(n_idx)])
    rd, nd = torch.from_numpy(r).cuda(), torch.from_numpy(n_idx).cuda()
    np.testing.assert_array_equal(qa_d[rd].cpu().numpy(), qa_r)
    np.testing.assert_array_equal(sa_d[rd].cpu().numpy().view(np.uint32), sa_r.view(np.uint32))
    np.testing.assert_array_equal(qw_d[nd].cpu().numpy(), qw_r)
    np.testing.assert_array_equal(sw_d[torch.from_numpy(nbs).cuda()].cpu().numpy().view(np.uint32),
                                  sw_r.view(np.uint32))
    y_ref = oracle.block_gemm(qa_r, sa_r, qw_r, sw_r)
    return check_gemm(y[rd][:, nd], y_ref, (qa_r, sa_r, qw_r, sw_r), f"{kind} M={M} N={N} K={K}")


def _sample(n, k, seed, must=()):
    rng = np.random.default_rng(seed)
    s = set(must) | set(rng.choice(n, min(n, k), replace=False).tolist())
    return np.array(sorted(s))


def _blocks(N, k, seed):
    NB = -(-N // 128)
    return _sample(NB, k, seed, must=(0, NB - 1))


def test_tiny_config():
    stats = _gemm_case("tiny", 16, 256, 256)
    assert stats["max_err_over_sum"] < 1e-5


@pytest.mark.parametrize("N,K", [(6144, 4096), (4096, 4096), (28672, 4096), (4096, 14336)])
@pytest.mark.parametrize("M", [1, 8, 32, 128])
def test_decode_llama3_8b(M, N, K):
    stats = _chain_case("llama", M, N, K, seed=1, blocks=_blocks(N, 24, N + M))
    assert stats["max_err_over_sum"] < 1e-4


@pytest.mark.parametrize("N,K", [(2112, 7168), (24576, 7168), (7168, 7168), (4096, 7168),
                                 (7168, 2048)])
def test_deepseek_v3_m64(N, K):
    stats = _chain_case("deepseek", 64, N, K, seed=2, blocks=_blocks(N, 24, N))
    assert stats["max_err_over_sum"] < 1e-4


def test_decode_exact_oracle_inputs():
    """The GEMM alone on oracle-quantized inputs, full output, split-K path."""
    stats = _gemm_case("llama", 8, 4096, 4096, seed=12)
    assert stats["max_err_over_sum"] < 1e-4


@pytest.mark.parametrize("M,N,K", [(2048, 4096, 4096), (2048, 6144, 4096), (2048, 4096, 14336)])
def test_prefill_llama3_8b(M, N, K):
    rows = _sample(M, 256, M, must=list(range(0, M, 128)) + [M - 1])
    stats = _chain_case("llama", M, N, K, seed=3, rows=rows, blocks=_blocks(N, 12, K))
    assert stats["max_err_over_sum"] < 1e-4


@pytest.mark.parametrize("M,N,K", [(8192, 28672, 4096), (8192, 4096, 14336), (2048, 128256, 4096),
                                   (8192, 6144, 4096), (8192, 4096, 4096), (2048, 28672, 4096),
                                   (8192, 128256, 4096)])
def test_prefill_llama3_8b_large(M, N, K):
    rows = _sample(M, 96, M, must=list(range(7, M, 128)) + [M - 1])
    stats = _chain_case("llama", M, N, K, seed=4, rows=rows, blocks=_blocks(N, 6, N))
    assert stats["max_err_over_sum"] < 1e-4


@pytest.mark.parametrize("N,K", [(2112, 7168), (24576, 7168), (7168, 7168), (4096, 7168),
                                 (7168, 2048)])
def test_deepseek_v3_m4096(N, K):
    M = 4096
    rows = _sample(M, 64, N, must=list(range(3, M, 128)) + [M - 1])
    stats = _chain_case("deepseek", M, N, K, seed=5, rows=rows, blocks=_blocks(N, 8, K))
    assert stats["max_err_over_sum"] < 1e-4


def test_prefill_exact_oracle_inputs():
    stats = _gemm_case("deepseek", 512, 1024, 1024, seed=13)
    assert stats["max_err_over_sum"] < 1e-4


@pytest.mark.parametrize("M,N,K", [(5, 8, 128), (3, 136, 256), (100, 520, 384), (200, 264, 640),
                                   (257, 264, 384), (300, 1032, 512), (130, 4104, 1024)])
def test_ragged_shapes(M, N, K):
    """Partial tiles on every side: M not a multiple of 16/128, N not a
    multiple of 128 or 256, single and few K-blocks; both operand orders."""
    stats = _gemm_case("deepseek", M, N, K, seed=6)
    assert stats["max_err_over_sum"] < 1e-4


@pytest.mark.parametrize("M", [64, 65, 128, 200, 256])
def test_operand_order_boundary_wide_n(M):
    """At 65..256 tokens a weight matrix wide enough for three quarters of a
    wave of 128 x 256 prefill tiles runs in prefill order, below 65 tokens in
    decode order: both sides of the switch, a half-filled second row tile
    (200) and a full one (256), on a 28672-row (gate+up) weight with a ragged
    last column tile avoided by N % 256 == 0 and a short K."""
    N, K = 28672, 512
    stats = _chain_case("llama", M, N, K, seed=30 + M, rows=_sample(M, 24, M, must=(0, M - 1)),
                        blocks=_blocks(N, 12, M))
    assert stats["max_err_over_sum"] < 1e-4


@pytest.mark.parametrize("M,N", [(65, 28672), (200, 14208), (128, 28288), (128, 28160)])
def test_fused_quantization_in_prefill_order_at_decode_sizes(M, N):
    """fp8_block_gemm_quant for 65..256 tokens on wide weights: the GEMM in
    either operand order, then the quantizer. On 148 SMs N = 28288 at M = 128
    is the narrowest width whose GEMM runs in prefill order (111 tiles of
    128 x 256) and 28160 the widest that stays in decode order; 28288 and 14208
    (M = 200, two row tiles) leave the last 256-column tile half empty. y equal
    to fp8_block_gemm's, codes and scales equal to the oracle's quantization of
    that y."""
    K = 384
    qa, sa, qw, sw = _quantized("llama", M, N, K, 5)
    args = [to_dev(a) for a in (qa, sa, qw, sw)]
    y_plain = fb.fp8_block_gemm(*args)
    y, qy, sy = fb.fp8_block_gemm_quant(*args)
    torch.cuda.synchronize()
    assert fb.get_device_error() == 0
    assert torch.equal(y, y_plain)
    q_ref, s_ref = oracle.quant_act_group128(y.cpu())
    np.testing.assert_array_equal(qy.cpu().numpy(), q_ref)
    np.testing.assert_array_equal(sy.cpu().numpy(), s_ref)


def test_zero_scales_and_extreme_values():
    M, N, K = 40, 272, 512
    x = synth.activations("deepseek", M, K, seed=7).float().numpy()
    x[3, :] = 0.0                     # all-zero token: every group scale is 0
    x[5, 128:256] = 0.0               # one zero group
    x[7, :] *= 1e30                   # huge activations
    w = synth.weights("deepseek", N, K, seed=7).float().numpy()
    w[:128, 256:384] = 0.0            # a zero weight block
    qa, sa = oracle.quant_act_group128(torch.from_numpy(x).to(torch.bfloat16))
    qw, sw = oracle.quant_weight_block128(torch.from_numpy(w).to(torch.bfloat16))
    y = _run(qa, sa, qw, sw)
    check_gemm(y, oracle.block_gemm(qa, sa, qw, sw), (qa, sa, qw, sw), "edge values")
    assert torch.all(y[3] == 0)


@pytest.mark.parametrize("M,N,K", [(1, 4096, 4096), (128, 6144, 4096), (2048, 4096, 4096)])
def test_deterministic_bytes(M, N, K):
    qa, sa, qw, sw = _quantized("llama", M, N, K, 8)
    args = [to_dev(a) for a in (qa, sa, qw, sw)]
    ys = [fb.fp8_block_gemm(*args) for _ in range(5)]
    torch.cuda.synchronize()
    for y in ys[1:]:
        assert torch.equal(y.view(torch.int16), ys[0].view(torch.int16))


def test_end_to_end_linear_matches_oracle():
    """quantize on the GPU then GEMM on the GPU, against the oracle chain."""
    M, N, K = 32, 6144, 4096
    x = synth.activations("llama", M, K, seed=9)
    w = synth.weights("llama", N, K, seed=9)
    qw, sw = fb.fp8_quant_weight_block128(to_dev(w))
    y = fb.fp8_linear(to_dev(x), qw, sw)
    torch.cuda.synchronize()
    qa_r, sa_r = oracle.quant_act_group128(x)
    qw_r, sw_r = oracle.quant_weight_block128(w)
    check_gemm(y, oracle.block_gemm(qa_r, sa_r, qw_r, sw_r), (qa_r, sa_r, qw_r, sw_r), "linear")


def test_output_guard_bands_untouched():
    """Output written exactly in place: canary bytes around y stay intact and
    every element of y is overwritten."""
    M, N, K = 37, 1032, 512
    qa, sa, qw, sw = _quantized("deepseek", M, N, K, 10)
    pad = 4096
    buf = torch.full((pad + M * N + pad,), -7.0, dtype=torch.bfloat16, device="cuda")
    buf[pad:pad + M * N] = float("nan")
    y = buf[pad:pad + M * N].view(M, N)
    fb.fp8_block_gemm(to_dev(qa), to_dev(sa), to_dev(qw), to_dev(sw), y=y)
    torch.cuda.synchronize()
    assert torch.all(buf[:pad] == -7.0) and torch.all(buf[pad + M * N:] == -7.0)
    assert not torch.isnan(y).any()


@pytest.mark.parametrize("M", [8, 64])
def test_bounded_wait_reports_timeout_and_recovers(M):
    """A wait limit of one cycle makes the kernel give up its first wait that
    is not already satisfied: it records FP8BS_ERR_DEVICE_TIMEOUT, drains its
    own copies and MMAs, and the next call with the default limit is correct.
    Both shapes split K over a cluster of 4 CTAs: M = 8 reduces by pushing
    partial rows into the owner CTA's receive buffer, M = 64 by reading the
    other CTAs' shared memory."""
    N, K = 4096, 4096
    qa, sa, qw, sw = _quantized("llama", M, N, K, 11)
    args = [to_dev(a) for a in (qa, sa, qw, sw)]
    fb.get_device_error()
    try:
        fb.set_wait_limit(1)
        fb.fp8_block_gemm(*args)
        assert fb.get_device_error() == 6
    finally:
        fb.set_wait_limit(0)
    y = fb.fp8_block_gemm(*args)
    assert fb.get_device_error() == 0
    check_gemm(y, oracle.block_gemm(qa, sa, qw, sw), (qa, sa, qw, sw), "after timeout")


@pytest.mark.parametrize("M,N,K", [(8, 4096, 4096), (128, 6144, 4096), (300, 640, 512),
                                   (2048, 6144, 4096), (4096, 2048, 1024), (8192, 4096, 14336),
                                   (1, 28672, 4096), (8, 9600, 512), (16, 14336, 384),
                                   (37, 14336, 384), (64, 28672, 256), (100, 12288, 512),
                                   (128, 28160, 384)])
def test_gemm_with_fused_next_layer_quantization(M, N, K):
    """fp8_block_gemm_quant gives fp8_block_gemm's y, byte for byte, and the
    next layer's 1x128 codes and scales of that bf16 y exactly as the oracle's
    activation quantizer computes them; with M > 256 (the fused epilogue) also
    when y itself is not written. N = 640 leaves the second warpgroup of the
    last column tile without a group. Up to 16 tokens with at least 75 row
    tiles (N >= 9600) the decode-order tiles run unsplit and quantize in the
    epilogue from the staged Y (M = 1, 8, 16); 17..256 tokens, and the split
    shapes (4096 and 6144 rows), write Y and run the quantizer (M = 37, 64,
    100, 128)."""
    qa, sa, qw, sw = _quantized("llama", M, N, K, 3)
    args = [to_dev(a) for a in (qa, sa, qw, sw)]
    y_plain = fb.fp8_block_gemm(*args)
    y, qy, sy = fb.fp8_block_gemm_quant(*args)
    torch.cuda.synchronize()
    assert fb.get_device_error() == 0
    assert torch.equal(y, y_plain)
    q_ref, s_ref = oracle.quant_act_group128(y.cpu())
    np.testing.assert_array_equal(qy.cpu().numpy(), q_ref)
    np.testing.assert_array_equal(sy.cpu().numpy(), s_ref)
    if M > 256:
        y2, qy2, sy2 = fb.fp8_block_gemm_quant(*args, want_y=False)
        torch.cuda.synchronize()
        assert y2 is None
        assert torch.equal(qy2, qy) and torch.equal(sy2, sy)


def test_fused_epilogue_timeout_leaves_outputs_and_recovers():
    """The fused prefill epilogue (M > 256) under a one-cycle wait limit: the
    call records FP8BS_ERR_DEVICE_TIMEOUT and writes no code or scale (the
    canary values stay), and the next call with the default limit gives the
    exact codes and scales."""
    M, N, K = 512, 1024, 1024
    qa, sa, qw, sw = _quantized("llama", M, N, K, 14)
    args = [to_dev(a) for a in (qa, sa, qw, sw)]
    qy = torch.full((M, N), 0x5A, dtype=torch.uint8, device="cuda")
    sy = torch.full((M, N // 128), -3.0, dtype=torch.float32, device="cuda")
    fb.get_device_error()
    try:
        fb.set_wait_limit(1)
        fb.fp8_block_gemm_quant(*args, qy=qy, sy=sy, want_y=False)
        assert fb.get_device_error() == 6
    finally:
        fb.set_wait_limit(0)
    assert torch.all(qy == 0x5A) and torch.all(sy == -3.0)
    y_plain = fb.fp8_block_gemm(*args)
    _, qy2, sy2 = fb.fp8_block_gemm_quant(*args, qy=qy, sy=sy, want_y=False)
    assert fb.get_device_error() == 0
    q_ref, s_ref = oracle.quant_act_group128(y_plain.cpu())
    np.testing.assert_array_equal(qy2.cpu().numpy(), q_ref)
    np.testing.assert_array_equal(sy2.cpu().numpy().view(np.uint32), s_ref.view(np.uint32))

"""GPU parity of the quantizers and the 2:4 compressor against the oracle:
E4M3 bytes, scales and metadata must be bit-exact."""

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


def _act_case(x, rows=None):
    qa, sa = fb.fp8_quant_act_group128(to_dev(x))
    torch.cuda.synchronize()
    qa, sa = qa.cpu().numpy(), sa.cpu().numpy()
    xs = x if rows is None else x[rows]
    q_ref, s_ref = oracle.quant_act_group128(xs)
    if rows is not None:
        qa, sa = qa[rows], sa[rows]
    np.testing.assert_array_equal(sa.view(np.uint32), s_ref.view(np.uint32))
    np.testing.assert_array_equal(qa, q_ref)


def test_act_quant_tiny_config():
    _act_case(synth.activations("tiny", 16, 256, seed=0))


@pytest.mark.parametrize("M", [1, 8, 32, 128])
@pytest.mark.parametrize("K", [4096, 14336])
def test_act_quant_decode_shapes(M, K):
    _act_case(synth.activations("llama", M, K, seed=1))


@pytest.mark.parametrize("M,K", [(2048, 4096), (4096, 7168), (8192, 14336)])
def test_act_quant_prefill_shapes_sampled_rows(M, K):
    kind = "deepseek" if K == 7168 else "llama"
    x = synth.activations(kind, M, K, seed=2)
    rows = np.unique(np.concatenate([[0, M - 1], np.random.default_rng(M).choice(M, 190, replace=False)]))
    _act_case(x, rows=rows)


@pytest.mark.parametrize("M", [3, 5, 33, 256, 257])
def test_act_quant_ragged_group_counts(M):
    # M * K / 128 not a multiple of 4: the last warp's unit is partial
    _act_case(synth.activations("deepseek", M, 384, seed=M))


def test_act_quant_edge_values():
    x = np.zeros((8, 512), np.float32)
    x[0, :] = 0.0
    x[0, 1::3] = -0.0                                   # all-zero group with signed zeros
    x[1, :128] = np.linspace(-448, 448, 128)            # amax 448: s = 1
    x[2, :128] = 2.0 ** -133                            # smallest bf16 subnormal amax
    x[2, 5] = -(2.0 ** -130)
    x[3, :] = 3.0e38                                    # near bf16 max
    x[3, 7] = -3.3e38
    vals = oracle.e4m3_decode(np.arange(256, dtype=np.uint8))
    vals = vals[np.isfinite(vals)]
    x[4, :254] = vals                                   # every code value, s = 1
    mids = (np.sort(np.unique(vals))[1:] + np.sort(np.unique(vals))[:-1]) / 2
    x[5, :len(mids)] = mids[:512]                       # ties: round-to-even path
    x[5, 0] = 448.0
    x[6, :] = np.random.default_rng(0).standard_normal(512) * 1e-30
    x[7, ::2] = 1.0
    x[7, 1::2] = -1e-8                                  # tiny next to a large amax
    xb = torch.from_numpy(x.astype(np.float32)).to(torch.bfloat16)
    _act_case(xb)


def _weight_case(w, row_blocks=None):
    qw, sw = fb.fp8_quant_weight_block128(to_dev(w))
    torch.cuda.synchronize()
    qw, sw = qw.cpu().numpy(), sw.cpu().numpy()
    N = w.shape[0]
    if row_blocks is None:
        q_ref, s_ref = oracle.quant_weight_block128(w)
        np.testing.assert_array_equal(sw.view(np.uint32), s_ref.view(np.uint32))
        np.testing.assert_array_equal(qw, q_ref)
        return
    for nb in row_blocks:
        r0, r1 = nb * 128, min(N, nb * 128 + 128)
        q_ref, s_ref = oracle.quant_weight_block128(w[r0:r1])
        np.testing.assert_array_equal(sw[nb:nb + 1].view(np.uint32), s_ref.view(np.uint32))
        np.testing.assert_array_equal(qw[r0:r1], q_ref)


def test_weight_quant_tiny_and_ragged():
    _weight_case(synth.weights("tiny", 256, 256, seed=0))
    _weight_case(synth.weights("deepseek", 130, 384, seed=1))
    _weight_case(synth.weights("deepseek", 2112, 7168, seed=2))


@pytest.mark.parametrize("N,K", [(6144, 4096), (4096, 14336), (128256, 4096)])
def test_weight_quant_full_shapes_sampled_blocks(N, K):
    w = synth.weights("llama", N, K, seed=3)
    NB = -(-N // 128)
    blocks = sorted(set([0, NB - 1] + list(np.random.default_rng(N).choice(NB, 6, replace=False))))
    _weight_case(w, row_blocks=blocks)


def test_weight_quant_zero_and_edge_blocks():
    w = np.zeros((256, 256), np.float32)
    w[0:128, 0:128] = -0.0                      # an all-zero block (signed zeros)
    w[128:, 128:] = 3.0e38
    w[128, 200] = -3.3e38
    w[0:128, 128:] = np.random.default_rng(1).standard_normal((128, 128)) * 1e-38
    _weight_case(torch.from_numpy(w).to(torch.bfloat16))


def _prune_case(w, row_blocks=None):
    vals, meta, sw, wp = fb.prune24_compress(to_dev(w), want_pruned=True)
    torch.cuda.synchronize()
    vals, meta, sw = vals.cpu().numpy(), meta.cpu().numpy(), sw.cpu().numpy()
    wp = wp.float().cpu().numpy()
    N = w.shape[0]
    blocks = [None] if row_blocks is None else row_blocks
    for nb in blocks:
        r0, r1 = (0, N) if nb is None else (nb * 128, min(N, nb * 128 + 128))
        s0, s1 = (0, sw.shape[0]) if nb is None else (nb, nb + 1)
        v_ref, m_ref, s_ref, wp_ref = oracle.prune24_compress(w[r0:r1])
        np.testing.assert_array_equal(meta[r0:r1], m_ref)
        np.testing.assert_array_equal(vals[r0:r1], v_ref)
        np.testing.assert_array_equal(sw[s0:s1].view(np.uint32), s_ref.view(np.uint32))
        np.testing.assert_array_equal(wp[r0:r1].view(np.uint32), wp_ref.view(np.uint32))


def test_prune_small_with_ties():
    rng = np.random.default_rng(7)
    w = rng.integers(-3, 4, size=(200, 256)).astype(np.float32) * 0.25
    w[0, :8] = [0.0, -0.0, 0.0, -0.0, 1.0, -1.0, 1.0, -1.0]
    _prune_case(torch.from_numpy(w).to(torch.bfloat16))


@pytest.mark.parametrize("N,K", [(14336, 4096), (4096, 14336)])
def test_prune_sparse_config_sampled_blocks(N, K):
    w = synth.weights("llama", N, K, seed=5)
    NB = -(-N // 128)
    blocks = sorted(set([0, NB - 1] + list(np.random.default_rng(K).choice(NB, 4, replace=False))))
    _prune_case(w, row_blocks=blocks)


def _all_patterns_matrix():
    """Rows of 256 groups of 4 covering every assignment of 4 magnitude levels
    to the 4 positions of a group (4^4 patterns, so every tie structure), for
    three level sets: small multiples of 0.25, adjacent bf16 values, and the
    extremes of the bf16 magnitude range (0, smallest subnormal, the two
    largest finite values). Signs are random per element."""
    levels = [np.array([0x0000, 0x3E80, 0x3F00, 0x3F40], np.uint16),   # 0, .25, .5, .75
              np.array([0x3F80, 0x3F81, 0x3F82, 0x3F83], np.uint16),   # adjacent bf16
              np.array([0x0000, 0x0001, 0x7F7E, 0x7F7F], np.uint16)]   # range ends
    idx = np.array(np.meshgrid(*[np.arange(4)] * 4, indexing="ij")).reshape(4, -1).T  # [256, 4]
    rng = np.random.default_rng(11)
    rows = []
    for lv in levels:
        for r in range(128):
            perm = np.roll(idx, r, axis=0)               # each row holds every pattern
            bits = lv[perm].reshape(-1)
            sign = rng.integers(0, 2, size=bits.shape).astype(np.uint16) << 15
            rows.append(bits | sign)
    return torch.from_numpy(np.stack(rows).view(np.int16)).view(torch.bfloat16)


def test_prune_every_tie_pattern():
    w = _all_patterns_matrix()                      # [384, 1024]
    _prune_case(w)
    # the path without the pruned output writes the same bytes
    a = fb.prune24_compress(to_dev(w), want_pruned=True)
    b = fb.prune24_compress(to_dev(w))
    torch.cuda.synchronize()
    for x, y in zip(a[:3], b[:3]):
        assert torch.equal(x.view(torch.uint8), y.view(torch.uint8))

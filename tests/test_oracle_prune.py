"""Pins of the oracle's 2:4 pruning and compression: brute force over the six
pairs of each group, torch.topk on tie-free inputs (the selection the 2:4 mask
example computes), and format invariants."""

import itertools

import numpy as np
import torch

import oracle
from fp8_block_scaled_group128_b200 import synth


def _brute_force_pair(group):
    """Kept pair by exhaustive ranking: sort positions by (-|w|, index)."""
    order = sorted(range(4), key=lambda i: (-abs(float(group[i])), i))
    return tuple(sorted(order[:2]))


def test_brute_force_on_small_groups_with_ties():
    rng = np.random.default_rng(0)
    # small integer magnitudes make ties (and +-0) frequent
    w = rng.integers(-3, 4, size=(64, 128)).astype(np.float32)
    w[0, :4] = [0.0, -0.0, 0.0, -0.0]
    i0, i1 = oracle.fp8_oracle.prune24_select(w)
    for n in range(w.shape[0]):
        for g in range(w.shape[1] // 4):
            assert (i0[n, g], i1[n, g]) == _brute_force_pair(w[n, 4 * g:4 * g + 4])
    assert (i0[0, 0], i1[0, 0]) == (0, 1)      # all-zero group keeps {0, 1}


def test_matches_topk_selection_on_tie_free_inputs():
    # The 2:4 mask example ("Déployer la parcimonie 2:4 avec FP8 sur Hopper",
    # Exemples pratiques 1) keeps the top-2 |w| of each group of 4 along K.
    rng = np.random.default_rng(11)
    # distinct magnitudes within each group by construction: a permutation of
    # {1, 2, 3, 4} times a per-group power of two, with random signs
    perm = np.argsort(rng.random((96, 128, 4)), axis=-1) + 1.0
    scale = np.exp2(rng.integers(-12, 2, size=(96, 128, 1)))
    sign = np.where(rng.random((96, 128, 4)) < 0.5, -1.0, 1.0)
    wf = torch.from_numpy((perm * scale * sign).reshape(96, 512).astype(np.float32))
    g = wf.reshape(96, 128, 4).abs()
    assert (g.sort(dim=-1).values.diff(dim=-1) > 0).all(), "inputs must be tie-free"
    top = g.topk(k=2, dim=-1).indices
    mask = torch.zeros_like(g, dtype=torch.bool).scatter_(-1, top, True)
    i0, i1 = oracle.fp8_oracle.prune24_select(wf.numpy())
    idx = np.arange(4)
    ours = (idx == i0[..., None]) | (idx == i1[..., None])
    np.testing.assert_array_equal(ours, mask.numpy())


def test_compressed_format_invariants():
    w = synth.weights("llama", 200, 384, seed=4)
    vals, meta, sw, wp = oracle.prune24_compress(w)
    N, K = 200, 384
    assert vals.shape == (N, K // 2) and meta.shape == (N, K // 8) and sw.shape == (2, 3)
    nib = np.stack([meta & 0xF, meta >> 4], axis=-1).reshape(N, K // 4)
    i0, i1 = nib & 3, nib >> 2
    assert np.all(i0 < i1)
    # exactly two nonzeros per group on Gaussian weights; pruned zeros are +0
    g = wp.reshape(N, K // 4, 4)
    assert np.all((g != 0).sum(-1) == 2)
    assert not np.any(np.signbit(g[g == 0]))
    # kept magnitudes dominate dropped ones
    wf = w.float().numpy().reshape(N, K // 4, 4)
    kept = np.abs(np.where(g != 0, wf, np.nan))
    drop = np.abs(np.where(g == 0, wf, np.nan))
    assert np.all(np.nanmin(kept, -1) >= np.nanmax(drop, -1))
    # the pruned matrix keeps the original values exactly where kept
    np.testing.assert_array_equal(np.where(g != 0, g, 0), np.where(g != 0, wf, 0))
    # decompression equals quantizing the pruned weights densely
    qd, sd = oracle.quant_weight_block128(wp)
    np.testing.assert_array_equal(oracle.decompress24(vals, meta), qd)
    np.testing.assert_array_equal(sw, sd)


def test_block_scales_unchanged_by_pruning():
    """Each group's largest magnitude is always kept, so every block's amax
    (and scale) equals the unpruned one."""
    w = synth.weights("deepseek", 256, 512, seed=6)
    _, _, sw_sparse, _ = oracle.prune24_compress(w)
    _, sw_dense = oracle.quant_weight_block128(w)
    np.testing.assert_array_equal(sw_sparse, sw_dense)


def test_meta_nibble_encoding_all_pairs():
    for (a, b) in itertools.combinations(range(4), 2):
        w = np.zeros((1, 128), np.float32)
        w[0, a], w[0, b] = 2.0, -3.0
        w[0, 4 + a], w[0, 4 + b] = 1.0, 1.0
        vals, meta, sw, _ = oracle.prune24_compress(w)
        assert meta[0, 0] == (a | b << 2) | ((a | b << 2) << 4)
        # vals hold the codes in position order: 2/s and -3/s with s = 3/448
        q = oracle.e4m3_encode(np.array([2.0, -3.0], np.float32) / (np.float32(3) / np.float32(448)))
        assert tuple(vals[0, :2]) == tuple(q)

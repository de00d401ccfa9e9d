"""Pins of the oracle's 2:4 pruning and compression: brute force over the six
pairs of each group, an independent stable-sort ranking on tie-free inputs,
and format invariants. Every pin runs against both statements of the oracle
(C++ and numpy)."""

import itertools

import numpy as np
import torch

from fp8_block_scaled_group128_b200 import synth


def _select(impl, w):
    """Kept positions (i0, i1) of every group, read back from the metadata
    nibbles that prune24_compress writes."""
    _, meta, _, _ = impl.prune24_compress(w)
    N = meta.shape[0]
    nib = np.stack([meta & 0xF, meta >> 4], axis=-1).reshape(N, -1)
    return (nib & 3).astype(np.int64), (nib >> 2).astype(np.int64)


def _brute_force_pair(group):
    """Kept pair by exhaustive ranking: sort positions by (-|w|, index)."""
    order = sorted(range(4), key=lambda i: (-abs(float(group[i])), i))
    return tuple(sorted(order[:2]))


def test_brute_force_on_small_groups_with_ties(impl):
    rng = np.random.default_rng(0)
    # small integer magnitudes make ties (and +-0) frequent
    w = rng.integers(-3, 4, size=(64, 128)).astype(np.float32)
    w[0, :4] = [0.0, -0.0, 0.0, -0.0]
    i0, i1 = _select(impl, w)
    for n in range(w.shape[0]):
        for g in range(w.shape[1] // 4):
            assert (i0[n, g], i1[n, g]) == _brute_force_pair(w[n, 4 * g:4 * g + 4])
    assert (i0[0, 0], i1[0, 0]) == (0, 1)      # all-zero group keeps {0, 1}


def test_matches_magnitude_ranking_on_tie_free_inputs(impl):
    # The two largest |w| of each group of 4 along K are kept ("Déployer la
    # parcimonie 2:4 avec FP8 sur Hopper", pipeline step 4): on inputs with
    # distinct magnitudes the kept set is the first two positions of a
    # descending stable sort of |w|.
    rng = np.random.default_rng(11)
    # distinct magnitudes within each group by construction: a permutation of
    # {1, 2, 3, 4} times a per-group power of two, with random signs
    perm = np.argsort(rng.random((96, 128, 4)), axis=-1) + 1.0
    scale = np.exp2(rng.integers(-12, 2, size=(96, 128, 1)))
    sign = np.where(rng.random((96, 128, 4)) < 0.5, -1.0, 1.0)
    wf = (perm * scale * sign).reshape(96, 512).astype(np.float32)
    mag = np.abs(wf.reshape(96, 128, 4))
    assert (np.diff(np.sort(mag, axis=-1), axis=-1) > 0).all(), "inputs must be tie-free"
    first_two = np.argsort(-mag, axis=-1, kind="stable")[..., :2]
    want = np.zeros(mag.shape, bool)
    np.put_along_axis(want, first_two, True, axis=-1)
    i0, i1 = _select(impl, wf)
    idx = np.arange(4)
    ours = (idx == i0[..., None]) | (idx == i1[..., None])
    np.testing.assert_array_equal(ours, want)


def test_compressed_format_invariants(impl):
    w = synth.weights("llama", 200, 384, seed=4)
    vals, meta, sw, wp = impl.prune24_compress(w)
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
    qd, sd = impl.quant_weight_block128(wp)
    np.testing.assert_array_equal(impl.decompress24(vals, meta), qd)
    np.testing.assert_array_equal(sw, sd)


def test_block_scales_unchanged_by_pruning(impl):
    """Each group's largest magnitude is always kept, so every block's amax
    (and scale) equals the unpruned one."""
    w = synth.weights("deepseek", 256, 512, seed=6)
    _, _, sw_sparse, _ = impl.prune24_compress(w)
    _, sw_dense = impl.quant_weight_block128(w)
    np.testing.assert_array_equal(sw_sparse, sw_dense)


def test_meta_nibble_encoding_all_pairs(impl):
    for (a, b) in itertools.combinations(range(4), 2):
        w = np.zeros((1, 128), np.float32)
        w[0, a], w[0, b] = 2.0, -3.0
        w[0, 4 + a], w[0, 4 + b] = 1.0, 1.0
        vals, meta, sw, _ = impl.prune24_compress(w)
        assert meta[0, 0] == (a | b << 2) | ((a | b << 2) << 4)
        # vals hold the codes in position order: 2/s and -3/s with s = 3/448
        q = impl.e4m3_encode(np.array([2.0, -3.0], np.float32) / (np.float32(3) / np.float32(448)))
        assert tuple(vals[0, :2]) == tuple(q)

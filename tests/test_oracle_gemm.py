"""Pins of the oracle's block-scaled GEMMs: a hand-computed product, exact
integer and power-of-two cases, and brute-force dequantize-then-matmul in
float64 torch (an independent route to the same sum)."""

import numpy as np
import torch

import oracle
from fp8_block_scaled_group128_b200 import synth


def test_hand_computed_two_by_two():
    # K = 256 (two K-blocks), M = N = 2.
    qa = np.zeros((2, 256), np.uint8)
    qa[0, :128] = 0x38            # 1.0
    qa[0, 128:] = 0x40            # 2.0
    qa[1, 0] = 0xC0               # -2.0, only one nonzero
    sa = np.array([[0.5, 0.25], [3.0, 7.0]], np.float32)
    qw = np.zeros((2, 256), np.uint8)
    qw[0, :] = 0x38               # 1.0 everywhere
    qw[1, 128:] = 0x30            # 0.5 in the second K-block only
    sw = np.array([[1.0, 2.0]], np.float32)
    y = oracle.block_gemm(qa, sa, qw, sw)
    # y00 = 0.5*1*(128*1*1) + 0.25*2*(128*2*1) = 64 + 128 = 192
    # y01 = 0 + 0.25*2*(128*2*0.5) = 64
    # y10 = 3*1*(-2*1) = -6 ; y11 = 0
    np.testing.assert_array_equal(y, np.array([[192.0, 64.0], [-6.0, 0.0]]))


def test_ragged_n_uses_row_block_scales():
    # N = 130: rows 128, 129 take the second scale row.
    qa = np.full((1, 128), 0x38, np.uint8)
    sa = np.ones((1, 1), np.float32)
    qw = np.full((130, 128), 0x38, np.uint8)
    sw = np.array([[1.0], [0.5]], np.float32)
    y = oracle.block_gemm(qa, sa, qw, sw)
    assert np.all(y[0, :128] == 128.0) and np.all(y[0, 128:] == 64.0)
    y_cols = oracle.block_gemm(qa, sa, qw, sw, cols=[127, 128, 3])
    np.testing.assert_array_equal(y_cols[0], [128.0, 64.0, 128.0])


def test_exact_integer_case():
    rng = np.random.default_rng(2)
    ints = np.array([oracle.e4m3_encode(np.array([v], np.float32))[0] for v in range(-16, 17)], np.uint8)
    qa = rng.choice(ints, size=(5, 384))
    qw = rng.choice(ints, size=(7, 384))
    ones_a = np.ones((5, 3), np.float32)
    ones_w = np.ones((1, 3), np.float32)
    y = oracle.block_gemm(qa, ones_a, qw, ones_w)
    a = oracle.e4m3_decode(qa).astype(np.int64)
    w = oracle.e4m3_decode(qw).astype(np.int64)
    np.testing.assert_array_equal(y, (a @ w.T).astype(np.float64))   # integer arithmetic


def test_matches_dequantize_then_matmul_float64():
    M, N, K = 9, 300, 640                 # ragged N, several K-blocks, M != N != K
    x = synth.activations("deepseek", M, K, seed=1)
    w = synth.weights("deepseek", N, K, seed=1)
    qa, sa = oracle.quant_act_group128(x)
    qw, sw = oracle.quant_weight_block128(w)
    y = oracle.block_gemm(qa, sa, qw, sw)
    # dequantize every element with its own scale, then one float64 matmul
    a = torch.from_numpy(oracle.e4m3_decode(qa)) * torch.from_numpy(sa.astype(np.float64)).repeat_interleave(128, 1)
    sw_rows = torch.from_numpy(sw.astype(np.float64)).repeat_interleave(128, 0)[:N]
    wd = torch.from_numpy(oracle.e4m3_decode(qw)) * sw_rows.repeat_interleave(128, 1)
    ref = (a @ wd.T).numpy()
    np.testing.assert_allclose(y, ref, rtol=1e-12, atol=1e-12 * np.abs(ref).max())
    # and the quantized product approximates the bf16 product
    exact = (x.double() @ w.double().T).numpy()
    bound = oracle.gemm_error_bound(qa, sa, qw, sw, rel=0.2)
    assert np.all(np.abs(y - exact) <= bound + 1e-30)


def test_power_of_two_scales_exact():
    rng = np.random.default_rng(3)
    qa = rng.integers(0, 256, size=(4, 256)).astype(np.uint8)
    qw = rng.integers(0, 256, size=(3, 256)).astype(np.uint8)
    qa[(qa & 0x7F) == 0x7F] = 0x38     # no NaN codes
    qw[(qw & 0x7F) == 0x7F] = 0x38
    sa = np.exp2(rng.integers(-8, 8, size=(4, 2))).astype(np.float32)
    sw = np.exp2(rng.integers(-8, 8, size=(1, 2))).astype(np.float32)
    y = oracle.block_gemm(qa, sa, qw, sw)
    a = oracle.e4m3_decode(qa)
    w = oracle.e4m3_decode(qw)
    want = np.zeros((4, 3))
    for m in range(4):
        for n in range(3):
            for k in range(256):
                want[m, n] += a[m, k] * sa[m, k // 128] * w[n, k] * sw[0, k // 128]
    np.testing.assert_array_equal(y, want)   # every term and partial sum exact


def test_sparse_equals_dense_on_pruned_weights():
    x = synth.activations("llama", 6, 512, seed=8)
    w = synth.weights("llama", 260, 512, seed=8)
    qa, sa = oracle.quant_act_group128(x)
    vals, meta, sw, wp = oracle.prune24_compress(w)
    qd, sd = oracle.quant_weight_block128(wp)
    ys = oracle.sparse24_gemm(qa, sa, vals, meta, sw)
    yd = oracle.block_gemm(qa, sa, qd, sd)
    np.testing.assert_array_equal(ys, yd)
    cols = [0, 129, 259]
    np.testing.assert_array_equal(oracle.sparse24_gemm(qa, sa, vals, meta, sw, cols=cols), yd[:, cols])


def test_bf16_ulp():
    assert oracle.bf16_ulp(np.array([1.0]))[0] == 2.0 ** -7
    assert oracle.bf16_ulp(np.array([-3.0]))[0] == 2.0 ** -6
    assert oracle.bf16_ulp(np.array([0.0]))[0] == 2.0 ** -133

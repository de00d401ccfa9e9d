"""Pins of the oracle's block-scaled GEMMs: a hand-computed product, exact
integer and power-of-two cases, and brute-force dequantize-then-matmul in
float64 torch (an independent route to the same sum)."""

import numpy as np
import torch

import oracle
from fp8_block_scaled_group128_b200 import synth


def test_hand_computed_two_by_two(impl):
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
    y = impl.block_gemm(qa, sa, qw, sw)
    # y00 = 0.5*1*(128*1*1) + 0.25*2*(128*2*1) = 64 + 128 = 192
    # y01 = 0 + 0.25*2*(128*2*0.5) = 64
    # y10 = 3*1*(-2*1) = -6 ; y11 = 0
    np.testing.assert_array_equal(y, np.array([[192.0, 64.0], [-6.0, 0.0]]))


def test_ragged_n_uses_row_block_scales(impl):
    # N = 130: rows 128, 129 take the second scale row.
    qa = np.full((1, 128), 0x38, np.uint8)
    sa = np.ones((1, 1), np.float32)
    qw = np.full((130, 128), 0x38, np.uint8)
    sw = np.array([[1.0], [0.5]], np.float32)
    y = impl.block_gemm(qa, sa, qw, sw)
    assert np.all(y[0, :128] == 128.0) and np.all(y[0, 128:] == 64.0)
    y_cols = impl.block_gemm(qa, sa, qw, sw, cols=[127, 128, 3])
    np.testing.assert_array_equal(y_cols[0], [128.0, 64.0, 128.0])


def test_exact_integer_case(impl):
    rng = np.random.default_rng(2)
    ints = np.array([impl.e4m3_encode(np.array([v], np.float32))[0] for v in range(-16, 17)], np.uint8)
    qa = rng.choice(ints, size=(5, 384))
    qw = rng.choice(ints, size=(7, 384))
    ones_a = np.ones((5, 3), np.float32)
    ones_w = np.ones((1, 3), np.float32)
    y = impl.block_gemm(qa, ones_a, qw, ones_w)
    a = impl.e4m3_decode(qa).astype(np.int64)
    w = impl.e4m3_decode(qw).astype(np.int64)
    np.testing.assert_array_equal(y, (a @ w.T).astype(np.float64))   # integer arithmetic


def test_matches_dequantize_then_matmul_float64(impl):
    M, N, K = 9, 300, 640                 # ragged N, several K-blocks, M != N != K
    x = synth.activations("deepseek", M, K, seed=1)
    w = synth.weights("deepseek", N, K, seed=1)
    qa, sa = impl.quant_act_group128(x)
    qw, sw = impl.quant_weight_block128(w)
    y = impl.block_gemm(qa, sa, qw, sw)
    # dequantize every element with its own scale, then one float64 matmul
    a = torch.from_numpy(impl.e4m3_decode(qa)) * torch.from_numpy(sa.astype(np.float64)).repeat_interleave(128, 1)
    sw_rows = torch.from_numpy(sw.astype(np.float64)).repeat_interleave(128, 0)[:N]
    wd = torch.from_numpy(impl.e4m3_decode(qw)) * sw_rows.repeat_interleave(128, 1)
    ref = (a @ wd.T).numpy()
    np.testing.assert_allclose(y, ref, rtol=1e-12, atol=1e-12 * np.abs(ref).max())
    # and the quantized product approximates the bf16 product
    exact = (x.double() @ w.double().T).numpy()
    bound = impl.gemm_error_bound(qa, sa, qw, sw, rel=0.2)
    assert np.all(np.abs(y - exact) <= bound + 1e-30)


def test_power_of_two_scales_exact(impl):
    rng = np.random.default_rng(3)
    qa = rng.integers(0, 256, size=(4, 256)).astype(np.uint8)
    qw = rng.integers(0, 256, size=(3, 256)).astype(np.uint8)
    qa[(qa & 0x7F) == 0x7F] = 0x38     # no NaN codes
    qw[(qw & 0x7F) == 0x7F] = 0x38
    sa = np.exp2(rng.integers(-8, 8, size=(4, 2))).astype(np.float32)
    sw = np.exp2(rng.integers(-8, 8, size=(1, 2))).astype(np.float32)
    y = impl.block_gemm(qa, sa, qw, sw)
    a = impl.e4m3_decode(qa)
    w = impl.e4m3_decode(qw)
    want = np.zeros((4, 3))
    for m in range(4):
        for n in range(3):
            for k in range(256):
                want[m, n] += a[m, k] * sa[m, k // 128] * w[n, k] * sw[0, k // 128]
    np.testing.assert_array_equal(y, want)   # every term and partial sum exact


def test_sparse_equals_dense_on_pruned_weights(impl):
    x = synth.activations("llama", 6, 512, seed=8)
    w = synth.weights("llama", 260, 512, seed=8)
    qa, sa = impl.quant_act_group128(x)
    vals, meta, sw, wp = impl.prune24_compress(w)
    qd, sd = impl.quant_weight_block128(wp)
    ys = impl.sparse24_gemm(qa, sa, vals, meta, sw)
    yd = impl.block_gemm(qa, sa, qd, sd)
    np.testing.assert_array_equal(ys, yd)
    cols = [0, 129, 259]
    np.testing.assert_array_equal(impl.sparse24_gemm(qa, sa, vals, meta, sw, cols=cols), yd[:, cols])


def test_bf16_ulp(impl):
    assert impl.bf16_ulp(np.array([1.0]))[0] == 2.0 ** -7
    assert impl.bf16_ulp(np.array([-3.0]))[0] == 2.0 ** -6
    assert impl.bf16_ulp(np.array([0.0]))[0] == 2.0 ** -133


def _two_by_two_operands():
    """The operands of test_hand_computed_two_by_two."""
    qa = np.zeros((2, 256), np.uint8)
    qa[0, :128] = 0x38            # 1.0
    qa[0, 128:] = 0x40            # 2.0
    qa[1, 0] = 0xC0               # -2.0
    sa = np.array([[0.5, 0.25], [3.0, 7.0]], np.float32)
    qw = np.zeros((2, 256), np.uint8)
    qw[0, :] = 0x38
    qw[1, 128:] = 0x30            # 0.5
    sw = np.array([[1.0, 2.0]], np.float32)
    return qa, sa, qw, sw


def test_error_bound_hand_computed(impl):
    """The parity tolerance rel * sum_k |a_k w_k| on hand-computed operands.
    sum |a w|: y00 = 0.5*1*128 + 0.25*2*(128*2*1) = 192; y01 = 0.25*2*(128*2*0.5)
    = 64; y10 = 3*1*|-2*1| = 6; y11 = 0 (row 1 meets only zero weights)."""
    qa, sa, qw, sw = _two_by_two_operands()
    np.testing.assert_array_equal(impl.gemm_error_bound(qa, sa, qw, sw, rel=1.0),
                                  [[192.0, 64.0], [6.0, 0.0]])
    # the default rel is the parity bound's 1e-2
    np.testing.assert_allclose(impl.gemm_error_bound(qa, sa, qw, sw),
                               [[1.92, 0.64], [0.06, 0.0]], rtol=1e-15)
    np.testing.assert_array_equal(impl.gemm_error_bound(qa, sa, qw, sw, cols=[1], rel=1.0),
                                  [[64.0], [0.0]])


def test_error_bound_counts_magnitudes_not_the_signed_sum(impl):
    """Terms of opposite sign cancel in y but not in the bound: a = (+1 x 64,
    -1 x 64), w = 1 gives y = 0 and sum |a w| = 128; a negative weight block
    and a negative code change nothing."""
    qa = np.zeros((1, 128), np.uint8)
    qa[0, :64] = 0x38
    qa[0, 64:] = 0xB8             # -1.0
    qw = np.full((2, 128), 0x38, np.uint8)
    qw[1] = 0xB8
    sa = np.ones((1, 1), np.float32)
    sw = np.array([[0.25]], np.float32)
    np.testing.assert_array_equal(impl.block_gemm(qa, sa, qw, sw), [[0.0, 0.0]])
    np.testing.assert_array_equal(impl.gemm_error_bound(qa, sa, qw, sw, rel=1.0), [[32.0, 32.0]])


def test_error_bound_ragged_row_blocks(impl):
    """N = 130: rows 128, 129 take the second scale row; K = 256 with
    different block scales per K-block; sum |a w| = sum_kb 128 * |sa| * |sw|."""
    qa = np.full((1, 256), 0x40, np.uint8)      # 2.0
    sa = np.array([[1.0, 0.5]], np.float32)
    qw = np.full((130, 256), 0xB0, np.uint8)    # -0.5
    sw = np.array([[1.0, 4.0], [0.125, 8.0]], np.float32)
    b = impl.gemm_error_bound(qa, sa, qw, sw, rel=1.0)
    # rows < 128: 128*2*0.5*(1*1 + 0.5*4) = 384 ; rows 128, 129: 128*(0.125 + 0.5*8) = 528
    assert np.all(b[0, :128] == 384.0) and np.all(b[0, 128:] == 528.0)
    np.testing.assert_array_equal(impl.gemm_error_bound(qa, sa, qw, sw, cols=[129, 0], rel=1.0),
                                  [[528.0, 384.0]])


def test_cpp_and_numpy_statements_agree():
    """The two statements of the oracle give the same codes, scales, metadata,
    pruned weights and GEMM outputs, bit for bit, on every workload kind (and
    bounds equal up to the summation order of sum |a w|)."""
    import oracle
    c, n = oracle.cpp_oracle, oracle.numpy_oracle
    for kind, M, N, K, seed in (("tiny", 16, 256, 256, 0), ("llama", 33, 520, 1024, 1),
                                ("deepseek", 9, 300, 640, 2)):
        x = synth.activations(kind, M, K, seed=seed)
        w = synth.weights(kind, N, K, seed=seed)
        for f in ("quant_act_group128", "quant_weight_block128", "prune24_compress",
                  "quant_act_group128_ue8m0", "quant_weight_block128_ue8m0"):
            arg = x if f.startswith("quant_act") else w
            for a, b in zip(getattr(c, f)(arg), getattr(n, f)(arg)):
                np.testing.assert_array_equal(np.asarray(a).view(np.uint8), np.asarray(b).view(np.uint8))
        qa, sa = c.quant_act_group128(x)
        qw, sw = c.quant_weight_block128(w)
        vals, meta, sws, _ = c.prune24_compress(w)
        np.testing.assert_array_equal(c.block_gemm(qa, sa, qw, sw), n.block_gemm(qa, sa, qw, sw))
        np.testing.assert_array_equal(c.sparse24_gemm(qa, sa, vals, meta, sws),
                                      n.sparse24_gemm(qa, sa, vals, meta, sws))
        np.testing.assert_array_equal(c.decompress24(vals, meta), n.decompress24(vals, meta))
        np.testing.assert_allclose(c.gemm_error_bound(qa, sa, qw, sw),
                                   n.gemm_error_bound(qa, sa, qw, sw), rtol=1e-13)


def test_cpp_oracle_result_does_not_depend_on_thread_count():
    import oracle
    x = synth.activations("llama", 5, 512, seed=3)
    w = synth.weights("llama", 260, 512, seed=3)
    qa, sa = oracle.quant_act_group128(x)
    qw, sw = oracle.quant_weight_block128(w)
    y_all = oracle.block_gemm(qa, sa, qw, sw)
    try:
        oracle.set_threads(1)
        assert oracle.threads() == 1
        np.testing.assert_array_equal(oracle.block_gemm(qa, sa, qw, sw), y_all)
        np.testing.assert_array_equal(oracle.quant_weight_block128(w)[0], qw)
    finally:
        oracle.set_threads(0)


def test_grouped_gemm_hand_computed(impl):
    """Two experts, K = 128: a row of 1.0 codes (scale 1) against expert 0
    (codes 1.0, scale 1) gives 128; against expert 1 (codes 1.5, scale 2)
    128 * 1.5 * 2 = 384; a padding row (-1) has no result (NaN)."""
    qa = np.full((3, 128), 0x38, np.uint8)
    sa = np.ones((3, 1), np.float32)
    qw = np.stack([np.full((8, 128), 0x38, np.uint8), np.full((8, 128), 0x3C, np.uint8)])
    sw = np.array([[[1.0]], [[2.0]]], np.float32)
    y = impl.grouped_gemm(qa, sa, qw, sw, np.array([0, 1, -1], np.int32))
    np.testing.assert_array_equal(y[0], np.full(8, 128.0))
    np.testing.assert_array_equal(y[1], np.full(8, 384.0))
    assert np.all(np.isnan(y[2]))


def test_grouped_gemm_reduces_to_the_dense_gemm(impl):
    """One expert holding every row is the dense GEMM; an expert whose weights
    are another's with every block scale times 4 gives exactly 4x its rows."""
    x = synth.activations("deepseek", 10, 384, seed=12)
    w = synth.weights("deepseek", 260, 384, seed=12)
    qa, sa = impl.quant_act_group128(x)
    qw, sw = impl.quant_weight_block128(w)
    np.testing.assert_array_equal(
        impl.grouped_gemm(qa, sa, qw[None], sw[None], np.zeros(10, np.int32)),
        impl.block_gemm(qa, sa, qw, sw))
    mi = np.array([1, 0, 0, 1, -1, 1, 0, 0, 1, 1], np.int32)
    y = impl.grouped_gemm(qa, sa, np.stack([qw, qw]), np.stack([sw, sw * 4]), mi)
    dense = impl.block_gemm(qa, sa, qw, sw)
    np.testing.assert_array_equal(y[mi == 0], dense[mi == 0])
    np.testing.assert_array_equal(y[mi == 1], 4.0 * dense[mi == 1])
    assert np.all(np.isnan(y[mi == -1]))


def test_swiglu_closed_forms(impl):
    """silu(g) = g * sigmoid(g): sigmoid(ln 3) = 3/4 and sigmoid(-ln 3) = 1/4,
    silu(0) = 0, silu(g) -> g for large g and -> 0 for very negative g."""
    import math
    ln3 = math.log(3.0)
    g = np.array([0.0, ln3, -ln3, 40.0, -800.0, 1.0])
    u = np.array([5.0, 2.0, 2.0, 1.0, 3.0, -1.0])
    h = impl.swiglu(g, u)
    want = np.array([0.0, 2 * 0.75 * ln3, 2 * -0.25 * ln3, 40.0, 0.0, -1.0 / (1.0 + math.exp(-1.0))])
    np.testing.assert_allclose(h, want, rtol=1e-15, atol=1e-300)
    assert abs(h[4]) < 1e-300


def test_swiglu_bound_hand_computed_and_slope_below_1_1(impl):
    """The tolerance at g = ln 3, u = 2, tg = 0.1, tu = 0.2:
    1.1 * 0.1 * (2 + 0.2) + (0.75 ln 3) * 0.2 + 1e-5 * (1.5 ln 3); and the
    slope of silu, by central differences on a fine grid, stays below 1.1
    in magnitude (the constant the bound uses)."""
    import math
    ln3 = math.log(3.0)
    b = impl.swiglu_error_bound(np.array([ln3]), np.array([2.0]), np.array([0.1]), np.array([0.2]))
    want = 1.1 * 0.1 * 2.2 + 0.75 * ln3 * 0.2 + 1e-5 * 1.5 * ln3
    np.testing.assert_allclose(b, [want], rtol=1e-14)
    z = np.linspace(-30, 30, 600001)
    eps = 1e-6
    slope = (impl.swiglu(z + eps, np.ones_like(z)) - impl.swiglu(z - eps, np.ones_like(z))) / (2 * eps)
    assert np.abs(slope).max() < 1.1 and np.abs(slope).max() > 1.09


def test_gemm_swiglu_hand_computed(impl):
    """I = 128, K = 128: every activation 1.0, gate weights 1.0 with block
    scale ln(3)/128, up weights 0.5 with scale 1/32: g = ln 3, u = 128 * 0.5
    / 32 = 2, so h = 2 * 0.75 * ln 3 for every output."""
    import math
    qa = np.full((2, 128), 0x38, np.uint8)
    sa = np.ones((2, 1), np.float32)
    qw = np.concatenate([np.full((128, 128), 0x38, np.uint8), np.full((128, 128), 0x30, np.uint8)])
    s_gate = np.float32(math.log(3.0) / 128)
    sw = np.array([[s_gate], [1.0 / 32]], np.float32)
    h, tol = impl.gemm_swiglu(qa, sa, qw, sw)
    g = 128 * float(s_gate)
    np.testing.assert_allclose(h, np.full((2, 128), g / (1 + math.exp(-g)) * 2.0), rtol=1e-15)
    assert np.all(tol > 0)

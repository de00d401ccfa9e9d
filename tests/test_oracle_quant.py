"""Pins of the oracle's activation and weight quantizers: a hand-worked group,
closed-form scales, and invariants that follow from scale = amax/448."""

import numpy as np
import torch

import oracle
from fp8_block_scaled_group128_b200 import synth


def test_worked_activation_groups(impl, golden):
    rows = golden("act_group_worked.txt")
    x = np.zeros((1, 384), np.float32)
    x[0, 128 + 64:256] = -0.0
    want = {}
    scales = {}
    for r in rows:
        if r[0] == "scale":
            scales[int(r[1])] = float(r[2])
        else:
            g, i, v, code = int(r[1]), int(r[2]), float(r[3]), int(r[4], 16)
            x[0, 128 * g + i] = np.float32(v)
            want[128 * g + i] = code
    xb = torch.from_numpy(x).to(torch.bfloat16)
    assert torch.equal(xb.float(), torch.from_numpy(x)), "fixture values must be bf16-exact"
    q, s = impl.quant_act_group128(xb)
    for g, sv in scales.items():
        assert s[0, g] == np.float32(sv)
    for k in range(384):
        if k in want:
            assert q[0, k] == want[k], (k, hex(q[0, k]), hex(want[k]))
        elif 128 + 64 <= k < 256:
            assert q[0, k] == 0x80
        else:
            assert q[0, k] == 0x00


def test_scale_closed_forms_and_max_code(impl):
    x = synth.activations("llama", 7, 512, seed=3).float().numpy()
    q, s = impl.quant_act_group128(x)
    amax = np.abs(x.reshape(7, 4, 128)).max(axis=2)
    np.testing.assert_array_equal(s, (amax / np.float32(448)).astype(np.float32))
    # the element with the group's largest magnitude always lands on +-448
    mag = (q.reshape(7, 4, 128) & 0x7F)
    assert np.all(mag.max(axis=2) == 0x7E)
    # amax = 2 gives s = fl32(2/448); amax = 448 gives s = 1
    g = np.zeros((2, 128), np.float32)
    g[0, 5] = -2.0
    g[1, 17] = 448.0
    _, s2 = impl.quant_act_group128(g)
    assert s2[0, 0] == np.float32(2.0) / np.float32(448.0)
    assert s2[1, 0] == np.float32(1.0)


def test_round_trip_exact_for_power_of_two_scales(impl):
    rng = np.random.default_rng(5)
    vals = impl.e4m3_decode(np.arange(256, dtype=np.uint8))
    vals = vals[np.isfinite(vals)]
    for p in (-20, -3, 0, 2):
        codes_v = rng.choice(vals, size=(3, 256))
        codes_v[:, 0] = 448.0            # amax = 448 * 2^p, so s = 2^p exactly
        codes_v[:, 128] = -448.0
        x = (codes_v * 2.0 ** p).astype(np.float32)
        q, s = impl.quant_act_group128(x)
        assert np.all(s == np.float32(2.0 ** p))
        np.testing.assert_array_equal(impl.e4m3_decode(q) * 2.0 ** p, x.astype(np.float64))


def test_quantization_error_within_half_ulp(impl):
    x = synth.activations("deepseek", 16, 1024, seed=9).float().numpy()
    q, s = impl.quant_act_group128(x)
    deq = impl.e4m3_decode(q) * np.repeat(s.astype(np.float64), 128, axis=1)
    r = np.abs(x.astype(np.float64) / np.repeat(s.astype(np.float64), 128, axis=1))
    _, ex = np.frexp(np.maximum(r, 2.0 ** -6))
    half_ulp = np.ldexp(1.0, ex - 1 - 3) / 2       # half the E4M3 spacing at x/s
    # one extra fp32 rounding of x/s (relative 2^-24) is allowed on top
    tol = (half_ulp + r * 2.0 ** -23) * np.repeat(s.astype(np.float64), 128, axis=1)
    assert np.all(np.abs(deq - x) <= tol)


def test_zero_and_tiny_groups(impl):
    x = np.zeros((3, 128), np.float32)
    x[0, ::2] = -0.0
    x[1, 3] = 2.0 ** -133          # the smallest bf16 subnormal
    x[2, 0] = -2.0 ** -126
    x[2, 1] = 2.0 ** -127
    q, s = impl.quant_act_group128(x)
    assert s[0, 0] == 0 and np.all(q[0, ::2] == 0x80) and np.all(q[0, 1::2] == 0x00)
    assert s[1, 0] > 0                 # a subnormal fp32 scale, never 0 for amax > 0
    assert q[1, 3] == 0x7E             # amax / s saturates or lands on 448
    assert q[2, 0] == 0xFE


def test_weight_blocks_ragged_rows_and_worked_scales(impl):
    # rows 0..127: block amax 0.875 -> s = 0.875/448 = 2^-9 ; rows 128..129: 3.5 -> 2^-7
    w = np.zeros((130, 256), np.float32)
    w[5, 7] = -0.875
    w[100, 3] = 0.4375           # / 2^-9 = 224 -> 0x76
    w[128, 0] = 3.5
    w[129, 1] = 0.02734375       # / 2^-7 = 3.5 -> 0x46
    w[3, 200] = 1.0              # second K-block of the first row-block: s = 1/448
    qw, sw = impl.quant_weight_block128(w)
    assert sw.shape == (2, 2)
    assert sw[0, 0] == np.float32(2.0 ** -9) and sw[1, 0] == np.float32(2.0 ** -7)
    assert sw[1, 1] == 0 and sw[0, 1] == np.float32(1.0) / np.float32(448)
    assert qw[5, 7] == 0xFE and qw[100, 3] == 0x76 and qw[128, 0] == 0x7E and qw[129, 1] == 0x46
    assert qw[3, 200] == 0x7E


def test_weight_quant_equals_groupwise_rule_on_each_block(impl):
    """Each 128x128 block quantized alone with its own amax gives the same
    bytes as the whole-matrix call (blocks do not interact)."""
    w = synth.weights("deepseek", 300, 384, seed=2).float().numpy()
    qw, sw = impl.quant_weight_block128(w)
    for nb in range(3):
        for kb in range(3):
            blk = w[nb * 128:(nb + 1) * 128, kb * 128:(kb + 1) * 128]
            flat = blk.reshape(1, -1)
            s = np.float32(np.abs(flat).max()) / np.float32(448)
            assert sw[nb, kb] == s
            q_blk = impl.e4m3_encode((blk / s).astype(np.float32))
            np.testing.assert_array_equal(qw[nb * 128:(nb + 1) * 128, kb * 128:(kb + 1) * 128], q_blk)

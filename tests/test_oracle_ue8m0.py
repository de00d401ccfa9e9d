"""Pins of the oracle's UE8M0 scale variant ("FP8 à granularité fine",
section "Format d'échelle UE8M0": scales stored as float8_e8m0fnu, a bare
power of two). Hand-worked scale codes, the format's decode, and invariants
that follow from "the smallest power of two s with 448 * s >= amax". Every
pin runs against both statements of the oracle (C++ and numpy)."""

import numpy as np
import torch

from fp8_block_scaled_group128_b200 import synth


def _num(s):
    return float.fromhex(s) if s.lower().startswith(("0x", "-0x")) else float(s)


def test_scale_code_landmarks(impl, golden):
    rows = [r for r in golden("ue8m0_landmarks.txt") if r[0] == "amax"]
    assert len(rows) >= 15
    amax = np.array([_num(r[1]) for r in rows], np.float32)
    assert np.all(amax.astype(np.float64) == [_num(r[1]) for r in rows]), "fixture must be fp32-exact"
    codes = impl.ue8m0_of_amax(amax)
    np.testing.assert_array_equal(codes, [int(r[3]) for r in rows])
    np.testing.assert_array_equal(codes.astype(int) - 127, [max(int(r[2]), -127) for r in rows])


def test_decode_is_two_to_the_code_minus_127(impl):
    codes = np.arange(255, dtype=np.uint8)
    v = impl.ue8m0_decode(codes)
    want = np.array([2.0 ** (c - 127) for c in range(255)], np.float64)
    np.testing.assert_array_equal(v.astype(np.float64), want)
    assert np.isnan(impl.ue8m0_decode(np.array([255], np.uint8))[0])


def test_scale_is_the_smallest_power_of_two_without_saturation(impl):
    rng = np.random.default_rng(0)
    amax = (np.exp2(rng.uniform(-100, 100, 20000)) * rng.uniform(1, 2, 20000)).astype(np.float32)
    s = impl.ue8m0_decode(impl.ue8m0_of_amax(amax)).astype(np.float64)
    a = amax.astype(np.float64)
    assert np.all(448.0 * s >= a)            # nothing saturates
    assert np.all(448.0 * s / 2 < a)         # and half of it would not do


def test_activation_groups(impl):
    x = synth.activations("deepseek", 9, 640, seed=4).float().numpy()
    x[2, :128] = 0.0
    x[3, 128:256] = -0.0
    q, s8 = impl.quant_act_group128_ue8m0(x)
    amax = np.abs(x.reshape(9, 5, 128)).max(axis=2)
    np.testing.assert_array_equal(s8, impl.ue8m0_of_amax(amax))
    s = impl.ue8m0_decode(s8)
    # codes are e4m3 of x / s (division by a power of two: exact here)
    want = impl.e4m3_encode((x.reshape(9, 5, 128) / s[:, :, None]).astype(np.float32))
    np.testing.assert_array_equal(q.reshape(9, 5, 128), want)
    # the largest element of every nonzero group lands in (224, 448], i.e.
    # on a code of magnitude 0x76..0x7E; zero groups encode signed zeros
    mag = (q.reshape(9, 5, 128) & 0x7F).max(axis=2)
    nz = amax > 0
    assert np.all((mag[nz] >= 0x76) & (mag[nz] <= 0x7E))
    assert s8[2, 0] == 0 and np.all(q[2, :128] == 0x00) and np.all(q[3, 128:256] == 0x80)


def test_power_of_two_round_trip_is_exact(impl):
    rng = np.random.default_rng(1)
    vals = impl.e4m3_decode(np.arange(256, dtype=np.uint8))
    vals = vals[np.isfinite(vals)]
    for p in (-30, -2, 0, 5):
        v = rng.choice(vals, size=(2, 256))
        v[:, 0] = 448.0                       # amax = 448 * 2^p: s = 2^p exactly
        v[:, 128] = -448.0
        x = (v * 2.0 ** p).astype(np.float32)
        q, s8 = impl.quant_act_group128_ue8m0(x)
        assert np.all(s8 == 127 + p)
        np.testing.assert_array_equal(impl.e4m3_decode(q) * 2.0 ** p, x.astype(np.float64))


def test_weight_blocks_ragged_rows(impl):
    w = np.zeros((130, 256), np.float32)
    w[5, 7] = -0.875                          # block (0, 0): amax 0.875 -> 2^-9 (code 118)
    w[100, 3] = 0.4375                        # / 2^-9 = 224 -> 0x76
    w[128, 0] = 3.0                           # block (1, 0): 3 -> 2^-7 (code 120); 3 / 2^-7 = 384
    w[3, 200] = 1.0                           # block (0, 1): 1 -> 2^-8 (code 119); 256 -> 0x78
    qw, s8 = impl.quant_weight_block128_ue8m0(w)
    np.testing.assert_array_equal(s8, [[118, 119], [120, 0]])
    assert qw[5, 7] == 0xFE and qw[100, 3] == 0x76 and qw[128, 0] == 0x7C and qw[3, 200] == 0x78
    # the same block rule as the fp32-scale quantizer, with the scale replaced
    wt = synth.weights("deepseek", 300, 384, seed=2)
    q1, c1 = impl.quant_weight_block128_ue8m0(wt)
    wf = wt.float().numpy()
    for nb in range(3):
        for kb in range(3):
            blk = wf[nb * 128:(nb + 1) * 128, kb * 128:(kb + 1) * 128]
            assert c1[nb, kb] == impl.ue8m0_of_amax(np.float32(np.abs(blk).max()))
            s = impl.ue8m0_decode(c1[nb, kb])
            np.testing.assert_array_equal(q1[nb * 128:(nb + 1) * 128, kb * 128:(kb + 1) * 128],
                                          impl.e4m3_encode((blk / s).astype(np.float32)))


def test_gemm_with_power_of_two_scales_by_hand(impl):
    # K = 256: y = 2^(ca-127) * 2^(cw-127) * partial per K-block, summed
    qa = np.zeros((1, 256), np.uint8)
    qa[0, :128] = 0x38                       # 1.0
    qa[0, 128:] = 0xC0                       # -2.0
    qw = np.full((2, 256), 0x30, np.uint8)   # 0.5
    sa8 = np.array([[127 + 1, 127 - 3]], np.uint8)      # 2, 1/8
    sw8 = np.array([[127 + 4, 127]], np.uint8)          # 16, 1
    y = impl.block_gemm_ue8m0(qa, sa8, qw, sw8)
    # 2*16*(128*0.5) + (1/8)*1*(128*-2*0.5) = 2048 - 16 = 2032
    np.testing.assert_array_equal(y, [[2032.0, 2032.0]])
    np.testing.assert_array_equal(impl.gemm_error_bound_ue8m0(qa, sa8, qw, sw8, rel=1.0),
                                  [[2064.0, 2064.0]])


def test_ue8m0_error_is_at_most_twice_the_fp32_scale_error_bound():
    """The power-of-two scale loses at most one bit of the E4M3 range: the
    quantization error of each element is at most half an E4M3 ulp of x / s
    times s, with s < 2 * amax / 448."""
    import oracle
    x = synth.activations("llama", 16, 1024, seed=9).float().numpy()
    q, s8 = oracle.quant_act_group128_ue8m0(x)
    s = np.repeat(oracle.ue8m0_decode(s8).astype(np.float64), 128, axis=1)
    deq = oracle.e4m3_decode(q) * s
    r = np.abs(x.astype(np.float64) / s)
    _, ex = np.frexp(np.maximum(r, 2.0 ** -6))
    half_ulp = np.ldexp(1.0, ex - 1 - 3) / 2
    assert np.all(np.abs(deq - x) <= half_ulp * s)
    assert torch.is_tensor(torch.zeros(1))

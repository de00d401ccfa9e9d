"""Helpers shared by the GPU parity tests (no oracle arithmetic here)."""

import json
import os

import numpy as np
import pytest
import torch

import oracle


def require_gpu():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    major, minor = torch.cuda.get_device_capability()
    if (major, minor) != (10, 0):
        pytest.skip(f"needs sm_100 (B200), found sm_{major}{minor}")
    from fp8_block_scaled_group128_b200.build import build
    build()


def to_dev(a, dtype=None):
    t = a if isinstance(a, torch.Tensor) else torch.from_numpy(np.ascontiguousarray(a))
    if dtype is not None:
        t = t.to(dtype)
    return t.contiguous().cuda()


def _dequant_abs(q, s_rows):
    """|E4M3 value| x its scale, float64, with torch's own float8_e4m3fn decode
    (a library routine, independent of the oracle); s_rows [rows, K/128]."""
    v = torch.from_numpy(np.ascontiguousarray(q)).view(torch.float8_e4m3fn).to(torch.float64).abs()
    return v * torch.from_numpy(np.abs(np.asarray(s_rows, np.float64))).repeat_interleave(128, 1)


def independent_abs_sum(qa, sa, qw, sw, cols=None):
    """sum_k |a_k w_k| per output, computed here with one float64 matmul of
    the dequantized magnitudes (weight row n uses scale row n // 128)."""
    n = np.arange(qw.shape[0]) if cols is None else np.asarray(cols, np.int64)
    a = _dequant_abs(qa, sa)
    w = _dequant_abs(np.asarray(qw)[n], np.asarray(sw)[n // 128])
    return (a @ w.T).numpy()


def check_gemm(y_gpu, y_ref, operands, label="", cols=None):
    """The GEMM parity bar: |y - y_ref| <= 1e-2 * sum_k |a_k w_k| + 1 bf16 ulp
    of the reference, on every compared output. `operands` = (qa, sa, qw, sw)
    of the compared rows (qw, sw for all weight rows; `cols` picks the
    compared ones). The oracle's bound is checked against sum |a w| computed
    independently here. Returns summary statistics."""
    bound = oracle.gemm_error_bound(*operands, cols=cols)
    abs_sum = independent_abs_sum(*operands, cols=cols)
    np.testing.assert_allclose(bound, 1e-2 * abs_sum, rtol=1e-9, atol=0.0)
    y = y_gpu.float().cpu().numpy().astype(np.float64)
    err = np.abs(y - y_ref)
    tol = bound + oracle.bf16_ulp(y_ref)
    bad = err > tol
    if bad.any():
        i = np.argwhere(bad)[0]
        raise AssertionError(
            f"{label}: {bad.sum()} of {bad.size} outputs outside the bound; first at {tuple(i)}: "
            f"gpu={y[tuple(i)]!r} ref={y_ref[tuple(i)]!r} tol={tol[tuple(i)]!r}")
    # error beyond the final bf16 rounding, relative to sum_k |a_k w_k|
    excess = np.maximum(err - 0.5 * oracle.bf16_ulp(y_ref), 0.0)
    rel = excess / np.maximum(abs_sum, 1e-300)
    y_rn = torch.from_numpy(y_ref).to(torch.bfloat16).double().numpy()
    stats = {"label": label, "n": int(y.size),
             "max_err_over_sum": float(rel.max(initial=0.0)),
             "frac_equal_rn": float((y == y_rn).mean()) if y.size else 1.0}
    log = os.environ.get("FP8BS_PARITY_LOG")
    if log:
        with open(log, "a") as f:
            f.write(json.dumps(stats) + "\n")
    return stats

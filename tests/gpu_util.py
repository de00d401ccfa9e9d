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


def check_gemm(y_gpu, y_ref, bound, label=""):
    """The GEMM parity bar: |y - y_ref| <= 1e-2 * sum_k |a_k w_k| + 1 bf16 ulp
    of the reference, on every compared output. Returns summary statistics."""
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
    rel = excess / np.maximum(bound / 1e-2, 1e-300)
    y_rn = torch.from_numpy(y_ref).to(torch.bfloat16).double().numpy()
    stats = {"label": label, "n": int(y.size),
             "max_err_over_sum": float(rel.max(initial=0.0)),
             "frac_equal_rn": float((y == y_rn).mean()) if y.size else 1.0}
    log = os.environ.get("FP8BS_PARITY_LOG")
    if log:
        with open(log, "a") as f:
            f.write(json.dumps(stats) + "\n")
    return stats

"""The quantizers' scale division (Markstein's FMA correction on a once-per-
scale reciprocal) against CUDA's IEEE division __fdiv_rn, bit for bit, over
every bf16 amax and every bf16 x with |x| <= amax."""

import ctypes
import os
import subprocess

import pytest

from gpu_util import require_gpu

pytestmark = pytest.mark.gpu

HERE = os.path.dirname(os.path.abspath(__file__))


def test_scale_division_matches_ieee_exhaustively(tmp_path):
    require_gpu()
    from fp8_block_scaled_group128_b200.build import ARCH, nvcc
    so = tmp_path / "div_check.so"
    subprocess.run([nvcc()] + ARCH + ["-O3", "-std=c++17", "-shared", "-Xcompiler", "-fPIC",
                    "-I", os.path.join(os.path.dirname(HERE), "include"),
                    os.path.join(HERE, "cuda", "div_check.cu"), "-o", str(so)], check=True)
    lib = ctypes.CDLL(str(so))
    out = (ctypes.c_ulonglong * 5)()
    assert lib.div_check(out) == 0
    checked, bad_q, bad_c, amax_bits, x_bits = list(out)
    assert checked > 1_000_000_000
    assert (bad_q, bad_c) == (0, 0), (
        f"{bad_q} quotient and {bad_c} code mismatches of {checked}; "
        f"first at amax=0x{amax_bits:04x} x=0x{x_bits & 0xFFFF:04x}")

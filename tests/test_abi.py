"""Host-side checks of the C ABI: the library loads, exports every symbol the
header declares, and rejects bad arguments before touching a GPU."""

import ctypes
import os
import re

import pytest

from fp8_block_scaled_group128_b200 import binding
from fp8_block_scaled_group128_b200.build import build

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "fp8bs.h")


@pytest.fixture(scope="module")
def lib():
    build()
    return binding.lib()


def _declared_functions():
    text = open(HEADER).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    names = re.findall(r"^\s*(?:const\s+)?[A-Za-z_][\w\s\*]*?\b([a-z_][a-z0-9_]*)\s*\(", text, flags=re.M)
    return sorted(set(n for n in names if n not in ("if", "defined")))


def test_header_declares_the_five_operations():
    names = _declared_functions()
    for n in ("fp8_quant_act_group128", "fp8_quant_weight_block128", "fp8_block_gemm",
              "prune24_compress", "fp8_sparse24_gemm"):
        assert n in names


def test_library_exports_every_declared_symbol(lib):
    for n in _declared_functions():
        assert hasattr(lib, n), n
    assert set(_declared_functions()) <= set(binding.SIGNATURES)


def test_status_strings_and_version(lib):
    assert lib.fp8bs_status_string(0) == b"ok"
    assert b"128" in lib.fp8bs_status_string(2)
    assert lib.fp8bs_version() >= 100


def test_workspace_query_has_no_device_dependency(lib):
    assert lib.fp8bs_gemm_workspace_bytes(1, 4096, 4096, 0) == 0


BAD = ctypes.c_void_p(0x1000)
MIS = ctypes.c_void_p(0x1004)    # 4-byte aligned only
MIS2 = ctypes.c_void_p(0x1002)   # 2-byte aligned


@pytest.mark.parametrize("K", [0, 100, 129, -128])
def test_shape_errors_before_any_launch(lib, K):
    assert lib.fp8_quant_act_group128(BAD, 4, K, BAD, BAD, None) == 2
    assert lib.fp8_quant_weight_block128(BAD, 4, K, BAD, BAD, None) == 2
    assert lib.prune24_compress(BAD, 4, K, BAD, BAD, BAD, None, None) == 2
    assert lib.fp8_block_gemm(BAD, BAD, BAD, BAD, BAD, 4, 8, K, None, 0, None) == 2
    assert lib.fp8_sparse24_gemm(BAD, BAD, BAD, BAD, BAD, BAD, 4, 8, K, None, 0, None) == 2


def test_negative_sizes_and_gemm_n_alignment(lib):
    assert lib.fp8_quant_act_group128(BAD, -1, 128, BAD, BAD, None) == 2
    assert lib.fp8_block_gemm(BAD, BAD, BAD, BAD, BAD, 4, 12, 128, None, 0, None) == 2
    assert lib.fp8_block_gemm(BAD, BAD, BAD, BAD, BAD, -4, 16, 128, None, 0, None) == 2


def test_empty_problems_are_noops(lib):
    assert lib.fp8_quant_act_group128(None, 0, 128, None, None, None) == 0
    assert lib.fp8_quant_weight_block128(None, 0, 128, None, None, None) == 0
    assert lib.prune24_compress(None, 0, 128, None, None, None, None, None) == 0
    assert lib.fp8_block_gemm(None, None, None, None, None, 0, 16, 128, None, 0, None) == 0
    assert lib.fp8_block_gemm(None, None, None, None, None, 5, 0, 128, None, 0, None) == 0


def test_null_and_misaligned_pointers(lib):
    assert lib.fp8_quant_act_group128(None, 4, 128, BAD, BAD, None) == 1
    assert lib.fp8_quant_act_group128(MIS, 4, 128, BAD, BAD, None) == 3
    assert lib.fp8_block_gemm(BAD, BAD, BAD, None, BAD, 4, 8, 128, None, 0, None) == 1
    assert lib.fp8_block_gemm(BAD, BAD, MIS, BAD, BAD, 4, 8, 128, None, 0, None) == 3
    assert lib.prune24_compress(BAD, 4, 128, BAD, BAD, BAD, MIS, None) == 3


def test_fused_quantization_argument_checks(lib):
    """fp8_block_gemm_quant: whole 1x128 groups of y (N % 128), the codes and
    scales are required, and y is required when M <= 256 (that path quantizes
    the stored y); all checked before any launch."""
    g = lib.fp8_block_gemm_quant
    assert g(BAD, BAD, BAD, BAD, BAD, BAD, BAD, 4, 136, 128, None, 0, None) == 2
    assert g(BAD, BAD, BAD, BAD, BAD, BAD, BAD, 4, 128, 100, None, 0, None) == 2
    assert g(BAD, BAD, BAD, BAD, BAD, None, BAD, 4, 128, 128, None, 0, None) == 1
    assert g(BAD, BAD, BAD, BAD, BAD, BAD, None, 4, 128, 128, None, 0, None) == 1
    assert g(BAD, BAD, BAD, BAD, None, BAD, BAD, 256, 128, 128, None, 0, None) == 1
    assert g(BAD, BAD, BAD, BAD, BAD, MIS, BAD, 4, 128, 128, None, 0, None) == 3
    assert g(None, None, None, None, None, None, None, 0, 128, 128, None, 0, None) == 0


def test_grouped_and_ue8m0_argument_checks(lib):
    """The grouped GEMMs need E >= 1 and m_indices; the UE8M0 entry points
    follow the same shape, pointer and alignment rules; all before any launch."""
    for g in (lib.fp8_grouped_gemm, lib.fp8_grouped_gemm_ue8m0):
        assert g(BAD, BAD, BAD, BAD, BAD, BAD, 4, 8, 128, 0, None, 0, None) == 2     # E = 0
        assert g(BAD, BAD, BAD, BAD, None, BAD, 4, 8, 128, 2, None, 0, None) == 1    # m_indices
        assert g(BAD, BAD, BAD, BAD, BAD, BAD, 4, 12, 128, 2, None, 0, None) == 2    # N % 8
        assert g(BAD, BAD, BAD, BAD, MIS2, BAD, 4, 8, 128, 2, None, 0, None) == 3    # alignment
        assert g(BAD, MIS, BAD, MIS, MIS, BAD, 4, 8, 128, 2, None, 0, None) != 3     # 4 B is enough
        assert g(None, None, None, None, None, None, 0, 8, 128, 2, None, 0, None) == 0
    assert lib.fp8_block_gemm_ue8m0(BAD, BAD, BAD, BAD, BAD, 4, 8, 100, None, 0, None) == 2
    assert lib.fp8_block_gemm_ue8m0(BAD, None, BAD, BAD, BAD, 4, 8, 128, None, 0, None) == 1
    assert lib.fp8_quant_act_group128_ue8m0(BAD, 4, 129, BAD, BAD, None) == 2
    assert lib.fp8_quant_weight_block128_ue8m0(MIS, 4, 128, BAD, BAD, None) == 3
    # UE8M0 code arrays are bytes: no alignment rule (a 2-byte offset is not an error)
    assert lib.fp8_block_gemm_ue8m0(BAD, BAD, BAD, None, BAD, 4, 8, 128, None, 0, None) == 1
    assert lib.fp8_quant_act_group128_ue8m0(None, 0, 128, None, None, None) == 0


def test_swiglu_argument_checks(lib):
    """I must be a positive multiple of 128; codes and scales are required; h
    is optional; M == 0 or I == 0 is a no-op."""
    f = lib.fp8_gemm_swiglu_quant
    assert f(BAD, BAD, BAD, BAD, BAD, BAD, BAD, 4, 136, 128, None, 0, None) == 2
    assert f(BAD, BAD, BAD, BAD, BAD, BAD, BAD, 4, 128, 100, None, 0, None) == 2
    assert f(BAD, BAD, BAD, BAD, BAD, None, BAD, 4, 128, 128, None, 0, None) == 1
    assert f(BAD, BAD, BAD, BAD, MIS, BAD, BAD, 4, 128, 128, None, 0, None) == 3
    assert f(None, None, None, None, None, None, None, 0, 128, 128, None, 0, None) == 0
    # decode-sized M needs a scratch y [M][2I] bf16
    assert lib.fp8bs_swiglu_workspace_bytes(8, 14336) == 8 * 2 * 14336 * 2
    assert lib.fp8bs_swiglu_workspace_bytes(257, 14336) == 0
    assert f(BAD, BAD, BAD, BAD, BAD, BAD, BAD, 8, 128, 128, None, 0, None) == 4
    assert f(BAD, BAD, BAD, BAD, BAD, BAD, BAD, 8, 128, 128, BAD, 4095, None) == 4


def test_gather_columns_argument_checks(lib):
    g = lib.fp8_gather_columns
    assert g(BAD, 0, 4, 8, BAD, None) == 2          # P >= 1
    assert g(BAD, 2, 4, 12, BAD, None) == 2         # Np % 8
    assert g(None, 2, 4, 8, BAD, None) == 1
    assert g(MIS, 2, 4, 8, BAD, None) == 3
    assert g(None, 2, 0, 8, None, None) == 0

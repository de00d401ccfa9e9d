"""Fine-grained (block-scaled, group-128) FP8 linear layer for NVIDIA B200.

The computation runs in libfp8bs.so (hand-written sm_100a CUDA kernels behind
a C ABI, include/fp8bs.h); this package is its thin Python binding plus the
seeded synthetic input generators.
"""

from .binding import (  # noqa: F401
    Fp8bsError,
    fp8_block_gemm,
    fp8_block_gemm_quant,
    fp8_block_gemm_ue8m0,
    fp8_gather_columns,
    fp8_gemm_swiglu_quant,
    fp8_gemm_swiglu_quant_noalloc,
    fp8_grouped_gemm,
    fp8_grouped_gemm_ue8m0,
    fp8_linear,
    fp8_quant_act_group128_ue8m0,
    fp8_quant_weight_block128_ue8m0,
    fp8_quant_act_group128,
    fp8_quant_weight_block128,
    fp8_sparse24_gemm,
    gemm_workspace_bytes,
    get_device_error,
    lib,
    prune24_compress,
    set_wait_limit,
)

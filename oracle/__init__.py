"""CPU oracle for the fine-grained (block-scaled, group-128) FP8 linear layer.

TEST INFRASTRUCTURE ONLY. Only the tests, ``__graft_entry__.smoke()`` and the
``cpu_baseline`` leg / reference arm of ``bench.py`` may import this package;
the library in ``fp8_block_scaled_group128_b200`` never does, and shares no
code with it.

Two statements of the same definitions, written separately:

* ``fp8_oracle.cpp`` (plain C++17, double precision for the GEMM, fp32 where
  the method fixes fp32: the scale and the element division; threaded over
  independent outputs), reached through ``fp8_oracle_cpp`` -- the oracle the
  GPU parity tests and the CPU baseline use, exported at package level;
* ``fp8_oracle`` (numpy) -- the same arithmetic written a second time; the
  CPU tests check both against the same pins and against each other.
"""

from . import fp8_oracle as numpy_oracle  # noqa: F401
from . import fp8_oracle_cpp as cpp_oracle  # noqa: F401
from .fp8_oracle_cpp import (  # noqa: F401
    E4M3_MAX,
    GROUP,
    bf16_ulp,
    block_gemm,
    block_gemm_ue8m0,
    decompress24,
    e4m3_decode,
    e4m3_encode,
    gemm_abs_sum,
    gemm_error_bound,
    gemm_error_bound_ue8m0,
    gemm_swiglu,
    grouped_gemm,
    grouped_gemm_ue8m0,
    prune24_compress,
    quant_act_group128,
    quant_act_group128_ue8m0,
    quant_weight_block128,
    quant_weight_block128_ue8m0,
    set_threads,
    sparse24_gemm,
    swiglu,
    swiglu_error_bound,
    threads,
    ue8m0_decode,
    ue8m0_of_amax,
)

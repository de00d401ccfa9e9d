"""CPU oracle for the fine-grained (block-scaled, group-128) FP8 linear layer.

TEST INFRASTRUCTURE ONLY. Only the tests, ``__graft_entry__.smoke()`` and the
``cpu_baseline`` leg of ``bench.py`` may import this package; the library in
``fp8_block_scaled_group128_b200`` never does, and shares no code with it.

Everything is plain numpy, with floating point in fp64 except where the method
fixes fp32 (the scale and the element division, see ``fp8_oracle``).
"""

from .fp8_oracle import (  # noqa: F401
    E4M3_MAX,
    GROUP,
    e4m3_encode,
    e4m3_decode,
    quant_act_group128,
    quant_weight_block128,
    prune24_compress,
    decompress24,
    block_gemm,
    sparse24_gemm,
    gemm_error_bound,
    bf16_ulp,
)

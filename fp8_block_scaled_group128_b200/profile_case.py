"""Run one step of the path on one shape, a few times, for a profiler.

    python -m fp8_block_scaled_group128_b200.profile_case KIND M N K ITERS

KIND is one of quant_act, quant_weight, prune24, dense_gemm, sparse_gemm,
ue8m0_gemm, swiglu (N = 2I: the gate+up GEMM with SwiGLU and the next layer's
quantization, codes only), grouped_gemm and grouped_ue8m0 (M routed token
rows over 8 experts with the seeded uneven layout, each expert's rows padded
to 128; N, K per expert).
The inputs are the seeded synthetic llama tensors of that shape (deepseek for
the grouped kinds), prepared on the device by the library's own kernels before
the ITERS launches of the kernel under test (select those with the profiler's
kernel-name filter). Prints the mean device time of the ITERS launches (CUDA
events). One kernel and one shape per run, so that a profiler capture stays
small.
"""

import sys

import torch

from . import binding as fb
from . import synth


def main(argv):
    kind, M, N, K, iters = argv[0], int(argv[1]), int(argv[2]), int(argv[3]), int(argv[4])
    dev = torch.device("cuda", 0)
    torch.cuda.set_device(dev)
    if kind in ("quant_weight", "prune24", "dense_gemm", "sparse_gemm", "ue8m0_gemm", "swiglu"):
        w = synth.weights("llama", N, K, seed=0).to(dev)
    if kind in ("quant_act", "dense_gemm", "sparse_gemm", "ue8m0_gemm", "swiglu"):
        x = synth.activations("llama", max(M, 1), K, seed=0).to(dev)

    if kind == "quant_act":
        qa = torch.empty(M, K, dtype=torch.uint8, device=dev)
        sa = torch.empty(M, K // 128, dtype=torch.float32, device=dev)
        fn = lambda: fb.fp8_quant_act_group128(x, qa=qa, sa=sa)  # noqa: E731
    elif kind == "quant_weight":
        qw = torch.empty(N, K, dtype=torch.uint8, device=dev)
        sw = torch.empty(-(-N // 128), K // 128, dtype=torch.float32, device=dev)
        fn = lambda: fb.fp8_quant_weight_block128(w, qw=qw, sw=sw)  # noqa: E731
    elif kind == "prune24":
        vals = torch.empty(N, K // 2, dtype=torch.uint8, device=dev)
        meta = torch.empty(N, K // 8, dtype=torch.uint8, device=dev)
        sw = torch.empty(-(-N // 128), K // 128, dtype=torch.float32, device=dev)
        fn = lambda: fb.prune24_compress(w, vals=vals, meta=meta, sw=sw)  # noqa: E731
    elif kind in ("dense_gemm", "sparse_gemm"):
        qa, sa = fb.fp8_quant_act_group128(x)
        y = torch.empty(M, N, dtype=torch.bfloat16, device=dev)
        if kind == "dense_gemm":
            qw, sw = fb.fp8_quant_weight_block128(w)
            fn = lambda: fb.fp8_block_gemm(qa, sa, qw, sw, y=y)  # noqa: E731
        else:
            vals, meta, sw, _ = fb.prune24_compress(w)
            fn = lambda: fb.fp8_sparse24_gemm(qa, sa, vals, meta, sw, y=y)  # noqa: E731
        del w
    elif kind == "swiglu":
        qa, sa = fb.fp8_quant_act_group128(x)
        qw, sw = fb.fp8_quant_weight_block128(w)
        qh = torch.empty(M, N // 2, dtype=torch.uint8, device=dev)
        sh = torch.empty(M, N // 256, dtype=torch.float32, device=dev)
        need = fb.lib().fp8bs_swiglu_workspace_bytes(M, N // 2)
        ws = torch.empty(max(need, 16), dtype=torch.uint8, device=dev)
        fn = lambda: fb.fp8_gemm_swiglu_quant(qa, sa, qw, sw, qh=qh, sh=sh, want_h=False,  # noqa: E731
                                              workspace=ws)
        del w
    elif kind == "ue8m0_gemm":
        qa, sa = fb.fp8_quant_act_group128_ue8m0(x)
        qw, sw = fb.fp8_quant_weight_block128_ue8m0(w)
        y = torch.empty(M, N, dtype=torch.bfloat16, device=dev)
        fn = lambda: fb.fp8_block_gemm_ue8m0(qa, sa, qw, sw, y=y)  # noqa: E731
        del w
    elif kind in ("grouped_gemm", "grouped_ue8m0"):
        E = synth.MOE_EXPERTS
        mi, _ = synth.moe_layout(E, M, seed=3)
        Mp = mi.numel()
        x = synth.activations("deepseek", Mp, K, seed=3).to(dev)
        w = synth.expert_weights("deepseek", E, N, K, seed=3).to(dev)
        mid = mi.to(dev)
        qw = torch.empty(E, N, K, dtype=torch.uint8, device=dev)
        NB, KB = -(-N // 128), K // 128
        if kind == "grouped_gemm":
            qa, sa = fb.fp8_quant_act_group128(x)
            sw = torch.empty(E, NB, KB, dtype=torch.float32, device=dev)
            for e in range(E):
                fb.fp8_quant_weight_block128(w[e], qw=qw[e], sw=sw[e])
            gemm = fb.fp8_grouped_gemm
        else:
            qa, sa = fb.fp8_quant_act_group128_ue8m0(x)
            sw = torch.empty(E, NB, KB, dtype=torch.uint8, device=dev)
            for e in range(E):
                fb.fp8_quant_weight_block128_ue8m0(w[e], qw=qw[e], sw8=sw[e])
            gemm = fb.fp8_grouped_gemm_ue8m0
        y = torch.empty(Mp, N, dtype=torch.bfloat16, device=dev)
        fn = lambda: gemm(qa, sa, qw, sw, mid, y=y)  # noqa: E731
        del w, x
    else:
        raise SystemExit(f"unknown kind {kind!r}")
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record()
    for _ in range(iters):
        fn()
    e1.record()
    torch.cuda.synchronize()
    if fb.get_device_error() != 0:
        raise SystemExit("device error")
    us = e0.elapsed_time(e1) / iters * 1e3
    gemm_kind = kind.endswith("gemm") or kind in ("swiglu", "grouped_ue8m0")
    extra = f", {2.0 * M * N * K / (us * 1e-6) / 1e12:.1f} TFLOP/s" if gemm_kind else ""
    print(f"{kind} M={M} N={N} K={K}: {us:.2f} us/launch over {iters} launches{extra}")


if __name__ == "__main__":
    main(sys.argv[1:])

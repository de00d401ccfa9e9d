#!/usr/bin/env python
"""Benchmark of the fine-grained FP8 linear-layer path on B200.

One pass of the path covers the decode-shaped Llama-3-8B linears ((N, K) =
QKV (6144, 4096), O (4096, 4096), gate+up (28672, 4096), down (4096, 14336);
tokens M in {1, 8, 32, 128}):

  1. weight quantization of the four bf16 weights (128x128 blocks)
  2. 2:4 prune + compress of the four weights
  3. for each M: the four activation quantizations (1x128 groups), the four
     dense block-scaled GEMMs, the four 2:4 sparse block-scaled GEMMs

The metric is HBM throughput (algorithmic bytes of every launch / device
time), with the dominant kernel's roofline fraction against the measured copy
bandwidth. Inputs are seeded synthetic bf16 tensors; the per-pass working set
(~2.7 GB) is far larger than L2 and every weight is re-read only after more
than L2's worth of other traffic. A pass is captured once as a CUDA graph and
replayed. A counted step is `passes` replays of that graph, with `passes`
chosen so that the timed region lasts at least about a second whatever
--steps says (the clock record and the per-kernel split then rest on many
samples); the last passes of the timed region use copies of the graph with an
event wherever the launch kind changes, for the live per-kernel split.

The same JSON line also carries a "prefill" section (the dense GEMM on the
prefill-shaped linears, M in {2048, 8192}, the four Llama-3-8B linears and the
LM head, with fp32 scales and with UE8M0 scales; the 2:4 GEMM at M = 4096; in
TFLOP/s against the dense FP8 tensor peak), a "quantize" section (the
quantizers at bandwidth-bound sizes, in GB/s against the copy bandwidth) and
an "accuracy" section (both scale formats against the exact product).

Usage:
  python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]
Multi-GPU (replicas, weak scaling; no collective on the data path):
  python -m torch.distributed.run --nnodes=1 --nproc-per-node N \\
      --master-addr 127.0.0.1 --master-port P bench.py --gpus N
"""

import argparse
import datetime
import hashlib
import json
import math
import os
import statistics
import subprocess
import sys
import tempfile
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

import torch  # noqa: E402

METRIC = "block-scaled FP8 GEMM TFLOP/s and decode GB/s, % of B200 roofline"
UNIT = "GB/s"
WORKLOAD = "decode-shaped Llama-3-8B linears, M in {1,8,32,128}"
LINEARS = ((6144, 4096), (4096, 4096), (28672, 4096), (4096, 14336))
TOKENS = (1, 8, 32, 128)
FALLBACK_HBM_GBS = 6650.0
L2_BYTES = 126 * 1024 * 1024
MIN_TIMED_S = 1.2          # the timed region lasts at least this long
KERNELS = ("quant_weight", "prune24", "quant_act", "dense_gemm", "sparse_gemm")
# Rows of the path the step runs.
ROWS = KERNELS
# The oracle's bounded sample of a pass: every weight row, and the token rows
# for these M only.
ORACLE_SAMPLE_M = (1, 8)


# ----------------------------------------------------------------- bytes --

def kernel_bytes(kind, M, N, K):
    """Algorithmic bytes of one launch: every input read once, every output
    written once (E4M3 = 1 B, bf16 = 2 B, scale = 4 B, metadata = K/8 B/row)."""
    KB, NB = K // 128, -(-N // 128)
    if kind == "quant_act":
        return 2 * M * K + M * K + 4 * M * KB
    if kind == "quant_weight":
        return 2 * N * K + N * K + 4 * NB * KB
    if kind == "prune24":
        return 2 * N * K + N * K // 2 + N * K // 8 + 4 * NB * KB
    if kind == "dense_gemm":
        return N * K + 4 * NB * KB + M * K + 4 * M * KB + 2 * M * N
    if kind == "sparse_gemm":
        return N * K // 2 + N * K // 8 + 4 * NB * KB + M * K + 4 * M * KB + 2 * M * N
    raise ValueError(kind)


def step_launches():
    """(kind, M, N, K) of every launch of one pass, in issue order: the weight
    rows, then per token count M the four activation quantizations, the four
    dense GEMMs and the four 2:4 GEMMs (same-kind launches back to back, so
    the live per-kernel split needs an event only where the kind changes)."""
    out = [("quant_weight", 0, N, K) for N, K in LINEARS]
    out += [("prune24", 0, N, K) for N, K in LINEARS]
    for M in TOKENS:
        for kind in ("quant_act", "dense_gemm", "sparse_gemm"):
            out += [(kind, M, N, K) for N, K in LINEARS]
    return [l for l in out if l[0] in ROWS]


def step_bytes():
    return sum(kernel_bytes(*l) for l in step_launches())


def oracle_sample_launches():
    """The launches of a pass the CPU oracle runs as its bounded sample."""
    return [l for l in step_launches()
            if l[0] in ("quant_weight", "prune24") or l[1] in ORACLE_SAMPLE_M]


def bench_config(world, passes):
    """The `config` object of the JSON line (the same for both arms)."""
    return {"workload": WORKLOAD, "rows": list(ROWS), "linears_NK": [list(l) for l in LINEARS],
            "tokens_M": list(TOKENS), "global_batch": sum(TOKENS) * passes * world,
            "passes_per_step": passes, "pass_bytes": step_bytes(),
            "launches_per_pass": len(step_launches()),
            "parallelism": f"replicas x{world} (token data parallel, no collective)",
            "l2": "working set per pass ~2.7 GB >> 126 MB L2; every weight is re-read only "
                  "after >126 MB of other traffic; CUDA-graph replay"}


# ------------------------------------------------------------ GPU step --

class Step:
    """Device buffers of one pass and the launches through the C ABI."""

    def __init__(self, device, seed=0):
        from fp8_block_scaled_group128_b200 import synth
        self.dev = device
        self.w = {}
        self.x = {}
        for N, K in LINEARS:
            self.w[(N, K)] = synth.weights("llama", N, K, seed=seed).to(device)
        # one activation per (M, linear), as the inputs of a layer's four
        # linears are four different tensors
        for M in TOKENS:
            for i, (N, K) in enumerate(LINEARS):
                self.x[(M, N, K)] = synth.activations("llama", M, K, seed=seed + 101 * i).to(device)
        e = lambda *s, dt: torch.empty(*s, dtype=dt, device=device)  # noqa: E731
        self.qw, self.sw, self.vals, self.meta, self.sws = {}, {}, {}, {}, {}
        for N, K in LINEARS:
            NB, KB = -(-N // 128), K // 128
            self.qw[(N, K)] = e(N, K, dt=torch.uint8)
            self.sw[(N, K)] = e(NB, KB, dt=torch.float32)
            self.vals[(N, K)] = e(N, K // 2, dt=torch.uint8)
            self.meta[(N, K)] = e(N, K // 8, dt=torch.uint8)
            self.sws[(N, K)] = e(NB, KB, dt=torch.float32)
        self.qa, self.sa, self.y, self.ys = {}, {}, {}, {}
        for M in TOKENS:
            for N, K in LINEARS:
                self.qa[(M, N, K)] = e(M, K, dt=torch.uint8)
                self.sa[(M, N, K)] = e(M, K // 128, dt=torch.float32)
                self.y[(M, N, K)] = e(M, N, dt=torch.bfloat16)
                self.ys[(M, N, K)] = e(M, N, dt=torch.bfloat16)

    def launches(self):
        """(kind, thunk) for every launch of one pass, in issue order."""
        from fp8_block_scaled_group128_b200 import binding as fb
        out = []
        for N, K in LINEARS:
            out.append(("quant_weight", lambda N=N, K=K: fb.fp8_quant_weight_block128(
                self.w[(N, K)], qw=self.qw[(N, K)], sw=self.sw[(N, K)])))
        for N, K in LINEARS:
            out.append(("prune24", lambda N=N, K=K: fb.prune24_compress(
                self.w[(N, K)], vals=self.vals[(N, K)], meta=self.meta[(N, K)],
                sw=self.sws[(N, K)])))
        for M in TOKENS:
            for N, K in LINEARS:
                out.append(("quant_act", lambda M=M, N=N, K=K: fb.fp8_quant_act_group128(
                    self.x[(M, N, K)], qa=self.qa[(M, N, K)], sa=self.sa[(M, N, K)])))
            for N, K in LINEARS:
                out.append(("dense_gemm", lambda M=M, N=N, K=K: fb.fp8_block_gemm(
                    self.qa[(M, N, K)], self.sa[(M, N, K)], self.qw[(N, K)], self.sw[(N, K)],
                    y=self.y[(M, N, K)])))
            for N, K in LINEARS:
                out.append(("sparse_gemm", lambda M=M, N=N, K=K: fb.fp8_sparse24_gemm(
                    self.qa[(M, N, K)], self.sa[(M, N, K)], self.vals[(N, K)],
                    self.meta[(N, K)], self.sws[(N, K)], y=self.ys[(M, N, K)])))
        return [(k, f) for k, f in out if k in ROWS]

    def run(self):
        """Issue one pass eagerly on the current stream."""
        for _, f in self.launches():
            f()

    def host_inputs(self):
        """Pinned host copies of the step's inputs (for the end-to-end run)."""
        return ({k: v.cpu().pin_memory() for k, v in self.w.items()},
                {k: v.cpu().pin_memory() for k, v in self.x.items()})


class ClockSampler:
    """nvidia-smi samples (every 200 ms) of SM clock and throttle reasons
    while the timed region runs."""

    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, index):
        self.index = index
        self.proc = None
        self.out = None
        self._own_file = None   # the temporary file this sampler created

    def __enter__(self):
        try:
            fd, path = tempfile.mkstemp(prefix="fp8bs_clocks_", suffix=".csv")
            self._own_file = path
            self.out = os.fdopen(fd, "w+")
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", str(self.index), "--query-gpu=" + self.FIELDS,
                 "--format=csv,noheader,nounits", "-lms", "200"],
                stdout=self.out, stderr=subprocess.DEVNULL)
        except (OSError, FileNotFoundError):
            self.proc = None
        time.sleep(0.3)
        return self

    def __exit__(self, *exc):
        if self.proc is not None:
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except subprocess.TimeoutExpired:
                self.proc.kill()

    def summary(self):
        if self.out is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"]}
        self.out.flush()
        self.out.seek(0)
        rows = [l.strip().split(", ") for l in self.out.read().splitlines() if l.strip()]
        self.out.close()
        if self._own_file is not None:
            try:
                os.remove(self._own_file)
            except OSError:
                pass
            self._own_file = None
        sm, mx, reasons = [], [], set()
        names = ("hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap")
        for r in rows:
            if len(r) < 9:
                continue
            try:
                sm.append(float(r[1]))
                mx.append(float(r[2]))
            except ValueError:
                continue
            for nm, v in zip(names, r[5:9]):
                if v.strip().lower() == "active":
                    reasons.add(nm)
        if not sm:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["no samples"]}
        loaded = [s for s in sm if s > 0.5 * max(sm)] or sm
        return {"sm_mhz": statistics.median(loaded), "sm_max_mhz": max(mx),
                "samples": len(sm), "reasons": sorted(reasons)}


# ------------------------------------------------------------- helpers --

def measured_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(p) as f:
            d = json.load(f)
        return float(d["hbm_gbs"]), "measured"
    except (OSError, KeyError, ValueError):
        return FALLBACK_HBM_GBS, "fallback"


def source_hash():
    """Hash of the CUDA sources, to tell whether recorded ncu traffic is stale."""
    h = hashlib.sha256()
    csrc = os.path.join(ROOT, "fp8_block_scaled_group128_b200", "csrc")
    for name in sorted(os.listdir(csrc)):
        with open(os.path.join(csrc, name), "rb") as f:
            h.update(name.encode() + f.read())
    return h.hexdigest()[:16]


def recorded_traffic(kind):
    """DRAM bytes / algorithmic bytes of `kind`, from the committed per-kernel
    ncu captures (one kernel, a few launches each), or None if absent or
    taken on different kernel sources."""
    p = os.path.join(ROOT, "profiles", "traffic.json")
    try:
        with open(p) as f:
            d = json.load(f)
    except (OSError, ValueError):
        return None
    if d.get("source_hash") != source_hash():
        return None
    v = d.get("kernels", {}).get(kind)
    try:
        return float(v["dram_bytes"]) / float(v["algorithmic_bytes"])
    except (TypeError, KeyError, ValueError, ZeroDivisionError):
        return None


def dist_info():
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    return rank, world, local


def max_over_ranks(value, world):
    """Max of a float over all ranks (identity for one process)."""
    if world == 1:
        return value
    import torch.distributed as dist
    t = torch.tensor([value], dtype=torch.float64,
                     device="cuda" if dist.get_backend() == "nccl" else "cpu")
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def barrier(world):
    if world > 1:
        import torch.distributed as dist
        dist.barrier()


def passes_per_step(steps, pass_ms, min_timed_s=MIN_TIMED_S):
    """Graph replays per counted step so that `steps` steps last at least
    `min_timed_s`."""
    return max(1, math.ceil(min_timed_s * 1e3 / (max(steps, 1) * max(pass_ms, 1e-3))))


def copies_beyond_l2(bytes_per_copy, cap=16):
    """Input copies to rotate over so that back-to-back launches never find
    their inputs in L2 (working set at least twice the L2 size)."""
    return max(1, min(cap, math.ceil(2 * L2_BYTES / max(bytes_per_copy, 1))))


# ------------------------------------------------- prefill and quantize --

def fp8_tensor_peak():
    """Dense FP8 tensor peak (TFLOP/s): the measured cuBLAS bf16 burst figure
    times 2, the nominal fp8 : bf16 dense ratio of B200 (4.5 : 2.25 PFLOP/s)."""
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(p) as f:
            return 2.0 * float(json.load(f)["bf16_tflops"]), "measured bf16 burst x 2"
    except (OSError, KeyError, ValueError):
        return 2.0 * 1590.0, "fallback bf16 1.59 PF/s x 2"


def _time_graph(fns, stream, world, reps):
    """Mean device time (ms) of one call, from a CUDA graph of `reps` calls
    that cycle through `fns` (one warm-up replay, three timed; CUDA events on
    the launching stream; max over ranks)."""
    from fp8_block_scaled_group128_b200 import binding as fb
    with torch.cuda.stream(stream):
        for f in fns:
            f()
    stream.synchronize()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g, stream=stream):
        for i in range(reps):
            fns[i % len(fns)]()
    with torch.cuda.stream(stream):
        g.replay()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    with torch.cuda.stream(stream):
        e0.record()
        for _ in range(3):
            g.replay()
        e1.record()
    stream.synchronize()
    assert fb.get_device_error(stream) == 0
    del g
    return max_over_ranks(e0.elapsed_time(e1) / (3 * reps), world)


def run_prefill(dev, stream, world, reps=12):
    """Prefill-shaped GEMMs timed on their own: the dense GEMM at M in {2048,
    8192} on the four Llama-3-8B linears and the LM head, with fp32 scales
    ("dense") and with UE8M0 scales ("ue8m0", the tensor cores' block
    scaling); the 2:4 GEMM at M = 4096 on its two shapes; and on the down
    projection at M = 8192 the GEMM with the next layer's 1x128 quantization
    fused into its epilogue ("fused", codes only) against the GEMM followed by
    the activation quantizer ("separate"). Each shape rotates over enough
    copies of its quantized inputs that back-to-back launches find none of
    them in L2. Inputs: the seeded synthetic llama tensors, quantized /
    compressed on the device before timing."""
    from fp8_block_scaled_group128_b200 import binding as fb
    from fp8_block_scaled_group128_b200 import synth
    peak, peak_src = fp8_tensor_peak()
    shapes = [(kind, M, N, K) for N, K in synth.LLAMA3_8B_LINEARS + (synth.LLAMA3_8B_LM_HEAD,)
              for M in synth.PREFILL_M for kind in ("dense", "ue8m0")]
    shapes += [("sparse", 4096, N, K) for N, K in synth.SPARSE_LINEARS]
    shapes += [(kind, 8192, 4096, 14336) for kind in ("fused", "separate")]
    # the gated MLP's gate+up GEMM with SwiGLU and the down projection's
    # quantization fused (codes only), at decode and prefill token counts; the
    # plain gate+up GEMM of the same shape is the dense row (or timed here)
    shapes += [(kind, M, 28672, 4096) for M in (8, 128) for kind in ("swiglu", "dense")]
    shapes += [("swiglu", M, 28672, 4096) for M in synth.PREFILL_M]
    shapes = [sh + ("llama",) for sh in shapes]
    # the DeepSeek-V3 linears (their own weight and activation statistics) at
    # M = 4096, both scale formats
    shapes += [(kind, 4096, N, K, "deepseek") for N, K in synth.DEEPSEEK_V3_LINEARS
               for kind in ("dense", "ue8m0")]
    rows = []
    tot = {g: [0.0, 0.0] for g in ("dense", "ue8m0", "ds_dense", "ds_ue8m0")}
    wcache = {}
    for kind, M, N, K, wl in shapes:
        with torch.cuda.stream(stream):
            key = (wl, N, K)
            if key not in wcache:
                wcache.clear()
                torch.cuda.empty_cache()
                wcache[key] = synth.weights(wl, N, K, seed=7).to(dev)
            w = wcache[key]
            if kind == "sparse":
                wq = list(fb.prune24_compress(w)[:3])
            elif kind == "ue8m0":
                wq = list(fb.fp8_quant_weight_block128_ue8m0(w))
            else:
                wq = list(fb.fp8_quant_weight_block128(w))
            x = synth.activations(wl, M, K, seed=7).to(dev)
            qa, sa = (fb.fp8_quant_act_group128_ue8m0(x) if kind == "ue8m0"
                      else fb.fp8_quant_act_group128(x))
            del x
            in_bytes = M * K + (N * K * 5 // 8 if kind == "sparse" else N * K)
            n_cp = copies_beyond_l2(in_bytes, cap=8)
            ins = [(qa.clone(), sa.clone(), [t.clone() for t in wq]) for _ in range(n_cp - 1)]
            ins.append((qa, sa, wq))
            y = torch.empty(M, N, dtype=torch.bfloat16, device=dev)
            qy = torch.empty(M, N, dtype=torch.uint8, device=dev)
            sy = torch.empty(M, N // 128, dtype=torch.float32, device=dev)
            qh_sw = torch.empty(M, N // 2, dtype=torch.uint8, device=dev)
            sh_sw = torch.empty(M, N // 256, dtype=torch.float32, device=dev)
        fns = []
        for a, s, wqq in ins:
            if kind == "dense":
                fns.append(lambda a=a, s=s, wqq=wqq: fb.fp8_block_gemm(a, s, wqq[0], wqq[1], y=y))
            elif kind == "ue8m0":
                fns.append(lambda a=a, s=s, wqq=wqq: fb.fp8_block_gemm_ue8m0(
                    a, s, wqq[0], wqq[1], y=y))
            elif kind == "sparse":
                fns.append(lambda a=a, s=s, wqq=wqq: fb.fp8_sparse24_gemm(
                    a, s, wqq[0], wqq[1], wqq[2], y=y))
            elif kind == "fused":
                fns.append(lambda a=a, s=s, wqq=wqq: fb.fp8_block_gemm_quant(
                    a, s, wqq[0], wqq[1], qy=qy, sy=sy, want_y=False))
            elif kind == "swiglu":
                fns.append(lambda a=a, s=s, wqq=wqq: fb.fp8_gemm_swiglu_quant(
                    a, s, wqq[0], wqq[1], qh=qh_sw, sh=sh_sw, want_h=False))
            else:
                fns.append(lambda a=a, s=s, wqq=wqq: (
                    fb.fp8_block_gemm(a, s, wqq[0], wqq[1], y=y),
                    fb.fp8_quant_act_group128(y, qa=qy, sa=sy)))
        ms = _time_graph(fns, stream, world, reps)
        # algorithmic FLOPs: 2MNK dense; MNK (the kept half) for 2:4
        flop = (1.0 if kind == "sparse" else 2.0) * M * N * K
        tf = flop / (ms * 1e-3) / 1e12
        rows.append({"gemm": kind, "workload": wl, "M": M, "N": N, "K": K,
                     "us": round(ms * 1e3, 1), "TFLOP/s": round(tf, 1), "frac": round(tf / peak, 4),
                     "input_copies": n_cp})
        group = kind if wl == "llama" else "ds_" + kind
        if group in tot and (wl != "llama" or M in synth.PREFILL_M):
            tot[group][0] += flop
            tot[group][1] += ms
        del fns, ins, qa, sa, wq, y, qy, sy, qh_sw, sh_sw
    wcache.clear()
    torch.cuda.empty_cache()
    rows += run_grouped(dev, stream, world, peak, reps)
    agg = {k: v[0] / (v[1] * 1e-3) / 1e12 for k, v in tot.items()}
    return {"bound": "tensor", "unit": "TFLOP/s", "peak": round(peak, 1), "peak_source": peak_src,
            "dense_achieved": round(agg["dense"], 1), "dense_frac": round(agg["dense"] / peak, 4),
            "ue8m0_achieved": round(agg["ue8m0"], 1), "ue8m0_frac": round(agg["ue8m0"] / peak, 4),
            "deepseek_dense_achieved": round(agg["ds_dense"], 1),
            "deepseek_dense_frac": round(agg["ds_dense"] / peak, 4),
            "deepseek_ue8m0_achieved": round(agg["ds_ue8m0"], 1),
            "deepseek_ue8m0_frac": round(agg["ds_ue8m0"] / peak, 4),
            "note": "dense: fp32 scales (per-K-block promotion), 2MNK FLOPs; ue8m0: power-of-two "
                    "scales applied by the block-scaled MMA; dense/ue8m0_achieved average the "
                    "llama prefill shapes, deepseek_* the DeepSeek-V3 linears at M = 4096; 2:4: "
                    "MNK FLOPs (nonzero work) against the dense peak; fused / separate: the down "
                    "projection with the next layer's 1x128 quantization in the epilogue / after "
                    "it (M = 8192; not in dense_achieved); swiglu: gate+up GEMM with SwiGLU and "
                    "the down projection's quantization (codes only; one kernel where the gate+up "
                    "GEMM runs in prefill order, here M > 64), against the plain gate+up GEMM; "
                    "inputs rotated over copies so that none is in L2 at its launch",
            "shapes": rows}


def run_grouped(dev, stream, world, peak, reps=12):
    """The grouped (mixture-of-experts) GEMMs on the DeepSeek-V3 expert
    linears (gate+up N=4096 K=7168, down N=7168 K=2048): 8 experts, 4096
    routed token rows with uneven loads, each expert's rows padded to 128
    (synth.moe_layout), fp32 and UE8M0 scales. FLOPs count the routed rows
    only (2 x routed x N x K)."""
    from fp8_block_scaled_group128_b200 import binding as fb
    from fp8_block_scaled_group128_b200 import synth
    out = []
    E, routed = synth.MOE_EXPERTS, synth.MOE_ROUTED_ROWS
    for N, K in synth.MOE_LINEARS:
        mi, _ = synth.moe_layout(E, routed, seed=3)
        M = mi.numel()
        with torch.cuda.stream(stream):
            x = synth.activations("deepseek", M, K, seed=3).to(dev)
            w = synth.expert_weights("deepseek", E, N, K, seed=3).to(dev)
            mid = mi.to(dev)
            NB, KB = -(-N // 128), K // 128
            for fmt in ("fp32", "ue8m0"):
                qw = torch.empty(E, N, K, dtype=torch.uint8, device=dev)
                if fmt == "fp32":
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
                y = torch.empty(M, N, dtype=torch.bfloat16, device=dev)
                n_cp = copies_beyond_l2(M * K + E * N * K, cap=4)
                ins = [(qa, sa, qw, sw)] + [(qa.clone(), sa.clone(), qw.clone(), sw.clone())
                                            for _ in range(n_cp - 1)]
                fns = [lambda i=i: gemm(*i, mid, y=y) for i in ins]
                ms = _time_graph(fns, stream, world, reps)
                tf = 2.0 * routed * N * K / (ms * 1e-3) / 1e12
                out.append({"gemm": f"grouped_{fmt}", "experts": E, "M_routed": routed,
                            "M_padded": M, "N": N, "K": K, "us": round(ms * 1e3, 1),
                            "TFLOP/s": round(tf, 1), "frac": round(tf / peak, 4),
                            "input_copies": n_cp})
                del fns, ins, qa, sa, qw, sw, y
            del x, w
        torch.cuda.empty_cache()
    return out


def run_accuracy(dev):
    """Accuracy of the two scale formats on prefill-shaped linears (the llama
    QKV at M = 2048 and the DeepSeek-V3 (7168, 7168) linear at M = 4096):
    relative Frobenius error and largest error / largest |y| of the GPU output
    against the exact product of the bf16 inputs (float64 on the host), on 64
    sampled token rows x 512 sampled output columns."""
    import numpy as np
    from fp8_block_scaled_group128_b200 import binding as fb
    from fp8_block_scaled_group128_b200 import synth
    out = []
    for kind, M, N, K in (("llama", 2048, 6144, 4096), ("deepseek", 4096, 7168, 7168)):
        x = synth.activations(kind, M, K, seed=11)
        w = synth.weights(kind, N, K, seed=11)
        rng = np.random.default_rng(M + N)
        r = torch.from_numpy(np.sort(rng.choice(M, 64, replace=False)))
        c = torch.from_numpy(np.sort(rng.choice(N, 512, replace=False)))
        exact = x[r].double() @ w[c].double().T
        xd, wd = x.to(dev), w.to(dev)
        res = {"workload": kind, "M": M, "N": N, "K": K}
        for name, qa_f, qw_f, g_f in (
                ("fp32_scale", fb.fp8_quant_act_group128, fb.fp8_quant_weight_block128,
                 fb.fp8_block_gemm),
                ("ue8m0", fb.fp8_quant_act_group128_ue8m0, fb.fp8_quant_weight_block128_ue8m0,
                 fb.fp8_block_gemm_ue8m0)):
            y = g_f(*qa_f(xd), *qw_f(wd))
            ys = y[r.to(dev)][:, c.to(dev)].double().cpu()
            err = ys - exact
            res[name] = {"rel_fro": float(err.norm() / exact.norm()),
                         "max_abs_over_max_y": float(err.abs().max() / exact.abs().max())}
        del xd, wd
        out.append(res)
    torch.cuda.empty_cache()
    return out


QUANT_SHAPES = (("quant_act", 8192, 0, 14336), ("quant_act", 8192, 0, 4096),
                ("quant_act", 2048, 0, 4096), ("quant_weight", 0, 128256, 4096),
                ("quant_weight", 0, 28672, 4096), ("prune24", 0, 128256, 4096),
                ("prune24", 0, 28672, 4096))


def run_quantize(dev, stream, world, reps=12):
    """The quantizers at bandwidth-bound sizes (prefill activations, the LM
    head and gate+up weights), each rotating over enough input copies that no
    launch finds its input in L2; GB/s of algorithmic bytes against the
    measured copy bandwidth."""
    from fp8_block_scaled_group128_b200 import binding as fb
    from fp8_block_scaled_group128_b200 import synth
    hbm, kind_src = measured_peaks()
    rows = []
    for kind, M, N, K in QUANT_SHAPES:
        rows_in = M if kind == "quant_act" else N
        n_cp = copies_beyond_l2(2 * rows_in * K, cap=8)
        with torch.cuda.stream(stream):
            if kind == "quant_act":
                src = synth.activations("llama", M, K, seed=5).to(dev)
            else:
                src = synth.weights("llama", N, K, seed=5).to(dev)
            ins = [src] + [src.clone() for _ in range(n_cp - 1)]
            NB = -(-rows_in // 128)
            if kind == "quant_act":
                q = torch.empty(M, K, dtype=torch.uint8, device=dev)
                s = torch.empty(M, K // 128, dtype=torch.float32, device=dev)
                fns = [lambda t=t: fb.fp8_quant_act_group128(t, qa=q, sa=s) for t in ins]
            elif kind == "quant_weight":
                q = torch.empty(N, K, dtype=torch.uint8, device=dev)
                s = torch.empty(NB, K // 128, dtype=torch.float32, device=dev)
                fns = [lambda t=t: fb.fp8_quant_weight_block128(t, qw=q, sw=s) for t in ins]
            else:
                v = torch.empty(N, K // 2, dtype=torch.uint8, device=dev)
                m = torch.empty(N, K // 8, dtype=torch.uint8, device=dev)
                s = torch.empty(NB, K // 128, dtype=torch.float32, device=dev)
                fns = [lambda t=t: fb.prune24_compress(t, vals=v, meta=m, sw=s) for t in ins]
        ms = _time_graph(fns, stream, world, reps)
        gbs = kernel_bytes(kind, M, N, K) / (ms * 1e-3) / 1e9
        rows.append({"kernel": kind, "M": M, "N": N, "K": K, "us": round(ms * 1e3, 1),
                     "GB/s": round(gbs, 1), "frac": round(gbs / hbm, 4), "input_copies": n_cp})
        del fns, ins, src
        torch.cuda.empty_cache()
    return {"bound": "hbm", "unit": "GB/s", "peak": hbm,
            "peak_source": f"{kind_src} copy bandwidth", "shapes": rows}


# ------------------------------------------------------------ CPU side --

class OracleSample:
    """The CPU oracle (C++, all host cores) on a bounded sample of a pass:
    every weight row of the four linears and the token rows at M in
    ORACLE_SAMPLE_M, with the same seeded inputs as the GPU pass. Inputs are
    generated and widened to fp32 once, outside the timing."""

    def __init__(self, seed=0):
        import numpy as np
        import oracle
        from fp8_block_scaled_group128_b200 import synth
        self.oracle = oracle
        self.launches = oracle_sample_launches()
        self.bytes = sum(kernel_bytes(*l) for l in self.launches)
        self.w = {nk: synth.weights("llama", *nk, seed=seed).float().numpy() for nk in LINEARS}
        self.x = {}
        for M in ORACLE_SAMPLE_M:
            for i, nk in enumerate(LINEARS):
                self.x[(M,) + nk] = np.ascontiguousarray(
                    synth.activations("llama", M, nk[1], seed=seed + 101 * i).float().numpy())
        self.cores = oracle.threads()
        self.desc = (f"every weight row of the four linears and the token rows at M in "
                     f"{list(ORACLE_SAMPLE_M)} ({len(self.launches)} of the pass's "
                     f"{len(step_launches())} launches, {self.bytes / 1e9:.3f} GB of algorithmic "
                     f"traffic); C++ oracle on {self.cores} host threads")

    def run(self):
        o = self.oracle
        qw, sp, qa = {}, {}, {}
        for kind, M, N, K in self.launches:
            nk = (N, K)
            if kind == "quant_weight":
                qw[nk] = o.quant_weight_block128(self.w[nk])
            elif kind == "prune24":
                sp[nk] = o.prune24_compress(self.w[nk])[:3]
            elif kind == "quant_act":
                qa[(M,) + nk] = o.quant_act_group128(self.x[(M,) + nk])
            elif kind == "dense_gemm":
                o.block_gemm(*qa[(M,) + nk], *qw[nk])
            elif kind == "sparse_gemm":
                o.sparse24_gemm(*qa[(M,) + nk], *sp[nk])

    def time(self, budget_s):
        """Repeat the sample for at least `budget_s` seconds (at least once);
        returns (GB/s, seconds, repetitions)."""
        reps, t0 = 0, time.perf_counter()
        while True:
            self.run()
            reps += 1
            el = time.perf_counter() - t0
            if el >= budget_s:
                break
        return self.bytes * reps / el / 1e9, el, reps


# ---------------------------------------------------------------- arms --

def run_ours(args, rank, world, local):
    from fp8_block_scaled_group128_b200 import binding as fb
    from fp8_block_scaled_group128_b200.build import build
    if rank == 0 or not os.path.exists(fb.LIB_PATH):
        build()
    barrier(world)
    dev = torch.device("cuda", local)
    torch.cuda.set_device(dev)
    fb.lib()
    step = Step(dev, seed=rank)
    stream = torch.cuda.Stream(dev)
    launches = step_launches()
    per_pass_launches = len(launches)

    # eager warm-up (also runs the one-time per-device setup of the library)
    with torch.cuda.stream(stream):
        for _ in range(max(1, args.warmup)):
            step.run()
    stream.synchronize()
    assert fb.get_device_error(stream) == 0

    # A pass is captured as one CUDA graph and replayed (host launch cost stays
    # out of the device timing). The last R passes of the timed region replay
    # copies of the graph that also hold an event record node wherever the
    # launch kind changes (external events; each copy its own events): every
    # kind's device time over those R passes is measured live inside the timed
    # region, a run of same-kind launches as one span. Event nodes cost a few
    # microseconds each, so the other passes run the plain graph.
    launches_fns = step.launches()
    # (kind, index of the first launch, index past the last) of each run
    groups = []
    for i, (kind, _) in enumerate(launches_fns):
        if groups and groups[-1][0] == kind:
            groups[-1][2] = i + 1
        else:
            groups.append([kind, i, i + 1])

    def capture(with_events):
        evs = [torch.cuda.Event(enable_timing=True, external=True)
               for _ in range(len(groups) + 1)] if with_events else None
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g, stream=stream):
            if evs:
                evs[0].record()
            for gi, (_, a, b) in enumerate(groups):
                for _, fn in launches_fns[a:b]:
                    fn()
                if evs:
                    evs[gi + 1].record()
        return g, evs

    plain, _ = capture(False)
    # graph warm-up, which also sizes the counted step
    t0 = torch.cuda.Event(enable_timing=True)
    t1 = torch.cuda.Event(enable_timing=True)
    with torch.cuda.stream(stream):
        for _ in range(args.warmup):
            plain.replay()
        t0.record()
        for _ in range(5):
            plain.replay()
        t1.record()
    stream.synchronize()
    pass_ms = max_over_ranks(t0.elapsed_time(t1) / 5, world)
    passes = passes_per_step(args.steps, pass_ms, args.min_timed_s)
    total_passes = passes * args.steps
    R = min(10, total_passes)
    evented = [capture(True) for _ in range(R)]
    stream.synchronize()
    with torch.cuda.stream(stream):
        for g, _ in evented:
            g.replay()
    torch.cuda.synchronize()

    barrier(world)
    with ClockSampler(local) as clocks:
        torch.cuda.synchronize()
        with torch.cuda.stream(stream):
            t0.record()
            for _ in range(total_passes - R):
                plain.replay()
            for g, _ in evented:
                g.replay()
            t1.record()
        torch.cuda.synchronize()
        barrier(world)
    total_ms = t0.elapsed_time(t1)
    kernel_ms = {k: 0.0 for k in ROWS}
    for _, evs in evented:
        for gi, (kind, _, _) in enumerate(groups):
            kernel_ms[kind] += evs[gi].elapsed_time(evs[gi + 1]) / R
    assert fb.get_device_error(stream) == 0
    ms_step = max_over_ranks(total_ms / args.steps, world)

    sb = step_bytes()
    value = sb * passes * world / (ms_step * 1e-3) / 1e9
    hbm_peak, peak_kind = measured_peaks()

    breakdown = {}
    for k in ROWS:
        kb = sum(kernel_bytes(*l) for l in launches if l[0] == k)
        n = sum(1 for l in launches if l[0] == k)
        ms = kernel_ms[k]
        breakdown[k] = {"launches_per_pass": n, "ms_per_pass": round(ms, 4),
                        "GB/s": round(kb / (ms * 1e-3) / 1e9, 1) if ms > 0 else None,
                        "frac": round(kb / (ms * 1e-3) / 1e9 / hbm_peak, 4) if ms > 0 else None}
    dominant = max(ROWS, key=lambda k: kernel_ms[k])
    dom_launches = [l for l in launches if l[0] == dominant]
    dom_bytes_per_launch = sum(kernel_bytes(*l) for l in dom_launches) / len(dom_launches)
    dom_ms_per_launch = kernel_ms[dominant] / len(dom_launches)
    achieved = dom_bytes_per_launch / (dom_ms_per_launch * 1e-3) / 1e9
    ratio = recorded_traffic(dominant)
    roofline = {"bound": "hbm", "kernel": dominant, "achieved": round(achieved, 1),
                "peak": hbm_peak, "unit": "GB/s", "frac": round(achieved / hbm_peak, 4),
                "peak_source": f"{peak_kind} copy bandwidth (MEASURED_PEAKS.json hbm_gbs)"
                if peak_kind == "measured" else "fallback 6.65 TB/s",
                "algorithmic_bytes_per_launch": round(dom_bytes_per_launch),
                "traffic": None if ratio is None else round(ratio * dom_bytes_per_launch),
                "traffic_source": "profiles/traffic.json: DRAM bytes / algorithmic bytes of "
                                  "per-kernel ncu captures, times the algorithmic bytes per "
                                  "launch" if ratio is not None else "no capture on these sources"}

    # end to end: pinned host inputs -> device, one pass through the C ABI,
    # device -> host read of every output Y
    h_w, h_x = step.host_inputs()
    h2d = sum(t.numel() * t.element_size() for t in h_w.values()) + \
        sum(t.numel() * t.element_size() for t in h_x.values())
    d2h = sum(t.numel() * t.element_size() for t in step.y.values()) + \
        sum(t.numel() * t.element_size() for t in step.ys.values())
    out_host = {k: torch.empty(v.shape, dtype=v.dtype).pin_memory() for k, v in step.y.items()}
    outs_host = {k: torch.empty(v.shape, dtype=v.dtype).pin_memory() for k, v in step.ys.items()}
    e2e_steps = max(1, min(args.steps, 5))

    def e2e_once():
        for k, v in h_w.items():
            step.w[k].copy_(v, non_blocking=True)
        for k, v in h_x.items():
            step.x[k].copy_(v, non_blocking=True)
        step.run()
        for k, v in step.y.items():
            out_host[k].copy_(v, non_blocking=True)
        for k, v in step.ys.items():
            outs_host[k].copy_(v, non_blocking=True)

    with torch.cuda.stream(stream):
        e2e_once()
    stream.synchronize()
    barrier(world)
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    with torch.cuda.stream(stream):
        e0.record()
        for _ in range(e2e_steps):
            e2e_once()
        e1.record()
    stream.synchronize()
    e2e_ms = max_over_ranks(e0.elapsed_time(e1) / e2e_steps, world)
    e2e = {"value": round(sb * world / (e2e_ms * 1e-3) / 1e9, 2), "unit": UNIT,
           "ms_per_step": round(e2e_ms, 3), "passes_per_step": 1,
           "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h}

    result = {
        "metric": METRIC, "value": round(value, 1), "unit": UNIT, "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": round(ms_step, 4),
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
        "dtype": "e4m3 x e4m3 -> fp32 accumulate, bf16 out",
        "data": "synthetic (seeded bf16, Llama-3-8B linear shapes)",
        "config": bench_config(world, passes),
        "timed_region_s": round(total_ms * 1e-3, 3),
        "roofline": roofline,
        "kernels": breakdown,
        "e2e": e2e,
        "gpu_launches": per_pass_launches * total_passes,
        "clocks": clocks.summary(),
    }
    if not args.no_sections:
        result["quantize"] = run_quantize(dev, stream, world)
        result["prefill"] = run_prefill(dev, stream, world)
        result["accuracy"] = run_accuracy(dev)
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        sample = OracleSample(seed=0)
        sample.run()   # first touch of the oracle's buffers, untimed
        v, el, reps = sample.time(args.cpu_budget)
        result["cpu_baseline"] = {"value": round(v, 4), "unit": UNIT, "cores": sample.cores,
                                  "kind": "oracle", "sample": f"{sample.desc}; {reps} repetition(s)",
                                  "seconds": round(el, 2)}
    del plain, evented
    return result


def run_reference(args, rank, world):
    """The oracle as it stands (C++, fp64 GEMM, every host core) on the host:
    each counted step is one run of the bounded sample of a pass, timed by the
    host clock. Rank 0 alone runs; other ranks return without work."""
    if rank != 0:
        return None
    sample = OracleSample(seed=0)
    for _ in range(max(1, args.warmup)):
        sample.run()
    times = []
    t_all = time.perf_counter()
    for _ in range(args.steps):
        t0 = time.perf_counter()
        sample.run()
        times.append(time.perf_counter() - t0)
    wall = time.perf_counter() - t_all
    ms = 1e3 * wall / max(args.steps, 1)
    v = sample.bytes * args.steps / wall / 1e9
    cfg = bench_config(world, 1)
    cfg["sample"] = sample.desc
    cfg["sample_bytes"] = sample.bytes
    return {
        "impl": "reference", "metric": METRIC, "value": round(v, 4), "unit": UNIT,
        "n_gpus": world, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": round(ms, 1), "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "C++ oracle: fp32 quantization arithmetic, fp64 GEMM",
        "data": "synthetic (seeded bf16, Llama-3-8B linear shapes)",
        "config": cfg, "timed_region_s": round(wall, 2),
        "step_s_min_max": [round(min(times), 3), round(max(times), 3)],
        "cpu_baseline": {"value": round(v, 4), "unit": UNIT, "cores": sample.cores,
                         "kind": "oracle", "sample": sample.desc},
        "e2e": {"value": round(v, 4), "unit": UNIT, "h2d_bytes_per_step": 0,
                "d2h_bytes_per_step": 0},
    }


def main():
    ap = argparse.ArgumentParser(description=__doc__.split("\n")[0])
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=1000)
    ap.add_argument("--warmup", type=int, default=10)
    ap.add_argument("--impl", choices=("ours", "reference"), default="ours")
    ap.add_argument("--cpu-budget", type=float, default=15.0,
                    help="seconds of oracle work for the CPU baseline sample")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--min-timed-s", type=float, default=MIN_TIMED_S,
                    help="shortest timed region; a counted step replays the pass graph often "
                         "enough to reach it (0: one pass per step, e.g. under a profiler)")
    ap.add_argument("--no-sections", action="store_true",
                    help="skip the prefill and quantize sections of the JSON line")
    args = ap.parse_args()
    if args.warmup < 3 and args.impl == "ours":
        ap.error("--warmup must be >= 3")
    rank, world, local = dist_info()
    if world > 1:
        import torch.distributed as dist
        backend = "nccl" if args.impl == "ours" else "gloo"
        if backend == "nccl":
            torch.cuda.set_device(local)
        dist.init_process_group(backend, timeout=datetime.timedelta(seconds=120))
    try:
        if args.impl == "reference":
            res = run_reference(args, rank, world)
        else:
            res = run_ours(args, rank, world, local)
        if rank == 0 and res is not None:
            print(json.dumps(res), flush=True)
    finally:
        if world > 1:
            import torch.distributed as dist
            dist.destroy_process_group()


if __name__ == "__main__":
    main()

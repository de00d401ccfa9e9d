"""Host-side logic of bench.py: launch list, algorithmic bytes, the
max-over-ranks reduction on a 2-rank gloo group, clock parsing, and the
staleness check of recorded ncu traffic."""

import io
import os
import socket

import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

import bench


def test_step_launch_list_and_bytes():
    launches = bench.step_launches()
    kinds = [l[0] for l in launches]
    assert len(launches) == 4 + 4 + 16 * 3
    assert kinds.count("dense_gemm") == 16 and kinds.count("sparse_gemm") == 16
    # one weight read of the O projection at M = 1: N*K bytes of codes dominate
    b = bench.kernel_bytes("dense_gemm", 1, 4096, 4096)
    assert b == 4096 * 4096 + 4 * 32 * 32 + 4096 + 4 * 32 + 2 * 4096
    assert bench.kernel_bytes("sparse_gemm", 1, 4096, 4096) < 0.7 * b
    assert bench.kernel_bytes("quant_weight", 0, 128, 128) == 3 * 16384 + 4
    assert bench.kernel_bytes("prune24", 0, 128, 128) == 2 * 16384 + 8192 + 2048 + 4
    assert abs(bench.step_bytes() - 2.697e9) < 0.01e9


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    p = s.getsockname()[1]
    s.close()
    return p


def _worker(rank, world, port, out):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        v = bench.max_over_ranks(1.5 + rank, world)
        bench.barrier(world)
        out[rank] = v
    finally:
        dist.destroy_process_group()


def test_max_over_ranks_gloo_two_ranks():
    world = 2
    port = _free_port()
    out = mp.get_context("spawn").Manager().dict()
    mp.start_processes(_worker, args=(world, port, out), nprocs=world, start_method="spawn")
    assert dict(out) == {0: 2.5, 1: 2.5}


def test_counted_step_lasts_long_enough():
    # 20 steps of a 0.75 ms pass: 80 passes per step (1.2 s); long passes: 1
    assert bench.passes_per_step(20, 0.75) == 80
    assert bench.passes_per_step(20, 0.75) * 20 * 0.75e-3 >= bench.MIN_TIMED_S
    assert bench.passes_per_step(1000, 5.0) == 1
    assert bench.copies_beyond_l2(16 << 20, cap=16) == 16
    assert bench.copies_beyond_l2(1 << 30) == 1


def test_oracle_sample_is_a_subset_of_the_pass():
    s = bench.oracle_sample_launches()
    assert set(s) <= set(bench.step_launches())
    assert {l[0] for l in s} == set(bench.ROWS)
    assert all(l[1] in bench.ORACLE_SAMPLE_M for l in s if l[0] not in ("quant_weight", "prune24"))
    cfg = bench.bench_config(1, 3)
    assert cfg["passes_per_step"] == 3 and cfg["global_batch"] == 3 * sum(bench.TOKENS)


def test_clock_summary_parses_reasons():
    c = bench.ClockSampler(0)
    c.out = io.StringIO(
        "0, 1965, 1965, 700.1, 0x0, Not Active, Not Active, Not Active, Not Active\n"
        "0, 1800, 1965, 990.0, 0x4, Not Active, Not Active, Not Active, Active\n"
        "0, 120, 1965, 90.0, 0x1, Not Active, Not Active, Not Active, Not Active\n")
    s = c.summary()   # parses the rows; deletes nothing it did not create
    assert s["sm_max_mhz"] == 1965 and s["sm_mhz"] == 1882.5
    assert s["reasons"] == ["sw_power_cap"]


def test_recorded_traffic_requires_matching_sources(tmp_path, monkeypatch):
    monkeypatch.setattr(bench, "ROOT", str(tmp_path))
    csrc = tmp_path / "fp8_block_scaled_group128_b200" / "csrc"
    csrc.mkdir(parents=True)
    (csrc / "a.cu").write_text("x")
    (tmp_path / "profiles").mkdir()
    h = bench.source_hash()
    (tmp_path / "profiles" / "traffic.json").write_text(
        '{"source_hash": "%s", "kernels": {"prune24": {"dram_bytes": 123, '
        '"algorithmic_bytes": 246}}}' % h)
    assert bench.recorded_traffic("prune24") == 0.5
    (csrc / "a.cu").write_text("changed")
    assert bench.recorded_traffic("prune24") is None

"""Host-side logic of bench.py (CPU only): clock parsing, whole-job aggregation, the max-over-ranks
timing reduction on a 2-rank gloo group, profile bookkeeping, and the reference arm on non-zero ranks."""
import io
import json
import os
import socket
import sys
from contextlib import redirect_stdout

import pytest
import torch.multiprocessing as mp

import bench


def test_clock_summary():
    lines = ["0, 1900, 1965, 700.5, 0x0000000000000000, Not Active, Not Active, Not Active, Not Active",
             "0, 1800, 1965, 990.0, 0x0000000000000004, Not Active, Not Active, Not Active, Active",
             "0, 1850, 1965, 995.0, 0x0000000000000004, Not Active, Not Active, Not Active, Active",
             "garbage"]
    s = bench.summarize_clock_lines(lines)
    assert s["sm_mhz"] == 1850 and s["sm_max_mhz"] == 1965 and s["reasons"] == ["sw_power_cap"]
    assert s["samples"] == 3


def test_aggregate_value_counts_every_rank():
    b = bench.decode_step_bytes()
    assert abs(b - 3625975808 - 32 * sum(2 * K + 2 * N for _, K, N in bench.DECODE_SHAPES)) < 1
    assert bench.aggregate_value(1e9, 10, 4, 2.0) == pytest.approx(20.0)


def test_profiled_traffic_requires_matching_source(tmp_path):
    p = tmp_path / "traffic.json"
    h = bench.source_hash(bench.KERNEL_SOURCES["gemv_kernel"])
    p.write_text(json.dumps({"gemv_kernel": {"source_hash": h, "bytes_per_launch": 123.5}}))
    assert bench.profiled_traffic("gemv_kernel", str(p)) == 123.5
    assert bench.profiled_traffic("gemm_kernel", str(p)) is None
    p.write_text(json.dumps({"gemv_kernel": {"source_hash": "0000", "bytes_per_launch": 123.5}}))
    assert bench.profiled_traffic("gemv_kernel", str(p)) is None
    assert bench.profiled_traffic("gemv_kernel", str(tmp_path / "missing.json")) is None


def test_gpus_flag_must_match_world_size(monkeypatch, capsys):
    monkeypatch.setenv("WORLD_SIZE", "1")
    assert bench.main(["--gpus", "8", "--impl", "reference", "--steps", "1"]) == 2
    assert "WORLD_SIZE" in capsys.readouterr().err


def test_pack_and_linear_byte_counts():
    assert bench.gemv_bytes(1, 14336, 4096) == pytest.approx(14336 * 4096 * 0.51953125 + 2 * 4096 + 2 * 14336)
    assert bench.pack_bytes(14336, 4096) == pytest.approx(2 * 14336 * 4096 + 2 * 4096 + 14336 * 4096 * 0.51953125)


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, world, port, q):
    import torch.distributed as dist

    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank), WORLD_SIZE=str(world))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        bench.barrier()
        t = bench.reduce_max(1.0 + rank)          # each rank's "seconds"
        v = bench.aggregate_value(1e9, 5, world, t)
        q.put((rank, t, v))
    finally:
        dist.destroy_process_group()


def test_replica_timing_max_over_ranks_gloo():
    world = 2
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_rank_main, args=(r, world, port, q)) for r in range(world)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(timeout=120)
        assert p.exitcode == 0
    res = sorted(q.get(timeout=10) for _ in range(world))
    assert [r[1] for r in res] == [2.0, 2.0]            # every rank sees the slowest rank's time
    assert all(r[2] == pytest.approx(1e9 * 5 * 2 / 2.0 / 1e9) for r in res)


def test_reference_arm_silent_on_nonzero_rank(monkeypatch):
    monkeypatch.setenv("RANK", "1")
    monkeypatch.setenv("WORLD_SIZE", "2")
    buf = io.StringIO()
    with redirect_stdout(buf):
        rc = bench.main(["--gpus", "2", "--impl", "reference", "--steps", "1", "--warmup", "3"])
    assert rc == 0 and buf.getvalue() == ""

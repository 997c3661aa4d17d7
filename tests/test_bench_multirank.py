"""bench.py's multi-rank host logic on CPU with two gloo ranks: the timed
totals are the maximum over ranks on every rank, and the reference arm runs
and prints on rank 0 only (the other ranks exit without work)."""
from __future__ import annotations

import io
import os
import socket
import sys
from contextlib import redirect_stdout

import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, world, port, out):
    import datetime
    import torch.distributed as dist
    sys.path.insert(0, ROOT)
    import bench
    dist.init_process_group("gloo", init_method=f"tcp://127.0.0.1:{port}", rank=rank, world_size=world,
                            timeout=datetime.timedelta(seconds=60))
    try:
        got = bench.max_over_ranks([1.0 + rank, 10.0 - rank, 3.5], world, "cpu")
        buf = io.StringIO()

        class Args:
            workload, steps, warmup = "chain8", 1, 0
        if rank != 0:
            with redirect_stdout(buf):
                bench.run_reference(Args, rank, world)       # returns at once on ranks > 0
        out[rank] = (got, buf.getvalue())
        dist.barrier()
    finally:
        dist.destroy_process_group()


def test_max_over_ranks_and_rank0_only_reference():
    world = 2
    mgr = mp.get_context("spawn").Manager()
    out = mgr.dict()
    mp.start_processes(_rank_main, args=(world, _free_port(), out), nprocs=world, join=True, start_method="spawn")
    for r in range(world):
        got, printed = out[r]
        assert got == [2.0, 10.0, 3.5]
        assert printed == ""


def test_max_over_ranks_single_rank_is_identity():
    sys.path.insert(0, ROOT)
    import bench
    assert bench.max_over_ranks([1.5, 2], 1, "cpu") == [1.5, 2.0]


def test_alu_roof_fields():
    """The FP32-ALU roof of the per-shape lines: SMs x 128 lanes x 2 flops x
    the SM clock; a line's fraction is its 2*M*N*K flops over its time."""
    import types
    import bench
    fake = types.SimpleNamespace(cuda=types.SimpleNamespace(
        get_device_properties=lambda dev: types.SimpleNamespace(multi_processor_count=148)))
    peak = bench.alu_peak_tflops(fake, 0, 1965.0)
    assert abs(peak - 148 * 128 * 2 * 1965e6 / 1e12) < 1e-9
    assert abs(bench.alu_peak_tflops(fake, 0, None) - peak) < 1e-9      # no clock sample: the boost clock
    r = bench.alu_roof(2 * 8 * 4096 * 4096, 10.0, peak)                   # 268 Mflop in 10 us
    assert abs(r["alu_tflops"] - 26.84) < 0.01 and abs(r["alu_frac"] - 26.8435 / peak) < 1e-3
    assert bench.alu_roof(None, 10.0, peak) == {} and bench.alu_roof(1e9, 10.0, None) == {}

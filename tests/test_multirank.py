"""The multi-process plumbing bench.py uses for N > 1 (one process per GPU on the GPUs): a barrier,
the max over ranks of the measured time, and rank 0 alone printing, run here as two gloo ranks
on the CPU."""
import os
import socket
import sys

import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, world, port, results):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank), WORLD_SIZE=str(world))
    sys.path.insert(0, ROOT)
    import bench
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        barrier, max_over_ranks = bench._dist_helpers(world, torch.device("cpu"))
        barrier()
        results[rank] = max_over_ranks(1.5 + rank)  # each rank's "time"; all must see the max
    finally:
        dist.destroy_process_group()


def test_max_over_ranks_gloo():
    world = 2
    port = _free_port()
    with mp.Manager() as mgr:
        results = mgr.dict()
        mp.spawn(_rank_main, args=(world, port, results), nprocs=world, join=True)
        assert dict(results) == {0: 2.5, 1: 2.5}


def test_single_rank_helpers_are_identity():
    sys.path.insert(0, ROOT)
    import bench
    barrier, max_over_ranks = bench._dist_helpers(1, torch.device("cpu"))
    barrier()
    assert max_over_ranks(3.25) == 3.25


def test_reference_arm_other_ranks_print_nothing(capsys):
    sys.path.insert(0, ROOT)
    import bench

    class Args:
        config, steps, warmup, ref_step_seconds, nsa_seqlens = 1, 1, 3, 1.0, ""

    bench.run_reference(Args(), rank=1, world=2)
    assert capsys.readouterr().out == ""


def test_reference_arm_json_line():
    """bench.py --impl reference on the CPU: one JSON line with the contract's keys, the oracle's
    own arithmetic type, and end-to-end copies of zero bytes (it never touches a device)."""
    import json
    import subprocess
    r = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference", "--config", "1",
                        "--steps", "1", "--warmup", "3", "--ref-step-seconds", "1"],
                       capture_output=True, text=True, timeout=600, cwd=ROOT)
    assert r.returncode == 0, r.stderr[-2000:]
    lines = [x for x in r.stdout.splitlines() if x.startswith("{")]
    assert len(lines) == 1
    d = json.loads(lines[0])
    for key in ("impl", "metric", "value", "unit", "n_gpus", "steps", "warmup", "ms_per_step", "higher_is_better",
                "scaling", "vs_baseline", "dtype", "data", "config", "cpu_baseline", "e2e"):
        assert key in d, key
    assert d["impl"] == "reference" and d["dtype"] == "f64" and d["steps"] == 1 and d["value"] > 0
    assert d["e2e"]["h2d_bytes_per_step"] == 0 and d["e2e"]["d2h_bytes_per_step"] == 0
    assert d["cpu_baseline"]["kind"] == "oracle" and d["cpu_baseline"]["value"] == d["value"]


def test_roofline_spec_fraction():
    sys.path.insert(0, ROOT)
    import bench
    r = bench.with_spec({"unit": "GB/s", "achieved": 4000.0})
    assert r["spec_peak"] == 8000.0 and r["frac_of_spec"] == 0.5
    r = bench.with_spec({"unit": "TFLOP/s", "achieved": 1125.0})
    assert r["spec_peak"] == 2250.0 and r["frac_of_spec"] == 0.5
    assert bench.with_spec(None) is None
    assert bench.with_spec({"unit": "GB/s", "achieved": None})["frac_of_spec"] is None

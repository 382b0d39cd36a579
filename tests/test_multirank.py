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


def _shard_rank_main(rank, world, port, results):
    """One rank of the sharded block-sparse problem: its balanced range of (batch, kv head) slices,
    computed here by the fp64 oracle slice by slice (the CPU stand-in for the rank's GPU calls)."""
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank), WORLD_SIZE=str(world))
    sys.path.insert(0, ROOT)
    import numpy as np

    from oracle import attention as A
    from selected_attention_b200 import shard
    q, k, v, do, mask, bx, by, scale = _shard_problem()
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        N2 = k.shape[1]
        G = q.shape[1] // N2
        starts, segs = shard.split(mask, N2, world, rank)
        got = {}
        for b0, b1, g0, g1 in segs:
            hq, hk = slice(g0 * G, g1 * G), slice(g0, g1)
            r = A.bsa_backward(q[b0:b1, hq], k[b0:b1, hk], v[b0:b1, hk], do[b0:b1, hq], mask[b0:b1, hq], bx, by, 2,
                               scale)
            got[(b0, b1, g0, g1)] = r
        # the ranks agree on the cut and together cover every slice once
        all_starts = [None] * world
        dist.all_gather_object(all_starts, starts.tolist())
        assert all(s == all_starts[0] for s in all_starts)
        results[rank] = got
    finally:
        dist.destroy_process_group()


def _shard_problem():
    import numpy as np
    rng = np.random.default_rng(17)
    B, N1, N2, S, D, blk = 3, 4, 2, 96, 16, 32
    f = lambda *s: rng.standard_normal(s)  # noqa: E731
    nb = S // blk
    mask = (rng.random((B, N1, nb, nb)) < 0.5).astype(np.uint8)
    mask[..., np.arange(nb), np.arange(nb)] = 1
    mask[0] = 1  # uneven weights: batch 0 holds more selected tiles
    return f(B, N1, S, D), f(B, N2, S, D), f(B, N2, S, D), f(B, N1, S, D), mask, blk, blk, 1 / np.sqrt(D)


def test_sharded_slices_gloo_match_whole_problem():
    """Two gloo ranks split a block-sparse problem into contiguous (batch, kv head) ranges
    balanced by selected tiles (bsa_partition); the union of their per-slice results equals the
    whole problem's, element for element: the slices need no exchange (no collective on the
    data path)."""
    import numpy as np

    from oracle import attention as A
    world = 2
    port = _free_port()
    with mp.Manager() as mgr:
        results = mgr.dict()
        mp.spawn(_shard_rank_main, args=(world, port, results), nprocs=world, join=True)
        res = dict(results)
    q, k, v, do, mask, bx, by, scale = _shard_problem()
    full = A.bsa_backward(q, k, v, do, mask, bx, by, 2, scale)
    G = q.shape[1] // k.shape[1]
    covered = np.zeros((q.shape[0], k.shape[1]), int)
    for rank in range(world):
        assert res[rank], f"rank {rank} got no slices"
        for (b0, b1, g0, g1), r in res[rank].items():
            covered[b0:b1, g0:g1] += 1
            hq, hk = slice(g0 * G, g1 * G), slice(g0, g1)
            for i, part in enumerate((hq, hk, hk, hq, hq)):  # dq, dk, dv, out, lse
                np.testing.assert_allclose(r[i], full[i][b0:b1, part], rtol=0, atol=1e-12)
    assert np.all(covered == 1)


def _job_rank_main(rank, world, port, results):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank), WORLD_SIZE=str(world))
    sys.path.insert(0, ROOT)
    import bench
    from workloads import synth
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        w, mask, pieces, starts = bench.bsa_job(synth.workload(1), world, rank)
        G = w.N1 // w.N2
        vp = sum(bench.visible_pairs_bsa(mask[b0:b1, g0 * G:g1 * G], w.block, w.block, w.S, w.S)
                 for b0, b1, g0, g1 in pieces)
        total = bench.sum_over_ranks(world, torch.device("cpu"), vp)
        results[rank] = (w.B, pieces, vp, total, bench.visible_pairs_bsa(mask, w.block, w.block, w.S, w.S))
    finally:
        dist.destroy_process_group()


def test_bench_job_split_gloo():
    """bench.py's N-rank job (the workload's batches times N, split by slices): each rank's pieces,
    the job's credited work summed over ranks, and full coverage, as two gloo ranks."""
    world = 2
    port = _free_port()
    with mp.Manager() as mgr:
        results = mgr.dict()
        mp.spawn(_job_rank_main, args=(world, port, results), nprocs=world, join=True)
        res = dict(results)
    B = res[0][0]
    assert B == 2 * 1  # the tiny workload has one batch
    covered = set()
    for rank in range(world):
        _, pieces, vp, total, job_total = res[rank]
        assert pieces and total == job_total == res[0][2] + res[1][2]
        for b0, b1, g0, g1 in pieces:
            for b in range(b0, b1):
                for g in range(g0, g1):
                    assert (b, g) not in covered
                    covered.add((b, g))
    assert len(covered) == B * 2  # every (batch, kv head) slice of the job, once

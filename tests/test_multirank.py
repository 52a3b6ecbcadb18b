"""Host-side logic of the multi-process bench path, on CPU with two `gloo` ranks.

The layer shards as independent problems (one layer per rank, weak scaling, no
data-path collective); the only cross-rank traffic is the barrier and the
max-over-ranks reduction of the timings.  These tests run that reduction and the
whole-job aggregate on two real processes.
"""
import contextlib
import io
import os
import socket
import sys

import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)


def _free_port() -> int:
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, world, port, out):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank),
                      WORLD_SIZE=str(world), LOCAL_RANK=str(rank))
    import datetime
    import bench
    from video_dit_dynamic_b200 import inputs
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
    try:
        # rank r reports timings that make it the slowest on exactly one key
        timings = {"elapsed": 10.0 + 5.0 * rank, "att": 3.0 - rank, "pool": 1.0, "sel": 0.5 + 0.25 * rank}
        red = bench.max_over_ranks(dist, "cpu", timings)
        # the bench's per-rank inputs: same shape, independent data (seed = rank)
        wl = inputs.WORKLOADS["tiny"]
        q, _, _ = inputs.make_qkv(wl, seed=rank, device="cpu")
        gathered = [torch.empty_like(q) for _ in range(world)]
        dist.all_gather(gathered, q)
        same = bool(torch.equal(gathered[0], gathered[1]))
        # the reference arm prints on rank 0 only; other ranks exit without work
        buf = io.StringIO()
        if rank != 0:
            args = type("A", (), {"gpus": world, "steps": 1, "warmup": 3})()
            with contextlib.redirect_stdout(buf):
                ret = bench.run_reference(args, wl)
            assert ret is None
        dist.barrier()
        out.put((rank, red, same, buf.getvalue(), bench.dist_env()))
    finally:
        dist.destroy_process_group()


def test_two_rank_max_reduction_and_aggregate():
    world = 2
    ctx = mp.get_context("spawn")
    out = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_rank_main, args=(r, world, port, out)) for r in range(world)]
    for p in procs:
        p.start()
    res = {}
    try:
        for _ in range(world):
            rank, red, same, printed, env = out.get(timeout=120)
            res[rank] = (red, same, printed, env)
    finally:
        for p in procs:
            p.join(timeout=60)
            if p.is_alive():
                p.kill()
    assert all(p.exitcode == 0 for p in procs)
    want = {"elapsed": 15.0, "att": 3.0, "pool": 1.0, "sel": 0.75}
    for rank in range(world):
        red, same, printed, env = res[rank]
        assert red == pytest.approx(want)
        assert not same, "ranks must run independent layers"
        assert env == (world, rank, rank)
        if rank != 0:
            assert printed == ""


def test_job_value_counts_every_rank_over_the_slowest():
    import bench
    # two ranks, 1e12 FLOP each, slowest step 2 ms -> 2e12 / 2e-3 s = 1000 TFLOP/s
    assert bench.job_tflops(1e12, 2, 2.0) == pytest.approx(1000.0)
    assert bench.job_tflops(1e12, 1, 2.0) == pytest.approx(500.0)
    assert bench.max_over_ranks(None, "cpu", {"a": 1.5}) == {"a": 1.5}


def test_kernel_spread_and_cpu_baseline_sample():
    import bench
    from video_dit_dynamic_b200 import inputs
    assert bench.spread([3.0, 1.0, 2.0, 5.0]) == {"ms_median": 2.5, "ms_best": 1.0}
    wl = inputs.WORKLOADS["tiny"]
    k = bench.keep_count(wl.num_blocks, wl.keep)
    q, kt, v = inputs.make_qkv(wl, seed=0, device="cpu")
    # the GPU arm's baseline: the reference arm's sample, repeated, with its spread, plus one core
    r = bench.gpu_arm_cpu_baseline(wl, k, q, kt, v, repeats=2)
    assert r["kind"] == "oracle" and r["value"] > 0 and r["cores"] >= 1
    assert r["spread"]["samples"] == 2
    assert r["spread"]["min_TFLOP/s"] <= r["value"] <= r["spread"]["max_TFLOP/s"]
    sc = r["single_core"]
    assert sc["cores"] == 1 and sc["value"] > 0 and "one core" in sc["sample"]
    # both arms time the same sample: the same heads' bits go in whichever tensors they come from
    a = bench.cpu_sample_inputs(wl, q, kt, v)
    b = bench.cpu_sample_inputs(wl)
    assert all(x.shape == y.shape and x.dtype == y.dtype for x, y in zip(a, b))
    assert all((x == y).all() for x, y in zip(a, b))  # seed 0 on the host in both

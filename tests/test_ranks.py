"""Multi-rank plumbing of bench.py on CPU: two gloo ranks on 127.0.0.1.

`bench.py --gpus N` runs one process per GPU; the units (b, h) are independent, so every
rank draws its own batch and the ranks meet only for barriers and the max-over-ranks time
(weak scaling, no data-path collective).  These tests run the same functions over gloo:
the rendezvous from the launcher's environment variables, the barrier, the MAX all-reduce
of the timed region, the per-rank input seeds, the whole-job throughput, and the reference
arm's rule that only rank 0 runs and prints.
"""
import contextlib
import io
import os
import socket
import sys

import pytest
import torch
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, world, port, out):
    os.environ.update({"RANK": str(rank), "LOCAL_RANK": str(rank), "WORLD_SIZE": str(world),
                       "MASTER_ADDR": "127.0.0.1", "MASTER_PORT": str(port)})
    import bench

    got_world, got_rank, _, pg = bench.dist_setup(None)
    cpu = torch.device("cpu")
    res = {"world": got_world, "rank": got_rank}
    bench.barrier(pg, cpu)
    # every rank times a different duration; the reported time is the slowest rank's
    res["ms_max"] = bench.max_over_ranks(pg, 10.0 + 5.0 * rank, cpu)
    # each rank's synthetic batch comes from its own seed
    g = torch.Generator().manual_seed(bench.rank_seed(rank))
    x = torch.randn(8, generator=g)
    xs = [torch.empty_like(x) for _ in range(world)]
    pg.all_gather(xs, x)
    res["batches_distinct"] = all(not torch.equal(xs[i], xs[j]) for i in range(world) for j in range(i))
    res["value"] = bench.job_tokens_per_s(got_world, 32 * 3136, 100, res["ms_max"])
    # the reference arm: ranks other than 0 return at once and print nothing
    if rank != 0:
        buf = io.StringIO()
        with contextlib.redirect_stdout(buf):
            bench.run_reference(type("A", (), {"steps": 1, "warmup": 3})())
        res["reference_output"] = buf.getvalue()
    bench.barrier(pg, cpu)
    pg.destroy_process_group()
    out.put(res)


@pytest.mark.timeout(300)
def test_two_gloo_ranks():
    world = 2
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_rank_main, args=(r, world, port, q)) for r in range(world)]
    for p in procs:
        p.start()
    res = sorted((q.get(timeout=240) for _ in range(world)), key=lambda r: r["rank"])
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    assert [r["rank"] for r in res] == [0, 1]
    assert all(r["world"] == world for r in res)
    # MAX over ranks: both see the slowest rank's 15 ms
    assert all(r["ms_max"] == 15.0 for r in res)
    assert all(r["batches_distinct"] for r in res)
    # whole-job tokens/s: both ranks' tokens over the slowest time
    assert res[0]["value"] == pytest.approx(2 * 32 * 3136 * 100 / 0.015)
    assert res[1]["reference_output"] == ""



def test_single_rank_needs_no_process_group():
    import bench

    env = {k: os.environ.pop(k) for k in ("WORLD_SIZE", "RANK", "LOCAL_RANK") if k in os.environ}
    try:
        world, rank, _, pg = bench.dist_setup(None)
    finally:
        os.environ.update(env)
    assert (world, rank, pg) == (1, 0, None)
    assert bench.max_over_ranks(None, 3.5, torch.device("cpu")) == 3.5
    assert bench.job_tokens_per_s(1, 1000, 10, 2.0) == pytest.approx(5e6)

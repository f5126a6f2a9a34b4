"""Multi-rank host logic of bench.py on CPU: two gloo ranks on 127.0.0.1.

The benchmark runs independent replicas (one problem per GPU, no collective on
the data path); the only cross-rank steps are the barriers that bracket the
timed region and the max-over-ranks reduction of the elapsed time.  These are
exercised here without a GPU.
"""
import io
import json
import os
import socket
import sys
import contextlib

import pytest
import torch.distributed as dist
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, out_dir):
    os.environ.update({"RANK": str(rank), "WORLD_SIZE": str(world), "LOCAL_RANK": str(rank),
                       "MASTER_ADDR": "127.0.0.1", "MASTER_PORT": str(port)})
    sys.path.insert(0, ROOT)
    import datetime
    import bench
    r, w, lr = bench.dist_env()
    dist.init_process_group("gloo", rank=r, world_size=w,
                            timeout=datetime.timedelta(seconds=60))
    try:
        bench.barrier(w)
        # rank r reports (r + 1) * 1.5 ms; every rank must see the slowest
        got = bench.max_over_ranks((r + 1) * 1.5, w)
        bench.barrier(w)
        # the reference arm: rank 0 alone runs and prints; others exit 0 at once
        buf = io.StringIO()
        if r != 0:
            with contextlib.redirect_stdout(buf):
                rc = bench.main(["--impl", "reference", "--steps", "1", "--warmup", "3",
                                 "--gpus", str(w)])
        else:
            rc = 0
        with open(os.path.join(out_dir, f"rank{r}.json"), "w") as f:
            json.dump({"rank": r, "world": w, "local": lr, "max": got, "ref_rc": rc,
                       "ref_out": buf.getvalue()}, f)
    finally:
        dist.destroy_process_group()


def test_two_rank_barrier_and_max(tmp_path):
    world = 2
    port = _free_port()
    ctx = mp.get_context("spawn")
    procs = [ctx.Process(target=_worker, args=(r, world, port, str(tmp_path)))
             for r in range(world)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(timeout=180)
    for p in procs:
        if p.is_alive():
            p.kill()
            pytest.fail("gloo rank did not finish")
        assert p.exitcode == 0
    res = [json.load(open(tmp_path / f"rank{r}.json")) for r in range(world)]
    for r, d in enumerate(res):
        assert d["rank"] == r and d["world"] == world and d["local"] == r
        assert d["max"] == pytest.approx(3.0)
    # rank 1 of the reference arm does no work and prints nothing
    assert res[1]["ref_rc"] == 0 and res[1]["ref_out"] == ""


def test_single_rank_passthrough():
    sys.path.insert(0, ROOT)
    import bench
    assert bench.max_over_ranks(2.5, 1) == 2.5
    bench.barrier(1)  # no process group needed for one rank

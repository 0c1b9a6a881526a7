"""The benchmark's multi-rank plumbing on CPU: two gloo ranks on 127.0.0.1.

bench.py runs one process per GPU under torchrun; the only collective it makes
is the max over ranks of the measured times. These tests run that path with
world size 2 and the gloo backend, no GPU: the max reduction, the barrier, the
rank-0-only JSON line, and the reference arm's rank filter.
"""

import io
import json
import os
import socket
import sys
from contextlib import redirect_stdout

import pytest
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port():
    with socket.socket(socket.AF_INET, socket.SOCK_STREAM) as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, out_dir):
    os.environ.update(RANK=str(rank), WORLD_SIZE=str(world), LOCAL_RANK=str(rank), MASTER_ADDR="127.0.0.1",
                      MASTER_PORT=str(port))
    sys.path.insert(0, ROOT)
    import bench

    r, w, local = bench.dist_env()
    assert (r, w, local) == (rank, world, rank)
    dist = bench.init_dist(w, "gloo")
    bench.barrier(dist)
    got = bench.reduce_max(dist, 10.0 + 5.0 * rank)
    buf = io.StringIO()
    with redirect_stdout(buf):
        bench.finish_line(r, {"rank": r, "max": got})
    # the reference arm does its work on rank 0 only; the other ranks return at once
    args = type("A", (), {"steps": 1, "warmup": 0})()
    rc = bench.run_reference(args, r, w) if r != 0 else 0
    bench.barrier(dist)
    dist.destroy_process_group()
    with open(os.path.join(out_dir, f"rank{rank}.json"), "w") as fh:
        json.dump({"max": got, "printed": buf.getvalue(), "rc": rc}, fh)


def test_two_gloo_ranks_reduce_and_print_once(tmp_path):
    world = 2
    port = _free_port()
    ctx = mp.get_context("spawn")
    procs = [ctx.Process(target=_worker, args=(r, world, port, str(tmp_path))) for r in range(world)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(120)
    for p in procs:
        if p.is_alive():
            p.kill()
            pytest.fail("a rank did not finish")
        assert p.exitcode == 0
    res = [json.load(open(tmp_path / f"rank{r}.json")) for r in range(world)]
    assert all(r["max"] == 15.0 for r in res)  # max over ranks, seen by every rank
    line = json.loads(res[0]["printed"])
    assert line == {"rank": 0, "max": 15.0}
    assert res[1]["printed"] == ""  # only rank 0 prints
    assert res[1]["rc"] == 0

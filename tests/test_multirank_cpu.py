"""The N > 1 plumbing of bench.py on CPU: two gloo ranks on 127.0.0.1.

The path shards into independent (batch, head) units, so N GPUs run N replicas with no
collective on the data path; the only cross-rank steps are the barriers around the timed
region and the max over ranks of the device times.  These tests run those steps as two
processes with the gloo backend."""
import io
import os
import socket
import sys
from contextlib import redirect_stdout

import pytest
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, world, port, queue):
    sys.path.insert(0, ROOT)
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), WORLD_SIZE=str(world),
                      RANK=str(rank), LOCAL_RANK=str(rank))
    import bench
    import torch.distributed as dist
    w, r, local = bench.dist_setup(world, backend="gloo")
    assert (w, r, local) == (world, rank, rank)
    bench.barrier(w)
    # each rank reports its own time; every rank must see the slowest one
    slowest = bench.max_over_ranks(w, 1.5 + rank)
    rate = bench.whole_job_rate(1e12, w, slowest)
    bench.barrier(w)
    dist.destroy_process_group()
    queue.put((rank, slowest, rate))


def _run_two_ranks(world):
    """Runs the ranks once on a fresh port; None if a rank failed (the port picked can be
    taken by another process between the probe and the rendezvous)."""
    port = _free_port()
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    procs = [ctx.Process(target=_rank_main, args=(r, world, port, q)) for r in range(world)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(timeout=120)
    if any(p.exitcode != 0 for p in procs):
        for p in procs:
            if p.is_alive():
                p.kill()
        return None
    return sorted(q.get(timeout=10) for _ in range(world))


def test_two_gloo_ranks_take_the_max_and_aggregate():
    world = 2
    res = None
    for _ in range(3):
        res = _run_two_ranks(world)
        if res is not None:
            break
    assert res is not None, "the two gloo ranks failed three times"
    for rank, slowest, rate in res:
        assert slowest == pytest.approx(1.5 + world - 1)
        # 1e12 units per rank, 2 ranks, slowest 2.5 ms -> 8e14 units/s for the whole job
        assert rate == pytest.approx(1e12 * world / 2.5e-3)


def _reference_rank(rank, world, queue):
    sys.path.insert(0, ROOT)
    os.environ.update(WORLD_SIZE=str(world), RANK=str(rank), LOCAL_RANK=str(rank))
    import bench
    buf = io.StringIO()
    with redirect_stdout(buf):
        rc = bench.main(["--impl", "reference", "--gpus", str(world), "--steps", "1",
                         "--warmup", "0", "--cpu-budget", "1"])
    queue.put((rank, rc, buf.getvalue()))


@pytest.mark.slow
def test_reference_arm_prints_on_rank_zero_only():
    world = 2
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    procs = [ctx.Process(target=_reference_rank, args=(r, world, q)) for r in range(world)]
    for p in procs:
        p.start()
    res = sorted(q.get(timeout=600) for _ in range(world))
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    (r0, rc0, out0), (r1, rc1, out1) = res
    assert rc0 == 0 and rc1 == 0
    assert out1 == ""
    import json
    line = json.loads(out0.strip().splitlines()[-1])
    assert line["impl"] == "reference" and line["n_gpus"] == world
    assert line["value"] > 0 and line["e2e"]["h2d_bytes_per_step"] == 0

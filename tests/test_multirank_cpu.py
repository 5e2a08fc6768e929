"""The N > 1 plumbing of bench.py on CPU: two gloo ranks on 127.0.0.1.

The path shards into independent (batch, head) units, so each of N GPUs runs its own slice
of them (whole batch entries, or whole KV-head groups when the batch does not divide) with
no collective on the data path; the only cross-rank steps are the barriers around the timed
region and the max over ranks of the device times.  These tests run those steps as two
processes with the gloo backend, and check that the ranks' slices tile every workload and
hold the whole workload's input numbers."""
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
    # this rank's slice of every workload, as bench.py takes it
    import workloads
    parts = {}
    for wl in workloads.ALL:
        p = bench.my_part(wl, w)
        parts[wl.name] = (p.b0, p.B, p.hk0, p.Hkv, p.Hq)
    # and the input numbers of a small GQA workload's slice (B = 1: split by KV heads)
    import dataclasses
    small = dataclasses.replace(workloads.SWA_GQA, B=1, Nq=16, Nk=16, d=64)
    q, k, v = workloads.make_inputs(bench.my_part(small, w))
    bench.barrier(w)
    dist.destroy_process_group()
    # plain arrays (bf16 -> float32 is exact): tensors would be shared with the parent through
    # this process's memory, which is gone once it exits
    queue.put((rank, slowest, rate, parts, tuple(t.float().numpy() for t in (q, k, v))))


def _run_two_ranks(world):
    """Runs the ranks once on a fresh port; None if a rank failed (the port picked can be
    taken by another process between the probe and the rendezvous)."""
    port = _free_port()
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    procs = [ctx.Process(target=_rank_main, args=(r, world, port, q)) for r in range(world)]
    for p in procs:
        p.start()
    # read the results before joining: a child cannot exit while its queue data is unread
    res = []
    try:
        for _ in range(world):
            res.append(q.get(timeout=120))
    except Exception:
        res = None
    for p in procs:
        p.join(timeout=60)
    if res is None or any(p.exitcode != 0 for p in procs):
        for p in procs:
            if p.is_alive():
                p.kill()
        return None
    return sorted(res, key=lambda r: r[0])


def test_two_gloo_ranks_take_the_max_and_aggregate():
    world = 2
    res = None
    for _ in range(3):
        res = _run_two_ranks(world)
        if res is not None:
            break
    assert res is not None, "the two gloo ranks failed three times"
    for rank, slowest, rate, _, _ in res:
        assert slowest == pytest.approx(1.5 + world - 1)
        # 1e12 units per rank, 2 ranks, slowest 2.5 ms -> 8e14 units/s for the whole job
        assert rate == pytest.approx(1e12 * world / 2.5e-3)
    import torch
    import workloads
    for wl in workloads.ALL:
        got = [parts[wl.name] for _, _, _, parts, _ in res]
        if wl.B % world == 0:
            # whole batch entries: consecutive, disjoint, covering [0, B), all heads each
            assert [g[0] for g in got] == [r * wl.B // world for r in range(world)]
            assert all(g[1] == wl.B // world and g[3] == wl.Hkv for g in got)
        else:
            # whole KV-head groups with their query heads, covering [0, Hkv)
            assert wl.Hkv % world == 0
            assert [g[2] for g in got] == [r * wl.Hkv // world for r in range(world)]
            assert all(g[1] == wl.B and g[3] == wl.Hkv // world and
                       g[4] == wl.Hq // world for g in got)
    import dataclasses
    small = dataclasses.replace(workloads.SWA_GQA, B=1, Nq=16, Nk=16, d=64)
    full = workloads.make_inputs(small)
    for i in range(3):
        got = torch.cat([torch.from_numpy(r[4][i]) for r in res], dim=1)
        assert torch.equal(got, full[i].float())


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

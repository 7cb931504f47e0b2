"""Host logic of the N>1 bench path on CPU: two gloo ranks.

The convolution shards as independent replicas (every rank runs the whole
layer on its own seeded inputs; no collective on the data path), so what
needs checking across ranks is the timing plumbing: the barrier, and the
maximum over ranks that turns per-rank device times into the job time.
"""
import os
import socket
import sys

import pytest
import torch
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, q):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank), WORLD_SIZE=str(world),
                      LOCAL_RANK=str(rank))
    sys.path.insert(0, ROOT)
    import bench
    try:
        w, r, lr = bench.dist_env()
        assert (w, r, lr) == (world, rank, rank)
        dist = bench.init_dist(world, "gloo")
        bench.barrier(world)
        # per-rank device times: the job time is the slowest rank's
        got = bench.max_over_ranks(10.0 + 3.5 * rank, world)
        bench.barrier(world)
        # rank inputs are distinct draws (seed + 1000 * rank), same shapes
        from quantized_conv3d_implicit_b200 import workloads
        wl = bench.dataclass_replace(workloads.WORKLOADS[workloads.SMALL],
                                     seed=workloads.WORKLOADS[workloads.SMALL].seed + 1000 * rank)
        x = workloads.make_inputs(wl)["x"]
        xs = [torch.empty_like(x) for _ in range(world)]
        dist.all_gather(xs, x)
        distinct = not torch.equal(xs[0], xs[1])
        dist.destroy_process_group()
        q.put((rank, got, distinct, None))
    except Exception as e:  # noqa: BLE001 - reported to the parent
        q.put((rank, None, None, repr(e)))


def test_two_rank_barrier_and_max_over_ranks():
    world = 2
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, world, port, q)) for r in range(world)]
    for p in procs:
        p.start()
    res = [q.get(timeout=120) for _ in range(world)]
    for p in procs:
        p.join(timeout=60)
    for rank, got, distinct, err in res:
        assert err is None, f"rank {rank}: {err}"
        assert got == pytest.approx(13.5)
        assert distinct
    assert all(p.exitcode == 0 for p in procs)


def test_single_rank_helpers_are_identity():
    sys.path.insert(0, ROOT)
    import bench
    assert bench.max_over_ranks(4.25, 1) == 4.25
    bench.barrier(1)  # no process group needed


def test_traffic_is_reported_only_for_the_profiled_kernel_sources(monkeypatch):
    sys.path.insert(0, ROOT)
    import bench
    t = bench.profiled_traffic("wan_mid_384_bf16")
    assert t is None or t > 0
    # a different source set no longer matches the recorded hash: no figure
    monkeypatch.setattr(bench, "KERNEL_SOURCES", ("conv3d_igemm_basic.cu",))
    assert bench.profiled_traffic("wan_mid_384_bf16") is None
    assert bench.profiled_traffic("no_such_workload") is None

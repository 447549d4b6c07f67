"""The N > 1 path of bench.py on CPU: two gloo ranks each take their own shard of requests (no
data-path collective), and the measurement reduces the candidate total (sum) and the time (max)
over ranks."""
import os
import socket

import pytest
import torch.multiprocessing as mp


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    p = s.getsockname()[1]
    s.close()
    return p


def _worker(rank, world, port, q, shard="own"):
    import datetime

    import torch.distributed as dist
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank), WORLD_SIZE=str(world))
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
    import bench
    workload, requests = ("dca", 4) if shard == "own" else ("rocs_forward_e2e", 0)
    mine, total, ms_max = bench.shard_totals(workload, rank, world, requests, local_ms=10.0 + rank, shard=shard)
    bench.barrier(world)
    dist.destroy_process_group()
    q.put((rank, mine, total, ms_max))


def _run(world, shard):
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, world, port, q, shard)) for r in range(world)]
    for p in procs:
        p.start()
    out = sorted(q.get(timeout=120) for _ in procs)
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    return out


def test_two_rank_weak_scaling_bookkeeping():
    import bench
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    out = sorted(q.get(timeout=120) for _ in procs)
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    shards = [bench.make_case("dca", r, 4).B_C for r in range(2)]
    assert [o[1] for o in out] == shards
    for _, _, total, ms_max in out:
        assert total == sum(shards)
        assert ms_max == 11.0
    # each rank's shard is its own draw of requests (different seed), same shapes
    a, b = bench.make_case("glm_stack", 0, 8), bench.make_case("glm_stack", 1, 8)
    assert a.B_R == b.B_R == 8 and not (a.counts == b.counts).all()


def test_two_rank_strong_scaling_partition():
    """--shard lpt: both ranks build the same batch and keep their parts of the LPT request
    partition; the parts are disjoint, cover every request and its candidates, and the ranks'
    work is balanced."""
    import numpy as np

    import bench
    from request_candidate_sharing_b200 import rocs
    out = _run(2, "lpt")
    full = bench.make_case("rocs_forward_e2e", 0)
    for _, _, total, ms_max in out:
        assert total == full.B_C
        assert ms_max == 11.0
    part = rocs.partition_requests(full.counts, 2, bench.SHARD_COST_R, bench.SHARD_COST_C)
    cases = [bench.make_case("rocs_forward_e2e", r, 0, "lpt", 2) for r in range(2)]
    assert [o[1] for o in out] == [c.B_C for c in cases]
    assert sorted(np.concatenate([c.counts for c in cases]).tolist()) == sorted(full.counts.tolist())
    for r, c in enumerate(cases):
        assert np.array_equal(c.counts, full.counts[part == r])
    work = [bench.SHARD_COST_R * c.B_R + bench.SHARD_COST_C * c.B_C for c in cases]
    assert max(work) / (sum(work) / 2) < 1.01

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


def _worker(rank, world, port, q):
    import datetime

    import torch.distributed as dist
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank), WORLD_SIZE=str(world))
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
    import bench
    mine, total, ms_max = bench.shard_totals("dca", rank, world, 4, local_ms=10.0 + rank)
    bench.barrier(world)
    dist.destroy_process_group()
    q.put((rank, mine, total, ms_max))


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

"""The N > 1 path on CPU: world size 2 over gloo (127.0.0.1). Checks that the
sequence shards partition the job, that the timed region reduces to the max
over ranks, and that throughput aggregates every rank's work."""
import os
import socket

import pytest
import torch.multiprocessing as mp

from token_recurrent_decoding_b200 import ranks


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, n_global, q):
    import datetime

    import torch.distributed as dist
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world,
                            timeout=datetime.timedelta(seconds=60))
    try:
        lo, hi = ranks.shard_range(n_global, rank, world)
        my_time = 1.0 + rank * 0.5  # rank 1 is the slow one
        t = ranks.max_over_ranks(my_time, dist)
        units = ranks.max_over_ranks(float(hi - lo), dist)  # exercised twice, same order
        dist.barrier()
        q.put((rank, lo, hi, t, units))
    finally:
        dist.destroy_process_group()


@pytest.mark.parametrize("n_global", [256, 1024, 7])
def test_two_ranks_gloo(n_global):
    world = 2
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, world, port, n_global, q)) for r in range(world)]
    for p in procs:
        p.start()
    out = [q.get(timeout=120) for _ in range(world)]
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    out.sort()
    covered = []
    for rank, lo, hi, t, _ in out:
        covered.extend(range(lo, hi))
        assert t == 1.5  # the max over ranks, seen identically by both
    assert covered == list(range(n_global))
    sizes = [hi - lo for _, lo, hi, _, _ in out]
    assert max(sizes) - min(sizes) <= 1
    assert ranks.job_throughput(sizes, 1.5) == pytest.approx(n_global / 1.5)


def test_single_process_is_identity():
    assert ranks.shard_range(10, 0, 1) == (0, 10)
    assert ranks.max_over_ranks(3.25) == 3.25
    with pytest.raises(ValueError):
        ranks.shard_range(10, 2, 2)

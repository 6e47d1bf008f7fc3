"""Host logic of the multi-process benchmark path on CPU: two gloo ranks.

The layer does not shard here (one GPU per replica), so the only
cross-rank step is the timing reduction: every rank's time is replaced by the
maximum over ranks, and the reference arm runs on rank 0 only."""
import os
import socket
import sys

import pytest
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def worker(rank, world, port, q):
    import datetime
    sys.path.insert(0, ROOT)
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank), WORLD_SIZE=str(world),
                      LOCAL_RANK=str(rank))
    import torch.distributed as dist
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
    import bench
    got = bench.max_over_ranks(10.0 + 5.0 * rank)
    env = bench.dist_env()

    class A:  # minimal argument record for the reference arm
        steps, warmup, gpus = 1, 0, world
    rc = bench.run_reference(A, None) if rank != 0 else None   # non-zero ranks return at once
    dist.barrier()
    dist.destroy_process_group()
    q.put((rank, got, env, rc))


@pytest.mark.timeout(180)
def test_two_gloo_ranks_reduce_time_to_the_maximum():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = free_port()
    procs = [ctx.Process(target=worker, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    out = sorted(q.get(timeout=150) for _ in procs)
    for p in procs:
        p.join(timeout=30)
        assert p.exitcode == 0
    assert [o[1] for o in out] == [15.0, 15.0]
    assert [o[2] for o in out] == [(2, 0, 0), (2, 1, 1)]
    assert out[1][3] == 0          # rank 1 of the reference arm exits without work


def test_single_process_is_identity():
    sys.path.insert(0, ROOT)
    import bench
    assert bench.max_over_ranks(3.5) == 3.5

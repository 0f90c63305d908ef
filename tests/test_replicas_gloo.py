"""bench.py's multi-GPU path on the CPU: the path does not shard, so N GPUs run N
independent replicas and the job's time is the slowest rank's.  Two gloo ranks
check the max-over-ranks reduction and that only rank 0 reports."""

import os
import socket

import torch.multiprocessing as tmp


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank(rank, world, port, out):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank),
                      WORLD_SIZE=str(world), LOCAL_RANK=str(rank))
    import torch.distributed as dist

    import bench

    dist.init_process_group("gloo", rank=rank, world_size=world)
    ws, r, local = bench._dist()
    got = bench.max_over_ranks(100.0 + 7.0 * rank, dist)
    dist.barrier()
    dist.destroy_process_group()
    out.put((r, ws, local, got))


def test_max_over_ranks_two_gloo_ranks():
    ctx = tmp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_rank, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    res = sorted(q.get(timeout=120) for _ in procs)
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    assert [r[0] for r in res] == [0, 1] and all(r[1] == 2 for r in res)
    assert all(r[3] == 107.0 for r in res)


def test_single_rank_is_identity():
    import bench

    assert bench.max_over_ranks(3.5) == 3.5

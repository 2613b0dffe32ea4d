"""Host-side logic of the multi-rank benchmark on CPU: two gloo ranks."""
import os
import socket

import torch
import torch.multiprocessing as mp


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    p = s.getsockname()[1]
    s.close()
    return p


def _worker(rank, world, port, q):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank), WORLD_SIZE=str(world),
                      LOCAL_RANK=str(rank))
    import bench
    r, w, loc = bench.dist_env()
    assert (r, w, loc) == (rank, world, rank)
    dist = bench.init_dist(w, "gloo")
    cpu = torch.device("cpu")
    bench.barrier(w, cpu)
    m = bench.max_over_ranks(10.0 + rank, w, cpu)
    seeds = [None] * w
    dist.all_gather_object(seeds, bench.rank_seed(rank))
    q.put((rank, m, seeds))
    dist.destroy_process_group()


def test_two_gloo_ranks():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    res = [q.get(timeout=120) for _ in procs]
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    for rank, m, seeds in res:
        assert m == 11.0                         # max over ranks
        assert len(set(seeds)) == 2              # every rank has its own checkpoint

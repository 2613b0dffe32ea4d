"""The compressed all-gather's exchange on CPU ranks (gloo): every rank's container (the
oracle's, for the shard it holds) reaches every rank through one all-gather of sizes and
one of padded containers, and decoding them gives the gathered tensor. The CUDA path (the
library's compress and batched decompress around the same exchange) is in
test_gpu_collective.py."""
import datetime
import os
import socket

import numpy as np
import pytest
import torch
import torch.multiprocessing as mp


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    p = s.getsockname()[1]
    s.close()
    return p


def _shard(rank, n):
    g = torch.Generator().manual_seed(100 + rank)
    x = (torch.randn(n, generator=g) * (0.01 * (rank + 1))).to(torch.bfloat16)
    if rank == 1:
        x[: n // 2] = 0  # a shard that compresses much better: containers differ in size
    return x


def _worker(rank, world, port, n, q):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    import torch.distributed as dist
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
    try:
        import oracle
        from lossless_float_weight_b200 import collective as C
        c = torch.from_numpy(oracle.compress("bf16", _shard(rank, n), n, chunk_bytes=8192, S=512))
        buf, sizes, slot = C.exchange_containers(c)
        got = [oracle.decompress("bf16", buf[r * slot: r * slot + sizes[r]].numpy(), n, chunk_bytes=8192)
               for r in range(world)]
        q.put((rank, sizes, slot, [g.tobytes() for g in got]))
    finally:
        dist.destroy_process_group()


@pytest.mark.parametrize("world", [2, 3])
def test_exchange_containers(world):
    n = 4096 * 5 + 8
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, world, port, n, q)) for r in range(world)]
    for p in procs:
        p.start()
    res = sorted(q.get(timeout=120) for _ in procs)
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    want = [_shard(r, n).view(torch.uint8).numpy().tobytes() for r in range(world)]
    for rank, sizes, slot, got in res:
        assert got == want                      # every rank decodes every shard
        assert slot % 16 == 0 and slot >= max(sizes)
        assert sizes == res[0][1]
    assert res[0][1][1] < res[0][1][0]           # the half-zero shard's container is smaller

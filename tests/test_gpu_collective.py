"""The compressed all-gather on one B200: with one rank it gives the shard back; with
shards of several ranks laid out as the all-gather delivers them (containers padded to
a common 16-byte slot), one batched decode gives the gathered tensor."""
import pytest
import torch

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def z():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from lossless_float_weight_b200 import zipnn
    return zipnn


def test_one_rank(z):
    from lossless_float_weight_b200 import collective as C
    x = (torch.randn(300000, generator=torch.Generator().manual_seed(3)) * 0.02).to(torch.bfloat16).cuda()
    out, slot = C.all_gather_compressed(x)
    assert torch.equal(out.view(torch.int16), x.view(torch.int16))
    assert slot < x.numel() * 2  # the container is what moves


def test_slots_of_several_ranks(z):
    """Four shards of unequal compressibility: containers of four sizes in slots of the
    largest, decoded in one launch into one tensor."""
    n = 262144 * 3 + 1000
    shards = []
    for r in range(4):
        x = (torch.randn(n, generator=torch.Generator().manual_seed(r)) * 0.01 * (r + 1)).to(torch.bfloat16)
        if r == 2:
            x[::3] = 0
        shards.append(x.cuda())
    conts = [z.compress(x) for x in shards]
    sizes = [c.numel() for c in conts]
    slot = -(-max(sizes) // 16) * 16
    buf = torch.zeros(4 * slot, dtype=torch.uint8, device="cuda")
    for r, c in enumerate(conts):
        buf[r * slot: r * slot + sizes[r]].copy_(c)
    out = torch.empty(4 * n, dtype=torch.bfloat16, device="cuda")
    ws = z.batch_workspace(4)
    z.decompress_batch_into([buf[r * slot: r * slot + sizes[r]] for r in range(4)], sizes,
                            [out[r * n: (r + 1) * n] for r in range(4)], ws)
    torch.cuda.synchronize()
    assert z.status(ws) == z.OK
    assert torch.equal(out.view(torch.int16), torch.cat(shards).view(torch.int16))
    assert len(set(sizes)) == 4


def _peer_worker(rank, world, port, n, q):
    import datetime
    import os
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    import torch.distributed as dist
    torch.cuda.set_device(0)  # every rank on the one GPU: no kernel waits on another's
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
    try:
        from lossless_float_weight_b200 import collective as C
        x = _peer_shard(rank, n).cuda()
        out, moved = C.all_gather_compressed(x, peer_read=True)
        want = torch.cat([_peer_shard(r, n) for r in range(world)])
        q.put((rank, bool(torch.equal(out.cpu().view(torch.int16), want.view(torch.int16))), moved))
    finally:
        dist.destroy_process_group()


def _peer_shard(rank, n):
    g = torch.Generator().manual_seed(500 + rank)
    x = (torch.randn(n, generator=g) * 0.01 * (rank + 1)).to(torch.bfloat16)
    if rank == 1:
        x[::4] = 0  # containers of different sizes
    return x


@pytest.mark.parametrize("world", [2, 3])
def test_peer_read_across_processes(z, world):
    """The decode fused with the transfer: each process shares its container through CUDA
    IPC and one batched decode per process reads the others' containers in place (here
    processes on one GPU, so the reads stay on the device; between GPUs they cross NVLink).
    Every process gets the whole gathered tensor, and no container travels in an
    all-gather."""
    import socket
    import torch.multiprocessing as mp
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    port = s.getsockname()[1]
    s.close()
    n = 262144 * 2 + 4096
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    procs = [ctx.Process(target=_peer_worker, args=(r, world, port, n, q)) for r in range(world)]
    for p in procs:
        p.start()
    res = sorted(q.get(timeout=180) for _ in procs)
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    assert [r[1] for r in res] == [True] * world
    assert all(r[2] == 0 for r in res)

"""One container from shards, on CPU ranks (gloo): the partition of a tensor's chunks over
ranks, the all-gather of one payload size per shard and rank, the exclusive scan, and every
rank writing its pieces into one file at the scanned offsets.

No GPU here: each rank's shard container is the oracle's container of its value range,
and the relocated chunk table (the library's zipnn_shard_tables on a GPU, tested in
test_gpu_shard.py) is stood in for by shifting each entry's offset by the shard's place.
The file the ranks write must equal the oracle's container of the whole tensor."""
import datetime
import os
import socket
import struct

import numpy as np
import pytest
import torch
import torch.multiprocessing as mp

CB = 4096  # 2048 BF16 values a chunk: many chunks on a small tensor


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    p = s.getsockname()[1]
    s.close()
    return p


def _tensor(n):
    g = torch.Generator().manual_seed(n)
    return (torch.randn(n, generator=g) * 0.02).to(torch.bfloat16)


def _relocate_stand_in(shard, n_total, chunk_lo, base, payload_total):
    """The test's own shift of a shard's chunk table into the whole container, and the whole
    header (only the fields that differ from the shard's: n, chunks, offsets, total)."""
    off_codes, off_payload, total = struct.unpack_from("<QQQ", shard, 32)
    n_chunks = struct.unpack_from("<I", shard, 24)[0]
    chunks = -(-n_total // (CB // 2))
    off_codes_g = 64 + 16 * 2 * chunks
    off_payload_g = off_codes_g + (off_payload - off_codes)
    table = bytearray(shard[64: 64 + 16 * 2 * n_chunks].tobytes())
    for k in range(2 * n_chunks):
        off = struct.unpack_from("<Q", table, 16 * k + 8)[0]
        struct.pack_into("<Q", table, 16 * k + 8, off + off_payload_g + base - off_payload)
    header = bytearray(shard[:64].tobytes())
    struct.pack_into("<Q", header, 8, n_total)
    struct.pack_into("<I", header, 24, chunks)
    struct.pack_into("<QQQ", header, 32, off_codes_g, off_payload_g, off_payload_g + payload_total)
    return table, header


def _worker(rank, world, port, path, n, q):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    import torch.distributed as dist
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
    try:
        import oracle
        from lossless_float_weight_b200 import shard as SH
        x = _tensor(n)
        lo, hi = SH.partition(n, "bf16", world, CB)[rank]
        v_lo, v_hi = SH.value_range(n, "bf16", lo, hi, CB)
        shard = oracle.compress("bf16", x[v_lo:v_hi].contiguous(), v_hi - v_lo, chunk_bytes=CB, S=512)
        off_payload, total = struct.unpack_from("<QQ", shard, 40)
        all_sizes = SH.exchange_sizes(torch.tensor([total - off_payload], dtype=torch.int64))
        base, payload_total = SH.payload_base(all_sizes, rank)
        table, header = _relocate_stand_in(shard, n, lo, base[0], payload_total[0])
        pl = SH.Placement("bf16", torch.from_numpy(shard), n, lo, base[0], payload_total[0],
                          torch.frombuffer(table, dtype=torch.uint8),
                          torch.frombuffer(header, dtype=torch.uint8) if lo == 0 else None, CB)
        fd = os.open(path, os.O_WRONLY)
        pl.write(fd)
        os.close(fd)
        dist.barrier()
        q.put((rank, all_sizes.tolist(), base[0], pl.total_bytes))
    finally:
        dist.destroy_process_group()


@pytest.mark.parametrize("n,world", [(2048 * 9 + 77, 2), (2048 * 4, 3)])
def test_shards_make_one_container(tmp_path, orc, n, world):
    path = str(tmp_path / "whole.znn")
    open(path, "wb").close()
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, world, port, path, n, q)) for r in range(world)]
    for p in procs:
        p.start()
    res = sorted(q.get(timeout=120) for _ in procs)
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    whole = orc.compress("bf16", _tensor(n), n, chunk_bytes=CB, S=512)
    got = np.fromfile(path, dtype=np.uint8)
    assert got.size == whole.size and np.array_equal(got, whole)
    # every rank saw the same sizes; bases are their exclusive scan; all agree on the total
    sizes = [s[0] for s in res[0][1]]
    assert all(r[1] == res[0][1] for r in res)
    assert [r[2] for r in res] == [sum(sizes[:k]) for k in range(world)]
    assert all(r[3] == whole.size for r in res)


def test_partition_is_whole_contiguous_chunks():
    from lossless_float_weight_b200 import shard as SH
    for n, world in ((10 * 131072, 4), (131072 * 3 + 5, 8), (7, 2), (131072 * 148, 8)):
        parts = SH.partition(n, "bf16", world)
        chunks = -(-n // 131072)
        assert parts[0][0] == 0 and parts[-1][1] == chunks and len(parts) == world
        assert all(a[1] == b[0] for a, b in zip(parts, parts[1:]))
        sizes = [hi - lo for lo, hi in parts]
        assert max(sizes) - min(sizes) <= 1 and sizes == sorted(sizes, reverse=True)
        spans = [SH.value_range(n, "bf16", lo, hi) for lo, hi in parts]
        assert spans[0][0] == 0 and spans[-1][1] == n
        assert all(a[1] == b[0] for a, b in zip(spans, spans[1:]))
    # FP4 counts values, two to a byte: chunk_bytes 256 holds 512 values
    assert SH.partition(1536, "fp4_e2m1", 3, 256) == [(0, 1), (1, 2), (2, 3)]

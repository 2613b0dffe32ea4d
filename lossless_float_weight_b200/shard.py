"""One container from shards compressed on several GPUs.

A tensor of n values is cut into contiguous ranges of whole chunks, one per rank (one
process per GPU). Each rank compresses its range with the library as a tensor of its own,
and the container of the whole tensor is assembled from the shards: the header, every
shard's chunk-table entries with their payload offsets moved, the shared records, then
the shards' payload sections in rank order. It equals, byte for byte, the container one
call on the whole tensor writes ("ZipNN: Lossless Compression for AI Models", abstract:
chunks are independent, so the work splits with no exchange of data).

The only exchange between ranks is one u64 per shard and rank, the shards' payload
sizes, gathered with torch.distributed (NCCL between GPUs, gloo on CPU) and scanned into
each shard's place. This module holds host orchestration only: the partition, the
all-gather, and placing bytes at the scanned offsets (a file write at each offset, or a
copy). The sizes and the relocated tables come from the library's kernels
(zipnn_shard_sizes, zipnn_shard_tables).
"""
import ctypes
import os
import struct

import torch

from . import zipnn as Z

HEADER_BYTES = 64
ENTRY_BYTES = 16
_N_STREAMS = {Z.BF16: 2, Z.FP32: 4, Z.FP8_E4M3: 3, Z.FP4_E2M1: 3}


def values_per_chunk(dtype, chunk_bytes=Z.DEFAULT_CHUNK_BYTES):
    return int(chunk_bytes * Z._VALUES_PER_BYTE[Z.dtype_code(dtype)])


def partition(n, dtype, world, chunk_bytes=Z.DEFAULT_CHUNK_BYTES):
    """Contiguous whole-chunk ranges [(chunk_lo, chunk_hi), ...] for ranks 0..world-1, as
    even as whole chunks allow (the first C mod world ranks take one chunk more; a rank gets
    no chunk when there are fewer chunks than ranks)."""
    m0 = values_per_chunk(dtype, chunk_bytes)
    chunks = -(-n // m0)
    q, r = divmod(chunks, world)
    out, lo = [], 0
    for k in range(world):
        hi = lo + q + (1 if k < r else 0)
        out.append((lo, hi))
        lo = hi
    return out


def value_range(n, dtype, chunk_lo, chunk_hi, chunk_bytes=Z.DEFAULT_CHUNK_BYTES):
    """The values [v_lo, v_hi) of the chunks [chunk_lo, chunk_hi) of a tensor of n values."""
    m0 = values_per_chunk(dtype, chunk_bytes)
    return min(n, chunk_lo * m0), min(n, chunk_hi * m0)


def exchange_sizes(local_sizes, group=None):
    """All-gather of every rank's shard payload sizes: local_sizes is a 1-D int64 tensor
    (one entry per shard, the same count on every rank); returns (world, count), rank-major.
    Without a process group (or with one rank) the local sizes are the whole answer."""
    import torch.distributed as dist
    flat = local_sizes.reshape(-1).contiguous()
    if not dist.is_available() or not dist.is_initialized() or dist.get_world_size(group) == 1:
        return flat.reshape(1, -1)
    world = dist.get_world_size(group)
    out = torch.empty(world * flat.numel(), dtype=flat.dtype, device=flat.device)  # flat: gloo wants 1-D
    dist.all_gather_into_tensor(out, flat, group=group)
    return out.reshape(world, -1)


def payload_base(all_sizes, rank):
    """Exclusive scan over ranks: for each shard, the payload bytes of the shards before
    rank's, and the total over all ranks (host ints, from a (world, count) tensor)."""
    a = all_sizes.to("cpu", torch.int64)
    base = a[:rank].sum(dim=0) if rank else torch.zeros(a.shape[1], dtype=torch.int64)
    return [int(v) for v in base], [int(v) for v in a.sum(dim=0)]


def _items(containers, n_totals, chunk_los, tables=None, headers=None):
    count = len(containers)
    arr = (Z.ShardItem * count)()
    for i, c in enumerate(containers):
        arr[i] = Z.ShardItem(c.data_ptr(), c.numel(), n_totals[i], chunk_los[i],
                             tables[i].data_ptr() if tables is not None else None,
                             headers[i].data_ptr() if headers is not None and headers[i] is not None else None)
    return arr


def shard_sizes(containers, n_totals, chunk_los, stream=None, out=None, ws=None):
    """Payload bytes of each shard container (a device int64 tensor), by the library.
    Asynchronous; with `out` and `ws` given it allocates nothing."""
    dev = containers[0].device
    if ws is None:
        ws = torch.empty(Z.zipnn_shard_workspace_bytes(len(containers)), dtype=torch.uint8, device=dev)
    if out is None:
        out = torch.empty(len(containers), dtype=torch.int64, device=dev)
    Z.check(Z.zipnn_shard_sizes(len(containers), _items(containers, n_totals, chunk_los), out.data_ptr(),
                                ws.data_ptr(), ws.numel(), Z._stream(stream)), "zipnn_shard_sizes")
    return out, ws


def table_bytes(dtype, n_shard, chunk_bytes=Z.DEFAULT_CHUNK_BYTES):
    """Bytes of the chunk-table entries of a shard of n_shard values."""
    dt = Z.dtype_code(dtype)
    return ENTRY_BYTES * _N_STREAMS[dt] * -(-n_shard // values_per_chunk(dt, chunk_bytes))


def shard_tables(dtype, containers, n_totals, chunk_los, all_sizes, rank, world, chunk_bytes=Z.DEFAULT_CHUNK_BYTES,
                 stream=None, tables=None, headers=None, ws=None):
    """Each shard's chunk-table entries in the whole container's coordinates (device
    uint8 tensors) and, for shards that start at chunk 0, the whole header (64 device
    bytes; None for the others), by the library. all_sizes: (world, count) device int64.
    Asynchronous; with `tables`, `headers` and `ws` given it allocates and reads nothing."""
    dt = Z.dtype_code(dtype)
    dev = containers[0].device
    if tables is None:
        tables, headers = [], []
        for c, lo in zip(containers, chunk_los):
            n_shard = struct.unpack_from("<Q", c[8:16].cpu().numpy().tobytes())[0]
            tables.append(torch.empty(table_bytes(dt, n_shard, chunk_bytes), dtype=torch.uint8, device=dev))
            headers.append(torch.empty(HEADER_BYTES, dtype=torch.uint8, device=dev) if lo == 0 else None)
    if ws is None:
        ws = torch.empty(Z.zipnn_shard_workspace_bytes(len(containers)), dtype=torch.uint8, device=dev)
    sizes = all_sizes.reshape(-1).contiguous()
    Z.check(Z.zipnn_shard_tables(dt, chunk_bytes, len(containers),
                                 _items(containers, n_totals, chunk_los, tables, headers), sizes.data_ptr(),
                                 rank, world, ws.data_ptr(), ws.numel(), Z._stream(stream)), "zipnn_shard_tables")
    return tables, headers, ws


class Placement:
    """Where one shard's pieces go in the whole container (byte offsets) and what they are
    (device byte tensors). `header` and `records` are set on the rank holding chunk 0."""

    def __init__(self, dtype, container, n_total, chunk_lo, base, total, table, header, chunk_bytes):
        dt = Z.dtype_code(dtype)
        ns = _N_STREAMS[dt]
        h = container[:HEADER_BYTES].cpu().numpy().tobytes()
        off_codes, off_payload, total_local = struct.unpack_from("<QQQ", h, 32)
        chunks = -(-n_total // values_per_chunk(dt, chunk_bytes))
        off_codes_g = HEADER_BYTES + ENTRY_BYTES * ns * chunks
        self.off_payload_g = off_codes_g + (off_payload - off_codes)
        self.total_bytes = self.off_payload_g + total
        self.pieces = [(HEADER_BYTES + ENTRY_BYTES * ns * chunk_lo, table),
                       (self.off_payload_g + base, container[off_payload:total_local])]
        if header is not None:
            self.pieces += [(0, header), (off_codes_g, container[off_codes:off_payload])]

    def write(self, fd):
        """pwrite every piece at its offset of an open file (each rank writes its own)."""
        for off, t in self.pieces:
            b = t.cpu().numpy().tobytes()
            if b:
                os.pwrite(fd, b, off)

    def copy_into(self, whole):
        """Copy every piece into `whole` (a uint8 tensor holding the whole container)."""
        for off, t in self.pieces:
            if t.numel():
                whole[off: off + t.numel()].copy_(t, non_blocking=True)


def compress_sharded(x_local, n_total, chunk_lo, chunk_bytes=Z.DEFAULT_CHUNK_BYTES, plan=None, group=None,
                     rank=None, world=None, stream=None):
    """This rank's part of the whole container of a tensor split over ranks: compress the
    local values (the chunks from chunk_lo on), exchange the payload sizes, relocate the
    chunk table. Every rank of the group calls it (the same collective on each). Returns
    a Placement, or None on a rank whose range holds no chunk."""
    import torch.distributed as dist
    if rank is None:
        rank = dist.get_rank(group) if dist.is_initialized() else 0
    if world is None:
        world = dist.get_world_size(group) if dist.is_initialized() else 1
    dt = Z.dtype_code(x_local.dtype)
    if x_local.numel() == 0:  # fewer chunks than ranks: this rank has none, but still exchanges
        all_sizes = exchange_sizes(torch.zeros(1, dtype=torch.int64, device=x_local.device), group)
        return None
    cont = Z.compress(x_local, chunk_bytes=chunk_bytes, plan=plan, stream=stream)
    sizes, _ = shard_sizes([cont], [n_total], [chunk_lo], stream)
    all_sizes = exchange_sizes(sizes, group)
    tables, headers, ws = shard_tables(dt, [cont], [n_total], [chunk_lo], all_sizes, rank, world, chunk_bytes, stream)
    Z.check(Z.status(ws, stream), "zipnn_shard_tables status")
    base, total = payload_base(all_sizes, rank)
    return Placement(dt, cont, n_total, chunk_lo, base[0], total[0], tables[0], headers[0], chunk_bytes)

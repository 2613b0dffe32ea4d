"""All-gather with the payload moved compressed.

Every rank holds a shard of the same number of values; every rank needs all of them (the
all-gather of a sharded checkpoint's weights before use). Each rank compresses its shard
with the library, the ranks exchange their container sizes (one u64 each) and then the
containers themselves (one all-gather of byte buffers padded to the largest container),
and every rank decodes all the containers in one batched launch straight into the
gathered tensor. What crosses the link is the containers: about two thirds of a BF16
weight shard ("ZipNN: Lossless Compression for AI Models", abstract: compression reduces
the movement of model weights).

`exchange_containers` is the collective part alone (torch.distributed, NCCL between GPUs
or gloo on CPU); `all_gather_compressed` adds the compress and the batched decompress,
which run in the CUDA library. With peer_read the all-gather of containers is replaced by
`share_containers` (CUDA IPC views of the peers' containers) and the decode reads the
peers' memory itself: the transfer and the decode are one kernel. Its loads are plain,
never multicast, bulk copies and loads.
"""
import torch

from . import zipnn as Z


def exchange_containers(container, group=None):
    """All-gather of one container per rank (a 1-D uint8 tensor, its exact size): the
    sizes first (one int64 per rank), then the containers padded to the largest one, so
    the all-gather moves world x max-size bytes. Returns (buffer, sizes, slot): rank r's
    container is buffer[r * slot : r * slot + sizes[r]] (slot is a multiple of 16, so
    every container starts 16-byte aligned). Without a process group, one rank."""
    import torch.distributed as dist
    dev = container.device
    if not dist.is_available() or not dist.is_initialized() or dist.get_world_size(group) == 1:
        return container, [container.numel()], -(-container.numel() // 16) * 16
    world = dist.get_world_size(group)
    sizes_t = torch.empty(world, dtype=torch.int64, device=dev)
    dist.all_gather_into_tensor(sizes_t, torch.tensor([container.numel()], dtype=torch.int64, device=dev),
                                group=group)
    sizes = [int(v) for v in sizes_t.cpu()]
    slot = -(-max(sizes) // 16) * 16
    mine = torch.zeros(slot, dtype=torch.uint8, device=dev)
    mine[: container.numel()].copy_(container)
    buf = torch.empty(world * slot, dtype=torch.uint8, device=dev)
    dist.all_gather_into_tensor(buf, mine, group=group)
    return buf, sizes, slot


def share_containers(container, group=None):
    """Every rank's container, readable in place: this rank's own tensor and, for each peer,
    a view of the peer's device memory opened through CUDA IPC (the handles travel in one
    all-gather of small host objects). A kernel that reads a peer's view reads the peer's
    memory directly: over NVLink between GPUs, with nothing copied first. Peer access is
    enabled from this device to each peer's. Returns (views, sizes). Every rank keeps its
    container alive, and unchanged, until all ranks are done reading (a barrier)."""
    import torch.distributed as dist
    from torch.multiprocessing.reductions import reduce_tensor, rebuild_cuda_tensor
    world, rank = dist.get_world_size(group), dist.get_rank(group)
    _, args = reduce_tensor(container)
    objs = [None] * world
    dist.all_gather_object(objs, (container.numel(), container.device.index, args), group=group)
    here = container.device.index
    views = []
    for r, (n, dev, a) in enumerate(objs):
        if r == rank:
            views.append(container)
            continue
        if dev != here and torch.cuda.can_device_access_peer(here, dev):
            _enable_peer_access(here, dev)
        views.append(rebuild_cuda_tensor(*a))
    return views, [n for n, _, _ in objs]


def _enable_peer_access(here, peer):
    from cuda.bindings import runtime as rt
    with torch.cuda.device(here):
        err, = rt.cudaDeviceEnablePeerAccess(peer, 0)
    if err not in (rt.cudaError_t.cudaSuccess, rt.cudaError_t.cudaErrorPeerAccessAlreadyEnabled):
        raise RuntimeError(f"cudaDeviceEnablePeerAccess({peer}) from device {here}: {err}")
    rt.cudaGetLastError()  # an already-enabled peer leaves its code behind


def all_gather_compressed(x_local, group=None, chunk_bytes=Z.DEFAULT_CHUNK_BYTES, stream=None, peer_read=False):
    """The gathered tensor (rank r's shard at [r * n, (r + 1) * n) of the flattened result,
    n = x_local's values), with the shards moved compressed. Every rank of the group calls
    it with a shard of the same dtype and size.

    peer_read=False: the containers travel in one all-gather (exchange_containers), then
    one batched decode. peer_read=True (the decode fused with the transfer): the ranks
    share their containers in place (share_containers) and one batched decode reads the
    peers' containers where they are, so each peer's bitstream crosses the link once,
    straight into the shared memory of the block that decodes it, and its sign/fraction
    bytes straight into registers; the decoded values land in local memory. Barriers on
    both sides keep every container complete while it is read and alive until every rank
    is done.

    Returns (gathered, bytes each rank contributed to an all-gather of containers: the
    padded slot, or 0 with peer_read)."""
    import torch.distributed as dist
    world = dist.get_world_size(group) if dist.is_available() and dist.is_initialized() else 1
    xf = x_local.reshape(-1)
    if (xf.numel() * xf.element_size()) % 16:
        raise ValueError("all_gather_compressed: a shard must be a multiple of 16 bytes (each lands 16-byte aligned)")
    cont = Z.compress(xf, chunk_bytes=chunk_bytes, stream=stream)  # synchronises: the container is complete
    n = xf.numel()
    out = torch.empty(world * n, dtype=xf.dtype, device=xf.device)
    outs = [out[r * n: (r + 1) * n] for r in range(world)]
    ws = Z.batch_workspace(world, xf.device)
    if peer_read and world > 1:
        views, sizes = share_containers(cont, group)
        dist.barrier(group=group)  # every rank's container is complete before anyone reads it
        Z.decompress_batch_into(views, sizes, outs, ws, chunk_bytes, stream=stream)
        Z.check(Z.status(ws, stream), "all_gather_compressed: decompress")  # synchronises
        del views
        dist.barrier(group=group)  # every rank is done reading before any container is freed
        return out, 0
    buf, sizes, slot = exchange_containers(cont, group)
    items = [buf[r * slot: r * slot + sizes[r]] for r in range(world)]
    Z.decompress_batch_into(items, sizes, outs, ws, chunk_bytes, stream=stream)
    Z.check(Z.status(ws, stream), "all_gather_compressed: decompress")
    return out, slot

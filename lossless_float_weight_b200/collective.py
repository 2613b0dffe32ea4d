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
which run in the CUDA library. No peer memory is read by a kernel here: the containers
arrive through the all-gather into local memory first.
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


def all_gather_compressed(x_local, group=None, chunk_bytes=Z.DEFAULT_CHUNK_BYTES, stream=None):
    """The gathered tensor (rank r's shard at [r * n, (r + 1) * n) of the flattened result,
    n = x_local's values), with the shards moved compressed. Every rank of the group calls
    it with a shard of the same dtype and size. Returns (gathered, bytes moved per rank
    into the all-gather of containers)."""
    import torch.distributed as dist
    world = dist.get_world_size(group) if dist.is_available() and dist.is_initialized() else 1
    xf = x_local.reshape(-1)
    if (xf.numel() * xf.element_size()) % 16:
        raise ValueError("all_gather_compressed: a shard must be a multiple of 16 bytes (each lands 16-byte aligned)")
    cont = Z.compress(xf, chunk_bytes=chunk_bytes, stream=stream)
    buf, sizes, slot = exchange_containers(cont, group)
    out = torch.empty(world * xf.numel(), dtype=xf.dtype, device=xf.device)
    n = xf.numel()
    items = [buf[r * slot: r * slot + sizes[r]] for r in range(world)]
    outs = [out[r * n: (r + 1) * n] for r in range(world)]
    ws = Z.batch_workspace(world, xf.device)
    Z.decompress_batch_into(items, sizes, outs, ws, chunk_bytes, stream=stream)
    Z.check(Z.status(ws, stream), "all_gather_compressed: decompress")
    return out, slot

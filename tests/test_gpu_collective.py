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

"""Batched decompress (zipnn_decompress_batch): one launch over the chunks of many
containers must give, for every item, exactly the tensor zipnn_decompress gives alone.
B200 only. Containers come from the per-tensor compress, whose bytes the parity tests
pin to the oracle; the oracle's own containers are decoded here too."""
import numpy as np
import pytest
import torch

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def z():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from lossless_float_weight_b200 import zipnn
    return zipnn


def _batch(z, xs, conts, chunk_bytes=262144):
    outs = [torch.empty_like(x) for x in xs]
    ws = z.batch_workspace(len(xs))
    z.decompress_batch_into(conts, [c.numel() for c in conts], outs, ws, chunk_bytes)
    torch.cuda.synchronize()
    assert z.status(ws) == z.OK
    for i, (x, y) in enumerate(zip(xs, outs)):
        assert torch.equal(y.view(torch.uint8), x.view(torch.uint8)), i
    return outs


def test_mixed_sizes_and_container_shapes(z, orc):
    g = torch.Generator().manual_seed(5)
    xs, conts = [], []
    for i, n in enumerate([1, 17, 4096, 131071, 131072, 131073, 400000, 1048576, 3]):
        x = (torch.randn(n, generator=g) * (0.005 * (i + 1))).to(torch.bfloat16).cuda()
        xs.append(x)
        conts.append(z.compress(x, subblock=(64, 512, 1024, 256)[i % 4]))
    # one container from the oracle, one all-zero tensor (ZERO streams)
    xo = (torch.randn(200001, generator=g) * 0.02).to(torch.bfloat16)
    ref = orc.compress("bf16", xo.view(torch.uint8).numpy(), xo.numel(), chunk_bytes=262144, S=512)
    xs.append(xo.cuda())
    conts.append(torch.from_numpy(ref).cuda())
    xs.append(torch.zeros(70000, dtype=torch.bfloat16, device="cuda"))
    conts.append(z.compress(xs[-1]))
    _batch(z, xs, conts)


def test_plan_coded_members(z):
    from lossless_float_weight_b200 import workloads as W
    kv = W.kv_cache(shape=(1, 2, 2, 2, 1024, 128), device="cuda")  # 8 chunks, flat
    plan = z.Plan.create(kv, groups=4, seed=0)
    half = kv.numel() // 2
    parts = [kv[:half].contiguous(), kv[half:].contiguous()]
    conts = [z.compress(p, plan=plan) for p in parts] + [z.compress(parts[0])]
    _batch(z, parts + [parts[0]], conts)


@pytest.mark.parametrize("dtype", ["fp32", "fp8"])
def test_other_dtypes(z, dtype):
    from lossless_float_weight_b200 import workloads as W
    if dtype == "fp32":
        xs = [W.fp32_tensor(n=n, device="cuda") for n in (5, 65536, 100003, 300000)]
        xs.append(xs[-1].to(torch.bfloat16).to(torch.float32))  # clean: ZERO low planes
    else:
        xs = [W.fp8_tensor(rows=r, cols=4096, device="cuda").reshape(-1) for r in (1, 64, 200)]
    _batch(z, xs, [z.compress(x) for x in xs])


def test_many_small_items(z):
    # 1100 items: the block-to-item search takes several 32-way rounds
    g = torch.Generator().manual_seed(7)
    sizes = torch.randint(1, 300000, (1100,), generator=g).tolist()
    xs = [(torch.randn(n, generator=g) * 0.03).to(torch.bfloat16).cuda() for n in sizes]
    _batch(z, xs, [z.compress(x) for x in xs])


def test_a_corrupt_member_is_reported(z):
    g = torch.Generator().manual_seed(9)
    xs = [(torch.randn(300000, generator=g) * 0.02).to(torch.bfloat16).cuda() for _ in range(3)]
    conts = [z.compress(x) for x in xs]
    bad = conts[1].clone()
    bad[0] ^= 1  # magic
    outs = [torch.empty_like(x) for x in xs]
    ws = z.batch_workspace(3)
    z.decompress_batch_into([conts[0], bad, conts[2]], [c.numel() for c in conts], outs, ws)
    torch.cuda.synchronize()
    assert z.status(ws) == z.ERR_CORRUPT
    # the intact members still decode
    assert torch.equal(outs[0].view(torch.uint8), xs[0].view(torch.uint8))
    assert torch.equal(outs[2].view(torch.uint8), xs[2].view(torch.uint8))


def test_argument_errors(z):
    x = torch.zeros(100, dtype=torch.bfloat16, device="cuda")
    c = z.compress(x)
    ws = z.batch_workspace(2)
    with pytest.raises(z.ZipnnError):
        z.decompress_batch_into([c, c], [c.numel(), c.numel()], [x, x.to(torch.float32)], ws)
    with pytest.raises(z.ZipnnError):
        z.decompress_batch_into([c], [c.numel()], [x], ws[:100])


def test_checkpoint_7b_in_one_launch(z):
    from lossless_float_weight_b200 import workloads as W
    shapes = W.checkpoint_7b_shapes()
    sig = W.checkpoint_7b_sigmas(len(shapes))
    xs, conts = [], []
    for t, (name, shape) in enumerate(shapes):
        x = W.checkpoint_7b_tensor(t, shape, sig[t], "cuda").reshape(-1)
        c = z.compress(x)
        xs.append(x)
        conts.append(c[: z.compressed_size(c)])
    assert sum(x.numel() for x in xs) * 2 == 13214154752
    _batch(z, xs, conts)

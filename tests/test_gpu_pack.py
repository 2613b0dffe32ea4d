"""Packed exponent tuples on the GPU (NeuralZip, abstract: recurring exponent tuples
represented by packed exponents, chosen by the setup), against the oracle: the packed
plan (list and codes) built on the device equals the oracle's, every container equals the
oracle's byte for byte, and every decode gives back the input exactly (B200 only)."""
import numpy as np
import pytest
import torch

import golden_util as GU

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def z():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from lossless_float_weight_b200 import zipnn
    return zipnn


def _host(t):
    return t.detach().contiguous().cpu().reshape(-1).view(torch.uint8).numpy()


def _export_fields(data):
    """(K, plain lens [G, 256], packed lens [G, 256], list) of an exported BF16 plan."""
    G, K = data[5], data[6]
    b = np.frombuffer(data, dtype=np.uint8)

    def unpack(off):
        rec = b[off: off + 128 * G].reshape(G, 128)
        out = np.zeros((G, 256), dtype=np.uint8)
        out[:, 0::2] = rec & 15
        out[:, 1::2] = rec >> 4
        return out
    plain = unpack(8)
    packed = unpack(8 + 128 * G) if K else np.zeros((G, 256), dtype=np.uint8)
    lst = list(b[8 + 256 * G: 8 + 256 * G + K]) if K else []
    return K, plain, packed, lst


def _check(z, orc, x, groups, cb=262144, S=512, max_pack=15, seed=0, name=""):
    xd = x.reshape(-1).cuda()
    n = xd.numel()
    plan = z.Plan.create(xd, groups=groups, seed=seed, chunk_bytes=cb, max_pack=max_pack)
    lens, assign, _, _ = orc.plan_build("bf16", _host(x), n, cb, groups=groups, seed=seed)
    exps, plens = orc.plan_pack(_host(x), assign, groups, max_pack, n=n, chunk_bytes=cb)
    assert plan.assignment() == assign.tolist(), name
    data = plan.export()
    K, plain, packed, lst = _export_fields(data)
    assert K == len(exps) and lst == list(exps), name
    assert np.array_equal(plain, lens[0]) and np.array_equal(packed, plens), name
    got = z.compress(xd, chunk_bytes=cb, plan=plan, subblock=S).cpu().numpy()
    ref = orc.compress("bf16", _host(x), n, chunk_bytes=cb, S=S, plan_lens=lens, pack=(exps, plens), threads=8)
    assert got.size == ref.size, f"{name}: size {got.size} != oracle {ref.size}"
    bad = np.nonzero(got != ref)[0]
    assert bad.size == 0, f"{name}: {bad.size} bytes differ, first at {bad[:5]}"
    y = z.decompress(torch.from_numpy(got).cuda(), torch.bfloat16, n, chunk_bytes=cb)
    assert torch.equal(y.view(torch.uint8).cpu(), xd.view(torch.uint8).cpu()), name
    # an imported copy of the plan codes the same container
    p2 = z.Plan.from_bytes(data)
    got2 = z.compress(xd, chunk_bytes=cb, plan=p2, subblock=S).cpu().numpy()
    assert np.array_equal(got2, got), name
    return got, plan


def test_golden_packed_pairs(z, orc):
    """The hand-derived container: built on the device from the device's own packed plan."""
    fx = GU.load("bf16_packed_pairs.json")
    x = GU.packed_pairs_input().cuda()
    plan = z.Plan.create(x, groups=1, chunk_bytes=128, max_pack=2)
    got = z.compress(x, chunk_bytes=128, plan=plan, subblock=16).cpu().numpy()
    assert np.array_equal(got, GU.expected_bytes(fx))
    y = z.decompress(torch.from_numpy(GU.expected_bytes(fx).copy()).cuda(), torch.bfloat16, 64, chunk_bytes=128)
    assert torch.equal(y.cpu(), x.cpu())


def test_packed_plan_parity_kv(z, orc):
    from lossless_float_weight_b200 import workloads as W
    kv = W.kv_cache(shape=(2, 2, 4, 4, 4096, 128), seed=2).reshape(-1)  # 128 chunks
    got, _ = _check(z, orc, kv, groups=8, name="kv")
    modes = got[64: 64 + 32 * 128: 16][0::2]
    assert (modes == 4).sum() > 64


@pytest.mark.parametrize("case", ["tail", "odd", "big_chunks", "short_subblocks", "few_exponents", "max_pack_3",
                                  "partial_runs"])
def test_packed_plan_parity_shapes(z, orc, case):
    """Escapes, an odd value count (the last chunk cannot pack), chunks of 1024 sub-blocks
    (four rounds of the encoder's scan), sub-blocks of 16 values, fewer distinct exponents
    than the list holds, and a short list."""
    g = torch.Generator().manual_seed(7)
    if case == "tail":
        v = torch.randn(262144 * 3 + 4096, generator=g, dtype=torch.float64) * 0.02
        t = torch.rand(v.numel(), generator=g) < 0.01
        v[t] *= torch.pow(2.0, -torch.randint(12, 21, (int(t.sum()),), generator=g).to(torch.float64))
        _check(z, orc, v.to(torch.bfloat16), groups=4, cb=65536, name=case)
    elif case == "odd":
        x = (torch.randn(131072 * 3 + 777, generator=g) * 0.05).to(torch.bfloat16)
        got, _ = _check(z, orc, x, groups=2, cb=65536, name=case)
        assert got[64 + 32 * 12] != 4  # the last (odd) chunk's exponent entry
    elif case == "big_chunks":
        x = (torch.randn(524288 * 2 + 1000, generator=g) * 0.02).to(torch.bfloat16)
        _check(z, orc, x, groups=2, cb=1 << 20, name=case)
    elif case == "short_subblocks":
        x = (torch.randn(200000, generator=g) * 0.02).to(torch.bfloat16)
        _check(z, orc, x, groups=3, cb=65536, S=16, name=case)
    elif case == "few_exponents":
        E = torch.randint(124, 130, (300000,), generator=g)
        x = torch.pow(2.0, (E - 127).to(torch.float64)).to(torch.bfloat16)
        _check(z, orc, x, groups=2, cb=65536, name=case)
    elif case == "max_pack_3":
        x = (torch.randn(400000, generator=g) * 0.02).to(torch.bfloat16)
        _check(z, orc, x, groups=2, cb=65536, max_pack=3, name=case)
    else:  # a last chunk of 1000 values: its second sub-block's 244 pairs leave one lane 4
        x = (torch.randn(65536 * 2 + 1000, generator=g) * 0.02).to(torch.bfloat16)
        got, _ = _check(z, orc, x, groups=2, cb=131072, name=case)
        assert got[64 + 32 * 2] == 4  # the last chunk's exponent stream is PACK


def test_packed_with_zero_runs(z, orc):
    """Pruned weights (60% of the 32-value blocks all zero): PACK exponent streams next to
    ZRUN sign/fraction planes, which the BF16 encode writes while the packed encode writes
    the exponents."""
    g = torch.Generator().manual_seed(11)
    v = (torch.randn(262144 * 2 + 8192, generator=g) * 0.02)
    blocks = v.view(-1, 32)
    blocks[torch.rand(blocks.shape[0], generator=g) < 0.6] = 0
    x = v.to(torch.bfloat16)
    got, _ = _check(z, orc, x, groups=2, cb=262144, name="pruned")
    modes = got[64: 64 + 16 * 2 * 5: 16]
    assert 4 in modes[0::2].tolist() and 3 in modes[1::2].tolist()


def test_packed_with_zero_runs_unstaged(z, orc):
    """The same pruned weights in 1 MiB chunks: bitstreams too long for the shared-memory
    window, so PACK exponents beside ZRUN planes go through the per-stream readers."""
    g = torch.Generator().manual_seed(12)
    v = (torch.randn(524288 * 2 + 4096, generator=g) * 0.02)
    blocks = v.view(-1, 32)
    blocks[torch.rand(blocks.shape[0], generator=g) < 0.5] = 0
    x = v.to(torch.bfloat16)
    got, _ = _check(z, orc, x, groups=2, cb=1 << 20, name="pruned, 1 MiB chunks")
    modes = got[64: 64 + 16 * 2 * 3: 16]
    assert 4 in modes[0::2].tolist() and 3 in modes[1::2].tolist()


def test_packed_plan_reuse_and_batch(z, orc):
    """A packed plan built on one tensor codes another as the oracle does; the batched
    decode takes PACK containers with others."""
    from lossless_float_weight_b200 import workloads as W
    a = W.kv_cache(shape=(1, 2, 4, 4, 4096, 128), seed=3).reshape(-1)
    b = W.kv_cache(shape=(1, 2, 4, 4, 4096, 128), seed=4).reshape(-1)
    plan = z.Plan.create(a.cuda(), groups=4, max_pack=15)
    lens, assign, _, _ = orc.plan_build("bf16", _host(a), a.numel(), 262144, groups=4)
    exps, plens = orc.plan_pack(_host(a), assign, 4, 15, n=a.numel())
    got = z.compress(b.cuda(), plan=plan).cpu().numpy()
    ref = orc.compress("bf16", _host(b), b.numel(), plan_lens=lens, pack=(exps, plens), threads=8)
    assert np.array_equal(got, ref)
    plain = z.compress(a.cuda())
    conts = [torch.from_numpy(got).cuda(), plain]
    outs = [torch.empty(b.numel(), dtype=torch.bfloat16, device="cuda"),
            torch.empty(a.numel(), dtype=torch.bfloat16, device="cuda")]
    ws = torch.empty(z.zipnn_decompress_batch_workspace_bytes(2), dtype=torch.uint8, device="cuda")
    z.decompress_batch_into(conts, [c.numel() for c in conts], outs, ws, 262144)
    z.check(z.status(ws, None), "batch")
    assert torch.equal(outs[0].cpu(), b) and torch.equal(outs[1].cpu(), a)


def test_packed_container_damage(z):
    """A byte after the list, a list longer than 15, and a PACK entry naming a plain
    record are refused (status 3), with every read inside the container."""
    fx = GU.load("bf16_packed_pairs.json")
    good = GU.expected_bytes(fx).copy()
    for pos, val in ((352 + 5, 1), (58, 16), (64 + 4, 0)):
        bad = good.copy()
        bad[pos] = val
        with pytest.raises(z.ZipnnError) as e:
            z.decompress(torch.from_numpy(bad).cuda(), torch.bfloat16, 64, chunk_bytes=128)
        assert e.value.status == 3


def test_packed_plan_arguments(z):
    x = torch.zeros(4096, dtype=torch.float32, device="cuda")
    with pytest.raises(z.ZipnnError):
        z.Plan.create(x, groups=2, max_pack=3)  # packed exponents are BF16 only
    y = torch.zeros(4096, dtype=torch.bfloat16, device="cuda")
    with pytest.raises(z.ZipnnError):
        z.Plan.create(y, groups=2, max_pack=16)

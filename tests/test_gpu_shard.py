"""One container from shards, on one B200: the library's zipnn_shard_sizes and
zipnn_shard_tables for every shard of a tensor split over `world` ranks (the ranks run one
after another in this process; no kernel waits on another rank's), the exclusive scan of
the sizes, and the assembled container equal, byte for byte, to the single-call container
and to the oracle's."""
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


def _assemble(z, x, world, cb, plan=None):
    """Compress x split over `world` ranks and assemble the whole container (device)."""
    from lossless_float_weight_b200 import shard as SH
    dt = z.dtype_code(x.dtype)
    n = z.nvalues(x)
    per_elem = 2 if dt == z.FP4_E2M1 else 1
    parts = SH.partition(n, dt, world, cb)
    conts, sizes = [], []
    for lo, hi in parts:
        v_lo, v_hi = SH.value_range(n, dt, lo, hi, cb)
        if v_hi == v_lo:
            conts.append(None)
            sizes.append(torch.zeros(1, dtype=torch.int64, device="cuda"))
            continue
        c = z.compress(x[v_lo // per_elem: v_hi // per_elem], chunk_bytes=cb, plan=plan)
        s, ws = SH.shard_sizes([c], [n], [lo])
        assert z.status(ws) == z.OK
        conts.append(c)
        sizes.append(s)
    all_sizes = torch.stack(sizes)  # (world, 1), rank-major: what the all-gather gives every rank
    whole = None
    for r, (lo, hi) in enumerate(parts):
        if conts[r] is None:
            continue
        tables, headers, ws = SH.shard_tables(dt, [conts[r]], [n], [lo], all_sizes, r, world, cb)
        assert z.status(ws) == z.OK
        base, total = SH.payload_base(all_sizes, r)
        pl = SH.Placement(dt, conts[r], n, lo, base[0], total[0], tables[0], headers[0], cb)
        if whole is None:
            whole = torch.full((pl.total_bytes,), 0xEE, dtype=torch.uint8, device="cuda")
        pl.copy_into(whole)
    torch.cuda.synchronize()
    return whole


CASES = [
    ("bf16", 131072 * 5 + 999, 2, 262144),
    ("bf16", 131072 * 5 + 999, 3, 262144),
    ("bf16", 2048 * 40 + 1, 4, 4096),
    ("bf16", 2048 * 3, 8, 4096),        # more ranks than chunks
    ("fp32", 65536 * 3 + 17, 2, 262144),
    ("fp8_e4m3", 1 << 20, 3, 65536),
    ("fp4_e2m1", (1 << 20) + 4, 2, 65536),
    ("bf16", 300001, 1, 262144),
]


def _input(name, n):
    from lossless_float_weight_b200 import workloads as W
    g = torch.Generator().manual_seed(n)
    if name == "bf16":
        return (torch.randn(n, generator=g) * 0.02).to(torch.bfloat16)
    if name == "fp32":
        return (torch.randn(n, generator=g) * 0.02).float()
    if name == "fp8_e4m3":
        return W.fp8_tensor(rows=n // 4096, cols=4096, seed=n)
    return W.fp4_tensor(rows=2, cols=n // 2, seed=n)


@pytest.mark.parametrize("name,n,world,cb", CASES)
def test_shards_equal_one_call(z, orc, name, n, world, cb):
    x = _input(name, n)
    xd = x.reshape(-1).cuda()
    whole = _assemble(z, xd, world, cb).cpu().numpy()
    one = z.compress(xd, chunk_bytes=cb).cpu().numpy()
    assert whole.size == one.size and np.array_equal(whole, one)
    ref = orc.compress(name, x.reshape(-1), z.nvalues(x), chunk_bytes=cb, S=512, threads=8)
    assert np.array_equal(whole, ref)


def test_shards_with_a_plan(z, orc):
    """Shared records: every shard carries the plan's records; the assembled container
    holds them once, at its own off_codes."""
    from lossless_float_weight_b200 import workloads as W
    x = W.kv_cache(shape=(2, 2, 2, 2, 4096, 128), device="cuda")
    plan = z.Plan.create(x, groups=4, seed=0)
    whole = _assemble(z, x, 3, 262144, plan=plan).cpu().numpy()
    one = z.compress(x, plan=plan).cpu().numpy()
    assert np.array_equal(whole, one)


def test_shards_with_a_packed_plan(z):
    """A plan with packed exponents: the shards carry its packed records and list too, and
    the assembled container equals the single call's."""
    from lossless_float_weight_b200 import workloads as W
    x = W.kv_cache(shape=(2, 2, 2, 2, 4096, 128), device="cuda")
    plan = z.Plan.create(x, groups=4, seed=0, max_pack=15)
    whole = _assemble(z, x, 3, 262144, plan=plan).cpu().numpy()
    one = z.compress(x, plan=plan).cpu().numpy()
    assert one[58] == 15 and np.array_equal(whole, one)


def test_shard_tables_batch_and_mismatch(z):
    """Several tensors in one call (as a multi-tensor checkpoint uses it), and a shard
    whose size or range does not match: CORRUPT, nothing written for it."""
    from lossless_float_weight_b200 import shard as SH
    xs = [(torch.randn(131072 * k + 5, generator=torch.Generator().manual_seed(k)) * 0.01).to(torch.bfloat16).cuda()
          for k in (1, 2, 3)]
    conts = [z.compress(x) for x in xs]
    ns = [x.numel() for x in xs]
    sizes, ws = SH.shard_sizes(conts, ns, [0, 0, 0])
    assert z.status(ws) == z.OK
    tables, headers, ws = SH.shard_tables("bf16", conts, ns, [0, 0, 0], sizes.reshape(1, -1), 0, 1)
    assert z.status(ws) == z.OK
    for c, t, h in zip(conts, tables, headers):
        assert torch.equal(t, c[64: 64 + t.numel()]) and torch.equal(h, c[:64])  # one shard: nothing moves
    bad = sizes.clone().reshape(1, -1)
    bad[0, 1] += 16
    _, _, ws = SH.shard_tables("bf16", conts, ns, [0, 0, 0], bad, 0, 1)
    assert z.status(ws) == z.ERR_CORRUPT
    # chunks [1, 3) of a tensor of ns[0] + 131079 values would hold ns[0] + 7 values, not ns[0]
    _, _, ws = SH.shard_tables("bf16", conts[:1], [ns[0] + 131079], [1], sizes[:1].reshape(1, 1), 0, 1)
    assert z.status(ws) == z.ERR_CORRUPT

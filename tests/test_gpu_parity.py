"""Parity of the CUDA path with the CPU oracle (B200 only).

Every compressed container must equal the oracle's byte for byte, and every
decompressed tensor must equal the input byte for byte (integer work: bit-exact is the
only bar). Inputs come from lossless_float_weight_b200.workloads, seeded; the oracle
sees the same bytes copied to the host.
"""
import numpy as np
import pytest
import torch

import container_util as CU
import golden_util as GU

pytestmark = pytest.mark.gpu

S_DEFAULT = 512
CB = 262144


@pytest.fixture(scope="module")
def z():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from lossless_float_weight_b200 import zipnn
    return zipnn


def _host_bytes(t):
    return t.detach().contiguous().cpu().reshape(-1).view(torch.uint8).numpy()


def _check_roundtrip(z, orc, x, name, chunk_bytes=CB, subblock=S_DEFAULT, plan=None, plan_lens=None):
    dtype = {torch.bfloat16: "bf16", torch.float32: "fp32", torch.float8_e4m3fn: "fp8_e4m3",
             torch.float4_e2m1fn_x2: "fp4_e2m1"}[x.dtype]
    xd = x.reshape(-1).cuda()
    cont = z.compress(xd, chunk_bytes=chunk_bytes, plan=plan, subblock=subblock)
    got = cont.cpu().numpy()
    ref = orc.compress(dtype, _host_bytes(x), z.nvalues(x), chunk_bytes=chunk_bytes, S=subblock, plan_lens=plan_lens,
                       threads=8)
    assert got.size == ref.size, f"{name}: size {got.size} != oracle {ref.size}"
    bad = np.nonzero(got != ref)[0]
    assert bad.size == 0, f"{name}: {bad.size} bytes differ, first at {bad[:5]}"
    y = z.decompress(cont, x.dtype, x.numel(), chunk_bytes=chunk_bytes)
    assert torch.equal(y.view(torch.uint8).cpu(), x.reshape(-1).contiguous().view(torch.uint8).cpu()), name
    # and the GPU decodes the oracle's container
    y2 = z.decompress(torch.from_numpy(ref).cuda(), x.dtype, x.numel(), chunk_bytes=chunk_bytes)
    assert torch.equal(y2.view(torch.uint8).cpu(), x.reshape(-1).contiguous().view(torch.uint8).cpu()), name
    return got


def test_bf16_small_config(z, orc):
    from lossless_float_weight_b200 import workloads as W
    x = W.bf16_small()
    c = _check_roundtrip(z, orc, x, "bf16 1M")
    assert 0.64 <= c.size / (2 * x.numel()) <= 0.68


def test_golden_containers(z, orc):
    x = GU.three_chunk_input().cuda()
    fx = GU.load("bf16_three_chunks.json")
    got = z.compress(x, chunk_bytes=512, subblock=64).cpu().numpy()
    assert np.array_equal(got, GU.expected_bytes(fx))
    y = z.decompress(torch.from_numpy(GU.expected_bytes(fx).copy()).cuda(), torch.bfloat16, 517, chunk_bytes=512)
    assert torch.equal(y.cpu(), x.cpu())


# every hand-derived golden container: (fixture, input builder, shared-code plan?)
GOLDEN_ALL = [
    ("bf16_three_chunks.json", GU.three_chunk_input, False),
    ("bf16_shared_code.json", GU.three_chunk_input, True),
    ("fp8_two_chunks.json", GU.fp8_two_chunk_input, False),
    ("fp8_shared_code.json", GU.fp8_two_chunk_input, True),
    ("fp32_clean_two_chunks.json", GU.fp32_clean_two_chunk_input, False),
    ("fp4_two_chunks.json", GU.fp4_two_chunk_input, False),
    ("bf16_zero_runs.json", GU.zero_runs_input, False),
]


@pytest.mark.parametrize("name,make,with_plan", GOLDEN_ALL)
def test_golden_containers_every_dtype(z, name, make, with_plan):
    """The library writes each hand-derived container byte for byte and decodes it back.
    A fixture's hand-written plan enters through zipnn_plan_import: its exported form is
    "ZNP1", dtype, groups, two zero bytes, then the container's shared records."""
    fx = GU.load(name)
    src = GU.load(fx["input"]["same_as"]) if "same_as" in fx["input"] else fx
    exp = GU.expected_bytes(fx)
    h = fx["header"]
    plan = None
    if with_plan:
        blob = b"ZNP1" + bytes([h["dtype"], h["n_groups"], 0, 0]) + exp[h["off_codes"]: h["off_payload"]].tobytes()
        plan = z.Plan.from_bytes(blob)
    x = make().cuda()
    got = z.compress(x, chunk_bytes=src["input"]["chunk_bytes"], subblock=src["input"]["S"], plan=plan)
    got = got.cpu().numpy()
    assert got.size == exp.size and np.array_equal(got, exp), np.nonzero(got[: exp.size] != exp[: got.size])[0][:8]
    y = z.decompress(torch.from_numpy(exp.copy()).cuda(), x.dtype, x.numel(), chunk_bytes=src["input"]["chunk_bytes"])
    assert torch.equal(y.cpu().view(torch.uint8), x.cpu().view(torch.uint8))


@pytest.mark.parametrize("n", [1, 7, 8, 15, 16, 17, 1023, 4095, 4096, 4097, 131071, 131072, 131073, 400000])
def test_bf16_ragged_sizes(z, orc, n):
    x = (torch.randn(n, generator=torch.Generator().manual_seed(n)) * 0.02).to(torch.bfloat16)
    _check_roundtrip(z, orc, x, f"bf16 n={n}")


@pytest.mark.parametrize("chunk_bytes,subblock", [(16, 16), (4096, 64), (65536, 256), (262144, 1024),
                                                  (1 << 20, 2048), (262144, 65536),
                                                  # more sub-blocks than decode threads: two per thread,
                                                  # one or several batches, a partly filled batch
                                                  (262144, 256), (262144, 128), (131072, 16), (262144, 48),
                                                  (262144, 272)])
def test_bf16_chunk_and_subblock_shapes(z, orc, chunk_bytes, subblock):
    x = (torch.randn(300001, generator=torch.Generator().manual_seed(1)) * 0.05).to(torch.bfloat16)
    _check_roundtrip(z, orc, x, f"cb={chunk_bytes} S={subblock}", chunk_bytes=chunk_bytes, subblock=subblock)


def test_every_bf16_and_fp8_pattern(z, orc):
    rng = np.random.default_rng(0)
    pats = torch.from_numpy(rng.permutation(np.arange(65536, dtype=np.int64)).astype(np.int16))
    _check_roundtrip(z, orc, pats.view(torch.bfloat16), "bf16 patterns", chunk_bytes=4096, subblock=64)
    _check_roundtrip(z, orc, torch.arange(65536, dtype=torch.int32).to(torch.int16).view(torch.bfloat16),
                     "bf16 ordered patterns", chunk_bytes=4096)
    f8 = torch.from_numpy(np.tile(np.arange(256, dtype=np.uint8), 500)).view(torch.float8_e4m3fn)
    _check_roundtrip(z, orc, f8, "fp8 patterns", chunk_bytes=4096, subblock=128)


def test_constant_and_zero_tensors(z, orc):
    for x in (torch.zeros(300000, dtype=torch.bfloat16), torch.ones(300000, dtype=torch.bfloat16),
              torch.full((70000,), -2.5, dtype=torch.float32), torch.zeros(70000, dtype=torch.float32),
              torch.zeros(90000, dtype=torch.uint8).view(torch.float8_e4m3fn)):
        _check_roundtrip(z, orc, x, f"constant {x.dtype}")


def test_bf16_largest_chunk(z, orc):
    # chunk_bytes = 2^28, the largest the ABI takes: a chunk of 2^27 values (4096 encode
    # tiles, 262,144 sub-blocks, a bitstream far beyond the shared-memory window) and a
    # second chunk of 5 values
    cb = 1 << 28
    n = (1 << 27) + 5
    x = (torch.randn(n, generator=torch.Generator().manual_seed(13)) * 0.02).to(torch.bfloat16)
    _check_roundtrip(z, orc, x, "bf16 2^28-byte chunks", chunk_bytes=cb)
    h = z.histogram(x.cuda(), chunk_bytes=cb).cpu().numpy()
    hb = _host_bytes(x)
    for c, (lo, hi) in enumerate(((0, 1 << 27), (1 << 27, n))):
        assert np.array_equal(h[c, 0].astype(np.uint64), orc.histogram("bf16", hb, lo, hi, 0)), c


def _mixed_modes_bf16():
    # one tensor whose chunks take every pair of stream modes: zeros (ZERO, ZERO), weights
    # (HUFF, RAW), positive powers of two (HUFF, ZERO), every bit pattern at random
    # (RAW, RAW), and a ragged tail of weights (HUFF, RAW)
    m0 = 131072
    g = torch.Generator().manual_seed(11)
    parts = [torch.zeros(m0), torch.randn(m0, generator=g) * 0.02,
             torch.pow(2.0, -torch.randint(1, 20, (m0,), generator=g).float()), None,
             torch.randn(1001, generator=g) * 0.02]
    pat = torch.randint(0, 65536, (m0,), generator=g, dtype=torch.int32).to(torch.int16).view(torch.bfloat16)
    return torch.cat([p.to(torch.bfloat16) if p is not None else pat for p in parts])


def test_bf16_mixed_chunk_modes(z, orc):
    import struct
    x = _mixed_modes_bf16()
    got = _check_roundtrip(z, orc, x, "bf16 mixed modes")
    modes = [struct.unpack_from("<I", got, 64 + 16 * k)[0] & 0xFF for k in range(10)]
    assert modes == [1, 1, 2, 0, 2, 1, 0, 0, 2, 0]  # ZERO 1, HUFF 2, RAW 0; (exp, sign/fraction) per chunk
    # decoded in one batch beside a tensor of weights
    w = (torch.randn(300001, generator=torch.Generator().manual_seed(12)) * 0.03).to(torch.bfloat16)
    conts = [z.compress(x.cuda()), z.compress(w.cuda())]
    outs = [torch.empty(t.numel(), dtype=torch.bfloat16, device="cuda") for t in (x, w)]
    ws = z.batch_workspace(2)
    z.decompress_batch_into(conts, [c.numel() for c in conts], outs, ws)
    torch.cuda.synchronize()
    assert z.status(ws) == z.OK
    for o, t in zip(outs, (x, w)):
        assert torch.equal(o.view(torch.int16).cpu(), t.view(torch.int16))


def test_fp32_and_clean(z, orc):
    from lossless_float_weight_b200 import workloads as W
    x = W.fp32_tensor(n=(1 << 21) + 333)
    c = _check_roundtrip(z, orc, x, "fp32")
    assert 0.82 <= c.size / (4 * x.numel()) <= 0.85
    xc = x.to(torch.bfloat16).to(torch.float32)
    c = _check_roundtrip(z, orc, xc, "fp32 clean")
    assert c.size / (4 * x.numel()) < 0.35


def test_fp32_special_values(z, orc):
    rng = np.random.default_rng(2)
    bits = rng.integers(0, 2 ** 32, size=100000, dtype=np.uint64).astype(np.uint32)
    specials = np.array([0.0, -0.0, np.inf, -np.inf, np.nan, 1e-45, -1e-45, 3.4028235e38], dtype=np.float32)
    x = np.concatenate([specials.view(np.uint32), bits]).view(np.int32)
    _check_roundtrip(z, orc, torch.from_numpy(x).view(torch.float32), "fp32 bits", chunk_bytes=4096)


def test_fp8(z, orc):
    from lossless_float_weight_b200 import workloads as W
    q = W.fp8_tensor(rows=600, cols=4096)
    q = torch.cat([q, q[:777]])
    c = _check_roundtrip(z, orc, q, "fp8")
    assert c.size / q.numel() < 0.9


def _spread_bf16(n, binades, seed):
    from lossless_float_weight_b200 import workloads as W
    return W.spread_bf16(n, binades, seed)


@pytest.mark.parametrize("binades", [6, 9, 10, 16])
def test_bf16_high_entropy_exponents(z, orc, binades):
    # the three decode paths: the 48 KB window with the two-symbol table, the 56 KB window
    # with the single-symbol table (9, and 10 at the limit), and the global-memory reader
    x = _spread_bf16(131072 * 3 + 1001, binades, binades)
    _check_roundtrip(z, orc, x, f"bf16 {binades} binades")
    _check_roundtrip(z, orc, x, f"bf16 {binades} binades S=256", subblock=256)
    conts = [z.compress(x.cuda()), z.compress(x.cuda(), subblock=1024)]
    outs = [torch.empty(x.numel(), dtype=torch.bfloat16, device="cuda") for _ in conts]
    ws = z.batch_workspace(2)
    z.decompress_batch_into(conts, [c.numel() for c in conts], outs, ws)
    torch.cuda.synchronize()
    assert z.status(ws) == z.OK
    for o in outs:
        assert torch.equal(o.view(torch.int16).cpu(), x.view(torch.int16))


def test_bf16_wide_window_corrupt(z, orc):
    # chunk 0's bitstream (53 KB) is in flight into shared memory when its code record
    # fails the Kraft check; flips in its last 8 KB (the part kept in the table region)
    # are detected or decode, never fault
    import struct
    x = _spread_bf16(131072 * 2, 9, 3)
    c = z.compress(x.cuda()).cpu().numpy()
    off0 = struct.unpack_from("<Q", c, 64 + 8)[0]
    end0 = struct.unpack_from("<Q", c, 64 + 16 + 8)[0]
    assert 48 * 1024 < end0 - off0 - 128 - 4 * 256 <= 56 * 1024
    ws = torch.zeros(256, dtype=torch.uint8, device="cuda")
    out = torch.empty(x.numel(), dtype=torch.bfloat16, device="cuda")
    d = c.copy(); d[off0: off0 + 128] = 0x11
    z.decompress_into(torch.from_numpy(d).cuda(), d.size, out, ws)
    assert z.status(ws) == z.ERR_CORRUPT
    assert orc.decompress_status("bf16", d, x.numel()) == orc.ECORRUPT
    rng = np.random.default_rng(9)
    for _ in range(20):
        d = c.copy()
        d[int(rng.integers(end0 - 8192, end0))] ^= 1 << int(rng.integers(0, 8))
        z.decompress_into(torch.from_numpy(d).cuda(), d.size, out, ws)
        assert z.status(ws) in (z.OK, z.ERR_CORRUPT)
    torch.cuda.synchronize()


def _fp4(raw):
    return torch.from_numpy(np.ascontiguousarray(raw, dtype=np.uint8)).view(torch.float4_e2m1fn_x2)


def test_fp4(z, orc):
    from lossless_float_weight_b200 import workloads as W
    q = W.fp4_tensor(rows=512, cols=4096)  # 2,097,152 values, 4 chunks
    got = _check_roundtrip(z, orc, q, "fp4")
    assert got.size < 0.95 * q.numel()  # the exponent plane compresses
    _check_roundtrip(z, orc, q, "fp4 S=64", chunk_bytes=65536, subblock=64)


def test_every_fp4_byte_pattern_and_ragged_sizes(z, orc):
    pats = np.arange(256, dtype=np.uint8)
    rng = np.random.default_rng(11)
    _check_roundtrip(z, orc, _fp4(np.tile(pats, 64)), "fp4 patterns", chunk_bytes=4096, subblock=64)
    _check_roundtrip(z, orc, _fp4(rng.permutation(np.tile(pats, 700))), "fp4 shuffled", chunk_bytes=65536)
    for nbytes in (1, 9, 8192, 8193, 131073, 200001):  # 2 .. 400002 values; ragged last chunks
        _check_roundtrip(z, orc, _fp4(rng.integers(0, 256, nbytes, dtype=np.uint8)), f"fp4 {nbytes} B",
                         chunk_bytes=65536)
    # FP4 values come in pairs: an odd count is an argument error
    out = torch.empty(1024, dtype=torch.uint8, device="cuda")
    ws = torch.empty(1 << 20, dtype=torch.uint8, device="cuda")
    assert z.zipnn_compress(z.FP4_E2M1, out.data_ptr(), 7, CB, None, out.data_ptr(), out.numel(), ws.data_ptr(),
                            ws.numel(), None) == z.ERR_INVALID_ARG


def test_fp4_plan_and_batch(z, orc):
    from lossless_float_weight_b200 import workloads as W
    q = W.fp4_tensor(rows=1024, cols=4096, seed=2)  # 16 chunks of 64 KiB
    plan = z.Plan.create(q.cuda(), groups=4, seed=1, chunk_bytes=65536)
    lens, assign, _, _ = orc.plan_build("fp4_e2m1", _host_bytes(q), z.nvalues(q), 65536, groups=4, seed=1)
    assert plan.assignment() == assign.tolist()
    _check_roundtrip(z, orc, q, "fp4 plan", chunk_bytes=65536, plan=plan, plan_lens=lens)
    xs = [W.fp4_tensor(rows=r, cols=4096, seed=r, device="cuda") for r in (1, 64, 300)]
    conts = [z.compress(x, chunk_bytes=65536) for x in xs]
    outs = [torch.empty_like(x) for x in xs]
    ws = z.batch_workspace(len(xs))
    z.decompress_batch_into(conts, [c.numel() for c in conts], outs, ws, 65536)
    torch.cuda.synchronize()
    assert z.status(ws) == z.OK
    for x, y in zip(xs, outs):
        assert torch.equal(y.view(torch.uint8), x.view(torch.uint8))


def test_histogram_entry_point(z, orc):
    from lossless_float_weight_b200 import workloads as W
    for x, dt, cb in ((W.bf16_small(n=500001), "bf16", CB), (W.fp8_tensor(rows=70, cols=4096), "fp8_e4m3", 65536),
                      (W.fp32_tensor(n=100003), "fp32", 65536)):
        h = z.histogram(x.cuda(), chunk_bytes=cb).cpu().numpy()
        vb = {"bf16": 2, "fp32": 4, "fp8_e4m3": 1}[dt]
        m0 = cb // vb
        hb = _host_bytes(x)
        n = x.numel()
        for c in range(h.shape[0]):
            for e in range(h.shape[1]):
                ref = orc.histogram(dt, hb, c * m0, min(n, (c + 1) * m0), e)
                assert np.array_equal(h[c, e].astype(np.uint64), ref), (dt, c, e)


def test_code_lengths_entry_point(z, orc):
    rng = np.random.default_rng(3)
    hists = []
    for t in range(400):
        # the first half: alphabets of at most 32 symbols (the builder's register path)
        a = int(rng.integers(2, 33)) if t < 200 else int(rng.integers(2, 257))
        kind = t % 5
        f = np.zeros(256, dtype=np.int64)
        if kind == 0:
            f[:a] = rng.integers(0, 50, size=a)
        elif kind == 1:
            f[:a] = (1e9 * rng.random(a) ** 12).astype(np.int64)
        elif kind == 2:  # Fibonacci weights: the deepest possible trees
            a = min(a, 60)
            fib = [1, 1]
            while len(fib) < a:
                fib.append(fib[-1] + fib[-2])
            f[:a] = np.array(fib[:a], dtype=np.int64)[rng.permutation(a)]
        elif kind == 3:  # many ties
            f[:a] = rng.integers(1, 4, size=a)
        else:
            f[:a] = rng.integers(0, 2 ** 40, size=a)
        hists.append(f)
    H = torch.from_numpy(np.stack(hists)).cuda()
    got = z.code_lengths(H).cpu().numpy()
    for i, f in enumerate(hists):
        assert np.array_equal(got[i], orc.limited_lengths(f.astype(np.uint64))), i


def test_plan_parity(z, orc):
    from lossless_float_weight_b200 import workloads as W
    kv = W.kv_cache(shape=(2, 2, 4, 4, 4096, 128))  # 128 chunks
    plan = z.Plan.create(kv.cuda(), groups=8, seed=0)
    lens, assign, iters, _ = orc.plan_build("bf16", _host_bytes(kv), kv.numel(), CB, groups=8, seed=0)
    assert plan.assignment() == assign.tolist()
    exported = plan.export()
    # export = "ZNP1", dtype, groups, 2 zero bytes, 4-bit length records
    assert exported[:4] == b"ZNP1" and exported[4] == 0 and exported[5] == 8
    rec = np.frombuffer(exported[8:], dtype=np.uint8).reshape(8, 128)
    got_lens = np.zeros((8, 256), dtype=np.uint8)
    got_lens[:, 0::2] = rec & 15
    got_lens[:, 1::2] = rec >> 4
    assert np.array_equal(got_lens, lens[0])
    _check_roundtrip(z, orc, kv, "kv with plan", plan=plan, plan_lens=lens)
    # the plan applies to another tensor (reuse), and survives export/import
    other = W.kv_cache(shape=(1, 2, 4, 4, 4096, 128), seed=5)
    p2 = z.Plan.from_bytes(exported)
    _check_roundtrip(z, orc, other, "kv reuse", plan=p2, plan_lens=lens)


def test_plan_transfer_between_layers(z, orc):
    # a plan built on one checkpoint tensor codes another layer's tensor exactly as the oracle does
    from lossless_float_weight_b200 import workloads as W
    shapes = W.checkpoint_7b_shapes()
    sig = W.checkpoint_7b_sigmas(len(shapes))
    a = W.checkpoint_7b_tensor(0, shapes[0][1], sig[0], "cpu").reshape(-1)    # layer 0 q, 128 chunks
    b = W.checkpoint_7b_tensor(12, shapes[12][1], sig[12], "cpu").reshape(-1)  # layer 1 up projection
    plan = z.Plan.create(a.cuda(), groups=8, seed=0)
    lens, assign, _, _ = orc.plan_build("bf16", _host_bytes(a), a.numel(), CB, groups=8, seed=0)
    assert plan.assignment() == assign.tolist()
    _check_roundtrip(z, orc, b, "plan from another layer", plan=plan, plan_lens=lens)


def test_plan_fp8_and_small(z, orc):
    from lossless_float_weight_b200 import workloads as W
    q = W.fp8_tensor(rows=512, cols=4096)
    plan = z.Plan.create(q.cuda(), groups=4, seed=3, chunk_bytes=65536)
    lens, assign, _, _ = orc.plan_build("fp8_e4m3", _host_bytes(q), q.numel(), 65536, groups=4, seed=3)
    assert plan.assignment() == assign.tolist()
    _check_roundtrip(z, orc, q, "fp8 plan", chunk_bytes=65536, plan=plan, plan_lens=lens)
    x = W.bf16_small(n=300000)  # 3 chunks <= 8 groups: identity grouping
    plan = z.Plan.create(x.cuda(), groups=8)
    lens, assign, _, _ = orc.plan_build("bf16", _host_bytes(x), x.numel(), CB, groups=8, seed=0)
    assert plan.assignment() == [0, 1, 2]
    _check_roundtrip(z, orc, x, "bf16 identity plan", plan=plan, plan_lens=lens)


def test_plan_dtype_mismatch(z):
    from lossless_float_weight_b200 import workloads as W
    x = W.bf16_small(n=300000).cuda()
    plan = z.Plan.create(x, groups=2)
    f = torch.zeros(1000, dtype=torch.float32, device="cuda")
    with pytest.raises(z.ZipnnError) as ei:
        z.compress(f, plan=plan)
    assert ei.value.status == z.ERR_PLAN_MISMATCH


def test_corrupt_containers_report_status(z, orc):
    import struct
    from lossless_float_weight_b200 import workloads as W
    x = W.bf16_small(n=300000)
    c = z.compress(x.cuda()).cpu().numpy()
    off0 = struct.unpack_from("<Q", c, 64 + 8)[0]
    cases = []
    d = c.copy(); d[0] ^= 1; cases.append(d)
    cases.append(c[: c.size - 16].copy())
    d = c.copy(); struct.pack_into("<Q", d, 48, c.size + 16); cases.append(d)
    d = c.copy(); struct.pack_into("<Q", d, 64 + 16 + 8, 10 ** 9); cases.append(d)
    d = c.copy(); d[64] = 7; cases.append(d)
    d = c.copy(); d[off0 + 63] = 0xFF; cases.append(d)
    d = c.copy(); d[off0: off0 + 128] = 0x11; cases.append(d)
    d = c.copy(); struct.pack_into("<I", d, off0 + 128, 5); cases.append(d)
    d = c.copy(); struct.pack_into("<I", d, off0 + 128 + 4, 0x7FFFFFFF); cases.append(d)
    ws = torch.zeros(256, dtype=torch.uint8, device="cuda")
    out = torch.empty(300000, dtype=torch.bfloat16, device="cuda")
    for i, d in enumerate(cases):
        dd = torch.from_numpy(d).cuda()
        z.decompress_into(dd, dd.numel(), out, ws)
        assert z.status(ws) == z.ERR_CORRUPT, i
        assert orc.decompress_status("bf16", d, 300000) == orc.ECORRUPT, i
    # wrong n / dtype for a valid container
    cd = torch.from_numpy(c).cuda()
    z.decompress_into(cd, cd.numel(), out[:299999], ws)
    assert z.status(ws) == z.ERR_CORRUPT
    # random bit flips: either detected or decoded, never a fault
    rng = np.random.default_rng(4)
    for _ in range(30):
        d = c.copy()
        d[int(rng.integers(64, c.size))] ^= 1 << int(rng.integers(0, 8))
        dd = torch.from_numpy(d).cuda()
        z.decompress_into(dd, dd.numel(), out, ws)
        assert z.status(ws) in (z.OK, z.ERR_CORRUPT)
    torch.cuda.synchronize()


def test_argument_errors(z):
    x = torch.zeros(1000, dtype=torch.bfloat16, device="cuda")
    ws = z.workspace(z.BF16, 1000)
    out = torch.empty(100000, dtype=torch.uint8, device="cuda")
    with pytest.raises(z.ZipnnError) as ei:
        z.compress_into(x, out[:10], ws)
    assert ei.value.status == z.ERR_OUT_TOO_SMALL
    with pytest.raises(z.ZipnnError) as ei:
        z.compress_into(x, out, ws, chunk_bytes=100)
    assert ei.value.status == z.ERR_INVALID_ARG
    with pytest.raises(z.ZipnnError) as ei:
        z.compress_into(x[1:], out, ws)  # 2-byte aligned pointer
    assert ei.value.status == z.ERR_INVALID_ARG
    with pytest.raises(z.ZipnnError) as ei:
        z.compress_into(x, out, ws, subblock=24)
    assert ei.value.status == z.ERR_INVALID_ARG


def _pruned_bf16(rows, cols, seed, every=3):
    g = torch.Generator().manual_seed(seed)
    x = (torch.randn(rows, cols, generator=g) * 0.02).to(torch.bfloat16)
    x[torch.arange(rows) % every == 0] = 0  # pruned rows: runs of zero sign/fraction bytes
    return x.reshape(-1)


@pytest.mark.parametrize("chunk_bytes,subblock", [(262144, 512), (4096, 64), (1 << 20, 512), (65536, 16)])
def test_zero_runs_bf16(z, orc, chunk_bytes, subblock):
    """Pruned rows make ZRUN sign/fraction planes; 1 MiB chunks (16384 blocks) take the
    generic decode instead of the staged one. Ragged sizes end in a short block."""
    import container_util as CU
    for n_extra in (0, 77):
        x = torch.cat([_pruned_bf16(600, 1000, chunk_bytes), (torch.randn(n_extra) * 0.02).to(torch.bfloat16)])
        got = _check_roundtrip(z, orc, x, "bf16 pruned", chunk_bytes=chunk_bytes, subblock=subblock)
        h, mode, code, off, ends = CU.payload_spans(got)
        assert 3 in mode[1::2].tolist()


def test_zero_runs_fp32(z, orc):
    g = torch.Generator().manual_seed(21)
    y = (torch.randn(1 << 20, generator=g) * 0.02).float()
    clean = (torch.arange(1 << 20) // 96) % 3 == 0  # runs of clean values, not aligned to blocks
    y[clean] = y[clean].bfloat16().float()
    y[5000:9000] = 0
    got = _check_roundtrip(z, orc, y, "fp32 partly clean")
    import container_util as CU
    h, mode, code, off, ends = CU.payload_spans(got)
    assert 3 in mode.reshape(-1, 4)[:, 2].tolist() and 3 in mode.reshape(-1, 4)[:, 3].tolist()


def test_zero_runs_corrupt(z, orc):
    """A ZRUN bitmap that marks every block asks for more kept bytes than the payload holds:
    CORRUPT on the staged and on the generic path, never a fault."""
    import container_util as CU
    for cb in (262144, 1 << 20):
        x = _pruned_bf16(300, 1000, 5, every=2)
        c = z.compress(x.cuda(), chunk_bytes=cb).cpu().numpy()
        h, mode, code, off, ends = CU.payload_spans(c)
        k = [i for i in range(1, len(mode), 2) if mode[i] == 3][0]
        d = c.copy()
        d[off[k]: off[k] + 16] = 0xFF
        ws = torch.zeros(256, dtype=torch.uint8, device="cuda")
        out = torch.empty(x.numel(), dtype=torch.bfloat16, device="cuda")
        z.decompress_into(torch.from_numpy(d).cuda(), d.size, out, ws, chunk_bytes=cb)
        assert z.status(ws) == z.ERR_CORRUPT
        assert orc.decompress_status("bf16", d, x.numel(), chunk_bytes=cb) == orc.ECORRUPT


@pytest.mark.parametrize("name", ["bf16", "fp32", "fp8_e4m3"])
def test_input_16_byte_aligned_only(z, orc, name):
    """A tensor that starts 16 bytes past a 32-byte boundary (the encode then reads it with
    128-bit loads instead of 256-bit ones): the same container as the oracle's."""
    from lossless_float_weight_b200 import workloads as W
    g = torch.Generator().manual_seed(16)
    n = 131072 * 3 + 4096
    if name == "bf16":
        x = (torch.randn(n + 8, generator=g) * 0.02).to(torch.bfloat16)
        shift = 8
    elif name == "fp32":
        x = (torch.randn(n + 4, generator=g) * 0.02).float()
        shift = 4
    else:
        x = W.fp8_tensor(rows=(n + 4096) // 4096, cols=4096, seed=16).reshape(-1)
        shift = 16
    base = x.cuda()
    assert base.data_ptr() % 32 == 0
    xd = base[shift:shift + n]
    assert xd.data_ptr() % 32 == 16
    cont = z.compress(xd).cpu().numpy()
    ref = orc.compress(name, _host_bytes(x[shift:shift + n]), n, chunk_bytes=CB, S=S_DEFAULT, threads=8)
    assert np.array_equal(cont, ref)
    y = z.decompress(torch.from_numpy(ref).cuda(), x.dtype, n)
    assert torch.equal(y.view(torch.uint8).cpu(), torch.from_numpy(_host_bytes(x[shift:shift + n]).copy()))


@pytest.mark.parametrize("dtype", ["fp8_e4m3", "fp4_e2m1"])
def test_sub_byte_stream_modes(z, orc, dtype):
    """FP8 and FP4 chunks whose mantissa or sign stream is ZERO (non-negative values;
    values with a zero mantissa), whose counts end inside a 32-value step, and whose
    sub-block size is not a multiple of 32 (the decode's other path): every container the
    oracle's, every decode exact."""
    from lossless_float_weight_b200 import workloads as W
    if dtype == "fp8_e4m3":
        q = W.fp8_tensor(rows=80, cols=4096, seed=5).reshape(-1)
        b = q.view(torch.uint8)
        cases = {"no sign": (b & 0x7F), "no mantissa": (b & 0xF8), "neither": (b & 0x78), "as is": b}
        mk = lambda t: t.contiguous().view(torch.float8_e4m3fn)
    else:
        q = W.fp4_tensor(rows=80, cols=2048, seed=5).reshape(-1)
        b = q.view(torch.uint8)
        cases = {"no sign": (b & 0x77), "no mantissa": (b & 0xEE), "neither": (b & 0x66), "as is": b}
        mk = lambda t: t.contiguous().view(torch.float4_e2m1fn_x2)
    for name, t in cases.items():
        x = mk(t)
        _check_roundtrip(z, orc, x, f"{dtype} {name}", chunk_bytes=65536)
        cut = mk(t[: t.numel() - 2 * 37])  # counts that end inside a step
        _check_roundtrip(z, orc, cut, f"{dtype} {name} ragged", chunk_bytes=65536, subblock=512)
        _check_roundtrip(z, orc, cut, f"{dtype} {name} S=48", chunk_bytes=65536, subblock=48)


def test_fp4_plan_with_long_exponent_codes(z, orc):
    """An FP4 plan whose exponent code has a 12-bit length (a valid prefix code, though no
    Huffman code of four symbols has one): a 12-bit window then need not hold four whole
    codes, so the decode takes its two-symbol table. The plan is written by hand as the
    export format ("ZNP1", dtype, groups, two zero bytes, then the records: 4-bit lengths,
    two symbols a byte, 16 bytes a record)."""
    import struct
    lens_e, lens_m = [1, 2, 3, 12], [1, 1]
    rec_e = bytes([lens_e[0] | lens_e[1] << 4, lens_e[2] | lens_e[3] << 4]) + bytes(14)
    rec_m = bytes([lens_m[0] | lens_m[1] << 4]) + bytes(15)
    blob = b"ZNP1" + struct.pack("<BBH", z.FP4_E2M1, 1, 0) + rec_e + rec_m
    plan = z.Plan.from_bytes(blob)
    plan_lens = np.zeros((2, 1, 256), dtype=np.uint8)
    plan_lens[0, 0, :4] = lens_e
    plan_lens[1, 0, :2] = lens_m
    # exponents mostly 0 and 1, one in a thousand 3: the plan's code beats RAW
    rng = np.random.default_rng(44)
    n = 700000
    e = rng.choice(4, size=n, p=[0.6, 0.3, 0.099, 0.001]).astype(np.uint8)
    nib = (e << 1) | rng.integers(0, 2, n, dtype=np.uint8) | (rng.integers(0, 2, n, dtype=np.uint8) << 3)
    q = _fp4((nib[0::2] | (nib[1::2] << 4)).astype(np.uint8))
    c = _check_roundtrip(z, orc, q, "fp4 long exponent code", chunk_bytes=65536, plan=plan, plan_lens=plan_lens)
    assert c.size < 0.95 * (n // 2)  # the exponent stream is coded

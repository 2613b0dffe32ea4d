"""Parity at the full sizes of the five workloads (B200 only).

The oracle cannot compress 13 GB in a test, so at full size the checks are:
  * every chunk payload of a sample of chunks equals, byte for byte, the oracle's
    container for that chunk alone (payload bytes do not depend on their offset);
  * the chunk table is a valid layout (offsets are the running sum, in order);
  * decompress(compress(x)) == x for every tensor (a property at any size);
  * the grouping plan of the K/V cache equals the oracle's (assignment and group codes).
Workloads: the 7B-shaped BF16 checkpoint (per-tensor calls, as the benchmark times),
FP32 268,435,456 values and its clean variant, FP8 E4M3 262,144 x 4096, and the BF16
K/V cache [32, 2, 16, 8, 4096, 128] with an 8-group plan.
"""
import numpy as np
import pytest
import torch

import container_util as CU

pytestmark = pytest.mark.gpu

CB = 262144
S = 512


@pytest.fixture(scope="module")
def z():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from lossless_float_weight_b200 import zipnn
    return zipnn


NAMES = {torch.bfloat16: "bf16", torch.float32: "fp32", torch.float8_e4m3fn: "fp8_e4m3"}
VB = {"bf16": 2, "fp32": 4, "fp8_e4m3": 1}


def _check(z, orc, x, sample, plan=None, plan_lens=None, rng=None):
    """Compress x (device) with the library; compare sampled chunks with the oracle;
    check the layout and the round trip. Returns the container size."""
    dtype = NAMES[x.dtype]
    xf = x.reshape(-1)
    n = xf.numel()
    cont = z.compress(xf, chunk_bytes=CB, plan=plan)
    host = cont.cpu().numpy()
    h, mode, code, off, ends = CU.payload_spans(host)
    ns = h["n_streams"]
    m0 = CB // VB[dtype]
    assert h["n"] == n and h["n_chunks"] == -(-n // m0) and h["S"] == S
    # layout: offsets are the running sum of the payload sizes, in entry order
    assert off[0] == h["off_payload"] and np.all(np.diff(off) >= 0) and h["total_bytes"] == host.size
    assert np.all(off % 16 == 0)
    C = h["n_chunks"]
    picks = sorted(set([0, C - 1] + [int(c) for c in rng.integers(0, C, size=sample)]))
    for c in picks:
        lo, hi = c * m0, min(n, (c + 1) * m0)
        part = xf[lo:hi].contiguous().cpu().view(torch.uint8).numpy()
        ref = orc.compress(dtype, part, hi - lo, chunk_bytes=CB, S=S, plan_lens=plan_lens)
        rh, rmode, rcode, roff, rends = CU.payload_spans(ref)
        for s in range(ns):
            k = c * ns + s
            assert mode[k] == rmode[s] and code[k] == rcode[s], (c, s)
            got = host[off[k]: ends[k]]
            exp = ref[roff[s]: rends[s]]
            assert got.size == exp.size and np.array_equal(got, exp), (c, s)
    y = z.decompress(cont, x.dtype, n, chunk_bytes=CB)
    assert torch.equal(y.view(torch.uint8), xf.view(torch.uint8))
    return host.size


def test_checkpoint_7b_full(z, orc):
    from lossless_float_weight_b200 import workloads as W
    rng = np.random.default_rng(0)
    shapes = W.checkpoint_7b_shapes()
    sig = W.checkpoint_7b_sigmas(len(shapes))
    total_in = total_out = 0
    for t, (name, shape) in enumerate(shapes):
        x = W.checkpoint_7b_tensor(t, shape, sig[t], "cuda")
        total_out += _check(z, orc, x, sample=2 if t < 224 else 6, rng=rng)
        total_in += x.numel() * 2
        del x
    assert total_in == 13214154752
    assert 0.64 <= total_out / total_in <= 0.68


def test_fp32_full(z, orc):
    from lossless_float_weight_b200 import workloads as W
    rng = np.random.default_rng(1)
    x = W.fp32_tensor(n=268435456, device="cuda")
    r = _check(z, orc, x, sample=6, rng=rng) / (4 * x.numel())
    assert 0.82 <= r <= 0.85
    xc = x.to(torch.bfloat16).to(torch.float32)
    del x
    r = _check(z, orc, xc, sample=6, rng=rng) / (4 * xc.numel())
    assert r < 0.35


def test_fp8_full(z, orc):
    from lossless_float_weight_b200 import workloads as W
    rng = np.random.default_rng(2)
    q = W.fp8_tensor(rows=262144, cols=4096, device="cuda")
    r = _check(z, orc, q, sample=6, rng=rng) / q.numel()
    assert r < 0.9


def test_kv_cache_plan_full(z, orc):
    from lossless_float_weight_b200 import workloads as W
    rng = np.random.default_rng(3)
    kv = W.kv_cache(device="cuda")
    assert kv.numel() * 2 == 8589934592
    plan = z.Plan.create(kv, groups=8, seed=0, chunk_bytes=CB)
    host = kv.cpu()
    lens, assign, iters, _ = orc.plan_build("bf16", host.view(torch.uint8).numpy(), kv.numel(), CB, groups=8, seed=0)
    del host
    assert plan.assignment() == assign.tolist()
    rec = np.frombuffer(plan.export()[8:], dtype=np.uint8).reshape(8, 128)
    got = np.zeros((8, 256), dtype=np.uint8)
    got[:, 0::2] = rec & 15
    got[:, 1::2] = rec >> 4
    assert np.array_equal(got, lens[0])
    _check(z, orc, kv, sample=6, plan=plan, plan_lens=lens, rng=rng)

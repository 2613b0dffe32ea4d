"""Parity at the full sizes of the five workloads (B200 only).

Every container the library writes at full size is compared, byte for byte, with the
oracle's container for the same tensor (the oracle runs chunk-parallel on all host
cores), and decompress(compress(x)) == x is checked on the device. Workloads: the
7B-shaped BF16 checkpoint (225 tensors, one call each, as the benchmark makes them), FP32
268,435,456 values and its clean variant, FP8 E4M3 262,144 x 4096, FP4 E2M1 at the FP8
shape, and the BF16 K/V cache [32, 2, 16, 8, 4096, 128] with an 8-group plan (whose
grouping and group codes are compared with the oracle's first).
"""
import os

import numpy as np
import pytest
import torch

import container_util as CU

pytestmark = pytest.mark.gpu

CB = 262144
S = 512
THREADS = os.cpu_count() or 1


@pytest.fixture(scope="module")
def z():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from lossless_float_weight_b200 import zipnn
    return zipnn


NAMES = {torch.bfloat16: "bf16", torch.float32: "fp32", torch.float8_e4m3fn: "fp8_e4m3",
         torch.float4_e2m1fn_x2: "fp4_e2m1"}


def _check(z, orc, x, plan=None, plan_lens=None):
    """Compress x (device) with the library and with the oracle; the two containers must be
    equal byte for byte; the library's decompress must give x back. Returns the size."""
    dtype = NAMES[x.dtype]
    xf = x.reshape(-1)
    n = z.nvalues(xf)
    cont = z.compress(xf, chunk_bytes=CB, plan=plan)
    host = cont.cpu().numpy()
    h = CU.header(host)
    assert h["n"] == n and h["S"] == S and h["total_bytes"] == host.size
    ref = orc.compress(dtype, xf.cpu(), n, chunk_bytes=CB, S=S, plan_lens=plan_lens, threads=THREADS)
    assert ref.size == host.size, (ref.size, host.size)
    if not np.array_equal(host, ref):
        bad = np.nonzero(host != ref)[0]
        raise AssertionError(f"{bad.size} bytes differ, the first at {bad[:8]}")
    del ref
    y = z.decompress(cont, x.dtype, xf.numel(), chunk_bytes=CB)
    assert torch.equal(y.view(torch.uint8), xf.view(torch.uint8))
    return host.size


def test_checkpoint_7b_full(z, orc):
    from lossless_float_weight_b200 import workloads as W
    shapes = W.checkpoint_7b_shapes()
    sig = W.checkpoint_7b_sigmas(len(shapes))
    total_in = total_out = 0
    for t, (name, shape) in enumerate(shapes):
        x = W.checkpoint_7b_tensor(t, shape, sig[t], "cuda")
        total_out += _check(z, orc, x)
        total_in += x.numel() * 2
        del x
    assert total_in == 13214154752
    assert 0.64 <= total_out / total_in <= 0.68


def test_fp32_full(z, orc):
    from lossless_float_weight_b200 import workloads as W
    x = W.fp32_tensor(n=268435456, device="cuda")
    r = _check(z, orc, x) / (4 * x.numel())
    assert 0.82 <= r <= 0.85
    xc = x.to(torch.bfloat16).to(torch.float32)
    del x
    r = _check(z, orc, xc) / (4 * xc.numel())
    assert r < 0.35


def test_fp8_full(z, orc):
    from lossless_float_weight_b200 import workloads as W
    q = W.fp8_tensor(rows=262144, cols=4096, device="cuda")
    r = _check(z, orc, q) / q.numel()
    assert r < 0.9


def test_fp4_full(z, orc):
    from lossless_float_weight_b200 import workloads as W
    q = W.fp4_tensor(rows=262144, cols=4096, device="cuda")
    r = _check(z, orc, q) / q.numel()
    assert r < 1.0


def test_kv_cache_plan_full(z, orc):
    from lossless_float_weight_b200 import workloads as W
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
    r = _check(z, orc, kv, plan=plan, plan_lens=lens) / (2 * kv.numel())
    assert r < 0.8

"""Limits of the CUDA path (B200 only): the code builder on counts across the whole 64-bit
range, and the decoupled look-back's bounded wait made to run out on a healthy launch."""
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


def test_code_lengths_on_64bit_counts(z, orc):
    """Counts at and above 2^56 (where a packed (count << 8 | symbol) key would overflow)
    give the oracle's lengths; each histogram's total stays below 2^64."""
    rng = np.random.default_rng(11)
    hists = []
    for t in range(120):
        a = int(rng.integers(2, 33)) if t < 60 else int(rng.integers(33, 257))
        f = np.zeros(256, dtype=np.uint64)
        kind = t % 4
        if kind == 0:    # every count in [2^56, 2^57): ties in the top bits, order from the low ones
            f[:a] = (np.uint64(1) << np.uint64(56)) + rng.integers(0, 1 << 20, size=a).astype(np.uint64)
        elif kind == 1:  # huge and tiny counts together, total below 2^63
            f[:a] = rng.integers(1, 1000, size=a).astype(np.uint64)
            f[int(rng.integers(0, a))] = np.uint64((1 << 62) + int(rng.integers(0, 1 << 40)))
        elif kind == 2:  # equal huge counts: the symbol decides every tie
            f[:a] = np.uint64(1 << 57)
        else:            # counts spread over [2^50, 2^58)
            f[:a] = (2.0 ** rng.uniform(50, 58, size=a)).astype(np.uint64)
        hists.append(f)
    H = torch.from_numpy(np.stack(hists).view(np.int64)).cuda()
    got = z.code_lengths(H).cpu().numpy()
    for i, f in enumerate(hists):
        assert np.array_equal(got[i], orc.limited_lengths(f)), i


def _many_tiles(dtype):
    g = torch.Generator().manual_seed(5)
    x = torch.randn(3 * 1000 * 1024, generator=g) * 0.02
    return x.to(dtype)


@pytest.mark.parametrize("dtype,chunk_bytes", [(torch.bfloat16, 4096), (torch.float32, 4096)])
def test_lookback_wait_runs_out(z, orc, dtype, chunk_bytes):
    """With a look-back limit of one poll, a wait whose predecessor has not published yet
    gives up: the call ends, the status is OK or TIMEOUT (never a fault), every write stays
    inside the output (a guard band after it stays untouched), and the process goes on.
    With 4 KiB chunks, BF16 has 3000 chunk-table entries (three layout tiles that wait on
    each other) and FP32 12000 (twelve)."""
    name = {torch.bfloat16: "bf16", torch.float32: "fp32"}[dtype]
    x = _many_tiles(dtype).cuda()
    n = x.numel()
    cap = z.zipnn_max_compressed_bytes(z.dtype_code(dtype), n, chunk_bytes)
    guard = 1 << 16
    out = torch.full((cap + guard,), 0xA5, dtype=torch.uint8, device="cuda")
    ws = z.workspace(z.dtype_code(dtype), n, chunk_bytes)
    statuses = set()
    try:
        z.zipnn_test_lookback_limit(1)
        for _ in range(5):
            z.compress_into(x, out[:cap], ws, chunk_bytes)
            statuses.add(z.status(ws))
    finally:
        z.zipnn_test_lookback_limit(0)
    assert statuses <= {z.OK, z.ERR_TIMEOUT}, statuses
    assert bool((out[cap:] == 0xA5).all())
    # the default limit again: the same call is exact
    z.compress_into(x, out[:cap], ws, chunk_bytes)
    assert z.status(ws) == z.OK
    size = z.compressed_size(out)
    ref = orc.compress(name, x.cpu(), n, chunk_bytes=chunk_bytes, S=512, threads=8)
    assert size == ref.size and np.array_equal(out[:size].cpu().numpy(), ref)

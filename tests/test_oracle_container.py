"""Pins for the oracle's container: hand-derived golden bytes, round trips over every
bit pattern, and corruption handling (CPU only)."""
import struct

import numpy as np
import pytest
import torch

import golden_util as GU


def test_golden_three_chunks(orc):
    fx = GU.load("bf16_three_chunks.json")
    x = GU.three_chunk_input()
    got = orc.compress("bf16", x, chunk_bytes=fx["input"]["chunk_bytes"], S=fx["input"]["S"])
    exp = GU.expected_bytes(fx)
    assert got.size == exp.size
    bad = np.nonzero(got != exp)[0]
    assert bad.size == 0, f"first differing byte {bad[:8]}"
    y = orc.decompress("bf16", got, 517, chunk_bytes=512)
    assert np.array_equal(y, x.view(torch.uint8).numpy())


def test_golden_shared_code(orc):
    fx = GU.load("bf16_shared_code.json")
    x = GU.three_chunk_input()
    got = orc.compress("bf16", x, chunk_bytes=512, S=64, plan_lens=GU.plan_lens(fx))
    exp = GU.expected_bytes(fx)
    assert got.size == exp.size
    assert np.array_equal(got, exp), np.nonzero(got != exp)[0][:8]
    y = orc.decompress("bf16", got, 517, chunk_bytes=512)
    assert np.array_equal(y, x.view(torch.uint8).numpy())


def _roundtrip(orc, dtype, x, chunk_bytes, S=1024, threads=1):
    raw = orc._bytes_view(x)
    n = orc.values_in(dtype, raw.size)
    c = orc.compress(dtype, raw, n, chunk_bytes=chunk_bytes, S=S, threads=threads)
    assert c.size <= orc.max_compressed_bytes(dtype, n, chunk_bytes)
    assert c.size % 16 == 0
    y = orc.decompress(dtype, c, n, chunk_bytes=chunk_bytes, threads=threads)
    assert np.array_equal(y, raw)
    return c


def test_every_bf16_bit_pattern(orc):
    pats = np.arange(65536, dtype=np.uint16)
    rng = np.random.default_rng(0)
    _roundtrip(orc, "bf16", pats, 4096)                 # in order: exponent runs
    _roundtrip(orc, "bf16", rng.permutation(pats), 4096, S=64)  # shuffled
    _roundtrip(orc, "bf16", pats, 131072)               # a single chunk


def test_every_fp8_bit_pattern(orc):
    pats = np.arange(256, dtype=np.uint8)
    rng = np.random.default_rng(1)
    _roundtrip(orc, "fp8_e4m3", np.tile(pats, 64), 4096)
    _roundtrip(orc, "fp8_e4m3", rng.permutation(np.tile(pats, 300)), 4096, S=128)


def test_fp32_special_values(orc):
    rng = np.random.default_rng(2)
    specials = np.array([0.0, -0.0, np.inf, -np.inf, np.nan, 1e-45, -1e-45, 1.17549435e-38,
                         3.4028235e38, -3.4028235e38, 1.0, -1.0], dtype=np.float32)
    bits = rng.integers(0, 2 ** 32, size=50000, dtype=np.uint64).astype(np.uint32)
    x = np.concatenate([specials.view(np.uint32), bits, np.full(7, 0x7FC00001, np.uint32)])
    _roundtrip(orc, "fp32", x, 4096)
    _roundtrip(orc, "fp32", x, 1 << 20)


def test_edge_sizes_and_constant_tensors(orc):
    for n in (1, 2, 7, 8, 9, 1023, 1024, 1025, 131071, 131073):
        x = (torch.randn(n, generator=torch.Generator().manual_seed(n)) * 0.02).to(torch.bfloat16)
        _roundtrip(orc, "bf16", x, 262144)
        _roundtrip(orc, "bf16", x, 16, S=16)
    zeros = torch.zeros(300000, dtype=torch.bfloat16)
    c = _roundtrip(orc, "bf16", zeros, 262144)
    assert c.size == 64 + 16 * 2 * 3  # header and table only: every entry is ZERO
    ones = torch.ones(300000, dtype=torch.bfloat16)
    c = _roundtrip(orc, "bf16", ones, 262144)
    # exponent 127 everywhere: one symbol, one bit each, well below RAW
    assert c[64] == 2
    _roundtrip(orc, "fp32", torch.zeros(5000), 4096)
    _roundtrip(orc, "fp8_e4m3", torch.zeros(5000, dtype=torch.uint8), 4096)


def test_thread_count_does_not_change_bytes(orc):
    from lossless_float_weight_b200 import workloads as W
    x = W.bf16_small()
    a = orc.compress("bf16", x, threads=1)
    b = orc.compress("bf16", x, threads=5)
    assert np.array_equal(a, b)


def _corrupt_cases(c):
    cases = []
    # bad magic
    d = c.copy(); d[0] ^= 1; cases.append(("magic", d))
    # truncated container
    cases.append(("truncated", c[: c.size - 16].copy()))
    # total_bytes beyond the buffer
    d = c.copy(); struct.pack_into("<Q", d, 48, c.size + 16); cases.append(("total", d))
    # entry offset out of order
    d = c.copy(); struct.pack_into("<Q", d, 64 + 16 + 8, 10 ** 9); cases.append(("offset", d))
    # bad mode
    d = c.copy(); d[64] = 7; cases.append(("mode", d))
    # length record with a length above 12 (local code of chunk 0)
    off0 = struct.unpack_from("<Q", c, 64 + 8)[0]
    d = c.copy(); d[off0 + 63] = 0xFF; cases.append(("length>12", d))
    # length record that breaks the Kraft inequality: make every symbol length 1
    d = c.copy(); d[off0: off0 + 128] = 0x11; cases.append(("kraft", d))
    # sub-block index not starting at 0
    d = c.copy(); struct.pack_into("<I", d, off0 + 128, 5); cases.append(("idx0", d))
    # sub-block index beyond the bitstream
    d = c.copy(); struct.pack_into("<I", d, off0 + 128 + 4, 0x7FFFFFFF); cases.append(("idx", d))
    return cases


def test_corruption_is_reported(orc):
    from lossless_float_weight_b200 import workloads as W
    x = W.bf16_small(n=300000)
    c = orc.compress("bf16", x)
    assert c[64] == 2  # chunk 0 exponent stream is HUFF
    for name, d in _corrupt_cases(c):
        st = orc.decompress_status("bf16", d, 300000)
        assert st == orc.ECORRUPT, name
    # header / argument mismatch
    assert orc.decompress_status("bf16", c, 299999) == orc.ECORRUPT
    assert orc.decompress_status("fp32", c, 150000) == orc.ECORRUPT
    # flipped bits inside the bitstream either fail the index check or decode to
    # different values, never crash
    rng = np.random.default_rng(3)
    off0 = struct.unpack_from("<Q", c, 64 + 8)[0]
    for _ in range(20):
        d = c.copy()
        d[off0 + 128 + 512 + int(rng.integers(0, 20000))] ^= 1 << int(rng.integers(0, 8))
        assert orc.decompress_status("bf16", d, 300000) in (orc.OK, orc.ECORRUPT)


# Hand-derived containers of the other dtypes: FP8 (a HUFF exponent and a HUFF mantissa,
# 3-bit and 1-bit RAW packing, a 4-bit RAW exponent, a ragged chunk), the same FP8 input
# with a two-group plan (shared records of both entropy streams), a clean FP32 tensor
# (ZERO low fraction planes) and FP4 (2-bit and 1-bit packing).
GOLDEN_OTHER = [
    ("fp8_two_chunks.json", "fp8_e4m3", GU.fp8_two_chunk_input, False),
    ("fp8_shared_code.json", "fp8_e4m3", GU.fp8_two_chunk_input, True),
    ("fp32_clean_two_chunks.json", "fp32", GU.fp32_clean_two_chunk_input, False),
    ("fp4_two_chunks.json", "fp4_e2m1", GU.fp4_two_chunk_input, False),
    ("bf16_zero_runs.json", "bf16", GU.zero_runs_input, False),
]


@pytest.mark.parametrize("name,dtype,make,with_plan", GOLDEN_OTHER)
def test_golden_other_dtypes(orc, name, dtype, make, with_plan):
    fx = GU.load(name)
    src = GU.load(fx["input"]["same_as"]) if "same_as" in fx["input"] else fx
    x = make()
    n = src["input"]["n"]
    got = orc.compress(dtype, x, n, chunk_bytes=src["input"]["chunk_bytes"], S=src["input"]["S"],
                       plan_lens=GU.plan_lens(fx) if with_plan else None)
    exp = GU.expected_bytes(fx)
    assert got.size == exp.size, (got.size, exp.size)
    bad = np.nonzero(got != exp)[0]
    assert bad.size == 0, f"first differing bytes at {bad[:8]}"
    y = orc.decompress(dtype, got, n, chunk_bytes=src["input"]["chunk_bytes"])
    assert np.array_equal(y, orc._bytes_view(x))


def _entry_modes(c):
    import container_util as CU
    h, mode, code, off, ends = CU.payload_spans(c)
    return h, mode, off, ends


def test_zero_runs_round_trip_and_choice(orc):
    """Byte planes with zeroed blocks take ZRUN exactly when it is strictly smaller than
    RAW; the exponent (an entropy stream) never does; every case round-trips."""
    g = torch.Generator().manual_seed(12)
    # BF16 rows of 256 values; some rows zeroed (pruned), so whole 32-value blocks are zero
    x = (torch.randn(64, 256, generator=g) * 0.02).to(torch.bfloat16)
    x[torch.arange(64) % 3 == 0] = 0
    c = _roundtrip(orc, "bf16", x.reshape(-1), 4096, S=64)
    h, mode, off, ends = _entry_modes(c)
    assert set(mode[1::2].tolist()) == {3}         # every sign/fraction plane: ZRUN
    assert 3 not in mode[0::2].tolist()            # exponent: HUFF or RAW
    # the ZRUN payload: bitmap of 2048/32 = 64 blocks (16 bytes) + kept bytes
    for k in range(1, len(mode), 2):
        assert ends[k] - off[k] < 2048              # smaller than RAW
    # FP32 where every other 32-value block is clean: the two low planes keep half their
    # blocks (whole clean chunks would be ZERO instead)
    y = (torch.randn(1 << 16, generator=g) * 0.02).float()
    clean = (torch.arange(1 << 16) // 32) % 2 == 0
    y[clean] = y[clean].bfloat16().float()
    c = _roundtrip(orc, "fp32", y, 1 << 16)
    h, mode, off, ends = _entry_modes(c)
    assert mode.reshape(-1, 4)[:, 2:].tolist() == [[3, 3]] * 4
    # a plane with no zero block stays RAW; all zero stays ZERO
    z = (torch.randn(4096, generator=g) * 0.02).to(torch.bfloat16)
    c = _roundtrip(orc, "bf16", z, 8192)
    assert _entry_modes(c)[1][1] == 0
    c = _roundtrip(orc, "bf16", torch.zeros(4096, dtype=torch.bfloat16), 8192)
    assert _entry_modes(c)[1].tolist() == [1, 1]


def test_zero_runs_break_even(orc):
    """ZRUN costs a 16-byte bitmap (padded) for a 4096-byte plane of 128 blocks; one zero
    block saves 32 bytes but the kept bytes pad to 16 again: 16 + 4064 = 4080 < 4096, so
    one zero block already makes ZRUN; the RAW tie (never here) would keep RAW."""
    g = torch.Generator().manual_seed(13)
    x = (torch.randn(4096, generator=g) * 0.02).to(torch.bfloat16)
    x[:32] = 0
    c = _roundtrip(orc, "bf16", x, 8192)
    h, mode, off, ends = _entry_modes(c)
    assert mode[1] == 3 and ends[1] - off[1] == 16 + 4064


def test_zero_runs_corruption(orc):
    import container_util as CU
    g = torch.Generator().manual_seed(14)
    x = (torch.randn(4096, generator=g) * 0.02).to(torch.bfloat16)
    x[:1024] = 0
    c = orc.compress("bf16", x, 4096, chunk_bytes=8192, S=64)
    h, mode, off, ends = _entry_modes(c)
    assert mode[1] == 3
    d = c.copy(); d[64] = 3                           # ZRUN on the exponent (entropy) stream
    assert orc.decompress_status("bf16", d, 4096, chunk_bytes=8192) == orc.ECORRUPT
    d = c.copy(); d[off[1]: off[1] + 16] = 0xFF        # every block marked: data too short
    assert orc.decompress_status("bf16", d, 4096, chunk_bytes=8192) == orc.ECORRUPT

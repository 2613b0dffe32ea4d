"""Pins for the oracle's FP4 (E2M1) support (CPU only).

"Lossless Compression of Neural Network Components: Weights, Checkpoints, and K/V
Caches in Low-Precision Formats" (abstract) extends the exponent/mantissa split to FP4.
Reading: a byte holds two E2M1 values, value 2i in its low nibble and 2i+1 in its high
nibble; a nibble is sign (bit 3), exponent (bits 2..1), mantissa (bit 0); the streams
are [exponent, mantissa, sign], exponent and mantissa entropy-coded independently."""
import numpy as np
import pytest

# E2M1 magnitudes by (exponent, mantissa): exponent 0 is subnormal (m * 0.5), else
# (1 + m / 2) * 2^(e - 1)
E2M1 = {(0, 0): 0.0, (0, 1): 0.5, (1, 0): 1.0, (1, 1): 1.5, (2, 0): 2.0, (2, 1): 3.0, (3, 0): 4.0, (3, 1): 6.0}


def _fields(orc, byte):
    b = np.array([byte], dtype=np.uint8)
    out = []
    for s in range(3):
        h = orc.histogram("fp4_e2m1", b, 0, 2, s)
        out.append(h)
    return out


def test_field_split_of_a_hand_worked_byte(orc):
    # 0xB5 = 1011 0101: value 0 = 0101 (+, e 2, m 1 = 3.0), value 1 = 1011 (-, e 1, m 1 = -1.5)
    he, hm, hs = _fields(orc, 0xB5)
    assert he[:4].tolist() == [0, 1, 1, 0]
    assert hm[:2].tolist() == [0, 2]
    assert hs[:2].tolist() == [1, 1]
    assert E2M1[(2, 1)] == 3.0 and E2M1[(1, 1)] == 1.5


def test_nibble_fields_match_the_e2m1_value_table(orc):
    # every nibble: its fields are (sign, exponent, mantissa) of the E2M1 value it encodes
    table = [0.0, 0.5, 1.0, 1.5, 2.0, 3.0, 4.0, 6.0]
    for nib in range(16):
        he, hm, hs = _fields(orc, nib | (nib << 4))  # both values the same nibble
        e, m, s = int(np.argmax(he)), int(np.argmax(hm)), int(np.argmax(hs))
        assert he[e] == 2 and hm[m] == 2 and hs[s] == 2
        assert (-1) ** s * E2M1[(e, m)] == (-1 if nib & 8 else 1) * table[nib & 7]


def _roundtrip(orc, raw, chunk_bytes, S=512, threads=1):
    n = orc.values_in("fp4_e2m1", raw.size)
    c = orc.compress("fp4_e2m1", raw, n, chunk_bytes=chunk_bytes, S=S, threads=threads)
    assert c.size <= orc.max_compressed_bytes("fp4_e2m1", n, chunk_bytes) and c.size % 16 == 0
    assert c[6] == 3 and c[7] == 3  # dtype FP4, three streams
    y = orc.decompress("fp4_e2m1", c, n, chunk_bytes=chunk_bytes, threads=threads)
    assert np.array_equal(y, raw)
    return c


def test_every_fp4_byte_pattern(orc):
    pats = np.arange(256, dtype=np.uint8)
    rng = np.random.default_rng(4)
    _roundtrip(orc, np.tile(pats, 64), 4096)
    _roundtrip(orc, rng.permutation(np.tile(pats, 300)), 4096, S=128)
    _roundtrip(orc, rng.permutation(np.tile(pats, 1000)), 65536, threads=4)


def test_ragged_sizes_and_odd_counts(orc):
    rng = np.random.default_rng(5)
    for nbytes in (1, 2, 9, 2047, 2048, 2049, 100001):
        raw = rng.integers(0, 256, size=nbytes, dtype=np.uint8)
        _roundtrip(orc, raw, 2048, S=64)
    with pytest.raises(orc.OracleError):  # values come in byte pairs
        orc.compress("fp4_e2m1", np.zeros(4, dtype=np.uint8), 7, chunk_bytes=2048)


def test_quantised_gaussian_compresses(orc):
    # as the FP8 workload: N(0, 1) times a per-row scale (rows of 4096, log-uniform in
    # [0.25, 4]), rounded to the nearest E2M1 value (ties to the smaller magnitude), saturating at 6
    rng = np.random.default_rng(6)
    rows = 256
    scale = np.exp(rng.uniform(np.log(0.25), np.log(4.0), size=rows))
    x = (rng.standard_normal((rows, 4096)) * scale[:, None]).reshape(-1)
    grid = np.array([0.0, 0.5, 1.0, 1.5, 2.0, 3.0, 4.0, 6.0])
    code = np.abs(np.abs(x)[:, None] - grid[None, :]).argmin(axis=1) | ((x < 0) << 3)
    raw = (code[0::2] | (code[1::2] << 4)).astype(np.uint8)
    c = _roundtrip(orc, raw, 262144)
    # the exponent plane is skewed, so the container is smaller than the input
    assert c.size < 0.95 * raw.size


def test_plan_with_two_entropy_streams(orc):
    # a plan holds one code per group for the exponent and one for the mantissa
    rng = np.random.default_rng(8)
    raw = rng.choice(np.array([0x10, 0x21, 0x32, 0x05, 0x13, 0x20], dtype=np.uint8), size=1 << 18)
    n = orc.values_in("fp4_e2m1", raw.size)
    lens, assign, iters, _ = orc.plan_build("fp4_e2m1", raw, n, 16384, groups=3, seed=0)
    assert lens.shape == (2, 3, 256) and assign.size == 16 and iters >= 1
    assert np.all(lens[0, :, 4:] == 0) and np.all(lens[1, :, 2:] == 0)  # alphabets of 4 and 2
    c = orc.compress("fp4_e2m1", raw, n, chunk_bytes=16384, plan_lens=lens)
    assert np.array_equal(orc.decompress("fp4_e2m1", c, n, chunk_bytes=16384), raw)

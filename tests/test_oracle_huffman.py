"""Pins for the oracle's code construction (CPU only).

What pins it, other than itself:
  * hand-worked tie-break vectors (reading: ties by (weight, order), leaves before merged
    nodes), with the canonical code values of RFC 1951 section 3.2.2 worked by hand;
  * brute force over every complete prefix code on alphabets of at most 8 symbols;
  * the Kraft equality and the textbook entropy bound H <= L < H + 1 (the THEORY-599
    note, "Implied entropy", leans on the same bound);
  * a hand-worked run of the length limiter.
"""
import itertools
import math

import numpy as np
import pytest


def kraft(lens):
    return sum(2.0 ** -int(x) for x in lens if x)


def test_tie_break_hand_worked(orc):
    # {0:1, 1:1, 2:2}: merge 0 and 1 (order 0 < 1), then symbol 2 with the merged node.
    assert list(orc.huffman_lengths([1, 1, 2])) == [2, 2, 1]
    # four equal weights: 0+1, then 2+3 (leaves before the weight-2 node), then the two.
    assert list(orc.huffman_lengths([1, 1, 1, 1])) == [2, 2, 2, 2]
    # {0:2, 1:1, 2:1, 3:2}: 1+2 -> (2, 256); then leaves 0 and 3 (orders 0, 3 < 256)
    # -> (4, 257); then (2,256)+(4,257): all lengths 2.
    assert list(orc.huffman_lengths([2, 1, 1, 2])) == [2, 2, 2, 2]
    # {0:1, 1:1, 2:2, 3:2}: 0+1 -> (2,256); then leaf 2 (order 2) with leaf 3 -> (4,257);
    # then (2,256)+(4,257): all 2.
    assert list(orc.huffman_lengths([1, 1, 2, 2])) == [2, 2, 2, 2]
    # {0:1, 1:1, 2:1}: 0+1 -> (2,256); leaf 2 (weight 1) + (2,256): lengths 2,2,1.
    assert list(orc.huffman_lengths([1, 1, 1])) == [2, 2, 1]
    # a single present symbol gets one bit; absent symbols get none.
    assert list(orc.huffman_lengths([0, 0, 7, 0])) == [0, 0, 1, 0]
    assert list(orc.huffman_lengths([0, 0, 0])) == [0, 0, 0]


def test_canonical_codes_hand_worked(orc):
    # lengths {2,2,1}: symbol 2 = "0", symbol 0 = "10", symbol 1 = "11"
    assert list(orc.canonical_codes([2, 2, 1])) == [0b10, 0b11, 0b0]
    # RFC 1951 section 3.2.2 example: lengths (3,3,3,3,3,2,4,4) for A..H give
    # A=010 B=011 C=100 D=101 E=110 F=00 G=1110 H=1111.
    assert list(orc.canonical_codes([3, 3, 3, 3, 3, 2, 4, 4])) == [
        0b010, 0b011, 0b100, 0b101, 0b110, 0b00, 0b1110, 0b1111]


def _brute_force_min_cost(freqs):
    """Minimum of sum f*len over every complete prefix code (Kraft sum exactly 1).

    For a multiset of lengths the cheapest assignment gives the shortest lengths to the
    largest frequencies (rearrangement inequality), so enumerating non-decreasing
    length sequences covers every complete code."""
    f = sorted([x for x in freqs if x > 0], reverse=True)
    n = len(f)
    if n == 1:
        return f[0]
    best = None
    for lens in itertools.combinations_with_replacement(range(1, n), n):
        if sum(2.0 ** -x for x in lens) != 1.0:
            continue
        cost = sum(a * b for a, b in zip(f, lens))
        best = cost if best is None else min(best, cost)
    return best


def test_brute_force_optimal_small_alphabets(orc):
    rng = np.random.default_rng(0)
    for trial in range(300):
        a = int(rng.integers(2, 9))
        f = rng.integers(0, 6 if trial % 2 else 1000, size=a)
        if trial % 5 == 0:
            f[: a // 2] = f[0]  # force ties
        if np.count_nonzero(f) < 2:
            f[0], f[1] = 3, 3
        lens = orc.huffman_lengths(f)
        cost = int(np.sum(f.astype(np.int64) * lens))
        assert cost == _brute_force_min_cost(f.tolist()), (f, lens)
        # the limiter never fires on 8 symbols (the longest possible code is 7 bits)
        assert list(orc.limited_lengths(f)) == list(lens)


def test_kraft_equality_and_entropy_bound(orc):
    rng = np.random.default_rng(1)
    for trial in range(200):
        a = int(rng.integers(2, 257))
        if trial % 3 == 0:
            f = rng.integers(0, 50, size=a)
        else:  # geometric-like skew, as the exponent histograms of the pages
            f = (1e6 * rng.random(a) ** 8).astype(np.int64)
        if np.count_nonzero(f) < 2:
            f[:2] = [1, 2]
        lens = orc.huffman_lengths(f)
        assert kraft(lens) == 1.0
        assert all((f > 0) == (lens > 0))
        p = f[f > 0] / f.sum()
        H = float(-(p * np.log2(p)).sum())
        L = float((f * lens).sum() / f.sum())
        assert H - 1e-12 <= L < H + 1
        lim = orc.limited_lengths(f)
        assert lim.max() <= 12 and kraft(lim) == 1.0
        assert all((f > 0) == (lim > 0))


def test_limiter_hand_worked(orc):
    f = [1, 1, 2, 4, 8, 16]
    assert list(orc.huffman_lengths(f)) == [5, 5, 4, 3, 2, 1]
    # halved once: [1,1,1,2,4,8]; 0+1 -> (2,256); leaf 2 (w1) + leaf 3 (w2) -> (3,257);
    # (2,256)+(3,257) -> (5,258); leaf 4 (w4) + (5,258) -> (9,259); leaf 5 + (9,259).
    assert list(orc.limited_lengths(f, lmax=4)) == [4, 4, 4, 4, 2, 1]
    # no change when the longest code already fits
    assert list(orc.limited_lengths(f, lmax=5)) == [5, 5, 4, 3, 2, 1]


def test_limiter_fires_on_bf16_chunks(orc):
    from lossless_float_weight_b200 import workloads as W
    x = W.bf16_small()
    fired = 0
    for c in range(8):
        h = orc.histogram("bf16", x, c * 131072, (c + 1) * 131072, 0)
        un = orc.huffman_lengths(h)
        lim = orc.limited_lengths(h)
        assert lim.max() <= 12 and kraft(lim) == 1.0
        fired += un.max() > 12
        # the limit costs little: within 0.01 bit per symbol of the unlimited code
        cu = float((h * un).sum()) / h.sum()
        cl = float((h * lim).sum()) / h.sum()
        assert cu <= cl < cu + 0.01
    assert fired > 0


def test_single_symbol_and_two_symbol_cases(orc):
    assert list(orc.limited_lengths([0] * 255 + [5])) == [0] * 255 + [1]
    lens = orc.limited_lengths([10 ** 9] + [1] + [0] * 254)
    assert list(lens[:2]) == [1, 1]
    assert math.isclose(kraft(lens), 1.0)

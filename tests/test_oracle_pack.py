"""Pins for the oracle's packed exponent tuples (NeuralZip, abstract: recurring exponent
tuples represented by packed exponents, chosen by the setup).

Reading under test (BF16): the setup lists the K <= 15 most frequent exponents; the
exponents of values (2j, 2j+1) form one pair symbol, their list indices as nibbles (15 for
an exponent not in the list, whose 8 bits follow the pair's code); each group gets a
packed code over the pair symbols, and a chunk takes the shared code, plain or packed,
that codes it in the fewest bits. The pins: a hand-derived golden container, brute force
for the list and the pair counts, an independent decoder of PACK payloads written here
from the format, and the cheapest-code rule checked against costs computed here.
"""
import collections
import struct

import numpy as np
import pytest
import torch

import golden_util as GU


def _exponents(x):
    return [(v >> 7) & 0xFF for v in x.view(torch.int16).tolist()]


def _spread(n, binades, seed, sigma_shift=0):
    g = torch.Generator().manual_seed(seed)
    m = 1 + torch.rand(n, generator=g, dtype=torch.float64)
    e = torch.randint(0, binades, (n,), generator=g)
    s = torch.where(torch.rand(n, generator=g) < 0.5, -1.0, 1.0).to(torch.float64)
    return (s * m * torch.pow(2.0, -(e + 1 + sigma_shift).to(torch.float64))).to(torch.bfloat16)


def test_golden_packed_pairs(orc):
    """The hand-derived container: the plan the oracle builds on the input equals the
    fixture's hand-derived plan, and the container equals the fixture byte for byte."""
    fx = GU.load("bf16_packed_pairs.json")
    x = GU.packed_pairs_input()
    cb, S = fx["input"]["chunk_bytes"], fx["input"]["S"]
    lens, assign, _, _ = orc.plan_build("bf16", x, chunk_bytes=cb, groups=1)
    exps, plens = orc.plan_pack(x, assign, 1, fx["plan"]["max_pack"], chunk_bytes=cb)
    want_lens = GU.plan_lens(fx)
    want_plens = np.zeros((1, 256), dtype=np.uint8)
    for sym, ln in fx["plan"]["packed_lens"]["0"].items():
        want_plens[0, int(sym)] = ln
    assert np.array_equal(lens, want_lens)
    assert list(exps) == fx["plan"]["packed_exponents"]
    assert np.array_equal(plens, want_plens)
    c = orc.compress("bf16", x, chunk_bytes=cb, S=S, plan_lens=want_lens,
                     pack=(np.array(fx["plan"]["packed_exponents"], dtype=np.uint8), want_plens))
    assert np.array_equal(c, GU.expected_bytes(fx))
    y = orc.decompress("bf16", c, x.numel(), chunk_bytes=cb)
    assert np.array_equal(y, x.view(torch.uint8).numpy())


@pytest.mark.parametrize("case", ["gauss", "ties", "few", "many"])
def test_pack_list_is_most_frequent(orc, case):
    """The list is the exponents sorted by (count descending, exponent ascending), cut at
    max_pack or at the exponents present."""
    if case == "gauss":
        x = (torch.randn(50000, generator=torch.Generator().manual_seed(1)) * 0.02).to(torch.bfloat16)
    elif case == "ties":  # exponents 120..129, each 64 times, then 3 more of 125
        E = [120 + (i % 10) for i in range(640)] + [125] * 3
        x = torch.tensor([2.0 ** (e - 127) for e in E], dtype=torch.float64).to(torch.bfloat16)
    elif case == "few":  # three exponents only
        E = [126, 127, 127, 128] * 100
        x = torch.tensor([2.0 ** (e - 127) for e in E], dtype=torch.float64).to(torch.bfloat16)
    else:
        x = _spread(30000, 40, seed=2)
    E = _exponents(x)
    cnt = collections.Counter(E)
    order = sorted(cnt, key=lambda e: (-cnt[e], e))
    for max_pack in (1, 2, 7, 15):
        assign = np.zeros(-(-len(E) // 4096), dtype=np.uint32)
        exps, _ = orc.plan_pack(x, assign, 1, max_pack, chunk_bytes=8192)
        assert list(exps) == order[:max_pack]


def test_pack_histogram_brute_force(orc):
    """Pair symbols and escapes counted here value by value."""
    x = _spread(4000, 24, seed=3)
    E = _exponents(x)
    exps = [int(v) for v in np.random.default_rng(0).choice(np.arange(100, 130), 11, replace=False)]
    for lo, m in [(0, 4000), (6, 100), (1000, 2)]:
        h, esc = orc.pack_histogram(x, lo, m, exps)
        want = np.zeros(256, dtype=np.uint64)
        w_esc = 0
        for j in range(lo, lo + m, 2):
            a = exps.index(E[j]) if E[j] in exps else 15
            b = exps.index(E[j + 1]) if E[j + 1] in exps else 15
            want[a * 16 + b] += 1
            w_esc += (a == 15) + (b == 15)
        assert np.array_equal(h, want) and esc == w_esc


# ---- an independent reader of the container format (written from the format rules) ----

def _canonical(lens):
    """Canonical codes (RFC 1951, 3.2.2) as {(length, code): symbol}."""
    out, code = {}, 0
    for ln in range(1, 13):
        for sym in range(len(lens)):
            if lens[sym] == ln:
                out[(ln, code)] = sym
                code += 1
        code <<= 1
    return out


def _record(buf, pos, a=256):
    return [(buf[pos + i // 2] >> (4 * (i & 1))) & 15 for i in range(a)]


class _Bits:
    def __init__(self, data, t=0):
        self.d, self.t = data, t

    def bit(self):
        b = (self.d[self.t >> 3] >> (7 - (self.t & 7))) & 1
        self.t += 1
        return b

    def fixed(self, w):
        v = 0
        for _ in range(w):
            v = v << 1 | self.bit()
        return v

    def symbol(self, table):
        code = 0
        for ln in range(1, 13):
            code = code << 1 | self.bit()
            if (ln, code) in table:
                return table[(ln, code)]
        raise AssertionError("no code")


def _read(buf, m0, n):
    """Header fields, entries and, for every PACK entry, the decoded exponents with the
    bit offset found at each S-th value."""
    buf = bytes(buf)
    K, G, S = buf[58], buf[57], struct.unpack_from("<I", buf, 20)[0]
    C = struct.unpack_from("<I", buf, 24)[0]
    off_codes, off_payload = struct.unpack_from("<QQ", buf, 32)
    exps = list(buf[off_payload - 16: off_payload - 16 + K])
    assert not any(buf[off_payload - 16 + K: off_payload])
    ents = [struct.unpack_from("<BxxxIQ", buf, 64 + 16 * k) for k in range(2 * C)]
    decoded = {}
    for c in range(C):
        mode, code, off = ents[2 * c]
        if mode != 4:
            continue
        m = min(m0, n - c * m0)
        assert G <= code < 2 * G
        table = _canonical(_record(buf, off_codes + 128 * code))  # BF16: 2G records of 128 bytes
        nsub = -(-m // S)
        idx = struct.unpack_from(f"<{nsub}I", buf, off)
        bs = buf[off + ((4 * nsub + 15) // 16) * 16:]
        rd = _Bits(bs)
        out = []
        for i in range(0, m, 2):
            if i % S == 0:
                assert rd.t == idx[i // S]
            s = rd.symbol(table)
            for nib in (s >> 4, s & 15):
                out.append(rd.fixed(8) if nib == 15 else exps[nib])
        decoded[c] = (out, rd.t)
    return K, G, exps, ents, decoded


@pytest.mark.parametrize("kind", ["gauss", "tail", "kv"])
def test_packed_container_read_independently(orc, kind):
    """Every PACK entry decodes, with the reader written here, to the input's exponents;
    every pair's code and escapes lie where the index says; the group's packed code is
    the limited Huffman code of its member chunks' pair counts (counted here); and each
    chunk's exponent stream takes the code, plain or packed, with the fewest bits."""
    cb = 8192
    m0 = cb // 2
    if kind == "gauss":
        x = (torch.randn(m0 * 6 + 1000, generator=torch.Generator().manual_seed(4)) * 0.02).to(torch.bfloat16)
    elif kind == "tail":  # weights with 1% of values 2^-12 .. 2^-20 smaller: escapes
        g = torch.Generator().manual_seed(5)
        v = torch.randn(m0 * 5 + 12, generator=g, dtype=torch.float64) * 0.02
        tail = torch.rand(v.numel(), generator=g) < 0.01
        v[tail] *= torch.pow(2.0, -torch.randint(12, 21, (int(tail.sum()),), generator=g).to(torch.float64))
        x = v.to(torch.bfloat16)
    else:
        from lossless_float_weight_b200 import workloads as W
        x = W.kv_cache(shape=(1, 2, 2, 2, 64, 128), seed=1).reshape(-1)
    n = x.numel()
    G = 3
    lens, assign, _, _ = orc.plan_build("bf16", x, chunk_bytes=cb, groups=G)
    exps, plens = orc.plan_pack(x, assign, G, 15, chunk_bytes=cb)
    buf = orc.compress("bf16", x, chunk_bytes=cb, S=512, plan_lens=lens, pack=(exps, plens))
    K, G2, exps2, ents, decoded = _read(buf, m0, n)
    assert (K, G2, exps2) == (len(exps), G, list(exps))
    E = _exponents(x)
    C = -(-n // m0)
    # the packed code of each group from pair counts taken here
    for g in range(G):
        total = np.zeros(256, dtype=np.uint64)
        for c in range(C):
            m = min(m0, n - c * m0)
            if assign[c] != g or m % 2:
                continue
            for j in range(c * m0, c * m0 + m, 2):
                a = list(exps).index(E[j]) if E[j] in exps else 15
                b = list(exps).index(E[j + 1]) if E[j + 1] in exps else 15
                total[a * 16 + b] += 1
        want = orc.limited_lengths(total) if total.any() else np.zeros(256, np.uint8)
        assert np.array_equal(plens[g], want)
    picked = collections.Counter()
    escapes = 0
    for c in range(C):
        m = min(m0, n - c * m0)
        seg = E[c * m0: c * m0 + m]
        mode, code, off = ents[2 * c]
        picked[mode] += 1
        if mode == 4:
            out, end_bit = decoded[c]
            assert out == seg
            escapes += sum(e not in exps for e in seg)
            nxt = ents[2 * c + 1][2]
            assert (end_bit + 7) // 8 <= nxt - off
        # costs computed here: plain group codes, then packed ones (escapes 8 bits each)
        h = collections.Counter(seg)
        costs = []
        for g in range(G):
            lg = lens[0, g]
            if all(lg[s] for s in h):
                costs.append((sum(h[s] * int(lg[s]) for s in h), 2, g))
        if m % 2 == 0:
            pairs = collections.Counter()
            esc = 0
            for j in range(0, m, 2):
                a = list(exps).index(seg[j]) if seg[j] in exps else 15
                b = list(exps).index(seg[j + 1]) if seg[j + 1] in exps else 15
                pairs[a * 16 + b] += 1
                esc += (a == 15) + (b == 15)
            for g in range(G):
                if all(plens[g][s] for s in pairs):
                    costs.append((sum(pairs[s] * int(plens[g][s]) for s in pairs) + 8 * esc, 4, g))
        if not costs:
            assert mode in (0, 2) and (mode == 0 or code == 0xFFFFFFFF)
            continue
        best = costs[0]
        for cst in costs[1:]:
            if cst[0] < best[0]:
                best = cst
        nsub = -(-m // 512)
        size = ((4 * nsub + 15) // 16) * 16 + ((best[0] + 7) // 8 + 15) // 16 * 16
        raw = ((m + 15) // 16) * 16
        if size < raw:
            assert (mode, code) == (best[1], best[2] + (G if best[1] == 4 else 0))
        else:
            assert mode == 0
    assert picked[4] > 0
    assert kind != "tail" or escapes > 10
    y = orc.decompress("bf16", buf, n, chunk_bytes=cb, threads=4)
    assert np.array_equal(y, x.view(torch.uint8).numpy())


def test_no_packing_is_the_plain_plan(orc):
    """max_pack 0 lists nothing, and the container is the plain plan's byte for byte;
    the packed container of an odd-length tensor leaves its odd last chunk unpacked."""
    x = (torch.randn(4096 * 3 + 7, generator=torch.Generator().manual_seed(6)) * 0.02).to(torch.bfloat16)
    lens, assign, _, _ = orc.plan_build("bf16", x, chunk_bytes=8192, groups=2)
    exps, plens = orc.plan_pack(x, assign, 2, 0, chunk_bytes=8192)
    assert len(exps) == 0 and not plens.any()
    a = orc.compress("bf16", x, chunk_bytes=8192, plan_lens=lens)
    b = orc.compress("bf16", x, chunk_bytes=8192, plan_lens=lens, pack=(exps, plens))
    assert np.array_equal(a, b)
    exps, plens = orc.plan_pack(x, assign, 2, 15, chunk_bytes=8192)
    c = orc.compress("bf16", x, chunk_bytes=8192, plan_lens=lens, pack=(exps, plens))
    modes = [c[64 + 32 * k] for k in range(4)]
    assert modes[3] != 4 and 4 in modes[:3]
    y = orc.decompress("bf16", c, x.numel(), chunk_bytes=8192)
    assert np.array_equal(y, x.view(torch.uint8).numpy())


def test_packed_header_checks(orc):
    """The decoder refuses a list with more than 15 entries, a non-zero byte after the
    list, and a PACK entry whose code is a plain record."""
    fx = GU.load("bf16_packed_pairs.json")
    good = GU.expected_bytes(fx).copy()
    assert orc.decompress_status("bf16", good, 64, chunk_bytes=128) == 0
    bad = good.copy()
    bad[58] = 16
    assert orc.decompress_status("bf16", bad, 64, chunk_bytes=128) == 3
    bad = good.copy()
    bad[352 + 5] = 1
    assert orc.decompress_status("bf16", bad, 64, chunk_bytes=128) == 3
    bad = good.copy()
    bad[64 + 4] = 0  # code 0: the plain record
    assert orc.decompress_status("bf16", bad, 64, chunk_bytes=128) == 3

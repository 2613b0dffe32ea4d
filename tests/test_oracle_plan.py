"""Pins for the oracle's grouping step, the reusable setup of "NeuralZip: Reusable Setup
for Fast Lossless Compression" (abstract: chunks with similar exponent distributions
share one Huffman code). The pages give no grouping algorithm; the Lloyd k-means
reading is pinned here by the published SplitMix64 sequence and by properties that any
correct Lloyd run has: a fixed point at convergence, non-increasing inertia, identity
grouping when there are no more chunks than groups, and recovery of well-separated
clusters. The shared-code choice is pinned by brute force over the groups."""
import struct

import numpy as np
import torch


def test_splitmix64_published_sequence(orc):
    # Reference outputs of SplitMix64 (Steele, Lea, Flood 2014; Vigna's splitmix64.c)
    # for the state 1234567.
    assert orc.splitmix64_sequence(1234567, 5) == [
        6457827717110365317, 3203168211198807973, 9817491932198370423,
        4593380528125082431, 16408922859458223821]


def _chunks_with_sigmas(sigmas, m0=4096, seed=0):
    g = torch.Generator().manual_seed(seed)
    parts = [(torch.randn(m0, generator=g) * s).to(torch.bfloat16) for s in sigmas]
    return torch.cat(parts)


def _features(orc, x, m0, C):
    X = np.zeros((C, 256))
    for c in range(C):
        X[c] = orc.histogram("bf16", x, c * m0, (c + 1) * m0, 0) / m0
    return X


def test_fixed_point_and_monotone_inertia(orc):
    rng = np.random.default_rng(0)
    sig = np.exp(rng.uniform(np.log(1e-4), np.log(10.0), size=40))
    x = _chunks_with_sigmas(sig)
    lens, assign, iters, inertia = orc.plan_build("bf16", x, chunk_bytes=8192, groups=6, seed=0)
    assert iters < 100
    assert np.all(np.diff(inertia) <= 1e-12 * inertia[0])
    X = _features(orc, x, 4096, 40)
    for j in range(6):
        mem = assign == j
        if mem.any():
            mu = X[mem].mean(axis=0)
            # every member is nearer to its own centre than to any other group's
            for c in np.nonzero(mem)[0]:
                d_own = ((X[c] - mu) ** 2).sum()
                for k in range(6):
                    if k != j and (assign == k).any():
                        d_k = ((X[c] - X[assign == k].mean(axis=0)) ** 2).sum()
                        assert d_own <= d_k + 1e-12
    # a group's code has a length for exactly the symbols its members use
    for j in range(6):
        used = np.zeros(256, bool)
        for c in np.nonzero(assign == j)[0]:
            used |= X[c] > 0
        assert np.array_equal(lens[0, j] > 0, used)
        if used.sum() >= 2:
            assert sum(2.0 ** -int(l) for l in lens[0, j] if l) == 1.0
            assert lens[0, j].max() <= 12


def test_separable_groups_are_recovered(orc):
    # three far-apart exponent distributions, four chunks each, interleaved: the only
    # sensible 3-grouping is by distribution, and every seed here reaches it
    sig = [1e-6, 1.0, 1e4] * 4
    x = _chunks_with_sigmas(sig, seed=1)
    truth = np.array([0, 1, 2] * 4)
    for seed in range(6):
        lens, assign, iters, inertia = orc.plan_build("bf16", x, chunk_bytes=8192, groups=3, seed=seed)
        assert iters < 100
        # a bijection between groups and distributions
        pairs = set(zip(truth.tolist(), assign.tolist()))
        assert len(pairs) == 3 and len({a for _, a in pairs}) == 3, (seed, assign)


def test_few_chunks_are_their_own_group(orc):
    x = _chunks_with_sigmas([0.01, 0.5, 3.0])
    lens, assign, iters, _ = orc.plan_build("bf16", x, chunk_bytes=8192, groups=8, seed=0)
    assert list(assign) == [0, 1, 2]
    assert iters == 0
    assert (lens[0, 3:] == 0).all()
    for c in range(3):
        h = orc.histogram("bf16", x, c * 4096, (c + 1) * 4096, 0)
        assert np.array_equal(lens[0, c], orc.limited_lengths(h))


def test_plan_is_deterministic_and_seed_dependent(orc):
    rng = np.random.default_rng(5)
    x = _chunks_with_sigmas(np.exp(rng.uniform(-9, 2, size=30)), seed=2)
    a = orc.plan_build("bf16", x, chunk_bytes=8192, groups=4, seed=0)
    b = orc.plan_build("bf16", x, chunk_bytes=8192, groups=4, seed=0)
    assert np.array_equal(a[0], b[0]) and np.array_equal(a[1], b[1])


def test_shared_code_choice_is_minimum_cost(orc):
    rng = np.random.default_rng(7)
    x = _chunks_with_sigmas(np.exp(rng.uniform(-9, 2, size=24)), seed=3)
    lens, assign, _, _ = orc.plan_build("bf16", x, chunk_bytes=8192, groups=4, seed=0)
    c = orc.compress("bf16", x, chunk_bytes=8192, plan_lens=lens)
    G = 4
    for ch in range(24):
        mode, code = c[64 + 32 * ch], struct.unpack_from("<I", c, 64 + 32 * ch + 4)[0]
        h = orc.histogram("bf16", x, ch * 4096, (ch + 1) * 4096, 0)
        costs = []
        for g in range(G):
            ok = np.all(lens[0, g][h > 0] > 0)
            costs.append(int((h * lens[0, g]).sum()) if ok else None)
        elig = [g for g in range(G) if costs[g] is not None]
        if mode == 2 and code != 0xFFFFFFFF:
            g = code
            assert costs[g] == min(costs[e] for e in elig)
            assert g == min(e for e in elig if costs[e] == costs[g])
        elif mode == 2:
            assert not elig  # a local code only when no group is eligible
    y = orc.decompress("bf16", c, x.numel(), chunk_bytes=8192)
    assert np.array_equal(y, x.view(torch.uint8).numpy())


def test_fp8_plan_has_two_entropy_streams(orc):
    from lossless_float_weight_b200 import workloads as W
    q = W.fp8_tensor(rows=64, cols=4096).view(torch.uint8).numpy()
    lens, assign, _, _ = orc.plan_build("fp8_e4m3", q, chunk_bytes=4096, groups=4, seed=0)
    assert lens.shape == (2, 4, 256)
    assert (lens[0, :, 16:] == 0).all() and (lens[1, :, 8:] == 0).all()
    c = orc.compress("fp8_e4m3", q, chunk_bytes=4096, plan_lens=lens)
    assert np.array_equal(orc.decompress("fp8_e4m3", c, q.size, chunk_bytes=4096), q)

"""Seeded synthetic inputs shared by the tests, the smoke check and the benchmark.

This module only draws random numbers and casts them; it holds none of the codec's
arithmetic. The recipes stand in for the trained checkpoints and K/V caches that the
pages measure (ZipNN's BF16/FP32 models, FP8 weights and K/V caches), which are not
available here:

* ``bf16_small``: 1,048,576 values N(0, 0.02^2) from CPU seed 0, rounded to BF16.
* ``checkpoint_7b``: the 225 tensors of a 7B-shaped BF16 checkpoint (32 layers of
  q, k, v, o 4096x4096 and gate, up, down 4096x11008, then a 32000x4096 embedding);
  tensor t has sigma_t = exp(U(ln 0.005, ln 0.05)) (225 draws, CPU seed 0) and values
  N(0, 1) * sigma_t from a generator seeded t + 1 on the tensor's device.
* ``fp32_tensor``: N(0, 0.02^2) FP32; the "clean" variant is the same values rounded
  through BF16 (low 16 fraction bits zero).
* ``fp8_tensor``: rows of N(0, 1) * scale_r, scale_r = exp(U(ln 0.25, ln 4)) per
  4096-wide row, clamped to +-448 and cast to float8_e4m3fn (round to nearest).
* ``kv_cache``: [layers, 2, batch, heads, seq, dim] BF16 with per-channel std
  exp(ln 0.5 + N(0, 1)) for every (layer, k/v, head, dim), shared over batch and seq.
"""
import math

import torch

CHUNK_BYTES = 262144


def bf16_small(n=1048576, seed=0, sigma=0.02):
    g = torch.Generator("cpu").manual_seed(seed)
    return (torch.randn(n, generator=g) * sigma).to(torch.bfloat16)


def checkpoint_7b_shapes(layers=32, hidden=4096, mlp=11008, vocab=32000):
    shapes = []
    for layer in range(layers):
        for name in ("q", "k", "v", "o"):
            shapes.append((f"layers.{layer}.attn.{name}", (hidden, hidden)))
        for name in ("gate", "up", "down"):
            shapes.append((f"layers.{layer}.mlp.{name}", (hidden, mlp)))
    shapes.append(("embedding", (vocab, hidden)))
    return shapes


def checkpoint_7b_sigmas(count=225, seed=0):
    g = torch.Generator("cpu").manual_seed(seed)
    u = torch.rand(count, generator=g, dtype=torch.float64)
    lo, hi = math.log(0.005), math.log(0.05)
    return torch.exp(lo + (hi - lo) * u).tolist()


def checkpoint_7b_tensor(t, shape, sigma, device="cuda"):
    g = torch.Generator(device).manual_seed(t + 1)
    x = torch.randn(shape, generator=g, device=device, dtype=torch.float32)
    return (x * sigma).to(torch.bfloat16)


def checkpoint_7b(device="cuda", layers=32, hidden=4096, mlp=11008, vocab=32000):
    shapes = checkpoint_7b_shapes(layers, hidden, mlp, vocab)
    sig = checkpoint_7b_sigmas(len(shapes))
    return [(name, checkpoint_7b_tensor(t, shape, sig[t], device)) for t, (name, shape) in enumerate(shapes)]


def fp32_tensor(n=268435456, seed=0, sigma=0.02, clean=False, device="cpu", block=1 << 26):
    g = torch.Generator(device).manual_seed(seed)
    out = torch.empty(n, dtype=torch.float32, device=device)
    for lo in range(0, n, block):
        hi = min(n, lo + block)
        out[lo:hi] = torch.randn(hi - lo, generator=g, device=device) * sigma
    if clean:
        out = out.to(torch.bfloat16).to(torch.float32)
    return out


def fp8_tensor(rows=262144, cols=4096, seed=0, device="cpu", block_rows=16384):
    g = torch.Generator(device).manual_seed(seed)
    lo, hi = math.log(0.25), math.log(4.0)
    scale = torch.exp(lo + (hi - lo) * torch.rand(rows, 1, generator=g, device=device))
    out = torch.empty(rows, cols, dtype=torch.float8_e4m3fn, device=device)
    for r in range(0, rows, block_rows):
        r2 = min(rows, r + block_rows)
        x = torch.randn(r2 - r, cols, generator=g, device=device) * scale[r:r2]
        out[r:r2] = x.clamp(-448.0, 448.0).to(torch.float8_e4m3fn)
    return out.reshape(-1)


# E2M1 magnitudes in code order (codes 0..7) and the midpoints between them
FP4_GRID = (0.0, 0.5, 1.0, 1.5, 2.0, 3.0, 4.0, 6.0)
FP4_MIDPOINTS = (0.25, 0.75, 1.25, 1.75, 2.5, 3.5, 5.0)


def fp4_tensor(rows=262144, cols=4096, seed=0, device="cpu", block_rows=16384):
    """The FP8 recipe in FP4 (E2M1): N(0, 1) times a per-row scale log-uniform in
    [0.25, 4], rounded to the nearest E2M1 value (ties to the smaller magnitude),
    saturating at 6. Returns rows * cols values as torch.float4_e2m1fn_x2 (value 2i in
    the low nibble of element i)."""
    g = torch.Generator(device).manual_seed(seed)
    lo, hi = math.log(0.25), math.log(4.0)
    scale = torch.exp(lo + (hi - lo) * torch.rand(rows, 1, generator=g, device=device))
    mids = torch.tensor(FP4_MIDPOINTS, device=device)
    out = torch.empty(rows, cols // 2, dtype=torch.uint8, device=device)
    for r in range(0, rows, block_rows):
        r2 = min(rows, r + block_rows)
        x = torch.randn(r2 - r, cols, generator=g, device=device) * scale[r:r2]
        code = torch.bucketize(x.abs(), mids) | ((x < 0).to(torch.int64) << 3)
        out[r:r2] = (code[:, 0::2] | (code[:, 1::2] << 4)).to(torch.uint8)
    return out.reshape(-1).view(torch.float4_e2m1fn_x2)


def kv_cache(shape=(32, 2, 16, 8, 4096, 128), seed=0, device="cpu"):
    layers, kv, batch, heads, seq, dim = shape
    g = torch.Generator(device).manual_seed(seed)
    std = torch.exp(math.log(0.5) + torch.randn(layers, kv, 1, heads, 1, dim, generator=g, device=device))
    out = torch.empty(shape, dtype=torch.bfloat16, device=device)
    for layer in range(layers):
        x = torch.randn((kv, batch, heads, seq, dim), generator=g, device=device)
        out[layer] = (x * std[layer]).to(torch.bfloat16)
    return out.reshape(-1)


def spread_bf16(n, binades, seed):
    """BF16 values whose magnitudes are m * 2^-(e + 1), m uniform in [1, 2) and e uniform
    in {0, ..., binades - 1}, with a random sign: exponents uniform over the `binades`
    binades below 1 (rounding to BF16 lifts the few largest to 1.0), about
    log2(binades) bits of exponent entropy, more than trained weights have. A 256 KiB chunk's exponent bitstream comes to about 45 KB
    for 6 binades, 53 KB for 9, 56 KB for 10 and 65 KB for 16."""
    g = torch.Generator().manual_seed(seed)
    e = torch.randint(0, binades, (n,), generator=g).float()
    m = torch.rand(n, generator=g) + 1.0
    sgn = torch.randint(0, 2, (n,), generator=g).float() * 2 - 1
    return (sgn * m * torch.pow(2.0, -e - 1)).to(torch.bfloat16)

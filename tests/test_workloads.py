"""The synthetic inputs (lossless_float_weight_b200/workloads.py) follow the recipes of
the benchmark configurations: shapes, dtypes, value ranges, spreads and determinism.
CPU only; the large recipes are checked on smaller draws of the same generator."""
import math

import numpy as np
import torch

from lossless_float_weight_b200 import workloads as W


def test_checkpoint_shapes_and_sizes():
    shapes = W.checkpoint_7b_shapes()
    assert len(shapes) == 32 * 7 + 1 == 225
    sizes = [math.prod(s) for _, s in shapes]
    assert sum(sizes) == 6_607_077_376  # 13.21 GB of BF16
    assert shapes[0][1] == (4096, 4096) and shapes[4][1] == (4096, 11008) and shapes[-1][1] == (32000, 4096)
    assert sum(1 for _, s in shapes if s == (4096, 4096)) == 128
    assert sum(1 for _, s in shapes if s == (4096, 11008)) == 96


def test_checkpoint_sigmas_log_uniform():
    sig = np.array(W.checkpoint_7b_sigmas())
    assert sig.shape == (225,) and sig.min() >= 0.005 and sig.max() <= 0.05
    assert np.array_equal(sig, np.array(W.checkpoint_7b_sigmas()))  # seeded
    u = (np.log(sig) - math.log(0.005)) / (math.log(0.05) - math.log(0.005))
    assert abs(u.mean() - 0.5) < 0.06 and u.min() < 0.05 and u.max() > 0.95


def test_checkpoint_tensor_draw():
    x = W.checkpoint_7b_tensor(3, (512, 512), 0.01, device="cpu")
    assert x.dtype == torch.bfloat16 and x.shape == (512, 512)
    assert abs(x.float().std().item() / 0.01 - 1) < 0.02
    assert torch.equal(x, W.checkpoint_7b_tensor(3, (512, 512), 0.01, device="cpu"))
    assert not torch.equal(x, W.checkpoint_7b_tensor(4, (512, 512), 0.01, device="cpu"))


def test_bf16_small():
    x = W.bf16_small()
    assert x.dtype == torch.bfloat16 and x.numel() == 1_048_576
    assert abs(x.float().std().item() / 0.02 - 1) < 0.01 and abs(x.float().mean().item()) < 1e-4


def test_fp32_and_clean():
    x = W.fp32_tensor(n=1 << 20)
    c = W.fp32_tensor(n=1 << 20, clean=True)
    assert x.dtype == c.dtype == torch.float32 and abs(x.std().item() / 0.02 - 1) < 0.01
    assert torch.all((c.view(torch.int32) & 0xFFFF) == 0)  # low 16 fraction bits zero
    assert torch.equal(c, x.to(torch.bfloat16).to(torch.float32))


def test_fp8_rows_and_saturation():
    rows, cols = 256, 4096
    x = W.fp8_tensor(rows=rows, cols=cols)
    assert x.dtype == torch.float8_e4m3fn and x.numel() == rows * cols
    f = x.float().reshape(rows, cols)
    assert torch.isfinite(f).all() and f.abs().max().item() <= 448.0
    rms = f.pow(2).mean(dim=1).sqrt()  # the row's scale, up to sampling and rounding
    assert rms.min().item() > 0.2 and rms.max().item() < 4.5
    assert rms.max().item() / rms.min().item() > 8  # spread over most of [0.25, 4]


def test_fp4_values_on_the_grid():
    rows, cols = 64, 4096
    b = W.fp4_tensor(rows=rows, cols=cols).view(torch.uint8).reshape(rows, cols // 2)
    codes = torch.stack([b & 15, b >> 4], dim=-1).reshape(rows, cols)  # value 2i in the low nibble
    mag = torch.tensor(W.FP4_GRID)[(codes & 7).long()]
    val = torch.where(codes >= 8, -mag, mag)
    assert len(torch.unique(codes & 7)) == 8  # every magnitude occurs, 6 is the saturation
    rms = val.pow(2).mean(dim=1).sqrt()
    assert rms.min().item() > 0.15 and rms.max().item() < 4.5


def test_kv_cache_per_channel_spread():
    shape = (2, 2, 4, 2, 256, 16)
    x = W.kv_cache(shape=shape)
    assert x.dtype == torch.bfloat16 and x.numel() == math.prod(shape)
    f = x.float().reshape(shape)
    std = f.std(dim=(2, 4))  # per (layer, k/v, head, dim), over batch and sequence
    s = torch.log(std).flatten()
    assert abs(s.mean().item() - math.log(0.5)) < 0.35 and 0.7 < s.std().item() < 1.3


def test_spread_bf16_exponents():
    x = W.spread_bf16(100000, 9, 1)
    e = ((x.view(torch.int16).int() >> 7) & 0xFF).numpy()
    assert e.min() == 126 - 8 and e.max() <= 127  # 9 binades below 1; rounding lifts a few to 1.0
    counts = np.bincount(e - 118, minlength=10)
    assert counts[:9].min() > 0.9 * 100000 / 9 and counts[9] < 0.01 * 100000

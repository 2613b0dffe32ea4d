"""The oracle against the figures the pages print (CPU only).

Sources: THEORY-599 note on ZipNN, "The exponent distribution (Fig. 2, section III-A)"
(about 40 exponent values occur, the top 12 cover almost 99.9%), "Per-field
compressibility (Table II)" (exponent to about 33%, BF16 models to about 66.4%, FP32
to about 83%, clean FP32 33.7-48.1%), "Implied entropy" (about 1.6-2.6 bits).
The synthetic N(0, sigma) inputs stand in for the trained checkpoints measured there,
so the bands are wider than the printed figures; each measured value is printed.
"""
import struct

import numpy as np
import torch

from lossless_float_weight_b200 import workloads as W


def _payload_sizes(c, streams):
    n_chunks = struct.unpack_from("<I", c, 24)[0]
    total = struct.unpack_from("<Q", c, 48)[0]
    offs = [struct.unpack_from("<Q", c, 64 + 16 * k + 8)[0] for k in range(n_chunks * streams)] + [total]
    sizes = np.diff(np.array(offs, dtype=np.int64)).reshape(n_chunks, streams)
    return sizes


def test_exponent_statistics_bf16():
    x = W.bf16_small()
    e = (x.view(torch.int16).numpy().astype(np.uint16) >> 7) & 0xFF
    counts = np.bincount(e, minlength=256)
    distinct = int(np.count_nonzero(counts))
    top12 = float(np.sort(counts)[::-1][:12].sum()) / e.size
    p = counts[counts > 0] / e.size
    H = float(-(p * np.log2(p)).sum())
    print(f"distinct exponents {distinct}, top-12 share {top12:.5f}, entropy {H:.3f} bits")
    assert 15 <= distinct <= 50
    assert top12 >= 0.995
    assert 1.6 <= H <= 2.7


def test_bf16_ratios(orc):
    x = W.bf16_small()
    n = x.numel()
    c = orc.compress("bf16", x)
    sizes = _payload_sizes(c, 2)
    exp_frac = sizes[:, 0].sum() / n          # exponent plane: n bytes uncompressed
    sm_frac = sizes[:, 1].sum() / n
    total = c.size / (2 * n)
    print(f"exponent plane {exp_frac:.4f}, sign/fraction {sm_frac:.4f}, total {total:.4f}")
    assert 0.30 <= exp_frac <= 0.36
    assert sm_frac == 1.0
    assert 0.64 <= total <= 0.68


def test_fp32_ratios(orc):
    x = W.fp32_tensor(n=1 << 22)
    c = orc.compress("fp32", x, threads=4)
    total = c.size / (4 * x.numel())
    xc = x.to(torch.bfloat16).to(torch.float32)
    cc = orc.compress("fp32", xc, threads=4)
    clean = cc.size / (4 * x.numel())
    sizes = _payload_sizes(cc, 4)
    print(f"fp32 {total:.4f}, clean fp32 {clean:.4f}")
    assert 0.82 <= total <= 0.85
    assert 0.30 <= clean <= 0.49
    assert (sizes[:, 2] == 0).all() and (sizes[:, 3] == 0).all()  # low planes are ZERO
    assert np.array_equal(orc.decompress("fp32", cc, xc.numel(), threads=4), orc._bytes_view(xc))


def test_fp8_ratio_within_huffman_bounds(orc):
    q = W.fp8_tensor(rows=1024, cols=4096)
    raw = q.view(torch.uint8).numpy()
    c = orc.compress("fp8_e4m3", raw, threads=4)
    total = c.size / raw.size
    e = (raw >> 3) & 0xF
    p = np.bincount(e, minlength=16) / e.size
    p = p[p > 0]
    He = float(-(p * np.log2(p)).sum())
    print(f"fp8 total {total:.4f}, exponent entropy {He:.3f} bits")
    # sign 1 bit + mantissa 3 bits (RAW) + exponent within [H, H + 1) bits, plus framing
    assert (1 + 3 + He) / 8 - 0.005 <= total <= (1 + 3 + He + 1) / 8 + 0.01
    assert np.array_equal(orc.decompress("fp8_e4m3", c, raw.size, threads=4), raw)

"""The inputs of the GPU tests for high-entropy exponents (tests/test_gpu_parity.py) reach
the three ways the BF16 decode holds a chunk's exponent bitstream: within the 48 KB
shared-memory window, within the 56 KB wide window (the last 8 KB in the decode table's
first half), and beyond it (read from global memory). The sizes come from the oracle's
containers, so this holds whatever the CUDA path does."""
import struct

import numpy as np
import pytest
import torch

import oracle as orc
from lossless_float_weight_b200 import workloads as W

WINDOW, WIDE = 48 * 1024, 56 * 1024
M0, S = 131072, 512  # values per 256 KiB BF16 chunk; sub-block length


def _bitstream_bytes(x):
    """(mode, exponent bitstream bytes) of each chunk of the oracle's container."""
    c = np.asarray(orc.compress("bf16", x.view(torch.uint8).numpy()))
    n_chunks = struct.unpack_from("<I", c, 24)[0]
    out = []
    for ch in range(n_chunks):
        e = 64 + 32 * ch  # chunk table entry of the exponent stream; the next is the sign/fraction one
        mode, code = struct.unpack_from("<II", c, e)
        off = struct.unpack_from("<Q", c, e + 8)[0]
        end = struct.unpack_from("<Q", c, e + 16 + 8)[0]
        m = min(M0, x.numel() - ch * M0)
        rec = 128 if code == 0xFFFFFFFF else 0
        idx = (4 * -(-m // S) + 15) // 16 * 16
        out.append((mode & 0xFF, end - off - rec - idx))
    return out


@pytest.mark.parametrize("binades,lo,hi", [(6, 0, WINDOW), (9, WINDOW, WIDE), (10, WINDOW, WIDE),
                                           (16, WIDE, 1 << 20)])
def test_spread_inputs_reach_each_decode_window(binades, lo, hi):
    x = W.spread_bf16(M0 * 3 + 1001, binades, binades)  # as the GPU test draws it
    sizes = _bitstream_bytes(x)
    assert len(sizes) == 4
    for mode, b in sizes[:3]:
        assert mode == 2 and lo < b <= hi, (binades, b)  # HUFF, in the intended window
    assert sizes[3][1] < 1024  # the ragged last chunk


def test_wide_window_corruption_input():
    # the input of the corruption test: both chunks in the wide window
    for mode, b in _bitstream_bytes(W.spread_bf16(M0 * 2, 9, 3)):
        assert mode == 2 and WINDOW < b <= WIDE

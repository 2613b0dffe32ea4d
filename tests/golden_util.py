"""Readers for the hand-derived golden containers under tests/golden/.

The expected bytes are assembled from the fixture's hand-written fields only; nothing
here calls the oracle or the CUDA library.
"""
import json
import os
import struct

import numpy as np
import torch

GOLDEN = os.path.join(os.path.dirname(os.path.abspath(__file__)), "golden")


def load(name):
    with open(os.path.join(GOLDEN, name)) as f:
        return json.load(f)


def three_chunk_input():
    """The 517 BF16 values of bf16_three_chunks.json, built from their numeric meaning:
    (-1)^sign * (1 + fraction/128) * 2^(E - 127)."""
    vals = []
    E = [127, 127, 126, 128]
    for i in range(256):
        sign = -1.0 if (i >> 7) else 1.0
        vals.append(sign * (1.0 + (i & 127) / 128.0) * 2.0 ** (E[i % 4] - 127))
    vals += [0.0] * 256
    vals += [1.0] * 5
    x = torch.tensor(vals, dtype=torch.float64).to(torch.bfloat16)
    assert torch.equal(x.to(torch.float64), torch.tensor(vals, dtype=torch.float64))  # exact in BF16
    return x


def zero_runs_input():
    """The 296 BF16 values of bf16_zero_runs.json, from their numeric meaning."""
    vals = []
    for i in range(256):
        if 32 <= i < 96:
            vals.append(0.0)
        else:
            e = 127 if i % 2 == 0 else 126
            vals.append((-1.0) ** (i >> 7) * (1 + (i & 127) / 128) * 2.0 ** (e - 127))
    for j in range(40):
        vals.append(0.0 if j < 32 else 1 + (j - 32) / 128)
    x = torch.tensor(vals, dtype=torch.float64).to(torch.bfloat16)
    assert torch.equal(x.to(torch.float64), torch.tensor(vals, dtype=torch.float64))  # exact in BF16
    return x


def fp8_two_chunk_input():
    """The 293 FP8 E4M3 values of fp8_two_chunks.json: built from their numeric meaning
    (-1)^sign * (1 + M/8) * 2^(E - 7), cast to float8_e4m3fn, and checked against the
    bit layout the fixture states (sign bit 7, exponent bits 6..3, mantissa bits 2..0)."""
    E = [7, 7, 6, 9]
    M = [0] * 12 + [1, 1, 2, 3]
    vals, bits = [], []
    for i in range(256):
        s, e, m = int(i % 8 == 0), E[i % 4], M[i % 16]
        vals.append((-1.0) ** s * (1 + m / 8) * 2.0 ** (e - 7))
        bits.append(s << 7 | e << 3 | m)
    for j in range(37):
        vals.append(1 + (j % 8) / 8)
        bits.append(7 << 3 | (j % 8))
    x = torch.tensor(vals, dtype=torch.float64).to(torch.float8_e4m3fn)
    assert x.view(torch.uint8).tolist() == bits
    assert torch.equal(x.to(torch.float64), torch.tensor(vals, dtype=torch.float64))  # exact in E4M3
    return x


def fp32_clean_two_chunk_input():
    """The 261 FP32 values of fp32_clean_two_chunks.json, from their numeric meaning, with
    the stated fields checked: chunk 0 has zero fraction bits 15..0, chunk 1 fraction j+1."""
    E = [127, 127, 126, 128]
    vals, bits = [], []
    for i in range(256):
        b = 255 - i
        vals.append((-1.0) ** (b >> 7) * (1 + (b & 127) / 128) * 2.0 ** (E[i % 4] - 127))
        bits.append((b >> 7) << 31 | E[i % 4] << 23 | (b & 127) << 16)
    for j in range(5):
        vals.append(-2.0 * (1 + (j + 1) * 2.0 ** -23))
        bits.append(1 << 31 | 128 << 23 | (j + 1))
    x = torch.tensor(vals, dtype=torch.float64).to(torch.float32)
    assert torch.equal(x.to(torch.float64), torch.tensor(vals, dtype=torch.float64))  # exact in FP32
    assert [v & 0xFFFFFFFF for v in x.view(torch.int32).tolist()] == bits
    return x


def packed_pairs_input():
    """The 64 BF16 values of bf16_packed_pairs.json: 2^(E - 127) for the stated exponents
    (sign and fraction 0), with the exponent field (bits 14..7) checked."""
    E = [127, 127, 126, 127, 127, 127, 127, 126] * 8
    E[63] = 128
    vals = [2.0 ** (e - 127) for e in E]
    x = torch.tensor(vals, dtype=torch.float64).to(torch.bfloat16)
    assert torch.equal(x.to(torch.float64), torch.tensor(vals, dtype=torch.float64))  # exact in BF16
    assert [(v >> 7) & 0xFF for v in x.view(torch.int16).tolist()] == E
    return x


def _e2m1(nibble):
    """The number an E2M1 nibble stands for: sign bit 3, exponent bits 2..1, mantissa bit 0;
    exponent 0 is subnormal (mantissa * 0.5), else (1 + mantissa/2) * 2^(exponent - 1)."""
    s, e, m = nibble >> 3, (nibble >> 1) & 3, nibble & 1
    mag = m * 0.5 if e == 0 else (1 + m / 2) * 2.0 ** (e - 1)
    return -mag if s else mag


def fp4_two_chunk_input():
    """The 522 FP4 values of fp4_two_chunks.json as torch.float4_e2m1fn_x2 (value 2i in the
    low nibble of byte i). The nibbles are built from the rule's fields, and their numbers
    are checked against the E2M1 table of the workloads (0, 0.5, 1, 1.5, 2, 3, 4, 6)."""
    from lossless_float_weight_b200.workloads import FP4_GRID
    X = [1, 1, 1, 1, 1, 1, 0, 2]
    nib = []
    for v in range(512):
        nib.append(int(v % 4 == 3) << 3 | X[v % 8] << 1 | int(v % 8 == 1))
    for j in range(10):
        nib.append((3 - j % 4) << 1 | 1)
    assert [_e2m1(k) for k in range(8)] == list(FP4_GRID)
    assert nib[:8] == [0x2, 0x3, 0x2, 0xA, 0x2, 0x2, 0x0, 0xC]
    data = bytes(nib[2 * i] | nib[2 * i + 1] << 4 for i in range(len(nib) // 2))
    assert data[:4] == bytes.fromhex("32a222c0") and data[256:] == bytes.fromhex("5713571357")
    return torch.frombuffer(bytearray(data), dtype=torch.uint8).view(torch.float4_e2m1fn_x2)


def plan_lens(fx):
    """A fixture's hand-written plan as (entropy streams, groups, 256) length bytes."""
    G = fx["plan"]["n_groups"]
    by_stream = fx["plan"].get("lens_by_stream") or [fx["plan"]["lens"]]
    lens = np.zeros((len(by_stream), G, 256), dtype=np.uint8)
    for e, groups in enumerate(by_stream):
        for g, d in groups.items():
            for sym, ln in d.items():
                lens[e, int(g), int(sym)] = ln
    return lens


def _part_bytes(p):
    out = b""
    out += b"\0" * p.get("zeros_before", 0)
    if "hex" in p:
        out += bytes.fromhex(p["hex"])
    if "hex_repeat" in p:
        out += bytes.fromhex(p["hex_repeat"]) * p["times"]
    if "hex_range" in p:
        lo, hi = p["hex_range"]
        out += bytes(range(lo, hi + 1))
    if "hex_range_down" in p:
        hi, lo = p["hex_range_down"]
        out += bytes(range(hi, lo - 1, -1))
    if "u32" in p:
        raw = b"".join(struct.pack("<I", v) for v in p["u32"])
        out += raw + b"\0" * ((-len(raw)) % 16)
    out += b"\0" * p.get("zeros_after", 0)
    return out


def expected_bytes(fx):
    h = fx["header"]
    buf = bytearray(h["total_bytes"])
    struct.pack_into("<4sHBBQIIIIQQQBBHI", buf, 0, h["magic"].encode(), h["version"], h["dtype"],
                     h["n_streams"], h["n"], h["chunk_bytes"], h["S"], h["n_chunks"], h["n_shared"],
                     h["off_codes"], h["off_payload"], h["total_bytes"], h["lmax"], h["n_groups"],
                     h.get("n_packed", 0), 0)
    for k, e in enumerate(fx["entries"]):
        struct.pack_into("<BBHIQ", buf, 64 + 16 * k, e["mode"], 0, 0, e["code"], e["offset"])
    for r in fx.get("records", []):
        b = _part_bytes(r)
        buf[r["offset"]: r["offset"] + len(b)] = b
    for p in fx["payloads"]:
        b = b"".join(_part_bytes(x) for x in p["parts"])
        buf[p["offset"]: p["offset"] + len(b)] = b
    return np.frombuffer(bytes(buf), dtype=np.uint8)

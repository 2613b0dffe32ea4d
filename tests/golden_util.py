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


def plan_lens(fx):
    G = fx["plan"]["n_groups"]
    lens = np.zeros((1, G, 256), dtype=np.uint8)
    for g, d in fx["plan"]["lens"].items():
        for sym, ln in d.items():
            lens[0, int(g), int(sym)] = ln
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
                     h["off_codes"], h["off_payload"], h["total_bytes"], h["lmax"], h["n_groups"], 0, 0)
    for k, e in enumerate(fx["entries"]):
        struct.pack_into("<BBHIQ", buf, 64 + 16 * k, e["mode"], 0, 0, e["code"], e["offset"])
    for r in fx.get("records", []):
        b = _part_bytes(r)
        buf[r["offset"]: r["offset"] + len(b)] = b
    for p in fx["payloads"]:
        b = b"".join(_part_bytes(x) for x in p["parts"])
        buf[p["offset"]: p["offset"] + len(b)] = b
    return np.frombuffer(bytes(buf), dtype=np.uint8)

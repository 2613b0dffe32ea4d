"""Test helpers: read the header and chunk table of a container (host bytes)."""
import struct

import numpy as np

NO_CODE = 0xFFFFFFFF


def header(buf):
    f = struct.unpack_from("<4sHBBQIIIIQQQBBHI", bytes(buf[:64]))
    keys = ["magic", "version", "dtype", "n_streams", "n", "chunk_bytes", "S", "n_chunks", "n_shared",
            "off_codes", "off_payload", "total_bytes", "lmax", "n_groups", "pad0", "pad1"]
    return dict(zip(keys, f))


def entries(buf, n_entries):
    raw = np.frombuffer(bytes(buf[64: 64 + 16 * n_entries]), dtype=np.uint8).reshape(n_entries, 16)
    mode = raw[:, 0].astype(np.int64)
    code = raw[:, 4:8].copy().view("<u4").reshape(-1).astype(np.int64)
    off = raw[:, 8:16].copy().view("<u8").reshape(-1).astype(np.int64)
    return mode, code, off


def payload_spans(buf):
    """(mode, code, start, end) for every entry, end = next entry's offset or total."""
    h = header(buf)
    n_ent = h["n_chunks"] * h["n_streams"]
    mode, code, off = entries(buf, n_ent)
    ends = np.append(off[1:], h["total_bytes"])
    return h, mode, code, off, ends

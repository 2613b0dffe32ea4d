"""ctypes front of the plain C oracle (oracle/zipnn_oracle.c).

TEST INFRASTRUCTURE: imported only by tests/, by __graft_entry__.smoke() and by the
CPU-baseline leg of bench.py. The product package never imports this module.
"""
import ctypes
import os

import numpy as np

from . import build as _build

DTYPES = {"bf16": 0, "fp32": 1, "fp8_e4m3": 2, "fp4_e2m1": 3}
VALUES_PER_BYTE = {"bf16": 0.5, "fp32": 0.25, "fp8_e4m3": 1, "fp4_e2m1": 2}  # FP4: two per byte


def values_in(dtype, nbytes):
    """Values held in nbytes bytes."""
    return int(nbytes * VALUES_PER_BYTE[dtype])


def bytes_of(dtype, n):
    """Bytes that hold n values (FP4: n is even)."""
    return int(n / VALUES_PER_BYTE[dtype])
OK, EINVAL, ESMALL, ECORRUPT, EPLAN = 0, 1, 2, 3, 4
LMAX = 12

_lib = None


def lib():
    global _lib
    if _lib is None:
        path = _build.build()
        L = ctypes.CDLL(path)
        u8p = ctypes.POINTER(ctypes.c_uint8)
        u64p = ctypes.POINTER(ctypes.c_uint64)
        L.orc_huffman_lengths.argtypes = [u64p, ctypes.c_int, u8p]
        L.orc_limited_lengths.argtypes = [u64p, ctypes.c_int, ctypes.c_int, u8p]
        L.orc_canonical_codes.argtypes = [u8p, ctypes.c_int, ctypes.POINTER(ctypes.c_uint32)]
        L.orc_canonical_codes.restype = None
        L.orc_histogram.argtypes = [ctypes.c_int, ctypes.c_void_p, ctypes.c_uint64, ctypes.c_uint64,
                                    ctypes.c_int, u64p]
        L.orc_histogram.restype = None
        L.orc_max_compressed_bytes.argtypes = [ctypes.c_int, ctypes.c_uint64, ctypes.c_uint32, ctypes.c_uint32]
        L.orc_max_compressed_bytes.restype = ctypes.c_uint64
        L.orc_compress.argtypes = [ctypes.c_int, ctypes.c_void_p, ctypes.c_uint64, ctypes.c_uint32,
                                   ctypes.c_uint32, ctypes.c_void_p, ctypes.c_uint32, ctypes.c_void_p,
                                   ctypes.c_uint64, u64p, ctypes.c_int]
        L.orc_decompress.argtypes = [ctypes.c_int, ctypes.c_void_p, ctypes.c_uint64, ctypes.c_uint64,
                                     ctypes.c_uint32, ctypes.c_void_p, ctypes.c_int]
        L.orc_plan_build.argtypes = [ctypes.c_int, ctypes.c_void_p, ctypes.c_uint64, ctypes.c_uint32,
                                     ctypes.c_uint32, ctypes.c_uint64, ctypes.c_void_p, ctypes.c_void_p,
                                     ctypes.POINTER(ctypes.c_int), ctypes.c_void_p]
        L.orc_compress_packed.argtypes = [ctypes.c_int, ctypes.c_void_p, ctypes.c_uint64, ctypes.c_uint32,
                                          ctypes.c_uint32, ctypes.c_void_p, ctypes.c_uint32, ctypes.c_void_p,
                                          ctypes.c_void_p, ctypes.c_uint32, ctypes.c_void_p, ctypes.c_uint64, u64p,
                                          ctypes.c_int]
        L.orc_max_compressed_bytes_packed.argtypes = [ctypes.c_int, ctypes.c_uint64, ctypes.c_uint32,
                                                      ctypes.c_uint32, ctypes.c_uint32]
        L.orc_max_compressed_bytes_packed.restype = ctypes.c_uint64
        L.orc_pack_histogram.argtypes = [ctypes.c_void_p, ctypes.c_uint64, ctypes.c_uint64, ctypes.c_void_p,
                                         ctypes.c_uint32, u64p, u64p]
        L.orc_pack_histogram.restype = None
        L.orc_plan_pack.argtypes = [ctypes.c_void_p, ctypes.c_uint64, ctypes.c_uint32, ctypes.c_uint32,
                                    ctypes.c_void_p, ctypes.c_uint32, ctypes.c_void_p, ctypes.c_void_p,
                                    ctypes.POINTER(ctypes.c_uint32)]
        L.orc_splitmix64.argtypes = [u64p]
        L.orc_splitmix64.restype = ctypes.c_uint64
        _lib = L
    return _lib


def _u8(a):
    return a.ctypes.data_as(ctypes.POINTER(ctypes.c_uint8))


def _u64(a):
    return a.ctypes.data_as(ctypes.POINTER(ctypes.c_uint64))


def _bytes_view(data):
    """Accept a numpy array or a CPU torch tensor; return a contiguous uint8 numpy view."""
    if hasattr(data, "detach"):  # torch tensor (CPU)
        t = data.detach().contiguous()
        import torch
        data = t.view(torch.uint8).numpy() if t.dtype != torch.uint8 else t.numpy()
    a = np.ascontiguousarray(data)
    return a.view(np.uint8).reshape(-1)


def huffman_lengths(freq):
    f = np.ascontiguousarray(freq, dtype=np.uint64)
    out = np.zeros(len(f), dtype=np.uint8)
    st = lib().orc_huffman_lengths(_u64(f), len(f), _u8(out))
    assert st == OK
    return out


def limited_lengths(freq, lmax=LMAX):
    f = np.ascontiguousarray(freq, dtype=np.uint64)
    out = np.zeros(len(f), dtype=np.uint8)
    st = lib().orc_limited_lengths(_u64(f), len(f), lmax, _u8(out))
    assert st == OK
    return out


def canonical_codes(lens):
    ln = np.ascontiguousarray(lens, dtype=np.uint8)
    out = np.zeros(len(ln), dtype=np.uint32)
    lib().orc_canonical_codes(_u8(ln), len(ln), out.ctypes.data_as(ctypes.POINTER(ctypes.c_uint32)))
    return out


def histogram(dtype, data, lo, hi, stream):
    b = _bytes_view(data)
    a = 256
    h = np.zeros(a, dtype=np.uint64)
    lib().orc_histogram(DTYPES[dtype], b.ctypes.data, lo, hi, stream, _u64(h))
    return h


def max_compressed_bytes(dtype, n, chunk_bytes, n_groups=0, K=0):
    return int(lib().orc_max_compressed_bytes_packed(DTYPES[dtype], n, chunk_bytes, n_groups, K))


def compress(dtype, data, n=None, chunk_bytes=262144, S=512, plan_lens=None, threads=1, pack=None):
    """Return the container (numpy uint8) for the n values held in data. pack: the plan's
    packed exponents (exps, pack_lens[groups, 256]) as plan_pack returns them, or None."""
    b = _bytes_view(data)
    if n is None:
        n = values_in(dtype, b.size)
    assert b.size >= bytes_of(dtype, n)
    G = 0
    plan_ptr = None
    if plan_lens is not None:
        pl = np.ascontiguousarray(plan_lens, dtype=np.uint8)
        G = pl.shape[1]
        plan_ptr = pl.ctypes.data
    K, exps_ptr, plens_ptr = 0, None, None
    if pack is not None and len(pack[0]):
        ex = np.zeros(16, dtype=np.uint8)
        ex[: len(pack[0])] = np.asarray(pack[0], dtype=np.uint8)
        pk = np.ascontiguousarray(pack[1], dtype=np.uint8)
        K, exps_ptr, plens_ptr = len(pack[0]), ex.ctypes.data, pk.ctypes.data
    cap = max_compressed_bytes(dtype, n, chunk_bytes, G, K)
    out = np.zeros(cap, dtype=np.uint8)
    size = ctypes.c_uint64(0)
    st = lib().orc_compress_packed(DTYPES[dtype], b.ctypes.data, n, chunk_bytes, S, plan_ptr, G, plens_ptr,
                                   exps_ptr, K, out.ctypes.data, cap, ctypes.byref(size), threads)
    if st != OK:
        raise OracleError(st)
    return out[: size.value].copy()


def pack_histogram(data, lo, m, exps):
    """Pair-symbol counts (256) and escaped exponents of BF16 values [lo, lo + m)."""
    b = _bytes_view(data)
    ex = np.zeros(16, dtype=np.uint8)
    ex[: len(exps)] = np.asarray(exps, dtype=np.uint8)
    h = np.zeros(256, dtype=np.uint64)
    esc = np.zeros(1, dtype=np.uint64)
    lib().orc_pack_histogram(b.ctypes.data, lo, m, ex.ctypes.data, len(exps), _u64(h), _u64(esc))
    return h, int(esc[0])


def plan_pack(data, assign, groups, max_pack=15, n=None, chunk_bytes=262144):
    """Packed exponents of a BF16 plan: (exps (K bytes), pack_lens[groups, 256])."""
    b = _bytes_view(data)
    if n is None:
        n = values_in("bf16", b.size)
    a = np.ascontiguousarray(assign, dtype=np.uint32)
    ex = np.zeros(16, dtype=np.uint8)
    lens = np.zeros((groups, 256), dtype=np.uint8)
    K = ctypes.c_uint32(0)
    st = lib().orc_plan_pack(b.ctypes.data, n, chunk_bytes, groups, a.ctypes.data, max_pack, ex.ctypes.data,
                             lens.ctypes.data, ctypes.byref(K))
    if st != OK:
        raise OracleError(st)
    return ex[: K.value].copy(), lens


def decompress(dtype, container, n, chunk_bytes=262144, threads=1):
    """Return the n decoded values as raw bytes (numpy uint8)."""
    c = np.ascontiguousarray(container, dtype=np.uint8)
    out = np.zeros(bytes_of(dtype, n), dtype=np.uint8)
    st = lib().orc_decompress(DTYPES[dtype], c.ctypes.data, c.size, n, chunk_bytes, out.ctypes.data, threads)
    if st != OK:
        raise OracleError(st)
    return out


def decompress_status(dtype, container, n, chunk_bytes=262144):
    c = np.ascontiguousarray(container, dtype=np.uint8)
    out = np.zeros(bytes_of(dtype, n), dtype=np.uint8)
    return lib().orc_decompress(DTYPES[dtype], c.ctypes.data, c.size, n, chunk_bytes, out.ctypes.data, 1)


def n_entropy(dtype):
    return 2 if dtype in ("fp8_e4m3", "fp4_e2m1") else 1


def plan_build(dtype, data, n=None, chunk_bytes=262144, groups=8, seed=0):
    """Return (lens[n_entropy, groups, 256], assign[n_chunks], iterations, inertia list)."""
    b = _bytes_view(data)
    if n is None:
        n = values_in(dtype, b.size)
    m0 = values_in(dtype, chunk_bytes)
    C = -(-n // m0)
    lens = np.zeros((n_entropy(dtype), groups, 256), dtype=np.uint8)
    assign = np.zeros(C, dtype=np.uint32)
    inertia = np.zeros(100, dtype=np.float64)
    iters = ctypes.c_int(0)
    st = lib().orc_plan_build(DTYPES[dtype], b.ctypes.data, n, chunk_bytes, groups, seed, lens.ctypes.data,
                              assign.ctypes.data, ctypes.byref(iters), inertia.ctypes.data)
    if st != OK:
        raise OracleError(st)
    return lens, assign, iters.value, inertia[: iters.value].copy()


def splitmix64_sequence(seed, count):
    st = ctypes.c_uint64(seed)
    return [int(lib().orc_splitmix64(ctypes.byref(st))) for _ in range(count)]


class OracleError(RuntimeError):
    def __init__(self, code):
        super().__init__(f"oracle returned status {code}")
        self.code = code

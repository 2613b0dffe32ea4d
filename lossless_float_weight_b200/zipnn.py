"""Python binding of libzipnn_b200 (include/zipnn.h).

The functions named ``zipnn_*`` are the C ABI one to one (integers for pointers and
streams). The tensor helpers below them only allocate with PyTorch, marshal pointers
and streams, and copy between host and device; every step of the codec runs in the
CUDA library. Importing this module fails loudly if the library has not been built.
"""
import ctypes
import os

import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libzipnn_b200.so")

if not os.path.exists(LIB_PATH):
    raise ImportError(f"{LIB_PATH} is missing: build it with `python -m lossless_float_weight_b200.build` "
                      "(there is no CPU fallback)")

_lib = ctypes.CDLL(LIB_PATH)

BF16, FP32, FP8_E4M3, FP4_E2M1 = 0, 1, 2, 3
OK, ERR_INVALID_ARG, ERR_OUT_TOO_SMALL, ERR_CORRUPT, ERR_PLAN_MISMATCH, ERR_CUDA, ERR_UNSUPPORTED, ERR_TIMEOUT = range(8)
DEFAULT_CHUNK_BYTES = 262144
DEFAULT_SUBBLOCK = 512
MAX_GROUPS = 64

_u64, _u32, _vp, _sz, _i = ctypes.c_uint64, ctypes.c_uint32, ctypes.c_void_p, ctypes.c_size_t, ctypes.c_int


def _sig(name, res, *args):
    f = getattr(_lib, name)
    f.restype = res
    f.argtypes = list(args)
    return f


zipnn_max_compressed_bytes = _sig("zipnn_max_compressed_bytes", _sz, _i, _u64, _u32)
zipnn_workspace_bytes = _sig("zipnn_workspace_bytes", _sz, _i, _u64, _u32)
zipnn_compress = _sig("zipnn_compress", _i, _i, _vp, _u64, _u32, _vp, _vp, _sz, _vp, _sz, _vp)
zipnn_compress_ex = _sig("zipnn_compress_ex", _i, _i, _vp, _u64, _u32, _u32, _vp, _vp, _sz, _vp, _sz, _vp)
zipnn_decompress = _sig("zipnn_decompress", _i, _i, _vp, _sz, _u64, _u32, _vp, _vp, _sz, _vp)
zipnn_compressed_size = _sig("zipnn_compressed_size", _i, _vp, _vp, ctypes.POINTER(_u64))
zipnn_get_status = _sig("zipnn_get_status", _i, _vp, _vp)
zipnn_histogram = _sig("zipnn_histogram", _i, _i, _vp, _u64, _u32, _vp, _vp)
zipnn_code_lengths = _sig("zipnn_code_lengths", _i, _vp, _u32, _u32, _vp, _vp)
zipnn_plan_create = _sig("zipnn_plan_create", _i, _i, _vp, _u64, _u32, _u32, _u64, _vp, _sz, _vp,
                         ctypes.POINTER(_vp))
zipnn_plan_create_packed = _sig("zipnn_plan_create_packed", _i, _i, _vp, _u64, _u32, _u32, _u64, _u32, _vp, _sz,
                                _vp, ctypes.POINTER(_vp))
zipnn_plan_export = _sig("zipnn_plan_export", _i, _vp, _vp, _sz, ctypes.POINTER(_sz))
zipnn_plan_import = _sig("zipnn_plan_import", _i, _vp, _sz, ctypes.POINTER(_vp))
zipnn_plan_assignment = _sig("zipnn_plan_assignment", _i, _vp, _vp, _sz, ctypes.POINTER(_sz))
zipnn_plan_destroy = _sig("zipnn_plan_destroy", None, _vp)
zipnn_status_string = _sig("zipnn_status_string", ctypes.c_char_p, _i)
zipnn_timing_enable = _sig("zipnn_timing_enable", _i, _i)
zipnn_timing_collect = _sig("zipnn_timing_collect", _i, _vp, _vp, _u32)
zipnn_kernel_count = _sig("zipnn_kernel_count", _u32)
zipnn_kernel_name = _sig("zipnn_kernel_name", ctypes.c_char_p, _u32)
zipnn_compress_noalloc = _sig("zipnn_compress_noalloc", _i, _i, _vp, _u64, _u32, _vp, _sz, _vp)
zipnn_test_lookback_limit = _sig("zipnn_test_lookback_limit", _i, _u32)
NOALLOC_SCRATCH_BYTES = 8 << 20


class DecompressItem(ctypes.Structure):
    """zipnn_decompress_item: one tensor of a batched decompress."""
    _fields_ = [("in_", _vp), ("in_bytes", _u64), ("n", _u64), ("out", _vp)]


zipnn_decompress_batch_workspace_bytes = _sig("zipnn_decompress_batch_workspace_bytes", _sz, _u32)
zipnn_decompress_batch = _sig("zipnn_decompress_batch", _i, _i, _u32, _u32, ctypes.POINTER(DecompressItem), _vp,
                              _sz, _vp)

class ShardItem(ctypes.Structure):
    """zipnn_shard_item: one shard container and where its relocated pieces go."""
    _fields_ = [("shard", _vp), ("shard_bytes", _u64), ("n_total", _u64), ("chunk_lo", _u64),
                ("table_out", _vp), ("header_out", _vp)]


zipnn_shard_workspace_bytes = _sig("zipnn_shard_workspace_bytes", _sz, _u32)
zipnn_shard_sizes = _sig("zipnn_shard_sizes", _i, _u32, ctypes.POINTER(ShardItem), _vp, _vp, _sz, _vp)
zipnn_shard_tables = _sig("zipnn_shard_tables", _i, _i, _u32, _u32, ctypes.POINTER(ShardItem), _vp, _u32, _u32, _vp,
                          _sz, _vp)

C_ABI_NAMES = [
    "zipnn_max_compressed_bytes", "zipnn_workspace_bytes", "zipnn_compress", "zipnn_compress_ex",
    "zipnn_decompress", "zipnn_compressed_size", "zipnn_get_status", "zipnn_histogram", "zipnn_code_lengths",
    "zipnn_plan_create", "zipnn_plan_create_packed", "zipnn_plan_export", "zipnn_plan_import", "zipnn_plan_assignment", "zipnn_plan_destroy",
    "zipnn_status_string", "zipnn_timing_enable", "zipnn_timing_collect", "zipnn_kernel_count",
    "zipnn_kernel_name", "zipnn_compress_noalloc", "zipnn_decompress_batch_workspace_bytes",
    "zipnn_decompress_batch", "zipnn_test_lookback_limit", "zipnn_shard_workspace_bytes", "zipnn_shard_sizes",
    "zipnn_shard_tables",
]


class ZipnnError(RuntimeError):
    def __init__(self, status, what=""):
        msg = zipnn_status_string(status).decode()
        super().__init__(f"{what}: {msg} (status {status})" if what else f"{msg} (status {status})")
        self.status = status


def check(status, what=""):
    if status != OK:
        raise ZipnnError(status, what)


# ------------------------------------------------------------------ tensor helpers

# torch.float4_e2m1fn_x2 holds two FP4 values per element (one byte, the first value in
# the low nibble); the codec counts values, so n is twice numel() for it
_TORCH_DTYPES = {torch.bfloat16: BF16, torch.float32: FP32, torch.float8_e4m3fn: FP8_E4M3,
                 torch.float4_e2m1fn_x2: FP4_E2M1}
_VALUES_PER_ELEMENT = {BF16: 1, FP32: 1, FP8_E4M3: 1, FP4_E2M1: 2}
_VALUES_PER_BYTE = {BF16: 0.5, FP32: 0.25, FP8_E4M3: 1, FP4_E2M1: 2}


def nvalues(x):
    """Values held by the tensor x (FP4: two per element)."""
    return x.numel() * _VALUES_PER_ELEMENT[dtype_code(x.dtype)]


def dtype_code(x):
    if isinstance(x, int):
        return x
    if isinstance(x, str):
        return {"bf16": BF16, "fp32": FP32, "fp8_e4m3": FP8_E4M3, "fp4_e2m1": FP4_E2M1}[x]
    return _TORCH_DTYPES[x]


def _stream(stream):
    if stream is None:
        stream = torch.cuda.current_stream()
    return stream.cuda_stream if hasattr(stream, "cuda_stream") else int(stream)


def workspace(dtype, n, chunk_bytes=DEFAULT_CHUNK_BYTES, device="cuda"):
    nb = zipnn_workspace_bytes(dtype_code(dtype), n, chunk_bytes)
    if nb == 0:
        raise ZipnnError(ERR_INVALID_ARG, "workspace size")
    return torch.empty(nb, dtype=torch.uint8, device=device)


class Plan:
    """A reusable shared-code setup (owns the library's plan handle)."""

    def __init__(self, handle, dtype):
        self.handle = handle
        self.dtype = dtype

    @classmethod
    def create(cls, x, groups=8, seed=0, chunk_bytes=DEFAULT_CHUNK_BYTES, ws=None, stream=None, max_pack=0):
        """max_pack > 0 (BF16, at most 15): the plan also lists up to that many packed
        exponents and gives every group a packed code over exponent pairs."""
        dt = dtype_code(x.dtype)
        xf = x.reshape(-1)
        if ws is None:
            ws = workspace(dt, nvalues(xf), chunk_bytes, xf.device)
        h = _vp()
        check(zipnn_plan_create_packed(dt, xf.data_ptr(), nvalues(xf), chunk_bytes, groups, seed, max_pack,
                                       ws.data_ptr(), ws.numel(), _stream(stream), ctypes.byref(h)),
              "zipnn_plan_create_packed")
        return cls(h.value, dt)

    def export(self):
        n = _sz(0)
        check(zipnn_plan_export(self.handle, None, 0, ctypes.byref(n)), "zipnn_plan_export")
        buf = (ctypes.c_uint8 * n.value)()
        check(zipnn_plan_export(self.handle, buf, n.value, ctypes.byref(n)), "zipnn_plan_export")
        return bytes(buf)

    @classmethod
    def from_bytes(cls, data):
        h = _vp()
        buf = (ctypes.c_uint8 * len(data)).from_buffer_copy(data)
        check(zipnn_plan_import(buf, len(data), ctypes.byref(h)), "zipnn_plan_import")
        return cls(h.value, data[4])

    def assignment(self):
        n = _sz(0)
        check(zipnn_plan_assignment(self.handle, None, 0, ctypes.byref(n)), "zipnn_plan_assignment")
        buf = (ctypes.c_uint32 * max(1, n.value))()
        check(zipnn_plan_assignment(self.handle, buf, n.value, ctypes.byref(n)), "zipnn_plan_assignment")
        return list(buf)[: n.value]

    def close(self):
        if self.handle:
            zipnn_plan_destroy(self.handle)
            self.handle = None

    def __del__(self):
        try:
            self.close()
        except Exception:
            pass


def compress_into(x, out, ws, chunk_bytes=DEFAULT_CHUNK_BYTES, plan=None, subblock=0, stream=None):
    """Asynchronous: compress the device tensor x into the device byte tensor out."""
    dt = dtype_code(x.dtype)
    check(zipnn_compress_ex(dt, x.data_ptr(), nvalues(x), chunk_bytes, subblock, plan.handle if plan else None,
                            out.data_ptr(), out.numel(), ws.data_ptr(), ws.numel(), _stream(stream)),
          "zipnn_compress")


def decompress_into(container, nbytes, out, ws, chunk_bytes=DEFAULT_CHUNK_BYTES, stream=None):
    """Asynchronous: decompress nbytes of the device container into the device tensor out."""
    dt = dtype_code(out.dtype)
    check(zipnn_decompress(dt, container.data_ptr(), nbytes, nvalues(out), chunk_bytes, out.data_ptr(),
                           ws.data_ptr(), ws.numel(), _stream(stream)), "zipnn_decompress")


def batch_workspace(count, device="cuda"):
    """A workspace for zipnn_decompress_batch of `count` tensors."""
    return torch.empty(zipnn_decompress_batch_workspace_bytes(count), dtype=torch.uint8, device=device)


def decompress_batch_into(containers, nbytes, outs, ws, chunk_bytes=DEFAULT_CHUNK_BYTES, stream=None):
    """Asynchronous: decompress the device containers (nbytes[i] readable each) into the
    device tensors outs[i], all of one dtype, in one launch."""
    if not outs or len(containers) != len(outs) or len(nbytes) != len(outs):
        raise ZipnnError(ERR_INVALID_ARG, "zipnn_decompress_batch")
    dt = dtype_code(outs[0].dtype)
    if any(dtype_code(o.dtype) != dt for o in outs):
        raise ZipnnError(ERR_INVALID_ARG, "zipnn_decompress_batch: one dtype per batch")
    items = (DecompressItem * len(outs))(*[DecompressItem(c.data_ptr(), b, nvalues(o), o.data_ptr())
                                            for c, b, o in zip(containers, nbytes, outs)])
    check(zipnn_decompress_batch(dt, chunk_bytes, len(outs), items, ws.data_ptr(), ws.numel(), _stream(stream)),
          "zipnn_decompress_batch")


def compressed_size(out, stream=None):
    v = _u64(0)
    check(zipnn_compressed_size(out.data_ptr(), _stream(stream), ctypes.byref(v)), "zipnn_compressed_size")
    return v.value


def status(ws, stream=None):
    return zipnn_get_status(ws.data_ptr(), _stream(stream))


def compress(x, chunk_bytes=DEFAULT_CHUNK_BYTES, plan=None, subblock=0, stream=None):
    """Compress a CUDA tensor; returns the container as a CUDA uint8 tensor (synchronises)."""
    xf = x.reshape(-1)
    dt = dtype_code(xf.dtype)
    cap = zipnn_max_compressed_bytes(dt, nvalues(xf), chunk_bytes)
    if cap == 0:
        raise ZipnnError(ERR_INVALID_ARG, "zipnn_max_compressed_bytes")
    out = torch.empty(cap, dtype=torch.uint8, device=xf.device)
    ws = workspace(dt, nvalues(xf), chunk_bytes, xf.device)
    compress_into(xf, out, ws, chunk_bytes, plan, subblock, stream)
    size = compressed_size(out, stream)
    check(status(ws, stream), "compress status")
    return out[:size]


def decompress(container, dtype, shape, chunk_bytes=DEFAULT_CHUNK_BYTES, stream=None):
    """Decompress a CUDA container into a new CUDA tensor of the given dtype and shape
    (in elements of dtype: for torch.float4_e2m1fn_x2, pairs of values)."""
    n = 1
    for d in (shape if isinstance(shape, (tuple, list, torch.Size)) else (shape,)):
        n *= d
    out = torch.empty(n, dtype=dtype, device=container.device)
    ws = torch.empty(256, dtype=torch.uint8, device=container.device)
    decompress_into(container, container.numel(), out, ws, chunk_bytes, stream)
    check(status(ws, stream), "decompress status")
    return out.reshape(shape)


def compress_host(x_host, out_host, dev_in, dev_out, ws, chunk_bytes=DEFAULT_CHUNK_BYTES, plan=None, stream=None):
    """End-to-end compress of a pinned host tensor: H2D copy, compress, D2H copy of the
    container into the pinned host buffer out_host. Returns the container size."""
    dev_in.copy_(x_host.reshape(-1), non_blocking=True)
    compress_into(dev_in, dev_out, ws, chunk_bytes, plan, 0, stream)
    size = compressed_size(dev_out, stream)
    out_host[:size].copy_(dev_out[:size], non_blocking=True)
    return size


def decompress_host(container_host, nbytes, out_host, dev_in, dev_out, ws, chunk_bytes=DEFAULT_CHUNK_BYTES,
                    stream=None):
    """End-to-end decompress of a pinned host container into the pinned host tensor out_host."""
    dev_in[:nbytes].copy_(container_host[:nbytes], non_blocking=True)
    decompress_into(dev_in, nbytes, dev_out, ws, chunk_bytes, stream)
    out_host.reshape(-1).copy_(dev_out, non_blocking=True)


def kernel_times():
    """Collect the event timing of every kernel launched since the last call:
    {name: (total ms, launches)}. Waits for the recorded events."""
    k = zipnn_kernel_count()
    ms = (ctypes.c_double * k)()
    n = (ctypes.c_uint64 * k)()
    check(zipnn_timing_collect(ms, n, k), "zipnn_timing_collect")
    return {zipnn_kernel_name(i).decode(): (ms[i], n[i]) for i in range(k)}


def histogram(x, chunk_bytes=DEFAULT_CHUNK_BYTES, stream=None):
    """Per-chunk order-0 histograms of the entropy streams: (n_chunks, n_entropy, 256) int32."""
    xf = x.reshape(-1)
    dt = dtype_code(xf.dtype)
    m0 = int(chunk_bytes * _VALUES_PER_BYTE[dt])
    C = -(-nvalues(xf) // m0)
    ne = 2 if dt in (FP8_E4M3, FP4_E2M1) else 1
    out = torch.zeros((C, ne, 256), dtype=torch.int32, device=xf.device)
    check(zipnn_histogram(dt, xf.data_ptr(), nvalues(xf), chunk_bytes, out.data_ptr(), _stream(stream)),
          "zipnn_histogram")
    return out


def code_lengths(hist, alphabet=256, stream=None):
    """Length-limited Huffman code lengths for a (count, 256) int64 CUDA tensor."""
    h = hist.to(torch.int64).contiguous()
    out = torch.zeros(h.shape, dtype=torch.uint8, device=h.device)
    check(zipnn_code_lengths(h.data_ptr(), h.shape[0], alphabet, out.data_ptr(), _stream(stream)),
          "zipnn_code_lengths")
    return out

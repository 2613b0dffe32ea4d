"""The C-ABI library loads and exports every entry point include/zipnn.h declares, and
its host-only calls (sizes, argument checks) behave; no kernel is launched (CPU)."""
import ctypes
import os
import re

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "zipnn.h")


def _declared():
    src = open(HEADER).read()
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    return sorted(set(re.findall(r"\b(zipnn_[a-z_0-9]+)\s*\(", src)))


@pytest.fixture(scope="module")
def lib():
    from lossless_float_weight_b200 import build
    build.build()
    return ctypes.CDLL(build.LIB)


def test_every_declared_symbol_is_exported(lib):
    names = _declared()
    assert len(names) >= 15
    for name in names:
        assert hasattr(lib, name), name


def test_binding_covers_the_abi(lib):
    from lossless_float_weight_b200 import zipnn
    assert sorted(zipnn.C_ABI_NAMES) == _declared()


def test_sizes_match_the_oracle(lib, orc):
    from lossless_float_weight_b200 import zipnn as Z
    for dt, name in ((Z.BF16, "bf16"), (Z.FP32, "fp32"), (Z.FP8_E4M3, "fp8_e4m3")):
        for n in (1, 17, 131072, 6607077376 // 225, 10 ** 7 + 3):
            for cb in (4096, 262144):
                # room for 64 groups' records and, for BF16, their packed records and a list of 15
                K = 15 if name == "bf16" else 0
                assert Z.zipnn_max_compressed_bytes(dt, n, cb) == orc.max_compressed_bytes(name, n, cb, 64, K)
                assert Z.zipnn_workspace_bytes(dt, n, cb) > 0
    assert Z.zipnn_max_compressed_bytes(Z.BF16, 0, 262144) == 0
    assert Z.zipnn_max_compressed_bytes(Z.BF16, 10, 100) == 0      # not a multiple of 16
    assert Z.zipnn_max_compressed_bytes(7, 10, 262144) == 0        # bad dtype
    for n in (2, 18, 524288, 524290, 2 * 10 ** 7 + 6):               # FP4: values in pairs
        for cb in (4096, 262144):
            assert Z.zipnn_max_compressed_bytes(Z.FP4_E2M1, n, cb) == orc.max_compressed_bytes("fp4_e2m1", n, cb, 64)
    assert Z.zipnn_max_compressed_bytes(Z.FP4_E2M1, 7, 262144) == 0  # an odd FP4 count


def test_argument_errors_without_a_device(lib):
    from lossless_float_weight_b200 import zipnn as Z
    # null pointers and bad sizes are rejected before anything touches the device
    assert Z.zipnn_compress(Z.BF16, None, 10, 262144, None, None, 0, None, 0, None) == Z.ERR_INVALID_ARG
    assert Z.zipnn_decompress(Z.BF16, None, 0, 10, 262144, None, None, 0, None) == Z.ERR_INVALID_ARG
    assert Z.zipnn_code_lengths(None, 1, 256, None, None) == Z.ERR_INVALID_ARG
    assert Z.zipnn_plan_import(None, 0, None) == Z.ERR_INVALID_ARG
    assert Z.zipnn_status_string(Z.ERR_CORRUPT).startswith(b"corrupt")


def test_batch_argument_errors_without_a_device(lib):
    from lossless_float_weight_b200 import zipnn as Z
    fake = 1 << 20  # a 16-byte aligned address, never dereferenced: every case fails before a launch
    ws_bytes = Z.zipnn_decompress_batch_workspace_bytes(2)
    assert ws_bytes >= 256 + 2 * 40
    good = (Z.DecompressItem * 2)(Z.DecompressItem(fake, 4096, 1000, fake), Z.DecompressItem(fake, 4096, 5, fake))
    # no items, no workspace, an empty batch
    assert Z.zipnn_decompress_batch(Z.BF16, 262144, 2, None, fake, ws_bytes, None) == Z.ERR_INVALID_ARG
    assert Z.zipnn_decompress_batch(Z.BF16, 262144, 2, good, None, ws_bytes, None) == Z.ERR_INVALID_ARG
    assert Z.zipnn_decompress_batch(Z.BF16, 262144, 0, good, fake, ws_bytes, None) == Z.ERR_INVALID_ARG
    # a misaligned or null pointer, n = 0, a bad chunk size
    for bad in (Z.DecompressItem(fake + 8, 4096, 10, fake), Z.DecompressItem(fake, 4096, 10, None),
                Z.DecompressItem(fake, 4096, 0, fake)):
        items = (Z.DecompressItem * 2)(good[0], bad)
        assert Z.zipnn_decompress_batch(Z.BF16, 262144, 2, items, fake, ws_bytes, None) == Z.ERR_INVALID_ARG
    assert Z.zipnn_decompress_batch(Z.BF16, 1000, 2, good, fake, ws_bytes, None) == Z.ERR_INVALID_ARG
    # a workspace one byte short
    assert Z.zipnn_decompress_batch(Z.BF16, 262144, 2, good, fake, ws_bytes - 1, None) == Z.ERR_OUT_TOO_SMALL


def test_code_lengths_and_size_limits_without_a_device(lib):
    from lossless_float_weight_b200 import zipnn as Z
    fake = 1 << 20  # never dereferenced: each case is rejected before a launch
    for alphabet in (0, 257, 1000):
        assert Z.zipnn_code_lengths(fake, 1, alphabet, fake, None) == Z.ERR_INVALID_ARG
    assert Z.zipnn_code_lengths(fake, 1 << 31, 256, fake, None) == Z.ERR_INVALID_ARG
    # value counts at or above 2^56 are outside the library's range
    assert Z.zipnn_max_compressed_bytes(Z.BF16, 1 << 56, 262144) == 0
    assert Z.zipnn_workspace_bytes(Z.FP8_E4M3, (1 << 56) + 16, 262144) == 0
    assert Z.zipnn_compress(Z.BF16, fake, 1 << 56, 262144, None, fake, 1 << 62, fake, 1 << 40, None) \
        == Z.ERR_INVALID_ARG


def test_lookback_limit_is_a_host_setting(lib):
    from lossless_float_weight_b200 import zipnn as Z
    assert Z.zipnn_test_lookback_limit(1) == Z.OK
    assert Z.zipnn_test_lookback_limit(0) == Z.OK  # back to the default


def test_no_device_is_reported_as_unsupported(lib):
    import torch
    if torch.cuda.is_available():
        pytest.skip("a device is present")
    from lossless_float_weight_b200 import zipnn as Z
    fake = 1 << 20
    assert Z.zipnn_code_lengths(fake, 1, 256, fake, None) == Z.ERR_UNSUPPORTED
    assert Z.zipnn_compress_noalloc(Z.BF16, fake, 1000, 262144, fake, 1 << 20, None) == Z.ERR_UNSUPPORTED


def test_packed_plan_arguments_without_a_device(lib):
    """Packed exponents: a list longer than 15, or packing for a dtype other than BF16, is
    refused before anything touches the device; an exported plan whose list is longer than
    15, names packed exponents for FP8, or has a byte past its list, does not import."""
    import ctypes
    from lossless_float_weight_b200 import zipnn as Z
    fake = 1 << 20
    h = ctypes.c_void_p()
    assert Z.zipnn_plan_create_packed(Z.BF16, fake, 4096, 262144, 2, 0, 16, fake, 1 << 20, None,
                                      ctypes.byref(h)) == Z.ERR_INVALID_ARG
    assert Z.zipnn_plan_create_packed(Z.FP8_E4M3, fake, 4096, 262144, 2, 0, 3, fake, 1 << 20, None,
                                      ctypes.byref(h)) == Z.ERR_INVALID_ARG
    G = 1

    def plan_bytes(dt, K, pad_byte=0):
        # "ZNP1", dtype, groups, K, 0; one plain record (a 2-symbol code); K > 0: a packed
        # record and the list
        rec = bytearray(128 if dt == Z.BF16 else 16 * 2)
        rec[0] = 0x11
        body = bytes(rec)
        if K:
            prec = bytearray(128)
            prec[0] = 0x11
            lst = bytearray(16)
            lst[:min(K, 16)] = bytes(range(100, 100 + min(K, 16)))
            if pad_byte:
                lst[15] = pad_byte
            body += bytes(prec) + bytes(lst)
        return b"ZNP1" + bytes([dt, G, K, 0]) + body

    for data in (plan_bytes(Z.BF16, 16), plan_bytes(Z.FP8_E4M3, 2), plan_bytes(Z.BF16, 3, pad_byte=7)):
        buf = (ctypes.c_uint8 * len(data)).from_buffer_copy(data)
        assert Z.zipnn_plan_import(buf, len(data), ctypes.byref(h)) == Z.ERR_CORRUPT

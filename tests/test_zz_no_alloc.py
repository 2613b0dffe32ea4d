"""zipnn_compress_noalloc: the compress entry point for callers that cannot allocate
device memory (code whose device memory belongs to a framework's caching allocator it
cannot reach from C, or a latency-critical path that cannot afford the synchronisation
of a cudaMalloc/cudaFree pair). It must produce exactly the container zipnn_compress
produces, call after call, although its fixed scratch array keeps whatever the previous
call left there.
Collected last on purpose: a failure here leaves every other test already run."""
import ctypes

import pytest
import torch

pytestmark = pytest.mark.gpu

CB = 262144


def test_noalloc_matches_compress_on_two_calls():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from lossless_float_weight_b200 import workloads as W
    from lossless_float_weight_b200 import zipnn as Z
    stream = torch.cuda.current_stream().cuda_stream
    # a larger tensor first, then a smaller one, so the second call runs on scratch that
    # still holds the first call's histograms, descriptors and tables
    for n, seed in ((900001, 1), (300007, 2)):
        x = W.bf16_small(n=n, seed=seed).cuda()
        ref = Z.compress(x, chunk_bytes=CB)  # the existing entry point, with its own workspace
        cap = Z.zipnn_max_compressed_bytes(Z.BF16, n, CB)
        out = torch.full((cap,), 0xA5, dtype=torch.uint8, device="cuda")  # no pre-cleared output needed
        st = Z.zipnn_compress_noalloc(Z.BF16, x.data_ptr(), n, CB, out.data_ptr(), cap, stream)
        assert st == Z.OK, Z.zipnn_status_string(st)
        size = Z.compressed_size(out)
        assert size == ref.numel()
        assert torch.equal(out[:size], ref)
        y = Z.decompress(out[:size], torch.bfloat16, n, chunk_bytes=CB)
        assert torch.equal(y.view(torch.int16), x.view(torch.int16))


def test_noalloc_rejects_tensors_beyond_its_scratch():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from lossless_float_weight_b200 import zipnn as Z
    n = 1 << 33  # a workspace far beyond the fixed scratch: refused before any launch
    assert Z.zipnn_workspace_bytes(Z.BF16, n, CB) > Z.NOALLOC_SCRATCH_BYTES
    x = torch.zeros(16, dtype=torch.bfloat16, device="cuda")
    out = torch.zeros(16, dtype=torch.uint8, device="cuda")
    st = Z.zipnn_compress_noalloc(Z.BF16, x.data_ptr(), n, CB, out.data_ptr(), 16,
                                  torch.cuda.current_stream().cuda_stream)
    assert st == Z.ERR_UNSUPPORTED

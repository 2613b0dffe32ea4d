// noalloc.cu -- zipnn_compress_noalloc: compress without any allocation by the caller
// or the library. The workspace is a file-scope device array of fixed size, shared by
// every call on a device.
#include <mutex>

#include "zipnn.h"
#include "launch.h"

namespace {

// Scratch for zipnn_compress_noalloc. Every GPU on which the library is loaded holds
// it until the process exits.
static __device__ __align__(256) unsigned char g_noalloc_scratch[ZIPNN_NOALLOC_SCRATCH_BYTES];

std::mutex g_noalloc_mu;
void* g_noalloc_addr[128] = {nullptr};

}  // namespace

extern "C" zipnn_status zipnn_compress_noalloc(zipnn_dtype dtype, const void* src, uint64_t n, uint32_t chunk_bytes,
                                               void* out, size_t out_cap, zipnn_stream_t stream) {
  if (!src || !out) return ZIPNN_ERR_INVALID_ARG;
  const size_t need = zipnn_workspace_bytes(dtype, n, chunk_bytes);
  if (need == 0) return ZIPNN_ERR_INVALID_ARG;
  if (need > ZIPNN_NOALLOC_SCRATCH_BYTES) return ZIPNN_ERR_UNSUPPORTED;  // tensor beyond the fixed scratch
  // the same device check as zipnn_compress, before the module is touched: on a device
  // the kernels were not built for, the symbol lookup below would fail
  if (!zipnn::device_ok()) return ZIPNN_ERR_UNSUPPORTED;
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 128) {
    cudaGetLastError();
    return ZIPNN_ERR_CUDA;
  }
  void* ws = nullptr;
  {
    // once per device, with that device current: the device address of the array (the
    // host-side symbol is only a stand-in and must never reach a kernel)
    std::lock_guard<std::mutex> lock(g_noalloc_mu);
    if (!g_noalloc_addr[dev]) {
      void* p = nullptr;
      if (cudaGetSymbolAddress(&p, g_noalloc_scratch) != cudaSuccess || !p) {
        cudaGetLastError();  // leave no sticky error behind for the caller's own checks
        return ZIPNN_ERR_CUDA;
      }
      g_noalloc_addr[dev] = p;
    }
    ws = g_noalloc_addr[dev];
  }
  return zipnn_compress(dtype, src, n, chunk_bytes, nullptr, out, out_cap, ws, ZIPNN_NOALLOC_SCRATCH_BYTES, stream);
}

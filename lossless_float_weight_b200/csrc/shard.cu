// shard.cu -- one container from shards compressed on several GPUs.
//
// "ZipNN: Lossless Compression for AI Models" (abstract): a model is many tensors and
// its chunks are coded independently, so the work splits across GPUs with no exchange of
// data. A tensor of n values is cut into contiguous whole-chunk ranges, one per GPU; each
// GPU compresses its range as a tensor of its own (a shard container). The container of
// the whole tensor is the header, the shards' chunk tables with their payload offsets
// moved, the shared records (one plan for all shards), then the shards' payload sections
// one after another. A payload's bytes do not depend on where it lies, so the result is
// byte for byte the container one GPU would write. The only exchange is the exclusive
// scan of the shards' payload sizes.
//   k_shard_sizes : payload bytes of each shard container (total_bytes - off_payload);
//   k_shard_tables: given every rank's sizes, each shard's entries in the whole
//                   container's coordinates, and the whole header for the first shard.
#include <vector>

#include "zipnn.h"
#include "common.cuh"
#include "launch.h"

namespace zipnn {
namespace {

constexpr int kShardThreads = 256;

struct ShardItem {
  const uint8_t* shard;
  uint64_t shard_bytes, n_total, chunk_lo;
  uint8_t* table_out;
  uint8_t* header_out;
};

__device__ __forceinline__ uint64_t ld_u64(const uint8_t* p) { return *reinterpret_cast<const uint64_t*>(p); }

// Payload bytes of every shard; a header that is not a container's gives 0 and CORRUPT.
__global__ void k_shard_sizes(const ShardItem* __restrict__ items, uint32_t count, uint64_t* __restrict__ sizes,
                              uint32_t* status) {
  const uint32_t i = blockIdx.x * blockDim.x + threadIdx.x;
  if (i >= count) return;
  const uint8_t* h = items[i].shard;
  const bool fits = items[i].shard_bytes >= kHeaderBytes;
  const uint32_t magic = fits ? *reinterpret_cast<const uint32_t*>(h) : 0u;
  const uint64_t off_payload = fits ? ld_u64(h + 40) : 0, total = fits ? ld_u64(h + 48) : 0;
  if (magic != 0x314E4E5Au || total < off_payload || total > items[i].shard_bytes) {
    sizes[i] = 0;
    set_status(status, kStCorrupt);
    return;
  }
  sizes[i] = total - off_payload;
}

// One block per item. all_sizes is rank-major: all_sizes[r * count + i] is the payload
// size of item i on rank r. The shard must be the compressed values
// [chunk_lo * m0, min(n_total, (chunk_lo + its chunks) * m0)) with this dtype and chunk
// size; anything else is reported as CORRUPT and nothing is written.
template <int DT>
__global__ void __launch_bounds__(kShardThreads) k_shard_tables(const ShardItem* __restrict__ items, uint32_t count,
                                                                uint32_t chunk_bytes, const uint64_t* __restrict__ all_sizes,
                                                                uint32_t rank, uint32_t world, uint32_t* status) {
  constexpr int NS = n_streams(DT);
  __shared__ uint64_t s_delta;  // added to every local payload offset
  __shared__ uint32_t s_entries;
  __shared__ int s_bad;
  const ShardItem it = items[blockIdx.x];
  const uint32_t m0 = (uint32_t)(8ull * chunk_bytes / (uint32_t)value_bits(DT));
  if (threadIdx.x == 0 && it.shard_bytes < kHeaderBytes) {
    s_bad = 1;
    set_status(status, kStCorrupt);
  } else if (threadIdx.x == 0) {
    int bad = 0;
    const uint32_t* hv = reinterpret_cast<const uint32_t*>(it.shard);
    const uint64_t n = ld_u64(it.shard + 8), off_codes = ld_u64(it.shard + 32);
    const uint64_t off_payload = ld_u64(it.shard + 40), total = ld_u64(it.shard + 48);
    const uint32_t n_chunks = hv[6], G = (hv[14] >> 8) & 0xFF, K = (hv[14] >> 16) & 0xFF;
    const uint64_t C = ceil_div(it.n_total, m0);
    const uint64_t v_lo = it.chunk_lo * (uint64_t)m0;
    if (hv[0] != 0x314E4E5Au || hv[1] != (1u | ((uint32_t)DT << 16) | ((uint32_t)NS << 24))) bad = 1;
    if (hv[4] != chunk_bytes || v_lo >= it.n_total) bad = 1;
    if (!bad && (n != min64(it.n_total - v_lo, (uint64_t)n_chunks * m0) || n_chunks != ceil_div(n, m0))) bad = 1;
    if (G > kMaxGroups || K > kPackMax || off_codes != kHeaderBytes + (uint64_t)kEntryBytes * n_chunks * NS) bad = 1;
    if (off_payload != off_codes + code_section_bytes(DT, G, K) || total < off_payload || total > it.shard_bytes)
      bad = 1;
    // this shard's place among the shards of the item, and the whole payload size
    uint64_t base = 0, sum = 0;
    for (uint32_t r = 0; r < world; r++) {
      const uint64_t sz = all_sizes[(uint64_t)r * count + blockIdx.x];
      if (r < rank) base += sz;
      sum += sz;
    }
    if (all_sizes[(uint64_t)rank * count + blockIdx.x] != total - off_payload) bad = 1;
    const uint64_t off_codes_g = kHeaderBytes + (uint64_t)kEntryBytes * C * NS;
    const uint64_t off_payload_g = off_codes_g + code_section_bytes(DT, G, K);
    s_delta = off_payload_g + base - off_payload;
    s_entries = n_chunks * NS;
    s_bad = bad;
    if (bad) set_status(status, kStCorrupt);
    if (!bad && it.header_out) {
      uint32_t h[16];
      for (int i = 0; i < 16; i++) h[i] = hv[i];
      h[2] = (uint32_t)it.n_total;
      h[3] = (uint32_t)(it.n_total >> 32);
      h[6] = (uint32_t)C;
      h[8] = (uint32_t)off_codes_g;
      h[9] = (uint32_t)(off_codes_g >> 32);
      h[10] = (uint32_t)off_payload_g;
      h[11] = (uint32_t)(off_payload_g >> 32);
      const uint64_t tb = off_payload_g + sum;
      h[12] = (uint32_t)tb;
      h[13] = (uint32_t)(tb >> 32);
      for (int i = 0; i < 16; i++) reinterpret_cast<uint32_t*>(it.header_out)[i] = h[i];
    }
  }
  __syncthreads();
  if (s_bad) return;
  const uint64_t delta = s_delta;
  const uint4* src = reinterpret_cast<const uint4*>(it.shard + kHeaderBytes);
  uint4* dst = reinterpret_cast<uint4*>(it.table_out);
  for (uint32_t k = threadIdx.x; k < s_entries; k += kShardThreads) {
    uint4 e = src[k];
    const uint64_t off = (e.z | ((uint64_t)e.w << 32)) + delta;
    e.z = (uint32_t)off;
    e.w = (uint32_t)(off >> 32);
    dst[k] = e;
  }
}

}  // namespace
}  // namespace zipnn

using namespace zipnn;

namespace {

constexpr size_t kShardTableOffset = 256;  // the item table's place in ws, after the status word

inline bool aligned16p(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15) == 0; }

// Copy the host items into ws (stream-ordered) after clearing the status word.
zipnn_status stage_items(uint32_t count, const zipnn_shard_item* items, void* ws, size_t ws_bytes, cudaStream_t st,
                         ShardItem** dev_items) {
  if (!items || !ws || count == 0 || !aligned16p(ws)) return ZIPNN_ERR_INVALID_ARG;
  if (ws_bytes < zipnn_shard_workspace_bytes(count)) return ZIPNN_ERR_OUT_TOO_SMALL;
  std::vector<ShardItem> table(count);
  for (uint32_t i = 0; i < count; i++) {
    const zipnn_shard_item& s = items[i];
    if (!s.shard || !aligned16p(s.shard)) return ZIPNN_ERR_INVALID_ARG;
    table[i] = ShardItem{static_cast<const uint8_t*>(s.shard), s.shard_bytes, s.n_total, s.chunk_lo,
                         static_cast<uint8_t*>(s.table_out), static_cast<uint8_t*>(s.header_out)};
  }
  if (!device_ok()) return ZIPNN_ERR_UNSUPPORTED;
  *dev_items = reinterpret_cast<ShardItem*>(static_cast<uint8_t*>(ws) + kShardTableOffset);
  cudaError_t e = cudaMemsetAsync(ws, 0, 4, st);
  if (e == cudaSuccess) e = cudaMemcpyAsync(*dev_items, table.data(), count * sizeof(ShardItem), cudaMemcpyHostToDevice, st);
  return e == cudaSuccess ? ZIPNN_OK : ZIPNN_ERR_CUDA;
}

}  // namespace

extern "C" {

size_t zipnn_shard_workspace_bytes(uint32_t count) {
  return kShardTableOffset + (((size_t)count * sizeof(ShardItem) + 255) & ~(size_t)255);
}

zipnn_status zipnn_shard_sizes(uint32_t count, const zipnn_shard_item* items, uint64_t* sizes_out, void* ws,
                               size_t ws_bytes, zipnn_stream_t stream) {
  if (!sizes_out) return ZIPNN_ERR_INVALID_ARG;
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  ShardItem* dev = nullptr;
  zipnn_status zs = stage_items(count, items, ws, ws_bytes, st, &dev);
  if (zs != ZIPNN_OK) return zs;
  TimedLaunch t(kIdShard, st);
  k_shard_sizes<<<(count + kShardThreads - 1) / kShardThreads, kShardThreads, 0, st>>>(dev, count, sizes_out,
                                                                                    static_cast<uint32_t*>(ws));
  return cudaGetLastError() == cudaSuccess ? ZIPNN_OK : ZIPNN_ERR_CUDA;
}

zipnn_status zipnn_shard_tables(zipnn_dtype dtype, uint32_t chunk_bytes, uint32_t count, const zipnn_shard_item* items,
                                const uint64_t* all_sizes, uint32_t rank, uint32_t world, void* ws, size_t ws_bytes,
                                zipnn_stream_t stream) {
  if (!all_sizes || world == 0 || rank >= world) return ZIPNN_ERR_INVALID_ARG;
  if (dtype != ZIPNN_BF16 && dtype != ZIPNN_FP32 && dtype != ZIPNN_FP8_E4M3 && dtype != ZIPNN_FP4_E2M1)
    return ZIPNN_ERR_INVALID_ARG;
  if (chunk_bytes < 16 || chunk_bytes % 16 || chunk_bytes > (1u << 28)) return ZIPNN_ERR_INVALID_ARG;
  if (items)
    for (uint32_t i = 0; i < count; i++)
      if (!items[i].table_out || !aligned16p(items[i].table_out) ||
          (items[i].header_out && !aligned16p(items[i].header_out)) || items[i].n_total == 0)
        return ZIPNN_ERR_INVALID_ARG;
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  ShardItem* dev = nullptr;
  zipnn_status zs = stage_items(count, items, ws, ws_bytes, st, &dev);
  if (zs != ZIPNN_OK) return zs;
  uint32_t* status = static_cast<uint32_t*>(ws);
  TimedLaunch t(kIdShard, st);
  switch (dtype) {
    case ZIPNN_BF16: k_shard_tables<kBF16><<<count, kShardThreads, 0, st>>>(dev, count, chunk_bytes, all_sizes, rank, world, status); break;
    case ZIPNN_FP32: k_shard_tables<kFP32><<<count, kShardThreads, 0, st>>>(dev, count, chunk_bytes, all_sizes, rank, world, status); break;
    case ZIPNN_FP8_E4M3: k_shard_tables<kFP8><<<count, kShardThreads, 0, st>>>(dev, count, chunk_bytes, all_sizes, rank, world, status); break;
    default: k_shard_tables<kFP4><<<count, kShardThreads, 0, st>>>(dev, count, chunk_bytes, all_sizes, rank, world, status); break;
  }
  return cudaGetLastError() == cudaSuccess ? ZIPNN_OK : ZIPNN_ERR_CUDA;
}

}  // extern "C"

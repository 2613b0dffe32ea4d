// encode_cluster.cu -- BF16 encode with thread-block clusters.
//
// The same work as k_encode (encode.cu) for BF16 chunks of at most 8 tiles of 16384
// values: one cluster per chunk (cluster i encodes chunk i), one block per tile.
// Each block packs its exponent codes into shared memory, and its bit offset inside
// the chunk is the sum of the lower blocks' bit counts, read over distributed shared
// memory (DSMEM) after a cluster barrier: no global look-back between the tiles of a
// chunk, and no dependence between clusters. Words shared by two tiles are merged as
// in k_encode. A block arrives on the closing cluster barrier as soon as its DSMEM
// reads are done and waits on it only before it exits (its shared memory must outlive
// the other blocks' reads).
#include <cooperative_groups.h>

#include "common.cuh"
#include "fields.cuh"
#include "launch.h"

namespace cg = cooperative_groups;

namespace zipnn {

constexpr int kFValues = kGroupValues * kEncGroups;        // 64 values per thread
constexpr int kFStageWords = kTileValues * kLmax / 32 + 2;  // one tile's bitstream
constexpr int kFPrivStride = kFValues * kLmax / 32 + 1;     // odd: conflict-free
constexpr int kMaxCluster = 8;

struct FusedSmem {
  struct {
    uint32_t priv[kEncodeThreads * kFPrivStride];  // each thread's codes, packed from bit 0
    uint32_t stage[kFStageWords];                  // the tile's bitstream at its final alignment
  } pack;
  uint32_t enc[256];   // the chunk's code: len << 16 | code
  uint32_t warp[kEncodeThreads / 32];
  uint32_t tile_bits;  // this tile's exponent bits (read by later blocks over DSMEM)
};

// Merge a word shared by two tiles: the second arrival stores the union.
__device__ __forceinline__ void cluster_slot_merge(uint64_t* slot, uint32_t part, uint32_t* dst) {
  const uint64_t old = atomicAdd(reinterpret_cast<unsigned long long*>(slot), (1ull << 32) | (uint64_t)part);
  if ((old >> 32) == 1) *dst = bswap32((uint32_t)old | part);
}

// Exponent (s == 0) or sign/fraction byte (s == 1) of two BF16 values, in bytes 0 and 2.
__device__ __forceinline__ uint32_t bf16_pair_plane(uint32_t w, int s) {
  return s == 0 ? (w >> 7) & 0x00FF00FFu : (w & 0x007F007Fu) | ((w >> 8) & 0x00800080u);
}

__global__ void __launch_bounds__(kEncodeThreads) k_encode_bf16_cluster(const uint8_t* __restrict__ src, Geo g, Ws ws,
                                                                        uint8_t* __restrict__ out) {
  cg::cluster_group cluster = cg::this_cluster();
  const uint32_t T = cluster.num_blocks(), rank = cluster.block_rank();
  extern __shared__ __align__(16) uint8_t smem_raw[];
  FusedSmem& sm = *reinterpret_cast<FusedSmem*>(smem_raw);
  const int tid = threadIdx.x, lane = tid & 31;
  const uint32_t c = blockIdx.x / T;
  const uint64_t clo = (uint64_t)c * g.m0;
  const uint32_t m = (uint32_t)min64(g.m0, g.n - clo);
  const uint32_t tlo = rank * (uint32_t)kTileValues;
  const bool live = tlo < m;                                  // the block has values
  const bool last = live && tlo + (uint32_t)kTileValues >= m;  // the chunk's last tile
  const uint32_t v0 = tlo + tid * kFValues;
  const int cnt = v0 < m ? (int)min32(kFValues, m - v0) : 0;
  RawValues<kBF16, kFValues> raw;
  if (cnt > 0) load_values<kBF16, kFValues>(src + (clo + v0) * 2, cnt, raw);

  // the chunk's decisions and code, from the code build
  uint32_t mode[2], code0;
  uint64_t off[2];
  mode[0] = ws.emode[2ull * c];
  mode[1] = ws.emode[2ull * c + 1];
  code0 = ws.ecode[2ull * c];
  off[0] = ws.eoff[2ull * c];
  off[1] = ws.eoff[2ull * c + 1];
  if (mode[0] == kModeHuff) sm.enc[tid] = ws.enc[(uint64_t)c * 256 + tid];
  __syncthreads();
  const uint64_t nsub = ceil_div(m, g.S);

#pragma unroll
  for (int s = 0; s < 2; s++) {
    if (mode[s] != kModeRaw || !live) continue;
    // RAW byte plane (the sign/fraction bytes; an exponent stream that did not compress)
    if (cnt == kFValues) {
#pragma unroll
      for (int q = 0; q < kFValues / 16; q++) {
        uint32_t x[4];
#pragma unroll
        for (int k = 0; k < 4; k++)
          x[k] = __byte_perm(bf16_pair_plane(raw.w[8 * q + 2 * k], s), bf16_pair_plane(raw.w[8 * q + 2 * k + 1], s),
                             0x6420);
        *reinterpret_cast<uint4*>(out + off[s] + v0 + 16 * q) = make_uint4(x[0], x[1], x[2], x[3]);
      }
    } else {
#pragma unroll
      for (int q = 0; q < kFValues / 16; q++) {
        if (16 * q < cnt) {
          uint32_t x[4];
#pragma unroll
          for (int j = 0; j < 4; j++) {
            x[j] = 0;
#pragma unroll
            for (int b = 0; b < 4; b++) {
              const int i = 16 * q + 4 * j + b;
              if (i < cnt) x[j] |= symbol<kBF16, kFValues>(raw, s, i) << (8 * b);
            }
          }
          *reinterpret_cast<uint4*>(out + off[s] + v0 + 16 * q) = make_uint4(x[0], x[1], x[2], x[3]);
        }
      }
    }
  }

  if (mode[0] == kModeHuff) {
    const uint32_t rec = code0 == kNoCode ? record_bytes(kBF16, 0) : 0;
    const uint64_t idx_bytes = round16(4 * nsub);
    uint8_t* payload = out + off[0];
    uint32_t* idx = reinterpret_cast<uint32_t*>(payload + rec);
    uint32_t* bs = reinterpret_cast<uint32_t*>(payload + rec + idx_bytes);
    // the local code record heads the payload (4-bit lengths)
    if (rec && rank == 0 && tid < 128)
      payload[tid] = (uint8_t)((sm.enc[2 * tid] >> 16) | ((sm.enc[2 * tid + 1] >> 16) << 4));
    // pack my codes from bit 0 of my private words
    uint32_t* pw = sm.pack.priv + tid * kFPrivStride;
    uint32_t nw = 0, nfill = 0, mybits = 0;
    uint32_t qoff[kFValues / 16];
    uint64_t acc = 0;
    if (cnt == kFValues) {
      // two values (one input word) per step: the exponent of the low value is bits
      // 14..7, so its table entry is at byte offset (w >> 5) & 0x3FC, the high one's at
      // (w >> 21) & 0x3FC. The two codes (at most 24 bits) join before they enter the
      // accumulator, which then holds fewer than 56 pending bits: one flush test a pair.
      const uint8_t* encb = reinterpret_cast<const uint8_t*>(sm.enc);
#pragma unroll
      for (int j = 0; j < kFValues / 2; j++) {
        if ((j & 7) == 0) qoff[j >> 3] = nw * 32 + nfill;
        const uint32_t w = raw.w[j];
        const uint32_t e0 = *reinterpret_cast<const uint32_t*>(encb + ((w >> 5) & 0x3FCu));
        const uint32_t e1 = *reinterpret_cast<const uint32_t*>(encb + ((w >> 21) & 0x3FCu));
        const uint32_t l1 = e1 >> 16;
        const uint32_t l = (e0 >> 16) + l1;
        acc = (acc << l) | (((e0 & 0xFFFFu) << l1) | (e1 & 0xFFFFu));
        nfill += l;
        if (nfill >= 32) {
          nfill -= 32;
          pw[nw++] = (uint32_t)(acc >> nfill);
        }
      }
      mybits = nw * 32 + nfill;
    } else {
#pragma unroll
      for (int i = 0; i < kFValues; i++) {
        if ((i & 15) == 0) qoff[i >> 4] = mybits;
        if (i < cnt) {
          const uint32_t e = sm.enc[symbol<kBF16, kFValues>(raw, 0, i)];
          const uint32_t l = e >> 16;
          mybits += l;
          acc = (acc << l) | (e & 0xFFFFu);
          nfill += l;
          const bool full = nfill >= 32;
          nfill -= full ? 32u : 0u;
          const uint32_t word = (uint32_t)(acc >> nfill);
          if (full) pw[nw] = word;
          nw += full ? 1u : 0u;
        }
      }
    }
    if (nfill) pw[nw++] = (uint32_t)(acc << (32 - nfill));
    uint32_t tile_bits;
    const uint32_t myoff = block_exclusive_scan<kEncodeThreads>(mybits, sm.warp, tile_bits);
    if (tid == 0) sm.tile_bits = tile_bits;
    const uint32_t nw_max = (31 + tile_bits + 31) / 32;
    for (uint32_t i = tid; i < nw_max; i += kEncodeThreads) sm.pack.stage[i] = 0;
    cluster.sync();
    // this tile's bit offset in the chunk: the lower tiles' bits, lane r reading rank r
    const uint32_t lower = (uint32_t)lane < rank ? cluster.map_shared_rank(&sm, (unsigned)lane)->tile_bits : 0u;
    const uint64_t P = __reduce_add_sync(0xFFFFFFFFu, lower);
    cluster.barrier_arrive();
    if (cnt > 0) {
      uint32_t rr = v0 % g.S;
#pragma unroll
      for (int q = 0; q < kFValues / 16; q++) {
        if (rr == 0 && 16 * q < cnt) idx[(v0 + 16 * q) / g.S] = (uint32_t)(P + myoff + qoff[q]);
        rr += 16;
        if (rr >= g.S) rr -= g.S;
      }
    }
    if (mybits) {
      const uint32_t q0 = (uint32_t)(P & 31) + myoff;
      const uint32_t sh = q0 & 31, d0 = q0 >> 5, dlast = (q0 + mybits - 1) >> 5;
      uint32_t prev = 0;
      for (uint32_t k = 0; k <= dlast - d0; k++) {
        const uint32_t cur = k < nw ? pw[k] : 0u;
        const uint32_t o = (sh ? prev << (32 - sh) : 0u) | (cur >> sh);
        if (k == 0 || k == dlast - d0) atomicOr(sm.pack.stage + d0 + k, o);
        else sm.pack.stage[d0 + k] = o;
        prev = cur;
      }
    }
    __syncthreads();
    if (live) {
      const uint64_t end = P + tile_bits;
      const uint32_t nwt = (uint32_t)(((P & 31) + tile_bits + 31) >> 5);
      const uint64_t W0 = P >> 5;
      const uint64_t gtile = (uint64_t)c * g.tiles_per_chunk + rank;
      for (uint32_t i = tid; i < nwt; i += kEncodeThreads) {
        const uint32_t word = sm.pack.stage[i];
        uint32_t* dst = bs + W0 + i;
        if (i == 0 && (P & 31) != 0) cluster_slot_merge(ws.slot + gtile, word, dst);
        else if (i == nwt - 1 && (end & 31) != 0 && !last) cluster_slot_merge(ws.slot + gtile + 1, word, dst);
        else *dst = bswap32(word);
      }
      if (last) {
        const uint64_t padded_words = round16(ceil_div(end, 8)) / 4;
        for (uint64_t i = W0 + nwt + tid; i < padded_words; i += kEncodeThreads) bs[i] = 0;
        for (uint64_t i = nsub + tid; i < idx_bytes / 4; i += kEncodeThreads) idx[i] = 0;
      }
    }
  } else {
    cluster.barrier_arrive();
  }
  // no block leaves while another may still read its shared memory
  cluster.barrier_wait();
}

// Launch: one cluster of tiles_per_chunk blocks per chunk.
cudaError_t launch_encode_bf16_cluster(const void* src, const Geo& g, const Ws& ws, uint8_t* out, cudaStream_t st) {
  const size_t smem = sizeof(FusedSmem);
  static int done[128] = {0};
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  if (dev < 0 || dev >= 128 || !done[dev]) {
    e = cudaFuncSetAttribute(k_encode_bf16_cluster, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e == cudaSuccess) e = cudaFuncSetAttribute(k_encode_bf16_cluster, cudaFuncAttributePreferredSharedMemoryCarveout, 100);
    if (e != cudaSuccess) return e;
    if (dev >= 0 && dev < 128) done[dev] = 1;
  }
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(g.n_chunks * g.tiles_per_chunk, 1, 1);
  cfg.blockDim = dim3(kEncodeThreads, 1, 1);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = st;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = g.tiles_per_chunk;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, k_encode_bf16_cluster, static_cast<const uint8_t*>(src), g, ws, out);
}

bool cluster_encode_applies(const Geo& g) {
  return g.dt == kBF16 && g.tiles_per_chunk >= 1 && g.tiles_per_chunk <= kMaxCluster &&
         (uint64_t)g.n_chunks * g.tiles_per_chunk <= 0x7FFFFFFFull;
}

}  // namespace zipnn

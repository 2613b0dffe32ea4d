// encode.cu -- k_encode: writes every payload byte of an FP32 container (BF16 has
// k_encode_bf16, FP8 and FP4 k_encode_sub; the kernel is written for any type, and the
// sub-byte RAW branch below serves only those).
//
// One block per tile of 16384 values of one chunk; each of the 256 threads owns 64
// consecutive values, all loaded up front (128-bit loads) so that a block keeps
// 64 KB of input in flight.
//  * byte planes (the three fraction planes; an exponent that did not compress) go out
//    as 16-byte stores, RAW at the values' own offset, ZRUN only for marked blocks.
//  * HUFF: each thread sums the code lengths of its symbols; a block-wide warp-shuffle
//    scan gives its bit offset inside the tile; the tile's offset inside the chunk comes
//    from the previous tiles of the same chunk by single-pass decoupled look-back (one
//    warp inspects 32 predecessors at a time). Codes are emitted most significant bit
//    first into a shared staging buffer, whole words with plain stores and the two edge
//    words of each thread with shared atomicOr; the block then stores the staged words.
//    A word that straddles two tiles is merged in a workspace slot: each side adds
//    (1 << 32 | its bits) and the side that arrives second stores the complete word, so
//    no output pre-clearing and no wait between blocks is needed.
//  * the sub-block index idx[j] (bit offset of symbol j*S) is written by the thread
//    that owns symbol j*S; the first tile writes a local code record, the last tile the
//    zero padding.
#include <atomic>

#include "common.cuh"
#include "fields.cuh"
#include "launch.h"

namespace zipnn {

constexpr int kEncValues = kGroupValues * kEncGroups;     // values per thread
constexpr int kStageWords = kTileValues * kLmax / 32 + 2;  // staged bits of one stream
constexpr int kPrivStride = kEncValues * kLmax / 32 + 1;   // private words per thread (odd: conflict-free)

// Merge a word shared by two tiles: the second arrival stores the union.
__device__ __forceinline__ void slot_merge(uint64_t* slot, uint32_t part, uint32_t* dst) {
  const uint64_t old = atomicAdd(reinterpret_cast<unsigned long long*>(slot), (1ull << 32) | (uint64_t)part);
  if ((old >> 32) == 1) *dst = bswap32((uint32_t)old | part);
}

// Shared memory of one encode block.
template <int DT>
struct EncodeSmem {
  uint32_t priv[kEncodeThreads * kPrivStride];  // each thread's codes, packed from bit 0
  uint32_t stage[kStageWords];                  // the tile's bitstream, at its final bit alignment
  uint32_t enc[n_entropy(DT)][256];
  uint32_t warp[kEncodeThreads / 32];
  uint32_t zmap[32];  // ZRUN byte plane: the tile's block-bitmap words (16 of them)
  uint32_t zpre[32];  // marked blocks of the chunk before each of those words
  uint64_t prefix;
  uint64_t off[n_streams(DT)];
  uint32_t mode[n_streams(DT)], code[n_streams(DT)];
  uint32_t tile;
};

template <int DT>
__global__ void __launch_bounds__(kEncodeThreads) k_encode(const uint8_t* __restrict__ src, Geo g, Ws ws,
                                                           uint8_t* __restrict__ out) {
  constexpr int NS = n_streams(DT), NE = n_entropy(DT);
  constexpr int NB = DT == kFP8 || DT == kFP4 ? 3 : 1;  // streams that may be bit-packed
  extern __shared__ __align__(16) uint8_t smem_raw[];
  EncodeSmem<DT>& sm = *reinterpret_cast<EncodeSmem<DT>*>(smem_raw);
  const int tid = threadIdx.x;
  if (tid == 0) sm.tile = atomicAdd(&ws.status[1], 1u);
  __syncthreads();
  const uint32_t tile = sm.tile;
  const uint32_t c = tile / g.tiles_per_chunk, ti = tile % g.tiles_per_chunk;
  const uint64_t clo = (uint64_t)c * g.m0;
  const uint32_t m = (uint32_t)min64(g.m0, g.n - clo);
  const uint32_t tlo = ti * (uint32_t)kTileValues;
  if (tlo >= m) return;  // past the end of a ragged last chunk
  const bool last = tlo + (uint32_t)kTileValues >= m;

  const uint32_t v0 = tlo + tid * kEncValues;  // chunk-relative index of my first value
  const int cnt = v0 < m ? (int)min32(kEncValues, m - v0) : 0;
  RawValues<DT, kEncValues> raw;
  if (cnt > 0) load_values<DT, kEncValues>(src + value_offset(DT, clo + v0), cnt, raw);

  if (tid < NS) {
    const uint64_t k = (uint64_t)c * NS + tid;
    sm.mode[tid] = ws.emode[k];
    sm.code[tid] = ws.ecode[k];
    sm.off[tid] = ws.eoff[k];
  }
#pragma unroll
  for (int e = 0; e < NE; e++) sm.enc[e][tid] = ws.enc[((uint64_t)c * NE + e) * 256 + tid];
  __syncthreads();
  const uint64_t nsub = ceil_div(m, g.S);

#pragma unroll
  for (int s = 0; s < NS; s++) {
    const uint32_t mode = sm.mode[s];
    if (mode == kModeZero) continue;
    const int w = raw_width(DT, s);
    if (mode == kModeRaw && w == 8) {
      if constexpr (DT == kBF16) {
        if (cnt == kEncValues) {
          // two values at a time: the exponent is bits 14..7 of each half, the
          // sign/fraction byte bits 15 and 6..0
#pragma unroll
          for (int q = 0; q < kEncValues / 16; q++) {
            uint32_t x[4];
#pragma unroll
            for (int k = 0; k < 4; k++) {
              const uint32_t a = raw.w[8 * q + 2 * k], b = raw.w[8 * q + 2 * k + 1];
              const uint32_t ta = s == 0 ? (a >> 7) & 0x00FF00FFu : (a & 0x007F007Fu) | ((a >> 8) & 0x00800080u);
              const uint32_t tb = s == 0 ? (b >> 7) & 0x00FF00FFu : (b & 0x007F007Fu) | ((b >> 8) & 0x00800080u);
              x[k] = __byte_perm(ta, tb, 0x6420);
            }
            *reinterpret_cast<uint4*>(out + sm.off[s] + v0 + 16 * q) = make_uint4(x[0], x[1], x[2], x[3]);
          }
          continue;
        }
      }
#pragma unroll
      for (int q = 0; q < kEncValues / 16; q++) {
        if (16 * q < cnt) {
          uint32_t x[4];
#pragma unroll
          for (int j = 0; j < 4; j++) {
            x[j] = 0;
#pragma unroll
            for (int b = 0; b < 4; b++) {
              const int i = 16 * q + 4 * j + b;
              if (i < cnt) x[j] |= symbol<DT, kEncValues>(raw, s, i) << (8 * b);
            }
          }
          *reinterpret_cast<uint4*>(out + sm.off[s] + v0 + 16 * q) = make_uint4(x[0], x[1], x[2], x[3]);
        }
      }
      continue;
    }
    if (mode == kModeZrun) {
      if constexpr (n_byte_planes(DT) > 0) {
        // zero runs of a byte plane: the tile's 512 blocks are bitmap words 16 ti ..
        // 16 ti + 15; warp 0 loads them with each word's rank base (the chunk's marked
        // blocks before it) and writes them into the payload's bitmap (MSB first), the
        // last tile also the bitmap's zero padding
        constexpr uint32_t kTileWords = kTileValues / kZBlock / 32;
        const uint64_t map_bytes = zrun_map_bytes(m);
        if (tid < 32) {
          const uint32_t* map = ws.zmap + ((uint64_t)c * n_byte_planes(DT) + (s - 1)) * g.zwords;
          const uint32_t w0 = ti * kTileWords, used = (uint32_t)ceil_div(ceil_div(m, kZBlock), 32);
          uint32_t base = 0;
          for (uint32_t w = tid; w < w0; w += 32) base += __popc(__ldcg(map + w));
          base = __reduce_add_sync(0xFFFFFFFFu, base);
          const uint32_t word = (tid < (int)kTileWords && w0 + tid < used) ? __ldcg(map + w0 + tid) : 0u;
          const uint32_t pc = __popc(word);
          uint32_t incl = pc;
#pragma unroll
          for (int o = 1; o < 32; o <<= 1) {
            const uint32_t y = __shfl_up_sync(0xFFFFFFFFu, incl, o);
            if (tid >= o) incl += y;
          }
          sm.zmap[tid] = word;
          sm.zpre[tid] = base + incl - pc;
          uint32_t* mp = reinterpret_cast<uint32_t*>(out + sm.off[s]);
          if (tid < (int)kTileWords && w0 + tid < used) mp[w0 + tid] = __byte_perm(__brev(word), 0, 0x0123);
          if (last)
            for (uint32_t w = used + tid; w < map_bytes / 4; w += 32) mp[w] = 0;
        }
        __syncthreads();
        // my values are blocks v0 / 32 and v0 / 32 + 1: a marked block's bytes go to 32 x
        // (its rank) after the bitmap, in 16-byte groups (zero past cnt, so the chunk's
        // short last block ends with its padding); an unmarked block is not stored
        if (cnt > 0) {
          uint8_t* half[2];
#pragma unroll
          for (int h = 0; h < 2; h++) {
            const uint32_t lb = (v0 - tlo) / kZBlock + (uint32_t)h;
            const uint32_t word = sm.zmap[lb >> 5], bit = lb & 31u;
            half[h] = ((word >> bit) & 1u) ? out + sm.off[s] + map_bytes +
                                                 (uint64_t)(sm.zpre[lb >> 5] + __popc(word & ((1u << bit) - 1u))) * kZBlock
                                           : nullptr;
          }
#pragma unroll
          for (int q = 0; q < kEncValues / 16; q++) {
            if (16 * q < cnt && half[q >> 1]) {
              uint32_t x[4];
#pragma unroll
              for (int j = 0; j < 4; j++) {
                x[j] = 0;
#pragma unroll
                for (int b = 0; b < 4; b++) {
                  const int i = 16 * q + 4 * j + b;
                  if (i < cnt) x[j] |= symbol<DT, kEncValues>(raw, s, i) << (8 * b);
                }
              }
              *reinterpret_cast<uint4*>(half[q >> 1] + 16 * (q & 1)) = make_uint4(x[0], x[1], x[2], x[3]);
            }
          }
        }
        __syncthreads();  // the next stream's tables may reuse zmap / zpre
      }
      continue;
    }
    if (s >= NB) continue;  // unreachable: only streams < NB can be bit-packed
    if (mode == kModeRaw) {
      // a RAW stream of w < 8 bits a symbol: value v starts at bit v * w of the payload,
      // and my 64 values fill 2w whole words from word v0 * w / 32, so I pack them in
      // registers and store the words myself (no scan, no staging, no shared edge words).
      // The last value's word ends in zero bits; the chunk's last tile zeroes the words
      // after it up to the payload's 16-byte padding.
      static_assert(kEncValues * 1 % 32 == 0, "64 values of any width are whole words");
      uint32_t* words = reinterpret_cast<uint32_t*>(out + sm.off[s]);
      const uint32_t wbase = (uint32_t)((uint64_t)v0 * w / 32);
      if (cnt > 0) {
        uint64_t acc = 0;
        uint32_t nfill = 0, nw = 0;
#pragma unroll
        for (int i = 0; i < kEncValues; i++) {
          if (i < cnt) {
            acc = (acc << w) | symbol<DT, kEncValues>(raw, s, i);
            nfill += (uint32_t)w;
            if (nfill >= 32) {
              nfill -= 32;
              words[wbase + nw++] = bswap32((uint32_t)(acc >> nfill));
            }
          }
        }
        if (nfill) words[wbase + nw] = bswap32((uint32_t)(acc << (32 - nfill)));
      }
      if (last) {
        const uint64_t used = ceil_div((uint64_t)m * w, 32), padded = raw_payload(m, w) / 4;
        for (uint64_t i = used + tid; i < padded; i += kEncodeThreads) words[i] = 0;
      }
      continue;
    }
    const bool huff = mode == kModeHuff;
    const uint32_t* enc = sm.enc[s < NE ? s : 0];
    // pack my codes, most significant bit first, into my private words from bit 0
    uint32_t* pw = sm.priv + tid * kPrivStride;
    uint32_t mybits = 0, nw = 0, nfill = 0;
    uint32_t qoff[kEncValues / 16];
    uint64_t acc = 0;
    if (huff && cnt == kEncValues) {
      // the common case, without per-value guards; a full word is written (predicated)
      // whenever 32 bits are pending
#pragma unroll
      for (int i = 0; i < kEncValues; i++) {
        if ((i & 15) == 0) qoff[i >> 4] = mybits;
        const uint32_t e = enc[symbol<DT, kEncValues>(raw, s, i)];
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
    } else {
#pragma unroll
      for (int i = 0; i < kEncValues; i++) {
        if ((i & 15) == 0) qoff[i >> 4] = mybits;
        if (i < cnt) {
          const uint32_t sy = symbol<DT, kEncValues>(raw, s, i);
          uint32_t l, cv;
          if (huff) {
            const uint32_t e = enc[sy];
            l = e >> 16;
            cv = e & 0xFFFFu;
          } else {
            l = (uint32_t)w;
            cv = sy;
          }
          mybits += l;
          acc = (acc << l) | cv;
          nfill += l;
          if (nfill >= 32) {
            nfill -= 32;
            pw[nw++] = (uint32_t)(acc >> nfill);
          }
        }
      }
    }
    if (nfill) pw[nw++] = (uint32_t)(acc << (32 - nfill));
    uint32_t tile_bits;
    const uint32_t myoff = block_exclusive_scan<kEncodeThreads>(mybits, sm.warp, tile_bits);
    const uint32_t rec = (huff && sm.code[s] == kNoCode) ? record_bytes(DT, s) : 0;
    const uint64_t idx_bytes = huff ? round16(4 * nsub) : 0;
    uint8_t* payload = out + sm.off[s];
    uint32_t* bs = reinterpret_cast<uint32_t*>(payload + rec + idx_bytes);
    if (tid < 32) {
      if (huff) {
        const uint32_t e = s < NE ? s : 0;
        const uint64_t p =
            warp_lookback(ws.tile_desc + (uint64_t)e * g.n_tiles, tile, c * g.tiles_per_chunk, tile_bits, ws.status,
                          g.spin_limit);
        if (tid == 0) sm.prefix = p;
      } else if (tid == 0) {
        sm.prefix = (uint64_t)tlo * (uint64_t)w;
      }
    }
    const uint32_t nw_max = (31 + tile_bits + 31) / 32;
    for (uint32_t i = tid; i < nw_max; i += kEncodeThreads) sm.stage[i] = 0;
    __syncthreads();
    const uint64_t P = sm.prefix;
    if (huff && cnt > 0) {
      // sub-block index entries that fall at one of my 16-value groups
      uint32_t r = v0 % g.S;
      uint32_t* idx = reinterpret_cast<uint32_t*>(payload + rec);
#pragma unroll
      for (int q = 0; q < kEncValues / 16; q++) {
        if (r == 0 && 16 * q < cnt) idx[(v0 + 16 * q) / g.S] = (uint32_t)(P + myoff + qoff[q]);
        r += 16;
        if (r >= g.S) r -= g.S;
      }
    }
    if (mybits) {
      // move my words into the tile staging at bit (P mod 32) + myoff
      const uint32_t q0 = (uint32_t)(P & 31) + myoff;
      const uint32_t sh = q0 & 31, d0 = q0 >> 5, dlast = (q0 + mybits - 1) >> 5;
      uint32_t prev = 0;
      for (uint32_t k = 0; k <= dlast - d0; k++) {
        const uint32_t cur = k < nw ? pw[k] : 0u;
        const uint32_t o = (sh ? prev << (32 - sh) : 0u) | (cur >> sh);
        if (k == 0 || k == dlast - d0) atomicOr(sm.stage + d0 + k, o);
        else sm.stage[d0 + k] = o;
        prev = cur;
      }
    }
    __syncthreads();
    const uint64_t end = P + tile_bits;
    const uint32_t nwt = (uint32_t)(((P & 31) + tile_bits + 31) >> 5);
    const uint64_t W0 = P >> 5;
    const uint32_t e = s < NE ? s : 0;
    for (uint32_t i = tid; i < nwt; i += kEncodeThreads) {
      const uint32_t word = sm.stage[i];
      uint32_t* dst = bs + W0 + i;
      if (i == 0 && (P & 31) != 0) {
        slot_merge(ws.slot + (uint64_t)e * g.n_tiles + tile, word, dst);
      } else if (i == nwt - 1 && (end & 31) != 0 && !last) {
        slot_merge(ws.slot + (uint64_t)e * g.n_tiles + tile + 1, word, dst);
      } else {
        *dst = bswap32(word);
      }
    }
    if (last) {
      // zero padding after the bitstream, up to its 16-byte boundary
      const uint64_t padded_words = round16(ceil_div(end, 8)) / 4;
      for (uint64_t i = W0 + nwt + tid; i < padded_words; i += kEncodeThreads) bs[i] = 0;
      if (huff) {
        uint32_t* idx = reinterpret_cast<uint32_t*>(payload + rec);
        for (uint64_t i = nsub + tid; i < idx_bytes / 4; i += kEncodeThreads) idx[i] = 0;
      }
    }
    if (huff && rec && ti == 0) {
      const int A = alphabet(DT, s);
      if (tid < (int)rec) {
        uint32_t b = 0;
        if (2 * tid < A) b = (enc[2 * tid] >> 16) | ((enc[2 * tid + 1] >> 16) << 4);
        payload[tid] = (uint8_t)b;
      }
    }
    __syncthreads();
  }
}

template <int DT>
static cudaError_t encode_t(const void* src, const Geo& g, const Ws& ws, uint8_t* out, cudaStream_t st) {
  const size_t smem = sizeof(EncodeSmem<DT>);
  static std::atomic<int> done[128];
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  if (dev < 0 || dev >= 128 || !done[dev].load(std::memory_order_relaxed)) {
    e = cudaFuncSetAttribute(k_encode<DT>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e == cudaSuccess) e = cudaFuncSetAttribute(k_encode<DT>, cudaFuncAttributePreferredSharedMemoryCarveout, 100);
    if (e != cudaSuccess) return e;
    if (dev >= 0 && dev < 128) done[dev].store(1, std::memory_order_relaxed);
  }
  k_encode<DT><<<g.n_tiles, kEncodeThreads, smem, st>>>(static_cast<const uint8_t*>(src), g, ws, out);
  return cudaGetLastError();
}

// FP32 (BF16 has k_encode_bf16, FP8 and FP4 k_encode_sub).
cudaError_t launch_encode(const void* src, const Geo& g, const Ws& ws, uint8_t* out, cudaStream_t st) {
  if (g.dt != kFP32) return cudaErrorInvalidValue;
  return encode_t<kFP32>(src, g, ws, out, st);
}

}  // namespace zipnn

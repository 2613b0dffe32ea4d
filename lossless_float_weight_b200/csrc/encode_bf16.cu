// encode_bf16.cu -- k_encode_bf16: the encode of BF16 tensors.
//
// The container bytes the oracle writes for a BF16 tensor, with no wait between blocks. A tile is
// 32768 consecutive values of one chunk (one histogram tile); its exponent
// bits start, inside the chunk's bitstream, at the sum over the chunk's lower tiles of
// count(tile, e) * len(e). The histogram pass counts per tile and the code build turns
// the counts into tile offsets, so every tile knows its offset before it packs a bit.
// Blocks are persistent: each takes tiles blockIdx.x, blockIdx.x + gridDim.x, ... and
// encodes a tile in passes of kBPassValues values (kBThreads threads of 64 values);
// each pass starts where the previous one's bits end. Small blocks (four warps, eight
// per SM) keep the barriers of a pass short and let the blocks' load and compute phases
// interleave. In each pass it
//  * loads its 64 values per thread (256-bit loads; 128-bit ones where they start only
//    16-byte aligned) and writes the sign/fraction plane (and an exponent plane that
//    did not compress) with 32-byte stores (two 16-byte ones where only 16-byte aligned);
//  * packs its exponent codes, two per step, most significant bit first, into private
//    shared words from bit 0; a block scan gives each thread its bit offset in the tile;
//  * moves the private words into a staging copy of the tile's bitstream at its final
//    alignment (shared atomicOr on each thread's two edge words), then stores it with
//    coalesced 32-bit stores, clearing the staging words as it reads them. The word
//    shared by two passes is carried in shared memory into the next pass's first word. A word that straddles two tiles is merged in a workspace slot: each side adds
//    (1 << 32 | its bits) and the side that arrives second stores the complete word.
// The sub-block index idx[j] (bit offset of symbol j*S) is written by the thread that
// owns symbol j*S; the first tile writes a local code record, the last the padding.
// A PACK exponent stream (packed exponent pairs) is written by k_encode_pack, which also
// writes a RAW sign/fraction plane: such chunks are skipped here unless the plane is ZRUN.
#include <atomic>

#include "common.cuh"
#include "fields.cuh"
#include "launch.h"

namespace zipnn {

constexpr int kBThreads = 128;
constexpr int kBValues = kGroupValues * kEncGroups;             // 64 values per thread
constexpr int kBPassValues = kBThreads * kBValues;              // 8192
constexpr int kBPasses = kBf16TileValues / kBPassValues;        // 4
constexpr int kBStageWords = kBPassValues * kLmax / 32 + 2;     // one pass's bitstream
constexpr int kBPrivStride = kBValues * kLmax / 32 + 1;         // odd: conflict-free
static_assert(kBPasses * kBPassValues == kBf16TileValues, "a tile is a whole number of passes");
static_assert(kBThreads == 128, "the pass scan adds four warp totals");

struct Bf16EncodeSmem {
  uint32_t priv[kBThreads * kBPrivStride];  // each thread's codes, packed from bit 0
  uint32_t stage[kBStageWords];                  // the tile's bitstream at its final alignment
  uint32_t enc[256];                             // the chunk's code: len << 16 | code
  alignas(16) uint32_t warp[2][kBThreads / 32];  // warp bit totals, by pass parity
  uint32_t zmap[32];  // ZRUN sign/fraction plane: the tile's 32 block-bitmap words
  uint32_t zpre[32];  // marked blocks of the chunk before each of those words
  uint32_t carry[2];  // the bits of the word shared with the next pass, by pass parity
};

__device__ __forceinline__ void bf16_slot_merge(uint64_t* slot, uint32_t part, uint32_t* dst) {
  const uint64_t old = atomicAdd(reinterpret_cast<unsigned long long*>(slot), (1ull << 32) | (uint64_t)part);
  if ((old >> 32) == 1) *dst = bswap32((uint32_t)old | part);
}

// Exponent (s == 0) or sign/fraction byte (s == 1) of two BF16 values, in bytes 0 and 2.
__device__ __forceinline__ uint32_t bf16_pair_plane(uint32_t w, int s) {
  return s == 0 ? (w >> 7) & 0x00FF00FFu : (w & 0x007F007Fu) | ((w >> 8) & 0x00800080u);
}

// The plane bytes of the four BF16 values in words a and b, in value order. Sign/fraction
// (s == 1): the values' low bytes (fraction bits 6..0 under exponent bit 0) and high bytes
// (the sign over exponent bits 7..1), gathered by two byte permutes, then the sign bits
// taken from the high bytes and the rest from the low bytes (one bit select).
__device__ __forceinline__ uint32_t bf16_quad_plane(uint32_t a, uint32_t b, int s) {
  if (s == 0) return __byte_perm(bf16_pair_plane(a, 0), bf16_pair_plane(b, 0), 0x6420);
  const uint32_t lo = __byte_perm(a, b, 0x6420), hi = __byte_perm(a, b, 0x7531);
  return (lo & 0x7F7F7F7Fu) | (hi & 0x80808080u);
}

__global__ void __launch_bounds__(kBThreads, 8) k_encode_bf16(const uint8_t* __restrict__ src, Geo g, Ws ws,
                                                                   uint8_t* __restrict__ out) {
  extern __shared__ __align__(16) uint8_t smem_raw[];
  Bf16EncodeSmem& sm = *reinterpret_cast<Bf16EncodeSmem*>(smem_raw);
  const int tid = threadIdx.x;
  const uint32_t T = g.tiles_per_chunk;
  for (int i = tid; i < kBStageWords; i += kBThreads) sm.stage[i] = 0;

  for (uint32_t tile = blockIdx.x; tile < g.n_tiles; tile += gridDim.x) {
    const uint32_t c = tile / T, ti = tile - c * T;
    const uint64_t clo = (uint64_t)c * g.m0;
    const uint32_t m = (uint32_t)min64(g.m0, g.n - clo);
    const uint32_t tlo = ti * (uint32_t)kBf16TileValues;
    if (tlo >= m) continue;  // past the end of a ragged last chunk (uniform)
    // the chunk's decisions and code
    const uint32_t mode0 = ws.emode[2ull * c], mode1 = ws.emode[2ull * c + 1];
    if (mode0 == kModePack && mode1 != kModeZrun) continue;  // k_encode_pack writes both streams (uniform)
    const uint32_t code0 = ws.ecode[2ull * c];
    const uint64_t off0 = ws.eoff[2ull * c], off1 = ws.eoff[2ull * c + 1];
    uint64_t P = 0;  // the pass's bit offset in the chunk
    if (mode0 == kModeHuff) {
      for (int i = tid; i < 256; i += kBThreads) sm.enc[i] = ws.enc[(uint64_t)c * 256 + i];
      P = ws.tile_off[tile];
    }
    if (mode1 == kModeZrun && tid < 32) {
      // zero runs: the tile's 1024 blocks are bitmap words 32 ti .. 32 ti + 31; each word's
      // rank base is the chunk's marked blocks before it. The tile also writes its words of
      // the payload's bitmap (MSB first: bits reversed within each byte), and the last tile
      // the bitmap's zero padding.
      const uint32_t* map = ws.zmap + (uint64_t)c * g.zwords;
      const uint32_t w0 = ti * 32u, used = (uint32_t)ceil_div(ceil_div(m, kZBlock), 32);
      uint32_t base = 0;
      for (uint32_t w = tid; w < w0; w += 32) base += __popc(__ldcg(map + w));
      base = __reduce_add_sync(0xFFFFFFFFu, base);
      const uint32_t word = w0 + tid < used ? __ldcg(map + w0 + tid) : 0u;
      const uint32_t pc = __popc(word);
      uint32_t incl = pc;
#pragma unroll
      for (int o = 1; o < 32; o <<= 1) {
        const uint32_t y = __shfl_up_sync(0xFFFFFFFFu, incl, o);
        if (tid >= o) incl += y;
      }
      sm.zmap[tid] = word;
      sm.zpre[tid] = base + incl - pc;
      uint32_t* mp = reinterpret_cast<uint32_t*>(out + off1);
      if (w0 + tid < used) mp[w0 + tid] = __byte_perm(__brev(word), 0, 0x0123);
      if (tlo + (uint32_t)kBf16TileValues >= m)
        for (uint32_t w = used + tid; w < zrun_map_bytes(m) / 4; w += 32) mp[w] = 0;
    }
    __syncthreads();  // the code is visible; the previous tile's stores and clears are done
    const uint64_t nsub = ceil_div(m, g.S);
    const uint32_t rec = code0 == kNoCode ? record_bytes(kBF16, 0) : 0;
    const uint64_t idx_bytes = round16(4 * nsub);
    uint8_t* payload = out + off0;
    uint32_t* idx = reinterpret_cast<uint32_t*>(payload + rec);
    uint32_t* bs = reinterpret_cast<uint32_t*>(payload + rec + idx_bytes);

    for (int pass = 0; pass < kBPasses; pass++) {
      const uint32_t plo = tlo + pass * (uint32_t)kBPassValues;
      if (plo >= m) break;  // uniform
      const bool last = plo + (uint32_t)kBPassValues >= m;              // the chunk's last pass
      const bool tile_end = last || pass == kBPasses - 1;               // the tile's last pass
      const uint32_t v0 = plo + tid * kBValues;
      const int cnt = v0 < m ? (int)min32(kBValues, m - v0) : 0;
      RawValues<kBF16, kBValues> raw;
      const uint8_t* vp = src + (clo + v0) * 2;
      if (cnt == kBValues && (reinterpret_cast<uintptr_t>(vp) & 31) == 0) {
#pragma unroll
        for (int j = 0; j < kBValues / 16; j++) ld_nc_v8(vp + 32 * j, raw.w + 8 * j);
      } else if (cnt > 0) {
        load_values<kBF16, kBValues>(vp, cnt, raw);
      }

#pragma unroll
      for (int s = 0; s < 2; s++) {
        const uint32_t mode = s == 0 ? mode0 : mode1;
        if ((mode != kModeRaw && !(s == 1 && mode == kModeZrun)) || cnt == 0) continue;
        // a byte plane: RAW (the sign/fraction bytes; an exponent stream that did not
        // compress) at the values' own offset; ZRUN (sign/fraction bytes with zero runs):
        // my values are blocks v0 / 32 and v0 / 32 + 1, and a marked block's 32 bytes go to
        // 32 x (its rank among the chunk's marked blocks) after the bitmap; an unmarked
        // block is not stored
        uint8_t* half[2];
        if (mode == kModeRaw) {
          half[0] = out + (s == 0 ? off0 : off1) + v0;
          half[1] = half[0] + 32;
        } else {
          uint8_t* data = out + off1 + zrun_map_bytes(m);
#pragma unroll
          for (int h = 0; h < 2; h++) {
            const uint32_t lb = (v0 - tlo) / kZBlock + (uint32_t)h;  // block within the tile
            const uint32_t word = sm.zmap[lb >> 5], bit = lb & 31u;
            half[h] = ((word >> bit) & 1u)
                          ? data + (uint64_t)(sm.zpre[lb >> 5] + __popc(word & ((1u << bit) - 1u))) * kZBlock
                          : nullptr;
          }
        }
        if (cnt == kBValues) {
#pragma unroll
          for (int h = 0; h < 2; h++) {
            uint32_t x[8];
#pragma unroll
            for (int k = 0; k < 8; k++) x[k] = bf16_quad_plane(raw.w[16 * h + 2 * k], raw.w[16 * h + 2 * k + 1], s);
            if (!half[h]) continue;
            if ((reinterpret_cast<uintptr_t>(half[h]) & 31) == 0) {
              st_v8(half[h], x);
            } else {
              *reinterpret_cast<uint4*>(half[h]) = make_uint4(x[0], x[1], x[2], x[3]);
              *reinterpret_cast<uint4*>(half[h] + 16) = make_uint4(x[4], x[5], x[6], x[7]);
            }
          }
        } else {
          // the chunk's last values: 16-byte groups, zero past cnt (a ZRUN block's data
          // then ends with the zero padding to its 16-byte boundary)
#pragma unroll
          for (int q = 0; q < kBValues / 16; q++) {
            if (16 * q < cnt && half[q >> 1]) {
              uint32_t x[4];
#pragma unroll
              for (int j = 0; j < 4; j++) {
                x[j] = 0;
#pragma unroll
                for (int b = 0; b < 4; b++) {
                  const int i = 16 * q + 4 * j + b;
                  if (i < cnt) x[j] |= symbol<kBF16, kBValues>(raw, s, i) << (8 * b);
                }
              }
              *reinterpret_cast<uint4*>(half[q >> 1] + 16 * (q & 1)) = make_uint4(x[0], x[1], x[2], x[3]);
            }
          }
        }
      }
      if (mode0 != kModeHuff) continue;  // uniform

      // the local code record heads the payload (4-bit lengths)
      if (rec && ti == 0 && pass == 0)
        for (int i = tid; i < 128; i += kBThreads)
          payload[i] = (uint8_t)((sm.enc[2 * i] >> 16) | ((sm.enc[2 * i + 1] >> 16) << 4));
      // pack my codes from bit 0 of my private words
      uint32_t* pw = sm.priv + tid * kBPrivStride;
      uint32_t nw = 0, nfill = 0, mybits = 0;
      uint32_t qoff[kBValues / 16];
      uint64_t acc = 0;
      if (cnt == kBValues) {
        // two values (one input word) per step: the exponent of the low value is bits
        // 14..7, so its table entry is at byte offset (w >> 5) & 0x3FC, the high one's at
        // (w >> 21) & 0x3FC. The two codes (at most 24 bits) join before they enter the
        // accumulator, which then holds fewer than 56 pending bits: one flush test a pair.
        const uint8_t* encb = reinterpret_cast<const uint8_t*>(sm.enc);
#pragma unroll
        for (int j = 0; j < kBValues / 2; j++) {
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
        for (int i = 0; i < kBValues; i++) {
          if ((i & 15) == 0) qoff[i >> 4] = mybits;
          if (i < cnt) {
            const uint32_t e = sm.enc[symbol<kBF16, kBValues>(raw, 0, i)];
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
      // my bit offset in the pass: a warp scan, then the four warp totals, which every
      // thread adds itself after one barrier. The totals alternate between two slots by
      // pass parity: a slot is written again two passes later, after the barrier of the
      // pass between, when every thread has read it.
      uint32_t pass_bits, myoff;
      {
        const int lane = tid & 31, warp = tid >> 5;
        uint32_t x = mybits;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
          const uint32_t y = __shfl_up_sync(0xFFFFFFFFu, x, o);
          if (lane >= o) x += y;
        }
        if (lane == 31) sm.warp[pass & 1][warp] = x;
        __syncthreads();
        const uint4 t = *reinterpret_cast<const uint4*>(sm.warp[pass & 1]);
        pass_bits = t.x + t.y + t.z + t.w;
        myoff = x - mybits + (warp > 0 ? t.x : 0u) + (warp > 1 ? t.y : 0u) + (warp > 2 ? t.z : 0u);
      }
      if (cnt > 0) {
        uint32_t rr = v0 % g.S;
#pragma unroll
        for (int q = 0; q < kBValues / 16; q++) {
          if (rr == 0 && 16 * q < cnt) idx[(v0 + 16 * q) / g.S] = (uint32_t)(P + myoff + qoff[q]);
          rr += 16;
          if (rr >= g.S) rr -= g.S;
        }
      }
      if (mybits) {
        const uint32_t q0 = (uint32_t)(P & 31) + myoff;
        const uint32_t sh = q0 & 31, d0 = q0 >> 5, nk = ((q0 + mybits - 1) >> 5) - d0 + 1;
        uint32_t cur = pw[0];
        atomicOr(sm.stage + d0, __funnelshift_r(cur, 0u, sh));
        for (uint32_t k = 1; k + 1 < nk; k++) {
          const uint32_t prev = cur;
          cur = pw[k];
          sm.stage[d0 + k] = __funnelshift_r(cur, prev, sh);
        }
        if (nk > 1) atomicOr(sm.stage + d0 + nk - 1, __funnelshift_r(nk - 1 < nw ? pw[nk - 1] : 0u, cur, sh));
      }
      __syncthreads();
      const uint64_t end = P + pass_bits;
      const uint32_t nwt = (uint32_t)(((P & 31) + pass_bits + 31) >> 5);
      const uint64_t W0 = P >> 5;
      for (uint32_t i = 1 + tid; i + 1 < nwt; i += kBThreads) {  // middle words: plain
        const uint32_t word = sm.stage[i];
        sm.stage[i] = 0;
        bs[W0 + i] = bswap32(word);
      }
      if (tid < 2 && nwt > 0 && (tid == 0 || nwt > 1)) {  // edge words: thread 0 the first, 1 the last
        const uint32_t i = tid == 0 ? 0u : nwt - 1;
        uint32_t word = sm.stage[i];
        sm.stage[i] = 0;
        // the previous pass's last bits; a pass reads one carry slot and writes the other,
        // so the slot it reads is not written again before the barriers of the next pass
        if (i == 0 && pass > 0 && (P & 31) != 0) word |= sm.carry[(pass - 1) & 1];
        uint32_t* dst = bs + W0 + i;
        // (a first pass that is not the tile's last has kBPassValues values, so i == 0 and
        // the carried word are never the same word)
        if (i == nwt - 1 && (end & 31) != 0 && !tile_end) sm.carry[pass & 1] = word;  // completed by the next pass
        else if (i == 0 && pass == 0 && (P & 31) != 0) bf16_slot_merge(ws.slot + tile, word, dst);
        else if (i == nwt - 1 && (end & 31) != 0 && !last) bf16_slot_merge(ws.slot + tile + 1, word, dst);
        else *dst = bswap32(word);
      }
      P = end;
      if (last) {
        const uint64_t padded_words = round16(ceil_div(end, 8)) / 4;
        for (uint64_t i = W0 + nwt + tid; i < padded_words; i += kBThreads) bs[i] = 0;
        for (uint64_t i = nsub + tid; i < idx_bytes / 4; i += kBThreads) idx[i] = 0;
      }
    }
    __syncthreads();  // the tile's bitmap words are read before the next tile's setup
  }
}

// Launch: a persistent grid of as many blocks as fit on the device at once.
cudaError_t launch_encode_bf16(const void* src, const Geo& g, const Ws& ws, uint8_t* out, cudaStream_t st) {
  const size_t smem = sizeof(Bf16EncodeSmem);
  static std::atomic<int> resident[128];  // blocks per device, once the attributes are set
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  int per_device = dev >= 0 && dev < 128 ? resident[dev].load(std::memory_order_relaxed) : 0;
  if (!per_device) {
    e = cudaFuncSetAttribute(k_encode_bf16, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e == cudaSuccess) e = cudaFuncSetAttribute(k_encode_bf16, cudaFuncAttributePreferredSharedMemoryCarveout, 100);
    int per_sm = 0, sms = 0;
    if (e == cudaSuccess) e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, k_encode_bf16, kBThreads, smem);
    if (e == cudaSuccess) e = cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    if (e != cudaSuccess) return e;
    per_device = (per_sm > 0 ? per_sm : 1) * (sms > 0 ? sms : 1);
    if (dev >= 0 && dev < 128) resident[dev].store(per_device, std::memory_order_relaxed);
  }
  const uint32_t blocks = (uint32_t)min64((uint64_t)per_device, g.n_tiles);
  k_encode_bf16<<<blocks, kBThreads, smem, st>>>(static_cast<const uint8_t*>(src), g, ws, out);
  return cudaGetLastError();
}

}  // namespace zipnn

// encode_fp32.cu -- k_encode_fp32: the encode of FP32 tensors.
//
// The scheme of k_encode_bf16 for FP32's four streams (the exponent, then the byte
// planes p1 = sign over fraction bits 22..16, p2 = bits 15..8, p3 = bits 7..0): a tile is
// the 32768 values of one histogram slice, whose exponent counts gave its bit offset in
// the chunk's exponent bitstream, so no block waits on another. Blocks are persistent
// (four warps, eight per SM); each takes tiles blockIdx.x, blockIdx.x + gridDim.x, ... in
// passes of kFPass values (32 a thread: one zero-run block). In each pass a thread
//  * loads its 32 values (256-bit loads where its address is 32-byte aligned);
//  * writes its 32 bytes of each byte plane: RAW at the values' own offset; ZRUN at
//    32 x (the block's rank among the chunk's marked blocks) after the bitmap when its
//    block holds a non-zero byte, else nothing;
//  * packs its exponent codes, two values a step, into private shared words; a block scan
//    gives its bit offset; the words move into a staging copy of the pass's bitstream and
//    go out as coalesced 32-bit stores, with the word shared by two passes carried in
//    shared memory and a word shared by two tiles merged in a workspace slot.
#include <atomic>

#include "common.cuh"
#include "fields.cuh"
#include "launch.h"

namespace zipnn {

constexpr int kFThreads = 128;
constexpr int kFValues = 32;                                   // values a thread per pass
constexpr int kFPass = kFThreads * kFValues;                   // 4096
constexpr int kFPasses = kBf16TileValues / kFPass;             // 8
constexpr int kFStageWords = kFPass * kLmax / 32 + 2;          // one pass's bitstream
constexpr int kFPrivStride = kFValues * kLmax / 32 + 1;        // odd: conflict-free
static_assert(kFPasses * kFPass == kBf16TileValues, "a tile is a whole number of passes");
static_assert(kFValues == (int)kZBlock, "a thread's values are one zero-run block");
static_assert(kFThreads == 128, "the pass scan adds four warp totals");

struct Fp32EncodeSmem {
  uint32_t priv[kFThreads * kFPrivStride];
  uint32_t stage[kFStageWords];
  uint32_t enc[256];                             // the chunk's exponent code: len << 16 | code
  alignas(16) uint32_t warp[2][kFThreads / 32];  // warp bit totals, by pass parity
  uint32_t zmap[3][32];  // ZRUN planes: the tile's 32 block-bitmap words of each
  uint32_t zpre[3][32];  // marked blocks of the chunk before each of those words
  uint32_t carry[2];     // the bits of the word shared with the next pass, by pass parity
};

__device__ __forceinline__ void f32_slot_merge(uint64_t* slot, uint32_t part, uint32_t* dst) {
  const uint64_t old = atomicAdd(reinterpret_cast<unsigned long long*>(slot), (1ull << 32) | (uint64_t)part);
  if ((old >> 32) == 1) *dst = bswap32((uint32_t)old | part);
}

// Byte plane s (0: the exponent, 1..3: p1..p3) of the four FP32 values w[0..3], in value order.
__device__ __forceinline__ uint32_t f32_quad_plane(const uint32_t* w, int s) {
  if (s == 1) {
    // sign (byte 3, bit 7) over fraction bits 22..16 (byte 2, bits 6..0): one bit select
    const uint32_t lo = __byte_perm(__byte_perm(w[0], w[1], 0x0062), __byte_perm(w[2], w[3], 0x0062), 0x5410);
    const uint32_t hi = __byte_perm(__byte_perm(w[0], w[1], 0x0073), __byte_perm(w[2], w[3], 0x0073), 0x5410);
    return (lo & 0x7F7F7F7Fu) | (hi & 0x80808080u);
  }
  if (s == 0) {
    uint32_t e[4];
#pragma unroll
    for (int i = 0; i < 4; i++) e[i] = w[i] >> 23;  // exponent in bits 7..0 (over the sign)
    return __byte_perm(__byte_perm(e[0], e[1], 0x0040), __byte_perm(e[2], e[3], 0x0040), 0x5410);
  }
  const uint32_t sel = s == 2 ? 0x0051u : 0x0040u;  // byte 1 (p2) or byte 0 (p3) of each value
  return __byte_perm(__byte_perm(w[0], w[1], sel), __byte_perm(w[2], w[3], sel), 0x5410);
}

__global__ void __launch_bounds__(kFThreads, 8) k_encode_fp32(const uint8_t* __restrict__ src, Geo g, Ws ws,
                                                              uint8_t* __restrict__ out) {
  extern __shared__ __align__(16) uint8_t smem_raw[];
  Fp32EncodeSmem& sm = *reinterpret_cast<Fp32EncodeSmem*>(smem_raw);
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const uint32_t T = g.tiles_per_chunk;
  for (int i = tid; i < kFStageWords; i += kFThreads) sm.stage[i] = 0;

  for (uint32_t tile = blockIdx.x; tile < g.n_tiles; tile += gridDim.x) {
    const uint32_t c = tile / T, ti = tile - c * T;
    const uint64_t clo = (uint64_t)c * g.m0;
    const uint32_t m = (uint32_t)min64(g.m0, g.n - clo);
    const uint32_t tlo = ti * (uint32_t)kBf16TileValues;
    if (tlo >= m) continue;  // past the end of a ragged last chunk (uniform)
    uint32_t mode[4];
    uint64_t off[4];
#pragma unroll
    for (int s = 0; s < 4; s++) {
      mode[s] = ws.emode[4ull * c + s];
      off[s] = ws.eoff[4ull * c + s];
    }
    const uint32_t code0 = ws.ecode[4ull * c];
    uint64_t P = 0;  // the pass's bit offset in the chunk
    if (mode[0] == kModeHuff) {
      for (int i = tid; i < 256; i += kFThreads) sm.enc[i] = ws.enc[(uint64_t)c * 256 + i];
      P = ws.tile_off[tile];
    }
    if (warp < 3 && ws.emode[4ull * c + warp + 1] == kModeZrun) {
      // zero runs of plane warp + 1 (warp w takes plane w + 1): the tile's 1024 blocks are
      // bitmap words 32 ti .. 32 ti + 31, each with its rank base (the chunk's marked
      // blocks before it); the tile writes its words of the payload's bitmap (MSB first:
      // bits reversed within each byte), the last tile the bitmap's zero padding
      const int p = warp;
      const uint32_t* map = ws.zmap + ((uint64_t)c * 3 + p) * g.zwords;
      const uint32_t w0 = ti * 32u, used = (uint32_t)ceil_div(ceil_div(m, kZBlock), 32);
      uint32_t base = 0;
      for (uint32_t w = lane; w < w0; w += 32) base += __popc(__ldcg(map + w));
      base = __reduce_add_sync(0xFFFFFFFFu, base);
      const uint32_t word = w0 + lane < used ? __ldcg(map + w0 + lane) : 0u;
      const uint32_t pc = __popc(word);
      uint32_t incl = pc;
#pragma unroll
      for (int o = 1; o < 32; o <<= 1) {
        const uint32_t y = __shfl_up_sync(0xFFFFFFFFu, incl, o);
        if (lane >= o) incl += y;
      }
      sm.zmap[p][lane] = word;
      sm.zpre[p][lane] = base + incl - pc;
      uint32_t* mp = reinterpret_cast<uint32_t*>(out + ws.eoff[4ull * c + p + 1]);
      if (w0 + lane < used) mp[w0 + lane] = __byte_perm(__brev(word), 0, 0x0123);
      if (tlo + (uint32_t)kBf16TileValues >= m)
        for (uint32_t w = used + lane; w < zrun_map_bytes(m) / 4; w += 32) mp[w] = 0;
    }
    __syncthreads();  // code and bitmaps visible; the previous tile's stores and clears are done
    const uint64_t nsub = ceil_div(m, g.S);
    const uint32_t rec = code0 == kNoCode ? record_bytes(kFP32, 0) : 0;
    const uint64_t idx_bytes = round16(4 * nsub);
    uint8_t* payload = out + off[0];
    uint32_t* idx = reinterpret_cast<uint32_t*>(payload + rec);
    uint32_t* bs = reinterpret_cast<uint32_t*>(payload + rec + idx_bytes);

    for (int pass = 0; pass < kFPasses; pass++) {
      const uint32_t plo = tlo + pass * (uint32_t)kFPass;
      if (plo >= m) break;  // uniform
      const bool last = plo + (uint32_t)kFPass >= m;     // the chunk's last pass
      const bool tile_end = last || pass == kFPasses - 1;
      const uint32_t v0 = plo + tid * kFValues;
      const int cnt = v0 < m ? (int)min32(kFValues, m - v0) : 0;
      RawValues<kFP32, kFValues> raw;
      const uint8_t* vp = src + (clo + v0) * 4;
      if (cnt == kFValues && (reinterpret_cast<uintptr_t>(vp) & 31) == 0) {
#pragma unroll
        for (int j = 0; j < kFValues / 8; j++) ld_nc_v8(vp + 32 * j, raw.w + 8 * j);
      } else if (cnt > 0) {
        load_values<kFP32, kFValues>(vp, cnt, raw);  // zero past cnt
      } else {
#pragma unroll
        for (int j = 0; j < kFValues; j++) raw.w[j] = 0;
      }

      // byte planes (and an exponent stream that did not compress): my 32 bytes, 16-byte
      // groups up to cnt (values past cnt are zero, so a short last block ends in its padding)
#pragma unroll
      for (int s = 0; s < 4; s++) {
        const uint32_t md = mode[s];
        if (!(md == kModeRaw || (s > 0 && md == kModeZrun)) || cnt == 0) continue;
        uint8_t* dst;
        if (md == kModeRaw) {
          dst = out + off[s] + v0;
        } else {
          const uint32_t lb = (v0 - tlo) / kZBlock;  // my block within the tile
          const uint32_t word = sm.zmap[s - 1][lb >> 5], bit = lb & 31u;
          dst = ((word >> bit) & 1u) ? out + off[s] + zrun_map_bytes(m) +
                                           (uint64_t)(sm.zpre[s - 1][lb >> 5] + __popc(word & ((1u << bit) - 1u))) * kZBlock
                                     : nullptr;
        }
        if (!dst) continue;
        uint32_t x[8];
#pragma unroll
        for (int k = 0; k < 8; k++) x[k] = f32_quad_plane(raw.w + 4 * k, s);
        if (cnt == kFValues && (reinterpret_cast<uintptr_t>(dst) & 31) == 0) {
          st_v8(dst, x);
        } else {
          *reinterpret_cast<uint4*>(dst) = make_uint4(x[0], x[1], x[2], x[3]);
          if (cnt > 16) *reinterpret_cast<uint4*>(dst + 16) = make_uint4(x[4], x[5], x[6], x[7]);
        }
      }
      if (mode[0] != kModeHuff) continue;  // uniform

      // the local code record heads the payload (4-bit lengths)
      if (rec && ti == 0 && pass == 0)
        for (int i = tid; i < 128; i += kFThreads)
          payload[i] = (uint8_t)((sm.enc[2 * i] >> 16) | ((sm.enc[2 * i + 1] >> 16) << 4));
      // pack my codes from bit 0 of my private words: two values a step (the exponent is
      // bits 30..23, its table entry at byte offset (w >> 21) & 0x3FC); the two codes (at
      // most 24 bits) join before they enter the accumulator
      uint32_t* pw = sm.priv + tid * kFPrivStride;
      uint32_t nw = 0, nfill = 0;
      uint32_t qoff[kFValues / 16];
      uint64_t acc = 0;
      const uint8_t* encb = reinterpret_cast<const uint8_t*>(sm.enc);
      auto pack_codes = [&](bool all) {  // all: a whole pass, no test per value
#pragma unroll
        for (int j = 0; j < kFValues / 2; j++) {
          if ((j & 7) == 0) qoff[j >> 3] = nw * 32 + nfill;
          if (all || 2 * j < cnt) {
            const uint32_t e0 = *reinterpret_cast<const uint32_t*>(encb + ((raw.w[2 * j] >> 21) & 0x3FCu));
            const uint32_t e1 = all || 2 * j + 1 < cnt
                                    ? *reinterpret_cast<const uint32_t*>(encb + ((raw.w[2 * j + 1] >> 21) & 0x3FCu))
                                    : 0u;
            const uint32_t l1 = e1 >> 16;
            const uint32_t l = (e0 >> 16) + l1;
            acc = (acc << l) | (((e0 & 0xFFFFu) << l1) | (e1 & 0xFFFFu));
            nfill += l;
            if (nfill >= 32) {
              nfill -= 32;
              pw[nw++] = (uint32_t)(acc >> nfill);
            }
          }
        }
      };
      if (cnt == kFValues) pack_codes(true);
      else pack_codes(false);
      const uint32_t mybits = nw * 32 + nfill;
      if (nfill) pw[nw++] = (uint32_t)(acc << (32 - nfill));
      // my bit offset in the pass: a warp scan, then the four warp totals after one barrier
      // (two slots by pass parity: a slot is written again two passes later, after the
      // barriers of the pass between)
      uint32_t pass_bits, myoff;
      {
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
        for (int q = 0; q < kFValues / 16; q++) {
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
      for (uint32_t i = 1 + tid; i + 1 < nwt; i += kFThreads) {  // middle words: plain
        const uint32_t word = sm.stage[i];
        sm.stage[i] = 0;
        bs[W0 + i] = bswap32(word);
      }
      if (tid < 2 && nwt > 0 && (tid == 0 || nwt > 1)) {  // edge words: thread 0 the first, 1 the last
        const uint32_t i = tid == 0 ? 0u : nwt - 1;
        uint32_t word = sm.stage[i];
        sm.stage[i] = 0;
        if (i == 0 && pass > 0 && (P & 31) != 0) word |= sm.carry[(pass - 1) & 1];
        uint32_t* dst = bs + W0 + i;
        // (a pass that is not the tile's last holds kFPass values, at least 4096 bits, so
        // its first word and its carried last word are never the same word)
        if (i == nwt - 1 && (end & 31) != 0 && !tile_end) sm.carry[pass & 1] = word;  // completed by the next pass
        else if (i == 0 && pass == 0 && (P & 31) != 0) f32_slot_merge(ws.slot + tile, word, dst);
        else if (i == nwt - 1 && (end & 31) != 0 && !last) f32_slot_merge(ws.slot + tile + 1, word, dst);
        else *dst = bswap32(word);
      }
      P = end;
      if (last) {
        const uint64_t padded_words = round16(ceil_div(end, 8)) / 4;
        for (uint64_t i = W0 + nwt + tid; i < padded_words; i += kFThreads) bs[i] = 0;
        for (uint64_t i = nsub + tid; i < idx_bytes / 4; i += kFThreads) idx[i] = 0;
      }
    }
    __syncthreads();  // the tile's bitmaps and code are read before the next tile's setup
  }
}

// Launch: a persistent grid of as many blocks as fit on the device at once.
cudaError_t launch_encode_fp32(const void* src, const Geo& g, const Ws& ws, uint8_t* out, cudaStream_t st) {
  const size_t smem = sizeof(Fp32EncodeSmem);
  static std::atomic<int> resident[128];  // blocks per device, once the attributes are set
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  int per_device = dev >= 0 && dev < 128 ? resident[dev].load(std::memory_order_relaxed) : 0;
  if (!per_device) {
    e = cudaFuncSetAttribute(k_encode_fp32, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e == cudaSuccess) e = cudaFuncSetAttribute(k_encode_fp32, cudaFuncAttributePreferredSharedMemoryCarveout, 100);
    int per_sm = 0, sms = 0;
    if (e == cudaSuccess) e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, k_encode_fp32, kFThreads, smem);
    if (e == cudaSuccess) e = cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    if (e != cudaSuccess) return e;
    per_device = (per_sm > 0 ? per_sm : 1) * (sms > 0 ? sms : 1);
    if (dev >= 0 && dev < 128) resident[dev].store(per_device, std::memory_order_relaxed);
  }
  const uint32_t blocks = (uint32_t)min64((uint64_t)per_device, g.n_tiles);
  k_encode_fp32<<<blocks, kFThreads, smem, st>>>(static_cast<const uint8_t*>(src), g, ws, out);
  return cudaGetLastError();
}

}  // namespace zipnn

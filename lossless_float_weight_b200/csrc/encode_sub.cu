// encode_sub.cu -- k_encode_sub<DT>: the encode of FP8 (E4M3) and FP4 (E2M1) tensors.
//
// The same output as the oracle's encode of these types ("Lossless Compression for LLM
// Tensors", abstract: the exponent and the mantissa of FP8 and FP4 values are coded
// independently; the sign is stored as it is), built like the BF16 encode: a tile is the
// 32768 values of one histogram slice, and the histogram pass counted each tile's joint
// (exponent, mantissa) bins, so the code build knows the bit offset of every tile in
// both entropy streams before any tile packs a bit. No block waits on another.
// Blocks are persistent (four warps, eight per SM); each takes tiles blockIdx.x,
// blockIdx.x + gridDim.x, ... in passes of kSPass values (64 a thread). In each pass a
// thread loads its 64 values at once and, for every stream of the chunk:
//  * RAW (exponent 4 / 2 bits, mantissa 3 / 1, sign 1): value v's bits sit at v * width,
//    so the thread's 64 values fill whole words that it assembles with bit-parallel
//    shifts and masks and stores itself;
//  * HUFF: the codes of a group of symbols (two FP8 exponents or mantissas, four FP4
//    exponents, eight FP4 mantissas: one byte of the input) come from one lookup in a
//    table of the chunk's concatenated codes; they are packed most significant bit first
//    into private shared words, a block scan gives each thread its bit offset, the words
//    move into a staging copy of the pass's bitstream at its final alignment and go out
//    as coalesced 32-bit stores. The word shared by two passes is carried in shared
//    memory; a word shared by two tiles is merged in a workspace slot (each side adds
//    1 << 32 | its bits, the second arrival stores the whole word).
// A code whose grouped codes would not fit the table's 24 bits (only an imported plan can
// have one) is packed a symbol at a time, as are the chunk's last values.
#include <atomic>
#include <type_traits>

#include "common.cuh"
#include "fields.cuh"
#include "launch.h"

namespace zipnn {

constexpr int kSThreads = 128;
constexpr int kSValues = 64;                                       // values a thread per pass
constexpr int kSPass = kSThreads * kSValues;                       // 8192
constexpr int kSPasses = kBf16TileValues / kSPass;                 // 4
constexpr int kSStageWords = kSPass * kLmax / 32 + 2;              // one pass's bitstream
constexpr int kSPrivStride = kSValues * kLmax / 32 + 1;            // odd: conflict-free
static_assert(kSPasses * kSPass == kBf16TileValues, "a tile is a whole number of passes");
static_assert(kSThreads == 128, "the pass scan adds four warp totals");

// Symbols of entropy stream e in one table group: the symbols of one input byte.
__host__ __device__ constexpr int group_symbols(int dt, int e) { return 8 / raw_width(dt, e); }

struct SubEncodeSmem {
  uint32_t priv[kSThreads * kSPrivStride];  // each thread's codes, packed from bit 0
  uint32_t stage[kSStageWords];             // the pass's bitstream at its final alignment
  uint32_t tab[2][256];                     // per entropy stream: len << 24 | grouped codes
  uint32_t enc[2][16];                      // per entropy stream: len << 16 | code
  alignas(16) uint32_t warp[2][kSThreads / 32];  // warp bit totals, by scan parity
  uint32_t carry[2][2];                     // per stream, by pass parity: the word shared with the next pass
  uint32_t fast[2];                         // per stream: the grouped table holds every group
};

__device__ __forceinline__ void sub_slot_merge(uint64_t* slot, uint32_t part, uint32_t* dst) {
  const uint64_t old = atomicAdd(reinterpret_cast<unsigned long long*>(slot), (1ull << 32) | (uint64_t)part);
  if ((old >> 32) == 1) *dst = bswap32((uint32_t)old | part);
}

// Table index of group q (in value order) of entropy stream e: the group's symbols with
// the first in the lowest bits.
template <int DT, int E>
__device__ __forceinline__ uint32_t group_index(const uint32_t* w, int q) {
  if constexpr (DT == kFP8) {
    // word q / 2 holds values 4(q / 2) ..; pair q % 2 is its bytes 2(q % 2), 2(q % 2) + 1
    const uint32_t x = w[q >> 1];
    const uint32_t t = E == 0 ? (x >> 3) & 0x0F0F0F0Fu : x & 0x07070707u;
    const uint32_t u = E == 0 ? t | (t >> 4) : t | (t >> 5);
    return (u >> (16 * (q & 1))) & (E == 0 ? 0xFFu : 0x3Fu);
  } else if constexpr (E == 0) {
    // FP4 exponents (nibble bits 1..2): word q / 2 holds values 8(q / 2) ..; quad q % 2
    const uint32_t x = w[q >> 1];
    const uint32_t t = (x >> 1) & 0x33333333u;
    const uint32_t u = (t | (t >> 2)) & 0x0F0F0F0Fu;
    return ((u | (u >> 4)) >> (16 * (q & 1))) & 0xFFu;
  } else {
    // FP4 mantissas (nibble bit 0): the eight of word q
    uint32_t t = w[q] & 0x11111111u;
    t = (t | (t >> 3)) & 0x03030303u;
    t = (t | (t >> 6)) & 0x000F000Fu;
    return (t | (t >> 12)) & 0xFFu;
  }
}

// The memory words of RAW stream s for my 64 values (value v0 first), most significant
// bit first: FP8 exponent 8 words, mantissa 6, sign 2; FP4 exponent 4, mantissa 2, sign 2.
template <int DT, int S>
__device__ __forceinline__ void raw_words(const uint32_t* w, uint32_t* mw) {
  if constexpr (DT == kFP8 && S == 0) {
    // bytes (e0 << 4 | e1) and (e2 << 4 | e3) of each input word, two words a memory word
#pragma unroll
    for (int j = 0; j < 8; j++) {
      const uint32_t ta = (w[2 * j] >> 3) & 0x0F0F0F0Fu, tb = (w[2 * j + 1] >> 3) & 0x0F0F0F0Fu;
      mw[j] = __byte_perm((ta << 4) | (ta >> 8), (tb << 4) | (tb >> 8), 0x6420);
    }
  } else if constexpr (DT == kFP8 && S == 1) {
    // 12 bits an input word (m0 m1 m2 m3), 16 groups in 6 words
    uint64_t acc = 0;
    int nf = 0, k = 0;
#pragma unroll
    for (int j = 0; j < 16; j++) {
      const uint32_t t = w[j] & 0x07070707u;
      const uint32_t y = ((t & 7u) << 9) | ((t >> 2) & 0x1C0u) | ((t >> 13) & 0x38u) | (t >> 24);
      acc = (acc << 12) | y;
      nf += 12;
      if (nf >= 32) {
        nf -= 32;
        mw[k++] = bswap32((uint32_t)(acc >> nf));
      }
    }
  } else if constexpr (DT == kFP8) {
    // the four sign bits of an input word gathered by one multiply (value 0 highest)
#pragma unroll
    for (int h = 0; h < 2; h++) {
      uint32_t b = 0;
#pragma unroll
      for (int j = 0; j < 8; j++) b = (b << 4) | ((((w[8 * h + j] >> 7) & 0x01010101u) * 0x08040201u) >> 24);
      mw[h] = bswap32(b);
    }
  } else if constexpr (S == 0) {
    // FP4 exponents: bytes (e0 e1 e2 e3) and (e4 e5 e6 e7) of each input word
#pragma unroll
    for (int j = 0; j < 4; j++) {
      uint32_t v[2];
#pragma unroll
      for (int i = 0; i < 2; i++) {
        const uint32_t t = (w[2 * j + i] >> 1) & 0x33333333u;
        const uint32_t u = ((t << 2) | (t >> 4)) & 0x0F0F0F0Fu;
        v[i] = (u << 4) | (u >> 8);
      }
      mw[j] = __byte_perm(v[0], v[1], 0x6420);
    }
  } else {
    // FP4 mantissa (nibble bit 0) or sign (bit 3): eight bits an input word, value i at
    // bit i, then the bits of each byte reversed (value 0 highest)
    constexpr int B = S == 1 ? 0 : 3;
#pragma unroll
    for (int h = 0; h < 2; h++) {
      uint32_t l = 0;
#pragma unroll
      for (int j = 0; j < 4; j++) {
        uint32_t t = (w[4 * h + j] >> B) & 0x11111111u;
        t = (t | (t >> 3)) & 0x03030303u;
        t = (t | (t >> 6)) & 0x000F000Fu;
        l |= ((t | (t >> 12)) & 0xFFu) << (8 * j);
      }
      mw[h] = bswap32(__brev(l));
    }
  }
}

template <int DT>
__global__ void __launch_bounds__(kSThreads, 8) k_encode_sub(const uint8_t* __restrict__ src, Geo g, Ws ws,
                                                              uint8_t* __restrict__ out) {
  constexpr int NS = n_streams(DT);
  constexpr int WORDS = kSValues * value_bits(DT) / 32;  // input words a thread per pass
  extern __shared__ __align__(16) uint8_t smem_raw[];
  SubEncodeSmem& sm = *reinterpret_cast<SubEncodeSmem*>(smem_raw);
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const uint32_t T = g.tiles_per_chunk;
  for (int i = tid; i < kSStageWords; i += kSThreads) sm.stage[i] = 0;
  uint32_t ph = 0;  // scans so far: the parity of the warp-total slot

  for (uint32_t tile = blockIdx.x; tile < g.n_tiles; tile += gridDim.x) {
    const uint32_t c = tile / T, ti = tile - c * T;
    const uint64_t clo = (uint64_t)c * g.m0;
    const uint32_t m = (uint32_t)min64(g.m0, g.n - clo);
    const uint32_t tlo = ti * (uint32_t)kBf16TileValues;
    if (tlo >= m) continue;  // past the end of a ragged last chunk (uniform)
    uint32_t mode[NS];
    uint64_t off[NS];
#pragma unroll
    for (int s = 0; s < NS; s++) {
      mode[s] = ws.emode[(uint64_t)c * NS + s];
      off[s] = ws.eoff[(uint64_t)c * NS + s];
    }
    uint64_t P[2] = {0, 0};  // per entropy stream: the pass's bit offset in the chunk
#pragma unroll
    for (int e = 0; e < 2; e++) {
      if (mode[e] != kModeHuff) continue;  // uniform
      P[e] = ws.tile_off[(uint64_t)e * g.n_tiles + tile];
      const int A = alphabet(DT, e), K = group_symbols(DT, e), w = raw_width(DT, e);
      const uint32_t* enc = ws.enc + ((uint64_t)c * 2 + e) * 256;
      if (tid < A) sm.enc[e][tid] = enc[tid];
      // grouped codes: entry x holds the codes of the K symbols of x (first in the
      // lowest bits), concatenated first-most-significant, if they fit 24 bits
      uint32_t lmax = 0;
      for (int a = 0; a < A; a++) lmax = max(lmax, enc[a] >> 16);
      if (tid == 0) sm.fast[e] = (uint32_t)K * lmax <= 24u;
      for (int x = tid; x < (1 << (K * w)); x += kSThreads) {
        uint32_t code = 0, len = 0;
        for (int k = 0; k < K; k++) {
          const uint32_t ek = enc[(x >> (k * w)) & (A - 1)], l = ek >> 16;  // l <= 12
          code = (code << l) | (ek & 0xFFFFu);
          len += l;
        }
        sm.tab[e][x] = len <= 24 ? (len << 24) | (code & 0xFFFFFFu) : 0u;
      }
    }
    __syncthreads();  // tables visible; the previous tile's stores and clears are done
    const uint64_t nsub = ceil_div(m, g.S);

    for (int pass = 0; pass < kSPasses; pass++) {
      const uint32_t plo = tlo + pass * (uint32_t)kSPass;
      if (plo >= m) break;  // uniform
      const bool last = plo + (uint32_t)kSPass >= m;     // the chunk's last pass
      const bool tile_end = last || pass == kSPasses - 1;
      const uint32_t v0 = plo + tid * kSValues;
      const int cnt = v0 < m ? (int)min32(kSValues, m - v0) : 0;
      RawValues<DT, kSValues> raw;
      const uint8_t* vp = src + value_offset(DT, clo + v0);
      if (cnt == kSValues && (reinterpret_cast<uintptr_t>(vp) & 31) == 0) {
#pragma unroll
        for (int j = 0; j < WORDS / 8; j++) ld_nc_v8(vp + 32 * j, raw.w + 8 * j);
      } else if (cnt > 0) {
        load_values<DT, kSValues>(vp, cnt, raw);
      } else {
#pragma unroll
        for (int j = 0; j < WORDS; j++) raw.w[j] = 0;
      }

      // RAW streams of w < 8 bits: my words at word v0 * w / 32 of the payload; a thread of
      // the chunk's last values writes only the words the chunk uses (the rest of the
      // payload up to its 16-byte padding is zeroed by the chunk's last pass)
      auto raw_stream = [&](auto sc) {
        constexpr int s = decltype(sc)::value, w = raw_width(DT, s), nwm = kSValues * w / 32;
        if (mode[s] != kModeRaw) return;  // uniform
        uint32_t* words = reinterpret_cast<uint32_t*>(out + off[s]);
        const uint32_t wbase = (uint32_t)((uint64_t)v0 * w / 32);
        const uint32_t used = (uint32_t)ceil_div((uint64_t)m * w, 32);
        if (cnt > 0) {
          uint32_t mw[nwm];
          raw_words<DT, s>(raw.w, mw);
#pragma unroll
          for (int k = 0; k < nwm; k++)  // a whole pass's words all lie inside the stream
            if (cnt == kSValues || wbase + k < used) words[wbase + k] = mw[k];
        }
        if (last) {
          const uint64_t padded = raw_payload(m, w) / 4;
          for (uint64_t i = used + tid; i < padded; i += kSThreads) words[i] = 0;
        }
      };
      raw_stream(std::integral_constant<int, 0>{});
      raw_stream(std::integral_constant<int, 1>{});
      raw_stream(std::integral_constant<int, 2>{});

      auto huff_stream = [&](auto ec) {
        constexpr int e = decltype(ec)::value, K = group_symbols(DT, e);
        if (mode[e] != kModeHuff) return;  // uniform
        const uint32_t rec = ws.ecode[(uint64_t)c * NS + e] == kNoCode ? record_bytes(DT, e) : 0;
        const uint64_t idx_bytes = round16(4 * nsub);
        uint8_t* payload = out + off[e];
        uint32_t* idx = reinterpret_cast<uint32_t*>(payload + rec);
        uint32_t* bs = reinterpret_cast<uint32_t*>(payload + rec + idx_bytes);
        if (rec && ti == 0 && pass == 0 && tid < (int)rec) {
          // the local code record heads the payload (4-bit lengths)
          const int A = alphabet(DT, e);
          uint32_t b = 0;
          if (2 * tid < A) b = (sm.enc[e][2 * tid] >> 16) | ((sm.enc[e][2 * tid + 1] >> 16) << 4);
          payload[tid] = (uint8_t)b;
        }
        // pack my codes from bit 0 of my private words
        uint32_t* pw = sm.priv + tid * kSPrivStride;
        uint32_t nw = 0, nfill = 0;
        uint32_t qoff[kSValues / 16];
        uint64_t acc = 0;
        if (cnt == kSValues && sm.fast[e]) {
          const uint32_t* tab = sm.tab[e];
#pragma unroll
          for (int q = 0; q < kSValues / K; q++) {
            if ((q * K) % 16 == 0) qoff[q * K / 16] = nw * 32 + nfill;
            const uint32_t t = tab[group_index<DT, e>(raw.w, q)];
            const uint32_t l = t >> 24;
            acc = (acc << l) | (t & 0xFFFFFFu);
            nfill += l;
            if (nfill >= 32) {
              nfill -= 32;
              pw[nw++] = (uint32_t)(acc >> nfill);
            }
          }
        } else {
          uint32_t bits = 0;
#pragma unroll
          for (int i = 0; i < kSValues; i++) {
            if ((i & 15) == 0) qoff[i >> 4] = bits;
            if (i < cnt) {
              const uint32_t ek = sm.enc[e][symbol<DT, kSValues>(raw, e, i)];
              const uint32_t l = ek >> 16;
              bits += l;
              acc = (acc << l) | (ek & 0xFFFFu);
              nfill += l;
              if (nfill >= 32) {
                nfill -= 32;
                pw[nw++] = (uint32_t)(acc >> nfill);
              }
            }
          }
        }
        const uint32_t mybits = nw * 32 + nfill;
        if (nfill) pw[nw++] = (uint32_t)(acc << (32 - nfill));
        // my bit offset in the pass: a warp scan, then the four warp totals after one
        // barrier. The totals alternate between two slots by scan parity: a slot is written
        // again two scans later, after the barriers between, when every thread has read it.
        uint32_t pass_bits, myoff;
        {
          uint32_t x = mybits;
#pragma unroll
          for (int o = 1; o < 32; o <<= 1) {
            const uint32_t y = __shfl_up_sync(0xFFFFFFFFu, x, o);
            if (lane >= o) x += y;
          }
          if (lane == 31) sm.warp[ph & 1][warp] = x;
          __syncthreads();
          const uint4 t = *reinterpret_cast<const uint4*>(sm.warp[ph & 1]);
          ph++;
          pass_bits = t.x + t.y + t.z + t.w;
          myoff = x - mybits + (warp > 0 ? t.x : 0u) + (warp > 1 ? t.y : 0u) + (warp > 2 ? t.z : 0u);
        }
        const uint64_t Pe = P[e];
        if (cnt > 0) {
          uint32_t rr = v0 % g.S;
#pragma unroll
          for (int q = 0; q < kSValues / 16; q++) {
            if (rr == 0 && 16 * q < cnt) idx[(v0 + 16 * q) / g.S] = (uint32_t)(Pe + myoff + qoff[q]);
            rr += 16;
            if (rr >= g.S) rr -= g.S;
          }
        }
        if (mybits) {
          const uint32_t q0 = (uint32_t)(Pe & 31) + myoff;
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
        const uint64_t end = Pe + pass_bits;
        const uint32_t nwt = (uint32_t)(((Pe & 31) + pass_bits + 31) >> 5);
        const uint64_t W0 = Pe >> 5;
        for (uint32_t i = 1 + tid; i + 1 < nwt; i += kSThreads) {  // middle words: plain
          const uint32_t word = sm.stage[i];
          sm.stage[i] = 0;
          bs[W0 + i] = bswap32(word);
        }
        if (tid < 2 && nwt > 0 && (tid == 0 || nwt > 1)) {  // edge words: thread 0 the first, 1 the last
          const uint32_t i = tid == 0 ? 0u : nwt - 1;
          uint32_t word = sm.stage[i];
          sm.stage[i] = 0;
          if (i == 0 && pass > 0 && (Pe & 31) != 0) word |= sm.carry[e][(pass - 1) & 1];
          uint32_t* dst = bs + W0 + i;
          uint64_t* slot = ws.slot + (uint64_t)e * g.n_tiles;
          if (i == nwt - 1 && (end & 31) != 0 && !tile_end) sm.carry[e][pass & 1] = word;  // completed by the next pass
          else if (i == 0 && pass == 0 && (Pe & 31) != 0) sub_slot_merge(slot + tile, word, dst);
          else if (i == nwt - 1 && (end & 31) != 0 && !last) sub_slot_merge(slot + tile + 1, word, dst);
          else *dst = bswap32(word);
        }
        P[e] = end;
        if (last) {
          const uint64_t padded_words = round16(ceil_div(end, 8)) / 4;
          for (uint64_t i = W0 + nwt + tid; i < padded_words; i += kSThreads) bs[i] = 0;
          for (uint64_t i = nsub + tid; i < idx_bytes / 4; i += kSThreads) idx[i] = 0;
        }
        __syncthreads();  // the staging words are clear before the next stream or pass stages
      };
      huff_stream(std::integral_constant<int, 0>{});
      huff_stream(std::integral_constant<int, 1>{});
    }
  }
}

template <int DT>
static cudaError_t encode_sub_t(const void* src, const Geo& g, const Ws& ws, uint8_t* out, cudaStream_t st) {
  const size_t smem = sizeof(SubEncodeSmem);
  static std::atomic<int> resident[128];  // blocks per device, once the attributes are set
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  int per_device = dev >= 0 && dev < 128 ? resident[dev].load(std::memory_order_relaxed) : 0;
  if (!per_device) {
    e = cudaFuncSetAttribute(k_encode_sub<DT>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e == cudaSuccess) e = cudaFuncSetAttribute(k_encode_sub<DT>, cudaFuncAttributePreferredSharedMemoryCarveout, 100);
    int per_sm = 0, sms = 0;
    if (e == cudaSuccess) e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, k_encode_sub<DT>, kSThreads, smem);
    if (e == cudaSuccess) e = cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    if (e != cudaSuccess) return e;
    per_device = (per_sm > 0 ? per_sm : 1) * (sms > 0 ? sms : 1);
    if (dev >= 0 && dev < 128) resident[dev].store(per_device, std::memory_order_relaxed);
  }
  const uint32_t blocks = (uint32_t)min64((uint64_t)per_device, g.n_tiles);
  k_encode_sub<DT><<<blocks, kSThreads, smem, st>>>(static_cast<const uint8_t*>(src), g, ws, out);
  return cudaGetLastError();
}

cudaError_t launch_encode_sub(const void* src, const Geo& g, const Ws& ws, uint8_t* out, cudaStream_t st) {
  switch (g.dt) {
    case kFP8: return encode_sub_t<kFP8>(src, g, ws, out, st);
    case kFP4: return encode_sub_t<kFP4>(src, g, ws, out, st);
    default: return cudaErrorInvalidValue;
  }
}

}  // namespace zipnn

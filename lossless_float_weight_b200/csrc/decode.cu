// decode.cu -- k_decode: container -> tensor, the inverse of the split and the coding.
//
// One block per chunk. Every block checks the header against the call's arguments and
// its chunk's table entries; every read is bounded by the container size, so a damaged
// container yields ZIPNN_ERR_CORRUPT and never an out-of-bounds access.
// For each HUFF stream the block rebuilds the canonical code from its 4-bit lengths
// and fills a 4096-entry lookup table in shared memory. An entry of the table, indexed
// by the next 12 bits of the stream, holds the first code's symbol and length and,
// when the second code also ends inside those 12 bits, that symbol and the two codes'
// total length too, so the BF16 paths take two exponents per lookup (the window holds
// two whole codes for almost every pair of a weight tensor's exponents). Layout:
//   bits 0..3 first length | 4..7 total length of two codes, 0 if the window holds one
//   bit 15 no code starts with these bits | 16..23 first symbol | 24..31 second symbol
// Each thread then decodes whole sub-blocks of S symbols, starting at the bit
// offset idx[j], merges the streams back into BF16/FP32/FP8 words and writes them to
// HBM with 16-byte stores: no intermediate plane is materialised. A sub-block must end
// exactly where the next one starts.
#include <atomic>

#include "bulk.cuh"
#include "common.cuh"
#include "fields.cuh"
#include "huffman.cuh"
#include "launch.h"

namespace zipnn {

constexpr int kDecodeThreads = 256;
constexpr uint32_t kLutInvalid = 0x8000u;
constexpr uint32_t kQuadInvalid = 0x4000u;  // FP4 four-symbol entries: not four valid codes
// The wide window's table (11-bit windows): a window that starts a 12-bit code
constexpr uint32_t kLong11 = 0x4000u;
// A PACK stream's table entries hold the pair's exponents (bits 16..23 the first, 24..31
// the second) and these flags for an escaped one (whose 8 bits follow the code)
constexpr uint32_t kPackEscHi = 0x10u, kPackEscLo = 0x20u;

__device__ __forceinline__ uint32_t lut_symbol(uint32_t e) { return (e >> 16) & 0xFFu; }

__device__ const uint32_t kZeroWord[1] = {0};  // the word an empty stream reads

// Streams decoded through a code table: HUFF, and PACK (packed exponent pairs).
__device__ __forceinline__ bool coded(uint32_t mode) { return mode == kModeHuff || mode == kModePack; }

// Big-endian-within-word bit reader over 32-bit words [0, nwords); a read past the last
// word sees the last word (a valid stream never consumes those bits; one that does ends
// past its bound and is reported). buf holds nb valid bits, most significant first; the next two words
// are already loaded (q0, q1), so a refill never waits on memory that was requested
// less than two refills ago.
struct BitReader {
  const uint32_t* w;
  uint32_t pos, last;  // pos: next word to request; last: the last word a read may touch
  uint64_t buf;
  int nb;
  uint32_t q0, q1;     // the next two words as stored (byte-swapped when they enter buf)
  __device__ __forceinline__ uint32_t load(uint32_t i) const { return __ldg(w + min(i, last)); }
  __device__ __forceinline__ void init(const uint32_t* words, uint32_t nwords, uint64_t bit) {
    w = nwords ? words : kZeroWord;
    last = nwords ? nwords - 1 : 0;
    const uint32_t p0 = (uint32_t)(bit >> 5);
    buf = (uint64_t)bswap32(load(p0)) << 32;
    q0 = load(p0 + 1);
    q1 = load(p0 + 2);
    pos = p0 + 3;
    nb = 32;
    const int skip = (int)(bit & 31);
    buf <<= skip;
    nb -= skip;
    refill();
  }
  __device__ __forceinline__ void refill() {
    if (nb <= 32) {
      buf |= (uint64_t)bswap32(q0) << (32 - nb);
      nb += 32;
      q0 = q1;
      q1 = load(pos++);
    }
  }
  __device__ __forceinline__ uint32_t fixed(int width) {
    const uint32_t v = (uint32_t)(buf >> (64 - width));
    buf <<= width;
    nb -= width;
    return v;
  }
  __device__ __forceinline__ uint32_t huff(const uint32_t* lut, uint32_t& acc) {
    const uint32_t e = lut[buf >> 52];
    const uint32_t l = e & 15u;
    buf <<= l;
    nb -= (int)l;
    acc |= e;
    return lut_symbol(e);
  }
  __device__ __forceinline__ uint32_t peek12() const { return (uint32_t)(buf >> 52); }
  __device__ __forceinline__ void skip(uint32_t l) {
    buf <<= l;
    nb -= (int)l;
  }
  // absolute index of the next unread bit
  __device__ __forceinline__ uint64_t position() const { return (uint64_t)(pos - 2) * 32 - (uint64_t)nb; }
};

// Two symbols from either bit reader, returned in bits 16..31 (the first in 16..23).
// Needs a full 12-bit window on entry; when the window holds only one whole code the
// reader refills once between the two lookups.
template <class Reader>
__device__ __forceinline__ uint32_t huff_pair(Reader& br, const uint32_t* lut, uint32_t& acc) {
  const uint32_t e = lut[br.peek12()];
  acc |= e;
  const uint32_t lp = (e >> 4) & 15u;
  if (lp) {
    br.skip(lp);
    return e;
  }
  br.skip(e & 15u);
  br.refill();
  const uint32_t e2 = lut[br.peek12()];
  acc |= e2;
  br.skip(e2 & 15u);
  return (e & 0x00FF0000u) | ((e2 & 0x00FF0000u) << 8);
}

enum Kind : int { kKZero = 0, kKBytes = 1, kKBits = 2, kKHuff = 3, kKZrun = 4, kKPack = 5 };

struct StreamState {
  int kind, width;       // kKPack: width is the number of packed exponents K
  const uint8_t* pexp;   // kKPack: the packed exponents
  const uint8_t* bytes;  // kKBytes: this sub-block's first byte; kKZrun: the kept bytes
  BitReader br;
  const uint32_t* lut;
  uint32_t acc;
  // kKZrun: the block bitmap (MSB first), the kept bytes available, the sub-block's first
  // value in the chunk, and the marked blocks before the current one
  const uint8_t* zmap;
  uint64_t zlimit;
  uint32_t zbase, zrank, zmarked, zbad;
};

// Marked blocks before block b0 of a zero-run bitmap (MSB first within each byte).
__device__ __forceinline__ uint32_t zrun_rank(const uint8_t* map, uint32_t b0) {
  uint32_t r = 0;
  const uint32_t* w = reinterpret_cast<const uint32_t*>(map);
  for (uint32_t i = 0; i < (b0 >> 5); i++) r += __popc(__ldg(w + i));
  for (uint32_t i = (b0 >> 5) * 4; i < (b0 >> 3); i++) r += __popc((uint32_t)map[i]);
  if (b0 & 7u) r += __popc((uint32_t)map[b0 >> 3] >> (8 - (b0 & 7u)));
  return r;
}

// The symbols of one stream for GV consecutive values (GV a multiple of 2; n <= GV
// valid), packed into one register: symbol i at bits SB * i (SB = 4 for FP8 and FP4,
// whose symbols have at most 4 bits; 8 otherwise). v: the group's first value in the
// sub-block.
template <int GV, int SB, bool FULL>
__device__ __forceinline__ uint64_t next_packed(StreamState& st, int n, uint32_t v) {
  static_assert(GV * SB <= 64, "a group's symbols fit one register");
  uint64_t o = 0;
  switch (st.kind) {
    case kKHuff:
#pragma unroll
      for (int i = 0; i < GV; i += 2) {
        st.br.refill();
        uint32_t a, b;
        if (FULL) {  // two symbols a lookup when the 12-bit window holds both codes
          const uint32_t p = huff_pair(st.br, st.lut, st.acc);
          a = (p >> 16) & 0xFFu;
          b = p >> 24;
        } else {
          a = i < n ? st.br.huff(st.lut, st.acc) : 0u;
          b = i + 1 < n ? st.br.huff(st.lut, st.acc) : 0u;
        }
        o |= (uint64_t)(a | (b << SB)) << (SB * i);
      }
      break;
    case kKPack:
      if constexpr (SB == 8) {
        // packed exponent pairs: one code a pair (a refill leaves at least 32 bits: a
        // code and two escaped exponents take at most 28)
#pragma unroll
        for (int i = 0; i < GV; i += 2) {
          if (!FULL && i >= n) break;
          st.br.refill();
          const uint32_t e = st.lut[st.br.peek12()];  // a pair entry with its exponents
          st.acc |= e;
          st.br.skip(e & 15u);
          const uint32_t a = (e & kPackEscHi) ? st.br.fixed(8) : (e >> 16) & 0xFFu;
          const uint32_t b = (e & kPackEscLo) ? st.br.fixed(8) : e >> 24;
          o |= (uint64_t)(a | (b << 8)) << (8 * i);
        }
      }
      break;
    case kKBits:
#pragma unroll
      for (int i = 0; i < GV; i += 2) {
        st.br.refill();
        const uint32_t a = (FULL || i < n) ? st.br.fixed(st.width) : 0u;
        const uint32_t b = (FULL || i + 1 < n) ? st.br.fixed(st.width) : 0u;
        o |= (uint64_t)(a | (b << SB)) << (SB * i);
      }
      break;
    case kKBytes:
      if constexpr (SB == 8) {
        if (FULL) {
          if constexpr (GV == 8) {
            const uint2 q = __ldg(reinterpret_cast<const uint2*>(st.bytes + v));
            o = q.x | ((uint64_t)q.y << 32);
          } else {
            o = __ldg(reinterpret_cast<const uint32_t*>(st.bytes + v));
          }
        } else {
#pragma unroll
          for (int i = 0; i < GV; i++)
            if (i < n) o |= (uint64_t)st.bytes[v + i] << (8 * i);
        }
      }
      break;
    case kKZrun:
      if constexpr (SB == 8) {
        // zero runs: a group (GV divides 32) lies in one block; a block's bytes are kept
        // when its bitmap bit is set, at 32 x (marked blocks before it)
        const uint32_t vv = st.zbase + v;
        if (v == 0 || (vv & 31u) == 0) {
          if (v != 0) st.zrank += st.zmarked;
          st.zmarked = ((uint32_t)st.zmap[vv >> 8] >> (7 - ((vv >> 5) & 7u))) & 1u;
        }
        const uint64_t at = (uint64_t)st.zrank * kZBlock + (vv & 31u);
        if (st.zmarked && at + GV <= st.zlimit) {
          const uint8_t* src = st.bytes + at;
          if (FULL) {
            if constexpr (GV == 8) {
              const uint2 q = __ldg(reinterpret_cast<const uint2*>(src));
              o = q.x | ((uint64_t)q.y << 32);
            } else {
              o = __ldg(reinterpret_cast<const uint32_t*>(src));
            }
          } else {
#pragma unroll
            for (int i = 0; i < GV; i++)
              if (i < n) o |= (uint64_t)src[i] << (8 * i);
          }
        } else if (st.zmarked) {
          st.zbad = 1;  // kept bytes past the payload: corrupt
        }
      }
      break;
    default:
      break;
  }
  return o;
}

// FP8: eight 4-bit symbols (nibble i of x) as eight bytes, in two words.
__device__ __forceinline__ void nibbles_to_bytes(uint32_t x, uint32_t& w0, uint32_t& w1) {
  const uint32_t lo = x & 0x0F0F0F0Fu, hi = (x >> 4) & 0x0F0F0F0Fu;  // nibbles 0,2,4,6 / 1,3,5,7
  w0 = __byte_perm(lo, hi, 0x5140);
  w1 = __byte_perm(lo, hi, 0x7362);
}

// Two BF16 words (the merge) from two sign/fraction bytes, bytes 2*sf_hi and 2*sf_hi + 1
// of sf, and two exponents, bytes 2*ex_hi and 2*ex_hi + 1 of ex. Each sign/fraction byte
// is copied into both bytes of its 16-bit half; the mask keeps its fraction bits 6..0
// and, from the copy one byte up, its sign at bit 15; the exponent, moved to bits 7..14
// by a multiply by 128, adds in without carries (those bits are clear in the masked word).
__device__ __forceinline__ uint32_t bf16_merge_pair(uint32_t sf, int sf_hi, uint32_t ex, int ex_hi) {
  const uint32_t y = __byte_perm(sf, 0, sf_hi ? 0x3322 : 0x1100) & 0x807F807Fu;
  return __byte_perm(ex, 0, ex_hi ? 0x4342 : 0x4140) * 128u + y;
}

// BF16 with a HUFF exponent stream and a RAW (or ZERO) sign/fraction stream: the case
// of every chunk of a trained or Gaussian checkpoint. 16 values per step; the
// sign/fraction bytes of the next step are requested one step ahead.
// A packed exponent pair (PACK streams) from either bit reader: one code, whose table
// entry already holds the pair's two exponents (set when the table is built: the pair
// symbol's nibbles index the packed exponents) and flags for the escaped ones, whose
// 8 bits follow the code (first, then second). Returns the pair in bits 16..31 (the
// first in 16..23), as huff_pair does. Needs 28 bits in the reader.
template <class Reader>
__device__ __forceinline__ uint32_t pack_pair(Reader& br, const uint32_t* lut, uint32_t& acc) {
  const uint32_t e = lut[br.peek12()];
  acc |= e;
  br.skip(e & 15u);
  uint32_t a = (e >> 16) & 0xFFu, b = e >> 24;
  if (e & kPackEscHi) a = br.fixed(8);
  if (e & kPackEscLo) b = br.fixed(8);
  return (a << 16) | (b << 24);
}

template <bool SM_ZERO, bool PACK = false>
__device__ __forceinline__ int decode_bf16_fast(const uint32_t* lut, const uint8_t* smp, const uint32_t* bs,
                                                uint32_t bs_words, uint64_t start, uint64_t expect, bool exact,
                                                uint32_t count, uint8_t* __restrict__ dst,
                                                const uint8_t* pexp = nullptr, uint32_t valid = 0) {
  BitReader br;
  br.init(bs, bs_words, start);
  uint32_t acc = 0;
  const uint32_t full = count / 16;
  uint4 cur = make_uint4(0, 0, 0, 0), nxt = cur, nx2 = cur, nx3 = cur;
  if (!SM_ZERO) {
    const uint4* sp = reinterpret_cast<const uint4*>(smp);
    if (full > 0) cur = __ldg(sp);
    if (full > 1) nxt = __ldg(sp + 1);
    if (full > 2) nx2 = __ldg(sp + 2);
    if (full > 3) nx3 = __ldg(sp + 3);
  }
  for (uint32_t gi = 0; gi < full; gi++) {
    uint32_t pr[8];  // exponent pairs in bits 16..31
    if (PACK) {
#pragma unroll
      for (int i = 0; i < 8; i++) {
        br.refill();
        pr[i] = pack_pair(br, lut, acc);
      }
    } else {
#pragma unroll
      for (int i = 0; i < 8; i += 2) {
        br.refill();
        pr[i] = huff_pair(br, lut, acc);
        pr[i + 1] = huff_pair(br, lut, acc);
      }
    }
    const uint32_t x[4] = {cur.x, cur.y, cur.z, cur.w};
    if (!SM_ZERO) {
      cur = nxt;
      nxt = nx2;
      nx2 = nx3;
      if (gi + 4 < full) nx3 = __ldg(reinterpret_cast<const uint4*>(smp) + gi + 4);
    }
    uint32_t o[8];
#pragma unroll
    for (int q = 0; q < 8; q++) o[q] = bf16_merge_pair(SM_ZERO ? 0u : x[q >> 1], q & 1, pr[q], 1);
    uint4* d = reinterpret_cast<uint4*>(dst + (uint64_t)gi * 32);
    d[0] = make_uint4(o[0], o[1], o[2], o[3]);
    d[1] = make_uint4(o[4], o[5], o[6], o[7]);
  }
  if (PACK) {  // count is even
    for (uint32_t v = full * 16; v < count; v += 2) {
      br.refill();
      const uint32_t pr = pack_pair(br, lut, acc);
      const uint32_t b0 = SM_ZERO ? 0u : smp[v], b1 = SM_ZERO ? 0u : smp[v + 1];
      reinterpret_cast<uint16_t*>(dst)[v] = (uint16_t)merge_value<kBF16>((pr >> 16) & 0xFFu, b0, 0, 0);
      reinterpret_cast<uint16_t*>(dst)[v + 1] = (uint16_t)merge_value<kBF16>(pr >> 24, b1, 0, 0);
    }
  } else {
    for (uint32_t v = full * 16; v < count; v++) {
      br.refill();
      const uint32_t e = br.huff(lut, acc);
      const uint32_t b = SM_ZERO ? 0u : smp[v];
      reinterpret_cast<uint16_t*>(dst)[v] = (uint16_t)merge_value<kBF16>(e, b, 0, 0);
    }
  }
  const uint64_t pos = br.position();
  return (acc & kLutInvalid) || (exact ? pos != expect : pos > expect);
}

// FP8 and FP4 with a HUFF exponent stream and RAW (or ZERO: MZ, SZ) mantissa and sign
// streams, the case of every chunk whose mantissas are near uniform: one sub-block, 32
// values a step. The exponents come two a lookup; the step's RAW words (FP8: three
// mantissa words and one sign word, FP4: one of each; value v's bits at v * width, so a
// step of 32 values starts on a word) are requested two steps ahead into one of two
// register sets and kept as loaded (byte-swapped only when used, so no instruction waits
// on them early); their fields are
// spread into the output bytes or nibbles with shifts, masks and multiplies. QUAD (FP4
// exponents of at most 3 bits): four exponents a lookup. mwp / swp:
// the sub-block's first mantissa / sign word (S is a multiple of 32), or nullptr (ZERO).
// Returns nonzero if the stream is inconsistent.
template <int DT, bool MZ, bool SZ, bool QUAD = false>
__device__ __forceinline__ int decode_sub_fast(const uint32_t* lut, const uint32_t* bs, uint32_t bs_words,
                                               uint64_t start, uint64_t expect, bool exact, const uint32_t* mwp,
                                               const uint32_t* swp, uint32_t count, uint8_t* __restrict__ dst) {
  constexpr int WM = raw_width(DT, 1);  // mantissa bits: FP8 3, FP4 1
  BitReader br;
  br.init(bs, bs_words, start);
  uint32_t acc = 0, qacc = 0;  // OR of the entries: single / pair lookups, four-symbol lookups
  const uint32_t full = count / 32;
  // the RAW words of two steps in flight, as loaded: set 0 for even steps, set 1 for odd;
  // a set is refilled for the step two ahead right after its words are used
  uint32_t mw[2][WM], sw[2];
  auto fetch = [&](int k, uint32_t g) {
#pragma unroll
    for (int i = 0; i < WM; i++) mw[k][i] = MZ || g >= full ? 0u : __ldg(mwp + g * WM + i);
    sw[k] = SZ || g >= full ? 0u : __ldg(swp + g);
  };
  fetch(0, 0);
  fetch(1, 1);
  auto step = [&](uint32_t gi, int k, uint32_t* out16) {
    uint32_t pr[16];  // exponent pairs in bits 16..31 (QUAD: four exponents in bits 0..7 of pr[0..7])
    if constexpr (QUAD) {
#pragma unroll
      for (int i = 0; i < 8; i += 2) {
        br.refill();
#pragma unroll
        for (int j = 0; j < 2; j++) {
          const uint32_t e = lut[br.peek12()];
          qacc |= e;
          br.skip((e >> 4) & 15u);
          pr[i + j] = e >> 24;
        }
      }
    } else {
#pragma unroll
      for (int i = 0; i < 16; i += 2) {
        br.refill();
        pr[i] = huff_pair(br, lut, acc);
        pr[i + 1] = huff_pair(br, lut, acc);
      }
    }
    uint32_t M[WM];
#pragma unroll
    for (int i = 0; i < WM; i++) M[i] = bswap32(mw[k][i]);
    const uint32_t Sg = bswap32(sw[k]);
    fetch(k, gi + 2);
    if constexpr (DT == kFP8) {
      // byte of value 4k + i: sign << 7 | exponent << 3 | mantissa
      uint32_t o[8];
#pragma unroll
      for (int q = 0; q < 8; q++) {
        const uint32_t ew = __byte_perm(pr[2 * q], pr[2 * q + 1], 0x7632);
        const int a = 12 * q / 32, b = 12 * q % 32;  // the four mantissas: bits [12q, 12q + 12)
        const uint32_t y = __funnelshift_l(a + 1 < WM ? M[a + 1 < WM ? a + 1 : 0] : 0u, M[a], b) >> 20;
        const uint32_t mv = (y >> 9) | ((y << 2) & 0x700u) | ((y << 13) & 0x70000u) | ((y << 24) & 0x7000000u);
        const uint32_t sv = (((Sg >> (28 - 4 * q)) & 0xFu) * 0x80402010u) & 0x80808080u;
        o[q] = (ew << 3) | mv | sv;
      }
      uint8_t* dp = dst + (uint64_t)gi * 32;
      if ((reinterpret_cast<uintptr_t>(dp) & 31) == 0) {
        st_v8(dp, o);
      } else {
        uint4* d = reinterpret_cast<uint4*>(dp);
        d[0] = make_uint4(o[0], o[1], o[2], o[3]);
        d[1] = make_uint4(o[4], o[5], o[6], o[7]);
      }
    } else {
      // nibble of value 8q + i (value 2j the low nibble of byte j): sign << 3 |
      // exponent << 1 | mantissa; a byte of bits (value 8q first) spreads to bit 0 of the
      // eight nibbles after its bits are reversed
      auto spread = [](uint32_t byte) {
        uint32_t t = __brev(byte) >> 24;
        t = (t | (t << 12)) & 0x000F000Fu;
        t = (t | (t << 6)) & 0x03030303u;
        return (t | (t << 3)) & 0x11111111u;
      };
      uint32_t o[4];
#pragma unroll
      for (int q = 0; q < 4; q++) {
        uint32_t en;
        if constexpr (QUAD) {
          // eight 2-bit exponents (value 8q first, lowest) spread to nibbles
          uint32_t t = pr[2 * q] | (pr[2 * q + 1] << 8);
          t = (t | (t << 8)) & 0x00FF00FFu;
          t = (t | (t << 4)) & 0x0F0F0F0Fu;
          en = (t | (t << 2)) & 0x33333333u;
        } else {
          const uint32_t e0 = __byte_perm(pr[4 * q], pr[4 * q + 1], 0x7632);
          const uint32_t e1 = __byte_perm(pr[4 * q + 2], pr[4 * q + 3], 0x7632);
          en = __byte_perm(e0 | (e0 >> 4), e1 | (e1 >> 4), 0x6420);
        }
        const uint32_t mb = (M[0] >> (24 - 8 * q)) & 0xFFu, sb = (Sg >> (24 - 8 * q)) & 0xFFu;
        o[q] = (en << 1) | spread(mb) | (spread(sb) << 3);
      }
#pragma unroll
      for (int q = 0; q < 4; q++) out16[q] = o[q];
    }
  };
  for (uint32_t gi = 0; gi < full; gi += 2) {
    if constexpr (DT == kFP8) {
      step(gi, 0, nullptr);
      if (gi + 1 < full) step(gi + 1, 1, nullptr);
    } else {
      // FP4: the two steps' 16 bytes each go out as one 32-byte store where aligned
      uint32_t o8[8];
      step(gi, 0, o8);
      uint8_t* dp = dst + (uint64_t)gi * 16;
      if (gi + 1 < full) {
        step(gi + 1, 1, o8 + 4);
        if ((reinterpret_cast<uintptr_t>(dp) & 31) == 0) {
          st_v8(dp, o8);
        } else {
          *reinterpret_cast<uint4*>(dp) = make_uint4(o8[0], o8[1], o8[2], o8[3]);
          *reinterpret_cast<uint4*>(dp + 16) = make_uint4(o8[4], o8[5], o8[6], o8[7]);
        }
      } else {
        *reinterpret_cast<uint4*>(dp) = make_uint4(o8[0], o8[1], o8[2], o8[3]);
      }
    }
  }
  // the sub-block's last values (fewer than 32; FP4 an even number)
  auto bits_at = [](const uint32_t* p, uint32_t bit, int width) {
    const uint32_t i = bit >> 5, o = bit & 31;
    uint32_t x = bswap32(__ldg(p + i)) << o;
    if (o + width > 32) x |= bswap32(__ldg(p + i + 1)) >> (32 - o);
    return x >> (32 - width);
  };
  for (uint32_t v = full * 32; v < count; v++) {
    br.refill();
    const uint32_t e = br.huff(lut, acc);
    const uint32_t mv = MZ ? 0u : bits_at(mwp, v * WM, WM), sv = SZ ? 0u : bits_at(swp, v, 1);
    if constexpr (DT == kFP8) {
      dst[v] = (uint8_t)((sv << 7) | (e << 3) | mv);
    } else {
      const uint32_t nib = (sv << 3) | (e << 1) | mv;
      if (v & 1) dst[v >> 1] = (uint8_t)(dst[v >> 1] | (nib << 4));
      else dst[v >> 1] = (uint8_t)nib;
    }
  }
  const uint64_t pos = br.position();
  return (acc & kLutInvalid) || (qacc & (kLutInvalid | kQuadInvalid)) || (exact ? pos != expect : pos > expect);
}

// FP32 with a HUFF exponent stream and RAW (or ZERO: nullptr) byte planes p1 (sign and
// fraction bits 22..16), p2 (bits 15..8), p3 (bits 7..0): one sub-block, 16 values a
// step. The exponents come two a lookup. A value's upper half is a BF16 word (p1 byte, exponent), merged two at a
// time; its lower half is the p3 byte under the p2 byte; byte permutes join them. The
// step's plane bytes are requested before its exponents are decoded.
__device__ __forceinline__ int decode_fp32_fast(const uint32_t* lut, const uint32_t* bs, uint32_t bs_words,
                                                uint64_t start, uint64_t expect, bool exact, const uint8_t* p1,
                                                const uint8_t* p2, const uint8_t* p3, uint32_t count,
                                                uint8_t* __restrict__ dst) {
  BitReader br;
  br.init(bs, bs_words, start);
  uint32_t acc = 0;
  const uint32_t full = count / 16;
  const uint8_t* pl[3] = {p1, p2, p3};
  for (uint32_t gi = 0; gi < full; gi++) {
    // the step's plane bytes, requested before its exponents are decoded
    uint4 pv[3];
#pragma unroll
    for (int k = 0; k < 3; k++)
      pv[k] = pl[k] ? __ldg(reinterpret_cast<const uint4*>(pl[k]) + gi) : make_uint4(0, 0, 0, 0);
    uint32_t pr[8];  // exponent pairs in bits 16..31
#pragma unroll
    for (int i = 0; i < 8; i += 2) {
      br.refill();
      pr[i] = huff_pair(br, lut, acc);
      pr[i + 1] = huff_pair(br, lut, acc);
    }
    const uint32_t x[3][4] = {{pv[0].x, pv[0].y, pv[0].z, pv[0].w},
                              {pv[1].x, pv[1].y, pv[1].z, pv[1].w},
                              {pv[2].x, pv[2].y, pv[2].z, pv[2].w}};
    uint32_t o[16];
#pragma unroll
    for (int q = 0; q < 4; q++) {
      const uint32_t ew = __byte_perm(pr[2 * q], pr[2 * q + 1], 0x7632);  // exponents of values 4q..4q+3
      const uint32_t h01 = bf16_merge_pair(x[0][q], 0, ew, 0), h23 = bf16_merge_pair(x[0][q], 1, ew, 1);
      const uint32_t l01 = __byte_perm(x[2][q], x[1][q], 0x5140), l23 = __byte_perm(x[2][q], x[1][q], 0x7362);
      o[4 * q] = __byte_perm(l01, h01, 0x5410);
      o[4 * q + 1] = __byte_perm(l01, h01, 0x7632);
      o[4 * q + 2] = __byte_perm(l23, h23, 0x5410);
      o[4 * q + 3] = __byte_perm(l23, h23, 0x7632);
    }
    uint8_t* dp = dst + (uint64_t)gi * 64;
    if ((reinterpret_cast<uintptr_t>(dp) & 31) == 0) {
      st_v8(dp, o);
      st_v8(dp + 32, o + 8);
    } else {
      uint4* d = reinterpret_cast<uint4*>(dp);
#pragma unroll
      for (int q = 0; q < 4; q++) d[q] = make_uint4(o[4 * q], o[4 * q + 1], o[4 * q + 2], o[4 * q + 3]);
    }
  }
  for (uint32_t v = full * 16; v < count; v++) {
    br.refill();
    const uint32_t e = br.huff(lut, acc);
    reinterpret_cast<uint32_t*>(dst)[v] =
        merge_value<kFP32>(e, p1 ? p1[v] : 0u, p2 ? p2[v] : 0u, p3 ? p3[v] : 0u);
  }
  const uint64_t pos = br.position();
  return (acc & kLutInvalid) || (exact ? pos != expect : pos > expect);
}

// ---------------------------------------------------------------- staged BF16 path
// For a BF16 chunk whose exponent stream is HUFF (or PACK) and whose bitstream fits a 48 KB
// window, the whole bitstream is brought into shared memory by one TMA bulk copy
// (cp.async.bulk, completion on an mbarrier) while the block builds its lookup table.
// Then, in rounds, every thread decodes the next 32 exponents of its sub-block into
// its row of a shared buffer, and each warp merges its own 32 rows with the sign/fraction
// bytes (so a round needs only warp barriers, and the warps of a block run at their own
// pace): those are loaded as whole 32-byte sectors one round ahead of use, and the
// merged words leave as whole 64-byte row segments. Word k of row r sits at
// 8r + (k ^ (r / 4 mod 8)): the row-per-thread stores and the unit-per-thread loads
// of the merge both touch 32 distinct banks, with no padding.
constexpr uint32_t kWindowBytes = 48 * 1024;
// A bitstream of 48 to 56 KB (exponents of more than 3 bits on average, as in K/V
// caches) still decodes from shared memory: its last 8 KB go to the first half of the
// decode table's 16 KB, and the second half holds a two-symbol table of 11-bit windows
// (2048 u32 entries) instead of the 12-bit one.
constexpr uint32_t kWideWindowBytes = 56 * 1024;
constexpr uint32_t kWindowWords = kWindowBytes / 4, kWideWords = kWideWindowBytes / 4;
constexpr int kRound = 32;  // exponents of a sub-block decoded per round
constexpr int kRowWords = kRound / 4;
constexpr uint32_t kWaitLimit = 1u << 26;

struct StagedSmem {
  uint32_t bits[kWindowBytes / 4];
  uint32_t ex[kDecodeThreads * kRowWords];
  uint64_t bar;
};


// Bit reader over words in shared memory, by position: c holds words p and p + 1 (p in
// the high half), bp of its bits are consumed, q is word p + 2. A refill advances one word
// when bp reaches 32 (the next word is requested one refill ahead), so a 12-bit window at
// bp <= 52 lies inside c. WIDE: words from kWindowWords on are in a second region, w2.
template <bool WIDE = false>
struct SmemBitReader {
  const uint32_t* w;
  const uint32_t* w2;
  uint32_t p, end, bp, q;
  uint64_t c;
  // Word i of the bitstream. Past the end a reader sees the word at `end` (stale data or
  // the next buffer, always inside the block's shared memory): a valid sub-block never
  // consumes those bits, and one that does ends past its bound and is reported.
  __device__ __forceinline__ uint32_t ld(uint32_t i) const {
    i = min(i, end);
    if constexpr (WIDE) return bswap32(i < kWindowWords ? w[i] : w2[i - kWindowWords]);
    return bswap32(w[i]);
  }
  __device__ __forceinline__ void init(const uint32_t* words, uint32_t nwords, uint64_t bit,
                                       const uint32_t* words2 = nullptr) {
    w = words;
    w2 = words2;
    end = nwords;
    p = (uint32_t)(bit >> 5);
    c = ((uint64_t)ld(p) << 32) | ld(p + 1);
    q = ld(p + 2);
    bp = (uint32_t)(bit & 31);
  }
  // The 48 KB window loads its next word only when the reader advances (fewer shared
  // loads, so fewer bank conflicts on the table's lookups); the wide window selects.
  __device__ __forceinline__ void refill() {
    if constexpr (WIDE) {
      const bool t = bp >= 32;
      const uint32_t nq = ld(p + 3);
      c = t ? (c << 32) | q : c;
      q = t ? nq : q;
      p += t ? 1u : 0u;
      bp -= t ? 32u : 0u;
    } else if (bp >= 32) {
      c = (c << 32) | q;
      q = ld(p + 3);
      p++;
      bp -= 32;
    }
  }
  __device__ __forceinline__ uint32_t peek12() const { return (uint32_t)((c << bp) >> 52); }
  __device__ __forceinline__ void skip(uint32_t l) { bp += l; }
  __device__ __forceinline__ uint32_t fixed(int width) {
    const uint32_t v = (uint32_t)((c << bp) >> (64 - width));
    bp += (uint32_t)width;
    return v;
  }
  __device__ __forceinline__ uint32_t huff(const uint32_t* lut, uint32_t& acc) {
    const uint32_t e = lut[peek12()];
    bp += e & 15u;
    acc |= e;
    return lut_symbol(e);
  }
  __device__ __forceinline__ uint32_t peek11() const { return (uint32_t)((c << bp) >> 53); }
  __device__ __forceinline__ uint64_t position() const { return (uint64_t)p * 32 + bp; }
};

__device__ __forceinline__ uint32_t ex_word(uint32_t row, uint32_t k) {
  return row * kRowWords + (k ^ ((row >> 2) & (kRowWords - 1)));
}

// The wide window's table is indexed by 11 bits (2048 u32 entries in 8 KB, the room the
// window leaves): an entry holds the first code's symbol and length and, when the second
// code also ends inside the 11 bits, its symbol and the pair's length (the two-symbol
// layout of the 12-bit table); a window that starts a 12-bit code is kLong11, and that code
// is decoded from the canonical tables (its first value, index offset and limit).
struct Long12 {
  const uint8_t* sorted;
  uint32_t first, offset, limit;
};

__device__ __forceinline__ uint32_t huff12_long(SmemBitReader<true>& br, const Long12& lg, uint32_t& acc) {
  const uint32_t w12 = br.peek12();
  if (w12 >= lg.limit || w12 < lg.first) acc |= kLutInvalid;  // no 12-bit code here: corrupt
  br.skip(12);
  return lg.sorted[(lg.offset + w12 - lg.first) & 255u];
}

// One symbol from the 11-bit table.
__device__ __forceinline__ uint32_t huff11(SmemBitReader<true>& br, const uint32_t* lut, const Long12& lg,
                                           uint32_t& acc) {
  const uint32_t e = lut[br.peek11()];
  if (e & kLong11) return huff12_long(br, lg, acc);
  acc |= e;
  br.skip(e & 15u);
  return lut_symbol(e);
}

// Two symbols from the 11-bit table, in bits 16..31 as huff_pair returns them (refilling
// once between two lookups when the window holds one code).
__device__ __forceinline__ uint32_t huff_pair11(SmemBitReader<true>& br, const uint32_t* lut, const Long12& lg,
                                                uint32_t& acc) {
  const uint32_t e = lut[br.peek11()];
  uint32_t s0;
  if (e & kLong11) {
    s0 = huff12_long(br, lg, acc);
  } else {
    acc |= e;
    const uint32_t lp = (e >> 4) & 15u;
    if (lp) {
      br.skip(lp);
      return e;
    }
    br.skip(e & 15u);
    s0 = lut_symbol(e);
  }
  br.refill();
  const uint32_t s1 = huff11(br, lut, lg, acc);
  return (s0 << 16) | (s1 << 24);
}

// A packed exponent pair from the 11-bit table (as pack_pair).
__device__ __forceinline__ uint32_t pack_pair11(SmemBitReader<true>& br, const uint32_t* lut, const Long12& lg,
                                                const uint8_t* pexp, uint32_t valid, uint32_t& acc) {
  const uint32_t e = lut[br.peek11()];
  if (e & kLong11) {  // a 12-bit pair code: its symbol's nibbles index the list here
    const uint32_t p = huff12_long(br, lg, acc);
    const uint32_t hi = p >> 4, lo = p & 15u;
    uint32_t a = pexp[hi], b = pexp[lo];
    if (hi == kPackEsc) a = br.fixed(8);
    if (lo == kPackEsc) b = br.fixed(8);
    if (!((valid >> hi) & (valid >> lo) & 1u)) acc |= kLutInvalid;
    return (a << 16) | (b << 24);
  }
  acc |= e;
  br.skip(e & 15u);
  uint32_t a = (e >> 16) & 0xFFu, b = e >> 24;
  if (e & kPackEscHi) a = br.fixed(8);
  if (e & kPackEscLo) b = br.fixed(8);
  return (a << 16) | (b << 24);
}

// One chunk, all threads of the block; one sub-block per thread and batch. WIDE: the
// bitstream continues in `tail` after the window and lut is the 11-bit two-symbol table;
// else lut is the 12-bit two-symbol table. smp: the chunk's sign/fraction payload (RAW) or
// nullptr (ZERO); outc: the chunk's first output value. Returns nonzero if the stream is
// inconsistent.
// ZRUN: the sign/fraction plane has zero runs; smp is its kept bytes, zmap / zpre the
// chunk's block bitmap words (bit i of word w: block 32w + i) and the marked blocks before
// each word, in shared memory.
// ALLFULL: every sub-block of the chunk holds S values, S is a multiple of the round and
// the sub-blocks fill whole batches, so every round decodes 32 exponents a thread and every
// merge unit holds 8 values (the case of every chunk of a weight checkpoint).
// PACK: the exponent stream is packed pairs (pexp, valid as for pack_pair); S and every
// count are even.
// WIDE: lut is the 11-bit table of the wide window (lg: its 12-bit codes).
template <bool WIDE, bool ZRUN, bool ALLFULL, bool PACK>
__device__ int decode_bf16_staged(StagedSmem& st, const uint32_t* lut, const uint32_t* tail,
                                  const uint32_t* __restrict__ idx, uint32_t bs_words,
                                  const uint8_t* __restrict__ smp, uint32_t m, uint32_t S, uint32_t nsub,
                                  uint8_t* __restrict__ outc, uint32_t pre_start, uint32_t pre_next,
                                  const uint32_t* zmap, const uint32_t* zpre, const uint8_t* pexp,
                                  uint32_t valid, Long12 lg) {
  const int tid = threadIdx.x;
  int bad = 0;
  const uint64_t cap_bits = (uint64_t)bs_words * 32;
  const uint32_t rounds = (S + kRound - 1) / kRound;
  uint8_t* exb = reinterpret_cast<uint8_t*>(st.ex);
  for (uint32_t batch = 0; batch < nsub; batch += kDecodeThreads) {
    const uint32_t j = batch + tid;
    const uint32_t count = ALLFULL ? S : j < nsub ? min32(S, m - j * S) : 0;
    SmemBitReader<WIDE> br;
    uint32_t acc = 0;
    uint64_t expect = 0;
    bool exact = false;
    if (count) {
      // the first batch's bounds were loaded by the caller while it built the tables
      const uint64_t start = batch == 0 ? pre_start : __ldg(idx + j);
      exact = j + 1 < nsub;
      expect = exact ? (batch == 0 ? pre_next : __ldg(idx + j + 1)) : cap_bits;
      if ((j == 0 && start != 0) || start > cap_bits || expect < start || expect > cap_bits) bad = 1;
      br.init(st.bits, bs_words, bad ? 0 : start, tail);
    }
    // my merge units: unit p is part tid % 4 (values 8(tid % 4)..) of row 32w + 8p +
    // lane / 4 of the batch, a row of my own warp (w), so a warp merges only the rows its
    // lanes decoded and its rounds need no block barrier; ubase is the unit's first value
    // in round 0, urem the values its row has from there on
    uint32_t ubase[4], urem[4];
#pragma unroll
    for (int p = 0; p < 4; p++) {
      const uint32_t rw = ((uint32_t)tid & ~31u) + 8u * p + (((uint32_t)tid & 31u) >> 2);
      const uint32_t row = batch + rw, part = (uint32_t)tid & 3u;
      const uint32_t rc = row < nsub ? min32(S, m - row * S) : 0;
      ubase[p] = row * S + part * 8;
      urem[p] = rc > part * 8 ? rc - part * 8 : 0;
    }
    for (uint32_t r = 0; r < rounds; r++) {
      // sign/fraction bytes of this round's merge units, requested before the decode
      uint2 smv[4];
      uint32_t uval[4], ucnt[4];
#pragma unroll
      for (int p = 0; p < 4; p++) {
        const uint32_t off = r * kRound;
        const uint32_t n = ALLFULL ? 8u : off < urem[p] ? min32(8, urem[p] - off) : 0;
        uval[p] = ubase[p] + off;
        ucnt[p] = n;
        smv[p] = make_uint2(0, 0);
        const uint8_t* src = nullptr;
        if constexpr (ZRUN) {
          const uint32_t b = uval[p] >> 5, word = zmap[b >> 5], bit = b & 31u;
          if (n && ((word >> bit) & 1u))
            src = smp + (uint64_t)(zpre[b >> 5] + __popc(word & ((1u << bit) - 1u))) * kZBlock + (uval[p] & 31u);
        } else if (smp) {
          src = smp + uval[p];
        }
        if (src && n == 8) smv[p] = __ldg(reinterpret_cast<const uint2*>(src));
        else if (src && n) {
          uint32_t lo = 0, hi = 0;
          for (uint32_t i = 0; i < n; i++) {
            const uint32_t b = src[i];
            if (i < 4) lo |= b << (8 * i);
            else hi |= b << (8 * (i - 4));
          }
          smv[p] = make_uint2(lo, hi);
        }
      }
      // decode up to 32 exponents of my sub-block, two per lookup
      const uint32_t base = r * kRound;
      if (ALLFULL || base < count) {
        if (ALLFULL || base + kRound <= count) {
#pragma unroll
          for (int k = 0; k < kRowWords; k++) {
            if constexpr (PACK && WIDE) {
              br.refill();
              const uint32_t a = pack_pair11(br, lut, lg, pexp, valid, acc);
              br.refill();
              const uint32_t b = pack_pair11(br, lut, lg, pexp, valid, acc);
              st.ex[ex_word(tid, k)] = __byte_perm(a, b, 0x7632);
            } else if constexpr (PACK) {
              br.refill();
              const uint32_t a = pack_pair(br, lut, acc);
              br.refill();
              const uint32_t b = pack_pair(br, lut, acc);
              st.ex[ex_word(tid, k)] = __byte_perm(a, b, 0x7632);
            } else if constexpr (WIDE) {
              br.refill();
              const uint32_t a = huff_pair11(br, lut, lg, acc);
              const uint32_t b = huff_pair11(br, lut, lg, acc);
              st.ex[ex_word(tid, k)] = __byte_perm(a, b, 0x7632);
            } else {
              br.refill();
              const uint32_t a = huff_pair(br, lut, acc);
              const uint32_t b = huff_pair(br, lut, acc);
              st.ex[ex_word(tid, k)] = __byte_perm(a, b, 0x7632);
            }
          }
        } else {
          const uint32_t n = count - base;
          if constexpr (PACK) {
            for (uint32_t k = 0; k < n; k += 2) {
              br.refill();
              uint32_t pr;
              if constexpr (WIDE) pr = pack_pair11(br, lut, lg, pexp, valid, acc);
              else pr = pack_pair(br, lut, acc);
              exb[ex_word(tid, k >> 2) * 4 + (k & 3)] = (uint8_t)(pr >> 16);
              exb[ex_word(tid, k >> 2) * 4 + (k & 3) + 1] = (uint8_t)(pr >> 24);
            }
          } else {
            for (uint32_t k = 0; k < n; k++) {
              br.refill();
              uint32_t sym;
              if constexpr (WIDE) sym = huff11(br, lut, lg, acc);
              else sym = br.huff(lut, acc);
              exb[ex_word(tid, k >> 2) * 4 + (k & 3)] = (uint8_t)sym;
            }
          }
        }
      }
      __syncwarp();
      // merge and store
#pragma unroll
      for (int p = 0; p < 4; p++) {
        if (!ALLFULL && !ucnt[p]) continue;
        const uint32_t row = ((uint32_t)tid & ~31u) + 8u * p + (((uint32_t)tid & 31u) >> 2), part = (uint32_t)tid & 3u;
        const uint32_t es[2] = {st.ex[ex_word(row, 2 * part)], st.ex[ex_word(row, 2 * part + 1)]};
        const uint32_t xs[2] = {smv[p].x, smv[p].y};
        uint32_t o[4];
#pragma unroll
        for (int q = 0; q < 4; q++) o[q] = bf16_merge_pair(xs[q >> 1], q & 1, es[q >> 1], q & 1);
        uint8_t* d = outc + (uint64_t)uval[p] * 2;
        if (ALLFULL || ucnt[p] == 8) {
          *reinterpret_cast<uint4*>(d) = make_uint4(o[0], o[1], o[2], o[3]);
        } else {
#pragma unroll
          for (uint32_t i = 0; i < 8; i++)
            if (i < ucnt[p]) reinterpret_cast<uint16_t*>(d)[i] = (uint16_t)(o[i >> 1] >> (16 * (i & 1)));
        }
      }
      __syncwarp();
    }
    if (count) {
      const uint64_t pos = br.position();
      if ((acc & kLutInvalid) || (exact ? pos != expect : pos > expect)) bad = 1;
    }
  }
  return bad;
}

template <int DT>
struct DecodeSmem {
  uint32_t lut[n_entropy(DT)][4096];
  uint8_t sorted[n_entropy(DT)][256];     // symbols in canonical order: by length, then symbol
  uint8_t slen[n_entropy(DT)][256];       // length of sorted[k]
  uint16_t base[n_entropy(DT)][8][16];    // canonical index of warp w's first symbol of length l
  uint8_t cnt[n_entropy(DT)][8][16];      // symbols of length l among the 32 of warp w
  uint32_t kraft[n_entropy(DT)][8];       // per warp: sum of 2^(12 - len)
  uint32_t flags[n_entropy(DT)][8];       // per warp: 1 a length above 12, 2 a symbol present
  uint32_t limit[n_entropy(DT)][kLmax + 1];
  uint32_t first[n_entropy(DT)][kLmax + 1];
  uint32_t offset[n_entropy(DT)][kLmax + 1];
  // BF16 staged path with a ZRUN sign/fraction plane: the chunk's block bitmap (up to
  // kZStagedWords words, bit i of word w = block 32w + i), the marked blocks before each
  // word, and each warp's marked blocks while the prefix is built
  uint32_t zmap[DT == kBF16 ? 128 : 1], zpre[DT == kBF16 ? 128 : 1], ztot[4];
  uint32_t mode[n_streams(DT)], code[n_streams(DT)];
  uint64_t off[n_streams(DT)], end[n_streams(DT)];
  uint64_t off_codes;
  uint32_t S, G, K;                 // K: packed exponents (BF16), 0 for none
  uint8_t pack_exps[kPackListBytes];
  int bad, staged;
  int quad;  // FP4 exponent stream with codes of at most 3 bits: table entries hold 4 symbols
};

// three BF16 decode blocks share an SM: 228 KB of shared memory, 1 KB reserved per block
static_assert(sizeof(StagedSmem) + sizeof(DecodeSmem<kBF16>) + 1024 <= 233472 / 3, "BF16 decode: 3 blocks per SM");

// Fill the decode table of one HUFF stream from its canonical tables. Canonical codes
// left-aligned to 12 bits tile [0, limit[12]) in canonical order: code k covers
// 2^(12 - len_k) entries and the next code starts where it ends. Warp w fills entries
// [512w, 512w + 512), lane l the entries 512w + l + 32j (so each store of a warp covers 32
// consecutive entries, one per bank): the lane finds the code of its first entry from the
// length limits, then walks forward over the codes that end before its next entry.
// Entries from limit[12] on match no code (only when the Kraft sum is below 1). Entries
// are symbol << 16 | length.
__device__ __forceinline__ void fill_lut(uint32_t* lut, const uint8_t* sorted, const uint8_t* slen,
                                         const uint32_t* limit, const uint32_t* first, const uint32_t* offset) {
  const uint32_t x0 = (threadIdx.x >> 5) * 512u + (threadIdx.x & 31u), lim = limit[kLmax];
  uint32_t l = 1;
  while (l < (uint32_t)kLmax && x0 >= limit[l]) l++;
  uint32_t k = 0, end = 0;
  if (x0 < lim) {
    const uint32_t c = x0 >> (kLmax - l);
    k = offset[l] + c - first[l];
    end = (c + 1) << (kLmax - l);
  }
#pragma unroll 4
  for (uint32_t j = 0; j < 16; j++) {
    const uint32_t x = x0 + 32u * j;
    uint32_t e = kLutInvalid | 1u;
    if (x < lim) {
      while (x >= end) {  // codes that end before x (each ends inside [0, lim))
        k++;
        l = slen[k];
        end += 1u << (kLmax - l);
      }
      e = ((uint32_t)sorted[k] << 16) | l;
    }
    lut[x] = e;
  }
}

static_assert(kDecodeThreads * 16 == 4096, "fill_lut: 8 warps of 512 table entries");

// The wide window's 11-bit table (first codes only; the second codes follow): window x
// is the 12-bit window x << 1; a code of at most 11 bits there gives its symbol and length,
// a 12-bit code gives kLong11, and no code (a Kraft sum below 1) gives kLutInvalid.
__device__ __forceinline__ void fill_lut11(uint32_t* lut, const uint8_t* sorted, const uint32_t* limit,
                                           const uint32_t* first, const uint32_t* offset) {
  for (uint32_t x = threadIdx.x; x < 2048; x += kDecodeThreads) {
    const uint32_t w = x << 1;
    uint32_t e = kLutInvalid | 1u;
    if (w < limit[kLmax]) {
      uint32_t l = 1;
      while (l < (uint32_t)kLmax && w >= limit[l]) l++;
      if (l == (uint32_t)kLmax) e = kLong11 | (uint32_t)kLmax;
      else e = ((uint32_t)sorted[(offset[l] + (w >> (kLmax - l)) - first[l]) & 255u] << 16) | l;
    }
    lut[x] = e;
  }
}


constexpr uint32_t kZStagedWords = 128;  // zero-run bitmap words the staged path holds: 4096 blocks
static_assert(kDecodeThreads >= kZStagedWords, "one thread per bitmap word");

// FP8 and FP4 chunks with a HUFF exponent stream and RAW or ZERO mantissa and sign
// streams (sub_fast_ok): one sub-block per thread per pass through decode_sub_fast.
template <int DT>
__device__ __forceinline__ bool sub_fast_ok(const DecodeSmem<DT>& sm, uint32_t S) {
  return sm.mode[0] == kModeHuff && (sm.mode[1] == kModeRaw || sm.mode[1] == kModeZero) &&
         (sm.mode[2] == kModeRaw || sm.mode[2] == kModeZero) && S % 32 == 0;
}

template <int DT>
__device__ __forceinline__ void decode_sub_chunk(const uint8_t* __restrict__ in, const DecodeSmem<DT>& sm, uint32_t m,
                                                 uint32_t S, uint64_t nsub, uint64_t clo, uint8_t* __restrict__ out,
                                                 uint32_t* status) {
  const bool mraw = sm.mode[1] == kModeRaw, sraw = sm.mode[2] == kModeRaw;
  for (uint64_t j = threadIdx.x; j < nsub; j += kDecodeThreads) {
    const uint32_t sb_lo = (uint32_t)(j * S);
    const uint32_t count = min32(S, m - sb_lo);
    const uint32_t rec = sm.code[0] == kNoCode ? record_bytes(DT, 0) : 0;
    const uint32_t* idx = reinterpret_cast<const uint32_t*>(in + sm.off[0] + rec);
    const uint64_t bs_off = sm.off[0] + rec + round16(4 * nsub);
    const uint64_t cap_bits = (sm.end[0] - bs_off) * 8;
    const uint64_t start = __ldg(idx + j);
    const bool exact = j + 1 < nsub;
    const uint64_t expect = exact ? __ldg(idx + j + 1) : cap_bits;
    int bad = (j == 0 && start != 0) || start > cap_bits || expect < start || expect > cap_bits;
    const uint32_t* bs = reinterpret_cast<const uint32_t*>(in + bs_off);
    const uint32_t* mwp = reinterpret_cast<const uint32_t*>(in + sm.off[1]) + (uint64_t)sb_lo * raw_width(DT, 1) / 32;
    const uint32_t* swp = reinterpret_cast<const uint32_t*>(in + sm.off[2]) + sb_lo / 32;
    uint8_t* dst = out + value_offset(DT, clo + sb_lo);
    const uint32_t bw = (uint32_t)(cap_bits / 32);
    const uint64_t st0 = bad ? 0 : start;
    if (DT == kFP4 && sm.quad) {
      constexpr bool Q = DT == kFP4;
      if (mraw && sraw) bad |= decode_sub_fast<DT, false, false, Q>(sm.lut[0], bs, bw, st0, expect, exact, mwp, swp, count, dst);
      else if (mraw) bad |= decode_sub_fast<DT, false, true, Q>(sm.lut[0], bs, bw, st0, expect, exact, mwp, nullptr, count, dst);
      else if (sraw) bad |= decode_sub_fast<DT, true, false, Q>(sm.lut[0], bs, bw, st0, expect, exact, nullptr, swp, count, dst);
      else bad |= decode_sub_fast<DT, true, true, Q>(sm.lut[0], bs, bw, st0, expect, exact, nullptr, nullptr, count, dst);
    } else {
      if (mraw && sraw) bad |= decode_sub_fast<DT, false, false>(sm.lut[0], bs, bw, st0, expect, exact, mwp, swp, count, dst);
      else if (mraw) bad |= decode_sub_fast<DT, false, true>(sm.lut[0], bs, bw, st0, expect, exact, mwp, nullptr, count, dst);
      else if (sraw) bad |= decode_sub_fast<DT, true, false>(sm.lut[0], bs, bw, st0, expect, exact, nullptr, swp, count, dst);
      else bad |= decode_sub_fast<DT, true, true>(sm.lut[0], bs, bw, st0, expect, exact, nullptr, nullptr, count, dst);
    }
    if (bad) set_status(status, kStCorrupt);
  }
}

// FP32 chunks with a HUFF exponent stream and RAW or ZERO byte planes (fp32_fast_ok):
// one sub-block per thread per pass through decode_fp32_fast.
__device__ __forceinline__ bool fp32_fast_ok(const DecodeSmem<kFP32>& sm) {
  if (sm.mode[0] != kModeHuff) return false;
  for (int s = 1; s < 4; s++)
    if (sm.mode[s] != kModeRaw && sm.mode[s] != kModeZero) return false;
  return true;
}

__device__ __forceinline__ void decode_fp32_chunk(const uint8_t* __restrict__ in, const DecodeSmem<kFP32>& sm,
                                                  uint32_t m, uint32_t S, uint64_t nsub, uint64_t clo,
                                                  uint8_t* __restrict__ out, uint32_t* status) {
  for (uint64_t j = threadIdx.x; j < nsub; j += kDecodeThreads) {
    const uint32_t sb_lo = (uint32_t)(j * S);
    const uint32_t count = min32(S, m - sb_lo);
    const uint32_t rec = sm.code[0] == kNoCode ? record_bytes(kFP32, 0) : 0;
    const uint32_t* idx = reinterpret_cast<const uint32_t*>(in + sm.off[0] + rec);
    const uint64_t bs_off = sm.off[0] + rec + round16(4 * nsub);
    const uint64_t cap_bits = (sm.end[0] - bs_off) * 8;
    const uint64_t start = __ldg(idx + j);
    const bool exact = j + 1 < nsub;
    const uint64_t expect = exact ? __ldg(idx + j + 1) : cap_bits;
    int bad = (j == 0 && start != 0) || start > cap_bits || expect < start || expect > cap_bits;
    const uint8_t* pl[3];
#pragma unroll
    for (int k = 0; k < 3; k++) pl[k] = sm.mode[k + 1] == kModeRaw ? in + sm.off[k + 1] + sb_lo : nullptr;
    bad |= decode_fp32_fast(sm.lut[0], reinterpret_cast<const uint32_t*>(in + bs_off), (uint32_t)(cap_bits / 32),
                            bad ? 0 : start, expect, exact, pl[0], pl[1], pl[2], count,
                            out + value_offset(kFP32, clo + sb_lo));
    if (bad) set_status(status, kStCorrupt);
  }
}

// Every chunk the staged BF16 path does not take (FP32, FP8, FP4; BF16 with a RAW or PACK
// exponent stream, a bitstream over 56 KB, or a ZRUN plane of more than 4096 blocks): one
// sub-block per thread per pass, every stream read through its own reader (BF16 with a
// coded exponent stream and a RAW or ZERO sign/fraction plane: the register decoder,
// which takes PACK pairs too). All threads.
template <int DT>
__device__ __forceinline__ void decode_generic(const uint8_t* __restrict__ in, const DecodeSmem<DT>& sm, uint32_t m,
                                               uint32_t S, uint64_t nsub, uint64_t clo, uint8_t* __restrict__ out,
                                               uint32_t* status) {
  constexpr int NS = n_streams(DT), NE = n_entropy(DT), VB = value_bytes(DT);
  constexpr int GV = DT == kBF16 ? 8 : DT == kFP32 ? 4 : 16;  // values per store (16 bytes; FP4 8)
  const int tid = threadIdx.x;
  for (uint64_t j = tid; j < nsub; j += kDecodeThreads) {
    const uint32_t sb_lo = (uint32_t)(j * S);
    const uint32_t count = min32(S, m - sb_lo);
    if constexpr (DT == kBF16) {
      if (coded(sm.mode[0]) && (sm.mode[1] == kModeRaw || sm.mode[1] == kModeZero)) {
        const uint32_t rec = sm.code[0] == kNoCode ? record_bytes(DT, 0) : 0;
        const uint32_t* idx = reinterpret_cast<const uint32_t*>(in + sm.off[0] + rec);
        const uint64_t bs_off = sm.off[0] + rec + round16(4 * nsub);
        const uint64_t cap_bits = (sm.end[0] - bs_off) * 8;
        const uint64_t start = __ldg(idx + j);
        const bool exact = j + 1 < nsub;
        const uint64_t expect = exact ? __ldg(idx + j + 1) : cap_bits;
        int bad = (j == 0 && start != 0) || start > cap_bits || expect < start || expect > cap_bits;
        const uint32_t* bs = reinterpret_cast<const uint32_t*>(in + bs_off);
        uint8_t* dst = out + (clo + sb_lo) * VB;
        const uint8_t* smp = sm.mode[1] == kModeZero ? nullptr : in + sm.off[1] + sb_lo;
        const uint32_t bw = (uint32_t)(cap_bits / 32);
        const uint64_t from = bad ? 0 : start;
        if (sm.mode[0] == kModePack) {
          const uint32_t valid = ((1u << sm.K) - 1u) | (1u << kPackEsc);
          if (!smp) bad |= decode_bf16_fast<true, true>(sm.lut[0], smp, bs, bw, from, expect, exact, count, dst,
                                                        sm.pack_exps, valid);
          else bad |= decode_bf16_fast<false, true>(sm.lut[0], smp, bs, bw, from, expect, exact, count, dst,
                                                    sm.pack_exps, valid);
        } else if (!smp) {
          bad |= decode_bf16_fast<true>(sm.lut[0], smp, bs, bw, from, expect, exact, count, dst);
        } else {
          bad |= decode_bf16_fast<false>(sm.lut[0], smp, bs, bw, from, expect, exact, count, dst);
        }
        if (bad) set_status(status, kStCorrupt);
        continue;
      }
    }
    StreamState st[NS];
    uint64_t expect_end[NS];
    bool check_exact[NS];
    int bad = 0;
#pragma unroll
    for (int s = 0; s < NS; s++) {
      const uint32_t mode = sm.mode[s];
      const int w = raw_width(DT, s);
      st[s].acc = 0;
      st[s].width = w;
      st[s].lut = nullptr;
      st[s].bytes = nullptr;
      st[s].zbad = 0;
      check_exact[s] = false;
      expect_end[s] = 0;
      if (mode == kModeZero) {
        st[s].kind = kKZero;
      } else if (mode == kModeZrun) {
        // zero runs (a byte plane): the bitmap, then the kept bytes; the marked blocks
        // before my first block give my first rank
        const uint64_t map_bytes = zrun_map_bytes(m);
        st[s].kind = kKZrun;
        st[s].zmap = in + sm.off[s];
        st[s].bytes = in + sm.off[s] + map_bytes;
        st[s].zlimit = sm.end[s] - sm.off[s] - map_bytes;
        st[s].zbase = sb_lo;
        st[s].zrank = zrun_rank(st[s].zmap, sb_lo / kZBlock);
        st[s].zmarked = 0;
      } else if (mode == kModeRaw) {
        if (w == 8) {
          st[s].kind = kKBytes;
          st[s].bytes = in + sm.off[s] + sb_lo;
        } else {
          st[s].kind = kKBits;
          st[s].br.init(reinterpret_cast<const uint32_t*>(in + sm.off[s]), (uint32_t)((sm.end[s] - sm.off[s]) / 4),
                        (uint64_t)sb_lo * w);
        }
      } else {
        const int e = s < NE ? s : 0;
        const uint32_t rec = sm.code[s] == kNoCode ? record_bytes(DT, s) : 0;
        const uint32_t* idx = reinterpret_cast<const uint32_t*>(in + sm.off[s] + rec);
        const uint64_t bs_off = sm.off[s] + rec + round16(4 * nsub);
        const uint64_t cap_bits = (sm.end[s] - bs_off) * 8;
        const uint64_t start = __ldg(idx + j);
        if (j == 0 && start != 0) bad = 1;
        if (start > cap_bits) bad = 1;
        if (j + 1 < nsub) {
          expect_end[s] = __ldg(idx + j + 1);
          check_exact[s] = true;
          if (expect_end[s] < start || expect_end[s] > cap_bits) bad = 1;
        } else {
          expect_end[s] = cap_bits;
        }
        st[s].kind = mode == kModePack ? kKPack : kKHuff;
        st[s].width = (int)sm.K;
        st[s].pexp = sm.pack_exps;
        st[s].lut = sm.lut[e];
        st[s].br.init(reinterpret_cast<const uint32_t*>(in + bs_off), (uint32_t)(cap_bits / 32), bad ? 0 : start);
      }
    }
    uint8_t* dst = out + value_offset(DT, clo + sb_lo);
    constexpr int SB = DT == kFP8 || DT == kFP4 ? 4 : 8;
    const uint32_t full = count / GV;
    for (uint32_t gi = 0; gi < full; gi++) {
      uint64_t P[NS];
#pragma unroll
      for (int s = 0; s < NS; s++) P[s] = next_packed<GV, SB, true>(st[s], GV, gi * GV);
      if constexpr (DT == kFP4) {
        // nibble i is value i (value 2i is the low nibble of byte i): sign << 3 |
        // exponent << 1 | mantissa, lane by lane
        const uint64_t v = (P[2] << 3) | (P[0] << 1) | P[1];
        *reinterpret_cast<uint2*>(dst + (uint64_t)gi * 8) = make_uint2((uint32_t)v, (uint32_t)(v >> 32));
      } else if constexpr (DT == kFP8) {
        // byte i: sign << 7 | exponent << 3 | mantissa
        uint32_t wv[4];
#pragma unroll
        for (int h = 0; h < 2; h++) {
          uint32_t e0, e1, m0, m1, s0, s1;
          nibbles_to_bytes((uint32_t)(P[0] >> (32 * h)), e0, e1);
          nibbles_to_bytes((uint32_t)(P[1] >> (32 * h)), m0, m1);
          nibbles_to_bytes((uint32_t)(P[2] >> (32 * h)), s0, s1);
          wv[2 * h] = (s0 << 7) | (e0 << 3) | m0;
          wv[2 * h + 1] = (s1 << 7) | (e1 << 3) | m1;
        }
        *reinterpret_cast<uint4*>(dst + (uint64_t)gi * 16) = make_uint4(wv[0], wv[1], wv[2], wv[3]);
      } else if constexpr (DT == kBF16) {
        uint32_t wv[4];
#pragma unroll
        for (int q = 0; q < 4; q++)
          wv[q] = bf16_merge_pair((uint32_t)(P[1] >> (32 * (q >> 1))), q & 1, (uint32_t)(P[0] >> (32 * (q >> 1))), q & 1);
        *reinterpret_cast<uint4*>(dst + (uint64_t)gi * 16) = make_uint4(wv[0], wv[1], wv[2], wv[3]);
      } else {
        uint32_t wv[4];
#pragma unroll
        for (int q = 0; q < 4; q++)
          wv[q] = merge_value<DT>((uint32_t)(P[0] >> (8 * q)) & 0xFFu, (uint32_t)(P[1] >> (8 * q)) & 0xFFu,
                                  (uint32_t)(P[NS > 2 ? 2 : 0] >> (8 * q)) & 0xFFu,
                                  (uint32_t)(P[NS > 3 ? 3 : 0] >> (8 * q)) & 0xFFu);
        *reinterpret_cast<uint4*>(dst + (uint64_t)gi * 16) = make_uint4(wv[0], wv[1], wv[2], wv[3]);
      }
    }
    const uint32_t rem = count - full * GV;
    if (rem) {
      uint64_t P[NS];
#pragma unroll
      for (int s = 0; s < NS; s++) P[s] = next_packed<GV, SB, false>(st[s], (int)rem, full * GV);
      constexpr uint32_t mask = (1u << SB) - 1u;
      if constexpr (DT == kFP4) {  // rem is even: values come in byte pairs
#pragma unroll
        for (uint32_t i = 0; i < (uint32_t)GV; i += 2) {
          if (i >= rem) break;
          const uint32_t lo = merge_value<DT>((uint32_t)(P[0] >> (SB * i)) & mask, (uint32_t)(P[1] >> (SB * i)) & mask,
                                              (uint32_t)(P[2] >> (SB * i)) & mask, 0);
          const uint32_t hi = merge_value<DT>((uint32_t)(P[0] >> (SB * (i + 1))) & mask,
                                              (uint32_t)(P[1] >> (SB * (i + 1))) & mask,
                                              (uint32_t)(P[2] >> (SB * (i + 1))) & mask, 0);
          dst[(full * GV + i) / 2] = (uint8_t)(lo | (hi << 4));
        }
      } else {
#pragma unroll
        for (uint32_t i = 0; i < (uint32_t)GV; i++) {
          if (i >= rem) break;
          const uint32_t v = merge_value<DT>((uint32_t)(P[0] >> (SB * i)) & mask, (uint32_t)(P[1] >> (SB * i)) & mask,
                                             NS > 2 ? (uint32_t)(P[NS > 2 ? 2 : 0] >> (SB * i)) & mask : 0u,
                                             NS > 3 ? (uint32_t)(P[NS > 3 ? 3 : 0] >> (SB * i)) & mask : 0u);
          uint8_t* p = dst + (uint64_t)(full * GV + i) * VB;
          if constexpr (VB == 2) *reinterpret_cast<uint16_t*>(p) = (uint16_t)v;
          else if constexpr (VB == 4) *reinterpret_cast<uint32_t*>(p) = v;
          else *p = (uint8_t)v;
        }
      }
    }
#pragma unroll
    for (int s = 0; s < NS; s++) {
      if (st[s].kind == kKZrun && st[s].zbad) bad = 1;
      if (st[s].kind != kKHuff && st[s].kind != kKPack) continue;
      const uint64_t pos = st[s].br.position();
      if (st[s].acc & kLutInvalid) bad = 1;
      if (check_exact[s] ? pos != expect_end[s] : pos > expect_end[s]) bad = 1;
    }
    if (bad) set_status(status, kStCorrupt);
  }
}

template <int DT>
__device__ __noinline__ void decode_generic_apart(const uint8_t* __restrict__ in, const DecodeSmem<DT>& sm, uint32_t m,
                                                  uint32_t S, uint64_t nsub, uint64_t clo, uint8_t* __restrict__ out,
                                                  uint32_t* status) {
  decode_generic<DT>(in, sm, m, S, nsub, clo, out, status);
}

// Chunk c of the container `in` (in_bytes readable) of a tensor with geometry g, into
// `out` (the tensor's first value). All threads of the block.
template <int DT>
__device__ __forceinline__ void decode_chunk(const uint8_t* __restrict__ in, uint64_t in_bytes, const Geo& g,
                                             uint32_t c, uint8_t* __restrict__ out, uint32_t* status) {
  constexpr int NS = n_streams(DT), NE = n_entropy(DT), VB = value_bytes(DT);
  __shared__ __align__(16) DecodeSmem<DT> sm;  // 16-byte aligned: a bulk copy may target its table
  extern __shared__ __align__(128) uint8_t dyn_smem[];  // StagedSmem for BF16 launches
  const int tid = threadIdx.x;
  const uint64_t clo = (uint64_t)c * g.m0;
  const uint32_t m = (uint32_t)min64(g.m0, g.n - clo);

  if (tid == 0) {
    int bad = 0;
    uint64_t total = 0, off_codes = 0, off_payload = 0;
    uint32_t S = 0, G = 0, K = 0;
    const uint64_t entries = (uint64_t)g.n_chunks * NS;
    const uint64_t k0 = (uint64_t)c * NS;
    if (in_bytes < kHeaderBytes + kEntryBytes * (k0 + NS)) {
      bad = 1;
    } else {
      // the header and this chunk's entries (and the next one's offset) in one round trip;
      // every address is inside in_bytes
      uint4 hq[4], ent[NS + 1];
#pragma unroll
      for (int i = 0; i < 4; i++) hq[i] = reinterpret_cast<const uint4*>(in)[i];
#pragma unroll
      for (int s = 0; s <= NS; s++) {
        const uint64_t k = k0 + s;
        ent[s] = (s < NS || (k < entries && kHeaderBytes + kEntryBytes * (k + 1) <= in_bytes))
                     ? *reinterpret_cast<const uint4*>(in + kHeaderBytes + kEntryBytes * k)
                     : make_uint4(0, 0, 0, 0);
      }
      const uint32_t hv[16] = {hq[0].x, hq[0].y, hq[0].z, hq[0].w, hq[1].x, hq[1].y, hq[1].z, hq[1].w,
                               hq[2].x, hq[2].y, hq[2].z, hq[2].w, hq[3].x, hq[3].y, hq[3].z, hq[3].w};
      const uint64_t n = hv[2] | ((uint64_t)hv[3] << 32);
      S = hv[5];
      G = (hv[14] >> 8) & 0xFF;
      off_codes = hv[8] | ((uint64_t)hv[9] << 32);
      off_payload = hv[10] | ((uint64_t)hv[11] << 32);
      total = hv[12] | ((uint64_t)hv[13] << 32);
      if (hv[0] != 0x314E4E5Au || hv[1] != (1u | ((uint32_t)DT << 16) | ((uint32_t)NS << 24))) bad = 1;
      if (n != g.n || hv[4] != g.chunk_bytes || hv[6] != g.n_chunks) bad = 1;
      if (S == 0 || (S & 15) || S > 65536) bad = 1;
      K = (hv[14] >> 16) & 0xFF;
      if ((hv[14] & 0xFF) != (uint32_t)kLmax || (hv[14] >> 24) != 0 || hv[15] != 0) bad = 1;
      if (K > kPackMax || (K && (DT != kBF16 || G == 0))) bad = 1;
      if (G > kMaxGroups || hv[7] != G * NE + (K ? G : 0u)) bad = 1;
      if (off_codes != kHeaderBytes + entries * kEntryBytes) bad = 1;
      if (!bad && off_payload != off_codes + code_section_bytes(DT, G, K)) bad = 1;
      if (total > in_bytes || total < off_payload || (total & 15)) bad = 1;
      if (!bad && K) {
        // the list of packed exponents: K entries, then zeros
        const uint4 q = *reinterpret_cast<const uint4*>(in + off_payload - kPackListBytes);
        const uint32_t qw[4] = {q.x, q.y, q.z, q.w};
#pragma unroll
        for (int i = 0; i < 16; i++) {
          const uint32_t b = (qw[i >> 2] >> (8 * (i & 3))) & 0xFFu;
          sm.pack_exps[i] = (uint8_t)b;
          if (i >= (int)K && b) bad = 1;
        }
      }
#pragma unroll
      for (int s = 0; s < NS; s++) {
        const uint64_t k = k0 + s;
        const uint64_t off = ent[s].z | ((uint64_t)ent[s].w << 32);
        const uint64_t end = k + 1 < entries ? (ent[s + 1].z | ((uint64_t)ent[s + 1].w << 32)) : total;
        const uint32_t mode = ent[s].x & 0xFF;
        if ((ent[s].x >> 8) != 0 || mode > kModePack) bad = 1;
        if ((off & 15) || (end & 15) || off > end || end > total || off < off_payload) bad = 1;
        if (k == 0 && off != off_payload) bad = 1;
        const uint64_t extent = end - off;
        const int w = raw_width(DT, s);
        if (mode == kModeRaw) {
          if (ent[s].y != kNoCode || extent * 8 < (uint64_t)m * w) bad = 1;
        } else if (mode == kModeZero) {
          if (ent[s].y != kNoCode) bad = 1;
        } else if (mode == kModeZrun) {
          if (!is_byte_plane(DT, s) || ent[s].y != kNoCode || extent < zrun_map_bytes(m)) bad = 1;
        } else if (mode == kModeHuff && S != 0) {
          const uint64_t nsub = ceil_div(m, S);
          uint64_t need = round16(4 * nsub);
          if (!is_entropy(DT, s)) bad = 1;
          else if (ent[s].y == kNoCode) need += record_bytes(DT, s);
          else if (G == 0 || ent[s].y >= G * NE || ent[s].y / G != (uint32_t)s) bad = 1;
          if (extent < need) bad = 1;
        } else if (mode == kModePack && S != 0) {
          // packed exponent pairs: a BF16 exponent stream of whole pairs, a packed record
          if (DT != kBF16 || s != 0 || K == 0 || (m & 1u)) bad = 1;
          else if (ent[s].y < G * NE || ent[s].y >= G * NE + G) bad = 1;
          if (extent < round16(4 * ceil_div(m, S))) bad = 1;
        }
        sm.mode[s] = mode;
        sm.code[s] = ent[s].y;
        sm.off[s] = off;
        sm.end[s] = end;
      }
    }
    sm.off_codes = off_codes;
    sm.S = S;
    sm.G = G;
    sm.K = K;
    sm.bad = bad;
    sm.staged = 0;
    if constexpr (DT == kBF16) {
      // staged path: HUFF exponents, RAW or ZERO sign/fraction bytes, bitstream in the
      // window (1), or in the window and the table's first half (2, the wide window)
      if (!bad && coded(sm.mode[0]) && sm.mode[1] != kModeHuff &&
          (sm.mode[1] != kModeZrun || ceil_div(ceil_div(m, kZBlock), 32) <= kZStagedWords)) {
        const uint64_t nsub = ceil_div(m, S);
        const uint32_t rec = sm.code[0] == kNoCode ? record_bytes(DT, 0) : 0;
        const uint64_t bs_off = sm.off[0] + rec + round16(4 * nsub);
        const uint64_t bs_bytes = sm.end[0] > bs_off ? sm.end[0] - bs_off : 0;
        if (bs_off <= sm.end[0] && bs_bytes <= kWideWindowBytes && nsub <= 0xFFFFFFFFull) {
          StagedSmem& stg = *reinterpret_cast<StagedSmem*>(dyn_smem);
          mbar_init(&stg.bar, 1);
          mbar_expect_tx(&stg.bar, (uint32_t)bs_bytes);
          for (uint64_t o = 0; o < bs_bytes; o += 16384) {  // 16 KB pieces; 48 KB is a piece boundary
            const uint32_t nb = (uint32_t)min64(16384, bs_bytes - o);
            uint8_t* dst = o < kWindowBytes ? reinterpret_cast<uint8_t*>(stg.bits) + o
                                            : reinterpret_cast<uint8_t*>(sm.lut[0]) + (o - kWindowBytes);
            bulk_g2s(dst, in + bs_off + o, nb, &stg.bar);
          }
          sm.staged = bs_bytes <= kWindowBytes ? 1 : 2;
        }
      }
    }
  }
  __syncthreads();
  if (sm.bad) {
    if (tid == 0) set_status(status, kStCorrupt);
    return;
  }
  const uint32_t S = sm.S;
  const uint64_t nsub = ceil_div(m, S);
  const int warp = tid >> 5, lane = tid & 31;

  // BF16 staged path: this thread's first sub-block bounds, requested now so that the
  // loads return while the tables are built
  uint32_t idx_start = 0, idx_next = 0;
  if constexpr (DT == kBF16) {
    if (sm.staged && (uint64_t)tid < nsub) {
      const uint32_t rec = sm.code[0] == kNoCode ? record_bytes(DT, 0) : 0;
      const uint32_t* idx = reinterpret_cast<const uint32_t*>(in + sm.off[0] + rec);
      idx_start = __ldg(idx + tid);
      if ((uint64_t)tid + 1 < nsub) idx_next = __ldg(idx + tid + 1);
    }
  }

  // BF16 staged path, ZRUN sign/fraction plane: thread w < 128 takes bitmap word w (the
  // payload's bytes are MSB first: reversing the bits of each byte gives bit i = block
  // 32w + i) and its in-warp prefix of marked blocks; the warps' totals join below.
  const bool zstaged = DT == kBF16 && sm.staged && sm.mode[1] == kModeZrun;
  if (zstaged && tid < (int)kZStagedWords) {
    const uint32_t used = (uint32_t)ceil_div(ceil_div(m, kZBlock), 32);
    const uint32_t raw = tid < (int)used ? __ldg(reinterpret_cast<const uint32_t*>(in + sm.off[1]) + tid) : 0u;
    const uint32_t word = __byte_perm(__brev(raw), 0, 0x0123);
    const uint32_t pc = __popc(word);
    uint32_t incl = pc;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const uint32_t y = __shfl_up_sync(0xFFFFFFFFu, incl, o);
      if (lane >= o) incl += y;
    }
    sm.zmap[tid] = word;
    sm.zpre[tid] = incl - pc;
    if (lane == 31) sm.ztot[warp] = incl;
  }

  // Canonical tables of each HUFF stream, from its 4-bit code lengths. Thread t takes
  // symbol t: each warp counts its 32 symbols of every length (ballots) and each symbol's
  // rank among the warp's symbols of its length (match), with the Kraft sum, a length
  // above 12, and whether any symbol is present.
  uint32_t my_len[NE], my_rank[NE];
#pragma unroll
  for (int e = 0; e < NE; e++) {
    my_len[e] = 0;
    my_rank[e] = 0;
    if (!coded(sm.mode[e])) continue;  // uniform
    const uint8_t* rp = sm.code[e] == kNoCode ? in + sm.off[e]
                        : sm.mode[e] == kModePack
                            ? in + sm.off_codes + packed_record_pos(DT, sm.G, sm.code[e] - sm.G * NE)
                            : in + sm.off_codes + shared_record_pos(DT, sm.G, sm.code[e]);
    uint32_t l = 0;
    if (tid < alphabet(DT, e)) {
      const uint32_t b = rp[tid >> 1];
      l = (tid & 1) ? (b >> 4) : (b & 15u);
    }
    const uint32_t same = __match_any_sync(0xFFFFFFFFu, l);
    my_len[e] = l;
    my_rank[e] = __popc(same & lanemask_lt());
    uint32_t c = 0;
#pragma unroll
    for (int q = 1; q <= kLmax; q++) {
      const uint32_t b = __popc(__ballot_sync(0xFFFFFFFFu, l == (uint32_t)q));
      if (lane == q) c = b;
    }
    if (lane < 16) sm.cnt[e][warp][lane] = (uint8_t)c;
    const uint32_t kw = __reduce_add_sync(0xFFFFFFFFu, (l && l <= (uint32_t)kLmax) ? 1u << (kLmax - l) : 0u);
    const uint32_t fl = (__any_sync(0xFFFFFFFFu, l > (uint32_t)kLmax) ? 1u : 0u) | (__any_sync(0xFFFFFFFFu, l != 0) ? 2u : 0u);
    if (lane == 0) {
      sm.kraft[e][warp] = kw;
      sm.flags[e][warp] = fl;
    }
  }
  __syncthreads();
  if (zstaged && tid < (int)kZStagedWords) {
    uint32_t before = 0;
    for (int w = 0; w < (tid >> 5); w++) before += sm.ztot[w];
    sm.zpre[tid] += before;
    if (tid == 0) {
      // the kept bytes must lie inside the payload: 32 per marked block, less what a marked
      // short last block lacks, padded to 16
      const uint32_t total = sm.ztot[0] + sm.ztot[1] + sm.ztot[2] + sm.ztot[3];
      const uint64_t last = (m - 1) / kZBlock;
      uint64_t kept = (uint64_t)total * kZBlock;
      if ((m % kZBlock) && ((sm.zmap[last >> 5] >> (last & 31)) & 1u)) kept -= kZBlock - m % kZBlock;
      if (sm.end[1] - sm.off[1] < zrun_payload(m, kept)) sm.bad = 1;
    }
  }
  // warp e: lengths' counts, first codes (RFC 1951, 3.2.2: first[l] = (first[l-1] +
  // count[l-1]) << 1, i.e. the sum over q < l of count[q] << (l - q)), canonical index
  // offsets, left-aligned limits, and every warp's base index for each length; lane l
  // takes length l. A length above 12, no symbol, or a Kraft sum above 1 is corrupt.
  if (warp < NE && coded(sm.mode[warp])) {
    const int e = warp;
    uint32_t kraft = 0, fl = 0;
#pragma unroll
    for (int w = 0; w < 8; w++) {
      kraft += sm.kraft[e][w];
      fl |= sm.flags[e][w];
    }
    const bool in_range = lane >= 1 && lane <= kLmax;
    uint32_t count = 0;
    if (in_range)
#pragma unroll
      for (int w = 0; w < 8; w++) count += sm.cnt[e][w][lane];
    uint32_t incl = count;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const uint32_t y = __shfl_up_sync(0xFFFFFFFFu, incl, o);
      if (lane >= o) incl += y;
    }
    const uint32_t offs = incl - count;
    uint32_t fst = 0;
#pragma unroll
    for (int q = 1; q < kLmax; q++) {
      const uint32_t cq = __shfl_sync(0xFFFFFFFFu, count, q);
      if (q < lane) fst += cq << (lane - q);
    }
    if (lane <= kLmax) {
      sm.first[e][lane] = fst;
      sm.offset[e][lane] = offs;
      sm.limit[e][lane] = in_range ? (fst + count) << (kLmax - lane) : 0u;
    }
    if (in_range) {
      uint32_t run = offs;
#pragma unroll
      for (int w = 0; w < 8; w++) {
        sm.base[e][w][lane] = (uint16_t)run;
        run += sm.cnt[e][w][lane];
      }
    }
    if ((fl & 1u) || !(fl & 2u) || kraft > (1u << kLmax)) {
      if (lane == 0) sm.bad = 1;
    }
  }
  __syncthreads();
  if (sm.bad) {
    if (tid == 0) set_status(status, kStCorrupt);
    if constexpr (DT == kBF16) {
      // a bitstream copy may be in flight into this block's shared memory: let it land
      // (bounded) before the block exits
      if (sm.staged) {
        StagedSmem& stg = *reinterpret_cast<StagedSmem*>(dyn_smem);
        for (uint32_t k = 0; k < kWaitLimit && !mbar_try_wait(&stg.bar, 0); k++) __nanosleep(256);
      }
    }
    return;
  }
  // symbols in canonical order
#pragma unroll
  for (int e = 0; e < NE; e++) {
    if (!coded(sm.mode[e]) || !my_len[e]) continue;
    const uint32_t k = sm.base[e][warp][my_len[e]] + my_rank[e];
    sm.sorted[e][k] = (uint8_t)tid;
    sm.slen[e][k] = (uint8_t)my_len[e];
  }
  __syncthreads();
  // BF16 with the wide window: the 11-bit table in the table's second half (the bulk copy
  // may still be writing the first half)
  const bool wide = DT == kBF16 && sm.staged == 2;
  uint32_t* const lut11 = sm.lut[0] + (kWideWords - kWindowWords);
#pragma unroll
  for (int e = 0; e < NE; e++) {
    if (!coded(sm.mode[e])) continue;
    if (wide) fill_lut11(lut11, sm.sorted[e], sm.limit[e], sm.first[e], sm.offset[e]);
    else fill_lut(sm.lut[e], sm.sorted[e], sm.slen[e], sm.limit[e], sm.first[e], sm.offset[e]);
  }
  __syncthreads();
  const bool pack = DT == kBF16 && sm.mode[0] == kModePack;
  if (pack) {
    // a PACK stream: each entry's pair symbol becomes its two exponents (the list's entries
    // for its nibbles) and escape flags; a nibble past the list makes the entry invalid
    uint32_t* const t = wide ? lut11 : sm.lut[0];
    const uint32_t ne = wide ? 2048u : 4096u;
    for (uint32_t x = tid; x < ne; x += kDecodeThreads) {
      const uint32_t e = t[x];
      if (e & (kLutInvalid | kLong11)) continue;
      const uint32_t sym = lut_symbol(e), hi = sym >> 4, lo = sym & 15u;
      const bool bad = (hi != kPackEsc && hi >= sm.K) || (lo != kPackEsc && lo >= sm.K);
      const uint32_t a = hi == kPackEsc ? 0u : sm.pack_exps[hi], b = lo == kPackEsc ? 0u : sm.pack_exps[lo];
      t[x] = (e & 15u) | (hi == kPackEsc ? kPackEscHi : 0u) | (lo == kPackEsc ? kPackEscLo : 0u) |
             (bad ? kLutInvalid : 0u) | (a << 16) | (b << 24);
    }
    __syncthreads();
  }
  if (wide && !pack) {
    // the 11-bit table's second codes, as for the 12-bit table below (in place: the first
    // code's fields of an entry never change)
    for (uint32_t x = tid; x < 2048; x += kDecodeThreads) {
      const uint32_t e0 = lut11[x];
      if (e0 & (kLutInvalid | kLong11)) continue;
      const uint32_t l0 = e0 & 15u;
      if (l0 >= 11) continue;
      const uint32_t e1 = lut11[(x << l0) & 2047u];
      const uint32_t l1 = e1 & 15u;
      if (!(e1 & (kLutInvalid | kLong11)) && l0 + l1 <= 11)
        lut11[x] = e0 | ((l0 + l1) << 4) | ((e1 & 0x00FF0000u) << 8);
    }
    __syncthreads();
  }
  // second code of each window: the entry of the window shifted by the first length
  // decides it when that code ends inside the 12 known bits (a prefix code's entry does
  // not depend on the bits after the code). Updating in place is safe: the fields read
  // here (first length, first symbol, invalid flag) never change. Every 12-bit table (the
  // wide window's 11-bit table had its own pass above).
  if (!wide) {
    bool any = false;
    // FP4 exponents whose codes have at most 3 bits (every Huffman code of 4 symbols): any
    // 12-bit window holds 4 whole codes, so entry x also gets their total length (bits
    // 4..7) and the 4 symbols (2 bits each, the first lowest, bits 24..31), read from the
    // entries of the window shifted past each code; a window that is not 4 valid codes
    // gets kQuadInvalid (bit 14, which no other entry's computation reads)
    const bool quad = DT == kFP4 && sm.mode[0] == kModeHuff && sm.limit[0][3] == sm.limit[0][kLmax] &&
                      sub_fast_ok(sm, sm.S);  // only the fast path reads four-symbol entries
    if (tid == 0) sm.quad = quad;
#pragma unroll
    for (int e = 0; e < NE; e++) {
      if (sm.mode[e] != kModeHuff) continue;  // PACK entries hold exponents, not second codes
      any = true;
      if (e == 0 && quad) {
        for (uint32_t x = tid; x < 4096; x += kDecodeThreads) {
          uint32_t total = 0, syms = 0, inval = 0;
#pragma unroll
          for (int k = 0; k < 4; k++) {
            const uint32_t ek = sm.lut[0][(x << total) & 4095u];
            inval |= ek & kLutInvalid;
            syms |= ((ek >> 16) & 3u) << (2 * k);
            total += ek & 15u;
          }
          const uint32_t e0 = sm.lut[0][x];
          sm.lut[0][x] = (e0 & 0x00FF800Fu) | (total << 4) | (syms << 24) | (inval || total > (uint32_t)kLmax ? kQuadInvalid : 0u);
        }
        continue;
      }
      for (uint32_t x = tid; x < 4096; x += kDecodeThreads) {
        const uint32_t e0 = sm.lut[e][x];
        if (e0 & kLutInvalid) continue;
        const uint32_t l0 = e0 & 15u;
        const uint32_t e1 = sm.lut[e][(x << l0) & 4095u];
        const uint32_t l1 = e1 & 15u;
        if (!(e1 & kLutInvalid) && l0 + l1 <= (uint32_t)kLmax)
          sm.lut[e][x] = e0 | ((l0 + l1) << 4) | ((e1 & 0x00FF0000u) << 8);
      }
    }
    if (any) __syncthreads();
  }

  if constexpr (DT == kBF16) {
    if (sm.staged) {
      StagedSmem& stg = *reinterpret_cast<StagedSmem*>(dyn_smem);
      uint32_t spins = 0;
      while (!mbar_try_wait(&stg.bar, 0)) {
        if (++spins > kWaitLimit) {  // the copy never landed: report, keep waiting for it (bounded again)
          if (tid == 0) set_status(status, kStTimeout);
          for (uint32_t k = 0; k < kWaitLimit && !mbar_try_wait(&stg.bar, 0); k++) __nanosleep(1024);
          return;
        }
        __nanosleep(32);
      }
      const uint32_t rec = sm.code[0] == kNoCode ? record_bytes(DT, 0) : 0;
      const uint32_t* idx = reinterpret_cast<const uint32_t*>(in + sm.off[0] + rec);
      const uint64_t bs_off = sm.off[0] + rec + round16(4 * nsub);
      const uint32_t bs_words = (uint32_t)((sm.end[0] - bs_off) / 4);
      const uint8_t* smp = sm.mode[1] == kModeRaw    ? in + sm.off[1]
                           : sm.mode[1] == kModeZrun ? in + sm.off[1] + zrun_map_bytes(m)
                                                     : nullptr;
      const bool allfull = (uint64_t)m == nsub * S && S % kRound == 0 && nsub % kDecodeThreads == 0;
      int bad;
#define ZIPNN_STAGED(W, Z, F, P, L, T, ZM, ZP)                                                                \
  decode_bf16_staged<W, Z, F, P>(stg, L, T, idx, bs_words, smp, m, S, (uint32_t)nsub, out + clo * VB, idx_start, \
                                 idx_next, ZM, ZP, sm.pack_exps, valid, lg)
      const Long12 lg{sm.sorted[0], sm.first[0][kLmax], sm.offset[0][kLmax], sm.limit[0][kLmax]};
      const uint32_t valid = ((1u << sm.K) - 1u) | (1u << kPackEsc);
      if (sm.mode[0] == kModePack) {
        if (sm.mode[1] == kModeZrun) {
          if (wide) bad = allfull ? ZIPNN_STAGED(true, true, true, true, lut11, sm.lut[0], sm.zmap, sm.zpre)
                                  : ZIPNN_STAGED(true, true, false, true, lut11, sm.lut[0], sm.zmap, sm.zpre);
          else bad = allfull ? ZIPNN_STAGED(false, true, true, true, sm.lut[0], nullptr, sm.zmap, sm.zpre)
                             : ZIPNN_STAGED(false, true, false, true, sm.lut[0], nullptr, sm.zmap, sm.zpre);
        } else {
          if (wide) bad = allfull ? ZIPNN_STAGED(true, false, true, true, lut11, sm.lut[0], nullptr, nullptr)
                                  : ZIPNN_STAGED(true, false, false, true, lut11, sm.lut[0], nullptr, nullptr);
          else bad = allfull ? ZIPNN_STAGED(false, false, true, true, sm.lut[0], nullptr, nullptr, nullptr)
                             : ZIPNN_STAGED(false, false, false, true, sm.lut[0], nullptr, nullptr, nullptr);
        }
      } else if (sm.mode[1] == kModeZrun) {
        if (wide) bad = allfull ? ZIPNN_STAGED(true, true, true, false, lut11, sm.lut[0], sm.zmap, sm.zpre)
                                : ZIPNN_STAGED(true, true, false, false, lut11, sm.lut[0], sm.zmap, sm.zpre);
        else bad = allfull ? ZIPNN_STAGED(false, true, true, false, sm.lut[0], nullptr, sm.zmap, sm.zpre)
                           : ZIPNN_STAGED(false, true, false, false, sm.lut[0], nullptr, sm.zmap, sm.zpre);
      } else {
        if (wide) bad = allfull ? ZIPNN_STAGED(true, false, true, false, lut11, sm.lut[0], nullptr, nullptr)
                                : ZIPNN_STAGED(true, false, false, false, lut11, sm.lut[0], nullptr, nullptr);
        else bad = allfull ? ZIPNN_STAGED(false, false, true, false, sm.lut[0], nullptr, nullptr, nullptr)
                           : ZIPNN_STAGED(false, false, false, false, sm.lut[0], nullptr, nullptr, nullptr);
      }
#undef ZIPNN_STAGED
      if (bad) set_status(status, kStCorrupt);
      return;
    }
  }
  // FP8, FP4 and FP32 chunks of the common stream modes take their fast paths; the other
  // cases (a rare fallback) go one sub-block per thread per pass through every stream's
  // own reader, in a function of its own so that its register needs do not weigh on the
  // main paths
  if constexpr (DT == kFP8 || DT == kFP4) {
    if (sub_fast_ok(sm, S)) decode_sub_chunk<DT>(in, sm, m, S, nsub, clo, out, status);
    else decode_generic_apart<DT>(in, sm, m, S, nsub, clo, out, status);
  } else if constexpr (DT == kFP32) {
    if (fp32_fast_ok(sm)) decode_fp32_chunk(in, sm, m, S, nsub, clo, out, status);
    else decode_generic_apart<DT>(in, sm, m, S, nsub, clo, out, status);
  } else {
    decode_generic_apart<DT>(in, sm, m, S, nsub, clo, out, status);
  }
}

// Blocks per SM the decode kernels are built for: three (24 warps).
constexpr int decode_blocks_per_sm(int) { return 3; }

template <int DT>
__global__ void __launch_bounds__(kDecodeThreads, decode_blocks_per_sm(DT))
    k_decode(const uint8_t* __restrict__ in, uint64_t in_bytes, Geo g, uint8_t* __restrict__ out, uint32_t* status) {
  decode_chunk<DT>(in, in_bytes, g, blockIdx.x, out, status);
}

// The item whose chunks include global chunk b: the last i with items[i].chunk0 <= b
// (items[0].chunk0 == 0, increasing). One warp, a 32-way search: each round probes 32
// evenly spaced items and keeps the span after the last probe at or below b.
__device__ __forceinline__ uint32_t find_item(const DecodeItem* __restrict__ items, uint32_t count, uint64_t b) {
  const uint32_t lane = threadIdx.x & 31;
  uint32_t lo = 0, hi = count;  // the answer is in [lo, hi)
  while (hi - lo > 1) {
    const uint32_t step = (hi - lo + 31) / 32;
    const uint32_t p = lo + lane * step;
    const bool le = p < hi && items[p].chunk0 <= b;
    const uint32_t mask = __ballot_sync(0xFFFFFFFFu, le);  // bit 0 is set: items[lo].chunk0 <= b
    lo += (uint32_t)(31 - __clz(mask)) * step;
    hi = min32(lo + step, hi);
  }
  return lo;
}

// Many tensors in one launch: block b decodes global chunk b.
template <int DT>
__global__ void __launch_bounds__(kDecodeThreads, decode_blocks_per_sm(DT))
    k_decode_batch(const DecodeItem* __restrict__ items, uint32_t count, Geo g, uint32_t* status) {
  __shared__ uint32_t s_item;
  if (threadIdx.x < 32) {
    const uint32_t it = find_item(items, count, blockIdx.x);
    if (threadIdx.x == 0) s_item = it;
  }
  __syncthreads();
  const DecodeItem d = items[s_item];
  g.n = d.n;
  g.n_chunks = (uint32_t)ceil_div(d.n, g.m0);
  decode_chunk<DT>(d.in, d.in_bytes, g, (uint32_t)(blockIdx.x - d.chunk0), d.out, status);
}

// Dynamic shared memory (the BF16 staging window) once per device and kernel.
template <class K>
static cudaError_t decode_attributes(K kernel, size_t dyn, std::atomic<int>* done) {
  if (!dyn) return cudaSuccess;
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  if (dev >= 0 && dev < 128 && done[dev].load(std::memory_order_relaxed)) return cudaSuccess;
  e = cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)dyn);
  if (e == cudaSuccess) e = cudaFuncSetAttribute(kernel, cudaFuncAttributePreferredSharedMemoryCarveout, 100);
  if (e == cudaSuccess && dev >= 0 && dev < 128) done[dev].store(1, std::memory_order_relaxed);
  return e;
}

template <int DT>
static cudaError_t decode_t(const uint8_t* in, uint64_t in_bytes, const Geo& g, uint8_t* out, uint32_t* status,
                            cudaStream_t st) {
  const size_t dyn = DT == kBF16 ? sizeof(StagedSmem) : 0;
  static std::atomic<int> done[128];
  cudaError_t e = decode_attributes(k_decode<DT>, dyn, done);
  if (e != cudaSuccess) return e;
  k_decode<DT><<<g.n_chunks, kDecodeThreads, dyn, st>>>(in, in_bytes, g, out, status);
  return cudaGetLastError();
}

template <int DT>
static cudaError_t decode_batch_t(const DecodeItem* items, uint32_t count, const Geo& g, uint32_t total_chunks,
                                  uint32_t* status, cudaStream_t st) {
  const size_t dyn = DT == kBF16 ? sizeof(StagedSmem) : 0;
  static std::atomic<int> done[128];
  cudaError_t e = decode_attributes(k_decode_batch<DT>, dyn, done);
  if (e != cudaSuccess) return e;
  k_decode_batch<DT><<<total_chunks, kDecodeThreads, dyn, st>>>(items, count, g, status);
  return cudaGetLastError();
}

cudaError_t launch_decode(const uint8_t* in, uint64_t in_bytes, const Geo& g, uint8_t* out, uint32_t* status,
                          cudaStream_t st) {
  switch (g.dt) {
    case kBF16: return decode_t<kBF16>(in, in_bytes, g, out, status, st);
    case kFP32: return decode_t<kFP32>(in, in_bytes, g, out, status, st);
    case kFP8: return decode_t<kFP8>(in, in_bytes, g, out, status, st);
    default: return decode_t<kFP4>(in, in_bytes, g, out, status, st);
  }
}

cudaError_t launch_decode_batch(const DecodeItem* items, uint32_t count, const Geo& g, uint32_t total_chunks,
                                uint32_t* status, cudaStream_t st) {
  switch (g.dt) {
    case kBF16: return decode_batch_t<kBF16>(items, count, g, total_chunks, status, st);
    case kFP32: return decode_batch_t<kFP32>(items, count, g, total_chunks, status, st);
    case kFP8: return decode_batch_t<kFP8>(items, count, g, total_chunks, status, st);
    default: return decode_batch_t<kFP4>(items, count, g, total_chunks, status, st);
  }
}

}  // namespace zipnn

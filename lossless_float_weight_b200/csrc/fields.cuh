// fields.cuh -- the byte-plane split of BF16 / FP32 / FP8 (E4M3) / FP4 (E2M1) values and
// its inverse.
//
// Split ("ZipNN: Lossless Compression for AI Models", abstract; THEORY-599 note,
// "Per-field compressibility (Table II)"): the exponent field is one stream, the sign
// and fraction bytes are the others. FP8 keeps exponent and mantissa as separate
// entropy streams ("Lossless Compression of Neural Network Components ... in
// Low-Precision Formats", abstract) and the sign as a 1-bit stream; so does FP4, whose
// values come two to a byte (value 2i in the low nibble of byte i).
//   BF16 w : s0 = bits 14..7, s1 = sign(bit 15) << 7 | bits 6..0
//   FP32 u : s0 = bits 30..23, s1 = sign << 7 | bits 22..16, s2 = bits 15..8, s3 = bits 7..0
//   FP8  b : s0 = bits 6..3, s1 = bits 2..0, s2 = bit 7
//   FP4  v : s0 = bits 2..1, s1 = bit 0, s2 = bit 3 (of the nibble)
#pragma once
#include "common.cuh"

namespace zipnn {

// The raw 32-bit words of NV consecutive values held by one thread.
template <int DT, int NV>
struct RawValues {
  static constexpr int kWords = NV * value_bits(DT) / 32;
  uint32_t w[kWords];
};

// Load NV consecutive values (16-byte aligned); values at or beyond cnt read as 0 and
// are never fetched.
template <int DT, int NV>
__device__ __forceinline__ void load_values(const uint8_t* __restrict__ p, int cnt, RawValues<DT, NV>& r) {
  constexpr int W = RawValues<DT, NV>::kWords;
  if (cnt >= NV) {
#pragma unroll
    for (int j = 0; j < W / 4; j++) {
      const uint4 a = __ldg(reinterpret_cast<const uint4*>(p) + j);
      r.w[4 * j] = a.x;
      r.w[4 * j + 1] = a.y;
      r.w[4 * j + 2] = a.z;
      r.w[4 * j + 3] = a.w;
    }
  } else {
#pragma unroll
    for (int j = 0; j < W; j++) {
      uint32_t x = 0;
#pragma unroll
      for (int b = 0; b < 4; b++) {
        // the first value held by byte 4j + b
        const int v = DT == kFP4 ? 2 * (4 * j + b) : (4 * j + b) / value_bytes(DT);
        if (v < cnt) x |= (uint32_t)p[4 * j + b] << (8 * b);
      }
      r.w[j] = x;
    }
  }
}

// Symbol of stream s for value i (the split above).
template <int DT, int NV>
__device__ __forceinline__ uint32_t symbol(const RawValues<DT, NV>& r, int s, int i) {
  if constexpr (DT == kBF16) {
    const uint32_t v = (r.w[i >> 1] >> (16 * (i & 1))) & 0xFFFFu;
    return s == 0 ? (v >> 7) & 0xFFu : ((v >> 8) & 0x80u) | (v & 0x7Fu);
  } else if constexpr (DT == kFP32) {
    const uint32_t u = r.w[i];
    return s == 0 ? (u >> 23) & 0xFFu
                  : s == 1 ? ((u >> 24) & 0x80u) | ((u >> 16) & 0x7Fu) : s == 2 ? (u >> 8) & 0xFFu : u & 0xFFu;
  } else if constexpr (DT == kFP4) {
    const uint32_t v = (r.w[i >> 3] >> (4 * (i & 7))) & 0xFu;
    return s == 0 ? (v >> 1) & 3u : s == 1 ? v & 1u : v >> 3;
  } else {
    const uint32_t b = (r.w[i >> 2] >> (8 * (i & 3))) & 0xFFu;
    return s == 0 ? (b >> 3) & 0xFu : s == 1 ? b & 7u : b >> 7;
  }
}

// Merge: the inverse of the split for one value.
template <int DT>
__device__ __forceinline__ uint32_t merge_value(uint32_t s0, uint32_t s1, uint32_t s2, uint32_t s3) {
  if constexpr (DT == kBF16) {
    return ((s1 & 0x80u) << 8) | (s0 << 7) | (s1 & 0x7Fu);
  } else if constexpr (DT == kFP32) {
    return ((s1 & 0x80u) << 24) | (s0 << 23) | ((s1 & 0x7Fu) << 16) | (s2 << 8) | s3;
  } else if constexpr (DT == kFP4) {
    return (s2 << 3) | (s0 << 1) | s1;
  } else {
    return (s2 << 7) | (s0 << 3) | s1;
  }
}

}  // namespace zipnn

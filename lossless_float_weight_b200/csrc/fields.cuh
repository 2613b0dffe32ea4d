// fields.cuh -- the byte-plane split of BF16 / FP32 / FP8 (E4M3) values and its inverse.
//
// Split ("ZipNN: Lossless Compression for AI Models", abstract; THEORY-599 note,
// "Per-field compressibility (Table II)"): the exponent field is one stream, the sign
// and fraction bytes are the others. FP8 keeps exponent and mantissa as separate
// entropy streams ("Lossless Compression of Neural Network Components ... in
// Low-Precision Formats", abstract) and the sign as a 1-bit stream.
//   BF16 w : s0 = bits 14..7, s1 = sign(bit 15) << 7 | bits 6..0
//   FP32 u : s0 = bits 30..23, s1 = sign << 7 | bits 22..16, s2 = bits 15..8, s3 = bits 7..0
//   FP8  b : s0 = bits 6..3, s1 = bits 2..0, s2 = bit 7
#pragma once
#include "common.cuh"

namespace zipnn {

// Load the 16 values of one group (16 * value_bytes bytes at p, 16-byte aligned) and
// split them: sym[s][i] for stream s, value i. Values at or beyond `cnt` read as 0 and
// are never fetched, so a ragged tail does not read past the tensor.
template <int DT>
__device__ __forceinline__ void load_split16(const uint8_t* __restrict__ p, int cnt, uint32_t (&sym)[n_streams(DT)][16]) {
  if constexpr (DT == kBF16) {
    uint32_t w[8];
    if (cnt >= 16) {
      uint4 a = __ldg(reinterpret_cast<const uint4*>(p));
      uint4 b = __ldg(reinterpret_cast<const uint4*>(p) + 1);
      w[0] = a.x; w[1] = a.y; w[2] = a.z; w[3] = a.w; w[4] = b.x; w[5] = b.y; w[6] = b.z; w[7] = b.w;
    } else {
      const uint16_t* q = reinterpret_cast<const uint16_t*>(p);
#pragma unroll
      for (int j = 0; j < 8; j++) {
        uint32_t lo = 2 * j < cnt ? q[2 * j] : 0u;
        uint32_t hi = 2 * j + 1 < cnt ? q[2 * j + 1] : 0u;
        w[j] = lo | (hi << 16);
      }
    }
#pragma unroll
    for (int i = 0; i < 16; i++) {
      uint32_t v = (w[i >> 1] >> (16 * (i & 1))) & 0xFFFFu;
      sym[0][i] = (v >> 7) & 0xFFu;
      sym[1][i] = ((v >> 8) & 0x80u) | (v & 0x7Fu);
    }
  } else if constexpr (DT == kFP32) {
    uint32_t w[16];
    if (cnt >= 16) {
#pragma unroll
      for (int j = 0; j < 4; j++) {
        uint4 a = __ldg(reinterpret_cast<const uint4*>(p) + j);
        w[4 * j] = a.x; w[4 * j + 1] = a.y; w[4 * j + 2] = a.z; w[4 * j + 3] = a.w;
      }
    } else {
      const uint32_t* q = reinterpret_cast<const uint32_t*>(p);
#pragma unroll
      for (int j = 0; j < 16; j++) w[j] = j < cnt ? q[j] : 0u;
    }
#pragma unroll
    for (int i = 0; i < 16; i++) {
      uint32_t u = w[i];
      sym[0][i] = (u >> 23) & 0xFFu;
      sym[1][i] = ((u >> 24) & 0x80u) | ((u >> 16) & 0x7Fu);
      sym[2][i] = (u >> 8) & 0xFFu;
      sym[3][i] = u & 0xFFu;
    }
  } else {
    uint32_t w[4];
    if (cnt >= 16) {
      uint4 a = __ldg(reinterpret_cast<const uint4*>(p));
      w[0] = a.x; w[1] = a.y; w[2] = a.z; w[3] = a.w;
    } else {
#pragma unroll
      for (int j = 0; j < 4; j++) {
        uint32_t x = 0;
#pragma unroll
        for (int b = 0; b < 4; b++)
          if (4 * j + b < cnt) x |= (uint32_t)p[4 * j + b] << (8 * b);
        w[j] = x;
      }
    }
#pragma unroll
    for (int i = 0; i < 16; i++) {
      uint32_t b = (w[i >> 2] >> (8 * (i & 3))) & 0xFFu;
      sym[0][i] = (b >> 3) & 0xFu;
      sym[1][i] = b & 7u;
      sym[2][i] = b >> 7;
    }
  }
}

// The raw 32-bit words of NV consecutive values held by one thread.
template <int DT, int NV>
struct RawValues {
  static constexpr int kWords = NV * value_bytes(DT) / 4;
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
    constexpr int VB = value_bytes(DT);
#pragma unroll
    for (int j = 0; j < W; j++) {
      uint32_t x = 0;
#pragma unroll
      for (int b = 0; b < 4; b++)
        if ((4 * j + b) / VB < cnt) x |= (uint32_t)p[4 * j + b] << (8 * b);
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
  } else {
    return (s2 << 7) | (s0 << 3) | s1;
  }
}

}  // namespace zipnn

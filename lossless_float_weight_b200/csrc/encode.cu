// encode.cu -- k_encode: writes every payload byte of the container.
//
// One block per tile of 4096 values of one chunk; 256 threads own 16 values each.
//  * RAW byte planes (8-bit streams: BF16/FP32 sign+fraction bytes, an exponent that
//    did not compress): the thread's 16 bytes go out as one 16-byte store.
//  * bit streams (HUFF streams; FP8's 4-, 3- and 1-bit RAW streams): each thread sums
//    the code lengths of its 16 symbols; a block-wide warp-shuffle scan gives its bit
//    offset inside the tile; the tile's offset inside the chunk comes from the previous
//    tiles of the same chunk by single-pass decoupled look-back (fixed for RAW
//    streams). Codes are emitted most significant bit first into a shared staging
//    buffer, whole words with plain stores and the two edge words of each thread with
//    shared atomicOr; the block then stores the staged words. A word that straddles two
//    tiles is merged in a workspace slot: each side adds (1 << 32 | its bits) and the
//    side that arrives second stores the complete word, so no output pre-clearing and
//    no wait between blocks is needed for it.
//  * the sub-block index idx[j] (bit offset of symbol j*S) is written by the thread
//    that owns symbol j*S; the first tile writes a local code record, the last tile the
//    zero padding.
#include "common.cuh"
#include "fields.cuh"
#include "launch.h"

namespace zipnn {

constexpr int kStageWords = kTileValues * kLmax / 32 + 2;

// Pack this thread's codes, starting q bits into the staging buffer.
__device__ __forceinline__ void stage_bits(uint32_t* stage, uint32_t q, const uint32_t (&code)[16],
                                           const uint32_t (&len)[16]) {
  uint32_t wi = q >> 5;
  uint32_t fill = q & 31;
  const bool shared_head = fill != 0;
  bool first = true;
  uint64_t acc = 0;
#pragma unroll
  for (int i = 0; i < 16; i++) {
    if (len[i]) {
      acc |= (uint64_t)code[i] << (64 - fill - len[i]);
      fill += len[i];
      if (fill >= 32) {
        const uint32_t word = (uint32_t)(acc >> 32);
        if (first && shared_head) atomicOr(stage + wi, word);
        else stage[wi] = word;
        first = false;
        wi++;
        acc <<= 32;
        fill -= 32;
      }
    }
  }
  if (fill > 0) atomicOr(stage + wi, (uint32_t)(acc >> 32));
}

// Merge a word shared by two tiles: the second arrival stores the union.
__device__ __forceinline__ void slot_merge(uint64_t* slot, uint32_t part, uint32_t* dst) {
  const uint64_t old = atomicAdd(reinterpret_cast<unsigned long long*>(slot), (1ull << 32) | (uint64_t)part);
  if ((old >> 32) == 1) *dst = bswap32((uint32_t)old | part);
}

template <int DT>
__global__ void __launch_bounds__(kEncodeThreads) k_encode(const uint8_t* __restrict__ src, Geo g, Ws ws,
                                                           uint8_t* __restrict__ out) {
  constexpr int NS = n_streams(DT), NE = n_entropy(DT), VB = value_bytes(DT);
  constexpr int NB = DT == kFP8 ? 3 : 1;  // streams that may be bit-packed
  __shared__ uint32_t s_enc[NE][256];
  __shared__ uint32_t s_stage[kStageWords];
  __shared__ uint32_t s_warp[kEncodeThreads / 32];
  __shared__ uint32_t s_tile;
  __shared__ uint64_t s_prefix;
  __shared__ uint32_t s_mode[NS], s_code[NS];
  __shared__ uint64_t s_off[NS];
  const int tid = threadIdx.x;
  if (tid == 0) s_tile = atomicAdd(&ws.status[1], 1u);
  __syncthreads();
  const uint32_t tile = s_tile;
  const uint32_t c = tile / g.tiles_per_chunk, ti = tile % g.tiles_per_chunk;
  const uint64_t clo = (uint64_t)c * g.m0;
  const uint32_t m = (uint32_t)min64(g.m0, g.n - clo);
  const uint32_t tlo = ti * (uint32_t)kTileValues;
  if (tlo >= m) return;  // past the end of a ragged last chunk
  const bool last = tlo + (uint32_t)kTileValues >= m;
  if (tid < NS) {
    const uint64_t k = (uint64_t)c * NS + tid;
    s_mode[tid] = ws.emode[k];
    s_code[tid] = ws.ecode[k];
    s_off[tid] = ws.eoff[k];
  }
#pragma unroll
  for (int e = 0; e < NE; e++) s_enc[e][tid] = ws.enc[((uint64_t)c * NE + e) * 256 + tid];
  __syncthreads();

  const uint32_t v0 = tlo + tid * kGroupValues;  // chunk-relative index of my first value
  const int cnt = v0 < m ? (int)min32(kGroupValues, m - v0) : 0;
  uint32_t sym[NS][16];
  load_split16<DT>(src + (clo + v0) * VB, cnt, sym);
  const uint64_t nsub = ceil_div(m, g.S);

#pragma unroll
  for (int s = 0; s < NS; s++) {
    const uint32_t mode = s_mode[s];
    if (mode == kModeZero) continue;
    const int w = raw_width(DT, s);
    if (mode == kModeRaw && w == 8) {
      if (cnt > 0) {
        uint32_t x[4];
#pragma unroll
        for (int j = 0; j < 4; j++)
          x[j] = sym[s][4 * j] | (sym[s][4 * j + 1] << 8) | (sym[s][4 * j + 2] << 16) | (sym[s][4 * j + 3] << 24);
        *reinterpret_cast<uint4*>(out + s_off[s] + v0) = make_uint4(x[0], x[1], x[2], x[3]);
      }
      continue;
    }
    if (s >= NB) continue;  // unreachable: only streams < NB can be bit-packed
    const bool huff = mode == kModeHuff;
    uint32_t code[16], len[16], mybits = 0;
#pragma unroll
    for (int i = 0; i < 16; i++) {
      uint32_t l = 0, cv = 0;
      if (i < cnt) {
        if (huff) {
          const uint32_t e = s_enc[s < NE ? s : 0][sym[s][i]];
          l = e >> 16;
          cv = e & 0xFFFFu;
        } else {
          l = (uint32_t)w;
          cv = sym[s][i];
        }
      }
      code[i] = cv;
      len[i] = l;
      mybits += l;
    }
    uint32_t tile_bits;
    const uint32_t myoff = block_exclusive_scan<kEncodeThreads>(mybits, s_warp, tile_bits);
    const uint32_t rec = (huff && s_code[s] == kNoCode) ? record_bytes(DT, s) : 0;
    const uint64_t idx_bytes = huff ? round16(4 * nsub) : 0;
    uint8_t* payload = out + s_off[s];
    uint32_t* bs = reinterpret_cast<uint32_t*>(payload + rec + idx_bytes);
    if (tid == 0) {
      if (huff) {
        const uint32_t e = s < NE ? s : 0;
        s_prefix = lookback(ws.tile_desc + (uint64_t)e * g.n_tiles, tile, c * g.tiles_per_chunk, tile_bits, ws.status);
      } else {
        s_prefix = (uint64_t)tlo * (uint64_t)w;
      }
    }
    const uint32_t nw_max = (31 + tile_bits + 31) / 32;
    for (uint32_t i = tid; i < nw_max; i += kEncodeThreads) s_stage[i] = 0;
    __syncthreads();
    const uint64_t P = s_prefix;
    if (huff && cnt > 0 && (v0 % g.S) == 0)
      reinterpret_cast<uint32_t*>(payload + rec)[v0 / g.S] = (uint32_t)(P + myoff);
    stage_bits(s_stage, (uint32_t)(P & 31) + myoff, code, len);
    __syncthreads();
    const uint64_t end = P + tile_bits;
    const uint32_t nw = (uint32_t)(((P & 31) + tile_bits + 31) >> 5);
    const uint64_t W0 = P >> 5;
    for (uint32_t i = tid; i < nw; i += kEncodeThreads) {
      const uint32_t word = s_stage[i];
      uint32_t* dst = bs + W0 + i;
      const uint32_t e = s < NE ? s : 0;
      if (i == 0 && (P & 31) != 0) {
        slot_merge(ws.slot + (uint64_t)e * g.n_tiles + tile, word, dst);
      } else if (i == nw - 1 && (end & 31) != 0 && !last) {
        slot_merge(ws.slot + (uint64_t)e * g.n_tiles + tile + 1, word, dst);
      } else {
        *dst = bswap32(word);
      }
    }
    if (last) {
      // zero padding after the bitstream, up to its 16-byte boundary
      const uint64_t padded_words = round16(ceil_div(end, 8)) / 4;
      for (uint64_t i = W0 + nw + tid; i < padded_words; i += kEncodeThreads) bs[i] = 0;
      if (huff) {
        uint32_t* idx = reinterpret_cast<uint32_t*>(payload + rec);
        for (uint64_t i = nsub + tid; i < idx_bytes / 4; i += kEncodeThreads) idx[i] = 0;
      }
    }
    if (huff && rec && ti == 0) {
      const int A = alphabet(DT, s);
      const uint32_t e = s < NE ? s : 0;
      if (tid < (int)rec) {
        uint32_t b = 0;
        if (2 * tid < A) b = (s_enc[e][2 * tid] >> 16) | ((s_enc[e][2 * tid + 1] >> 16) << 4);
        payload[tid] = (uint8_t)b;
      }
    }
    __syncthreads();
  }
}

template <int DT>
static cudaError_t encode_t(const void* src, const Geo& g, const Ws& ws, uint8_t* out, cudaStream_t st) {
  k_encode<DT><<<g.n_tiles, kEncodeThreads, 0, st>>>(static_cast<const uint8_t*>(src), g, ws, out);
  return cudaGetLastError();
}

cudaError_t launch_encode(const void* src, const Geo& g, const Ws& ws, uint8_t* out, cudaStream_t st) {
  switch (g.dt) {
    case kBF16: return encode_t<kBF16>(src, g, ws, out, st);
    case kFP32: return encode_t<kFP32>(src, g, ws, out, st);
    default: return encode_t<kFP8>(src, g, ws, out, st);
  }
}

}  // namespace zipnn

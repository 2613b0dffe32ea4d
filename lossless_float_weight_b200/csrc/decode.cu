// decode.cu -- k_decode: container -> tensor, the inverse of the split and the coding.
//
// One block per chunk. Every block checks the header against the call's arguments and
// its chunk's table entries; every read is bounded by the container size, so a damaged
// container yields ZIPNN_ERR_CORRUPT and never an out-of-bounds access.
// For each HUFF stream the block rebuilds the canonical code from its 4-bit lengths
// and fills a 4096-entry lookup table in shared memory (12-bit window -> symbol,
// length). Each thread then decodes whole sub-blocks of S symbols, starting at the bit
// offset idx[j], merges the streams back into BF16/FP32/FP8 words and writes them to
// HBM with 16-byte stores: no intermediate plane is materialised. A sub-block must end
// exactly where the next one starts.
#include "common.cuh"
#include "fields.cuh"
#include "huffman.cuh"
#include "launch.h"

namespace zipnn {

constexpr int kDecodeThreads = 128;
constexpr uint32_t kLutInvalid = 0x8000u;

// Big-endian-within-word bit reader over 32-bit words [0, end); words past `end`
// read as zero. buf holds nb valid bits, most significant first.
struct BitReader {
  const uint32_t* w;
  uint32_t pos, end;
  uint64_t buf;
  int nb;
  __device__ __forceinline__ uint32_t load(uint32_t i) const { return i < end ? bswap32(__ldg(w + i)) : 0u; }
  __device__ __forceinline__ void init(const uint32_t* words, uint32_t nwords, uint64_t bit) {
    w = words;
    end = nwords;
    pos = (uint32_t)(bit >> 5);
    buf = (uint64_t)load(pos++) << 32;
    nb = 32;
    const int skip = (int)(bit & 31);
    buf <<= skip;
    nb -= skip;
    refill();
  }
  __device__ __forceinline__ void refill() {
    if (nb <= 32) {
      buf |= (uint64_t)load(pos++) << (32 - nb);
      nb += 32;
    }
  }
  __device__ __forceinline__ uint32_t fixed(int width) {
    const uint32_t v = (uint32_t)(buf >> (64 - width));
    buf <<= width;
    nb -= width;
    return v;
  }
  __device__ __forceinline__ uint32_t huff(const uint16_t* lut, uint32_t& acc) {
    const uint32_t e = lut[buf >> 52];
    const uint32_t l = e & 15u;
    buf <<= l;
    nb -= (int)l;
    acc |= e;
    return (e >> 4) & 0xFFu;
  }
  __device__ __forceinline__ uint64_t position() const { return (uint64_t)pos * 32 - (uint64_t)nb; }
};

enum Kind : int { kKZero = 0, kKBytes = 1, kKBits = 2, kKHuff = 3 };

struct StreamState {
  int kind, width;
  const uint8_t* bytes;  // kKBytes: this sub-block's first byte
  BitReader br;
  const uint16_t* lut;
  uint32_t acc;
};

// Decode GV consecutive symbols of one stream (GV a multiple of 2; n <= GV valid).
template <int GV, bool FULL>
__device__ __forceinline__ void next_symbols(StreamState& st, uint32_t (&o)[GV], int n, uint32_t v) {
  switch (st.kind) {
    case kKHuff:
#pragma unroll
      for (int i = 0; i < GV; i += 2) {
        st.br.refill();
        if (FULL || i < n) o[i] = st.br.huff(st.lut, st.acc);
        else o[i] = 0;
        if (FULL || i + 1 < n) o[i + 1] = st.br.huff(st.lut, st.acc);
        else o[i + 1] = 0;
      }
      break;
    case kKBits:
#pragma unroll
      for (int i = 0; i < GV; i += 2) {
        st.br.refill();
        o[i] = (FULL || i < n) ? st.br.fixed(st.width) : 0u;
        o[i + 1] = (FULL || i + 1 < n) ? st.br.fixed(st.width) : 0u;
      }
      break;
    case kKBytes:
      if (FULL) {
        if constexpr (GV == 16) {
          const uint4 q = __ldg(reinterpret_cast<const uint4*>(st.bytes + v));
          const uint32_t x[4] = {q.x, q.y, q.z, q.w};
#pragma unroll
          for (int i = 0; i < 16; i++) o[i] = (x[i >> 2] >> (8 * (i & 3))) & 0xFFu;
        } else if constexpr (GV == 8) {
          const uint2 q = __ldg(reinterpret_cast<const uint2*>(st.bytes + v));
#pragma unroll
          for (int i = 0; i < 8; i++) o[i] = ((i < 4 ? q.x : q.y) >> (8 * (i & 3))) & 0xFFu;
        } else {
          const uint32_t q = __ldg(reinterpret_cast<const uint32_t*>(st.bytes + v));
#pragma unroll
          for (int i = 0; i < GV; i++) o[i] = (q >> (8 * i)) & 0xFFu;
        }
      } else {
#pragma unroll
        for (int i = 0; i < GV; i++) o[i] = i < n ? (uint32_t)st.bytes[v + i] : 0u;
      }
      break;
    default:
#pragma unroll
      for (int i = 0; i < GV; i++) o[i] = 0;
  }
}

template <int DT>
struct DecodeSmem {
  uint16_t lut[n_entropy(DT)][4096];
  uint8_t lens[n_entropy(DT)][256];
  uint32_t enc[n_entropy(DT)][256];
  uint8_t sorted[n_entropy(DT)][256];
  uint32_t limit[n_entropy(DT)][kLmax + 1];
  uint32_t first[n_entropy(DT)][kLmax + 1];
  uint32_t offset[n_entropy(DT)][kLmax + 1];
  uint32_t mode[n_streams(DT)], code[n_streams(DT)];
  uint64_t off[n_streams(DT)], end[n_streams(DT)];
  uint64_t off_codes;
  uint32_t S, G;
  int bad;
};

template <int DT>
__global__ void __launch_bounds__(kDecodeThreads) k_decode(const uint8_t* __restrict__ in, uint64_t in_bytes, Geo g,
                                                           uint8_t* __restrict__ out, uint32_t* status) {
  constexpr int NS = n_streams(DT), NE = n_entropy(DT), VB = value_bytes(DT);
  constexpr int GV = DT == kBF16 ? 8 : DT == kFP32 ? 4 : 16;  // values per 16-byte store
  __shared__ DecodeSmem<DT> sm;
  const int tid = threadIdx.x;
  const uint32_t c = blockIdx.x;
  const uint64_t clo = (uint64_t)c * g.m0;
  const uint32_t m = (uint32_t)min64(g.m0, g.n - clo);

  if (tid == 0) {
    int bad = 0;
    const uint32_t* h = reinterpret_cast<const uint32_t*>(in);
    uint64_t total = 0, off_codes = 0, off_payload = 0;
    uint32_t S = 0, G = 0;
    if (in_bytes < kHeaderBytes) {
      bad = 1;
    } else {
      uint32_t hv[16];
      for (int i = 0; i < 16; i++) hv[i] = h[i];
      const uint64_t n = hv[2] | ((uint64_t)hv[3] << 32);
      S = hv[5];
      G = (hv[14] >> 8) & 0xFF;
      off_codes = hv[8] | ((uint64_t)hv[9] << 32);
      off_payload = hv[10] | ((uint64_t)hv[11] << 32);
      total = hv[12] | ((uint64_t)hv[13] << 32);
      const uint64_t entries = (uint64_t)g.n_chunks * NS;
      if (hv[0] != 0x314E4E5Au || hv[1] != (1u | ((uint32_t)DT << 16) | ((uint32_t)NS << 24))) bad = 1;
      if (n != g.n || hv[4] != g.chunk_bytes || hv[6] != g.n_chunks) bad = 1;
      if (S == 0 || (S & 15) || S > 65536) bad = 1;
      if ((hv[14] & 0xFF) != (uint32_t)kLmax || (hv[14] >> 16) != 0 || hv[15] != 0) bad = 1;
      if (G > kMaxGroups || hv[7] != G * NE) bad = 1;
      if (off_codes != kHeaderBytes + entries * kEntryBytes) bad = 1;
      if (!bad && off_payload != off_codes + shared_bytes(DT, G)) bad = 1;
      if (total > in_bytes || total < off_payload || (total & 15)) bad = 1;
    }
    if (!bad) {
      const uint64_t entries = (uint64_t)g.n_chunks * NS;
      for (int s = 0; s < NS && !bad; s++) {
        const uint64_t k = (uint64_t)c * NS + s;
        const uint4 ent = *reinterpret_cast<const uint4*>(in + kHeaderBytes + kEntryBytes * k);
        const uint64_t off = ent.z | ((uint64_t)ent.w << 32);
        uint64_t end = total;
        if (k + 1 < entries) {
          const uint4 nx = *reinterpret_cast<const uint4*>(in + kHeaderBytes + kEntryBytes * (k + 1));
          end = nx.z | ((uint64_t)nx.w << 32);
        }
        const uint32_t mode = ent.x & 0xFF;
        if ((ent.x >> 8) != 0 || mode > kModeHuff) bad = 1;
        if ((off & 15) || (end & 15) || off > end || end > total || off < off_payload) bad = 1;
        if (k == 0 && off != off_payload) bad = 1;
        const uint64_t extent = end - off;
        const int w = raw_width(DT, s);
        if (mode == kModeRaw) {
          if (ent.y != kNoCode || extent * 8 < (uint64_t)m * w) bad = 1;
        } else if (mode == kModeZero) {
          if (ent.y != kNoCode) bad = 1;
        } else if (mode == kModeHuff) {
          const uint64_t nsub = ceil_div(m, S);
          uint64_t need = round16(4 * nsub);
          if (!is_entropy(DT, s)) bad = 1;
          else if (ent.y == kNoCode) need += record_bytes(DT, s);
          else if (G == 0 || ent.y >= G * NE || ent.y / G != (uint32_t)s) bad = 1;
          if (extent < need) bad = 1;
        }
        sm.mode[s] = mode;
        sm.code[s] = ent.y;
        sm.off[s] = off;
        sm.end[s] = end;
      }
    }
    sm.off_codes = off_codes;
    sm.S = S;
    sm.G = G;
    sm.bad = bad;
  }
  __syncthreads();
  if (sm.bad) {
    if (tid == 0) set_status(status, kStCorrupt);
    return;
  }
  const uint32_t S = sm.S;

  // code lengths of the HUFF streams
#pragma unroll
  for (int e = 0; e < NE; e++) {
    if (sm.mode[e] != kModeHuff) continue;
    const uint8_t* rp = sm.code[e] == kNoCode
                            ? in + sm.off[e]
                            : in + sm.off_codes + shared_record_pos(DT, sm.G, sm.code[e]);
    const int A = alphabet(DT, e);
    for (int s = tid; s < 256; s += kDecodeThreads) {
      uint32_t l = 0;
      if (s < A) {
        const uint32_t b = rp[s >> 1];
        l = (s & 1) ? (b >> 4) : (b & 15u);
      }
      sm.lens[e][s] = (uint8_t)l;
    }
  }
  __syncthreads();
  // check each code (lengths <= 12, at least one symbol, Kraft sum <= 1), build the
  // canonical values and the decode tables
  const int warp = tid >> 5, lane = tid & 31;
  if (warp < NE && sm.mode[warp] == kModeHuff) {
    const int e = warp;
    uint32_t kraft = 0, present = 0, toolong = 0;
    for (int s = lane; s < 256; s += 32) {
      const uint32_t l = sm.lens[e][s];
      if (l > kLmax) toolong = 1;
      else if (l) {
        present++;
        kraft += 1u << (kLmax - l);
      }
    }
    for (int o = 16; o; o >>= 1) {
      kraft += __shfl_xor_sync(0xFFFFFFFFu, kraft, o);
      present += __shfl_xor_sync(0xFFFFFFFFu, present, o);
      toolong |= __shfl_xor_sync(0xFFFFFFFFu, toolong, o);
    }
    if (toolong || !present || kraft > (1u << kLmax)) {
      if (lane == 0) sm.bad = 1;
    } else {
      warp_canonical(sm.lens[e], sm.enc[e]);
      if (lane == 0) {
        uint32_t count[kLmax + 1] = {0};
        for (int s = 0; s < 256; s++) count[sm.lens[e][s]]++;
        uint32_t code = 0, offs = 0;
        count[0] = 0;
        sm.limit[e][0] = 0;
        for (int l = 1; l <= kLmax; l++) {
          code = (code + count[l - 1]) << 1;
          sm.first[e][l] = code;
          sm.offset[e][l] = offs;
          offs += count[l];
          sm.limit[e][l] = (code + count[l]) << (kLmax - l);
        }
      }
    }
  }
  __syncthreads();
  if (sm.bad) {
    if (tid == 0) set_status(status, kStCorrupt);
    return;
  }
#pragma unroll
  for (int e = 0; e < NE; e++) {
    if (sm.mode[e] != kModeHuff) continue;
    for (int s = tid; s < 256; s += kDecodeThreads) {
      const uint32_t v = sm.enc[e][s];
      const uint32_t l = v >> 16;
      if (l) sm.sorted[e][sm.offset[e][l] + (v & 0xFFFFu) - sm.first[e][l]] = (uint8_t)s;
    }
  }
  __syncthreads();
#pragma unroll
  for (int e = 0; e < NE; e++) {
    if (sm.mode[e] != kModeHuff) continue;
    for (uint32_t x = tid; x < 4096; x += kDecodeThreads) {
      uint32_t entry = kLutInvalid | 1u;
      if (x < sm.limit[e][kLmax]) {
        uint32_t l = 1;
#pragma unroll
        for (int j = 1; j < kLmax; j++) l += x >= sm.limit[e][j];
        const uint32_t sym = sm.sorted[e][sm.offset[e][l] + (x >> (kLmax - l)) - sm.first[e][l]];
        entry = (sym << 4) | l;
      }
      sm.lut[e][x] = (uint16_t)entry;
    }
  }
  __syncthreads();

  // decode: one sub-block per thread per pass
  const uint64_t nsub = ceil_div(m, S);
  for (uint64_t j = tid; j < nsub; j += kDecodeThreads) {
    const uint32_t sb_lo = (uint32_t)(j * S);
    const uint32_t count = min32(S, m - sb_lo);
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
      check_exact[s] = false;
      expect_end[s] = 0;
      if (mode == kModeZero) {
        st[s].kind = kKZero;
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
        st[s].kind = kKHuff;
        st[s].lut = sm.lut[e];
        st[s].br.init(reinterpret_cast<const uint32_t*>(in + bs_off), (uint32_t)(cap_bits / 32), bad ? 0 : start);
      }
    }
    uint8_t* dst = out + (clo + sb_lo) * VB;
    const uint32_t full = count / GV;
    for (uint32_t gi = 0; gi < full; gi++) {
      uint32_t sy[NS][GV];
#pragma unroll
      for (int s = 0; s < NS; s++) next_symbols<GV, true>(st[s], sy[s], GV, gi * GV);
      uint32_t wv[4];
#pragma unroll
      for (int q = 0; q < 4; q++) {
        if constexpr (DT == kBF16) {
          wv[q] = merge_value<DT>(sy[0][2 * q], sy[1][2 * q], 0, 0) |
                  (merge_value<DT>(sy[0][2 * q + 1], sy[1][2 * q + 1], 0, 0) << 16);
        } else if constexpr (DT == kFP32) {
          wv[q] = merge_value<DT>(sy[0][q], sy[1][q], sy[2][q], sy[3][q]);
        } else {
          uint32_t x = 0;
#pragma unroll
          for (int b = 0; b < 4; b++) x |= merge_value<DT>(sy[0][4 * q + b], sy[1][4 * q + b], sy[2][4 * q + b], 0) << (8 * b);
          wv[q] = x;
        }
      }
      *reinterpret_cast<uint4*>(dst + (uint64_t)gi * 16) = make_uint4(wv[0], wv[1], wv[2], wv[3]);
    }
    const uint32_t rem = count - full * GV;
    if (rem) {
      uint32_t sy[NS][GV];
#pragma unroll
      for (int s = 0; s < NS; s++) next_symbols<GV, false>(st[s], sy[s], (int)rem, full * GV);
      for (uint32_t i = 0; i < rem; i++) {
        const uint32_t v = merge_value<DT>(sy[0][i], sy[1][i], NS > 2 ? sy[NS > 2 ? 2 : 0][i] : 0,
                                           NS > 3 ? sy[NS > 3 ? 3 : 0][i] : 0);
        uint8_t* p = dst + (uint64_t)(full * GV + i) * VB;
        if constexpr (VB == 2) *reinterpret_cast<uint16_t*>(p) = (uint16_t)v;
        else if constexpr (VB == 4) *reinterpret_cast<uint32_t*>(p) = v;
        else *p = (uint8_t)v;
      }
    }
#pragma unroll
    for (int s = 0; s < NS; s++) {
      if (st[s].kind != kKHuff) continue;
      const uint64_t pos = st[s].br.position();
      if (st[s].acc & kLutInvalid) bad = 1;
      if (check_exact[s] ? pos != expect_end[s] : pos > expect_end[s]) bad = 1;
    }
    if (bad) set_status(status, kStCorrupt);
  }
}

template <int DT>
static cudaError_t decode_t(const uint8_t* in, uint64_t in_bytes, const Geo& g, uint8_t* out, uint32_t* status,
                            cudaStream_t st) {
  k_decode<DT><<<g.n_chunks, kDecodeThreads, 0, st>>>(in, in_bytes, g, out, status);
  return cudaGetLastError();
}

cudaError_t launch_decode(const uint8_t* in, uint64_t in_bytes, const Geo& g, uint8_t* out, uint32_t* status,
                          cudaStream_t st) {
  switch (g.dt) {
    case kBF16: return decode_t<kBF16>(in, in_bytes, g, out, status, st);
    case kFP32: return decode_t<kFP32>(in, in_bytes, g, out, status, st);
    default: return decode_t<kFP8>(in, in_bytes, g, out, status, st);
  }
}

}  // namespace zipnn

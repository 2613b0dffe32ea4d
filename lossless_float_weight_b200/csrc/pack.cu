// pack.cu -- packed exponent tuples ("NeuralZip: Reusable Setup for Fast Lossless
// Compression", abstract: the setup selectively represents recurring exponent tuples
// with packed exponents). BF16 only. The plan lists its tensor's K <= 15 most frequent
// exponents; the exponents of values 2j and 2j + 1 of a chunk form one 8-bit pair
// symbol, each exponent's index in the list as a nibble (first value high), kPackEsc for
// an exponent not in the list, whose 8 bits then follow the pair's code. Each group has a
// packed code over the pair symbols next to its plain code; a chunk takes whichever codes
// it in fewer bits (the code build decides).
//
//   k_pack_select     : (setup) the list, from the exponent counts of every chunk;
//   k_pack_hist       : per chunk, the pair-symbol counts and the escaped exponents;
//   k_pack_group_sums : (setup) each group's summed pair counts (chunks of whole pairs);
//   k_encode_pack     : per PACK chunk, the sub-block index and the bitstream (and a RAW
//                       sign/fraction plane).
#include "common.cuh"
#include "launch.h"

namespace zipnn {

constexpr int kPackThreads = 256;

// One block: the exponent counts summed over the chunks (thread t: exponent t), then the
// K most frequent exponents, a larger count first and equal counts by the smaller
// exponent. Writes the list (16 bytes, zero past K) and K.
__global__ void __launch_bounds__(kPackThreads) k_pack_select(const uint32_t* __restrict__ hist, uint32_t C,
                                                              uint32_t NE, uint32_t max_pack, uint8_t* exps_out,
                                                              uint32_t* k_out) {
  __shared__ uint64_t cnt[256];
  const int t = threadIdx.x;
  uint64_t s = 0;
  for (uint32_t c = 0; c < C; c++) s += hist[((uint64_t)c * NE) * 256 + t];
  cnt[t] = s;
  __syncthreads();
  if (t == 0) {
    bool taken[256];
    for (int i = 0; i < 256; i++) taken[i] = false;
    uint32_t K = 0;
    uint8_t list[kPackListBytes];
    for (uint32_t i = 0; i < kPackListBytes; i++) list[i] = 0;
    while (K < max_pack) {
      int best = -1;
      for (int i = 0; i < 256; i++)
        if (!taken[i] && cnt[i] && (best < 0 || cnt[i] > cnt[best])) best = i;
      if (best < 0) break;
      taken[best] = true;
      list[K++] = (uint8_t)best;
    }
    for (uint32_t i = 0; i < kPackListBytes; i++) exps_out[i] = list[i];
    *k_out = K;
  }
}

// Nibble table of a list: nib[x] = the index of exponent x in the list, else kPackEsc.
__device__ __forceinline__ void fill_nibbles(uint8_t* nib, const uint8_t* exps, uint32_t K) {
  for (int x = threadIdx.x; x < 256; x += blockDim.x) {
    uint32_t v = kPackEsc;
    for (int i = (int)K - 1; i >= 0; i--)
      if (exps[i] == x) v = (uint32_t)i;
    nib[x] = (uint8_t)v;
  }
}

// The sign/fraction bytes of the two BF16 values of a word (bit 15 over bits 6..0), in
// bytes 0 and 1.
__device__ __forceinline__ uint32_t sf_pair(uint32_t w) {
  const uint32_t t = (w & 0x007F007Fu) | ((w >> 8) & 0x00800080u);
  return (t & 0xFFu) | ((t >> 8) & 0xFF00u);
}

// The pair symbol of one 32-bit word of BF16 input (value 2j in the low half).
__device__ __forceinline__ uint32_t pair_symbol(uint32_t w, const uint8_t* nib) {
  return ((uint32_t)nib[(w >> 7) & 0xFFu] << 4) | nib[(w >> 23) & 0xFFu];
}

// One block per chunk: the pair-symbol counts of a chunk of whole pairs (per-warp counters
// in shared memory, summed at the end) and its escaped exponents; a chunk with an odd
// value count gets zeros (it cannot take a packed code).
__global__ void __launch_bounds__(kPackThreads) k_pack_hist(const uint8_t* __restrict__ src, Geo g, Ws ws,
                                                            PlanDev plan) {
  __shared__ uint32_t cnt[kPackThreads / 32][256];
  __shared__ uint8_t nib[256];
  __shared__ uint32_t s_esc[kPackThreads / 32];
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const uint32_t c = blockIdx.x;
  const uint64_t clo = (uint64_t)c * g.m0;
  const uint32_t m = (uint32_t)min64(g.m0, g.n - clo);
  for (int i = tid; i < (kPackThreads / 32) * 256; i += kPackThreads) (&cnt[0][0])[i] = 0;
  fill_nibbles(nib, plan.pack_exps, plan.pack_k);
  __syncthreads();
  uint32_t esc = 0;
  if (m % 2 == 0) {
    const uint32_t pairs = m / 2, quads = pairs / 4;
    const uint4* q = reinterpret_cast<const uint4*>(src + clo * 2);  // chunks start 16-byte aligned
    for (uint32_t i = tid; i < quads; i += kPackThreads) {
      const uint4 v = __ldg(q + i);
      const uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
      for (int j = 0; j < 4; j++) {
        const uint32_t s = pair_symbol(w[j], nib);
        atomicAdd(&cnt[warp][s], 1u);
        esc += ((s >> 4) == kPackEsc) + ((s & 15u) == kPackEsc);
      }
    }
    const uint32_t* wp = reinterpret_cast<const uint32_t*>(src + clo * 2);
    for (uint32_t i = quads * 4 + tid; i < pairs; i += kPackThreads) {
      const uint32_t s = pair_symbol(__ldg(wp + i), nib);
      atomicAdd(&cnt[warp][s], 1u);
      esc += ((s >> 4) == kPackEsc) + ((s & 15u) == kPackEsc);
    }
  }
  esc = __reduce_add_sync(0xFFFFFFFFu, esc);
  if (lane == 0) s_esc[warp] = esc;
  __syncthreads();
  uint32_t total = 0;
#pragma unroll
  for (int w = 0; w < kPackThreads / 32; w++) total += cnt[w][tid];
  ws.pack_hist[(uint64_t)c * 256 + tid] = total;
  if (tid == 0) {
    uint32_t e = 0;
    for (int w = 0; w < kPackThreads / 32; w++) e += s_esc[w];
    ws.pack_esc[c] = e;
  }
}

// Each group's summed pair counts over its member chunks (gsum: [G][256], cleared first).
__global__ void k_pack_group_sums(const uint32_t* __restrict__ pack_hist, const uint32_t* __restrict__ assign,
                                  uint32_t C, uint64_t* gsum) {
  const uint64_t t = (uint64_t)blockIdx.x * blockDim.x + threadIdx.x;
  if (t >= (uint64_t)C * 256) return;
  const uint32_t v = pack_hist[t];
  if (v) atomicAdd(reinterpret_cast<unsigned long long*>(gsum + (uint64_t)assign[t / 256] * 256 + t % 256),
                   (unsigned long long)v);
}

// One block per chunk whose exponent stream is PACK (others return at once); it also
// writes the chunk's sign/fraction plane when that is RAW. The payload
// [index of ceil(m / S) u32, padded][bitstream, padded] is zeroed first. Then, a round at
// a time, each warp takes one sub-block, lane l the pairs [p0 + l q, p0 + (l + 1) q) (q =
// ceil(pairs / 32); at most kPackRegPairs held in registers): each lane forms its pairs'
// bits (the code, then each escaped exponent's 8 bits: at most 28 a pair) and their
// total, a warp scan places the lanes' runs and the warps' totals (one barrier a round,
// double-buffered) place the sub-blocks after the rounds before; each lane then appends
// its bits to a 64-bit accumulator, flushing whole words into its own shared words, and
// moves those words to its bit offset with funnel shifts: plain stores for the middle
// words, atomicOr for the two it may share with its neighbours.
constexpr int kPackRegPairs = 8;
constexpr int kPackPrivWords = kPackRegPairs * 28 / 32 + 1;  // 8 pairs of at most 28 bits

__global__ void __launch_bounds__(kPackThreads) k_encode_pack(const uint8_t* __restrict__ src, Geo g, Ws ws,
                                                              PlanDev plan, uint8_t* __restrict__ out) {
  constexpr int NW = kPackThreads / 32;
  __shared__ uint32_t enc[256];
  __shared__ uint8_t nib[256];
  __shared__ uint32_t s_tot[2][NW];
  __shared__ uint32_t priv[kPackPrivWords + 1][kPackThreads];  // lane-major: conflict-free
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const uint32_t c = blockIdx.x;
  if (ws.emode[2ull * c] != kModePack) return;  // uniform
  const uint64_t clo = (uint64_t)c * g.m0;
  const uint32_t m = (uint32_t)min64(g.m0, g.n - clo);  // even: the code build checked it
  const uint32_t S = g.S;
  const uint64_t nsub = ceil_div(m, S);
  uint8_t* payload = out + ws.eoff[2ull * c];
  const uint64_t size = ws.esize[2ull * c];
  uint4* pz = reinterpret_cast<uint4*>(payload);
  for (uint64_t i = tid; i < size / 16; i += kPackThreads) pz[i] = make_uint4(0, 0, 0, 0);
  // a RAW sign/fraction plane is written here too, from the same loads (k_encode_bf16
  // skips these chunks); its padding to 16 bytes is zero
  uint8_t* plane = ws.emode[2ull * c + 1] == kModeRaw ? out + ws.eoff[2ull * c + 1] : nullptr;
  if (plane && tid < (int)(round16(m) - m)) plane[m + tid] = 0;
  enc[tid] = ws.enc[(uint64_t)c * 256 + tid];
  fill_nibbles(nib, plan.pack_exps, plan.pack_k);
  __syncthreads();
  uint32_t* idx = reinterpret_cast<uint32_t*>(payload);
  uint32_t* bs = reinterpret_cast<uint32_t*>(payload + round16(4 * nsub));
  const uint32_t* wp = reinterpret_cast<const uint32_t*>(src + clo * 2);
  // a pair's bits: the code, then each escaped exponent (value << 8 | length)
  auto pair_code = [&](uint32_t w, uint32_t& len) {
    const uint32_t a = nib[(w >> 7) & 0xFFu], b = nib[(w >> 23) & 0xFFu];
    const uint32_t e = enc[(a << 4) | b];
    uint32_t v = e & 0xFFFFu, l = e >> 16;
    if (a == kPackEsc) {
      v = (v << 8) | ((w >> 7) & 0xFFu);
      l += 8;
    }
    if (b == kPackEsc) {
      v = (v << 8) | ((w >> 23) & 0xFFu);
      l += 8;
    }
    len = l;
    return v;
  };
  uint32_t carry = 0;
  int buf = 0;
  for (uint64_t base = 0; base < nsub; base += NW, buf ^= 1) {
    const uint64_t j = base + warp;
    uint32_t a = 0, b = 0, q = 0;
    if (j < nsub) {
      const uint32_t p0 = (uint32_t)(j * S / 2), p1 = (uint32_t)min64(j * S + S, m) / 2;
      q = (p1 - p0 + 31) / 32;
      a = min32(p0 + lane * q, p1);
      b = min32(a + q, p1);
    }
    // a full run of 8: p0 (S / 2 j, S a multiple of 16) and 8 lane are multiples of 8 pairs,
    // so the run starts 32 bytes into the chunk's 16-byte aligned values
    const bool in_regs = q == (uint32_t)kPackRegPairs && b - a == (uint32_t)kPackRegPairs;
    uint32_t v[kPackRegPairs], l[kPackRegPairs];
    uint32_t bits = 0;
    if (in_regs) {
      const uint4 v0 = __ldg(reinterpret_cast<const uint4*>(wp + a));
      const uint4 v1 = __ldg(reinterpret_cast<const uint4*>(wp + a) + 1);
      const uint32_t w[kPackRegPairs] = {v0.x, v0.y, v0.z, v0.w, v1.x, v1.y, v1.z, v1.w};
#pragma unroll
      for (int i = 0; i < kPackRegPairs; i++) {
        v[i] = pair_code(w[i], l[i]);
        bits += l[i];
      }
      if (plane) {  // 16 values: 16 bytes at value 2a (a multiple of 16)
        uint32_t o[4];
#pragma unroll
        for (int k = 0; k < 4; k++) o[k] = sf_pair(w[2 * k]) | (sf_pair(w[2 * k + 1]) << 16);
        *reinterpret_cast<uint4*>(plane + 2 * (uint64_t)a) = make_uint4(o[0], o[1], o[2], o[3]);
      }
    } else {
      for (uint32_t p = a; p < b; p++) {
        uint32_t len;
        const uint32_t w = __ldg(wp + p);
        pair_code(w, len);
        bits += len;
        if (plane) {
          const uint32_t sf = sf_pair(w);
          plane[2 * (uint64_t)p] = (uint8_t)sf;
          plane[2 * (uint64_t)p + 1] = (uint8_t)(sf >> 8);
        }
      }
    }
    uint32_t incl = bits;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const uint32_t y = __shfl_up_sync(0xFFFFFFFFu, incl, o);
      if (lane >= o) incl += y;
    }
    if (lane == 31) s_tot[buf][warp] = incl;
    __syncthreads();
    uint32_t before = 0, round_total = 0;
#pragma unroll
    for (int k = 0; k < NW; k++) {
      const uint32_t t = s_tot[buf][k];
      if (k < warp) before += t;
      round_total += t;
    }
    const uint32_t sub_start = carry + before;
    if (j < nsub && lane == 0) idx[j] = sub_start;
    if (bits) {
      const uint32_t start = sub_start + incl - bits;
      if (in_regs) {
        // append the codes, whole words into my shared words (pending bits < 32 + 28)
        uint64_t acc = 0;
        uint32_t nfill = 0, nw = 0;
#pragma unroll
        for (int i = 0; i < kPackRegPairs; i++) {
          acc = (acc << l[i]) | v[i];
          nfill += l[i];
          if (nfill >= 32) {
            nfill -= 32;
            priv[nw++][tid] = (uint32_t)(acc >> nfill);
          }
        }
        if (nfill) priv[nw++][tid] = (uint32_t)(acc << (32 - nfill));
        // word k of my run goes to bitstream word d0 + k, shifted right by sh
        const uint32_t sh = start & 31u, d0 = start >> 5, nk = ((start + bits - 1) >> 5) - d0 + 1;
        uint32_t cur = priv[0][tid];
        atomicOr(bs + d0, bswap32(__funnelshift_r(cur, 0u, sh)));
        for (uint32_t k = 1; k + 1 < nk; k++) {
          const uint32_t prev = cur;
          cur = priv[k][tid];
          bs[d0 + k] = bswap32(__funnelshift_r(cur, prev, sh));
        }
        if (nk > 1) atomicOr(bs + d0 + nk - 1, bswap32(__funnelshift_r(nk - 1 < nw ? priv[nk - 1][tid] : 0u, cur, sh)));
      } else {
        // a long or short run (S other than 512, a chunk's last sub-block): bit by bit
        // merges of each pair's bits into the zeroed words
        uint32_t t = start;
        for (uint32_t p = a; p < b; p++) {
          uint32_t len;
          const uint32_t x = pair_code(__ldg(wp + p), len);
          // at most 28 bits: they span at most two words
          const uint32_t sh = t & 31u;
          const uint64_t placed = ((uint64_t)x << (64 - len)) >> sh;
          atomicOr(bs + (t >> 5), bswap32((uint32_t)(placed >> 32)));
          if (sh + len > 32) atomicOr(bs + (t >> 5) + 1, bswap32((uint32_t)placed));
          t += len;
        }
      }
    }
    carry += round_total;
  }
}

cudaError_t launch_pack_select(const uint32_t* hist, uint32_t C, uint32_t NE, uint32_t max_pack, uint8_t* exps,
                               uint32_t* k_out, cudaStream_t st) {
  k_pack_select<<<1, kPackThreads, 0, st>>>(hist, C, NE, max_pack, exps, k_out);
  return cudaGetLastError();
}

cudaError_t launch_pack_hist(const void* src, const Geo& g, const Ws& ws, const PlanDev& plan, cudaStream_t st) {
  k_pack_hist<<<g.n_chunks, kPackThreads, 0, st>>>(static_cast<const uint8_t*>(src), g, ws, plan);
  return cudaGetLastError();
}

cudaError_t launch_pack_group_sums(const uint32_t* pack_hist, const uint32_t* assign, uint32_t C, uint64_t* gsum,
                                   cudaStream_t st) {
  const uint64_t n = (uint64_t)C * 256;
  k_pack_group_sums<<<(uint32_t)((n + 255) / 256), 256, 0, st>>>(pack_hist, assign, C, gsum);
  return cudaGetLastError();
}

cudaError_t launch_encode_pack(const void* src, const Geo& g, const Ws& ws, const PlanDev& plan, uint8_t* out,
                               cudaStream_t st) {
  k_encode_pack<<<g.n_chunks, kPackThreads, 0, st>>>(static_cast<const uint8_t*>(src), g, ws, plan, out);
  return cudaGetLastError();
}

}  // namespace zipnn

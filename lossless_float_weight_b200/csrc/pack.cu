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
//   k_encode_pack     : per PACK chunk, the sub-block index and the bitstream.
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

// Bit writer over 32-bit words of a bitstream that is stored most significant bit first
// (byte 0 holds bits 0..7): bits before `start` in its first word, and after its end in
// its last word, belong to the neighbouring sub-blocks, so those two words are merged
// with atomicOr into the zeroed payload; every other word is this writer's alone.
struct PackWriter {
  uint32_t* words;
  uint64_t buf;   // pending bits, left-aligned
  int nb;         // pending bits in buf, counting the leading bits of a shared first word
  uint32_t wi;    // index of the word buf's top bits go to
  bool shared;    // the word at wi is shared with the previous sub-block
  __device__ __forceinline__ void init(uint32_t* w, uint64_t start) {
    words = w;
    buf = 0;
    nb = (int)(start & 31);
    wi = (uint32_t)(start >> 5);
    shared = nb != 0;
  }
  __device__ __forceinline__ void put(uint32_t v, int len) {
    buf |= (uint64_t)v << (64 - nb - len);
    nb += len;
    if (nb >= 32) {
      const uint32_t w = bswap32((uint32_t)(buf >> 32));
      if (shared) atomicOr(words + wi, w);
      else words[wi] = w;
      shared = false;
      buf <<= 32;
      nb -= 32;
      wi++;
    }
  }
  __device__ __forceinline__ void finish() {
    if (nb > 0) atomicOr(words + wi, bswap32((uint32_t)(buf >> 32)));
  }
};

// One block per chunk whose exponent stream is PACK (others return at once). The payload
// [index of ceil(m / S) u32, padded][bitstream, padded] is zeroed first. Then, a round at
// a time, each warp takes one sub-block, lane l the pairs [p0 + l q, p0 + (l + 1) q) (q =
// ceil(pairs / 32); at most 8 are held in registers): the lanes size their runs (code
// lengths plus 8 bits an escape), a warp scan places the runs, the warps' totals (one
// barrier a round, double-buffered) place the sub-blocks after the rounds before, and each
// lane writes its codes. The input is read once when S <= 512.
constexpr int kPackRegPairs = 8;

__global__ void __launch_bounds__(kPackThreads) k_encode_pack(const uint8_t* __restrict__ src, Geo g, Ws ws,
                                                              PlanDev plan, uint8_t* __restrict__ out) {
  constexpr int NW = kPackThreads / 32;
  __shared__ uint32_t enc[256];
  __shared__ uint8_t nib[256];
  __shared__ uint32_t s_tot[2][NW];
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
  enc[tid] = ws.enc[(uint64_t)c * 256 + tid];
  fill_nibbles(nib, plan.pack_exps, plan.pack_k);
  __syncthreads();
  uint32_t* idx = reinterpret_cast<uint32_t*>(payload);
  uint32_t* bs = reinterpret_cast<uint32_t*>(payload + round16(4 * nsub));
  const uint32_t* wp = reinterpret_cast<const uint32_t*>(src + clo * 2);
  auto pair_bits = [&](uint32_t w) {
    const uint32_t s = pair_symbol(w, nib);
    return (enc[s] >> 16) + 8u * (((s >> 4) == kPackEsc) + ((s & 15u) == kPackEsc));
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
    uint32_t w[kPackRegPairs];
    uint32_t bits = 0;
    if (in_regs) {
      const uint4 v0 = __ldg(reinterpret_cast<const uint4*>(wp + a));
      const uint4 v1 = __ldg(reinterpret_cast<const uint4*>(wp + a) + 1);
      w[0] = v0.x; w[1] = v0.y; w[2] = v0.z; w[3] = v0.w;
      w[4] = v1.x; w[5] = v1.y; w[6] = v1.z; w[7] = v1.w;
#pragma unroll
      for (int i = 0; i < kPackRegPairs; i++) bits += pair_bits(w[i]);
    } else {
      for (uint32_t p = a; p < b; p++) bits += pair_bits(__ldg(wp + p));
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
    if (a < b) {
      PackWriter wr;
      wr.init(bs, (uint64_t)sub_start + incl - bits);
      auto put_pair = [&](uint32_t x) {
        const uint32_t s = pair_symbol(x, nib);
        wr.put(enc[s] & 0xFFFFu, (int)(enc[s] >> 16));
        if ((s >> 4) == kPackEsc) wr.put((x >> 7) & 0xFFu, 8);
        if ((s & 15u) == kPackEsc) wr.put((x >> 23) & 0xFFu, 8);
      };
      if (in_regs) {
#pragma unroll
        for (int i = 0; i < kPackRegPairs; i++) put_pair(w[i]);
      } else {
        for (uint32_t p = a; p < b; p++) put_pair(__ldg(wp + p));
      }
      wr.finish();
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

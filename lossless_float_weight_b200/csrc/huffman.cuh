// huffman.cuh -- per-chunk canonical Huffman code construction on the GPU.
//
// THEORY-599 note on ZipNN, "Order-0 only (section III-A b)": the exponent stream is
// coded with a Huffman code built from its order-0 histogram. The pages leave the
// construction's details open; this library fixes them so that the code is a
// function of the histogram alone:
//  * ties: the two nodes with the smallest (weight, order) keys merge first, a leaf's
//    order being its symbol and the i-th merged node's order 256 + i (minimum-variance
//    Huffman). Leaves sorted by (weight, symbol) and merged nodes in creation order
//    form two queues whose heads give that minimum, a leaf winning a weight tie.
//    Weights are full 64-bit counts, compared as (weight, symbol) pairs;
//  * length limit 12: the code of the weights max(1, f >> k) for the smallest k >= 0
//    whose longest code is at most 12 bits. The eight warps of a block try eight
//    values of k at once;
//  * canonical code values by the deflate rule (RFC 1951, section 3.2.2).
#pragma once
#include "common.cuh"

namespace zipnn {

constexpr int kHuffWarps = 8;

struct HuffScratch {
  uint64_t sorted[256];  // leaf weights in ascending (weight, symbol) order
  uint64_t iw[256];      // leaf weights in symbol order, then merged-node weights
  uint8_t ssym[256];     // symbol of sorted leaf i
  uint8_t isym[256];     // symbol of leaf iw[i] (read only before the merge reuses iw)
  uint16_t lpar[256];    // parent (merged-node index) of sorted leaf i
  uint16_t ipar[256];    // parent of merged node i
  uint8_t idep[256];     // depth of merged node i
  uint8_t lens[256];     // result, by symbol
};

struct HuffBlockSmem {
  uint64_t f[256];
  HuffScratch w[kHuffWarps];
  int maxlen[kHuffWarps];
  uint64_t cost[2 * kMaxGroups];  // plain group codes, then packed ones
  uint32_t elig[2 * kMaxGroups];
  uint64_t red[kHuffWarps];
  uint32_t red32[kHuffWarps];
  int pick;
  uint32_t bits_lo, bits_hi;
};

__device__ __forceinline__ uint32_t lanemask_lt() {
  uint32_t m;
  asm("mov.u32 %0, %%lanemask_lt;" : "=r"(m));
  return m;
}

// The same code as warp_huffman below for 2 <= n <= 32 present symbols whose weights and
// symbols are in sc.iw[0..n) and sc.isym[0..n), with every per-node quantity in
// registers: lane p holds the p-th smallest leaf and the p-th merged node. The two-queue
// merge runs on all lanes in step (its indices and sums are warp-uniform) and fetches
// queue heads by shuffle; depths follow by pointer jumping towards the root.
__device__ inline int warp_huffman_regs(HuffScratch& sc, int n) {
  const int lane = threadIdx.x & 31;
  const uint64_t w = lane < n ? sc.iw[lane] : ~0ull;
  const uint32_t sy = lane < n ? sc.isym[lane] : 0xFFu;
  // rank of my leaf among the n leaves in (weight, symbol) order (symbols are distinct)
  int r = 0;
#pragma unroll
  for (int q = 0; q < 32; q++) {
    const uint64_t wq = __shfl_sync(0xFFFFFFFFu, w, q);
    const uint32_t sq = __shfl_sync(0xFFFFFFFFu, sy, q);
    r += q < n && (wq < w || (wq == w && sq < sy));
  }
  if (lane < n) {
    sc.sorted[r] = w;
    sc.ssym[r] = (uint8_t)sy;
  }
  __syncwarp();
  const uint64_t leaf_w = lane < n ? sc.sorted[lane] : ~0ull;
  const uint32_t leaf_s = sc.ssym[lane];
  uint64_t node_w = 0;
  uint32_t leaf_par = 0, node_par = 0;
  uint32_t li = 0, ii = 0;
  uint64_t lh = __shfl_sync(0xFFFFFFFFu, leaf_w, 0), ih = 0;
  for (int t = 0; t < n - 1; t++) {
    uint64_t sum = 0;
#pragma unroll
    for (int pick = 0; pick < 2; pick++) {
      // a leaf wins a weight tie; no merged node is available while ii == t
      if ((int)li < n && ((int)ii >= t || lh <= ih)) {
        if (lane == (int)li) leaf_par = (uint32_t)t;
        sum += lh;
        li++;
        lh = __shfl_sync(0xFFFFFFFFu, leaf_w, li & 31);
      } else {
        if (lane == (int)ii) node_par = (uint32_t)t;
        sum += ih;
        ii++;
        ih = __shfl_sync(0xFFFFFFFFu, node_w, ii & 31);
      }
    }
    if (lane == t) node_w = sum;
    if ((int)ii == t) ih = sum;  // the head is the node just made
  }
  // depth of merged node t below the root (node n - 2), by pointer jumping
  const int root = n - 2;
  uint32_t d = lane < root ? 1u : 0u;
  uint32_t up = lane < root ? node_par : (uint32_t)lane;
#pragma unroll
  for (int k = 0; k < 5; k++) {
    const uint32_t du = __shfl_sync(0xFFFFFFFFu, d, up & 31);
    const uint32_t uu = __shfl_sync(0xFFFFFFFFu, up, up & 31);
    d += du;
    up = uu;
  }
  const uint32_t len = __shfl_sync(0xFFFFFFFFu, d, leaf_par & 31) + 1;
  if (lane < n) sc.lens[leaf_s] = (uint8_t)len;
  __syncwarp();
  return (int)__reduce_max_sync(0xFFFFFFFFu, lane < n ? len : 0u);
}

// One warp: lengths of the Huffman code for the weights max(1, f >> k) of the present
// symbols of f[0..A). Returns the longest length (0 if no symbol is present).
__device__ inline int warp_huffman(const uint64_t* f, int A, int k, HuffScratch& sc) {
  const int lane = threadIdx.x & 31;
  int n = 0;
#pragma unroll
  for (int i = 0; i < 8; i++) {
    const int s = i * 32 + lane;
    const uint64_t fs = s < A ? f[s] : 0;
    const bool p = fs > 0;
    const uint32_t b = __ballot_sync(0xFFFFFFFFu, p);
    if (p) {
      uint64_t g = k < 64 ? (fs >> k) : 0;
      if (g == 0) g = 1;
      const int at = n + __popc(b & lanemask_lt());
      sc.iw[at] = g;
      sc.isym[at] = (uint8_t)s;
    }
    n += __popc(b);
  }
  for (int s = lane; s < 256; s += 32) sc.lens[s] = 0;
  __syncwarp();
  if (n == 0) return 0;
  if (n == 1) {
    if (lane == 0) sc.lens[sc.isym[0]] = 1;
    __syncwarp();
    return 1;
  }
  if (n <= 32) return warp_huffman_regs(sc, n);
  // rank sort of the distinct keys (weight, symbol)
  for (int p = lane; p < n; p += 32) {
    const uint64_t wp = sc.iw[p];
    const uint32_t sp = sc.isym[p];
    int r = 0;
    for (int q = 0; q < n; q++) {
      const uint64_t wq = sc.iw[q];
      r += wq < wp || (wq == wp && sc.isym[q] < sp);
    }
    sc.sorted[r] = wp;
    sc.ssym[r] = (uint8_t)sp;
  }
  __syncwarp();
  if (lane == 0) {
    // two-queue merge: node t (t = 0..n-2) joins the two smallest heads
    int li = 0, ii = 0;
    for (int t = 0; t < n - 1; t++) {
      uint64_t sum = 0;
#pragma unroll
      for (int pick = 0; pick < 2; pick++) {
        const bool leaf = li < n && (ii >= t || sc.sorted[li] <= sc.iw[ii]);
        if (leaf) {
          sum += sc.sorted[li];
          sc.lpar[li] = (uint16_t)t;
          li++;
        } else {
          sum += sc.iw[ii];
          sc.ipar[ii] = (uint16_t)t;
          ii++;
        }
      }
      sc.iw[t] = sum;
    }
    sc.idep[n - 2] = 0;
    for (int t = n - 3; t >= 0; t--) sc.idep[t] = (uint8_t)(sc.idep[sc.ipar[t]] + 1);
  }
  __syncwarp();
  int mx = 0;
  for (int p = lane; p < n; p += 32) {
    const int d = sc.idep[sc.lpar[p]] + 1;
    sc.lens[sc.ssym[p]] = (uint8_t)(d > 255 ? 255 : d);
    mx = d > mx ? d : mx;
  }
  __syncwarp();
  return __reduce_max_sync(0xFFFFFFFFu, (uint32_t)mx);
}

// Whole block (kHuffWarps warps): length-limited lengths of sm.f[0..A). Returns the
// index of the warp whose sm.w[].lens holds the result. Call with all threads.
__device__ inline int block_limited_lengths(HuffBlockSmem& sm, int A) {
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  for (int round = 0; round < 8; round++) {
    const int k = round * kHuffWarps + warp;
    const int mx = warp_huffman(sm.f, A, k, sm.w[warp]);
    if (lane == 0) sm.maxlen[warp] = mx;
    __syncthreads();
    int found = -1;
    for (int w = 0; w < kHuffWarps; w++)
      if (sm.maxlen[w] <= kLmax) {
        found = w;
        break;
      }
    __syncthreads();
    if (found >= 0) return found;
  }
  return 0;  // unreachable: at k = 63 every weight is 1 and lengths are <= 8
}

// One warp: canonical code values (RFC 1951, 3.2.2) for lens[0..256); writes
// enc[s] = len << 16 | code (0 for absent symbols). Lane k holds symbols 8k..8k+7.
// Lengths are visited in increasing order; the first code of a length follows from
// the previous length's first code and count, and within a length the codes go to
// the symbols in increasing order (a scan over lanes gives each lane its offset).
// Every per-length quantity lives in registers: no local-memory arrays.
__device__ inline void warp_canonical(const uint8_t* lens, uint32_t* enc) {
  const int lane = threadIdx.x & 31;
  uint32_t L[8], v[8];
#pragma unroll
  for (int i = 0; i < 8; i++) {
    L[i] = lens[lane * 8 + i];
    v[i] = 0;
  }
  uint32_t first = 0, prev_count = 0;
#pragma unroll
  for (int l = 1; l <= kLmax; l++) {
    first = (first + prev_count) << 1;
    uint32_t c = 0;
#pragma unroll
    for (int i = 0; i < 8; i++) c += L[i] == (uint32_t)l;
    uint32_t x = c;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const uint32_t y = __shfl_up_sync(0xFFFFFFFFu, x, o);
      if (lane >= o) x += y;
    }
    uint32_t next = first + x - c;
#pragma unroll
    for (int i = 0; i < 8; i++)
      if (L[i] == (uint32_t)l) v[i] = ((uint32_t)l << 16) | next++;
    prev_count = __shfl_sync(0xFFFFFFFFu, x, 31);
  }
#pragma unroll
  for (int i = 0; i < 8; i++) enc[lane * 8 + i] = v[i];
}

// Code choice for one (chunk, entropy stream) whose histogram is in sm.f[0..A) and
// which has at least one non-zero symbol; all threads of the block (kHuffWarps warps).
// With a plan ("NeuralZip: Reusable Setup for Fast Lossless Compression", abstract): a
// group is eligible when its code has a length for every symbol the chunk uses; the
// eligible group with the fewest coded bits wins (ties to the smaller group). With the
// plan's packed exponents (pack_hist: the chunk's 256 pair-symbol counts, pack_esc its
// escaped exponents; NULL when the chunk cannot take them) each group's packed code is a
// candidate too, at the pairs' code bits plus 8 a escape, and wins only with strictly
// fewer bits. Without an eligible candidate, or without a plan, the chunk gets its own
// limited Huffman code. The payload is HUFF (PACK) when strictly smaller than RAW. Thread
// 0 writes *mode, *code and *size; enc_out receives len << 16 | code for every symbol of
// the chosen code when the result is HUFF or PACK.
__device__ inline void decide_code(HuffBlockSmem& sm, int A, int w, uint32_t rec, uint64_t m, uint32_t S,
                                   const PlanDev& plan, uint32_t e, uint32_t* enc_out, uint32_t* mode,
                                   uint32_t* code, uint64_t* size, const uint32_t* pack_hist = nullptr,
                                   uint32_t pack_esc = 0) {
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  int group = -1;  // 0..G-1 plain group codes, G..2G-1 packed ones
  uint64_t bits = 0;
  const uint32_t G = plan.groups, cand = pack_hist ? 2 * G : G;
  if (G) {
    for (uint32_t gi = warp; gi < cand; gi += kHuffWarps) {
      const bool packed = gi >= G;
      const uint8_t* lg = packed ? plan.pack_lens + (uint64_t)(gi - G) * 256
                                 : plan.lens + ((uint64_t)e * G + gi) * 256;
      uint64_t cost = 0;
      bool ok = true;
      for (int s = lane; s < (packed ? 256 : A); s += 32) {
        const uint64_t f = packed ? (uint64_t)__ldcg(pack_hist + s) : sm.f[s];
        if (f) {
          ok = ok && lg[s] != 0;
          cost += f * lg[s];
        }
      }
      for (int o = 16; o; o >>= 1) cost += __shfl_xor_sync(0xFFFFFFFFu, cost, o);
      const bool all = __all_sync(0xFFFFFFFFu, ok);
      if (lane == 0) {
        sm.cost[gi] = cost + (packed ? 8ull * pack_esc : 0ull);
        sm.elig[gi] = all;
      }
    }
    __syncthreads();
    if (tid == 0) {
      int best = -1;
      for (uint32_t gi = 0; gi < cand; gi++)
        if (sm.elig[gi] && (best < 0 || sm.cost[gi] < sm.cost[best])) best = (int)gi;
      sm.pick = best;
    }
    __syncthreads();
    group = sm.pick;
    if (group >= 0) bits = sm.cost[group];
  }
  const uint8_t* lens = nullptr;
  if (group < 0) {
    const int wbest = block_limited_lengths(sm, A);
    lens = sm.w[wbest].lens;
    uint64_t part = tid < A ? sm.f[tid] * lens[tid] : 0;
    for (int o = 16; o; o >>= 1) part += __shfl_xor_sync(0xFFFFFFFFu, part, o);
    if (lane == 0) sm.red[warp] = part;
    __syncthreads();
    bits = 0;
    for (int i = 0; i < kHuffWarps; i++) bits += sm.red[i];
  }
  const bool packed = group >= (int)G;
  const uint64_t nsub = ceil_div(m, S);
  const uint64_t p_huff = (group < 0 ? rec : 0) + round16(4 * nsub) + round16(ceil_div(bits, 8));
  const uint64_t p_raw = raw_payload(m, w);
  if (p_huff < p_raw) {
    if (packed) {
      enc_out[tid] = plan.pack_enc[(uint64_t)(group - (int)G) * 256 + tid];
    } else if (group >= 0) {
      enc_out[tid] = plan.enc[((uint64_t)e * G + group) * 256 + tid];
    } else if (warp == 0) {
      warp_canonical(lens, enc_out);
    }
    if (tid == 0) {
      *mode = packed ? kModePack : kModeHuff;
      // packed codes exist for BF16 only (one entropy stream): group g's packed record
      // follows the G plain ones, record G + g, which is the candidate index
      *code = packed ? (uint32_t)group : group >= 0 ? e * G + (uint32_t)group : kNoCode;
      *size = p_huff;
    }
  } else if (tid == 0) {
    *mode = kModeRaw;
    *code = kNoCode;
    *size = p_raw;
  }
}

}  // namespace zipnn

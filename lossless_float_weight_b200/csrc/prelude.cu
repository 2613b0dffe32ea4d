// prelude.cu -- the compress steps before encoding:
//   k_split_hist_bf16 (BF16) / k_split_hist_tiles (FP32, FP8, FP4): byte-plane split +
//                    order-0 histogram per chunk (per-lane shared-memory counters) +
//                    all-zero detection per chunk stream, in persistent blocks; in a
//                    compress also the counts of each encode tile (and the zero-run
//                    block bitmaps of the byte planes);
//   k_build_chunks : one block per chunk after the histogram pass: per entropy stream a
//                    shared group code or a local length-limited Huffman code, then
//                    HUFF / RAW / ZERO (ZRUN for byte planes), and the tiles' bit offsets
//                    from their counts;
//   k_layout       : exclusive scan of payload sizes (single-pass decoupled look-back)
//                    into payload offsets; writes header, chunk table, shared records.
#include <atomic>

#include "bulk.cuh"
#include "common.cuh"
#include "fields.cuh"
#include "huffman.cuh"
#include "launch.h"

namespace zipnn {

constexpr int kHistThreads = 256;
constexpr uint32_t kHistSlice = 32768;  // values of one chunk per histogram tile
static_assert(kHistSlice == kBf16TileValues, "a histogram slice is one encode tile");

// BF16 and FP32 with a HUFF exponent stream: the bit offset of each encode tile in the chunk's
// bitstream, the running sum over the lower tiles of count(tile, e) * len(e), from the
// per-tile counts of the histogram pass. Warp w totals tiles w, w + 8, ...; a block
// scan turns the totals into offsets. The code builder's scratch is free by now.
__device__ void tile_offsets(const Geo& g, const Ws& ws, uint32_t c, const uint32_t* enc, HuffBlockSmem& sm) {
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const uint32_t T = g.tiles_per_chunk;
  const uint64_t m = min64(g.m0, g.n - (uint64_t)c * g.m0);
  uint8_t* lens = reinterpret_cast<uint8_t*>(sm.w[0].lens);
  uint32_t* tbits = reinterpret_cast<uint32_t*>(&sm.w[1]);  // T words: T <= 8192 fits 7 scratches
  static_assert(sizeof(HuffScratch) * (kHuffWarps - 1) >= 8192 * 4, "tile totals fit the builder scratch");
  lens[tid] = (uint8_t)(__ldcg(enc + tid) >> 16);
  __syncthreads();
  uint32_t L[8];
#pragma unroll
  for (int i = 0; i < 8; i++) L[i] = lens[lane * 8 + i];
  for (uint32_t t = warp; t < T; t += kHuffWarps) {
    uint32_t part = 0;
    if ((uint64_t)t * kBf16TileValues < m) {
      const uint4 q = __ldcg(reinterpret_cast<const uint4*>(ws.tile_hist + ((uint64_t)c * T + t) * 256) + lane);
      const uint32_t x[4] = {q.x, q.y, q.z, q.w};
#pragma unroll
      for (int i = 0; i < 8; i++) part += ((x[i >> 1] >> (16 * (i & 1))) & 0xFFFFu) * L[i];
    }
    part = __reduce_add_sync(0xFFFFFFFFu, part);
    if (lane == 0) tbits[t] = part;
  }
  __syncthreads();
  uint32_t carry = 0;
  for (uint32_t base = 0; base < T; base += kHuffWarps * 32) {
    const uint32_t t = base + tid;
    uint32_t total;
    const uint32_t before = block_exclusive_scan<kHuffWarps * 32>(t < T ? tbits[t] : 0u, sm.red32, total);
    if (t < T) ws.tile_off[(uint64_t)c * T + t] = carry + before;
    carry += total;
  }
}

// Byte plane s of chunk c (thread 0): ZERO when every byte is 0; else ZRUN when its
// payload (the block bitmap, then the bytes of the blocks that hold a non-zero byte) is
// strictly smaller than RAW; else RAW. kept = 32 x marked blocks (counted by the
// histogram pass), less what the chunk's short last block lacks when it is marked.
template <int DT>
__device__ void decide_byte_plane(const Geo& g, const Ws& ws, uint32_t c, int s) {
  constexpr int NS = n_streams(DT);
  if (threadIdx.x != 0) return;
  const uint32_t k = c * NS + s;
  const uint64_t m = min64(g.m0, g.n - (uint64_t)c * g.m0);
  const uint64_t plane = (uint64_t)c * n_byte_planes(DT) + (s - 1);
  const uint32_t* map = ws.zmap + plane * g.zwords;
  const uint64_t last = (m - 1) / kZBlock;
  uint64_t kept = (uint64_t)__ldcg(ws.zcount + plane) * kZBlock;
  if ((m % kZBlock) && ((__ldcg(map + last / 32) >> (last % 32)) & 1u)) kept -= kZBlock - m % kZBlock;
  const uint64_t raw = raw_payload(m, 8), zrun = zrun_payload(m, kept);
  const bool zero = __ldcg(ws.nonzero + k) == 0;
  ws.emode[k] = zero ? kModeZero : zrun < raw ? kModeZrun : kModeRaw;
  ws.ecode[k] = kNoCode;
  ws.esize[k] = zero ? 0 : zrun < raw ? zrun : raw;
}

// Per (chunk, entropy stream), one block of kHuffWarps warps: ZERO when every symbol is
// 0, else the code choice of decide_code.
template <int DT>
__device__ void build_chunk_table(const Geo& g, const Ws& ws, const PlanDev& plan, uint32_t c, uint32_t e,
                                  HuffBlockSmem& sm) {
  constexpr int NS = n_streams(DT), NE = n_entropy(DT);
  const int tid = threadIdx.x;
  const uint32_t k = c * NS + e;
  const uint64_t clo = (uint64_t)c * g.m0;
  const uint64_t m = min64(g.m0, g.n - clo);
  const int A = alphabet(DT, e), w = raw_width(DT, e);
  if (__ldcg(ws.nonzero + k) == 0) {
    if (tid == 0) {
      ws.emode[k] = kModeZero;
      ws.ecode[k] = kNoCode;
      ws.esize[k] = 0;
    }
    return;
  }
  const uint32_t* h = ws.hist + ((uint64_t)c * NE + e) * 256;
  sm.f[tid] = tid < A ? __ldcg(h + tid) : 0;
  __syncthreads();
  uint32_t* enc = ws.enc + ((uint64_t)c * NE + e) * 256;
  // packed exponents: BF16 exponent stream of a chunk of whole pairs
  const bool pack = DT == kBF16 && e == 0 && plan.pack_k && ws.pack_hist && m % 2 == 0;
  decide_code(sm, A, w, record_bytes(DT, e), m, g.S, plan, e, enc, ws.emode + k, ws.ecode + k, ws.esize + k,
              pack ? ws.pack_hist + (uint64_t)c * 256 : nullptr, pack ? __ldcg(ws.pack_esc + c) : 0u);
  if constexpr (DT == kBF16 || DT == kFP32) {
    if (ws.tile_off) {
      __syncthreads();
      if (ws.emode[k] == kModeHuff) tile_offsets(g, ws, c, enc, sm);
    }
  }
}

// FP8 and FP4, each entropy stream with a HUFF code: the bit offset of every encode tile
// of chunk c in the stream's bitstream, the running sum over the lower tiles of
// sum over the joint bins (e, m) of count(tile, e, m) * len(the stream's symbol of the
// bin). The tiles' joint counts are complete: this is the chunk's last histogram block.
template <int DT>
__device__ void joint_tile_offsets(const Geo& g, const Ws& ws, uint32_t c, HuffBlockSmem& hs) {
  constexpr int NS = n_streams(DT), A0 = alphabet(DT, 0), A1 = alphabet(DT, 1), AJ = A0 * A1;
  static_assert(AJ == (int)tile_bins(DT), "one counter a joint bin");
  const int tid = threadIdx.x;
  const uint32_t T = g.tiles_per_chunk;
#pragma unroll
  for (int e = 0; e < 2; e++) {
    if (ws.emode[(uint64_t)c * NS + e] != kModeHuff) continue;  // uniform
    constexpr int AMAX = A0 > A1 ? A0 : A1;
    uint32_t L[AMAX];
#pragma unroll
    for (int a = 0; a < AMAX; a++) L[a] = a < (e == 0 ? A0 : A1) ? ws.enc[((uint64_t)c * 2 + e) * 256 + a] >> 16 : 0u;
    uint32_t carry = 0;
    for (uint32_t base = 0; base < T; base += kHistThreads) {
      const uint32_t t = base + tid;
      uint32_t bits = 0;
      if (t < T) {
        const uint16_t* h = ws.tile_hist + ((uint64_t)c * T + t) * AJ;
#pragma unroll
        for (int b = 0; b < AJ; b++) bits += (uint32_t)__ldcg(h + b) * L[e == 0 ? b / A1 : b % A1];
      }
      uint32_t total;
      const uint32_t before = block_exclusive_scan<kHistThreads>(bits, hs.red32, total);
      if (t < T) ws.tile_off[(uint64_t)e * g.n_tiles + (uint64_t)c * T + t] = carry + before;
      carry += total;
    }
  }
}

// ---------------------------------------------------------------- BF16 histogram
// k_split_hist_bf16: the histogram pass of BF16, with loads that stay in flight.
// Blocks are persistent: each takes tiles (32768-value slices of a chunk) blockIdx.x,
// blockIdx.x + gridDim.x, ... Thread 0 streams the block's tiles, 16 KB pieces in
// order, through a ring of kHbStages shared-memory buffers with bulk copies, so up to
// kHbStages pieces are on their way while the block counts and sums columns. The code
// builds, latency-bound, are a kernel of their own (k_build_chunks) that follows.
// The counters are those of k_split_hist (one per exponent and lane), taking both
// halves of a word at a time; each tile's column sums are also its encode-tile counts.
// Thread t takes the 16-byte units t, t + 256, ... of a piece, so a warp's shared
// loads are conflict-free. Only the tensor's last piece can end in fewer than 8 values
// (chunks are whole multiples of 16 bytes); thread 0 loads those itself.
constexpr int kHbStages = 4;
constexpr uint32_t kHbPieceValues = 8192;  // 16 KB
constexpr size_t kHbRegion = 256 * 32 * 4;  // the counters
constexpr size_t kHbZbits = 32 * 4;         // the tile's zero-run bitmap: 1024 blocks
constexpr size_t kHbSmemBytes = kHbRegion + (size_t)kHbStages * kHbPieceValues * 2 + kHbStages * 8 + kHbZbits;
constexpr uint32_t kHbWaitLimit = 1u << 26;

// Values of tile `tile` (0 past the end of a ragged last chunk) and its first value.
__device__ __forceinline__ uint32_t hb_tile_values(const Geo& g, uint32_t tile, uint64_t& vlo) {
  const uint32_t c = tile / g.tiles_per_chunk, ti = tile - c * g.tiles_per_chunk;
  const uint64_t clo = (uint64_t)c * g.m0;
  const uint32_t m = (uint32_t)min64(g.m0, g.n - clo), lo = ti * kHistSlice;
  vlo = clo + lo;
  return lo < m ? min32(kHistSlice, m - lo) : 0u;
}

__global__ void __launch_bounds__(kHistThreads) k_split_hist_bf16(const uint8_t* __restrict__ src, Geo g,
                                                                  uint32_t* __restrict__ hist,
                                                                  uint32_t* __restrict__ nonzero, Ws ws) {
  extern __shared__ __align__(16) uint8_t smem_raw[];  // table, stages, barriers
  uint32_t* const sh = reinterpret_cast<uint32_t*>(smem_raw);
  uint8_t* const stages = smem_raw + kHbRegion;
  uint64_t* const bar = reinterpret_cast<uint64_t*>(stages + (size_t)kHbStages * kHbPieceValues * 2);
  uint32_t* const zbits = reinterpret_cast<uint32_t*>(bar + kHbStages);
  const int tid = threadIdx.x, lane = tid & 31;
  const uint32_t T = g.tiles_per_chunk;
  for (int i = tid; i < 256 * 32; i += kHistThreads) sh[i] = 0;
  if (tid < 32) zbits[tid] = 0;
  if (tid == 0)
    for (int s = 0; s < kHbStages; s++) mbar_init(bar + s, 1);
  __syncthreads();

  // thread 0's cursor: the next piece to load
  uint32_t p_tile = blockIdx.x, p_piece = 0;
  auto issue = [&](int s) {
    for (; p_tile < g.n_tiles; p_tile += gridDim.x, p_piece = 0) {
      uint64_t vlo;
      const uint32_t nv = hb_tile_values(g, p_tile, vlo);
      if (p_piece * kHbPieceValues >= nv) continue;
      const uint32_t bytes = (min32(kHbPieceValues, nv - p_piece * kHbPieceValues) & ~7u) * 2;
      fence_proxy_async_smem();  // the stage's earlier reads come first
      mbar_expect_tx(bar + s, bytes);
      if (bytes)
        bulk_g2s(stages + (size_t)s * kHbPieceValues * 2, src + (vlo + (uint64_t)p_piece * kHbPieceValues) * 2, bytes,
                 bar + s);
      p_piece++;
      return;
    }
  };
  if (tid == 0)
    for (int s = 0; s < kHbStages; s++) issue(s);

  // counter of exponent e for this lane: byte (e << 7) | (lane << 2) of the table, one
  // LOP3 from the value's word (the exponent field is bits 14..7 of the low value)
  uint8_t* const tab = reinterpret_cast<uint8_t*>(sh);
  const uint32_t l4 = (uint32_t)lane << 2;
  uint8_t* const zbytes = reinterpret_cast<uint8_t*>(zbits);
  const int warp = tid >> 5;
  constexpr int kUnits = (int)(kHbPieceValues / 8 / kHistThreads);  // 16-byte units a thread takes per piece
  uint32_t q = 0;  // pieces consumed
  for (uint32_t tile = blockIdx.x; tile < g.n_tiles; tile += gridDim.x) {
    uint64_t vlo;
    const uint32_t nv = hb_tile_values(g, tile, vlo);
    if (nv == 0) continue;  // uniform
    const uint32_t c = tile / T, sl = tile - c * T;
    uint32_t nzall = 0;   // OR of every word I counted
    uint32_t tail_nz = 0; // thread 0: OR of the sign/fraction bits of the tile's last < 8 values
    for (uint32_t p0 = 0; p0 < nv; p0 += kHbPieceValues, q++) {
      const int s = (int)(q % kHbStages);
      if (!mbar_wait_bounded(bar + s, (q / kHbStages) & 1u, kHbWaitLimit) && ws.status) set_status(ws.status, kStTimeout);
      const uint32_t pv = min32(kHbPieceValues, nv - p0), nb = pv & ~7u;
      const uint4* st4 = reinterpret_cast<const uint4*>(stages + (size_t)s * kHbPieceValues * 2);
      uint32_t my4 = 0;  // bit k: my unit of iteration k holds a non-zero sign/fraction byte
#pragma unroll
      for (int k = 0; k < kUnits; k++) {
        const uint32_t i = (uint32_t)(k * kHistThreads + tid);
        if (i * 8 < nb) {
          const uint4 v = st4[i];
          const uint32_t x[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
          for (int j = 0; j < 4; j++) {
            atomicAdd(reinterpret_cast<uint32_t*>(tab + ((x[j] & 0x7F80u) | l4)), 1u);
            atomicAdd(reinterpret_cast<uint32_t*>(tab + (((x[j] >> 16) & 0x7F80u) | l4)), 1u);
          }
          const uint32_t o = v.x | v.y | v.z | v.w;
          nzall |= o;
          my4 |= ((o & 0x807F807Fu) != 0 ? 1u : 0u) << k;
        }
      }
      // zero-run blocks (32 values: four units, four lanes): only a warp that saw a unit
      // with no non-zero sign/fraction byte records anything. In iteration k the warp's
      // 32 units are the tile's 8 blocks 8w + 64k + piece offset: a ballot of the zero
      // units, each nibble folded onto one bit (its four lanes all zero), the 8 bits
      // gathered into the byte of those blocks (a byte no other warp or iteration writes).
      if (ws.zmap && !__all_sync(0xFFFFFFFFu, my4 == (1u << kUnits) - 1u)) {
#pragma unroll
        for (int k = 0; k < kUnits; k++) {
          uint32_t b = __ballot_sync(0xFFFFFFFFu, ((my4 >> k) & 1u) == 0);
          b &= b >> 1;
          b &= b >> 2;
          b &= 0x11111111u;  // bit 4j: block j of the eight is all zero
          b = (b | (b >> 3)) & 0x03030303u;
          b = (b | (b >> 6)) & 0x000F000Fu;
          b = (b | (b >> 12)) & 0xFFu;
          if (lane == k) zbytes[p0 / (kZBlock * 8) + (uint32_t)(8 * k + warp)] = (uint8_t)b;
        }
      }
      if (tid == 0 && nb < pv) {
        const uint16_t* t = reinterpret_cast<const uint16_t*>(src) + vlo + p0 + nb;
        for (uint32_t i = 0; i < pv - nb; i++) {
          const uint32_t v = t[i];
          atomicAdd(reinterpret_cast<uint32_t*>(tab + ((v & 0x7F80u) | l4)), 1u);
          nzall |= v;
          tail_nz |= v & 0x807Fu;
        }
      }
      __syncthreads();  // stage s is read, and the tile's counts are complete after the last piece
      if (tid == 0) issue(s);
    }
    const uint32_t nz0 = __reduce_or_sync(0xFFFFFFFFu, nzall & 0x7F807F80u);
    const uint32_t nz1 = __reduce_or_sync(0xFFFFFFFFu, nzall & 0x807F807Fu);
    if (nonzero && lane == 0) {
      if (nz0) atomicOr(&nonzero[(uint64_t)c * 2], nz0);
      if (nz1) atomicOr(&nonzero[(uint64_t)c * 2 + 1], nz1);
    }
    // row b (exponent b): thread b sums it (eight 16-byte loads, rotated so that the
    // eight lanes of a quarter warp take eight different bank groups) and clears it
    {
      const int b = tid;
      uint4* row = reinterpret_cast<uint4*>(sh + b * 32);
      uint32_t sum = 0;
#pragma unroll
      for (int j = 0; j < 8; j++) {
        const int gi = (j + b) & 7;
        const uint4 v = row[gi];
        sum += v.x + v.y + v.z + v.w;
        row[gi] = make_uint4(0u, 0u, 0u, 0u);
      }
      if (sum) atomicAdd(&hist[(uint64_t)c * 256 + b], sum);
      if (ws.tile_hist) ws.tile_hist[((uint64_t)c * T + sl) * 256 + b] = (uint16_t)sum;
    }
    if (ws.zmap) {
      // the tile's last values (under 8, the tensor's end): a non-zero sign/fraction
      // byte there marks their block, whatever its earlier units held
      if (nv & 7u) {
        if (tid == 0 && tail_nz) {
          const uint32_t blk = (nv - 1) / kZBlock;
          zbytes[blk / 8] &= (uint8_t)~(1u << (blk % 8));
        }
        __syncthreads();
      }
      if (tid < 32) {
        // the tile's 32 bitmap words go out as plain stores: a block is marked when it
        // lies in the tile and is not all zero; the marked count goes into the chunk's
        const uint32_t nvb = ceil_div(nv, kZBlock), lo = (uint32_t)tid * 32u;
        const uint32_t valid = lo >= nvb ? 0u : nvb - lo >= 32u ? 0xFFFFFFFFu : (1u << (nvb - lo)) - 1u;
        const uint32_t word = ~zbits[tid] & valid, wi = sl * 32u + (uint32_t)tid;
        if (wi < g.zwords) ws.zmap[(uint64_t)c * g.zwords + wi] = word;
        const uint32_t marked = __reduce_add_sync(0xFFFFFFFFu, __popc(word));
        if (tid == 0 && marked) atomicAdd(ws.zcount + c, marked);
        zbits[tid] = 0;
      }
    }
    __syncthreads();  // every row and bitmap word is clear before the next tile's counts
  }
}

// FP32, FP8 and FP4 (BF16 has k_split_hist_bf16 below). THEORY-599 note, "Order-0 only
// (section III-A b)": the model of a chunk is the count of each symbol. The block keeps one
// counter per (symbol, lane) in shared memory, so the 32 lanes of a warp always add into
// 32 different banks (lane l owns column l); warps share the table through shared
// atomics, and a tile's column sums also clear it for the next tile. FP8 and FP4 count the
// joint (exponent, mantissa) bin, exponent * mantissa alphabet + mantissa, so one atomic
// counts both entropy streams (FP4 one atomic per byte, for its pair of joint bins).
// Blocks are persistent (each takes tiles blockIdx.x, blockIdx.x + gridDim.x, ...; a tile
// is one 32768-value slice of a chunk) and write the chunks' histograms and all-zero
// flags; in a compress (ws set) also each tile's counts (its encode-tile counts: FP32 the
// exponents, FP8/FP4 the joint bins) and FP32's zero-run block bits of the three fraction
// planes with each tile's marked count. The code builds follow in k_build_chunks, so no
// block waits on another and none stalls its stream of tiles on a build.
template <int DT>
__global__ void __launch_bounds__(kHistThreads, 3) k_split_hist_tiles(const uint8_t* __restrict__ src, Geo g,
                                                                     uint32_t* __restrict__ hist,
                                                                     uint32_t* __restrict__ nonzero, Ws ws) {
  constexpr bool F32 = DT == kFP32;
  constexpr int NS = n_streams(DT), NE = n_entropy(DT);
  constexpr int A0 = alphabet(DT, 0), A1 = NE > 1 ? alphabet(DT, 1) : 1, AJ = A0 * A1;
  constexpr int AC = DT == kFP4 ? AJ * AJ : AJ;
  // values a thread per pass: FP32 32 (one zero-run block), FP8 64, FP4 128 (64 bytes)
  constexpr int NV = F32 ? 32 : DT == kFP8 ? 64 : 128;
  extern __shared__ __align__(16) uint8_t smem_raw[];
  uint32_t* sh = reinterpret_cast<uint32_t*>(smem_raw);
  uint32_t* csum = sh + AC * 32;
  uint32_t* joint = csum + (AC > AJ ? AC : 0);
  uint8_t* const tab = reinterpret_cast<uint8_t*>(sh);
  __shared__ uint32_t s_zbits[3][32];  // FP32: the tile's zero-run block bits of each fraction plane
  const int tid = threadIdx.x, lane = tid & 31;
  const uint32_t l4 = (uint32_t)lane << 2;
  for (int i = tid; i < AC * 32; i += kHistThreads) sh[i] = 0;
  if (tid < 96) s_zbits[tid / 32][tid % 32] = 0;
  __syncthreads();
  const uint32_t T = g.tiles_per_chunk;
  for (uint32_t tile = blockIdx.x; tile < g.n_tiles; tile += gridDim.x) {
    const uint32_t c = tile / T, sl = tile - c * T;
    const uint64_t clo = (uint64_t)c * g.m0;
    const uint32_t m = (uint32_t)min64(g.m0, g.n - clo);
    const uint32_t lo = sl * kHistSlice, hi = min(lo + kHistSlice, m);
    if (lo >= m) continue;  // past the end of a ragged last chunk (uniform)
    uint32_t nzw = 0;  // OR of my words
    for (uint32_t t0 = lo; t0 < hi; t0 += kHistThreads * NV) {
      const uint32_t v0 = t0 + tid * NV;
      const int cnt = v0 < hi ? (int)min32(NV, hi - v0) : 0;
      if (cnt == 0) continue;
      RawValues<DT, NV> raw;
      const uint8_t* vp = src + value_offset(DT, clo + v0);
      constexpr int W = RawValues<DT, NV>::kWords;
      if (cnt == NV && (reinterpret_cast<uintptr_t>(vp) & 31) == 0) {
#pragma unroll
        for (int j = 0; j < W / 8; j++) ld_nc_v8(vp + 32 * j, raw.w + 8 * j);
      } else {
        load_values<DT, NV>(vp, cnt, raw);  // zero past cnt
      }
      if constexpr (F32) {
        // counter (exponent, lane) at byte exponent << 7 | lane << 2: bits 30..23 of the
        // value moved to 14..7; my 32 values are one zero-run block of every fraction plane
        uint32_t a = 0;
        if (cnt == NV) {  // a whole pass: no test per value
#pragma unroll
          for (int j = 0; j < NV; j++) {
            atomicAdd(reinterpret_cast<uint32_t*>(tab + (((raw.w[j] >> 16) & 0x7F80u) | l4)), 1u);
            a |= raw.w[j];
          }
        } else {
#pragma unroll
          for (int j = 0; j < NV; j++) {
            if (j < cnt) atomicAdd(reinterpret_cast<uint32_t*>(tab + (((raw.w[j] >> 16) & 0x7F80u) | l4)), 1u);
            a |= raw.w[j];
          }
        }
        nzw |= a;
        const uint32_t blk = (v0 - lo) / kZBlock;  // within the tile
        RawValues<DT, NV> o;
        o.w[0] = a;
#pragma unroll
        for (int s = 1; s < 4; s++)
          if (symbol<DT, NV>(o, s, 0)) atomicOr(&s_zbits[s - 1][blk / 32], 1u << (blk % 32));
      } else {
        // counter (bin, lane) at byte bin << 7 | lane << 2: FP8 bin = byte & 0x7F; FP4 bin =
        // (low nibble & 7) | (high nibble & 7) << 3
        const int nbytes = DT == kFP8 ? cnt : cnt / 2;  // FP4: cnt is even
        auto count_word = [&](uint32_t x, int k0, bool all) {
#pragma unroll
          for (int k = 0; k < 4; k++) {
            if (all || k0 + k < nbytes) {
              uint32_t off;
              if constexpr (DT == kFP8) {
                off = k == 0 ? (x << 7) & 0x3F80u : (x >> (8 * k - 7)) & 0x3F80u;
              } else {
                const uint32_t b = x >> (8 * k);
                off = ((b << 7) & 0x380u) | ((b << 6) & 0x1C00u);
              }
              atomicAdd(reinterpret_cast<uint32_t*>(tab + (off | l4)), 1u);
            }
          }
        };
        if (cnt == NV) {  // a whole pass: no test per byte
#pragma unroll
          for (int j = 0; j < W; j++) {
            nzw |= raw.w[j];
            count_word(raw.w[j], 4 * j, true);
          }
        } else {
#pragma unroll
          for (int j = 0; j < W; j++) {
            nzw |= raw.w[j];
            count_word(raw.w[j], 4 * j, false);
          }
        }
      }
    }
    // all-zero flags: every stream is a bit field, so the OR of the words (FP8/FP4 folded
    // onto the first value's bits) holds the OR of each stream's symbols
    {
      uint32_t x = __reduce_or_sync(0xFFFFFFFFu, nzw);
      if constexpr (!F32) {
        x |= x >> 16;
        x |= x >> 8;
        if constexpr (DT == kFP4) x |= x >> 4;
      }
      RawValues<DT, NV> o;
      o.w[0] = x;
      if (nonzero && lane == 0) {
#pragma unroll
        for (int s = 0; s < NS; s++) {
          const uint32_t v = symbol<DT, NV>(o, s, 0);
          if (v) atomicOr(&nonzero[(uint64_t)c * NS + s], v);
        }
      }
    }
    __syncthreads();  // the tile's counts and bitmaps are complete
    {
      // column sums: TPB threads a bin (FP4 4, FP8 2, FP32 1: every thread one share of
      // 32 / TPB lanes), joined by shuffles between neighbouring lanes; the rotation by the
      // bin keeps a warp's loads on 32 different banks
      constexpr int TPB = kHistThreads / AC >= 1 ? kHistThreads / AC : 1;
      static_assert(AC * TPB == kHistThreads, "one share a thread");
      const int b = tid / TPB, part = tid % TPB;
      uint32_t sum = 0;
#pragma unroll 8
      for (int i = 0; i < 32 / TPB; i++) {
        const int a = b * 32 + ((part * (32 / TPB) + i + b) & 31);
        sum += sh[a];
        sh[a] = 0;
      }
#pragma unroll
      for (int o = 1; o < TPB; o <<= 1) sum += __shfl_xor_sync(0xFFFFFFFFu, sum, o);
      if (part == 0) csum[b] = sum;
    }
    if constexpr (F32) {
      if (ws.zmap && tid < 96) {
        // the tile's bitmap words of each plane (plain stores; no other tile holds them),
        // their marked blocks into the chunk's count; then cleared
        const int p = tid / 32, wl = tid % 32;
        const uint32_t word = s_zbits[p][wl], wi = sl * 32u + (uint32_t)wl;
        if (wi < g.zwords) ws.zmap[((uint64_t)c * 3 + p) * g.zwords + wi] = word;
        const uint32_t marked = __reduce_add_sync(0xFFFFFFFFu, __popc(word));
        if (wl == 0 && marked) atomicAdd(ws.zcount + (uint64_t)c * 3 + p, marked);
        s_zbits[p][wl] = 0;
      }
    }
    __syncthreads();
    if constexpr (AC > AJ) {
      // FP4: bin x counts the pairs with x first plus the pairs with x second
      for (int x = tid; x < AJ; x += kHistThreads) {
        uint32_t sum = 0;
        for (int y = 0; y < AJ; y++) sum += csum[x | (y << 3)] + csum[y | (x << 3)];
        joint[x] = sum;
      }
      __syncthreads();
    }
    if (ws.tile_hist)
      for (int b = tid; b < AJ; b += kHistThreads) ws.tile_hist[(uint64_t)tile * AJ + b] = (uint16_t)joint[b];
    if constexpr (F32) {
      for (int b = tid; b < A0; b += kHistThreads)
        if (joint[b]) atomicAdd(&hist[(uint64_t)c * 256 + b], joint[b]);
    } else {
      for (int t = tid; t < A0 + A1; t += kHistThreads) {
        uint32_t sum = 0;
        if (t < A0) {
          for (int j = 0; j < A1; j++) sum += joint[t * A1 + j];
        } else {
          for (int e = 0; e < A0; e++) sum += joint[e * A1 + (t - A0)];
        }
        if (sum) atomicAdd(&hist[((uint64_t)c * 2 + (t < A0 ? 0 : 1)) * 256 + (t < A0 ? t : t - A0)], sum);
      }
    }
    __syncthreads();  // the sums are read before the next tile's fold writes them
  }
}

// One block per chunk (compress): the chunk's code choice
// (build_chunk_table) for each entropy stream and the tiles' bit offsets, once the
// histogram pass is complete.
template <int DT>
__global__ void __launch_bounds__(kHuffWarps * 32, 4) k_build_chunks(Geo g, Ws ws, PlanDev plan) {
  extern __shared__ __align__(16) uint8_t smem_raw[];
  HuffBlockSmem& hs = *reinterpret_cast<HuffBlockSmem*>(smem_raw);
#pragma unroll
  for (int e = 0; e < n_entropy(DT); e++) {
    build_chunk_table<DT>(g, ws, plan, blockIdx.x, (uint32_t)e, hs);
    __syncthreads();
  }
  if constexpr (n_entropy(DT) > 1) {
    if (ws.tile_off) joint_tile_offsets<DT>(g, ws, blockIdx.x, hs);
  }
#pragma unroll
  for (int s = 0; s < n_streams(DT); s++)
    if (is_byte_plane(DT, s)) decide_byte_plane<DT>(g, ws, blockIdx.x, s);
}

// Stand-alone code lengths for `count` histograms (u64 x 256 each); also used by the
// plan for its group codes. Optionally writes canonical code values.
__global__ void __launch_bounds__(kHuffWarps * 32) k_code_lengths(const uint64_t* __restrict__ hist, uint32_t alphabet_size,
                                                                 uint8_t* __restrict__ lens_out, uint32_t* __restrict__ enc_out) {
  extern __shared__ __align__(16) uint8_t smem_raw[];
  HuffBlockSmem& sm = *reinterpret_cast<HuffBlockSmem*>(smem_raw);
  const int tid = threadIdx.x, warp = tid >> 5;
  const uint64_t* h = hist + (uint64_t)blockIdx.x * 256;
  sm.f[tid] = tid < (int)alphabet_size ? h[tid] : 0;
  __syncthreads();
  const int wbest = block_limited_lengths(sm, (int)alphabet_size);
  const uint8_t* lens = sm.w[wbest].lens;
  lens_out[(uint64_t)blockIdx.x * 256 + tid] = lens[tid];
  if (enc_out && warp == 0) warp_canonical(lens, enc_out + (uint64_t)blockIdx.x * 256);
}

constexpr int kLayoutThreads = 256, kLayoutPer = 4, kLayoutTile = kLayoutThreads * kLayoutPer;

// Block-wide exclusive scan of 64-bit values (blockDim = kLayoutThreads).
__device__ inline uint64_t block_scan_u64(uint64_t v, uint64_t* s_warp, uint64_t& total) {
  constexpr int NW = kLayoutThreads / 32;
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  uint64_t x = v;
  for (int o = 1; o < 32; o <<= 1) {
    const uint64_t y = __shfl_up_sync(0xFFFFFFFFu, x, o);
    if (lane >= o) x += y;
  }
  if (lane == 31) s_warp[warp] = x;
  __syncthreads();
  uint64_t before = 0;
  for (int i = 0; i < warp; i++) before += s_warp[i];
  total = 0;
  for (int i = 0; i < NW; i++) total += s_warp[i];
  __syncthreads();
  return before + x - v;
}

// Layout: payload k (entry order) starts at off_payload + sum of sizes of entries < k.
// Entropy entries take their mode and size from the code build; raw-plane entries are
// ZERO when all their symbols are 0, else RAW.
template <int DT>
__global__ void __launch_bounds__(kLayoutThreads) k_layout(Geo g, Ws ws, PlanDev plan, uint8_t* __restrict__ out) {
  constexpr int NS = n_streams(DT), NE = n_entropy(DT);
  __shared__ uint64_t s_warp[kLayoutThreads / 32];
  __shared__ uint32_t s_tile;
  __shared__ uint64_t s_prefix;
  const int tid = threadIdx.x;
  if (tid == 0) s_tile = atomicAdd(&ws.status[2], 1u);
  __syncthreads();
  const uint32_t tile = s_tile;
  const uint32_t k0 = tile * kLayoutTile + tid * kLayoutPer;
  uint64_t size[kLayoutPer];
  uint32_t mode[kLayoutPer], code[kLayoutPer];
  uint64_t mine = 0;
#pragma unroll
  for (int i = 0; i < kLayoutPer; i++) {
    const uint32_t k = k0 + i;
    size[i] = 0;
    mode[i] = kModeZero;
    code[i] = kNoCode;
    if (k < g.n_entries) {
      const uint32_t s = k % NS;
      if (is_entropy(DT, (int)s) || is_byte_plane(DT, (int)s)) {
        mode[i] = ws.emode[k];
        code[i] = ws.ecode[k];
        size[i] = ws.esize[k];
      } else {
        const uint32_t c = k / NS;
        const uint64_t m = min64(g.m0, g.n - (uint64_t)c * g.m0);
        if (ws.nonzero[k]) {
          mode[i] = kModeRaw;
          size[i] = raw_payload(m, raw_width(DT, (int)s));
        }
        ws.emode[k] = mode[i];
        ws.ecode[k] = kNoCode;
        ws.esize[k] = size[i];
      }
      mine += size[i];
    }
  }
  uint64_t total;
  uint64_t before = block_scan_u64(mine, s_warp, total);
  if (tid < 32) {
    const uint64_t p = warp_lookback(ws.scan_desc, tile, 0, total, ws.status, g.spin_limit);
    if (tid == 0) s_prefix = p;
  }
  __syncthreads();
  uint64_t pos = g.off_payload + s_prefix + before;
#pragma unroll
  for (int i = 0; i < kLayoutPer; i++) {
    const uint32_t k = k0 + i;
    if (k < g.n_entries) {
      ws.eoff[k] = pos;
      uint4 ent;
      ent.x = mode[i];
      ent.y = code[i];
      ent.z = (uint32_t)pos;
      ent.w = (uint32_t)(pos >> 32);
      *reinterpret_cast<uint4*>(out + kHeaderBytes + (uint64_t)kEntryBytes * k) = ent;
      pos += size[i];
    }
  }
  const uint32_t n_layout_tiles = (uint32_t)ceil_div(g.n_entries, kLayoutTile);
  if (tile == n_layout_tiles - 1 && tid == 0) {
    uint32_t hdr[16];
    hdr[0] = 0x314E4E5Au;  // "ZNN1"
    hdr[1] = 1u | ((uint32_t)DT << 16) | ((uint32_t)NS << 24);
    hdr[2] = (uint32_t)g.n;
    hdr[3] = (uint32_t)(g.n >> 32);
    hdr[4] = g.chunk_bytes;
    hdr[5] = g.S;
    hdr[6] = g.n_chunks;
    hdr[7] = g.n_groups * NE + (g.n_packed ? g.n_groups : 0u);
    hdr[8] = (uint32_t)g.off_codes;
    hdr[9] = (uint32_t)(g.off_codes >> 32);
    hdr[10] = (uint32_t)g.off_payload;
    hdr[11] = (uint32_t)(g.off_payload >> 32);
    const uint64_t tb = g.off_payload + s_prefix + total;
    hdr[12] = (uint32_t)tb;
    hdr[13] = (uint32_t)(tb >> 32);
    hdr[14] = (uint32_t)kLmax | (g.n_groups << 8) | (g.n_packed << 16);
    hdr[15] = 0;
    for (int i = 0; i < 4; i++)
      reinterpret_cast<uint4*>(out)[i] = make_uint4(hdr[4 * i], hdr[4 * i + 1], hdr[4 * i + 2], hdr[4 * i + 3]);
  }
  // shared code records (4-bit lengths), written by the first tile
  if (tile == 0 && plan.groups) {
    for (int e = 0; e < NE; e++) {
      const int A = alphabet(DT, e);
      const uint32_t rb = record_bytes(DT, e);
      for (uint32_t gi = 0; gi < plan.groups; gi++) {
        const uint8_t* lg = plan.lens + ((uint64_t)e * plan.groups + gi) * 256;
        uint8_t* rp = out + g.off_codes + shared_record_pos(DT, plan.groups, (uint32_t)e * plan.groups + gi);
        for (uint32_t b = tid; b < rb; b += kLayoutThreads)
          rp[b] = (int)(2 * b) < A ? (uint8_t)(lg[2 * b] | (lg[2 * b + 1] << 4)) : 0;
      }
    }
    // packed records and the list of packed exponents
    if (g.n_packed) {
      for (uint32_t gi = 0; gi < plan.groups; gi++) {
        const uint8_t* lp = plan.pack_lens + (uint64_t)gi * 256;
        uint8_t* rp = out + g.off_codes + packed_record_pos(DT, plan.groups, gi);
        for (uint32_t b = tid; b < 128; b += kLayoutThreads) rp[b] = (uint8_t)(lp[2 * b] | (lp[2 * b + 1] << 4));
      }
      if (tid < (int)kPackListBytes) out[g.off_payload - kPackListBytes + tid] = plan.pack_exps[tid];
    }
  }
}

// ---------------------------------------------------------------- launchers

// Opt a kernel into more than 48 KB of dynamic shared memory, once per device. Slots:
// 3 k_code_lengths, 8 + DT k_build_chunks<DT>.
template <typename K>
static cudaError_t allow_smem(K kernel, size_t bytes, int slot) {
  static std::atomic<int> done[12][128];
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  if (dev >= 0 && dev < 128 && done[slot][dev].load(std::memory_order_relaxed)) return cudaSuccess;
  e = cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)bytes);
  if (e == cudaSuccess && dev >= 0 && dev < 128) done[slot][dev].store(1, std::memory_order_relaxed);
  return e;
}


// BF16: a persistent grid of as many histogram blocks as fit on the device at once.
static cudaError_t split_hist_bf16(const void* src, const Geo& g, uint32_t* hist, uint32_t* nonzero, const Ws* ws,
                                   const PlanDev& plan, cudaStream_t st) {
  static std::atomic<int> resident[128];  // blocks per device, once the attributes are set
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  int per_device = dev >= 0 && dev < 128 ? resident[dev].load(std::memory_order_relaxed) : 0;
  if (!per_device) {
    e = cudaFuncSetAttribute(k_split_hist_bf16, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)kHbSmemBytes);
    int per_sm = 0, sms = 0;
    if (e == cudaSuccess)
      e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, k_split_hist_bf16, kHistThreads, kHbSmemBytes);
    if (e == cudaSuccess) e = cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    if (e != cudaSuccess) return e;
    per_device = (per_sm > 0 ? per_sm : 1) * (sms > 0 ? sms : 1);
    if (dev >= 0 && dev < 128) resident[dev].store(per_device, std::memory_order_relaxed);
  }
  Ws w{};
  if (ws) w = *ws;
  const uint32_t blocks = (uint32_t)min64((uint64_t)per_device, g.n_tiles);
  k_split_hist_bf16<<<blocks, kHistThreads, kHbSmemBytes, st>>>(static_cast<const uint8_t*>(src), g, hist, nonzero,
                                                                  w);
  return cudaGetLastError();
}

template <int DT>
static cudaError_t build_chunks_t(const Geo& g, const Ws& ws, const PlanDev& plan, cudaStream_t st) {
  const cudaError_t e = allow_smem(k_build_chunks<DT>, sizeof(HuffBlockSmem), 8 + DT);
  if (e != cudaSuccess) return e;
  k_build_chunks<DT><<<g.n_chunks, kHuffWarps * 32, sizeof(HuffBlockSmem), st>>>(g, ws, plan);
  return cudaGetLastError();
}

cudaError_t launch_build_chunks(const Geo& g, const Ws& ws, const PlanDev& plan, cudaStream_t st) {
  switch (g.dt) {
    case kBF16: return build_chunks_t<kBF16>(g, ws, plan, st);
    case kFP32: return build_chunks_t<kFP32>(g, ws, plan, st);
    case kFP8: return build_chunks_t<kFP8>(g, ws, plan, st);
    default: return build_chunks_t<kFP4>(g, ws, plan, st);
  }
}

// FP32 / FP8 / FP4: a persistent grid of as many histogram blocks as fit on the device.
template <int DT>
static cudaError_t split_hist_tiles_t(const void* src, const Geo& g, uint32_t* hist, uint32_t* nonzero, const Ws& ws,
                                      cudaStream_t st) {
  constexpr size_t AJ = (size_t)alphabet(DT, 0) * (n_entropy(DT) > 1 ? alphabet(DT, 1) : 1);
  constexpr size_t AC = DT == kFP4 ? AJ * AJ : AJ;
  constexpr size_t smem = (AC * 32 + AC + AJ) * 4;
  static std::atomic<int> resident[128];  // blocks per device, once known
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  int per_device = dev >= 0 && dev < 128 ? resident[dev].load(std::memory_order_relaxed) : 0;
  if (!per_device) {
    int per_sm = 0, sms = 0;
    e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, k_split_hist_tiles<DT>, kHistThreads, smem);
    if (e == cudaSuccess) e = cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    if (e != cudaSuccess) return e;
    per_device = (per_sm > 0 ? per_sm : 1) * (sms > 0 ? sms : 1);
    if (dev >= 0 && dev < 128) resident[dev].store(per_device, std::memory_order_relaxed);
  }
  const uint32_t blocks = (uint32_t)min64((uint64_t)per_device, g.n_tiles);
  static_assert(smem <= 48 * 1024, "the default dynamic shared memory suffices");
  k_split_hist_tiles<DT><<<blocks, kHistThreads, smem, st>>>(static_cast<const uint8_t*>(src), g, hist, nonzero, ws);
  return cudaGetLastError();
}

cudaError_t launch_split_hist(const void* src, const Geo& g, uint32_t* hist, uint32_t* nonzero, const Ws* ws,
                              const PlanDev& plan, cudaStream_t st) {
  switch (g.dt) {
    case kBF16: return split_hist_bf16(src, g, hist, nonzero, ws, plan, st);
    case kFP32: return split_hist_tiles_t<kFP32>(src, g, hist, nonzero, ws ? *ws : Ws{}, st);
    case kFP8: return split_hist_tiles_t<kFP8>(src, g, hist, nonzero, ws ? *ws : Ws{}, st);
    default: return split_hist_tiles_t<kFP4>(src, g, hist, nonzero, ws ? *ws : Ws{}, st);
  }
}

cudaError_t launch_code_lengths(const uint64_t* hist, uint32_t count, uint32_t alphabet_size, uint8_t* lens,
                                uint32_t* enc, cudaStream_t st) {
  const size_t smem = sizeof(HuffBlockSmem);
  cudaError_t e = allow_smem(k_code_lengths, smem, 3);
  if (e != cudaSuccess) return e;
  if (count == 0) return cudaSuccess;
  k_code_lengths<<<count, kHuffWarps * 32, smem, st>>>(hist, alphabet_size, lens, enc);
  return cudaGetLastError();
}

template <int DT>
static cudaError_t layout_t(const Geo& g, const Ws& ws, const PlanDev& plan, uint8_t* out, cudaStream_t st) {
  const uint32_t tiles = (uint32_t)ceil_div(g.n_entries, kLayoutTile);
  k_layout<DT><<<tiles, kLayoutThreads, 0, st>>>(g, ws, plan, out);
  return cudaGetLastError();
}

cudaError_t launch_layout(const Geo& g, const Ws& ws, const PlanDev& plan, uint8_t* out, cudaStream_t st) {
  switch (g.dt) {
    case kBF16: return layout_t<kBF16>(g, ws, plan, out, st);
    case kFP32: return layout_t<kFP32>(g, ws, plan, out, st);
    case kFP8: return layout_t<kFP8>(g, ws, plan, out, st);
    default: return layout_t<kFP4>(g, ws, plan, out, st);
  }
}

uint32_t layout_tiles(uint32_t n_entries) { return (uint32_t)ceil_div(n_entries, kLayoutTile); }

}  // namespace zipnn

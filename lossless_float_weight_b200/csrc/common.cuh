// common.cuh -- device-side definitions shared by the kernels of libzipnn_b200.
//
// The container layout these constants describe is the one documented in
// include/zipnn.h. This file is the CUDA library's own statement of it; the CPU
// oracle under oracle/ states it independently.
#pragma once

#include <cstdint>
#include <cuda_runtime.h>
#include <cuda/atomic>

namespace zipnn {

constexpr int kLmax = 12;
constexpr uint32_t kNoCode = 0xFFFFFFFFu;
constexpr uint32_t kModeRaw = 0, kModeZero = 1, kModeHuff = 2, kModeZrun = 3, kModePack = 4;
// Packed exponents (BF16 with a plan that lists them): a pair of exponents is one 8-bit
// symbol, each exponent's index in the plan's list as a nibble, kPackEsc for one that is
// not listed (its 8 bits follow the pair's code). The list holds at most kPackMax entries
// and takes kPackListBytes at the end of the code section.
constexpr uint32_t kPackMax = 15, kPackEsc = 15, kPackListBytes = 16;
// Zero runs: a byte plane is taken in blocks of 32 symbols; ZRUN keeps a bitmap of the
// blocks that hold a non-zero byte and the bytes of those blocks only.
constexpr uint32_t kZBlock = 32;
constexpr int kBF16 = 0, kFP32 = 1, kFP8 = 2, kFP4 = 3;
constexpr int kHeaderBytes = 64, kEntryBytes = 16;
constexpr uint32_t kMaxGroups = 64;

// Device status codes (the public zipnn_status values).
constexpr uint32_t kStCorrupt = 3, kStTimeout = 7;

// Values per 128-bit group of one thread and groups per encode thread (BF16: 64 values).
constexpr int kGroupValues = 16;
constexpr int kEncGroups = 4;
// The encode tile (32768 values; the encode kernels take it in passes of their own
// blocks) is also one histogram tile, whose counts give its bit offsets.
constexpr int kBf16TileValues = 32768;
__host__ __device__ constexpr uint32_t tile_values(int) { return (uint32_t)kBf16TileValues; }
// Counters a tile keeps for its bit offsets: BF16 and FP32 the 256 exponents; FP8 and FP4
// the joint (exponent, mantissa) bins, exponent * mantissa alphabet + mantissa (FP8
// 16 x 8, FP4 4 x 2).
__host__ __device__ constexpr uint32_t tile_bins(int dt) { return dt == kFP8 ? 128u : dt == kFP4 ? 8u : 256u; }

__host__ __device__ constexpr int n_streams(int dt) { return dt == kBF16 ? 2 : dt == kFP32 ? 4 : 3; }
// FP8 and FP4 entropy-code exponent and mantissa independently
__host__ __device__ constexpr int n_entropy(int dt) { return dt == kFP8 || dt == kFP4 ? 2 : 1; }
// bits of one value (FP4: two values share a byte, the first in the low nibble)
__host__ __device__ constexpr int value_bits(int dt) { return dt == kBF16 ? 16 : dt == kFP32 ? 32 : dt == kFP8 ? 8 : 4; }
// bytes of one value where whole bytes hold whole values (BF16, FP32, FP8)
__host__ __device__ constexpr int value_bytes(int dt) { return dt == kBF16 ? 2 : dt == kFP32 ? 4 : 1; }
// byte offset of value v (for FP4, v is even)
__host__ __device__ constexpr uint64_t value_offset(int dt, uint64_t v) { return v * value_bits(dt) / 8; }
// bits per symbol of a stream stored RAW
__host__ __device__ constexpr int raw_width(int dt, int s) {
  return dt == kFP8 ? (s == 0 ? 4 : s == 1 ? 3 : 1) : dt == kFP4 ? (s == 0 ? 2 : 1) : 8;
}
__host__ __device__ constexpr int alphabet(int dt, int s) { return 1 << raw_width(dt, s); }
__host__ __device__ constexpr bool is_entropy(int dt, int s) { return s == 0 || ((dt == kFP8 || dt == kFP4) && s == 1); }
__host__ __device__ constexpr uint64_t min64(uint64_t a, uint64_t b) { return a < b ? a : b; }
__host__ __device__ constexpr uint32_t min32(uint32_t a, uint32_t b) { return a < b ? a : b; }
__host__ __device__ constexpr uint64_t round16(uint64_t x) { return (x + 15) & ~uint64_t(15); }
__host__ __device__ constexpr uint64_t ceil_div(uint64_t a, uint64_t b) { return (a + b - 1) / b; }
__host__ __device__ constexpr uint32_t record_bytes(int dt, int s) { return (uint32_t)round16(alphabet(dt, s) / 2); }
// Byte planes (8-bit streams that are not entropy-coded) may take zero runs: BF16's
// sign/fraction byte (stream 1) and FP32's three fraction planes (streams 1..3).
__host__ __device__ constexpr bool is_byte_plane(int dt, int s) { return !is_entropy(dt, s) && raw_width(dt, s) == 8; }
__host__ __device__ constexpr int n_byte_planes(int dt) { return dt == kBF16 ? 1 : dt == kFP32 ? 3 : 0; }
// ZRUN payload of m symbols with `kept` symbols in marked blocks: the bitmap, then the bytes.
__host__ __device__ constexpr uint64_t zrun_map_bytes(uint64_t m) { return round16(ceil_div(ceil_div(m, kZBlock), 8)); }
__host__ __device__ constexpr uint64_t zrun_payload(uint64_t m, uint64_t kept) { return zrun_map_bytes(m) + round16(kept); }
__host__ __device__ constexpr uint64_t raw_payload(uint64_t m, int w) { return round16(ceil_div(m * (uint64_t)w, 8)); }

// Bytes of all shared code records for g groups, and the position of record r.
__host__ __device__ inline uint64_t shared_bytes(int dt, uint32_t g) {
  uint64_t b = 0;
  for (int e = 0; e < n_entropy(dt); e++) b += (uint64_t)g * record_bytes(dt, e);
  return b;
}
__host__ __device__ inline uint64_t shared_record_pos(int dt, uint32_t g, uint32_t r) {
  uint32_t e = r / g, k = r % g;
  uint64_t pos = 0;
  for (uint32_t i = 0; i < e; i++) pos += (uint64_t)g * record_bytes(dt, (int)i);
  return pos + (uint64_t)k * record_bytes(dt, (int)e);
}

// The code section with K packed exponents: the plain records, then (K > 0) one packed
// record per group and the list.
__host__ __device__ inline uint64_t code_section_bytes(int dt, uint32_t g, uint32_t K) {
  return shared_bytes(dt, g) + (K ? (uint64_t)g * record_bytes(dt, 0) + kPackListBytes : 0);
}
__host__ __device__ inline uint64_t packed_record_pos(int dt, uint32_t g, uint32_t gi) {
  return shared_bytes(dt, g) + (uint64_t)gi * record_bytes(dt, 0);
}

// Geometry of one call.
struct Geo {
  int dt;
  uint64_t n;
  uint32_t chunk_bytes, m0, n_chunks, S;
  uint32_t n_groups;          // 0 without a plan
  uint32_t n_packed;          // packed exponents the plan lists (BF16), 0 for none
  uint32_t tiles_per_chunk;   // encode tiles (tile_values(dt) values) per chunk
  uint32_t n_tiles;           // n_chunks * tiles_per_chunk
  uint32_t n_entries;         // n_chunks * n_streams
  uint64_t off_codes, off_payload;
  uint32_t spin_limit;        // polls after which a look-back wait gives up (kSpinLimit by default)
  uint32_t zwords;            // words of one chunk's zero-run block bitmap: ceil(ceil(m0 / 32) / 32)
};

// Workspace carve-up (device pointers). The first group is cleared by every
// compress call; the rest is fully overwritten before it is read.
struct Ws {
  uint32_t* status;     // [0] status, [1] encode ticket, [2] layout ticket, [4 + c] chunk c's
                        // finished histogram blocks
  uint32_t* hist;       // [n_chunks][n_entropy][256]
  uint32_t* nonzero;    // [n_entries]: OR of the stream's symbols
  uint32_t* zmap;       // [n_chunks][n_byte_planes][zwords]: bit i of word w set when block
                        // 32w + i of the plane holds a non-zero byte
  uint32_t* zcount;     // [n_chunks][n_byte_planes]: blocks set in zmap
  uint64_t* scan_desc;  // [layout tiles] look-back descriptors
  uint64_t* slot;       // [n_tiles][n_entropy] shared boundary words
  uint64_t* esize;      // [n_entries] payload bytes
  uint32_t* emode;      // [n_entries]
  uint32_t* ecode;      // [n_entries]
  uint64_t* eoff;       // [n_entries] payload offsets
  uint32_t* enc;        // [n_chunks][n_entropy][256]: len << 16 | code
  uint16_t* tile_hist;  // [n_tiles][tile_bins] (compress): counts of each encode tile
  uint32_t* tile_off;   // [n_entropy][n_tiles] (compress): bit offset of each tile in its
                        // chunk's bitstream of that entropy stream
  uint32_t* pack_hist;  // [n_chunks][256] (BF16 with packed exponents): pair-symbol counts
  uint32_t* pack_esc;   // [n_chunks]: escaped exponents
};

// Device-side tables of a plan.
struct PlanDev {
  const uint8_t* lens;  // [n_entropy][groups][256]
  const uint32_t* enc;  // [n_entropy][groups][256]: len << 16 | code
  uint32_t groups;
  uint32_t pack_k;           // packed exponents listed (BF16), 0 for none
  const uint8_t* pack_exps;  // [16]: the list, then zeros
  const uint8_t* pack_lens;  // [groups][256]: packed code lengths
  const uint32_t* pack_enc;  // [groups][256]: len << 16 | code
};

__device__ __forceinline__ void set_status(uint32_t* st, uint32_t code) { atomicCAS(st, 0u, code); }

__device__ __forceinline__ uint32_t bswap32(uint32_t x) { return __byte_perm(x, 0, 0x0123); }

// 32 bytes to global memory in one 256-bit store (sm_100: st.global.v8; p 32-byte aligned).
__device__ __forceinline__ void st_v8(void* p, const uint32_t* r) {
  asm volatile("st.global.v8.b32 [%0], {%1,%2,%3,%4,%5,%6,%7,%8};"
               :: "l"(p), "r"(r[0]), "r"(r[1]), "r"(r[2]), "r"(r[3]), "r"(r[4]), "r"(r[5]), "r"(r[6]), "r"(r[7])
               : "memory");
}

// 32 bytes from global memory in one 256-bit load (sm_100: ld.global.v8; p 32-byte
// aligned), through the read-only path. A warp whose lanes read consecutive 128-byte
// runs asks L1 for one sector a lane per load instead of half a sector.
__device__ __forceinline__ void ld_nc_v8(const void* p, uint32_t* r) {
  asm volatile("ld.global.nc.v8.b32 {%0,%1,%2,%3,%4,%5,%6,%7}, [%8];"
               : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7])
               : "l"(p));
}

// ---------------------------------------------------------------- look-back
// Descriptor: bits 63..62 flag (0 empty, 1 aggregate, 2 inclusive prefix), 61..0 value.
constexpr uint64_t kFlagAgg = 1ull << 62, kFlagPrefix = 2ull << 62, kValueMask = (1ull << 62) - 1;
// Default spin limit for every wait on another block; after it the wait records a timeout
// and continues, so no kernel can hang on a descriptor that is never written. A call can
// lower it (Geo::spin_limit) so that a test can make a healthy wait run out.
constexpr uint32_t kSpinLimit = 1u << 22;

__device__ __forceinline__ void publish(uint64_t* d, uint64_t v) {
  cuda::atomic_ref<uint64_t, cuda::thread_scope_device> a(*d);
  a.store(v, cuda::memory_order_release);
}
__device__ __forceinline__ uint64_t observe(uint64_t* d) {
  cuda::atomic_ref<uint64_t, cuda::thread_scope_device> a(*d);
  return a.load(cuda::memory_order_acquire);
}

// Single-pass decoupled look-back, run by one whole warp: publish this tile's
// aggregate, then inspect the 32 nearest predecessors of the same segment (tiles
// first..tile-1) at once; the nearest one holding an inclusive prefix ends the walk,
// otherwise all 32 aggregates are summed and the window moves back. Publishes the
// inclusive prefix and returns the exclusive one (to every lane). Tiles are handed out
// in launch order (a ticket), so every predecessor has started and the walk ends; the
// spin limit only guards against bugs. A walk that gives up returns the part of the
// prefix it has summed, never more than the true prefix, so every offset derived from it
// stays inside the true extent (payloads may then overlap, and the status says timeout).
__device__ inline uint64_t warp_lookback(uint64_t* desc, uint32_t tile, uint32_t first, uint64_t aggregate,
                                         uint32_t* status, uint32_t limit = kSpinLimit) {
  const int lane = threadIdx.x & 31;
  if (tile == first) {
    if (lane == 0) publish(desc + tile, kFlagPrefix | aggregate);
    return 0;
  }
  if (lane == 0) publish(desc + tile, kFlagAgg | aggregate);
  uint64_t excl = 0;
  int64_t base = (int64_t)tile - 1;
  uint32_t spins = 0;
  while (true) {
    const int64_t j = base - lane;
    const uint64_t d = j >= (int64_t)first ? observe(desc + j) : kFlagPrefix;  // before the segment: prefix 0
    const uint32_t flag = (uint32_t)(d >> 62);
    const uint32_t not_ready = __ballot_sync(0xFFFFFFFFu, flag == 0);
    const uint32_t is_prefix = __ballot_sync(0xFFFFFFFFu, flag == 2);
    const int pl = is_prefix ? __ffs(is_prefix) - 1 : 32;  // nearest prefix
    const uint32_t need = pl == 32 ? 0xFFFFFFFFu : (uint32_t)((2ull << pl) - 1);
    if (not_ready & need) {
      if (++spins > limit) {
        if (lane == 0) set_status(status, kStTimeout);
        break;
      }
      __nanosleep(spins < 64 ? 32 : 256);
      continue;
    }
    uint64_t v = lane <= pl ? (d & kValueMask) : 0;
#pragma unroll
    for (int o = 16; o; o >>= 1) v += __shfl_xor_sync(0xFFFFFFFFu, v, o);
    excl += v;
    if (pl < 32) break;
    base -= 32;
  }
  if (lane == 0) publish(desc + tile, kFlagPrefix | (excl + aggregate));
  return excl;
}

// Block-wide exclusive scan of one 32-bit value per thread (blockDim = NT).
template <int NT>
__device__ __forceinline__ uint32_t block_exclusive_scan(uint32_t v, uint32_t* s_warp, uint32_t& total) {
  constexpr int NW = NT / 32;
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  uint32_t x = v;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    uint32_t y = __shfl_up_sync(0xFFFFFFFFu, x, o);
    if (lane >= o) x += y;
  }
  if (lane == 31) s_warp[warp] = x;
  __syncthreads();
  if (warp == 0) {
    uint32_t w = lane < NW ? s_warp[lane] : 0;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      uint32_t y = __shfl_up_sync(0xFFFFFFFFu, w, o);
      if (lane >= o) w += y;
    }
    if (lane < NW) s_warp[lane] = w;  // inclusive warp totals
  }
  __syncthreads();
  total = s_warp[NW - 1];
  uint32_t before = warp ? s_warp[warp - 1] : 0;
  uint32_t r = before + x - v;
  __syncthreads();
  return r;
}

}  // namespace zipnn

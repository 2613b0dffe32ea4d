// api.cu -- the C ABI of include/zipnn.h: argument checks, workspace carving, launches.
// No call here computes any part of the codec on the host: histograms, codes, layout,
// encoding, decoding and the plan's grouping all run in the kernels.
#include <atomic>
#include <cstdlib>
#include <cstring>
#include <new>
#include <vector>

#include "zipnn.h"
#include "common.cuh"
#include "launch.h"

using namespace zipnn;

struct zipnn_plan {
  int dt;
  uint32_t groups;
  uint8_t* d_lens;   // [n_entropy][groups][256]
  uint32_t* d_enc;   // [n_entropy][groups][256]
  std::vector<uint8_t> h_lens;
  std::vector<uint32_t> assign;
  // packed exponents (BF16): K listed, and one device block holding the list (16 bytes),
  // K as a u32, the packed lengths [groups][256] and their codes [groups][256]
  uint32_t pack_k = 0;
  uint8_t* d_pack = nullptr;
  std::vector<uint8_t> h_pack_exps, h_pack_lens;
};

namespace {

constexpr uint64_t kAlign = 256;
constexpr uint32_t kMaxChunkBytes = 1u << 28;
// Largest value count: a plan's group histograms sum up to n counts, and every count
// stays far below the 64-bit range of the code builder's weights.
constexpr uint64_t kMaxValues = 1ull << 56;

// Polls after which a look-back wait gives up (zipnn_test_lookback_limit; 0 = default).
std::atomic<uint32_t> g_spin_limit{0};

inline uint64_t align_up(uint64_t x) { return (x + kAlign - 1) & ~(kAlign - 1); }
inline bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15) == 0; }
inline bool valid_dtype(int dt) { return dt == kBF16 || dt == kFP32 || dt == kFP8 || dt == kFP4; }

bool make_geo(int dt, uint64_t n, uint32_t chunk_bytes, uint32_t S, uint32_t G, Geo& g, uint32_t K = 0) {
  if (!valid_dtype(dt) || n == 0 || n >= kMaxValues) return false;
  if (dt == kFP4 && n % 2) return false;  // FP4 values come in byte pairs
  if (chunk_bytes < 16 || chunk_bytes % 16 || chunk_bytes > kMaxChunkBytes) return false;
  if (S < 16 || S % 16 || S > 65536) return false;
  g.dt = dt;
  g.n = n;
  g.chunk_bytes = chunk_bytes;
  g.m0 = (uint32_t)(8ull * chunk_bytes / (uint32_t)value_bits(dt));
  const uint64_t chunks = ceil_div(n, g.m0);
  const uint64_t tpc = ceil_div(g.m0, tile_values(dt));
  if (chunks * (uint64_t)n_streams(dt) > 0x7FFFFFFFull || chunks * tpc > 0x7FFFFFFFull) return false;
  g.n_chunks = (uint32_t)chunks;
  g.S = S;
  g.n_groups = G;
  g.n_packed = K;
  g.tiles_per_chunk = (uint32_t)tpc;
  g.n_tiles = (uint32_t)(chunks * tpc);
  g.n_entries = (uint32_t)(chunks * n_streams(dt));
  g.off_codes = kHeaderBytes + (uint64_t)kEntryBytes * g.n_entries;
  g.off_payload = g.off_codes + code_section_bytes(dt, G, K);
  const uint32_t lim = g_spin_limit.load(std::memory_order_relaxed);
  g.spin_limit = lim ? lim : kSpinLimit;
  g.zwords = (uint32_t)ceil_div(ceil_div(g.m0, kZBlock), 32);
  return true;
}

struct WsPlan {
  uint64_t status, hist, nonzero, zmap, zcount, scan_desc, slot, zero_end;
  uint64_t esize, emode, ecode, eoff, enc, tile_hist, tile_off, pack_hist, pack_esc;
  uint64_t km_mu, km_perm, km_assign, km_changed, km_gsum, total;
  bool tile_counts;  // per-tile histograms and bit offsets (every compress)
  int dt;
};

WsPlan ws_plan(const Geo& g) {
  const uint64_t C = g.n_chunks, NE = (uint64_t)n_entropy(g.dt), K = g.n_entries;
  WsPlan p;
  p.dt = g.dt;
  uint64_t o = 0;
  p.status = o;     o = align_up(o + 16 + C * 4);  // status, tickets, per-chunk counters
  p.hist = o;       o = align_up(o + C * NE * 256 * 4);
  p.nonzero = o;    o = align_up(o + K * 4);
  p.zmap = o;       o = align_up(o + C * (uint64_t)n_byte_planes(g.dt) * g.zwords * 4);
  p.zcount = o;     o = align_up(o + C * (uint64_t)n_byte_planes(g.dt) * 4);
  p.scan_desc = o;  o = align_up(o + (uint64_t)layout_tiles(g.n_entries) * 8);
  p.slot = o;       o = align_up(o + NE * g.n_tiles * 8);
  p.zero_end = o;
  p.esize = o;      o = align_up(o + K * 8);
  p.emode = o;      o = align_up(o + K * 4);
  p.ecode = o;      o = align_up(o + K * 4);
  p.eoff = o;       o = align_up(o + K * 8);
  p.enc = o;        o = align_up(o + C * NE * 256 * 4);
  p.tile_counts = true;
  p.tile_hist = o;  o = align_up(o + (p.tile_counts ? (uint64_t)g.n_tiles * tile_bins(g.dt) * 2 : 0));
  p.tile_off = o;   o = align_up(o + (p.tile_counts ? NE * g.n_tiles * 4 : 0));
  p.pack_hist = o;  o = align_up(o + (g.dt == kBF16 ? C * 256 * 4 : 0));
  p.pack_esc = o;   o = align_up(o + (g.dt == kBF16 ? C * 4 : 0));
  p.km_mu = o;      o = align_up(o + (uint64_t)kMaxGroups * 256 * 8);
  p.km_perm = o;    o = align_up(o + C * 4);
  p.km_assign = o;  o = align_up(o + C * 4);
  p.km_changed = o; o = align_up(o + 4);
  p.km_gsum = o;    o = align_up(o + NE * kMaxGroups * 256 * 8);
  p.total = o;
  return p;
}

Ws carve(const WsPlan& p, void* base) {
  uint8_t* b = static_cast<uint8_t*>(base);
  Ws w;
  w.status = reinterpret_cast<uint32_t*>(b + p.status);
  w.hist = reinterpret_cast<uint32_t*>(b + p.hist);
  w.nonzero = reinterpret_cast<uint32_t*>(b + p.nonzero);
  w.zmap = n_byte_planes(p.dt) ? reinterpret_cast<uint32_t*>(b + p.zmap) : nullptr;
  w.zcount = n_byte_planes(p.dt) ? reinterpret_cast<uint32_t*>(b + p.zcount) : nullptr;
  w.scan_desc = reinterpret_cast<uint64_t*>(b + p.scan_desc);
  w.slot = reinterpret_cast<uint64_t*>(b + p.slot);
  w.esize = reinterpret_cast<uint64_t*>(b + p.esize);
  w.emode = reinterpret_cast<uint32_t*>(b + p.emode);
  w.ecode = reinterpret_cast<uint32_t*>(b + p.ecode);
  w.eoff = reinterpret_cast<uint64_t*>(b + p.eoff);
  w.enc = reinterpret_cast<uint32_t*>(b + p.enc);
  w.tile_hist = p.tile_counts ? reinterpret_cast<uint16_t*>(b + p.tile_hist) : nullptr;
  w.tile_off = p.tile_counts ? reinterpret_cast<uint32_t*>(b + p.tile_off) : nullptr;
  w.pack_hist = p.dt == kBF16 ? reinterpret_cast<uint32_t*>(b + p.pack_hist) : nullptr;
  w.pack_esc = p.dt == kBF16 ? reinterpret_cast<uint32_t*>(b + p.pack_esc) : nullptr;
  return w;
}

uint64_t max_bytes(const Geo& g) {
  uint64_t total = g.off_codes + code_section_bytes(g.dt, kMaxGroups, g.dt == kBF16 ? kPackMax : 0);
  const uint64_t full = g.n / g.m0, tail = g.n % g.m0;
  for (int s = 0; s < n_streams(g.dt); s++) {
    const int w = raw_width(g.dt, s);
    total += full * raw_payload(g.m0, w);
    if (tail) total += raw_payload(tail, w);
  }
  return total;
}

zipnn_status cuda_status(cudaError_t e) { return e == cudaSuccess ? ZIPNN_OK : ZIPNN_ERR_CUDA; }

PlanDev plan_dev(const zipnn_plan* p) {
  PlanDev d;
  d.lens = p ? p->d_lens : nullptr;
  d.enc = p ? p->d_enc : nullptr;
  d.groups = p ? p->groups : 0;
  d.pack_k = p ? p->pack_k : 0;
  d.pack_exps = p && p->d_pack ? p->d_pack : nullptr;
  d.pack_lens = p && p->d_pack ? p->d_pack + 32 : nullptr;
  d.pack_enc = p && p->d_pack ? reinterpret_cast<const uint32_t*>(p->d_pack + 32 + (size_t)p->groups * 256) : nullptr;
  return d;
}

}  // namespace

// The kernels are built for sm_100a only; the answer is cached per device (several host
// threads may ask at once).
bool zipnn::device_ok() {
  static std::atomic<int> cache[128];  // 0 unknown, 1 usable, 2 not
  int dev = 0, major = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) {
    cudaGetLastError();
    return false;
  }
  if (dev >= 0 && dev < 128) {
    const int c = cache[dev].load(std::memory_order_relaxed);
    if (c) return c == 1;
  }
  const bool ok = cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev) == cudaSuccess && major == 10;
  if (!ok) cudaGetLastError();
  if (dev >= 0 && dev < 128) cache[dev].store(ok ? 1 : 2, std::memory_order_relaxed);
  return ok;
}

extern "C" {

size_t zipnn_max_compressed_bytes(zipnn_dtype dtype, uint64_t n, uint32_t chunk_bytes) {
  Geo g;
  if (!make_geo(dtype, n, chunk_bytes, ZIPNN_DEFAULT_SUBBLOCK, 0, g)) return 0;
  return (size_t)max_bytes(g);
}

size_t zipnn_workspace_bytes(zipnn_dtype dtype, uint64_t n, uint32_t chunk_bytes) {
  Geo g;
  if (!make_geo(dtype, n, chunk_bytes, ZIPNN_DEFAULT_SUBBLOCK, 0, g)) return 0;
  return (size_t)ws_plan(g).total;
}

zipnn_status zipnn_compress_ex(zipnn_dtype dtype, const void* src, uint64_t n, uint32_t chunk_bytes, uint32_t subblock,
                               const zipnn_plan_t* plan, void* out, size_t out_cap, void* ws, size_t ws_bytes,
                               zipnn_stream_t stream) {
  if (subblock == 0) subblock = ZIPNN_DEFAULT_SUBBLOCK;
  if (!src || !out || !ws || !aligned16(src) || !aligned16(out) || !aligned16(ws)) return ZIPNN_ERR_INVALID_ARG;
  if (plan && plan->dt != (int)dtype) return ZIPNN_ERR_PLAN_MISMATCH;
  Geo g;
  if (!make_geo(dtype, n, chunk_bytes, subblock, plan ? plan->groups : 0, g, plan ? plan->pack_k : 0))
    return ZIPNN_ERR_INVALID_ARG;
  if (out_cap < max_bytes(g)) return ZIPNN_ERR_OUT_TOO_SMALL;
  const WsPlan wp = ws_plan(g);
  if (ws_bytes < wp.total) return ZIPNN_ERR_OUT_TOO_SMALL;
  if (!device_ok()) return ZIPNN_ERR_UNSUPPORTED;
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  const Ws w = carve(wp, ws);
  const PlanDev pd = plan_dev(plan);
  cudaError_t e = cudaMemsetAsync(ws, 0, wp.zero_end, st);
  if (e == cudaSuccess) {
    TimedLaunch t(kIdHist, st);
    e = launch_split_hist(src, g, w.hist, w.nonzero, &w, pd, st);
  }
  if (e == cudaSuccess && pd.pack_k) {
    TimedLaunch t(kIdPackHist, st);
    e = launch_pack_hist(src, g, w, pd, st);
  }
  if (e == cudaSuccess) {
    TimedLaunch t(kIdBuild, st);
    e = launch_build_chunks(g, w, pd, st);
  }
  if (e == cudaSuccess) {
    TimedLaunch t(kIdLayout, st);
    e = launch_layout(g, w, pd, static_cast<uint8_t*>(out), st);
  }
  if (e == cudaSuccess) {
    TimedLaunch t(kIdEncode, st);
    e = g.dt == kBF16 ? launch_encode_bf16(src, g, w, static_cast<uint8_t*>(out), st)
        : g.dt == kFP32 ? launch_encode_fp32(src, g, w, static_cast<uint8_t*>(out), st)
                        : launch_encode_sub(src, g, w, static_cast<uint8_t*>(out), st);
  }
  if (e == cudaSuccess && pd.pack_k) {
    TimedLaunch t(kIdPackEncode, st);
    e = launch_encode_pack(src, g, w, pd, static_cast<uint8_t*>(out), st);
  }
  return cuda_status(e);
}

zipnn_status zipnn_compress(zipnn_dtype dtype, const void* src, uint64_t n, uint32_t chunk_bytes,
                            const zipnn_plan_t* plan, void* out, size_t out_cap, void* ws, size_t ws_bytes,
                            zipnn_stream_t stream) {
  return zipnn_compress_ex(dtype, src, n, chunk_bytes, 0, plan, out, out_cap, ws, ws_bytes, stream);
}

zipnn_status zipnn_decompress(zipnn_dtype dtype, const void* in, size_t in_bytes, uint64_t n, uint32_t chunk_bytes,
                              void* out, void* ws, size_t ws_bytes, zipnn_stream_t stream) {
  if (!in || !out || !ws || !aligned16(in) || !aligned16(out) || !aligned16(ws)) return ZIPNN_ERR_INVALID_ARG;
  Geo g;
  if (!make_geo(dtype, n, chunk_bytes, ZIPNN_DEFAULT_SUBBLOCK, 0, g)) return ZIPNN_ERR_INVALID_ARG;
  if (ws_bytes < 256) return ZIPNN_ERR_OUT_TOO_SMALL;
  if (!device_ok()) return ZIPNN_ERR_UNSUPPORTED;
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  cudaError_t e = cudaMemsetAsync(ws, 0, 4, st);
  if (e == cudaSuccess) {
    TimedLaunch t(kIdDecode, st);
    e = launch_decode(static_cast<const uint8_t*>(in), in_bytes, g, static_cast<uint8_t*>(out),
                      static_cast<uint32_t*>(ws), st);
  }
  return cuda_status(e);
}

// Batched decompress workspace: the status word, then the device copy of the item table.
static constexpr size_t kBatchTableOffset = 256;

size_t zipnn_decompress_batch_workspace_bytes(uint32_t count) {
  return kBatchTableOffset + (size_t)align_up((uint64_t)count * sizeof(DecodeItem));
}

zipnn_status zipnn_decompress_batch(zipnn_dtype dtype, uint32_t chunk_bytes, uint32_t count,
                                    const zipnn_decompress_item* items, void* ws, size_t ws_bytes,
                                    zipnn_stream_t stream) {
  if (!items || !ws || count == 0 || !aligned16(ws)) return ZIPNN_ERR_INVALID_ARG;
  std::vector<DecodeItem> table(count);
  Geo g0;
  uint64_t chunks = 0;
  for (uint32_t i = 0; i < count; i++) {
    const zipnn_decompress_item& it = items[i];
    Geo g;
    if (!it.in || !it.out || !aligned16(it.in) || !aligned16(it.out)) return ZIPNN_ERR_INVALID_ARG;
    if (!make_geo(dtype, it.n, chunk_bytes, ZIPNN_DEFAULT_SUBBLOCK, 0, g)) return ZIPNN_ERR_INVALID_ARG;
    if (i == 0) g0 = g;
    table[i] = DecodeItem{static_cast<const uint8_t*>(it.in), it.in_bytes, it.n, static_cast<uint8_t*>(it.out), chunks};
    chunks += g.n_chunks;
    if (chunks > 0x7FFFFFFFull) return ZIPNN_ERR_INVALID_ARG;
  }
  if (ws_bytes < zipnn_decompress_batch_workspace_bytes(count)) return ZIPNN_ERR_OUT_TOO_SMALL;
  if (!device_ok()) return ZIPNN_ERR_UNSUPPORTED;
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  DecodeItem* dev_table = reinterpret_cast<DecodeItem*>(static_cast<uint8_t*>(ws) + kBatchTableOffset);
  cudaError_t e = cudaMemsetAsync(ws, 0, 4, st);
  // from pageable memory: the table is staged before the call returns
  if (e == cudaSuccess)
    e = cudaMemcpyAsync(dev_table, table.data(), (size_t)count * sizeof(DecodeItem), cudaMemcpyHostToDevice, st);
  if (e == cudaSuccess) {
    TimedLaunch t(kIdDecode, st);
    e = launch_decode_batch(dev_table, count, g0, (uint32_t)chunks, static_cast<uint32_t*>(ws), st);
  }
  return cuda_status(e);
}

zipnn_status zipnn_compressed_size(const void* out, zipnn_stream_t stream, uint64_t* bytes) {
  if (!out || !bytes) return ZIPNN_ERR_INVALID_ARG;
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  uint64_t v = 0;
  cudaError_t e = cudaMemcpyAsync(&v, static_cast<const uint8_t*>(out) + 48, 8, cudaMemcpyDeviceToHost, st);
  if (e == cudaSuccess) e = cudaStreamSynchronize(st);
  if (e != cudaSuccess) return ZIPNN_ERR_CUDA;
  *bytes = v;
  return ZIPNN_OK;
}

zipnn_status zipnn_get_status(const void* ws, zipnn_stream_t stream) {
  if (!ws) return ZIPNN_ERR_INVALID_ARG;
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  uint32_t v = 0;
  cudaError_t e = cudaMemcpyAsync(&v, ws, 4, cudaMemcpyDeviceToHost, st);
  if (e == cudaSuccess) e = cudaStreamSynchronize(st);
  if (e != cudaSuccess) return ZIPNN_ERR_CUDA;
  return (zipnn_status)v;
}

zipnn_status zipnn_histogram(zipnn_dtype dtype, const void* src, uint64_t n, uint32_t chunk_bytes, uint32_t* hist_out,
                             zipnn_stream_t stream) {
  if (!src || !hist_out || !aligned16(src)) return ZIPNN_ERR_INVALID_ARG;
  Geo g;
  if (!make_geo(dtype, n, chunk_bytes, ZIPNN_DEFAULT_SUBBLOCK, 0, g)) return ZIPNN_ERR_INVALID_ARG;
  if (!device_ok()) return ZIPNN_ERR_UNSUPPORTED;
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  cudaError_t e = cudaMemsetAsync(hist_out, 0, (size_t)g.n_chunks * n_entropy(dtype) * 256 * 4, st);
  if (e == cudaSuccess) e = launch_split_hist(src, g, hist_out, nullptr, nullptr, PlanDev{}, st);
  return cuda_status(e);
}

zipnn_status zipnn_code_lengths(const uint64_t* hist, uint32_t count, uint32_t alphabet, uint8_t* lens_out,
                                zipnn_stream_t stream) {
  if (!hist || !lens_out || alphabet < 1 || alphabet > 256 || count > 0x7FFFFFFFu) return ZIPNN_ERR_INVALID_ARG;
  if (!device_ok()) return ZIPNN_ERR_UNSUPPORTED;
  return cuda_status(launch_code_lengths(hist, count, alphabet, lens_out, nullptr, reinterpret_cast<cudaStream_t>(stream)));
}

static zipnn_status plan_alloc(int dt, uint32_t groups, zipnn_plan** out) {
  zipnn_plan* p = new (std::nothrow) zipnn_plan();
  if (!p) return ZIPNN_ERR_INVALID_ARG;
  p->dt = dt;
  p->groups = groups;
  const size_t recs = (size_t)n_entropy(dt) * groups;
  if (cudaMalloc(&p->d_lens, recs * 256) != cudaSuccess) {
    delete p;
    return ZIPNN_ERR_CUDA;
  }
  if (cudaMalloc(&p->d_enc, recs * 256 * 4) != cudaSuccess) {
    cudaFree(p->d_lens);
    delete p;
    return ZIPNN_ERR_CUDA;
  }
  p->h_lens.assign(recs * 256, 0);
  *out = p;
  return ZIPNN_OK;
}

static zipnn_status pack_alloc(zipnn_plan* p) {
  const size_t bytes = 32 + (size_t)p->groups * 256 * 5;
  if (cudaMalloc(&p->d_pack, bytes) != cudaSuccess) {
    cudaGetLastError();
    p->d_pack = nullptr;
    return ZIPNN_ERR_CUDA;
  }
  p->h_pack_exps.assign(kPackListBytes, 0);
  p->h_pack_lens.assign((size_t)p->groups * 256, 0);
  return ZIPNN_OK;
}

zipnn_status zipnn_plan_create(zipnn_dtype dtype, const void* src, uint64_t n, uint32_t chunk_bytes, uint32_t groups,
                               uint64_t seed, void* ws, size_t ws_bytes, zipnn_stream_t stream, zipnn_plan_t** plan) {
  return zipnn_plan_create_packed(dtype, src, n, chunk_bytes, groups, seed, 0, ws, ws_bytes, stream, plan);
}

zipnn_status zipnn_plan_create_packed(zipnn_dtype dtype, const void* src, uint64_t n, uint32_t chunk_bytes,
                                      uint32_t groups, uint64_t seed, uint32_t max_pack, void* ws, size_t ws_bytes,
                                      zipnn_stream_t stream, zipnn_plan_t** plan) {
  if (!src || !ws || !plan || !aligned16(src) || !aligned16(ws)) return ZIPNN_ERR_INVALID_ARG;
  if (max_pack > kPackMax || (max_pack && dtype != ZIPNN_BF16)) return ZIPNN_ERR_INVALID_ARG;
  if (groups < 1 || groups > kMaxGroups) return ZIPNN_ERR_INVALID_ARG;
  Geo g;
  if (!make_geo(dtype, n, chunk_bytes, ZIPNN_DEFAULT_SUBBLOCK, 0, g)) return ZIPNN_ERR_INVALID_ARG;
  const WsPlan wp = ws_plan(g);
  if (ws_bytes < wp.total) return ZIPNN_ERR_OUT_TOO_SMALL;
  if (!device_ok()) return ZIPNN_ERR_UNSUPPORTED;
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  uint8_t* b = static_cast<uint8_t*>(ws);
  const Ws w = carve(wp, ws);
  const int NE = n_entropy(dtype);
  KmeansDev k;
  k.hist = w.hist;
  k.C = g.n_chunks;
  k.A = (uint32_t)alphabet(dtype, 0);
  k.NE = (uint32_t)NE;
  k.G = groups;
  k.m0 = g.m0;
  k.n = n;
  k.mu = reinterpret_cast<double*>(b + wp.km_mu);
  k.perm = reinterpret_cast<uint32_t*>(b + wp.km_perm);
  k.assign = reinterpret_cast<uint32_t*>(b + wp.km_assign);
  k.changed = reinterpret_cast<uint32_t*>(b + wp.km_changed);
  k.gsum = reinterpret_cast<uint64_t*>(b + wp.km_gsum);
  zipnn_plan* p = nullptr;
  zipnn_status zs = plan_alloc(dtype, groups, &p);
  if (zs != ZIPNN_OK) return zs;
  cudaError_t e = cudaMemsetAsync(ws, 0, wp.zero_end, st);
  if (e == cudaSuccess) e = launch_split_hist(src, g, w.hist, nullptr, nullptr, PlanDev{}, st);
  if (e == cudaSuccess) {
    if (g.n_chunks <= groups) {
      e = launch_identity_assign(k.assign, k.C, st);
    } else {
      e = launch_kmeans_init(k, seed, st);
      for (int it = 0; it < 100 && e == cudaSuccess; it++) {
        uint32_t changed = 0;
        e = cudaMemsetAsync(k.changed, 0, 4, st);
        if (e == cudaSuccess) e = launch_kmeans_assign(k, st);
        if (e == cudaSuccess) e = cudaMemcpyAsync(&changed, k.changed, 4, cudaMemcpyDeviceToHost, st);
        if (e == cudaSuccess) e = cudaStreamSynchronize(st);
        if (e != cudaSuccess || !changed) break;
        e = launch_kmeans_update(k, st);
      }
    }
  }
  if (e == cudaSuccess) e = cudaMemsetAsync(k.gsum, 0, (size_t)NE * groups * 256 * 8, st);
  if (e == cudaSuccess) e = launch_group_sums(k, st);
  for (int ei = 0; ei < NE && e == cudaSuccess; ei++)
    e = launch_code_lengths(k.gsum + (size_t)ei * groups * 256, groups, (uint32_t)alphabet(dtype, ei),
                            p->d_lens + (size_t)ei * groups * 256, p->d_enc + (size_t)ei * groups * 256, st);
  if (e == cudaSuccess && max_pack) {
    // packed exponents: the list from the exponent counts, the chunks' pair counts, and
    // each group's packed code from its members' summed pair counts
    if (pack_alloc(p) != ZIPNN_OK) e = cudaErrorMemoryAllocation;
    uint32_t K = 0;
    if (e == cudaSuccess)
      e = launch_pack_select(w.hist, g.n_chunks, (uint32_t)NE, max_pack, p->d_pack,
                             reinterpret_cast<uint32_t*>(p->d_pack + 16), st);
    if (e == cudaSuccess) e = cudaMemcpyAsync(&K, p->d_pack + 16, 4, cudaMemcpyDeviceToHost, st);
    if (e == cudaSuccess) e = cudaStreamSynchronize(st);
    if (e == cudaSuccess && K) {
      p->pack_k = K;
      const PlanDev pd = plan_dev(p);
      e = launch_pack_hist(src, g, w, pd, st);
      if (e == cudaSuccess) e = cudaMemsetAsync(k.gsum, 0, (size_t)groups * 256 * 8, st);
      if (e == cudaSuccess) e = launch_pack_group_sums(w.pack_hist, k.assign, g.n_chunks, k.gsum, st);
      if (e == cudaSuccess)
        e = launch_code_lengths(k.gsum, groups, 256, p->d_pack + 32,
                                reinterpret_cast<uint32_t*>(p->d_pack + 32 + (size_t)groups * 256), st);
      if (e == cudaSuccess)
        e = cudaMemcpyAsync(p->h_pack_exps.data(), p->d_pack, kPackListBytes, cudaMemcpyDeviceToHost, st);
      if (e == cudaSuccess)
        e = cudaMemcpyAsync(p->h_pack_lens.data(), p->d_pack + 32, p->h_pack_lens.size(), cudaMemcpyDeviceToHost, st);
    }
  }
  if (e == cudaSuccess) {
    p->assign.resize(g.n_chunks);
    e = cudaMemcpyAsync(p->h_lens.data(), p->d_lens, p->h_lens.size(), cudaMemcpyDeviceToHost, st);
    if (e == cudaSuccess)
      e = cudaMemcpyAsync(p->assign.data(), k.assign, (size_t)g.n_chunks * 4, cudaMemcpyDeviceToHost, st);
    if (e == cudaSuccess) e = cudaStreamSynchronize(st);
  }
  if (e != cudaSuccess) {
    zipnn_plan_destroy(p);
    return ZIPNN_ERR_CUDA;
  }
  *plan = p;
  return ZIPNN_OK;
}

zipnn_status zipnn_plan_export(const zipnn_plan_t* plan, void* host_buf, size_t cap, size_t* bytes) {
  if (!plan || !bytes) return ZIPNN_ERR_INVALID_ARG;
  const int dt = plan->dt, NE = n_entropy(dt);
  const uint32_t G = plan->groups, K = plan->pack_k;
  const size_t need = 8 + code_section_bytes(dt, G, K);
  *bytes = need;
  if (!host_buf) return ZIPNN_OK;
  if (cap < need) return ZIPNN_ERR_OUT_TOO_SMALL;
  uint8_t* o = static_cast<uint8_t*>(host_buf);
  std::memset(o, 0, need);
  o[0] = 'Z';
  o[1] = 'N';
  o[2] = 'P';
  o[3] = '1';
  o[4] = (uint8_t)dt;
  o[5] = (uint8_t)G;
  o[6] = (uint8_t)K;
  for (int e = 0; e < NE; e++) {
    const int A = alphabet(dt, e);
    for (uint32_t gi = 0; gi < G; gi++) {
      const uint8_t* l = plan->h_lens.data() + ((size_t)e * G + gi) * 256;
      uint8_t* r = o + 8 + shared_record_pos(dt, G, (uint32_t)e * G + gi);
      for (int i = 0; i < A / 2; i++) r[i] = (uint8_t)(l[2 * i] | (l[2 * i + 1] << 4));
    }
  }
  if (K) {
    for (uint32_t gi = 0; gi < G; gi++) {
      const uint8_t* l = plan->h_pack_lens.data() + (size_t)gi * 256;
      uint8_t* r = o + 8 + packed_record_pos(dt, G, gi);
      for (int i = 0; i < 128; i++) r[i] = (uint8_t)(l[2 * i] | (l[2 * i + 1] << 4));
    }
    std::memcpy(o + need - kPackListBytes, plan->h_pack_exps.data(), K);
  }
  return ZIPNN_OK;
}

// 4-bit lengths of a record into l[0..A): every length at most 12, the Kraft sum at most 1,
// and the record's bytes past the alphabet zero.
static bool read_lengths(const uint8_t* r, int A, uint32_t rb, uint8_t* l) {
  uint64_t kraft = 0;
  for (int i = 0; i < A; i++) {
    l[i] = (i & 1) ? (r[i >> 1] >> 4) : (r[i >> 1] & 15);
    if (l[i] > kLmax) return false;
    if (l[i]) kraft += 1ull << (kLmax - l[i]);
  }
  for (uint32_t i = (uint32_t)A / 2; i < rb; i++)
    if (r[i]) return false;
  return kraft <= (1ull << kLmax);
}

zipnn_status zipnn_plan_import(const void* host_buf, size_t bytes, zipnn_plan_t** plan) {
  if (!host_buf || !plan || bytes < 8) return ZIPNN_ERR_INVALID_ARG;
  const uint8_t* in = static_cast<const uint8_t*>(host_buf);
  if (in[0] != 'Z' || in[1] != 'N' || in[2] != 'P' || in[3] != '1' || in[7]) return ZIPNN_ERR_CORRUPT;
  const int dt = in[4];
  const uint32_t groups = in[5], K = in[6];
  if (!valid_dtype(dt) || groups < 1 || groups > kMaxGroups) return ZIPNN_ERR_CORRUPT;
  if (K > kPackMax || (K && dt != kBF16)) return ZIPNN_ERR_CORRUPT;
  const size_t need = 8 + code_section_bytes(dt, groups, K);
  if (bytes < need) return ZIPNN_ERR_CORRUPT;
  for (size_t i = need - kPackListBytes + K; K && i < need; i++)
    if (in[i]) return ZIPNN_ERR_CORRUPT;
  if (!device_ok()) return ZIPNN_ERR_UNSUPPORTED;
  zipnn_plan* p = nullptr;
  zipnn_status zs = plan_alloc(dt, groups, &p);
  if (zs != ZIPNN_OK) return zs;
  const int NE = n_entropy(dt);
  bool ok = true;
  for (int e = 0; e < NE && ok; e++)
    for (uint32_t gi = 0; gi < groups && ok; gi++)
      ok = read_lengths(in + 8 + shared_record_pos(dt, groups, (uint32_t)e * groups + gi), alphabet(dt, e),
                        record_bytes(dt, e), p->h_lens.data() + ((size_t)e * groups + gi) * 256);
  if (ok && K) {
    if (pack_alloc(p) != ZIPNN_OK) {
      zipnn_plan_destroy(p);
      return ZIPNN_ERR_CUDA;
    }
    p->pack_k = K;
    std::memcpy(p->h_pack_exps.data(), in + need - kPackListBytes, kPackListBytes);
    for (uint32_t gi = 0; gi < groups && ok; gi++)
      ok = read_lengths(in + 8 + packed_record_pos(dt, groups, gi), 256, 128, p->h_pack_lens.data() + (size_t)gi * 256);
  }
  if (!ok) {
    zipnn_plan_destroy(p);
    return ZIPNN_ERR_CORRUPT;
  }
  cudaError_t e = cudaMemcpy(p->d_lens, p->h_lens.data(), p->h_lens.size(), cudaMemcpyHostToDevice);
  if (e == cudaSuccess) e = launch_canonical(p->d_lens, (uint32_t)NE * groups, p->d_enc, 0);
  if (e == cudaSuccess && K) {
    uint8_t head[32] = {0};
    std::memcpy(head, p->h_pack_exps.data(), kPackListBytes);
    std::memcpy(head + 16, &K, 4);
    e = cudaMemcpy(p->d_pack, head, 32, cudaMemcpyHostToDevice);
    if (e == cudaSuccess)
      e = cudaMemcpy(p->d_pack + 32, p->h_pack_lens.data(), p->h_pack_lens.size(), cudaMemcpyHostToDevice);
    if (e == cudaSuccess)
      e = launch_canonical(p->d_pack + 32, groups, reinterpret_cast<uint32_t*>(p->d_pack + 32 + (size_t)groups * 256), 0);
  }
  if (e == cudaSuccess) e = cudaDeviceSynchronize();
  if (e != cudaSuccess) {
    zipnn_plan_destroy(p);
    return ZIPNN_ERR_CUDA;
  }
  *plan = p;
  return ZIPNN_OK;
}

zipnn_status zipnn_plan_assignment(const zipnn_plan_t* plan, uint32_t* host_buf, size_t cap, size_t* count) {
  if (!plan || !count) return ZIPNN_ERR_INVALID_ARG;
  *count = plan->assign.size();
  if (!host_buf) return ZIPNN_OK;
  if (cap < plan->assign.size()) return ZIPNN_ERR_OUT_TOO_SMALL;
  std::memcpy(host_buf, plan->assign.data(), plan->assign.size() * 4);
  return ZIPNN_OK;
}

void zipnn_plan_destroy(zipnn_plan_t* plan) {
  if (!plan) return;
  if (plan->d_lens) cudaFree(plan->d_lens);
  if (plan->d_enc) cudaFree(plan->d_enc);
  if (plan->d_pack) cudaFree(plan->d_pack);
  delete plan;
}

zipnn_status zipnn_test_lookback_limit(uint32_t polls) {
  g_spin_limit.store(polls, std::memory_order_relaxed);
  return ZIPNN_OK;
}

const char* zipnn_status_string(zipnn_status status) {
  switch (status) {
    case ZIPNN_OK: return "ok";
    case ZIPNN_ERR_INVALID_ARG: return "invalid argument";
    case ZIPNN_ERR_OUT_TOO_SMALL: return "output or workspace too small";
    case ZIPNN_ERR_CORRUPT: return "corrupt container or arguments that do not match it";
    case ZIPNN_ERR_PLAN_MISMATCH: return "plan made for another dtype";
    case ZIPNN_ERR_CUDA: return "CUDA runtime error";
    case ZIPNN_ERR_UNSUPPORTED: return "unsupported device or size";
    case ZIPNN_ERR_TIMEOUT: return "device-side wait gave up";
  }
  return "unknown status";
}

}  // extern "C"

/*
 * zipnn.h -- C ABI of libzipnn_b200: ZipNN-style lossless compression of BF16, FP32,
 * FP8 (E4M3) and FP4 (E2M1) tensors on an NVIDIA B200 (sm_100a).
 *
 * What the calls compute, by page title and section:
 *  - "ZipNN: Lossless Compression for AI Models" (abstract) and the THEORY-599 note
 *    on it, "Per-field compressibility (Table II)": every value is split into its
 *    exponent field and its sign/fraction bytes; the exponent field is entropy-coded,
 *    the sign/fraction bytes are stored as they are ("raw"), omitted when a chunk of them
 *    is all zero (the "clean" models of the same table), or stored without their runs of
 *    zero bytes (ZRUN).
 *  - THEORY-599, "Order-0 only (section III-A b)": one order-0 symbol histogram and one
 *    Huffman code per chunk; no context model.
 *  - "Lossless Compression of Neural Network Components: Weights, Checkpoints, and K/V
 *    Caches in Low-Precision Formats" (abstract): FP8 and FP4 exponent and mantissa
 *    are entropy-coded independently.
 *  - "NeuralZip: Reusable Setup for Fast Lossless Compression" (abstract): chunks are
 *    grouped by the similarity of their exponent distributions, each group shares one
 *    Huffman code, and this setup (a "plan") is built once and reused. The same setup may
 *    also choose packed exponents for recurring exponent tuples (BF16; see PACK below).
 *
 * Container format (all integers little-endian; every section and payload starts on a
 * 16-byte boundary; every pad byte and pad bit is zero):
 *   header, 64 bytes: 'Z','N','N','1' | u16 version=1 | u8 dtype | u8 n_streams |
 *     u64 n | u32 chunk_bytes | u32 S | u32 n_chunks | u32 n_shared | u64 off_codes |
 *     u64 off_payload | u64 total_bytes | u8 L_MAX=12 | u8 n_groups | u8 n_packed |
 *     5 zero bytes
 *   chunk table at 64: one 16-byte entry per (chunk c, stream s), index k = c*n_streams+s:
 *     u8 mode (0 RAW, 1 ZERO, 2 HUFF, 3 ZRUN, 4 PACK) | 3 zero bytes | u32 code |
 *     u64 payload offset. code is the shared record index for a HUFF or PACK entry coded
 *     with a plan's code, and 0xFFFFFFFF otherwise.
 *   shared code records at off_codes (n_shared = n_groups * entropy streams, plus n_groups
 *     with packed exponents), record r = e*n_groups + g: code lengths, 4 bits each (byte
 *     i = len[2i] | len[2i+1] << 4), padded to 16 bytes (128 bytes for a 256-symbol
 *     alphabet, 16 for FP8's). With n_packed = K > 0 (BF16 only): record n_groups + g is
 *     group g's packed code over the 256 pair symbols, and the K packed exponents follow
 *     the records, padded with zeros to 16 bytes.
 *   payloads at off_payload in increasing k, each at the running offset:
 *     RAW : the chunk's symbols at a fixed width, most significant bit first, padded.
 *     ZERO: nothing (every symbol of that chunk and stream is 0).
 *     HUFF: [local code record if code == 0xFFFFFFFF] [u32 idx[ceil(m/S)], padded]
 *           [bitstream, padded]; idx[j] is the bit offset of symbol j*S.
 *     ZRUN: zero runs of a byte plane: the chunk's symbols in blocks of 32 (the last may
 *           be shorter); [one bit per block, most significant first, 1 when the block
 *           holds a non-zero byte, padded] [the bytes of the marked blocks, padded].
 *     PACK: packed exponent tuples (NeuralZip, abstract: recurring exponent tuples
 *           represented by packed exponents), a BF16 exponent stream of a chunk with an
 *           even value count: the exponents of values 2j and 2j+1 form the pair symbol
 *           i(first) << 4 | i(second), i(x) = x's index among the K packed exponents, or
 *           15 when x is not among them. [u32 idx[ceil(m/S)], padded] [bitstream, padded]:
 *           every pair's code, followed by the 8 bits of its first exponent when that
 *           one's index is 15, then of its second when that one's is; idx[j] is the bit
 *           offset of the pair of value j*S.
 *   Streams: BF16 [exponent, sign+fraction byte]; FP32 [exponent, sign + fraction
 *   bits 22..16, fraction bits 15..8, fraction bits 7..0]; FP8 E4M3 [exponent (4 bits),
 *   mantissa (3 bits), sign (1 bit)]; FP4 E2M1 [exponent (2 bits), mantissa (1 bit),
 *   sign (1 bit)]. Entropy-coded streams: the exponent, and for FP8 and FP4 also the
 *   mantissa. FP4 values come two to a byte, value 2i in the low nibble of byte i
 *   (sign bit 3, exponent bits 2..1, mantissa bit 0); n counts values and is even.
 *   Codes are canonical (RFC 1951 rule), at most 12 bits long.
 *   A stream is ZERO when all its symbols in the chunk are 0; an entropy stream is HUFF
 *   (PACK when the plan's packed code of a group codes it in strictly fewer bits than any
 *   plain shared code) when that payload is strictly smaller than RAW, else RAW; a byte plane (BF16's
 *   sign+fraction byte, FP32's three fraction planes) is ZRUN when that payload is
 *   strictly smaller than RAW, else RAW; the 1-bit sign streams of FP8 and FP4 are RAW.
 *
 * Conventions for every call:
 *  - n (values) is at most 2^56 - 1, and a tensor has at most 2^31 - 1 chunk entries.
 *  - Device pointers (src, out, in, ws) are owned by the caller, must be 16-byte
 *    aligned, and are only read or written on `stream`, in stream order.
 *  - Compress and decompress are asynchronous; they allocate nothing. Argument errors
 *    are returned before anything is launched. Errors found on the device (a corrupt
 *    container, a container that does not match the arguments) are written to the
 *    workspace and returned by zipnn_get_status.
 *  - `ws` is scratch owned by the caller, at least zipnn_workspace_bytes(...) bytes.
 *    One workspace must not be used by two calls that may run at the same time.
 */
#ifndef ZIPNN_H
#define ZIPNN_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

/* Same type as cudaStream_t; NULL is the legacy default stream. */
typedef struct CUstream_st* zipnn_stream_t;

typedef enum { ZIPNN_BF16 = 0, ZIPNN_FP32 = 1, ZIPNN_FP8_E4M3 = 2, ZIPNN_FP4_E2M1 = 3 } zipnn_dtype;

typedef enum {
  ZIPNN_OK = 0,
  ZIPNN_ERR_INVALID_ARG = 1,  /* bad pointer, size, alignment or dtype */
  ZIPNN_ERR_OUT_TOO_SMALL = 2, /* out_cap or ws_bytes below the required size */
  ZIPNN_ERR_CORRUPT = 3,       /* container damaged or not matching the arguments */
  ZIPNN_ERR_PLAN_MISMATCH = 4, /* plan made for another dtype */
  ZIPNN_ERR_CUDA = 5,          /* a CUDA runtime call failed */
  ZIPNN_ERR_UNSUPPORTED = 6,   /* no sm_100 device, or a size beyond the limits below */
  ZIPNN_ERR_TIMEOUT = 7        /* a bounded device-side wait gave up (never expected) */
} zipnn_status;

typedef struct zipnn_plan zipnn_plan_t; /* opaque; owns device code tables */

#define ZIPNN_DEFAULT_CHUNK_BYTES 262144u /* 256 KiB of uncompressed values per chunk */
#define ZIPNN_DEFAULT_SUBBLOCK 512u       /* symbols per sub-block index entry */
#define ZIPNN_MAX_GROUPS 64u
#define ZIPNN_LMAX 12u
#define ZIPNN_MAX_PACKED 15u

/* Upper bound of the container size for n values: header, chunk table, room for
 * ZIPNN_MAX_GROUPS shared records (and, for BF16, their packed records and a list of
 * ZIPNN_MAX_PACKED exponents), and every payload stored RAW (a HUFF payload is
 * only chosen when it is smaller). Returns 0 for invalid arguments.
 * chunk_bytes: a multiple of 16 in [16, 2^28]. */
size_t zipnn_max_compressed_bytes(zipnn_dtype dtype, uint64_t n, uint32_t chunk_bytes);

/* Bytes of device scratch that compress, decompress and plan creation need for n
 * values; the same size serves every call on tensors of at most n values. */
size_t zipnn_workspace_bytes(zipnn_dtype dtype, uint64_t n, uint32_t chunk_bytes);

/* Compress n values at `src` (device) into the container at `out` (device, out_cap
 * bytes, out_cap >= zipnn_max_compressed_bytes). Each chunk_bytes of input is one
 * chunk with its own order-0 histogram and Huffman code (THEORY-599, "Order-0 only");
 * with a plan, a chunk takes the cheapest shared group code that covers its symbols
 * (NeuralZip, abstract), or a local code when none does. The container size is
 * written at out+48 (read it with zipnn_compressed_size). Sub-blocks of
 * ZIPNN_DEFAULT_SUBBLOCK symbols. */
zipnn_status zipnn_compress(zipnn_dtype dtype, const void* src, uint64_t n, uint32_t chunk_bytes,
                            const zipnn_plan_t* plan, void* out, size_t out_cap, void* ws,
                            size_t ws_bytes, zipnn_stream_t stream);

/* As zipnn_compress with an explicit sub-block length S (a multiple of 16 in
 * [16, 65536]; 0 selects ZIPNN_DEFAULT_SUBBLOCK). A shorter S gives the decoder more
 * parallel work at 32 bits of index per S symbols. */
zipnn_status zipnn_compress_ex(zipnn_dtype dtype, const void* src, uint64_t n, uint32_t chunk_bytes,
                               uint32_t subblock, const zipnn_plan_t* plan, void* out, size_t out_cap,
                               void* ws, size_t ws_bytes, zipnn_stream_t stream);

/* Decompress the container `in` (device, in_bytes readable bytes) into n values at
 * `out` (device): the inverse of zipnn_compress, giving back every value bit for bit
 * ("ZipNN: Lossless Compression for AI Models", abstract: lossless, with decompression
 * speed as a goal). Each chunk's streams are decoded and merged back into whole values
 * (the inverse of the split of THEORY-599, "Per-field compressibility (Table II)").
 * The container must have been made for the same dtype, n and chunk_bytes; anything
 * else, and any damage found, sets ZIPNN_ERR_CORRUPT in the workspace (output contents
 * are then unspecified). Every read stays inside in_bytes. ws: at least 256 bytes (only
 * its status word is used). */
zipnn_status zipnn_decompress(zipnn_dtype dtype, const void* in, size_t in_bytes, uint64_t n,
                              uint32_t chunk_bytes, void* out, void* ws, size_t ws_bytes,
                              zipnn_stream_t stream);

/* One tensor of a batched decompress: its container `in` (device, 16-byte aligned, in_bytes
 * readable), its value count n and its output `out` (device, 16-byte aligned, n values). */
typedef struct zipnn_decompress_item {
  const void* in;
  uint64_t in_bytes;
  uint64_t n;
  void* out;
} zipnn_decompress_item;

/* Workspace bytes for zipnn_decompress_batch of `count` tensors. */
size_t zipnn_decompress_batch_workspace_bytes(uint32_t count);

/* Decompress `count` containers of one dtype and chunk_bytes in a single launch: one block
 * per chunk over all the tensors' chunks, so that many small tensors fill the device
 * together ("ZipNN: Lossless Compression for AI Models", abstract: a model is many
 * tensors). Each output equals what zipnn_decompress gives for that item alone. `items`
 * is a host array, read before the call returns; its table is copied (stream-ordered)
 * into `ws`, which must hold zipnn_decompress_batch_workspace_bytes(count) and must not be
 * reused until the call completes. Argument errors (null or misaligned pointers, a count
 * of 0, n or chunk_bytes outside the limits of zipnn_compress, more than 2^31 - 1 chunks in
 * all) return synchronously before any launch. Damage found in any container sets
 * ZIPNN_ERR_CORRUPT in the workspace status (outputs are then unspecified). */
zipnn_status zipnn_decompress_batch(zipnn_dtype dtype, uint32_t chunk_bytes, uint32_t count,
                                    const zipnn_decompress_item* items, void* ws, size_t ws_bytes,
                                    zipnn_stream_t stream);

/* Wait for `stream`, then read the container size from the header at `out`. */
zipnn_status zipnn_compressed_size(const void* out, zipnn_stream_t stream, uint64_t* bytes);

/* Wait for `stream`, then return the device-side status of the last call on `ws`. */
zipnn_status zipnn_get_status(const void* ws, zipnn_stream_t stream);

/* Order-0 histograms (step "split + histogram" alone; THEORY-599 note, "Order-0 only
 * (section III-A b)": the model of a chunk is the count of each exponent value, no
 * context): hist_out (device, u32, 4-byte aligned) receives n_chunks x n_entropy
 * x 256 counts for the entropy streams of every chunk, symbols past a stream's alphabet
 * 0. Asynchronous; arguments as for zipnn_compress. */
zipnn_status zipnn_histogram(zipnn_dtype dtype, const void* src, uint64_t n, uint32_t chunk_bytes,
                             uint32_t* hist_out, zipnn_stream_t stream);

/* Code lengths (step "code build" alone; THEORY-599 note, "Order-0 only (section III-A
 * b)": a Huffman code built from the order-0 histogram): for `count` histograms of 256
 * u64 counts (device), writes 256 length bytes each (device): minimum-variance Huffman
 * lengths with ties by (weight, order), limited to ZIPNN_LMAX by halving the counts.
 * Counts are full 64-bit values (compared as (count, symbol) pairs); each histogram's
 * total must stay below 2^64. Symbols at or above `alphabet` (1..256) must have count 0.
 * count is at most 2^31 - 1. Asynchronous. */
zipnn_status zipnn_code_lengths(const uint64_t* hist, uint32_t count, uint32_t alphabet, uint8_t* lens_out,
                                zipnn_stream_t stream);

/* Build a plan ("NeuralZip: Reusable Setup for Fast Lossless Compression", abstract:
 * chunks with similar exponent distributions are grouped and share a Huffman code, and
 * this setup is prepared once, before the encodings that use it) on the tensor at `src`:
 * k-means (Lloyd, SplitMix64(seed) seeding, at most 100 passes) over the chunks'
 * normalised exponent histograms into `groups` groups (1..ZIPNN_MAX_GROUPS), then one
 * length-limited Huffman code per group and entropy stream from the group's summed
 * histograms. Setup call: it allocates the plan's device tables (the caller releases
 * them with zipnn_plan_destroy) and synchronises `stream`. ws as for compress. */
zipnn_status zipnn_plan_create(zipnn_dtype dtype, const void* src, uint64_t n, uint32_t chunk_bytes,
                               uint32_t groups, uint64_t seed, void* ws, size_t ws_bytes,
                               zipnn_stream_t stream, zipnn_plan_t** plan);

/* As zipnn_plan_create, and for BF16 with max_pack in 1..ZIPNN_MAX_PACKED also packed
 * exponents ("NeuralZip: Reusable Setup for Fast Lossless Compression", abstract: the
 * setup selectively represents recurring exponent tuples with packed exponents): the
 * plan lists the K = min(max_pack, exponents present) most frequent exponents of the
 * tensor (a larger count first, equal counts by the smaller exponent), and each group
 * gets a second, packed code: the length-limited Huffman code of its member chunks'
 * summed pair-symbol counts (chunks with an odd value count excluded; a group without
 * pairs gets none). A chunk coded with such a plan takes the shared code, plain or
 * packed, with the fewest bits (PACK in the container format). max_pack 0 is
 * zipnn_plan_create; max_pack > 0 for another dtype, or above ZIPNN_MAX_PACKED, is
 * ZIPNN_ERR_INVALID_ARG. */
zipnn_status zipnn_plan_create_packed(zipnn_dtype dtype, const void* src, uint64_t n, uint32_t chunk_bytes,
                                      uint32_t groups, uint64_t seed, uint32_t max_pack, void* ws, size_t ws_bytes,
                                      zipnn_stream_t stream, zipnn_plan_t** plan);

/* Serialise a plan into host memory, so that the setup can be stored and transferred
 * to other tensors or another compatible model (NeuralZip, abstract: the setup is
 * precomputed, transferred and reused as the weights evolve): "ZNP1", u8 dtype, u8
 * groups, u8 K (packed exponents, 0 for none), 1 zero byte, then the code section as in
 * the container (plain records; with K > 0 the packed records and the list). *bytes receives the
 * size; host_buf may be NULL to query it; ZIPNN_ERR_OUT_TOO_SMALL if cap is short. */
zipnn_status zipnn_plan_export(const zipnn_plan_t* plan, void* host_buf, size_t cap, size_t* bytes);

/* Rebuild a plan from exported bytes (host memory; NeuralZip, abstract: a transferred
 * setup is reused without being rebuilt); allocates its device tables. Records whose
 * lengths exceed ZIPNN_LMAX or whose Kraft sum exceeds 1, K above ZIPNN_MAX_PACKED (or
 * above 0 for a dtype other than BF16), a non-zero byte past the list, or a damaged
 * header, give ZIPNN_ERR_CORRUPT. */
zipnn_status zipnn_plan_import(const void* host_buf, size_t bytes, zipnn_plan_t** plan);

/* Per-chunk group chosen by the plan's k-means (NeuralZip, abstract: grouping of chunks
 * by exponent distribution) for the tensor the plan was built on (host memory, n_chunks
 * entries; empty for an imported plan); *count receives the number of entries. */
zipnn_status zipnn_plan_assignment(const zipnn_plan_t* plan, uint32_t* host_buf, size_t cap, size_t* count);

/* Release a plan and its device tables (NULL is ignored). */
void zipnn_plan_destroy(zipnn_plan_t* plan);

/* ---- One container from shards compressed on several GPUs ---------------------------
 * "ZipNN: Lossless Compression for AI Models" (abstract): a model's chunks are coded
 * independently, so a tensor splits across GPUs into contiguous ranges of whole chunks
 * (only the last range may end in a partial chunk). Each GPU compresses its range with
 * zipnn_compress as a tensor of its own (a shard container; the same dtype, chunk_bytes,
 * sub-block length and plan on every GPU). The container of the whole tensor is
 *   [header][chunk table][shared records][payloads of shard 0][payloads of shard 1]...
 * where shard r's relocated entries (zipnn_shard_tables) go to byte
 * 64 + 16 * n_streams * chunk_lo_r, the shared records are bytes off_codes..off_payload of
 * any shard's container (put at the whole container's off_codes), and shard r's payload
 * section (bytes off_payload..total_bytes of its container) starts at the whole
 * container's off_payload plus the payload bytes of the shards before it. The result
 * equals, byte for byte, the container that one call on the whole tensor writes. The only
 * exchange between GPUs is one u64 per shard and rank: an all-gather of the output of
 * zipnn_shard_sizes. The caller moves the bytes (a file write at each offset, or a copy). */
typedef struct zipnn_shard_item {
  const void* shard;    /* device, 16-byte aligned: the shard container */
  uint64_t shard_bytes; /* readable bytes at shard */
  uint64_t n_total;     /* values of the whole tensor */
  uint64_t chunk_lo;    /* index in the whole tensor of the shard's first chunk */
  void* table_out;      /* device, 16-byte aligned: 16 * n_streams * (shard's chunks) bytes */
  void* header_out;     /* device, 16-byte aligned, 64 bytes, or NULL: the whole header */
} zipnn_shard_item;

/* Workspace bytes (device, 16-byte aligned) for zipnn_shard_sizes / zipnn_shard_tables of
 * `count` items: a status word and a copy of the item table. */
size_t zipnn_shard_workspace_bytes(uint32_t count);

/* sizes_out[i] (device u64) = payload bytes (total_bytes - off_payload) of items[i].shard.
 * `items` is a host array read before the call returns. Asynchronous; a shard that is
 * not a container gets 0 and sets ZIPNN_ERR_CORRUPT in the workspace status. */
zipnn_status zipnn_shard_sizes(uint32_t count, const zipnn_shard_item* items, uint64_t* sizes_out, void* ws,
                               size_t ws_bytes, zipnn_stream_t stream);

/* For each item i of this rank: writes its chunk-table entries, payload offsets moved to
 * the whole container (the shard's payload base is the sum of all_sizes[r * count + i]
 * over ranks r < rank), to table_out, and when header_out is not NULL the whole container's
 * header (total_bytes = its off_payload plus the sum over all ranks). all_sizes: device,
 * world * count u64, rank-major (the all-gather of every rank's zipnn_shard_sizes). A shard
 * that is not the values [chunk_lo * m0, ...) of a tensor of n_total values with this dtype
 * and chunk_bytes, or whose size differs from all_sizes, sets ZIPNN_ERR_CORRUPT (nothing is
 * written for it). Asynchronous. */
zipnn_status zipnn_shard_tables(zipnn_dtype dtype, uint32_t chunk_bytes, uint32_t count, const zipnn_shard_item* items,
                                const uint64_t* all_sizes, uint32_t rank, uint32_t world, void* ws, size_t ws_bytes,
                                zipnn_stream_t stream);

/* Compress without allocating (the pages have no counterpart of this call). For callers
 * that cannot allocate device memory: code whose device memory is owned by a framework's
 * caching allocator that it cannot reach from C (a cudaMalloc of its own would fight
 * that allocator for memory it has already reserved), and latency-critical paths that
 * cannot afford the device synchronisation a cudaMalloc/cudaFree pair implies. It
 * behaves as zipnn_compress without a
 * plan, but its workspace is a file-scope device array of ZIPNN_NOALLOC_SCRATCH_BYTES
 * (8 MiB) that every GPU loading the library holds until the process exits; tensors
 * whose zipnn_workspace_bytes exceed it are rejected with ZIPNN_ERR_UNSUPPORTED before
 * anything is launched. The caller still passes input and output. The first call on a
 * device looks up the array's device address with that device current, so make the
 * first call before any stream capture. All calls on a device share the array and it
 * keeps the previous call's contents (each call clears what must start at zero): calls
 * that may overlap on the GPU race, so issue them on one stream or order them. */
#define ZIPNN_NOALLOC_SCRATCH_BYTES (8u << 20)
zipnn_status zipnn_compress_noalloc(zipnn_dtype dtype, const void* src, uint64_t n, uint32_t chunk_bytes, void* out,
                                    size_t out_cap, zipnn_stream_t stream);

/* Test aid (not a step of the codec): the number of polls after which a wait on another
 * block of the same launch (the decoupled look-back of the layout scan) gives up and
 * records ZIPNN_ERR_TIMEOUT; 0 restores the default
 * (2^22). It applies to calls made after it, in every host thread. A wait that gives up
 * has summed only part of its prefix, so every offset it yields is at most the true one
 * and every write stays inside the output; the container is then invalid and the status
 * says so. Always returns ZIPNN_OK. */
zipnn_status zipnn_test_lookback_limit(uint32_t polls);

/* Kernel timing, a measurement aid (off by default; not a step of the codec). While
 * enabled, every kernel the library launches is bracketed by two CUDA events on its
 * stream. zipnn_timing_collect waits for the recorded events and writes, for kernel
 * ids 0..count-1, the summed duration in ms and the number of launches since the last
 * collect (either pointer may be NULL), then resets the totals. */
zipnn_status zipnn_timing_enable(int enable);
zipnn_status zipnn_timing_collect(double* ms, uint64_t* launches, uint32_t count);
uint32_t zipnn_kernel_count(void);
const char* zipnn_kernel_name(uint32_t id);

const char* zipnn_status_string(zipnn_status status);

#ifdef __cplusplus
}
#endif
#endif

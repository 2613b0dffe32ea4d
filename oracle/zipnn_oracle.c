/*
 * zipnn_oracle.c -- plain, slow, obviously-correct CPU oracle for the ZipNN-style
 * float-tensor codec.
 *
 * TEST INFRASTRUCTURE. Only tests, the smoke check and the benchmark's CPU baseline
 * load this file's library. The product (the CUDA library) shares nothing with it:
 * no header, no helper, no table. Everything here is written out step by step, in
 * the order the method states it, with no blocking or fusion.
 *
 * Method, by page title and section:
 *  - Field split: "ZipNN: Lossless Compression for AI Models", abstract; THEORY-599
 *    note, "Per-field compressibility (Table II)": the exponent field compresses,
 *    the sign and fraction bytes do not.
 *  - Order-0 histogram and Huffman code per chunk: THEORY-599 note, "Order-0 only
 *    (section III-A b)": Huffman after exponent extraction, no context model.
 *  - FP8 exponent and mantissa coded independently: "Lossless Compression of Neural
 *    Network Components: Weights, Checkpoints, and K/V Caches in Low-Precision
 *    Formats", abstract.
 *  - Grouped chunks with shared Huffman codes from a reusable setup: "NeuralZip:
 *    Reusable Setup for Fast Lossless Compression", abstract.
 *
 * Readings where the pages are silent:
 *  - Huffman ties: the two nodes with the smallest (weight, order) keys merge first;
 *    a leaf's order is its symbol value, the i-th merged node's order is 256 + i.
 *  - Length limit 12: halve every non-zero frequency (never below 1) and rebuild,
 *    until the longest code is at most 12 bits.
 *  - Canonical code values: the deflate rule (RFC 1951, section 3.2.2).
 *  - Container layout, sub-block index, ZERO/RAW/HUFF choice: the format stated under
 *    "layout rules" below; pinned by a hand-derived golden container, not by the pages.
 *  - Grouping: Lloyd's k-means with SplitMix64 seeding (parity unpinned by the pages:
 *    pinned only by invariants and small separable cases).
 *  - Packed exponent tuples (NeuralZip, abstract: recurring exponent tuples represented
 *    by packed exponents, chosen by the setup; the pages give no format). Reading, BF16
 *    only: the setup lists the K <= 15 most frequent exponents of its tensor; a pair of
 *    exponents at values (2j, 2j+1) becomes one 8-bit symbol, the two list indices as
 *    nibbles (first value high), 15 for an exponent not in the list, whose 8 bits then
 *    follow the pair's code. Each group gets a second code over these pair symbols, and
 *    a chunk takes whichever shared code, plain or packed, codes it in the fewest bits.
 */
#include "zipnn_oracle.h"

#include <pthread.h>
#include <stdlib.h>
#include <string.h>

#define LMAX 12
#define MAX_GROUPS 64
#define HEADER_BYTES 64
#define ENTRY_BYTES 16
#define MODE_RAW 0
#define MODE_ZERO 1
#define MODE_HUFF 2
#define MODE_ZRUN 3
#define MODE_PACK 4
#define PACK_MAX 15   /* packed exponents a plan may list; nibble 15 is the escape */
#define PACK_ESC 15
#define PACK_LIST_BYTES 16
#define ZRUN_BLOCK 32 /* symbols of one zero-run block */
#define NO_CODE 0xFFFFFFFFu

/* ------------------------------------------------------------------ field map */

int orc_n_streams(int dtype) { return dtype == ORC_BF16 ? 2 : dtype == ORC_FP32 ? 4 : 3; }
/* FP8 and FP4: exponent and mantissa are entropy-coded independently */
int orc_n_entropy(int dtype) { return dtype == ORC_FP8 || dtype == ORC_FP4 ? 2 : 1; }
/* bytes of one value (FP4: two values share a byte; see chunk_values) */
static int value_bytes(int dtype) { return dtype == ORC_BF16 ? 2 : dtype == ORC_FP32 ? 4 : 1; }
static int is_entropy(int dtype, int s) { return s == 0 || ((dtype == ORC_FP8 || dtype == ORC_FP4) && s == 1); }
/* bits per symbol when a stream is stored RAW */
static int raw_width(int dtype, int s) {
  if (dtype == ORC_FP8) return s == 0 ? 4 : s == 1 ? 3 : 1;
  if (dtype == ORC_FP4) return s == 0 ? 2 : 1;
  return 8;
}
int orc_alphabet(int dtype, int s) { return 1 << raw_width(dtype, s); }
/* bytes of one packed code record (4-bit lengths), rounded up to 16 */
static uint64_t round16(uint64_t x) { return (x + 15) & ~(uint64_t)15; }
static uint64_t record_bytes(int dtype, int s) { return round16((uint64_t)orc_alphabet(dtype, s) / 2); }

/* The split. BF16 w: exponent = bits 14..7; sign+fraction byte = sign in bit 7,
 * fraction bits 6..0. FP32 u: exponent = bits 30..23; p1 = sign + fraction bits
 * 22..16; p2 = fraction bits 15..8; p3 = bits 7..0. FP8 E4M3 b: exponent bits 6..3,
 * mantissa bits 2..0, sign bit 7. FP4 E2M1: value i is the low nibble of byte i/2
 * when i is even, the high nibble when odd; exponent = nibble bits 2..1, mantissa =
 * bit 0, sign = bit 3. Streams are numbered in that order. */
uint8_t orc_field(int dtype, const uint8_t* src, uint64_t i, int s) {
  if (dtype == ORC_BF16) {
    uint32_t w = (uint32_t)src[2 * i] | ((uint32_t)src[2 * i + 1] << 8);
    if (s == 0) return (uint8_t)((w >> 7) & 0xFF);
    return (uint8_t)(((w >> 8) & 0x80) | (w & 0x7F));
  }
  if (dtype == ORC_FP32) {
    uint32_t u = (uint32_t)src[4 * i] | ((uint32_t)src[4 * i + 1] << 8) |
                 ((uint32_t)src[4 * i + 2] << 16) | ((uint32_t)src[4 * i + 3] << 24);
    if (s == 0) return (uint8_t)((u >> 23) & 0xFF);
    if (s == 1) return (uint8_t)(((u >> 24) & 0x80) | ((u >> 16) & 0x7F));
    if (s == 2) return (uint8_t)((u >> 8) & 0xFF);
    return (uint8_t)(u & 0xFF);
  }
  if (dtype == ORC_FP4) {
    uint32_t v = (src[i / 2] >> (4 * (i % 2))) & 0xF;
    if (s == 0) return (uint8_t)((v >> 1) & 3);
    if (s == 1) return (uint8_t)(v & 1);
    return (uint8_t)(v >> 3);
  }
  {
    uint32_t b = src[i];
    if (s == 0) return (uint8_t)((b >> 3) & 0xF);
    if (s == 1) return (uint8_t)(b & 7);
    return (uint8_t)(b >> 7);
  }
}

/* The merge: the inverse of the split, writing value i. */
static void put_value(int dtype, uint8_t* dst, uint64_t i, const uint8_t* f) {
  if (dtype == ORC_BF16) {
    uint32_t w = ((uint32_t)(f[1] & 0x80) << 8) | ((uint32_t)f[0] << 7) | (f[1] & 0x7F);
    dst[2 * i] = (uint8_t)(w & 0xFF);
    dst[2 * i + 1] = (uint8_t)(w >> 8);
  } else if (dtype == ORC_FP32) {
    uint32_t u = ((uint32_t)(f[1] & 0x80) << 24) | ((uint32_t)f[0] << 23) |
                 ((uint32_t)(f[1] & 0x7F) << 16) | ((uint32_t)f[2] << 8) | f[3];
    dst[4 * i] = (uint8_t)(u & 0xFF);
    dst[4 * i + 1] = (uint8_t)((u >> 8) & 0xFF);
    dst[4 * i + 2] = (uint8_t)((u >> 16) & 0xFF);
    dst[4 * i + 3] = (uint8_t)(u >> 24);
  } else if (dtype == ORC_FP4) {
    uint32_t v = ((uint32_t)f[2] << 3) | ((uint32_t)f[0] << 1) | f[1];
    uint32_t sh = 4 * (uint32_t)(i % 2);
    dst[i / 2] = (uint8_t)((dst[i / 2] & ~(0xFu << sh)) | (v << sh));
  } else {
    dst[i] = (uint8_t)((f[2] << 7) | (f[0] << 3) | f[1]);
  }
}

void orc_histogram(int dtype, const uint8_t* src, uint64_t lo, uint64_t hi, int s, uint64_t* hist) {
  int a = orc_alphabet(dtype, s);
  for (int k = 0; k < a; k++) hist[k] = 0;
  for (uint64_t i = lo; i < hi; i++) hist[orc_field(dtype, src, i, s)]++;
}

/* ------------------------------------------------------------------ Huffman */

/* Huffman code lengths. Every present symbol is a node with key (weight, order).
 * Repeatedly take out the two nodes with the smallest keys and put back one node
 * whose weight is their sum; the i-th such node gets order 256 + i. A symbol's
 * length is the depth of its leaf. A lone symbol gets length 1. */
int orc_huffman_lengths(const uint64_t* freq, int alphabet, uint8_t* len) {
  uint64_t w[512];
  uint32_t order[512];
  int parent[512], alive[512], leaf_of[256];
  int nodes = 0, leaves = 0;
  if (alphabet < 1 || alphabet > 256) return ORC_EINVAL;
  for (int s = 0; s < alphabet; s++) {
    len[s] = 0;
    leaf_of[s] = -1;
    if (freq[s] > 0) {
      w[nodes] = freq[s];
      order[nodes] = (uint32_t)s;
      parent[nodes] = -1;
      alive[nodes] = 1;
      leaf_of[s] = nodes;
      nodes++;
      leaves++;
    }
  }
  if (leaves == 0) return ORC_OK;
  if (leaves == 1) {
    for (int s = 0; s < alphabet; s++)
      if (leaf_of[s] >= 0) len[s] = 1;
    return ORC_OK;
  }
  for (int merged = 0; merged < leaves - 1; merged++) {
    int pick[2];
    for (int t = 0; t < 2; t++) {
      int best = -1;
      for (int j = 0; j < nodes; j++) {
        if (!alive[j]) continue;
        if (best < 0 || w[j] < w[best] || (w[j] == w[best] && order[j] < order[best])) best = j;
      }
      alive[best] = 0;
      pick[t] = best;
    }
    w[nodes] = w[pick[0]] + w[pick[1]];
    order[nodes] = 256u + (uint32_t)merged;
    parent[nodes] = -1;
    alive[nodes] = 1;
    parent[pick[0]] = nodes;
    parent[pick[1]] = nodes;
    nodes++;
  }
  for (int s = 0; s < alphabet; s++) {
    if (leaf_of[s] < 0) continue;
    int depth = 0;
    for (int j = leaf_of[s]; parent[j] >= 0; j = parent[j]) depth++;
    len[s] = (uint8_t)depth;
  }
  return ORC_OK;
}

/* Lengths limited to lmax: with k = 0, 1, 2, ... build the code for the frequencies
 * max(1, f >> k) (zero stays zero) and keep the first one whose longest code fits. */
int orc_limited_lengths(const uint64_t* freq, int alphabet, int lmax, uint8_t* len) {
  uint64_t g[256];
  if (alphabet < 1 || alphabet > 256 || lmax < 1) return ORC_EINVAL;
  for (int k = 0; k < 64; k++) {
    int longest = 0;
    for (int s = 0; s < alphabet; s++) {
      if (freq[s] == 0) g[s] = 0;
      else g[s] = (freq[s] >> k) > 0 ? (freq[s] >> k) : 1;
    }
    orc_huffman_lengths(g, alphabet, len);
    for (int s = 0; s < alphabet; s++)
      if (len[s] > longest) longest = len[s];
    if (longest <= lmax) return ORC_OK;
  }
  return ORC_EINVAL; /* unreachable for alphabets up to 2^lmax symbols */
}

/* Canonical code values, RFC 1951 section 3.2.2: count the codes of each length,
 * compute the first code of each length, then number the symbols in increasing
 * order within each length. */
void orc_canonical_codes(const uint8_t* len, int alphabet, uint32_t* code) {
  uint32_t count[16] = {0}, next[16] = {0};
  for (int s = 0; s < alphabet; s++)
    if (len[s]) count[len[s]]++;
  uint32_t c = 0;
  count[0] = 0;
  for (int bits = 1; bits < 16; bits++) {
    c = (c + count[bits - 1]) << 1;
    next[bits] = c;
  }
  for (int s = 0; s < alphabet; s++) code[s] = len[s] ? next[len[s]]++ : 0;
}

/* ------------------------------------------------------------------ bit I/O */

/* Bit t of a bit string is bit (7 - t mod 8) of byte t / 8: most significant first. */
static void put_bits(uint8_t* buf, uint64_t* t, uint32_t value, int nbits) {
  for (int b = nbits - 1; b >= 0; b--) {
    if ((value >> b) & 1u) buf[*t >> 3] |= (uint8_t)(0x80u >> (*t & 7));
    (*t)++;
  }
}

static int get_bit(const uint8_t* buf, uint64_t cap_bits, uint64_t* t) {
  if (*t >= cap_bits) return -1;
  int bit = (buf[*t >> 3] >> (7 - (*t & 7))) & 1;
  (*t)++;
  return bit;
}

static void put_u32(uint8_t* p, uint32_t v) {
  for (int i = 0; i < 4; i++) p[i] = (uint8_t)(v >> (8 * i));
}
static void put_u64(uint8_t* p, uint64_t v) {
  for (int i = 0; i < 8; i++) p[i] = (uint8_t)(v >> (8 * i));
}
static uint32_t get_u32(const uint8_t* p) {
  uint32_t v = 0;
  for (int i = 0; i < 4; i++) v |= (uint32_t)p[i] << (8 * i);
  return v;
}
static uint64_t get_u64(const uint8_t* p) {
  uint64_t v = 0;
  for (int i = 0; i < 8; i++) v |= (uint64_t)p[i] << (8 * i);
  return v;
}

/* ------------------------------------------------------------------ layout rules */
/*
 * The container (little-endian; every section and payload starts on a 16-byte
 * boundary; every pad byte and pad bit is zero):
 *  - header, 64 bytes: "ZN" "N1"; version 1 (u16); dtype (u8); streams per chunk (u8);
 *    n values (u64); chunk_bytes (u32); S (u32); chunks (u32); shared records (u32);
 *    offset of the code section (u64); offset of the payloads (u64); total bytes
 *    (u64); L_MAX = 12 (u8); groups (u8); zeros to byte 64;
 *  - chunk table, 16 bytes per entry k = chunk * streams + stream: mode (u8: RAW 0,
 *    ZERO 1, HUFF 2) and three zero bytes; code (u32: the shared record's index, or
 *    0xFFFFFFFF for a code of the chunk's own); payload offset (u64);
 *  - code section: the shared records, those of entropy stream 0 for every group,
 *    then stream 1's; a record is the alphabet's code lengths, 4 bits each (symbol
 *    2i in the low nibble of byte i), rounded up to 16 bytes;
 *  - payloads in entry order, each offset the sum of the sizes before it: RAW, the
 *    stream's symbols at their fixed width, MSB first; ZERO, nothing; HUFF, the
 *    chunk's own record (when code is 0xFFFFFFFF), then the bit offset (u32) of every
 *    S-th symbol padded to 16 bytes, then the codes MSB first padded to 16 bytes;
 *    ZRUN (mode 3, zero runs of a byte plane), the chunk's symbols taken in blocks of 32
 *    (the last block may be shorter): one bit per block, MSB first, 1 when the block
 *    holds a non-zero symbol, padded to 16 bytes, then the symbols of the marked blocks
 *    in order, padded to 16 bytes.
 *  - packed exponents (BF16 with a plan that lists K > 0 exponents): header byte 58 is
 *    K; the code section holds, after the plain records, one packed record per group
 *    (a code over the 256 pair symbols), then the K listed exponents padded to 16 bytes;
 *    a PACK entry (mode 4, code = groups + g) holds the bit offset (u32) of every S-th
 *    value's pair padded to 16 bytes, then for every pair its code followed by the raw
 *    8 bits of each escaped exponent (first, then second), MSB first, padded to 16 bytes.
 *  - choice for a stream: ZERO when every symbol is 0. An entropy stream is HUFF when
 *    that payload is strictly smaller than RAW, else RAW. A byte plane (8-bit symbols
 *    that are not entropy-coded: BF16's sign/fraction byte, FP32's three fraction
 *    planes) is ZRUN when that payload is strictly smaller than RAW, else RAW. The 1-bit
 *    sign streams of FP8 and FP4 are RAW.
 */

static uint64_t ceil_div(uint64_t a, uint64_t b) { return (a + b - 1) / b; }

static uint64_t chunk_values(int dtype, uint32_t chunk_bytes) {
  return dtype == ORC_FP4 ? 2 * (uint64_t)chunk_bytes : chunk_bytes / (uint32_t)value_bytes(dtype);
}
/* FP4 values come in byte pairs */
static int bad_count(int dtype, uint64_t n) { return n == 0 || (dtype == ORC_FP4 && n % 2 != 0); }

static uint64_t table_end(int dtype, uint64_t n_chunks) {
  return HEADER_BYTES + (uint64_t)ENTRY_BYTES * n_chunks * (uint64_t)orc_n_streams(dtype);
}

/* bytes of all plain shared code records for n_groups groups */
static uint64_t shared_bytes(int dtype, uint32_t n_groups) {
  uint64_t b = 0;
  for (int s = 0; s < orc_n_entropy(dtype); s++) b += (uint64_t)n_groups * record_bytes(dtype, s);
  return b;
}

/* the code section with K packed exponents: plain records, packed records, the list */
static uint64_t code_section_bytes(int dtype, uint32_t n_groups, uint32_t K) {
  uint64_t b = shared_bytes(dtype, n_groups);
  if (K) b += (uint64_t)n_groups * record_bytes(dtype, 0) + PACK_LIST_BYTES;
  return b;
}

/* byte position of group g's packed record inside the code section */
static uint64_t packed_record_pos(int dtype, uint32_t n_groups, uint32_t g) {
  return shared_bytes(dtype, n_groups) + (uint64_t)g * record_bytes(dtype, 0);
}

/* byte position of shared record r = e * n_groups + g inside the code section */
static uint64_t shared_record_pos(int dtype, uint32_t n_groups, uint32_t r) {
  uint32_t e = r / n_groups, g = r % n_groups;
  uint64_t pos = 0;
  for (uint32_t k = 0; k < e; k++) pos += (uint64_t)n_groups * record_bytes(dtype, (int)k);
  return pos + (uint64_t)g * record_bytes(dtype, (int)e);
}

static uint64_t raw_payload_bytes(uint64_t m, int width) { return round16(ceil_div(m * (uint64_t)width, 8)); }

/* header, table, code section and every payload stored RAW: a HUFF, PACK or ZRUN
 * payload is only chosen when it is smaller */
uint64_t orc_max_compressed_bytes_packed(int dtype, uint64_t n, uint32_t chunk_bytes, uint32_t n_groups, uint32_t K) {
  uint64_t m0 = chunk_values(dtype, chunk_bytes);
  if (m0 == 0 || n == 0) return 0;
  uint64_t chunks = ceil_div(n, m0);
  uint64_t total = table_end(dtype, chunks) + code_section_bytes(dtype, n_groups, K);
  for (uint64_t c = 0; c < chunks; c++) {
    uint64_t m = (c + 1) * m0 <= n ? m0 : n - c * m0;
    for (int s = 0; s < orc_n_streams(dtype); s++) total += raw_payload_bytes(m, raw_width(dtype, s));
  }
  return total;
}

uint64_t orc_max_compressed_bytes(int dtype, uint64_t n, uint32_t chunk_bytes, uint32_t n_groups) {
  return orc_max_compressed_bytes_packed(dtype, n, chunk_bytes, n_groups, 0);
}

/* Nibble of exponent x in a pair symbol: its index in the plan's list, else the escape. */
static uint32_t pack_nibble(uint8_t x, const uint8_t* exps, uint32_t K) {
  for (uint32_t i = 0; i < K; i++)
    if (exps[i] == x) return i;
  return PACK_ESC;
}

/* Pair symbols of the BF16 values [lo, lo + m) (m even): the exponents of values
 * lo + 2j and lo + 2j + 1 give symbol nibble(first) << 4 | nibble(second). hist (256)
 * receives the symbol counts and *escapes the number of escaped exponents. */
void orc_pack_histogram(const void* src, uint64_t lo, uint64_t m, const uint8_t* exps, uint32_t K, uint64_t* hist,
                        uint64_t* escapes) {
  const uint8_t* in = (const uint8_t*)src;
  for (int k = 0; k < 256; k++) hist[k] = 0;
  *escapes = 0;
  for (uint64_t j = 0; j + 1 < m; j += 2) {
    uint32_t a = pack_nibble(orc_field(ORC_BF16, in, lo + j, 0), exps, K);
    uint32_t b = pack_nibble(orc_field(ORC_BF16, in, lo + j + 1, 0), exps, K);
    hist[(a << 4) | b]++;
    *escapes += (a == PACK_ESC) + (b == PACK_ESC);
  }
}

/* ------------------------------------------------------------------ compress */

typedef struct {
  uint8_t mode;
  uint32_t code; /* shared record index, or NO_CODE */
  uint64_t size;
  uint8_t* bytes; /* size bytes, owned */
} entry_t;

typedef struct {
  int dtype;
  const uint8_t* src;
  uint64_t n, m0, chunks;
  uint32_t S;
  const uint8_t* plan_lens;
  uint32_t n_groups;
  const uint8_t* pack_lens; /* n_groups x 256 packed-code lengths, when K > 0 */
  const uint8_t* pack_exps; /* the K listed exponents */
  uint32_t K;
  entry_t* entries;
  int thread, threads;
  int status;
} job_t;

/* Encode stream s of one chunk (values [lo, lo + m)) into one entry. */
static int encode_entry(const job_t* jb, uint64_t lo, uint64_t m, int s, entry_t* en) {
  int dt = jb->dtype, a = orc_alphabet(dt, s), w = raw_width(dt, s);
  uint8_t* sym = (uint8_t*)malloc(m);
  uint8_t len[256];
  uint32_t code[256];
  uint64_t hist[256];
  if (!sym) return ORC_EINVAL;
  int all_zero = 1;
  for (uint64_t i = 0; i < m; i++) {
    sym[i] = orc_field(dt, jb->src, lo + i, s);
    if (sym[i]) all_zero = 0;
  }
  en->code = NO_CODE;
  en->bytes = NULL;
  en->size = 0;
  if (all_zero) {
    en->mode = MODE_ZERO;
    free(sym);
    return ORC_OK;
  }
  uint64_t p_raw = raw_payload_bytes(m, w);
  en->mode = MODE_RAW;
  if (is_entropy(dt, s)) {
    int e = s; /* entropy streams are streams 0 (and 1 for FP8) */
    for (int k = 0; k < a; k++) hist[k] = 0;
    for (uint64_t i = 0; i < m; i++) hist[sym[i]]++;
    int use_group = -1;
    uint64_t best_bits = 0;
    if (jb->plan_lens) {
      /* a group is eligible if its code has a length for every present symbol;
       * the one with the fewest coded bits wins, ties to the smaller group */
      for (uint32_t g = 0; g < jb->n_groups; g++) {
        const uint8_t* lg = jb->plan_lens + ((uint64_t)e * jb->n_groups + g) * 256;
        int ok = 1;
        uint64_t bits = 0;
        for (int k = 0; k < a; k++) {
          if (hist[k] == 0) continue;
          if (lg[k] == 0) ok = 0;
          bits += hist[k] * lg[k];
        }
        if (ok && (use_group < 0 || bits < best_bits)) {
          use_group = (int)g;
          best_bits = bits;
        }
      }
    }
    /* packed exponents (BF16 exponent stream, even chunk and sub-block lengths): each
     * group's packed code competes with the plain codes; strictly fewer bits win */
    int use_pack = -1;
    if (jb->plan_lens && jb->K && dt == ORC_BF16 && s == 0 && m % 2 == 0 && jb->S % 2 == 0) {
      uint64_t hp[256], esc = 0;
      orc_pack_histogram(jb->src, lo, m, jb->pack_exps, jb->K, hp, &esc);
      for (uint32_t g = 0; g < jb->n_groups; g++) {
        const uint8_t* lp = jb->pack_lens + (uint64_t)g * 256;
        int ok = 1;
        uint64_t bits = 8 * esc;
        for (int k = 0; k < 256; k++) {
          if (hp[k] == 0) continue;
          if (lp[k] == 0) ok = 0;
          bits += hp[k] * lp[k];
        }
        if (ok && ((use_group < 0 && use_pack < 0) || bits < best_bits)) {
          use_pack = (int)g;
          best_bits = bits;
        }
      }
      if (use_pack >= 0) use_group = -1;
    }
    if (use_pack >= 0) {
      const uint8_t* lp = jb->pack_lens + (uint64_t)use_pack * 256;
      uint64_t nsub = ceil_div(m, jb->S);
      uint64_t p_pack = round16(4 * nsub) + round16(ceil_div(best_bits, 8));
      if (p_pack < p_raw) {
        en->mode = MODE_PACK;
        en->code = jb->n_groups * (uint32_t)orc_n_entropy(dt) + (uint32_t)use_pack;
        en->size = p_pack;
        en->bytes = (uint8_t*)calloc(p_pack, 1);
        if (!en->bytes) {
          free(sym);
          return ORC_EINVAL;
        }
        orc_canonical_codes(lp, 256, code);
        uint8_t* bs = en->bytes + round16(4 * nsub);
        uint64_t t = 0;
        for (uint64_t i = 0; i < m; i += 2) {
          if (i % jb->S == 0) put_u32(en->bytes + 4 * (i / jb->S), (uint32_t)t);
          uint32_t a = pack_nibble(sym[i], jb->pack_exps, jb->K), b = pack_nibble(sym[i + 1], jb->pack_exps, jb->K);
          uint32_t ps = (a << 4) | b;
          put_bits(bs, &t, code[ps], lp[ps]);
          if (a == PACK_ESC) put_bits(bs, &t, sym[i], 8);
          if (b == PACK_ESC) put_bits(bs, &t, sym[i + 1], 8);
        }
        free(sym);
        return ORC_OK;
      }
    }
    if (use_pack < 0) {
      if (use_group >= 0) memcpy(len, jb->plan_lens + ((uint64_t)e * jb->n_groups + (uint32_t)use_group) * 256, 256);
      else orc_limited_lengths(hist, a, LMAX, len);
      uint64_t bits = 0;
      for (int k = 0; k < a; k++) bits += hist[k] * len[k];
      uint64_t nsub = ceil_div(m, jb->S);
      uint64_t rec = use_group >= 0 ? 0 : record_bytes(dt, s);
      uint64_t p_huff = rec + round16(4 * nsub) + round16(ceil_div(bits, 8));
      if (p_huff < p_raw) {
        en->mode = MODE_HUFF;
        en->code = use_group >= 0 ? (uint32_t)e * jb->n_groups + (uint32_t)use_group : NO_CODE;
        en->size = p_huff;
        en->bytes = (uint8_t*)calloc(p_huff, 1);
        if (!en->bytes) {
          free(sym);
          return ORC_EINVAL;
        }
        uint8_t* p = en->bytes;
        if (rec) {
          for (int k = 0; k < a / 2; k++) p[k] = (uint8_t)(len[2 * k] | (len[2 * k + 1] << 4));
          p += rec;
        }
        orc_canonical_codes(len, a, code);
        uint8_t* bs = p + round16(4 * nsub);
        uint64_t t = 0;
        for (uint64_t i = 0; i < m; i++) {
          if (i % jb->S == 0) put_u32(p + 4 * (i / jb->S), (uint32_t)t);
          put_bits(bs, &t, code[sym[i]], len[sym[i]]);
        }
        free(sym);
        return ORC_OK;
      }
    }
  }
  if (!is_entropy(dt, s) && w == 8) {
    /* zero runs of a byte plane: mark every block of 32 symbols that holds a non-zero
     * one; keep only the marked blocks' symbols */
    uint64_t blocks = ceil_div(m, ZRUN_BLOCK), kept = 0;
    for (uint64_t b = 0; b < blocks; b++) {
      uint64_t lo = b * ZRUN_BLOCK, hi = lo + ZRUN_BLOCK < m ? lo + ZRUN_BLOCK : m;
      int marked = 0;
      for (uint64_t i = lo; i < hi; i++)
        if (sym[i]) marked = 1;
      if (marked) kept += hi - lo;
    }
    uint64_t map_bytes = round16(ceil_div(blocks, 8));
    uint64_t p_zrun = map_bytes + round16(ceil_div(kept * (uint64_t)w, 8));
    if (p_zrun < p_raw) {
      en->mode = MODE_ZRUN;
      en->size = p_zrun;
      en->bytes = (uint8_t*)calloc(p_zrun, 1);
      if (!en->bytes) {
        free(sym);
        return ORC_EINVAL;
      }
      uint64_t tm = 0, td = 0;
      for (uint64_t b = 0; b < blocks; b++) {
        uint64_t lo = b * ZRUN_BLOCK, hi = lo + ZRUN_BLOCK < m ? lo + ZRUN_BLOCK : m;
        int marked = 0;
        for (uint64_t i = lo; i < hi; i++)
          if (sym[i]) marked = 1;
        put_bits(en->bytes, &tm, (uint32_t)marked, 1);
        if (marked)
          for (uint64_t i = lo; i < hi; i++) put_bits(en->bytes + map_bytes, &td, sym[i], w);
      }
      free(sym);
      return ORC_OK;
    }
  }
  en->mode = MODE_RAW;
  en->size = p_raw;
  en->bytes = (uint8_t*)calloc(p_raw, 1);
  if (!en->bytes) {
    free(sym);
    return ORC_EINVAL;
  }
  uint64_t t = 0;
  for (uint64_t i = 0; i < m; i++) put_bits(en->bytes, &t, sym[i], w);
  free(sym);
  return ORC_OK;
}

static void* compress_worker(void* arg) {
  job_t* jb = (job_t*)arg;
  int ns = orc_n_streams(jb->dtype);
  for (uint64_t c = (uint64_t)jb->thread; c < jb->chunks; c += (uint64_t)jb->threads) {
    uint64_t lo = c * jb->m0;
    uint64_t m = lo + jb->m0 <= jb->n ? jb->m0 : jb->n - lo;
    for (int s = 0; s < ns; s++) {
      int st = encode_entry(jb, lo, m, s, &jb->entries[c * (uint64_t)ns + (uint64_t)s]);
      if (st != ORC_OK) jb->status = st;
    }
  }
  return NULL;
}

static int run_jobs(job_t* base, int threads, void* (*fn)(void*)) {
  if (threads < 1) threads = 1;
  if (threads > 256) threads = 256;
  job_t* jobs = (job_t*)malloc(sizeof(job_t) * (size_t)threads);
  pthread_t* th = (pthread_t*)malloc(sizeof(pthread_t) * (size_t)threads);
  if (!jobs || !th) {
    free(jobs);
    free(th);
    return ORC_EINVAL;
  }
  for (int t = 0; t < threads; t++) {
    jobs[t] = *base;
    jobs[t].thread = t;
    jobs[t].threads = threads;
    jobs[t].status = ORC_OK;
  }
  for (int t = 1; t < threads; t++) pthread_create(&th[t], NULL, fn, &jobs[t]);
  fn(&jobs[0]);
  for (int t = 1; t < threads; t++) pthread_join(th[t], NULL);
  int st = ORC_OK;
  for (int t = 0; t < threads; t++)
    if (jobs[t].status != ORC_OK) st = jobs[t].status;
  free(jobs);
  free(th);
  return st;
}

int orc_compress(int dtype, const void* src, uint64_t n, uint32_t chunk_bytes, uint32_t S,
                 const uint8_t* plan_lens, uint32_t n_groups, void* out, uint64_t cap,
                 uint64_t* out_bytes, int threads) {
  return orc_compress_packed(dtype, src, n, chunk_bytes, S, plan_lens, n_groups, NULL, NULL, 0, out, cap, out_bytes,
                             threads);
}

int orc_compress_packed(int dtype, const void* src, uint64_t n, uint32_t chunk_bytes, uint32_t S,
                        const uint8_t* plan_lens, uint32_t n_groups, const uint8_t* pack_lens,
                        const uint8_t* pack_exps, uint32_t K, void* out, uint64_t cap, uint64_t* out_bytes,
                        int threads) {
  if (dtype < 0 || dtype > 3 || !src || !out || bad_count(dtype, n) || S == 0) return ORC_EINVAL;
  if (chunk_bytes == 0 || chunk_bytes % (uint32_t)value_bytes(dtype) != 0) return ORC_EINVAL;
  if (plan_lens && (n_groups == 0 || n_groups > MAX_GROUPS)) return ORC_EINVAL;
  if (!plan_lens) n_groups = 0;
  if (K > PACK_MAX || (K && (dtype != ORC_BF16 || !plan_lens || !pack_lens || !pack_exps))) return ORC_EINVAL;
  int ns = orc_n_streams(dtype);
  uint64_t m0 = chunk_values(dtype, chunk_bytes);
  uint64_t chunks = ceil_div(n, m0);
  if (cap < orc_max_compressed_bytes_packed(dtype, n, chunk_bytes, n_groups, K)) return ORC_ESMALL;
  entry_t* entries = (entry_t*)calloc(chunks * (uint64_t)ns, sizeof(entry_t));
  if (!entries) return ORC_EINVAL;
  job_t jb;
  memset(&jb, 0, sizeof(jb));
  jb.dtype = dtype;
  jb.src = (const uint8_t*)src;
  jb.n = n;
  jb.m0 = m0;
  jb.chunks = chunks;
  jb.S = S;
  jb.plan_lens = plan_lens;
  jb.n_groups = n_groups;
  jb.pack_lens = pack_lens;
  jb.pack_exps = pack_exps;
  jb.K = K;
  jb.entries = entries;
  int st = run_jobs(&jb, threads, compress_worker);
  if (st == ORC_OK) {
    uint8_t* o = (uint8_t*)out;
    uint64_t off_codes = table_end(dtype, chunks);
    uint64_t off_payload = off_codes + code_section_bytes(dtype, n_groups, K);
    memset(o, 0, off_payload);
    /* header */
    o[0] = 'Z';
    o[1] = 'N';
    o[2] = 'N';
    o[3] = '1';
    o[4] = 1;
    o[5] = 0;
    o[6] = (uint8_t)dtype;
    o[7] = (uint8_t)ns;
    put_u64(o + 8, n);
    put_u32(o + 16, chunk_bytes);
    put_u32(o + 20, S);
    put_u32(o + 24, (uint32_t)chunks);
    put_u32(o + 28, n_groups * (uint32_t)orc_n_entropy(dtype) + (K ? n_groups : 0));
    put_u64(o + 32, off_codes);
    put_u64(o + 40, off_payload);
    o[56] = LMAX;
    o[57] = (uint8_t)n_groups;
    o[58] = (uint8_t)K;
    /* shared code records */
    for (int e = 0; e < orc_n_entropy(dtype) && n_groups; e++) {
      int a = orc_alphabet(dtype, e);
      for (uint32_t g = 0; g < n_groups; g++) {
        const uint8_t* lg = plan_lens + ((uint64_t)e * n_groups + g) * 256;
        uint8_t* rp = o + off_codes + shared_record_pos(dtype, n_groups, (uint32_t)e * n_groups + g);
        for (int k = 0; k < a / 2; k++) rp[k] = (uint8_t)(lg[2 * k] | (lg[2 * k + 1] << 4));
      }
    }
    /* packed records and the list of packed exponents */
    if (K) {
      for (uint32_t g = 0; g < n_groups; g++) {
        const uint8_t* lp = pack_lens + (uint64_t)g * 256;
        uint8_t* rp = o + off_codes + packed_record_pos(dtype, n_groups, g);
        for (int k = 0; k < 128; k++) rp[k] = (uint8_t)(lp[2 * k] | (lp[2 * k + 1] << 4));
      }
      memcpy(o + off_codes + code_section_bytes(dtype, n_groups, K) - PACK_LIST_BYTES, pack_exps, K);
    }
    /* chunk table and payloads, in entry order: offsets are the running sum */
    uint64_t pos = off_payload;
    for (uint64_t k = 0; k < chunks * (uint64_t)ns; k++) {
      uint8_t* te = o + HEADER_BYTES + ENTRY_BYTES * k;
      te[0] = entries[k].mode;
      put_u32(te + 4, entries[k].code);
      put_u64(te + 8, pos);
      if (entries[k].size) memcpy(o + pos, entries[k].bytes, entries[k].size);
      pos += entries[k].size;
    }
    put_u64(o + 48, pos);
    *out_bytes = pos;
  }
  for (uint64_t k = 0; k < chunks * (uint64_t)ns; k++) free(entries[k].bytes);
  free(entries);
  return st;
}

/* ------------------------------------------------------------------ decompress */

typedef struct {
  int dtype;
  const uint8_t* in;
  uint64_t in_bytes, n, m0, chunks, total, off_codes;
  uint32_t S, n_groups, K;
  const uint8_t* pack_exps; /* the K listed exponents, in the container */
  uint8_t* out;
  int thread, threads;
  int status;
} djob_t;

/* Read the 4-bit lengths of a code record and check it: every length at most 12, at
 * least one symbol, and the Kraft sum of 2^-len at most 1. */
static int read_record(const uint8_t* rp, int a, uint8_t* len) {
  uint64_t kraft = 0;
  int present = 0;
  for (int k = 0; k < a / 2; k++) {
    len[2 * k] = rp[k] & 0xF;
    len[2 * k + 1] = rp[k] >> 4;
  }
  for (int k = 0; k < a; k++) {
    if (len[k] > LMAX) return ORC_ECORRUPT;
    if (len[k]) {
      present++;
      kraft += (uint64_t)1 << (LMAX - len[k]);
    }
  }
  if (!present || kraft > ((uint64_t)1 << LMAX)) return ORC_ECORRUPT;
  return ORC_OK;
}

/* Canonical decoding of one symbol, one bit at a time: at each length l the codes
 * of that length are the values [first, first + count[l]). */
static int decode_symbol(const uint8_t* bs, uint64_t cap_bits, uint64_t* t, const uint32_t* count,
                         const uint8_t* sorted) {
  int64_t code = 0, first = 0, index = 0;
  for (int l = 1; l <= LMAX; l++) {
    int b = get_bit(bs, cap_bits, t);
    if (b < 0) return -1;
    code |= b;
    if (code >= first && code - first < (int64_t)count[l]) return sorted[index + (code - first)];
    index += count[l];
    first = (first + (int64_t)count[l]) << 1;
    code <<= 1;
  }
  return -1;
}

static int decode_entry(const djob_t* jb, uint64_t c, int s, uint64_t m, uint8_t* sym) {
  int dt = jb->dtype, a = orc_alphabet(dt, s), w = raw_width(dt, s), ns = orc_n_streams(dt);
  uint64_t k = c * (uint64_t)ns + (uint64_t)s;
  const uint8_t* te = jb->in + HEADER_BYTES + ENTRY_BYTES * k;
  uint8_t mode = te[0];
  uint32_t code_ix = get_u32(te + 4);
  uint64_t off = get_u64(te + 8);
  uint64_t end = k + 1 < jb->chunks * (uint64_t)ns ? get_u64(te + ENTRY_BYTES + 8) : jb->total;
  if (te[1] || te[2] || te[3]) return ORC_ECORRUPT;
  if (off % 16 || end % 16 || off > end || end > jb->total) return ORC_ECORRUPT;
  if (mode == MODE_ZERO) {
    if (code_ix != NO_CODE) return ORC_ECORRUPT;
    memset(sym, 0, m);
    return ORC_OK;
  }
  if (mode == MODE_RAW) {
    if (code_ix != NO_CODE) return ORC_ECORRUPT;
    uint64_t cap_bits = (end - off) * 8, t = 0;
    if (cap_bits < m * (uint64_t)w) return ORC_ECORRUPT;
    for (uint64_t i = 0; i < m; i++) {
      uint32_t v = 0;
      for (int b = 0; b < w; b++) v = (v << 1) | (uint32_t)get_bit(jb->in + off, cap_bits, &t);
      sym[i] = (uint8_t)v;
    }
    return ORC_OK;
  }
  if (mode == MODE_ZRUN) {
    if (code_ix != NO_CODE || is_entropy(dt, s) || w != 8) return ORC_ECORRUPT;
    uint64_t blocks = ceil_div(m, ZRUN_BLOCK), map_bytes = round16(ceil_div(blocks, 8));
    if (end - off < map_bytes) return ORC_ECORRUPT;
    const uint8_t* map = jb->in + off;
    const uint8_t* data = map + map_bytes;
    uint64_t data_bits = (end - off - map_bytes) * 8, td = 0, tm = 0;
    for (uint64_t b = 0; b < blocks; b++) {
      uint64_t lo = b * ZRUN_BLOCK, hi = lo + ZRUN_BLOCK < m ? lo + ZRUN_BLOCK : m;
      int marked = get_bit(map, map_bytes * 8, &tm);
      for (uint64_t i = lo; i < hi; i++) {
        uint32_t v = 0;
        if (marked) {
          if (td + (uint64_t)w > data_bits) return ORC_ECORRUPT;
          for (int k = 0; k < w; k++) v = (v << 1) | (uint32_t)get_bit(data, data_bits, &td);
        }
        sym[i] = (uint8_t)v;
      }
    }
    return ORC_OK;
  }
  if (mode == MODE_PACK) {
    /* pairs of exponents as packed symbols, escaped exponents inline */
    uint8_t plen[256];
    if (dt != ORC_BF16 || s != 0 || !jb->K || m % 2 || jb->S % 2) return ORC_ECORRUPT;
    uint32_t NE = (uint32_t)orc_n_entropy(dt);
    if (code_ix < jb->n_groups * NE || code_ix >= jb->n_groups * NE + jb->n_groups) return ORC_ECORRUPT;
    uint32_t g = code_ix - jb->n_groups * NE;
    if (read_record(jb->in + jb->off_codes + packed_record_pos(dt, jb->n_groups, g), 256, plen) != ORC_OK)
      return ORC_ECORRUPT;
    uint64_t nsub = ceil_div(m, jb->S), avail = end - off;
    const uint8_t* p = jb->in + off;
    if (avail < round16(4 * nsub)) return ORC_ECORRUPT;
    const uint8_t* bs = p + round16(4 * nsub);
    uint64_t cap_bits = (avail - round16(4 * nsub)) * 8;
    uint32_t count[LMAX + 1] = {0};
    uint8_t sorted[256];
    int ns_sorted = 0;
    for (int l = 1; l <= LMAX; l++)
      for (int k2 = 0; k2 < 256; k2++)
        if (plen[k2] == l) {
          sorted[ns_sorted++] = (uint8_t)k2;
          count[l]++;
        }
    if (get_u32(p) != 0) return ORC_ECORRUPT;
    for (uint64_t j = 0; j < nsub; j++) {
      uint64_t t = get_u32(p + 4 * j);
      if (t > cap_bits) return ORC_ECORRUPT;
      uint64_t lo = j * jb->S, hi = lo + jb->S < m ? lo + jb->S : m;
      for (uint64_t i = lo; i < hi; i += 2) {
        int v = decode_symbol(bs, cap_bits, &t, count, sorted);
        if (v < 0) return ORC_ECORRUPT;
        uint32_t nib[2] = {(uint32_t)v >> 4, (uint32_t)v & 15u};
        for (int h = 0; h < 2; h++) {
          if (nib[h] == PACK_ESC) {
            uint32_t x = 0;
            for (int b = 0; b < 8; b++) {
              int bit = get_bit(bs, cap_bits, &t);
              if (bit < 0) return ORC_ECORRUPT;
              x = (x << 1) | (uint32_t)bit;
            }
            sym[i + h] = (uint8_t)x;
          } else if (nib[h] < jb->K) {
            sym[i + h] = jb->pack_exps[nib[h]];
          } else {
            return ORC_ECORRUPT;
          }
        }
      }
      if (j + 1 < nsub && t != get_u32(p + 4 * (j + 1))) return ORC_ECORRUPT;
    }
    return ORC_OK;
  }
  if (mode != MODE_HUFF || !is_entropy(dt, s)) return ORC_ECORRUPT;
  uint8_t len[256];
  const uint8_t* p = jb->in + off;
  uint64_t avail = end - off;
  if (code_ix == NO_CODE) {
    uint64_t rec = record_bytes(dt, s);
    if (avail < rec) return ORC_ECORRUPT;
    if (read_record(p, a, len) != ORC_OK) return ORC_ECORRUPT;
    p += rec;
    avail -= rec;
  } else {
    if (jb->n_groups == 0 || code_ix / jb->n_groups != (uint32_t)s) return ORC_ECORRUPT;
    if (read_record(jb->in + jb->off_codes + shared_record_pos(dt, jb->n_groups, code_ix), a, len) != ORC_OK)
      return ORC_ECORRUPT;
  }
  uint64_t nsub = ceil_div(m, jb->S);
  if (avail < round16(4 * nsub)) return ORC_ECORRUPT;
  const uint8_t* bs = p + round16(4 * nsub);
  uint64_t cap_bits = (avail - round16(4 * nsub)) * 8;
  /* canonical order: symbols sorted by (length, symbol) */
  uint32_t count[LMAX + 1] = {0};
  uint8_t sorted[256];
  int ns_sorted = 0;
  for (int l = 1; l <= LMAX; l++)
    for (int k2 = 0; k2 < a; k2++)
      if (len[k2] == l) {
        sorted[ns_sorted++] = (uint8_t)k2;
        count[l]++;
      }
  if (get_u32(p) != 0) return ORC_ECORRUPT;
  for (uint64_t j = 0; j < nsub; j++) {
    uint64_t t = get_u32(p + 4 * j);
    if (t > cap_bits) return ORC_ECORRUPT;
    uint64_t lo = j * jb->S, hi = lo + jb->S < m ? lo + jb->S : m;
    for (uint64_t i = lo; i < hi; i++) {
      int v = decode_symbol(bs, cap_bits, &t, count, sorted);
      if (v < 0) return ORC_ECORRUPT;
      sym[i] = (uint8_t)v;
    }
    if (j + 1 < nsub && t != get_u32(p + 4 * (j + 1))) return ORC_ECORRUPT;
  }
  return ORC_OK;
}

static void* decompress_worker(void* arg) {
  djob_t* jb = (djob_t*)arg;
  int ns = orc_n_streams(jb->dtype);
  uint8_t* sym[4] = {NULL, NULL, NULL, NULL};
  for (int s = 0; s < ns; s++) {
    sym[s] = (uint8_t*)malloc(jb->m0);
    if (!sym[s]) jb->status = ORC_EINVAL;
  }
  for (uint64_t c = (uint64_t)jb->thread; c < jb->chunks && jb->status == ORC_OK; c += (uint64_t)jb->threads) {
    uint64_t lo = c * jb->m0;
    uint64_t m = lo + jb->m0 <= jb->n ? jb->m0 : jb->n - lo;
    for (int s = 0; s < ns && jb->status == ORC_OK; s++) {
      int st = decode_entry(jb, c, s, m, sym[s]);
      if (st != ORC_OK) jb->status = st;
    }
    if (jb->status != ORC_OK) break;
    for (uint64_t i = 0; i < m; i++) {
      uint8_t f[4] = {0, 0, 0, 0};
      for (int s = 0; s < ns; s++) f[s] = sym[s][i];
      put_value(jb->dtype, jb->out, lo + i, f);
    }
  }
  for (int s = 0; s < ns; s++) free(sym[s]);
  return NULL;
}

int orc_decompress(int dtype, const void* in, uint64_t in_bytes, uint64_t n, uint32_t chunk_bytes,
                   void* out, int threads) {
  const uint8_t* h = (const uint8_t*)in;
  if (dtype < 0 || dtype > 3 || !in || !out || bad_count(dtype, n)) return ORC_EINVAL;
  if (chunk_bytes == 0 || chunk_bytes % (uint32_t)value_bytes(dtype) != 0) return ORC_EINVAL;
  if (in_bytes < HEADER_BYTES) return ORC_ECORRUPT;
  if (h[0] != 'Z' || h[1] != 'N' || h[2] != 'N' || h[3] != '1' || h[4] != 1 || h[5] != 0) return ORC_ECORRUPT;
  int ns = orc_n_streams(dtype);
  uint64_t m0 = chunk_values(dtype, chunk_bytes);
  uint64_t chunks = ceil_div(n, m0);
  if (h[6] != dtype || h[7] != ns || get_u64(h + 8) != n || get_u32(h + 16) != chunk_bytes) return ORC_ECORRUPT;
  uint32_t S = get_u32(h + 20), n_groups = h[57], K = h[58];
  if (S == 0 || get_u32(h + 24) != chunks || h[56] != LMAX || n_groups > MAX_GROUPS) return ORC_ECORRUPT;
  if (K > PACK_MAX || (K && (dtype != ORC_BF16 || n_groups == 0))) return ORC_ECORRUPT;
  if (get_u32(h + 28) != n_groups * (uint32_t)orc_n_entropy(dtype) + (K ? n_groups : 0)) return ORC_ECORRUPT;
  if (h[59] || get_u32(h + 60)) return ORC_ECORRUPT;
  uint64_t off_codes = get_u64(h + 32), off_payload = get_u64(h + 40), total = get_u64(h + 48);
  if (off_codes != table_end(dtype, chunks) || off_payload != off_codes + code_section_bytes(dtype, n_groups, K))
    return ORC_ECORRUPT;
  if (total > in_bytes || total < off_payload) return ORC_ECORRUPT;
  /* the list of packed exponents: K entries, then zeros */
  for (uint32_t i = K; K && i < PACK_LIST_BYTES; i++)
    if (h[off_payload - PACK_LIST_BYTES + i]) return ORC_ECORRUPT;
  if (total > in_bytes || total < off_payload) return ORC_ECORRUPT;
  if (get_u64(h + HEADER_BYTES + 8) != off_payload) return ORC_ECORRUPT;
  djob_t jb;
  memset(&jb, 0, sizeof(jb));
  jb.dtype = dtype;
  jb.in = h;
  jb.in_bytes = in_bytes;
  jb.n = n;
  jb.m0 = m0;
  jb.chunks = chunks;
  jb.total = total;
  jb.off_codes = off_codes;
  jb.S = S;
  jb.n_groups = n_groups;
  jb.K = K;
  jb.pack_exps = K ? h + off_payload - PACK_LIST_BYTES : NULL;
  jb.out = (uint8_t*)out;
  if (threads < 1) threads = 1;
  if (threads > 256) threads = 256;
  djob_t* jobs = (djob_t*)malloc(sizeof(djob_t) * (size_t)threads);
  pthread_t* th = (pthread_t*)malloc(sizeof(pthread_t) * (size_t)threads);
  if (!jobs || !th) {
    free(jobs);
    free(th);
    return ORC_EINVAL;
  }
  for (int t = 0; t < threads; t++) {
    jobs[t] = jb;
    jobs[t].thread = t;
    jobs[t].threads = threads;
    jobs[t].status = ORC_OK;
  }
  for (int t = 1; t < threads; t++) pthread_create(&th[t], NULL, decompress_worker, &jobs[t]);
  decompress_worker(&jobs[0]);
  for (int t = 1; t < threads; t++) pthread_join(th[t], NULL);
  int st = ORC_OK;
  for (int t = 0; t < threads; t++)
    if (jobs[t].status != ORC_OK) st = jobs[t].status;
  free(jobs);
  free(th);
  return st;
}

/* ------------------------------------------------------------------ plan (grouping) */

uint64_t orc_splitmix64(uint64_t* state) {
  uint64_t z = (*state += 0x9E3779B97F4A7C15ull);
  z = (z ^ (z >> 30)) * 0xBF58476D1CE4E5B9ull;
  z = (z ^ (z >> 27)) * 0x94D049BB133111EBull;
  return z ^ (z >> 31);
}

/* squared Euclidean distance, summed over i in ascending order */
static double sq_distance(const double* a, const double* b, int dims) {
  double s = 0.0;
  for (int i = 0; i < dims; i++) {
    double t = a[i] - b[i];
    s = s + t * t;
  }
  return s;
}

/* Grouping by exponent-distribution similarity:
 *  1. x_c[i] = h_c[i] / m_c for the exponent stream of every chunk c.
 *  2. If there are no more chunks than groups, chunk c is group c.
 *  3. Otherwise pick the starting centres with a partial Fisher-Yates shuffle driven
 *     by SplitMix64(seed): for j < G, r = j + next() mod (C - j), swap, centre j =
 *     x of the chunk now at position j.
 *  4. Lloyd passes (at most 100): assign every chunk to its nearest centre (ties to
 *     the smaller group); stop when no assignment changed; else set every non-empty
 *     group's centre to the mean of its members (summed in ascending chunk order).
 *  5. Each group's code for each entropy stream is the length-limited Huffman code of
 *     the summed histograms of its members (an empty group gets no code). */
int orc_plan_build(int dtype, const void* src, uint64_t n, uint32_t chunk_bytes, uint32_t n_groups,
                   uint64_t seed, uint8_t* lens_out, uint32_t* assign_out, int* iters_out,
                   double* inertia_out) {
  if (dtype < 0 || dtype > 3 || !src || bad_count(dtype, n) || n_groups == 0 || n_groups > MAX_GROUPS) return ORC_EINVAL;
  if (chunk_bytes == 0 || chunk_bytes % (uint32_t)value_bytes(dtype) != 0) return ORC_EINVAL;
  const uint8_t* in = (const uint8_t*)src;
  int E = orc_n_entropy(dtype), A = orc_alphabet(dtype, 0);
  uint64_t m0 = chunk_values(dtype, chunk_bytes), C = ceil_div(n, m0), G = n_groups;
  uint64_t* hist = (uint64_t*)calloc(C * (uint64_t)E * 256, sizeof(uint64_t));
  double* x = (double*)calloc(C * (uint64_t)A, sizeof(double));
  double* mu = (double*)calloc(G * (uint64_t)A, sizeof(double));
  uint32_t* assign = (uint32_t*)malloc(C * sizeof(uint32_t));
  uint64_t* perm = (uint64_t*)malloc(C * sizeof(uint64_t));
  if (!hist || !x || !mu || !assign || !perm) {
    free(hist);
    free(x);
    free(mu);
    free(assign);
    free(perm);
    return ORC_EINVAL;
  }
  for (uint64_t c = 0; c < C; c++) {
    uint64_t lo = c * m0, hi = lo + m0 <= n ? lo + m0 : n;
    for (int e = 0; e < E; e++) orc_histogram(dtype, in, lo, hi, e, hist + (c * (uint64_t)E + (uint64_t)e) * 256);
    for (int i = 0; i < A; i++) x[c * (uint64_t)A + (uint64_t)i] = (double)hist[c * (uint64_t)E * 256 + (uint64_t)i] / (double)(hi - lo);
  }
  int iters = 0;
  if (C <= G) {
    for (uint64_t c = 0; c < C; c++) assign[c] = (uint32_t)c;
  } else {
    uint64_t state = seed;
    for (uint64_t c = 0; c < C; c++) perm[c] = c;
    for (uint64_t j = 0; j < G; j++) {
      uint64_t r = j + orc_splitmix64(&state) % (C - j);
      uint64_t tmp = perm[j];
      perm[j] = perm[r];
      perm[r] = tmp;
      memcpy(mu + j * (uint64_t)A, x + perm[j] * (uint64_t)A, sizeof(double) * (size_t)A);
    }
    for (uint64_t c = 0; c < C; c++) assign[c] = 0xFFFFFFFFu;
    for (int it = 0; it < 100; it++) {
      int changed = 0;
      double inertia = 0.0;
      for (uint64_t c = 0; c < C; c++) {
        uint32_t best = 0;
        double bd = sq_distance(x + c * (uint64_t)A, mu, A);
        for (uint64_t j = 1; j < G; j++) {
          double d = sq_distance(x + c * (uint64_t)A, mu + j * (uint64_t)A, A);
          if (d < bd) {
            bd = d;
            best = (uint32_t)j;
          }
        }
        if (assign[c] != best) changed = 1;
        assign[c] = best;
        inertia = inertia + bd;
      }
      if (inertia_out) inertia_out[it] = inertia;
      iters = it + 1;
      if (!changed) break;
      for (uint64_t j = 0; j < G; j++) {
        uint64_t members = 0;
        for (uint64_t c = 0; c < C; c++)
          if (assign[c] == j) members++;
        if (!members) continue;
        for (int i = 0; i < A; i++) {
          double s = 0.0;
          for (uint64_t c = 0; c < C; c++)
            if (assign[c] == j) s = s + x[c * (uint64_t)A + (uint64_t)i];
          mu[j * (uint64_t)A + (uint64_t)i] = s / (double)members;
        }
      }
    }
  }
  for (int e = 0; e < E; e++) {
    int a = orc_alphabet(dtype, e);
    for (uint64_t g = 0; g < G; g++) {
      uint64_t sum[256];
      int any = 0;
      for (int k = 0; k < 256; k++) sum[k] = 0;
      for (uint64_t c = 0; c < C; c++)
        if (assign[c] == g)
          for (int k = 0; k < a; k++) sum[k] += hist[(c * (uint64_t)E + (uint64_t)e) * 256 + (uint64_t)k];
      uint8_t* lo = lens_out + ((uint64_t)e * G + g) * 256;
      memset(lo, 0, 256);
      for (int k = 0; k < a; k++)
        if (sum[k]) any = 1;
      if (any) orc_limited_lengths(sum, a, LMAX, lo);
    }
  }
  if (assign_out) memcpy(assign_out, assign, C * sizeof(uint32_t));
  if (iters_out) *iters_out = iters;
  free(hist);
  free(x);
  free(mu);
  free(assign);
  free(perm);
  return ORC_OK;
}

/* Packed exponents of a plan (BF16; reading stated at the top of this file):
 *  1. count every exponent of the setup tensor;
 *  2. list the K = min(max_pack, exponents present) most frequent ones, a larger count
 *     first, equal counts by the smaller exponent;
 *  3. for each group, the length-limited Huffman code of the summed pair-symbol
 *     histograms of its member chunks that hold an even number of values (a group
 *     without such pairs gets no packed code).
 * exps_out: 16 bytes (the list, then zeros); lens_out: n_groups x 256; *K_out. */
int orc_plan_pack(const void* src, uint64_t n, uint32_t chunk_bytes, uint32_t n_groups, const uint32_t* assign,
                  uint32_t max_pack, uint8_t* exps_out, uint8_t* lens_out, uint32_t* K_out) {
  if (!src || n == 0 || !assign || n_groups == 0 || n_groups > MAX_GROUPS || max_pack > PACK_MAX) return ORC_EINVAL;
  if (chunk_bytes == 0 || chunk_bytes % 2 != 0) return ORC_EINVAL;
  const uint8_t* in = (const uint8_t*)src;
  uint64_t total[256];
  for (int k = 0; k < 256; k++) total[k] = 0;
  for (uint64_t i = 0; i < n; i++) total[orc_field(ORC_BF16, in, i, 0)]++;
  uint8_t taken[256];
  memset(taken, 0, sizeof(taken));
  memset(exps_out, 0, PACK_LIST_BYTES);
  uint32_t K = 0;
  while (K < max_pack) {
    int best = -1;
    for (int k = 0; k < 256; k++)
      if (!taken[k] && total[k] > 0 && (best < 0 || total[k] > total[best])) best = k;
    if (best < 0) break;
    taken[best] = 1;
    exps_out[K++] = (uint8_t)best;
  }
  *K_out = K;
  memset(lens_out, 0, (size_t)n_groups * 256);
  if (!K) return ORC_OK;
  uint64_t m0 = chunk_bytes / 2, C = ceil_div(n, m0);
  for (uint32_t g = 0; g < n_groups; g++) {
    uint64_t sum[256], hp[256], esc;
    int any = 0;
    for (int k = 0; k < 256; k++) sum[k] = 0;
    for (uint64_t c = 0; c < C; c++) {
      uint64_t lo = c * m0, m = lo + m0 <= n ? m0 : n - lo;
      if (assign[c] != g || m % 2) continue;
      orc_pack_histogram(in, lo, m, exps_out, K, hp, &esc);
      for (int k = 0; k < 256; k++) sum[k] += hp[k];
    }
    for (int k = 0; k < 256; k++)
      if (sum[k]) any = 1;
    if (any) orc_limited_lengths(sum, 256, LMAX, lens_out + (uint64_t)g * 256);
  }
  return ORC_OK;
}

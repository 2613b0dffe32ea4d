/*
 * zipnn_oracle.h -- plain CPU oracle for the ZipNN-style float-tensor codec.
 *
 * TEST INFRASTRUCTURE. Only tests, the smoke check and the benchmark's CPU
 * baseline call this code. The product library never links, loads or calls it,
 * and it shares no header, helper or table with the CUDA path.
 *
 * What it computes (sources by page title and section):
 *  - "ZipNN: Lossless Compression for AI Models" (abstract) and the THEORY-599
 *    note on it, "Per-field compressibility (Table II)": split each float into its
 *    exponent field and its sign/fraction bytes; only the exponent compresses.
 *  - THEORY-599, "Order-0 only (section III-A b)": one order-0 model (a symbol
 *    histogram) per chunk, Huffman-coded after the exponent is extracted.
 *  - "Lossless Compression of Neural Network Components ... in Low-Precision
 *    Formats" (abstract): FP8 and FP4 exponent and mantissa entropy-coded
 *    independently.
 *  - "NeuralZip: Reusable Setup for Fast Lossless Compression" (abstract): chunks
 *    grouped by exponent-distribution similarity share one Huffman code, chosen
 *    once by a reusable setup (the plan).
 * The byte layout of the container, the length limit and the grouping procedure
 * are not given by the pages; the readings this oracle implements are stated in
 * zipnn_oracle.c (the container layout under "layout rules").
 */
#ifndef ZIPNN_ORACLE_H
#define ZIPNN_ORACLE_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

/* dtypes */
#define ORC_BF16 0
#define ORC_FP32 1
#define ORC_FP8 2
#define ORC_FP4 3

/* return codes */
#define ORC_OK 0
#define ORC_EINVAL 1
#define ORC_ESMALL 2
#define ORC_ECORRUPT 3
#define ORC_EPLAN 4

/* Huffman lengths without a limit, deterministic ties (weight, then order;
 * leaves have order = symbol, the i-th merged node has order 256 + i). */
int orc_huffman_lengths(const uint64_t* freq, int alphabet, uint8_t* len);
/* Lengths limited to lmax by halving the frequencies until the code fits. */
int orc_limited_lengths(const uint64_t* freq, int alphabet, int lmax, uint8_t* len);
/* Canonical code values (deflate rule) for a length vector; code[s] = 0 if len 0. */
void orc_canonical_codes(const uint8_t* len, int alphabet, uint32_t* code);

/* Fields of value i of stream s (the split). */
uint8_t orc_field(int dtype, const uint8_t* src, uint64_t i, int s);
int orc_n_streams(int dtype);
int orc_n_entropy(int dtype);
int orc_alphabet(int dtype, int s);

/* Per-chunk order-0 histogram of stream s over values [lo, hi). */
void orc_histogram(int dtype, const uint8_t* src, uint64_t lo, uint64_t hi, int s, uint64_t* hist);

/* Upper bound on the container size. */
uint64_t orc_max_compressed_bytes(int dtype, uint64_t n, uint32_t chunk_bytes, uint32_t n_groups);

/* Compress n values at src into out (cap bytes). plan_lens (n_entropy x n_groups x 256
 * length bytes) may be NULL. threads >= 1 splits the chunk loop; output is independent
 * of the thread count. */
int orc_compress(int dtype, const void* src, uint64_t n, uint32_t chunk_bytes, uint32_t S,
                 const uint8_t* plan_lens, uint32_t n_groups, void* out, uint64_t cap,
                 uint64_t* out_bytes, int threads);

/* As orc_compress, with a plan's packed exponents (BF16): pack_lens (n_groups x 256
 * packed-code lengths) and pack_exps (K listed exponents); K = 0 is orc_compress. */
int orc_compress_packed(int dtype, const void* src, uint64_t n, uint32_t chunk_bytes, uint32_t S,
                        const uint8_t* plan_lens, uint32_t n_groups, const uint8_t* pack_lens,
                        const uint8_t* pack_exps, uint32_t K, void* out, uint64_t cap, uint64_t* out_bytes,
                        int threads);
uint64_t orc_max_compressed_bytes_packed(int dtype, uint64_t n, uint32_t chunk_bytes, uint32_t n_groups, uint32_t K);

/* Pair-symbol histogram of the BF16 values [lo, lo + m) (m even) for K listed exponents,
 * and the number of escaped exponents. */
void orc_pack_histogram(const void* src, uint64_t lo, uint64_t m, const uint8_t* exps, uint32_t K, uint64_t* hist,
                        uint64_t* escapes);

/* Packed exponents of a plan (BF16): the list (16 bytes) and each group's packed code
 * from the chunks' assignment. */
int orc_plan_pack(const void* src, uint64_t n, uint32_t chunk_bytes, uint32_t n_groups, const uint32_t* assign,
                  uint32_t max_pack, uint8_t* exps_out, uint8_t* lens_out, uint32_t* K_out);

/* Decompress a container into n values. */
int orc_decompress(int dtype, const void* in, uint64_t in_bytes, uint64_t n, uint32_t chunk_bytes,
                   void* out, int threads);

/* Plan: k-means over normalised exponent histograms, then one limited Huffman code per
 * (entropy stream, group) from the group's summed histogram.
 * lens_out: n_entropy x n_groups x 256 bytes; assign_out: n_chunks entries (may be NULL);
 * iters_out: number of assignment passes; inertia_out: per-pass total squared distance
 * (up to 100 doubles, may be NULL). */
int orc_plan_build(int dtype, const void* src, uint64_t n, uint32_t chunk_bytes, uint32_t n_groups,
                   uint64_t seed, uint8_t* lens_out, uint32_t* assign_out, int* iters_out,
                   double* inertia_out);

/* SplitMix64 step (Steele, Lea and Flood, 2014); exposed for tests. */
uint64_t orc_splitmix64(uint64_t* state);

#ifdef __cplusplus
}
#endif
#endif

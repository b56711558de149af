/*
 * zfref.h -- CPU oracle for the ZipFloat comparison codec (BF16).
 *
 * TEST INFRASTRUCTURE ONLY, like ehref.h: loaded by the tests, the smoke check
 * and the benchmark's CPU-baseline leg; the product library shares no source
 * with it.
 *
 * Source: "ZipFloat: An Ultra-fast and Lossless Floating-Point Compressor for
 * LLM Inference Systems", §3.1 (blocks of N_e values coded independently),
 * §3.2 (the dominant exponent range [MD - 6, MD - 6 + 8) and the remap of
 * Eq. 4: new = old - l_b) and §3.3 (a 3-bit dense array stored as bit planes,
 * a sparse array of 16-bit <11-bit index, 5-bit value> records for the
 * elements whose remapped exponent has a non-zero high part, raw
 * sign/mantissa bytes).
 *
 * Format fixed here (readings of the page, one per point):
 *   - block = 2048 consecutive values (the page's N_e = 2048); B = ceil(n/2048);
 *     the last block may be short;
 *   - MD = the most frequent exponent field of the block, ties to the smaller
 *     field; l_b = (MD - 6) mod 256; r = (e - l_b) mod 256 (8-bit arithmetic);
 *   - dense[b][p][w] (u32, p = 0..2, w = 0..63): bit i = bit p of r of element
 *     32w + i of block b (0 past the block's end);
 *   - for every element with r >= 8, in element order, the record
 *     (i << 5) | (r >> 3), i = index in the block (0..2047);
 *   - meta[b] = l_b | (records of block b) << 8;
 *   - sparse_off[b] = index of block b's first record: blocks in order here
 *     (the GPU reserves each block's range with an atomic, so only the
 *     per-block record lists are unique);
 *   - sign_mant[i] = (s << 7) | m7 (as in the Huffman format).
 * Functions return EHREF_OK or a negative EHREF_E* code.
 */
#ifndef ZFREF_H
#define ZFREF_H

#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

#define ZFREF_BLOCK 2048

uint64_t zfref_blocks(uint64_t n);

/* The block's dominant exponent MD (most frequent field, ties to the smaller)
 * and l_b = (MD - 6) mod 256. */
int zfref_block_base(const uint16_t *in, uint32_t count, uint32_t *md, uint32_t *lb);

/* Compresses n BF16 bit patterns.  sparse has room for sparse_cap records;
 * *n_records receives their total. */
int zfref_compress(const uint16_t *in, uint64_t n, uint8_t *sign_mant, uint32_t *meta,
                   uint32_t *dense, uint32_t *sparse_off, uint16_t *sparse,
                   uint64_t sparse_cap, uint64_t *n_records);

/* Inverse; n_records bounds every block's record range. */
int zfref_decompress(uint64_t n, const uint8_t *sign_mant, const uint32_t *meta,
                     const uint32_t *dense, const uint32_t *sparse_off,
                     const uint16_t *sparse, uint64_t n_records, uint16_t *out);

#ifdef __cplusplus
}
#endif
#endif

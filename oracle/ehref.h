/*
 * ehref.h -- CPU oracle for the split-exponent Huffman codec.
 *
 * TEST INFRASTRUCTURE ONLY.  This library is the plain, slow, single-threaded
 * statement of what the codec computes.  Only the test suite, the smoke check
 * and the CPU-baseline leg of the benchmark may load it.  The product library
 * (libexphuff) shares no source with it and never calls it.
 *
 * Sources the steps follow (page title, then section):
 *  - "70% Size, 100% Accuracy: Lossless LLM Compression for Efficient GPU
 *    Inference via Dynamic-Length Float" (DFloat11 news article), section
 *    "方法介绍": the exponent is Huffman-coded from the histogram of all
 *    exponents, the codes are bit-packed tightly into EncodedExponent, and the
 *    raw sign and mantissa go to a separate byte array PackedSignMantissa.
 *  - "Lossless Compression of Neural Network Components ... Low-Precision
 *    Formats" (paper summary), sections "方法详解" and "实验设计": exponent and
 *    mantissa are separated; each tensor is coded in fixed-size chunks.
 *  - "ZipFloat: An Ultra-fast and Lossless Floating-Point Compressor for LLM
 *    Inference Systems", section 2.1 (Table 2): the BF16 exponent field is the
 *    exponent plus 127.
 * Where the pages are silent (tie-breaks, bit order, chunk size, length limit)
 * the format below fixes one reading; each is listed in the header of
 * ehref.cpp.
 *
 * All pointers are HOST pointers.  Functions return EHREF_OK (0) or a
 * negative EHREF_E* code.
 */
#ifndef EHREF_H
#define EHREF_H

#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

/* EHREF_BYTES: every byte is its own symbol and there is no sign/mantissa
 * part -- the codec applied to FP4 block scale factors (E4M3 or E8M0 bytes),
 * which the paper summary ("结果分析") and the edgentiq blog ("Insights into
 * FP4 Compression") report compressible with Huffman coding. */
enum { EHREF_BF16 = 0, EHREF_FP8_E4M3 = 1, EHREF_BYTES = 2 };

enum {
  EHREF_OK = 0,
  EHREF_EINVAL = -1,      /* bad argument                                   */
  EHREF_EINFEASIBLE = -2, /* more distinct symbols than 2^max_code_len      */
  EHREF_ECAPACITY = -3,   /* output stream buffer too small                 */
  EHREF_ECORRUPT = -4     /* compressed data inconsistent                   */
};

/* 256 for BF16 (8-bit exponent field) and BYTES, 16 for FP8 E4M3 (4-bit
 * field). */
int ehref_alphabet(int dtype);

/* Step S1.  Per element: exponent field e[i] and the raw sign+mantissa
 * value sm[i] (BF16: (s<<7)|m7, FP8: (s<<3)|m3), one byte each. */
int ehref_split(int dtype, const void *in, uint64_t n, uint8_t *e, uint8_t *sm);

/* Inverse of ehref_split for one element stream. */
int ehref_merge(int dtype, const uint8_t *e, const uint8_t *sm, uint64_t n,
                void *out);

/* Histogram of exponent fields, cnt[A]. */
int ehref_histogram(int dtype, const void *in, uint64_t n, uint64_t *cnt);

/* Min-variance Huffman leaf depths (0 for absent symbols), before any length
 * limit or rank assignment.  Returns the maximum depth (>= 0). */
int ehref_huffman_depths(const uint64_t *cnt, int A, uint8_t *depth);

/* Package-merge lengths limited to Lmax (0 for absent symbols), before rank
 * assignment.  Needs at least 2 present symbols and at most 2^Lmax. */
int ehref_package_merge(const uint64_t *cnt, int A, int Lmax, uint8_t *len);

/* The full length rule of the format: Huffman, package-merge when the Huffman
 * depth exceeds Lmax, then rank assignment. */
int ehref_code_lengths(const uint64_t *cnt, int A, int Lmax, uint8_t *len);

/* Canonical codes from lengths (0-length symbols get code 0). */
int ehref_canonical_codes(const uint8_t *len, int A, uint32_t *code);

/* Sign/mantissa array in its stored layout: BF16 one byte per element; FP8
 * one nibble per element, element 2i in the low nibble of byte i; BYTES none. */
uint64_t ehref_sm_bytes(int dtype, uint64_t n);
int ehref_pack_sm(int dtype, const void *in, uint64_t n, uint8_t *sm_packed);

/* Encode the exponent stream with a given code: off[C+1] bit offsets, stream
 * bytes (zero-filled first, MSB-first bit order), total bits. */
uint64_t ehref_num_chunks(uint64_t n, uint32_t chunk);
int ehref_encode(int dtype, const void *in, uint64_t n, uint32_t chunk,
                 const uint8_t *len, const uint32_t *code, uint64_t *off,
                 uint8_t *stream, uint64_t stream_cap, uint64_t *total_bits);

/* Steps S1-S5 in order. */
int ehref_compress(int dtype, const void *in, uint64_t n, uint32_t chunk,
                   int Lmax, uint8_t *len, uint32_t *code, uint64_t *off,
                   uint8_t *stream, uint64_t stream_cap, uint8_t *sm_packed,
                   uint64_t *total_bits);

/* Step S6 for chunks [first, first+count): writes elements
 * [first*chunk, min(n, (first+count)*chunk)) to out (indexed from element
 * first*chunk, i.e. out points at the first decoded element). */
int ehref_decompress_chunks(int dtype, uint64_t n, uint32_t chunk,
                            const uint8_t *len, const uint32_t *code,
                            const uint64_t *off, const uint8_t *stream,
                            uint64_t stream_bytes, const uint8_t *sm_packed,
                            uint32_t first, uint32_t count, void *out);

/* Step S6 over all chunks. */
int ehref_decompress(int dtype, uint64_t n, uint32_t chunk, const uint8_t *len,
                     const uint32_t *code, const uint64_t *off,
                     const uint8_t *stream, uint64_t stream_bytes,
                     const uint8_t *sm_packed, void *out);

/* Optional value index (an auxiliary position array in the spirit of the
 * DFloat11 article's per-thread position variables, "方法介绍", kept outside
 * the stream): for chunk c and k = 0 .. chunk/EHREF_INDEX_STRIDE - 1, entry
 * index[c * (chunk / EHREF_INDEX_STRIDE) + k] is the bit offset, from the
 * chunk's first bit, of the code of value k * EHREF_INDEX_STRIDE of the
 * chunk; entries past the chunk's last value hold the chunk's total bits.
 * With it a decoder can start every run of EHREF_INDEX_STRIDE values at a
 * known bit without first finding code boundaries. */
#define EHREF_INDEX_STRIDE 128
int ehref_value_index(int dtype, const void *in, uint64_t n, uint32_t chunk,
                      const uint8_t *len, uint32_t *index);

/* Fixed-slot page store (online K/V cache compression).  A page of n values
 * (one chunk; 64 tokens x 8 heads x 128 dims = 65,536 for Llama-3.1-8B K/V) is
 * coded with a FROZEN codebook (len/code from earlier data) into a slot of
 * slot_bytes bytes: the codes MSB-first from bit 0 of the slot, the rest of
 * the slot zero.  The page is stored raw instead -- *raw = 1, slot untouched,
 * exponent fields copied to raw_exps (one byte each) -- when one of its
 * exponents has no code or when ceil(bits/8) + 16 > slot_bytes (the decoder
 * reads up to 16 bytes past the last code).  sm_packed receives the page's
 * sign/mantissa array in every case.  Sources: ZipFloat §3.3 and §4.2 (new KV
 * entries are compressed into preallocated slots and decompressed on reuse);
 * the paper summary "局限性" and "开放问题" (real-time K/V compression). */
int ehref_page_encode(int dtype, const void *in, uint64_t n, const uint8_t *len,
                      const uint32_t *code, uint8_t *slot, uint64_t slot_bytes,
                      uint8_t *sm_packed, uint8_t *raw_exps, uint64_t *bits,
                      int *raw);

/* Inverse: rebuilds the page's n values from its slot (or raw exponents). */
int ehref_page_decode(int dtype, uint64_t n, const uint8_t *len,
                      const uint32_t *code, const uint8_t *slot,
                      uint64_t slot_bytes, uint64_t bits, int raw,
                      const uint8_t *raw_exps, const uint8_t *sm_packed,
                      void *out);

/* Stored form of one compressed tensor (a format of this library; the pages
 * only say that weights are compressed offline and decompressed on the GPU:
 * the DFloat11 article, "方法介绍", and ZipFloat §4.2).  Little-endian:
 *   "EXHF", u16 version 1, u8 dtype, u8 lmax, u32 chunk, u32 flags (bit 0:
 *   value index present), u64 n, u64 number of chunks C, u64 code bits;
 *   six section entries {u64 offset, u64 length, u32 crc32, u32 0} for
 *   lengths (A bytes), codes (A u32), chunk bit offsets (C+1 u64), stream
 *   (ceil(bits/8) bytes), sign/mantissa bytes, value index (C*chunk/128 u32
 *   or length 0); the crc32 of the preceding 184 bytes and a zero u32;
 *   then the sections in that order from byte 192, each starting at a
 *   multiple of 16, zeros between them and after the last up to a multiple
 *   of 16.
 * crc32 is the IEEE 802.3 / zlib CRC (reflected polynomial 0xEDB88320,
 * initial and final XOR 0xFFFFFFFF).  index may be NULL.  Writes the
 * container to out (out_cap bytes) and its size to *size; with out == NULL
 * only the size is returned. */
int ehref_container_write(int dtype, uint64_t n, uint32_t chunk, int lmax,
                          const uint8_t *len, const uint32_t *code,
                          const uint64_t *chunk_bit_off, const uint8_t *stream,
                          uint64_t bits, const uint8_t *sm_packed,
                          const uint32_t *index, uint8_t *out, uint64_t out_cap,
                          uint64_t *size);

/* The crc32 of the container format, for tests. */
uint32_t ehref_crc32(const uint8_t *data, uint64_t len);

#ifdef __cplusplus
}
#endif
#endif

/*
 * exphuff.h -- libexphuff: lossless split-exponent Huffman codec for BF16 and
 * FP8 E4M3 tensors on NVIDIA B200 (sm_100a).
 *
 * What the codec computes (page title, then section):
 *  - "70% Size, 100% Accuracy: Lossless LLM Compression for Efficient GPU
 *    Inference via Dynamic-Length Float" (DFloat11 article), section
 *    "方法介绍": a Huffman code is built from the distribution of exponent
 *    values; the exponent codes are tightly bit-packed into a byte array
 *    (EncodedExponent) and the sign and mantissa bits are kept raw in a
 *    separate byte array (PackedSignMantissa).  Decompression rebuilds the
 *    exact original values on the GPU.
 *  - "Lossless Compression of Neural Network Components: Weights,
 *    Checkpoints, and K/V Caches in Low-Precision Formats" (paper summary),
 *    sections "方法详解" and "实验设计": exponent and mantissa are split, the
 *    exponent is Huffman-coded, FP8 is covered, and every tensor is coded in
 *    fixed-size chunks.
 *  - "ZipFloat: An Ultra-fast and Lossless Floating-Point Compressor for LLM
 *    Inference Systems", section 2.1: the BF16 exponent field is the exponent
 *    plus 127.
 *
 * Format (one compressed tensor of n elements, chunk size K, C = ceil(n/K)):
 *  - exponent field e: BF16 bits 14..7 (x>>7 & 0xFF, alphabet 256); FP8 E4M3
 *    bits 6..3 (x>>3 & 0xF, alphabet 16);
 *  - code_len[A]: Huffman code lengths, 0 for absent symbols, at most
 *    max_code_len (<= 32).  Minimum-variance Huffman; package-merge when the
 *    Huffman depth exceeds the limit; lengths dealt in ascending order to the
 *    symbols sorted by (count descending, symbol ascending).  A tensor with one
 *    distinct exponent gets length 1 (code "0");
 *  - code[A]: canonical codes in (length, symbol) order (RFC 1951 §3.2.2);
 *  - exp_stream: the codes of all elements in element order, MSB-first (bit
 *    p is bit 7-(p&7) of byte p>>3), chunks back to back with no padding, the
 *    last byte zero-padded; ceil(exp_stream_bits/8) meaningful bytes;
 *  - chunk_bit_off[C+1]: bit offset of each chunk's first code;
 *    chunk_bit_off[C] = exp_stream_bits;
 *  - sign_mant: BF16 one byte (s<<7)|m7 per element; FP8 one nibble
 *    (s<<3)|m3 per element, element 2i in the low nibble of byte i, the unused
 *    high nibble of an odd-length tensor zero; EH_BYTES none (the symbol is
 *    the whole byte; sign_mant may be NULL).
 *
 * Memory: every pointer passed to a compress/decompress call is a DEVICE
 * pointer on the current CUDA device, allocated and owned by the CALLER.  The
 * library allocates nothing on these paths; it needs a caller-provided
 * workspace whose size the *_workspace / *_bound queries return.  Device
 * pointers must be 16-byte aligned.  Streams are passed as `void *` holding a
 * cudaStream_t (NULL = legacy default stream).
 *
 * Errors: argument errors are returned immediately (nothing is launched).
 * Data errors found on the GPU (a corrupt stream, an invalid codebook) are
 * recorded in a status word inside the workspace; eh_get_status() waits for
 * the stream and returns it.  Kernels never trap and every wait in them is
 * bounded.  Functions are thread-safe as long as concurrent calls use
 * distinct workspaces.
 */
#ifndef EXPHUFF_H
#define EXPHUFF_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

#if defined(__GNUC__)
#define EH_API __attribute__((visibility("default")))
#else
#define EH_API
#endif

#define EH_DEFAULT_CHUNK_ELEMS 65536u /* elements per chunk (one K/V page)   */
#define EH_MAX_CODE_LEN 32u           /* longest code the format allows     */
#define EH_MAX_BATCH 16               /* tensors per batched launch         */
#define EH_NOALLOC_MAX_BATCH 8        /* tensors per eh_decompress_batch_noalloc */

/* EH_BYTES: every byte is its own symbol (alphabet 256) and there is no
 * sign/mantissa array -- for FP4 block scale factors (E4M3 or E8M0 bytes),
 * which the paper summary ("结果分析") and the edgentiq blog ("Insights into
 * FP4 Compression") report compressible with Huffman coding. */
typedef enum { EH_BF16 = 0, EH_FP8_E4M3 = 1, EH_BYTES = 2 } eh_dtype;

typedef enum {
  EH_OK = 0,
  EH_ERR_INVALID_ARG = 1, /* bad pointer, size, alignment or capacity      */
  EH_ERR_UNSUPPORTED = 2, /* dtype / chunk size / limit not supported      */
  EH_ERR_INFEASIBLE = 3,  /* more distinct exponents than 2^max_code_len   */
  EH_ERR_CUDA = 4,        /* a CUDA runtime call failed                    */
  EH_ERR_CORRUPT = 5,     /* compressed data or codebook inconsistent      */
  EH_ERR_TIMEOUT = 6,     /* a bounded wait inside a kernel gave up        */
  EH_ERR_NOMEM = 7        /* workspace smaller than required               */
} eh_status;

/* Fixes the format: dtype, chunk size, length limit. */
typedef struct {
  int32_t dtype;         /* eh_dtype                                        */
  uint32_t chunk_elems;  /* multiple of 1024 in [1024, 65536]               */
  uint32_t max_code_len; /* 1..32                                           */
  uint32_t reserved;     /* 0                                               */
} eh_plan_t;

/* One compressed tensor.  The caller allocates the device arrays (sizes from
 * eh_compress_bound); eh_compress fills them, n_chunks and exp_stream_bits. */
typedef struct {
  int32_t dtype;            /* eh_dtype, must match the plan                 */
  uint32_t n_chunks;        /* ceil(n / chunk_elems)                         */
  uint64_t n;               /* element count                                 */
  uint8_t *code_len;        /* device, [A] (A = 256 BF16, 16 FP8)            */
  uint32_t *code;           /* device, [A]                                   */
  uint64_t *chunk_bit_off;  /* device, [n_chunks + 1]                        */
  uint8_t *exp_stream;      /* device, exp_stream_cap bytes                  */
  uint64_t exp_stream_cap;  /* bytes; >= eh_compress_bound's stream_cap      */
  uint8_t *sign_mant;       /* device, n (BF16), ceil(n/2) (FP8), 0 (BYTES)  */
  uint64_t exp_stream_bits; /* total code bits (host copy)                   */
  uint32_t *value_index;    /* device, optional (NULL: none); see below      */
} eh_compressed_t;

/* Optional value index, outside the stream: entry c * (chunk_elems /
 * EH_INDEX_STRIDE) + k is the bit offset, from chunk c's first bit, of the
 * code of value k * EH_INDEX_STRIDE of the chunk; entries past a short last
 * chunk's end hold that chunk's bit count.  n_chunks * chunk_elems /
 * EH_INDEX_STRIDE u32 entries (4 bytes per 128 values, +1.6 % on BF16).
 * eh_compress fills it when value_index is non-NULL; eh_decompress then
 * starts every run of EH_INDEX_STRIDE values at its recorded bit instead of
 * finding code boundaries first (the DFloat11 article's per-thread position
 * variables, "方法介绍", kept beside the format rather than in it).  An index
 * that does not match the stream is reported as EH_ERR_CORRUPT. */
#define EH_INDEX_STRIDE 128

/* Fills *plan.  chunk_elems = 0 selects 65536; max_code_len = 0 selects 32.
 * Returns EH_ERR_UNSUPPORTED for other chunk sizes or limits. */
EH_API eh_status eh_plan(eh_plan_t *plan, int32_t dtype, uint32_t chunk_elems,
                  uint32_t max_code_len);

/* Sizes for compressing one tensor of n elements: stream_cap = bytes for
 * exp_stream (worst case n*max_code_len bits, rounded up to 16 bytes, plus
 * 16 bytes that the decoder may read past the last code), sm_bytes = bytes
 * for sign_mant, workspace_bytes = device workspace for eh_compress.
 * Any output pointer may be NULL. */
EH_API eh_status eh_compress_bound(const eh_plan_t *plan, uint64_t n,
                            uint64_t *stream_cap, uint64_t *sm_bytes,
                            uint64_t *workspace_bytes);

/* Workspace for eh_compress_batch over k tensors of ns[i] elements. */
EH_API eh_status eh_compress_batch_workspace(const eh_plan_t *plan, int k,
                                      const uint64_t *ns,
                                      uint64_t *workspace_bytes);

/* Compresses one tensor (steps: split + histogram, codebook, chunk offsets,
 * encode + sign/mantissa pack).  `in` holds n raw BF16 (uint16) or FP8
 * (uint8) values.  `out` is a host struct whose dtype, n and device pointers
 * the caller has set; the call writes the device arrays, out->n_chunks and
 * out->exp_stream_bits.  Waits for `stream` once, to return the bit count. */
EH_API eh_status eh_compress(const eh_plan_t *plan, const void *in, uint64_t n,
                      eh_compressed_t *out, void *workspace,
                      uint64_t workspace_bytes, void *stream);

/* Compresses k <= EH_MAX_BATCH tensors with one launch per step, one
 * codebook per tensor.  ins[i] has outs[i].n elements.  If bits_dev is NULL
 * the call waits for the stream and fills outs[i].exp_stream_bits; otherwise
 * it writes the k bit counts to the device array bits_dev[k] and returns
 * without waiting (outs[i].exp_stream_bits is then left untouched). */
EH_API eh_status eh_compress_batch(const eh_plan_t *plan, int k,
                            const void *const *ins, eh_compressed_t *outs,
                            uint64_t *bits_dev, void *workspace,
                            uint64_t workspace_bytes, void *stream);

/* Compression of one tensor split across GPUs, each rank holding a shard of
 * whole chunks (the codebook is built from the histogram of the whole tensor, as in
 * the DFloat11 article, "方法介绍").
 * Step 1, on every rank: eh_compress_shard_begin histograms the local shard
 * into counts (device, u64[A], overwritten) and writes its packed
 * sign/mantissa.  Between the steps the caller sums counts over the ranks
 * (one all-reduce of A u64 values).  Step 2: eh_compress_shard_finish builds
 * the codebook from the summed counts (every rank gets the same one), the
 * shard's chunk offsets (starting at bit 0 of the shard) and its stream.  The
 * global offset of a shard is the sum of the bit counts of the ranks before
 * it (one all-gather).  `out`, `workspace` (eh_compress_bound for the shard's
 * n) and `in` must be the same for both steps.  bits_dev as in
 * eh_compress_batch.  Decompression of a shard needs no communication. */
EH_API eh_status eh_compress_shard_begin(const eh_plan_t *plan, const void *in,
                                         eh_compressed_t *out, uint64_t *counts,
                                         void *workspace, uint64_t workspace_bytes,
                                         void *stream);
EH_API eh_status eh_compress_shard_finish(const eh_plan_t *plan, const void *in,
                                          eh_compressed_t *out,
                                          const uint64_t *counts, uint64_t *bits_dev,
                                          void *workspace, uint64_t workspace_bytes,
                                          void *stream);

/* Workspace for decompressing up to k tensors in one call. */
EH_API eh_status eh_decompress_workspace(const eh_plan_t *plan, int k,
                                  uint64_t *workspace_bytes);

/* Rebuilds the n original values into out (device, n*elem_size bytes).
 * Fully stream-ordered, no host wait; data errors go to the status word. */
EH_API eh_status eh_decompress(const eh_plan_t *plan, const eh_compressed_t *c,
                        void *out, void *workspace, uint64_t workspace_bytes,
                        void *stream);

/* Block-at-a-time decompression (the DFloat11 article, "方法介绍" and
 * "消融研究": a whole transformer block is decompressed in one go): k <=
 * EH_MAX_BATCH tensors, one launch over all of their chunks. */
EH_API eh_status eh_decompress_batch(const eh_plan_t *plan, int k,
                              const eh_compressed_t *cs, void *const *outs,
                              void *workspace, uint64_t workspace_bytes,
                              void *stream);

/* Decompresses chunks [first, first+count) of one tensor (e.g. K/V pages of
 * 64 tokens x 8 heads x 128 dims = 65,536 values).  out receives elements
 * [first*K, min(n, (first+count)*K)). */
EH_API eh_status eh_decompress_chunks(const eh_plan_t *plan, const eh_compressed_t *c,
                               uint32_t first, uint32_t count, void *out,
                               void *workspace, uint64_t workspace_bytes,
                               void *stream);

/* eh_decompress_batch without a workspace, for callers that cannot allocate
 * device memory where they decompress: runtimes that plan all device memory
 * ahead of time and forbid later allocations, and allocator callbacks that
 * must not re-enter the allocator.  There is no counterpart on the pages: it
 * is a packaging variant of block decompression.  The decoder's scratch
 * lives in a fixed device array inside the library (256 +
 * EH_NOALLOC_MAX_BATCH * 37,888 bytes, held by every GPU that uses the
 * library until the process exits); nothing is allocated.  k must be in
 * [1, EH_NOALLOC_MAX_BATCH], else EH_ERR_INVALID_ARG.  The first call on a
 * device looks up the array's device address (a failed lookup is retried by
 * the next call).  The call waits for `stream` (a device-to-host copy of the
 * status word and a stream synchronisation) and returns the call's status
 * (EH_OK or a data error), so it cannot be issued on a stream that is being
 * captured into a CUDA graph.  All calls share the array: calls that overlap
 * on the GPU race and must not be issued. */
EH_API eh_status eh_decompress_batch_noalloc(const eh_plan_t *plan, int k,
                                             const eh_compressed_t *cs,
                                             void *const *outs, void *stream);

/* ---- Fixed-slot page store: online K/V cache compression.
 * New K/V pages (one page = one chunk of chunk_elems values, e.g. 64 tokens x
 * 8 heads x 128 dims = 65,536) are coded with a FROZEN codebook (code_len /
 * code of an earlier eh_compress, e.g. of the prefill) into fixed-capacity
 * slots, and decoded on reuse (ZipFloat §3.3 and §4.2: KV entries go to
 * preallocated slots and are decompressed on demand; the paper summary,
 * "局限性": real-time K/V compression needs a high-throughput
 * implementation).  A page whose code does not fit its slot (ceil(bits/8) +
 * 16 > slot_bytes) or that holds an exponent without a code is stored raw:
 * its exponent fields (one byte each) go to the next free page of raw_pool.
 * All arrays are device arrays owned by the caller. */
#define EH_PAGE_RAW 0x80000000u /* page_meta: raw page; low 31 bits = raw index */
typedef struct {
  const uint8_t *code_len; /* device [A]: the frozen codebook                   */
  const uint32_t *code;    /* device [A]                                         */
  uint8_t *slots;          /* device [n_slots][slot_bytes]: codes from bit 0;
                              bytes past ceil(bits/8) are unspecified           */
  uint64_t slot_bytes;     /* multiple of 16                                     */
  uint32_t n_slots;
  uint32_t raw_cap;        /* pages raw_pool can hold                            */
  uint8_t *sign_mant;      /* device [n_slots][sm bytes of one page]             */
  uint32_t *page_meta;     /* device [n_slots]: code bits, or EH_PAGE_RAW | idx  */
  uint8_t *raw_pool;       /* device [raw_cap][chunk_elems] exponent bytes      */
  uint32_t *raw_used;      /* device counter of raw pages taken (zero it once)   */
} eh_page_store_t;

/* Codebook (code_len[A], code[A], device) from exponent counts (device
 * u64[A]), exactly as eh_compress builds it for a tensor with those counts.
 * To freeze a codebook for the page store that codes every exponent, pass the
 * counts of earlier data plus one for every symbol.  Stream-ordered;
 * workspace: the workspace_bytes of eh_compress_bound(plan, 0, ...). */
EH_API eh_status eh_codebook_from_counts(const eh_plan_t *plan, const uint64_t *counts,
                                         uint8_t *code_len, uint32_t *code,
                                         void *workspace, uint64_t workspace_bytes,
                                         void *stream);

/* Codes n_pages full pages (in: n_pages * chunk_elems values, page i first)
 * into the slots slot_ids[i] (device array).  Stream-ordered; a full raw pool
 * sets EH_ERR_NOMEM in the workspace status word.  Workspace: 256 bytes;
 * with 256 + 16 * n_pages bytes, calls of up to a few hundred pages code
 * each page with several CTAs (the result is the same). */
EH_API eh_status eh_pages_append(const eh_plan_t *plan, const eh_page_store_t *store,
                                 const void *in, uint32_t n_pages,
                                 const uint32_t *slot_ids, void *workspace,
                                 uint64_t workspace_bytes, void *stream);

/* Decodes the pages in slots slot_ids[i] (device array) into out (page i at
 * out + i * chunk_elems values).  Workspace: eh_decompress_workspace(plan, 1). */
EH_API eh_status eh_pages_read(const eh_plan_t *plan, const eh_page_store_t *store,
                               const uint32_t *slot_ids, uint32_t n_pages, void *out,
                               void *workspace, uint64_t workspace_bytes, void *stream);

/* The store's codebook is frozen, so its decode tables can be built once:
 * eh_pages_prepare builds them into `tables` (device, 256-byte aligned,
 * eh_decompress_workspace(plan, 1) bytes; an invalid codebook is recorded
 * there and every read with these tables reports EH_ERR_CORRUPT), and
 * eh_pages_read_prepared reads pages with them instead of rebuilding them
 * every call (workspace: 256 bytes, the call's status word).  The tables
 * must be prepared again if store->code_len or store->code change. */
EH_API eh_status eh_pages_prepare(const eh_plan_t *plan, const eh_page_store_t *store,
                                  void *tables, uint64_t tables_bytes, void *stream);
EH_API eh_status eh_pages_read_prepared(const eh_plan_t *plan, const eh_page_store_t *store,
                                        const void *tables, const uint32_t *slot_ids,
                                        uint32_t n_pages, void *out, void *workspace,
                                        uint64_t workspace_bytes, void *stream);

/* ---- Prefetcher: decompression straight into the operand buffers of the
 * next consumer (a GEMM), on a decode stream that runs ahead of the consumer
 * stream.  The DFloat11 article ("方法介绍") decompresses a whole transformer
 * block just before the block runs; the tile-level ANS paper summary (the
 * Lattice page, abstract) aligns decoding with the inference GEMMs.  Here a
 * ring of `depth` caller-owned slots holds decoded blocks: the decode of
 * block i+depth overlaps the consumer's work on blocks i..i+depth-1, and
 * CUDA events order the two streams, so nothing waits on the host.
 *
 * Use (one host thread per prefetcher):
 *   submit(b0) ... submit(b{depth-1})            fill the ring
 *   for each block i: acquire(slot_i, s)          s waits for the decode
 *                     <consumer work on s>        reads the slot
 *                     release(slot_i, s)          slot reusable after that work
 *                     submit(b{i+depth})          decode waits for the release
 * Slots are used round-robin.  submit() fails with EH_ERR_INVALID_ARG (and
 * does nothing) when its slot has not been released since its last submit;
 * acquire() needs a submitted slot and release() an acquired one. */
#define EH_PREFETCH_MAX_DEPTH 8
typedef struct eh_prefetch eh_prefetch;

/* Device workspace for a prefetcher of `depth` slots (1..EH_PREFETCH_MAX_DEPTH):
 * one decompression workspace of EH_MAX_BATCH tensors per slot. */
EH_API eh_status eh_prefetch_workspace(const eh_plan_t *plan, int depth,
                                       uint64_t *workspace_bytes);

/* Creates a prefetcher.  slots[depth]: device buffers of slot_bytes bytes
 * each, 256-byte aligned, owned by the caller; workspace: device, 256-byte
 * aligned, eh_prefetch_workspace() bytes, owned by the caller;
 * decode_stream: the stream the decodes run on (not the consumer's).
 * max_ctas caps the decoder's grid (0: one CTA per SM) so that a consumer
 * running at the same time keeps the other SMs.  The handle (host memory and
 * 2*depth CUDA events) is freed by eh_prefetch_destroy. */
EH_API eh_status eh_prefetch_create(const eh_plan_t *plan, int depth,
                                    void *const *slots, uint64_t slot_bytes,
                                    void *workspace, uint64_t workspace_bytes,
                                    void *decode_stream, uint32_t max_ctas,
                                    eh_prefetch **out);

/* Enqueues the decompression of k (1..EH_MAX_BATCH) tensors into the next
 * slot, after the consumer work released from that slot.  Tensor i lands at
 * byte offsets[i] of the slot (host array of k entries, filled here): each
 * tensor starts on a 256-byte boundary after the previous one.  *slot
 * receives the slot index.  EH_ERR_NOMEM when the tensors do not fit. */
EH_API eh_status eh_prefetch_submit(eh_prefetch *pf, int k, const eh_compressed_t *cs,
                                    uint64_t *offsets, int *slot);

/* Makes consumer_stream wait (on the GPU) for the slot's decode. */
EH_API eh_status eh_prefetch_acquire(eh_prefetch *pf, int slot, void *consumer_stream);

/* Marks the slot reusable once the work enqueued so far on consumer_stream
 * has run. */
EH_API eh_status eh_prefetch_release(eh_prefetch *pf, int slot, void *consumer_stream);

/* Waits for the slot's last decode and returns its status word (EH_OK or a
 * data error, as eh_get_status). */
EH_API eh_status eh_prefetch_status(eh_prefetch *pf, int slot);

/* Waits for the decode stream, destroys the events and frees the handle.
 * NULL is accepted. */
EH_API eh_status eh_prefetch_destroy(eh_prefetch *pf);

/* ---- ZipFloat comparison codec (BF16 only).  A different codec, kept beside
 * the Huffman format as a point of comparison for ratio and speed on the same
 * inputs.  "ZipFloat: An Ultra-fast and Lossless Floating-Point Compressor for
 * LLM Inference Systems": blocks of 2048 values (§3.1); per block the most
 * frequent exponent MD, l_b = (MD - 6) mod 256 and r = (e - l_b) mod 256
 * (§3.2, Eq. 4; ties in MD go to the smaller field); the low three bits of r
 * as three bit planes of 64 words per block (bit i of word w of plane p = bit
 * p of r of element 32w+i), and for r >= 8 a record (i << 5) | (r >> 3) with
 * i the index in the block (§3.3); sign/mantissa bytes (s << 7) | m7.
 * Each block's records are contiguous, in element order, at sparse_off[b];
 * the blocks' ranges are reserved with an atomic, so their order in `sparse`
 * depends on scheduling.  All arrays are device memory owned by the caller;
 * sign_mant and dense 16-byte aligned; n < 2^32. */
typedef struct {
  uint64_t n;            /* values                                          */
  uint8_t *sign_mant;    /* n bytes                                         */
  uint32_t *meta;        /* per block: l_b | (records of the block) << 8    */
  uint32_t *dense;       /* per block 3 planes x 64 words                   */
  uint32_t *sparse_off;  /* per block: index of its first record            */
  uint16_t *sparse;      /* sparse_cap records                              */
  uint64_t sparse_cap;   /* records the buffer holds (n always suffices)    */
  uint64_t n_records;    /* out: records written (when compress waits)      */
} eh_zf_t;

/* blocks = ceil(n / 2048) (length of meta and sparse_off; dense holds
 * 192 * blocks words); sparse_cap = n, which no input exceeds. */
EH_API eh_status eh_zf_bound(uint64_t n, uint64_t *blocks, uint64_t *sparse_cap);

/* Compresses n = out->n BF16 values from `in` (device, 16-byte aligned).
 * workspace: device, >= 256 bytes, 256-byte aligned (status word and the
 * record counter).  wait != 0: waits for the stream, fills out->n_records and
 * returns EH_ERR_NOMEM if the records overflowed sparse_cap.  Otherwise
 * fully stream-ordered (eh_get_status reports the overflow). */
EH_API eh_status eh_zf_compress(const void *in, eh_zf_t *out, void *workspace,
                                uint64_t workspace_bytes, int wait, void *stream);

/* Rebuilds the n values into out (device, 16-byte aligned).  Stream-ordered;
 * a block whose record range or indices are out of bounds is skipped and
 * sets EH_ERR_CORRUPT in the workspace's status word. */
EH_API eh_status eh_zf_decompress(const eh_zf_t *c, void *out, void *workspace,
                                  uint64_t workspace_bytes, void *stream);

/* Waits for `stream` and returns the status word of `workspace`: EH_OK,
 * EH_ERR_CORRUPT, EH_ERR_INFEASIBLE, EH_ERR_NOMEM or EH_ERR_TIMEOUT.  Every compress or
 * decompress call resets the word when it starts, so it describes the most
 * recent call that used this workspace. */
EH_API eh_status eh_get_status(void *workspace, void *stream);

/* ---- Stored form of one compressed tensor.  Weights are compressed once,
 * offline, and decompressed on the GPU when used (the DFloat11 article,
 * "方法介绍"; ZipFloat §4.2): these calls turn a compressed tensor into one
 * self-describing byte container and back.  Layout (little-endian): the
 * magic "EXHF", u16 version 1, u8 dtype, u8 max_code_len, u32 chunk_elems,
 * u32 flags (bit 0: value index present), u64 n, u64 n_chunks, u64
 * exp_stream_bits; six section entries {u64 offset, u64 length, u32 CRC-32,
 * u32 0} for code_len (A bytes), code (A u32), chunk_bit_off (n_chunks+1
 * u64), exp_stream (ceil(bits/8) bytes), sign_mant and value_index (length 0
 * when absent); the CRC-32 of the 184 bytes before it; then the sections at
 * 16-byte aligned offsets from byte 192, zero-padded, the total a multiple of
 * 16.  CRC-32 is the IEEE 802.3 / zlib one.  All pointers are HOST pointers:
 * the caller copies the device arrays to the host before writing and back to
 * device buffers (eh_compress_bound sizes, for the decoder's read-ahead)
 * after reading. */

/* Size in bytes of the container of an n-element tensor with that many code
 * bits (with_index != 0: with a value index). */
EH_API eh_status eh_container_size(const eh_plan_t *plan, uint64_t n, uint64_t exp_stream_bits,
                                   int with_index, uint64_t *bytes);

/* Writes the container of the tensor `c` (its dtype, n, n_chunks,
 * exp_stream_bits and HOST arrays; value_index may be NULL) to dst, which
 * must hold eh_container_size() bytes (else EH_ERR_NOMEM). */
EH_API eh_status eh_container_write(const eh_plan_t *plan, const eh_compressed_t *c, void *dst,
                                    uint64_t dst_bytes);

/* Checks a container (magic, version, plan, sizes, section layout, every
 * CRC-32; EH_ERR_CORRUPT on any mismatch) and fills *plan and *view, whose
 * array pointers point into src (exp_stream_cap = the stream's byte
 * length).  Padding and reserved bytes must be zero, so that a change to any
 * byte of a container is detected.  src_bytes may exceed the container's size
 * (a container inside a larger file): the bytes after it are not read. */
EH_API eh_status eh_container_read(const void *src, uint64_t src_bytes, eh_plan_t *plan,
                                   eh_compressed_t *view);

/* Test hook (not for production use).  The decoder finds the thread
 * boundaries of a chunk in fix-up rounds; a chunk still unresolved after the
 * round limit is reported as EH_ERR_TIMEOUT | corrupt, which consistent data
 * never reaches (the default limit exceeds the rounds any chunk can need).
 * This sets the limit for decompression calls issued afterwards from any
 * thread (rounds >= 1; 0 restores the default), so that tests can make this
 * bounded device-side wait give up and check that the error is reported
 * while the kernel returns normally. */
EH_API eh_status eh_debug_set_fixup_rounds(uint32_t rounds);

/* Static description of a status code. */
EH_API const char *eh_status_str(eh_status s);

/* Library version string, e.g. "libexphuff 0.1 sm_100a". */
EH_API const char *eh_version(void);

#ifdef __cplusplus
}
#endif
#endif /* EXPHUFF_H */

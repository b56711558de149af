// eh_internal.cuh -- shared device-side definitions of libexphuff.
//
// Launch descriptors, workspace layout, status flags and small device helpers
// used by the compress and decompress kernels.  The public interface is
// include/exphuff.h.
#pragma once

#include <cuda_runtime.h>
#include <utility>
#include <stdint.h>

#include "exphuff.h"

namespace eh {

constexpr int kThreads = 512;           // threads per CTA of the compress kernels
constexpr int kDecThreads = 1024;       // threads per CTA of the decoder (one CTA per SM)
constexpr int kMaxChunk = 65536;        // largest chunk (elements)
constexpr int kNumSub = 4;              // second-level decode tables per codebook

// status word flags (bitwise OR of everything a call observed)
constexpr uint32_t kFlagCorrupt = 1u;
constexpr uint32_t kFlagInfeasible = 2u;
constexpr uint32_t kFlagTimeout = 4u;
constexpr uint32_t kFlagNoRoom = 8u;   // raw page pool exhausted

__host__ __device__ inline int alphabet_of(int dtype) { return dtype == EH_FP8_E4M3 ? 16 : 256; }

// Per-tensor part of a launch.
constexpr uint32_t kIndexStride = EH_INDEX_STRIDE;  // values per value-index entry

struct Item {
  const void *in;          // compress: raw values
  void *out;               // decompress: output values
  uint64_t n;              // element count of the tensor
  uint64_t elem0;          // decompress_chunks: element index of out[0]
  uint32_t chunk0;         // global index of this tensor's first chunk in the launch
  uint32_t nchunks;        // chunks of this tensor processed by the launch
  uint32_t first_chunk;    // tensor-local index of the first processed chunk
  uint32_t total_chunks;   // chunks of the whole tensor
  uint8_t *code_len;       // [A]
  uint32_t *code;          // [A]
  uint64_t *off;           // [total_chunks + 1]
  uint8_t *stream;         // exp_stream
  uint64_t stream_cap;     // bytes
  uint8_t *sm;             // sign_mant
  uint32_t *vindex;        // optional value index [total_chunks][chunk_elems / kIndexStride]
  // workspace views
  uint64_t *counts;        // compress: [256] global histogram
  uint32_t *chist;         // compress: [total_chunks][A] per-chunk histograms
  uint64_t *cbits;         // compress: [total_chunks] code bits per chunk
  uint64_t *pm_scratch;    // compress: package-merge package weights
  uint64_t *bits_out;      // compress: total bits (workspace copy)
  uint64_t *bits_dev;      // compress: optional caller copy (may be null)
  void *lut;               // decompress: DecodeTables
  // page store mode (chunks live in fixed slots; null page_meta = tensor mode)
  const uint32_t *slot_ids;  // [nchunks] slot of each page of the call
  const uint32_t *page_meta; // [n_slots] code bits, or EH_PAGE_RAW | raw index
  const uint8_t *raw_pool;   // [raw_cap][chunk_elems] exponent bytes
  uint64_t slot_bytes;
  uint32_t n_slots;
  uint32_t raw_cap;
};

// Launch descriptor of the page append kernel.
struct PageLaunch {
  const void *in;
  const uint32_t *slot_ids;
  uint32_t n_pages;
  uint32_t page_elems;
  const uint8_t *code_len;
  const uint32_t *code;
  uint8_t *slots;
  uint64_t slot_bytes;
  uint32_t n_slots;
  uint32_t raw_cap;
  uint8_t *sm;
  uint32_t *page_meta;
  uint8_t *raw_pool;
  uint32_t *raw_used;
  uint32_t *status;
  uint32_t *part_bits;     // split append: [n_pages][kPageParts] code bits | missing << 31 (null: one CTA a page)
  int32_t dtype;
};
constexpr uint32_t kPageParts = 4;  // CTAs per page in the split append

struct Batch {
  Item item[EH_MAX_BATCH];
  uint32_t k;
  uint32_t total_chunks;   // sum of item[i].nchunks
  uint32_t chunk_elems;
  int32_t dtype;
  uint32_t max_code_len;
  uint32_t *status;        // workspace status word
  uint32_t *ticket;        // workspace counter for last-block-done patterns
  uint32_t fixup_rounds;   // decoder: fix-up rounds before giving up (0: the default)
};

// Item that owns global chunk g (linear scan; k <= 16).
__device__ __forceinline__ int find_item(const Batch &b, uint32_t g) {
  int i = 0;
  #pragma unroll 1
  while (i + 1 < (int)b.k && g >= b.item[i + 1].chunk0) i++;
  return i;
}

__device__ __forceinline__ uint32_t bswap32(uint32_t x) { return __byte_perm(x, 0, 0x0123); }

__device__ __forceinline__ void set_status(uint32_t *status, uint32_t flag) {
  atomicOr(status, flag);
}

// Decode tables for one codebook, built by the table kernel into the
// workspace and copied to shared memory by each decoding CTA.
//
// First level, indexed by the next kLutBits stream bits: .x holds the symbols
// (in the decoder's output form) of the first four complete codes, 8 bits
// each, first in the low byte; .y is a meta word:
//   bits  0..3  bits of all complete codes in the index bits
//   bit   4     zero (a wrap-mode shift by the whole word shifts by bits 0..3)
//   bits  5..15 a complete code starts at offset 1..11 (offset 0 always does)
//   bits 16..19 number of complete codes (0: the first code is longer than the
//               index; then the whole entry is zero)
//   bits 20..23 bits of the first (up to four) codes
//   bits 24..31 8 * their number
// Second level, for the first kNumSub prefixes (from sub0 on) of codes longer
// than the index, indexed by the 8 bits after the prefix.  u32 entry:
//   bits 0..7 symbol (output form), bits 8..13 code length (0: longer ->
//   search).  The search path handles any length up to 32 with the canonical
//   limits.
constexpr int kLutBits = 12;
constexpr uint32_t kMetaStartShift = 5;
struct alignas(16) DecodeTables {  // copied to shared memory in 16-byte words
  uint2 l1[1 << kLutBits];
  uint32_t sub[kNumSub][256];
  uint64_t lim[33];        // (first[L] + count[L]) << (32 - L): left-justified limits
  uint32_t first[33];      // first canonical code of length L
  uint32_t base[33];       // index in `sorted` of the first code of length L
  uint8_t sorted[256];     // symbols (output form) in (length, symbol) order
  uint32_t sub0;           // first prefix of a code longer than the index
  uint32_t gcd;            // gcd of the code lengths in use
  uint32_t maxlen;
  uint32_t nsym;
  uint32_t err;            // nonzero: codebook invalid
};

static_assert(sizeof(DecodeTables) % 16 == 0, "the decoder copies the tables in 16-byte words");
constexpr uint64_t kLutBytes = (sizeof(DecodeTables) + 255) & ~uint64_t(255);

__host__ __device__ inline uint64_t align256(uint64_t x) { return (x + 255) & ~uint64_t(255); }

// ---- host-side launch wrappers (defined in the .cu files)
// Programmatic dependent launch: a kernel launched with launch_pdl may start
// while the previous kernel of the stream is still running; it calls
// pdl_wait() before touching anything that kernel (or an earlier one) wrote.
// pdl_trigger() lets the next such kernel start before this one ends.
__device__ __forceinline__ void pdl_wait() { asm volatile("griddepcontrol.wait;" ::: "memory"); }
__device__ __forceinline__ void pdl_trigger() { asm volatile("griddepcontrol.launch_dependents;" ::: "memory"); }

template <typename... KArgs, typename... Args>
inline cudaError_t launch_pdl(void (*kernel)(KArgs...), dim3 grid, dim3 block, size_t smem, cudaStream_t s,
                              Args &&...args) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = smem;
  cfg.stream = s;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, kernel, std::forward<Args>(args)...);
}

cudaError_t launch_hist(const Batch &b, cudaStream_t s);
cudaError_t launch_book(const Batch &b, cudaStream_t s);
cudaError_t launch_offsets(const Batch &b, cudaStream_t s);
cudaError_t launch_encode(const Batch &b, cudaStream_t s);
cudaError_t launch_page_append(const PageLaunch &pl, cudaStream_t s);
cudaError_t launch_tables(const Batch &b, cudaStream_t s);
cudaError_t launch_decode(const Batch &b, cudaStream_t s, int num_sms);
cudaError_t configure_decode();  // once per device, before the first decode launch
cudaError_t configure_encode();  // once per device, before the first encode launch

// Validates a decompression call (k tensors, optional chunk ranges) and
// launches the table and decode kernels on `stream`.  max_ctas caps the
// decoder's grid (0: one CTA per SM), leaving SMs free for concurrent work.
eh_status decompress_impl(const eh_plan_t *plan, int k, const eh_compressed_t *cs, void *const *outs,
                          const uint32_t *firsts, const uint32_t *counts, void *workspace,
                          uint64_t workspace_bytes, void *stream, uint32_t max_ctas);

}  // namespace eh

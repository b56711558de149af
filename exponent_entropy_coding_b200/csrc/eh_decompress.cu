// eh_decompress.cu -- decompression kernels of libexphuff (sm_100a).
//
//   tables  sixteen CTAs per codebook: validate the code lengths and codes and
//           build the decode tables (a 12-bit first level giving, for the
//           index bits, the number, bits and start offsets of all complete
//           codes and the symbols and bits of the first four; 8-bit second
//           levels for codes of 13..20 bits; canonical limits for anything
//           longer);
//   decode  persistent CTAs of two independent groups, one chunk per group
//           at a time:
//             1. the chunk's bit range is copied into shared memory with one
//                bulk asynchronous copy (cp.async.bulk + mbarrier) when it
//                fits, else read from global memory;
//             2. every thread counts the codes of its own window of the
//                chunk's bits, starting speculatively at the window start and
//                recording the code boundaries of its first 64 bits;
//             3. fix-up: each thread restarts from the end of its
//                predecessor's codes and stops as soon as it lands on one of
//                its recorded boundaries (Huffman codes resynchronise after a
//                few codes);
//             4. group-wide exclusive scan of the per-thread code counts
//                gives every thread its first output index;
//             5. every thread decodes again from its true start and writes a
//                run of whole exponent words to shared memory: the run starts
//                at the first multiple of 4 (16 for a warp's first thread) at
//                or after its first code and ends where its successor's run
//                starts, so no word is shared and no buffer is cleared;
//             6. each warp merges its own runs with the sign/mantissa stream
//                as soon as they are written (no group barrier) and stores
//                them with 16-byte coalesced stores.
// The DFloat11 article ("方法介绍") describes compact LUTs sized for on-chip
// SRAM, a two-phase kernel coordinating where each thread reads and writes,
// and block-level decompression; here the per-thread start positions are not
// stored in the format but recovered by the self-synchronising fix-up.
#include "eh_internal.cuh"

namespace eh {
namespace {

constexpr uint32_t kMaskBits = 64;            // code starts recorded per thread
constexpr uint64_t kWaitLimitNs = 200000000ull;  // a stage copy not landed after 0.2 s is given up

// ---------------------------------------------------------------- tables
// kTabParts CTAs of 256 threads per codebook; each builds 1/kTabParts of the
// first level (one entry a thread), parts 0..kNumSub-1 one second-level table
// each, part 0 also the limits.
constexpr uint32_t kTabParts = 16;

// Smallest L in [1, 32] with x < lim[L], 33 if there is none (lim is
// nondecreasing for a valid code).
__device__ __forceinline__ uint32_t code_length_of(uint32_t x, const uint64_t *limL) {
  uint32_t lo = 1, hi = 33;
  while (lo < hi) {
    const uint32_t mid = (lo + hi) >> 1;
    if ((uint64_t)x < limL[mid]) hi = mid;
    else lo = mid + 1;
  }
  return lo;
}

// The form in which the decoder keeps a decoded symbol.  BF16 exponents are
// rotated right by one bit, (e >> 1) | (e & 1) << 7: the high bits then sit
// where the high byte of the BF16 value needs them and the low bit where the
// low byte does, so two byte permutes and one bit select rebuild two values.
__device__ __forceinline__ uint32_t out_form(int dtype, uint32_t e) {
  return dtype == EH_BF16 ? ((e >> 1) | ((e & 1u) << 7)) : e;
}

__global__ void __launch_bounds__(256) tables_kernel(const __grid_constant__ Batch b) {
  const uint32_t part = blockIdx.x % kTabParts;
  const Item &I = b.item[blockIdx.x / kTabParts];
  DecodeTables *T = (DecodeTables *)I.lut;
  const int A = alphabet_of(b.dtype);
  const int tid = threadIdx.x;
  __shared__ uint32_t cntL[33], firstL[33], baseL[33];
  __shared__ uint64_t limL[33];
  __shared__ uint8_t srt[256];
  __shared__ uint32_t err;
  __shared__ uint32_t wlen[8][33];  // per warp: symbols of each length

  pdl_trigger();
  pdl_wait();  // the codebooks may come from the kernels just before
  if (blockIdx.x == 0 && tid == 0) {
    *b.status = 0u;  // this call's status starts clean
    *b.ticket = 0u;
  }
  if (tid <= 32) cntL[tid] = 0;
  for (int i = tid; i < 8 * 33; i += 256) (&wlen[0][0])[i] = 0;
  if (tid == 0) err = 0;
  const uint32_t l = tid < A ? I.code_len[tid] : 0u;
  __syncthreads();
  if (l > 32) atomicOr(&err, 1u);
  else if (l) {
    atomicAdd(&cntL[l], 1u);
    atomicAdd(&wlen[tid >> 5][l], 1u);
  }
  const uint32_t nsym = __syncthreads_count(l > 0 && l <= 32);
  if (tid < 32) {
    // Canonical limits by one warp, lane L-1 for length L: with
    // a_L = count_L << (32 - L), the inclusive prefix of a is lim[L] and the
    // exclusive one, shifted down, is the first code of length L.
    const uint32_t L = tid + 1, cL = cntL[L];
    const uint64_t aL = (uint64_t)cL << (32 - L);
    uint64_t inc = aL;
    uint32_t idx = cL;
    #pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const uint64_t y = __shfl_up_sync(0xffffffffu, inc, o);
      const uint32_t z = __shfl_up_sync(0xffffffffu, idx, o);
      if (tid >= (uint32_t)o) {
        inc += y;
        idx += z;
      }
    }
    limL[L] = inc;
    firstL[L] = (uint32_t)((inc - aL) >> (32 - L));
    baseL[L] = idx - cL;
    // lengths in use: their gcd (largest d dividing all of them) and maximum
    const uint32_t used = __ballot_sync(0xffffffffu, cL != 0);
    uint32_t mult = 0;  // lengths that are multiples of d = L
    for (uint32_t k = L; k <= 32; k += L) mult |= 1u << (k - 1);
    const uint32_t divides = __ballot_sync(0xffffffffu, used && (used & ~mult) == 0);
    const uint64_t kraft = __shfl_sync(0xffffffffu, inc, 31);  // every lane takes part
    if (tid == 0 && kraft > (1ull << 32)) err = 1;
    if (tid == 0) {
      limL[0] = 0;
      firstL[0] = baseL[0] = cntL[0] = 0;
      if (I.n > 0 && nsym == 0) err = 1;
      if (part == 0) {
        T->gcd = divides ? 32u - __clz(divides) : 1u;
        T->maxlen = used ? 32u - __clz(used) : 0u;
        T->nsym = nsym;
      }
    }
  }
  __syncthreads();
  // symbol order (length, symbol); the stored codes must be the canonical ones
  // rank among the symbols of equal length below this one: earlier warps'
  // counts plus the matching lower lanes of this warp
  const uint32_t same = __match_any_sync(0xffffffffu, l);
  if (tid < A && l && l <= 32) {
    uint32_t k = __popc(same & ((1u << (tid & 31)) - 1u));
    for (int w = 0; w < (tid >> 5); w++) k += wlen[w][l];
    srt[baseL[l] + k] = (uint8_t)tid;
    if (I.code[tid] != firstL[l] + k) atomicOr(&err, 1u);
  }
  if (tid <= 32 && part == 0) {
    T->first[tid] = firstL[tid];
    T->base[tid] = baseL[tid];
    T->lim[tid] = limL[tid];
  }
  __syncthreads();
  if (err) {  // invalid codebook: nothing below may index with its values
    if (tid == 0 && part == 0) T->err = err;
    return;
  }
  if (part == 0) T->sorted[tid] = tid < (int)nsym ? (uint8_t)out_form(b.dtype, srt[tid]) : (uint8_t)0;

  // first level.  Codes longer than kLutBits fill the left-justified range
  // [lim[kLutBits], lim[32]), so their prefixes are consecutive from sub0 on:
  // the first kNumSub of them get a second-level table.
  constexpr uint32_t kShift = 32 - kLutBits;
  const uint32_t sub0 = (uint32_t)(limL[kLutBits] >> kShift);
  if (part == 0 && tid == 0) T->sub0 = sub0;
  constexpr uint32_t kPerPart = (1u << kLutBits) / kTabParts;
  for (uint32_t p = part * kPerPart + tid; p < (part + 1) * kPerPart; p += 256) {
    // every complete code inside the index bits (their number, bits and
    // starts), and the symbols of the first four
    uint32_t syms = 0, pos = 0, nc = 0, bnd = 0, pos4 = 0, nc4 = 0;
    while (pos < (uint32_t)kLutBits) {
      const uint32_t x = (p << kShift) << pos;  // next bits, left-justified, zero-filled
      const uint32_t L = code_length_of(x, limL);
      if (L > (uint32_t)kLutBits - pos) break;  // not complete inside the index bits
      if (nc < 4) {
        const uint32_t v = x >> (32 - L);
        syms |= out_form(b.dtype, srt[baseL[L] + v - firstL[L]]) << (8 * nc);
        pos4 = pos + L;
        nc4 = nc + 1;
      }
      bnd |= 1u << pos;
      pos += L;
      nc++;
    }
    uint32_t meta = 0;  // a prefix without a complete code: every field zero
    if (nc) meta = pos | ((bnd >> 1) << kMetaStartShift) | (nc << 16) | (pos4 << 20) | ((8u * nc4) << 24);
    T->l1[p] = make_uint2(syms, meta);
  }
  // second level (one table per part): codes of kLutBits+1 .. kLutBits+8 bits
  if (part < (uint32_t)kNumSub) {
    const uint32_t j = part;
    uint32_t e = 0;
    const uint32_t p = sub0 + j;
    if (((uint64_t)p << kShift) < limL[32]) {
      const uint32_t x = (p << kShift) | ((uint32_t)tid << (kShift - 8));
      for (uint32_t L = kLutBits + 1; L <= (uint32_t)kLutBits + 8; L++) {
        if ((uint64_t)x < limL[L]) {
          if (x >= (uint32_t)(limL[L - 1])) {
            const uint32_t v = x >> (32 - L);
            e = out_form(b.dtype, srt[baseL[L] + v - firstL[L]]) | (L << 8);
          }
          break;
        }
      }
    }
    T->sub[j][tid] = e;
  }
  if (tid == 0 && part == 0) T->err = err;
}

// ---------------------------------------------------------------- decode
// Accessors of a first-level meta word (see DecodeTables).
__device__ __forceinline__ uint32_t meta_starts(uint32_t m) {  // code starts at offsets 0..11
  return ((m >> (kMetaStartShift - 1)) & 0xFFEu) | 1u;
}
constexpr uint32_t kCountFields = 0x000F000Fu;  // bits of all codes | their number << 16

// 32 stream bits starting at bit q of a thread's frame (stream words are
// byte-swapped on load to MSB-first order).
// Shared-memory loads by 32-bit shared address.
__device__ __forceinline__ uint32_t lds32(uint32_t a) {
  uint32_t v;
  asm volatile("ld.shared.u32 %0, [%1];" : "=r"(v) : "r"(a));
  return v;
}
__device__ __forceinline__ uint2 lds64(uint32_t a) {
  uint2 v;
  asm volatile("ld.shared.v2.u32 {%0,%1}, [%2];" : "=r"(v.x), "=r"(v.y) : "r"(a));
  return v;
}
template <bool kSmem>
struct Peek {
  const uint32_t *w;
  __device__ __forceinline__ uint32_t word(uint32_t i) const {
    return bswap32(kSmem ? lds32((uint32_t)__cvta_generic_to_shared(w) + 4 * i) : __ldg(w + i));
  }
  __device__ __forceinline__ uint32_t operator()(uint32_t q) const {
    const uint32_t i = q >> 5;
    return __funnelshift_l(word(i + 1), word(i), q);  // the shift is taken modulo 32
  }
};

// The same 32 bits from two cached words: each call may move at most 32
// bits past the previous one (one word), and loads one new word when the
// position enters the next word.  The counting passes move at most 24 bits a
// lookup pair and at most 32 a code, and they are bound by shared-memory
// bandwidth: this halves their stream loads.
template <bool kSmem>
struct Cursor {
  Peek<kSmem> src;
  uint32_t i, a, b;  // a, b: stream words i, i+1
  __device__ __forceinline__ void seek(uint32_t q) {
    i = q >> 5;
    a = src.word(i);
    b = src.word(i + 1);
  }
  __device__ __forceinline__ uint32_t operator()(uint32_t q) {
    const uint32_t j = q >> 5;
    if (j != i) {  // j == i + 1
      a = b;
      b = src.word(j + 1);
      i = j;
    }
    return __funnelshift_l(b, a, q);
  }
};

__device__ __forceinline__ uint32_t lut_index(uint32_t x) { return x >> (32 - kLutBits); }

// A code longer than the first-level index (its prefix has no complete
// code): second-level table, else search of the canonical limits.  Returns
// the symbol (output form) | length << 8, or 0 for an invalid code.
__device__ __noinline__ uint32_t decode_long(const DecodeTables &T, uint32_t x) {
  const uint32_t si = lut_index(x) - T.sub0;
  if (si < (uint32_t)kNumSub) {
    const uint32_t e2 = T.sub[si][(x >> (24 - kLutBits)) & 0xFFu];
    if (e2 >> 8) return e2;
  }
  uint32_t L = kLutBits + 1;
  while (L <= 32 && (uint64_t)x >= T.lim[L]) L++;
  if (L > 32) return 0;
  const uint32_t v = L == 32 ? x : x >> (32 - L);
  return T.sorted[T.base[L] + (v - T.first[L])] | (L << 8);
}

// One counting step on the next 32 bits `x`, taking only codes that start in
// the next `lim` (>= 1) bits.  Returns the number of codes taken (0: invalid
// code), the bits up to the end of the last one and their starts as a bitmap.
__device__ __forceinline__ uint32_t count_step(const DecodeTables &T, uint32_t x, uint32_t lim, uint32_t &nbits,
                                               uint32_t &bnd) {
  const uint32_t tab = (uint32_t)__cvta_generic_to_shared(&T.l1[0]);
  const uint32_t m = lds32(tab + 8 * lut_index(x) + 4);
  uint32_t k = (m >> 16) & 15u;
  if (!k) {
    const uint32_t d = decode_long(T, x);
    bnd = 1u;
    nbits = d >> 8;
    return d ? 1u : 0u;
  }
  uint32_t nb = m & 15u, bm = meta_starts(m);
  if (nb > lim) {
    // codes starting at or after the limit belong to the next window
    const uint32_t keep = bm & ((1u << lim) - 1u);
    const uint32_t rest = bm >> lim;
    k = __popc(keep);
    nb = rest ? lim + __ffs(rest) - 1 : nb;
    bm = keep;
  }
  nbits = nb;
  bnd = bm;
  return k;
}

// The decoding CTA holds two independent groups of kGroupThreads threads.
// Each group decodes its own chunk into its own exponent buffer, so one
// group's memory-bound output overlaps the other's decode; the decode tables
// are shared.
constexpr uint32_t kGroupThreads = 512;
constexpr uint32_t kGroupWarps = kGroupThreads / 32;
constexpr uint32_t kNumGroups = kDecThreads / kGroupThreads;
constexpr uint32_t kGroupStage = 27136;  // bytes of stream staged per group

// Where one chunk's bits are and whether they fit a shared-memory stage.
struct ChunkInfo {
  int item;
  uint32_t c;       // tensor-local chunk index (page index of the call in page mode)
  uint32_t cnt;     // values in the chunk
  uint32_t nbits;   // code bits of the chunk
  uint32_t rel0;    // first bit of the chunk relative to byte `lo`
  uint32_t bytes;   // stream bytes staged (multiple of 16)
  uint64_t lo;      // first staged stream byte (multiple of 16)
  uint64_t sm_off;  // byte offset of the chunk's sign/mantissa array
  uint64_t out_off; // index in `out` of the chunk's first value
  uint32_t raw;     // page mode: raw page index + 1 (0: coded)
  bool ok;          // offsets consistent with the buffer
  bool fits;        // bits staged in shared memory
};

struct GroupSmem {
  alignas(128) uint32_t stage[kGroupStage / 4 + 16];  // bulk-copy target (stream bytes as stored)
  // decoded exponents (output form) of one chunk: value j at byte
  // j + 4 * (j / 128), so that runs starting about 128 values apart store to
  // different banks
  alignas(16) uint8_t exps[kMaxChunk + 4 * (kMaxChunk / 128)];
  uint32_t ends[kGroupThreads];                       // end bit of every thread's codes
  uint32_t wsum[2][kGroupWarps];                      // scan: warp totals, by round parity
  alignas(8) unsigned long long mbar;
  ChunkInfo next[2];                                  // the group's next chunk, by chunk parity
  uint32_t writers_done;                              // warps done reading the stage
  uint32_t issued;                                    // stage copies started
};

struct DecodeSmem {
  alignas(16) DecodeTables tabs;
  GroupSmem grp[kNumGroups];
  uint32_t abort_flag;
};
static_assert(sizeof(DecodeSmem) + 128 <= 232448, "decoder shared memory exceeds the per-CTA limit");

__device__ __forceinline__ uint32_t smem_u32(const void *p) {
  return (uint32_t)__cvta_generic_to_shared(p);
}

__device__ __forceinline__ void mbar_init(unsigned long long *bar, uint32_t count) {
  asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(smem_u32(bar)), "r"(count));
}

__device__ __forceinline__ void mbar_expect_tx(unsigned long long *bar, uint32_t bytes) {
  asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(smem_u32(bar)), "r"(bytes)
               : "memory");
}

__device__ __forceinline__ bool mbar_try_wait(unsigned long long *bar, uint32_t parity) {
  uint32_t ok;
  asm volatile(
      "{\n .reg .pred p;\n mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n selp.u32 %0, 1, 0, p;\n}"
      : "=r"(ok)
      : "r"(smem_u32(bar)), "r"(parity)
      : "memory");
  return ok != 0;
}

__device__ __forceinline__ uint64_t global_ns() {
  uint64_t t;
  asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
  return t;
}

// Waits for the phase `parity` of the barrier; false if it has not completed
// within kWaitLimitNs.
__device__ __forceinline__ bool mbar_wait_bounded(unsigned long long *bar, uint32_t parity) {
  if (mbar_try_wait(bar, parity)) return true;
  const uint64_t t0 = global_ns();
  for (;;) {
    for (int i = 0; i < 64; i++)
      if (mbar_try_wait(bar, parity)) return true;
    if (global_ns() - t0 > kWaitLimitNs) return false;
  }
}

__device__ __forceinline__ void bulk_g2s(void *dst, const void *src, uint32_t bytes, unsigned long long *bar) {
  asm volatile(
      "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(
          smem_u32(dst)),
      "l"(src), "r"(bytes), "r"(smem_u32(bar))
      : "memory");
}

__device__ __forceinline__ uint4 ld_nc16(const void *p) {
  uint4 v;
  asm volatile("ld.global.nc.L1::no_allocate.v4.u32 {%0,%1,%2,%3}, [%4];"
               : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w)
               : "l"(p));
  return v;
}

__device__ __forceinline__ uint2 ld_nc8(const void *p) {
  uint2 v;
  asm volatile("ld.global.nc.L1::no_allocate.v2.u32 {%0,%1}, [%2];" : "=r"(v.x), "=r"(v.y) : "l"(p));
  return v;
}

// Byte permute with the sign-replicating selector bit (PTX prmt, default
// mode: selector nibble bit 3 set = the selected byte's top bit repeated).
__device__ __forceinline__ uint32_t prmt(uint32_t a, uint32_t b, uint32_t sel) {
  uint32_t d;
  asm("prmt.b32 %0, %1, %2, %3;" : "=r"(d) : "r"(a), "r"(b), "r"(sel));
  return d;
}

// Named barrier shared by both groups (ids 1 and 2 are the groups' own).
constexpr uint32_t kStaggerBarrier = 3;
__device__ __forceinline__ void named_sync(uint32_t id, uint32_t n) {
  asm volatile("bar.sync %0, %1;" ::"r"(id), "r"(n) : "memory");
}
__device__ __forceinline__ void named_arrive(uint32_t id, uint32_t n) {
  asm volatile("bar.arrive %0, %1;" ::"r"(id), "r"(n) : "memory");
}

// Barriers of one group: named barrier `id` over kGroupThreads threads.
__device__ __forceinline__ bool gsync_or(uint32_t id, bool pred) {
  uint32_t r;
  asm volatile(
      "{\n .reg .pred pi, po;\n setp.ne.u32 pi, %1, 0;\n bar.red.or.pred po, %2, %3, pi;\n"
      " selp.u32 %0, 1, 0, po;\n}"
      : "=r"(r)
      : "r"((uint32_t)pred), "r"(id), "n"(kGroupThreads)
      : "memory");
  return r != 0;
}

// Exclusive scan of v over the group with one barrier, which also ORs `pred`
// over the group (*any).  Every warp reduces the warp totals itself.  wsum
// must alternate between consecutive calls (a warp may write the next call's
// total while another still reads this one's).
__device__ __forceinline__ uint32_t group_excl_scan_or(uint32_t v, bool pred, uint32_t *wsum, uint32_t *total,
                                                       bool *any, uint32_t id, uint32_t gtid) {
  const uint32_t lane = gtid & 31u, warp = gtid >> 5;
  uint32_t x = v;
  #pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const uint32_t y = __shfl_up_sync(0xffffffffu, x, o);
    if (lane >= (uint32_t)o) x += y;
  }
  if (lane == 31) wsum[warp] = x;
  *any = gsync_or(id, pred);
  const uint32_t t = lane < kGroupWarps ? wsum[lane] : 0u;
  *total = __reduce_add_sync(0xffffffffu, t);  // one warp reduction each
  const uint32_t pre = __reduce_add_sync(0xffffffffu, lane < warp ? t : 0u);
  return pre + x - v;
}

// A run of decoded symbols written as whole 32-bit words of the exponent
// buffer, which the run owns: four symbols to a word, first in the low byte.
// The current word is stored after every append, complete or not (a later
// append completes it), so no append branches.
struct RunWriter {
  uint32_t *base;
  uint32_t w;    // word being filled (exponents 4w .. 4w+3; stored at word w + w/32)
  uint32_t lo;   // its bytes so far (those above f are zero)
  uint32_t f;    // bits of it filled: 0, 8, 16 or 24
  __device__ __forceinline__ void init(uint8_t *exps, uint32_t j) {  // j: a multiple of 4
    base = (uint32_t *)exps;
    w = j >> 2;
    lo = 0;
    f = 0;
  }
  // up to four symbols, first in the low byte, zero above; k8 = 8 * count
  __device__ __forceinline__ void put(uint32_t syms, uint32_t k8) {
    const uint32_t t = lo | (syms << f);
    const uint32_t h = __funnelshift_l(syms, 0u, f);  // the bytes past the word; none for f = 0
    base[w + (w >> 5)] = t;
    f += k8;
    const bool full = f >= 32;
    lo = full ? h : t;
    w += full ? 1 : 0;
    f &= 31u;
  }
  // a run that ends inside a word (a chunk's last run): its last bytes
  __device__ __forceinline__ void finish() {
    if (f) base[w + (w >> 5)] = lo;
  }
};

// Steps 2-5 for one chunk whose bits are [rel0, rel0 + nbits) of `words`,
// decoded by one group.  Returns false (group-uniform) if the chunk is
// corrupt; else *r0, *r1 receive the warp's region [r0, r1) of the chunk's
// values (r0 a multiple of 16), whose exponents the warp's threads wrote.
template <bool kSmem>
__device__ bool decode_chunk(GroupSmem &G, const DecodeTables &T, const uint32_t *words, uint32_t rel0,
                             uint32_t nbits, uint32_t cnt, uint32_t id, uint32_t gtid, uint32_t *timeout,
                             uint32_t *r0, uint32_t *r1, bool late, uint32_t max_rounds) {
  const uint32_t lane = gtid & 31u;
  const uint32_t tab = (uint32_t)__cvta_generic_to_shared(&T.l1[0]);
  // window width: a multiple of the gcd of the code lengths, so that a
  // fixed-length code starts every window on a code boundary
  const uint32_t gq = T.gcd;
  uint32_t W = (nbits + kGroupThreads - 1) / kGroupThreads;
  if (gq > 1) W = (W + gq - 1) / gq * gq;
  const uint32_t ws = min(gtid * W, nbits), we = min(ws + W, nbits);
  // The thread's frame: frame bit q is chunk bit ws + q - q0.
  const uint32_t q0 = (rel0 + ws) & 31u;
  const uint32_t qe = q0 + (we - ws);
  Peek<kSmem> peek{words + ((rel0 + ws) >> 5)};
  Cursor<kSmem> cur{peek};
  cur.seek(q0);
  // Bulk counting runs while 2 * kLutBits bits of the window remain: two
  // first-level lookups per 32-bit peek, no window-end handling.
  constexpr uint32_t kBulk = 2 * kLutBits;

  // 2. speculative count of the own window; P = frame position | count << 16.
  //    Record where codes start in the window's first kMaskBits bits.
  uint32_t P = q0;
  uint64_t mask = 0;
  bool bad = false;
  // (a) while the recorded bits last
  for (;;) {
    const uint32_t q = P & 0xFFFFu;
    if (q + kBulk > qe || q >= q0 + kMaskBits) break;
    const uint32_t x = cur(q);
    const uint32_t m1 = lds32(tab + 8 * lut_index(x) + 4);
    const uint32_t off = q - q0;
    if (!(m1 & 0xF0000u)) {
      const uint32_t d = decode_long(T, x);
      if (!d) { bad = true; break; }
      mask |= 1ull << off;
      P += (d >> 8) + 0x10000u;
      continue;
    }
    // a prefix with no complete code has every field zero; a code always
    // starts right after the first lookup's codes
    const uint32_t m2 = lds32(tab + 8 * lut_index(__funnelshift_l(0u, x, m1)) + 4);
    mask |= (uint64_t)meta_starts(m1) << off;
    const uint32_t off2 = off + (m1 & 15u);
    if (off2 < kMaskBits) mask |= (uint64_t)meta_starts(m2) << off2;
    P += (m1 & kCountFields) + (m2 & kCountFields);
  }
  // (b) the rest of the window, counting only
  while (!bad) {
    const uint32_t q = P & 0xFFFFu;
    if (q + kBulk > qe) break;
    const uint32_t x = cur(q);
    const uint32_t m1 = lds32(tab + 8 * lut_index(x) + 4);
    if (!(m1 & 0xF0000u)) {
      const uint32_t d = decode_long(T, x);
      if (!d) { bad = true; break; }
      P += (d >> 8) + 0x10000u;
      continue;
    }
    const uint32_t m2 = lds32(tab + 8 * lut_index(__funnelshift_l(0u, x, m1)) + 4);
    P += (m1 & kCountFields) + (m2 & kCountFields);
  }
  // (c) the window's last bits, taking only codes that start inside it
  while (!bad) {
    const uint32_t q = P & 0xFFFFu;
    if (q >= qe) break;
    uint32_t nb, bnd;
    const uint32_t k = count_step(T, cur(q), qe - q, nb, bnd);
    if (!k) { bad = true; break; }
    const uint32_t off = q - q0;
    if (off < kMaskBits) mask |= (uint64_t)bnd << off;
    P += nb + (k << 16);
  }
  const uint32_t spec_end = bad ? we : ws + (P & 0xFFFFu) - q0, spec_n = P >> 16;
  const uint64_t spec_mask = bad ? 0ull : mask;
  uint32_t my_start = ws, my_end = spec_end, my_n = spec_n;
  G.ends[gtid] = my_end;
  if (gsync_or(id, late)) {  // the stage copy of some thread came late
    if (gtid == 0) *timeout |= 1u;
    return false;
  }

  // 3-4. fix-up round: restart from the predecessor's end until a code starts
  //    where a speculative one did (from there on the speculative count is
  //    right); then the scan of the counts, whose barrier also tells whether
  //    any end moved.  A successor may read an end in the round it moves,
  //    before or after the store: an older end only costs it another round.
  uint32_t o, total;
  for (uint32_t round = 0;; round++) {
    const uint32_t pred = gtid == 0 ? 0u : G.ends[gtid - 1];
    bool changed = false;
    if (gtid > 0 && pred != my_start) {
      my_start = pred;
      uint32_t q = pred - ws + q0, k = 0;
      bool synced = false, bad2 = false;
      cur.seek(q);
      while (q < qe) {
        uint32_t nb, bnd;
        const uint32_t kk = count_step(T, cur(q), qe - q, nb, bnd);
        if (!kk) { bad2 = true; break; }
        const uint32_t off = q - q0;
        if (off < kMaskBits) {
          const uint64_t common = ((uint64_t)bnd << off) & spec_mask;
          if (common) {
            const uint32_t s = __ffsll(common) - 1;  // offset from q0, >= off
            k += __popc(bnd & ((1u << (s - off)) - 1u));
            q = q0 + s;
            synced = true;
            break;
          }
        }
        q += nb;
        k += kk;
      }
      uint32_t new_end;
      if (synced) {
        my_n = k + spec_n - __popcll(spec_mask & ((1ull << (q - q0)) - 1ull));
        new_end = spec_end;
        bad = false;
      } else {
        my_n = k;
        new_end = bad2 ? we : ws + q - q0;
        bad = bad2;
      }
      changed = new_end != my_end;
      my_end = new_end;
    }
    if (changed) G.ends[gtid] = my_end;
    // a bad window adds a count no chunk has, so the total check fails
    bool any_changed;
    o = group_excl_scan_or(my_n + (bad ? 0x100000u : 0u), changed, G.wsum[round & 1], &total, &any_changed,
                           id, gtid);
    if (!any_changed) break;
    if (round + 1 >= max_rounds) {  // the round limit: more rounds than threads cannot happen for consistent data
      if (gtid == 0) *timeout |= 1u;
      total = ~0u;
      break;
    }
  }
  const bool ok = total == cnt && G.ends[kGroupThreads - 1] == nbits;
  if (!ok) return false;

  // 5. the thread's run: from the first multiple of 4 at or after its first
  //    output index, to where the next thread's run starts.
  //    The warp's region [rs, re) starts at the first multiple of 16 at or
  //    after its first thread's first output index; every run is clamped to
  //    it, so the runs of a warp tile exactly its region and no other warp
  //    stores into it.
  const uint32_t o1 = o + my_n;
  const uint32_t rs = __shfl_sync(0xffffffffu, gtid == 0 ? 0u : min((o + 15u) & ~15u, cnt), 0);
  const uint32_t re =
      __shfl_sync(0xffffffffu, gtid == kGroupThreads - 1 ? cnt : min((o1 + 15u) & ~15u, cnt), 31);
  const uint32_t a0 = lane == 0 ? rs : min(max((o + 3u) & ~3u, rs), re);
  const uint32_t a1 = lane == 31 ? re : min(max((o1 + 3u) & ~3u, rs), re);
  *r0 = rs;
  *r1 = re;
  if (a1 > a0) {
    uint32_t skip = a0 - o;  // codes before the run (the previous run's last ones)
    uint32_t rem8 = 8u * (a1 - a0);
    uint32_t q = (gtid == 0 ? 0u : G.ends[gtid - 1]) - ws + q0;
    RunWriter out;
    out.init(G.exps, a0);
    // skip, then take the rest of the lookup that crosses into the run
    while (skip) {
      const uint32_t x = peek(q);
      const uint2 e = lds64(tab + 8 * lut_index(x));
      uint32_t k = e.y >> 27, nb = (e.y >> 20) & 15u, syms = e.x;  // k: up to four codes
      if (!k) {
        const uint32_t d = decode_long(T, x);
        if (!d) break;
        syms = d & 0xFFu;
        nb = d >> 8;
        k = 1;
      }
      q += nb;
      if (k <= skip) {
        skip -= k;
        continue;
      }
      const uint32_t take8 = min(8u * (k - skip), rem8);
      out.put((syms >> (8 * skip)) & ((take8 >= 32 ? 0u : 1u << take8) - 1u), take8);
      rem8 -= take8;
      skip = 0;
    }
    // bulk: two lookups per 32-bit peek while more than eight symbols remain
    while (rem8 > 64) {
      const uint32_t x = peek(q);
      const uint2 e1 = lds64(tab + 8 * lut_index(x));
      if (e1.y < (1u << 24)) {  // no complete code in the index bits
        const uint32_t d = decode_long(T, x);
        if (!d) break;
        out.put(d & 0xFFu, 8);
        rem8 -= 8;
        q += d >> 8;
        continue;
      }
      const uint32_t s1 = e1.y >> 20;  // bits of the first codes (low 4 bits) | 8 * their number << 4
      const uint2 e2 = lds64(tab + 8 * lut_index(__funnelshift_l(0u, x, s1)));
      const uint32_t s2 = e2.y >> 20;
      out.put(e1.x, s1 >> 4);
      out.put(e2.x, s2 >> 4);
      q += (s1 & 15u) + (s2 & 15u);
      rem8 -= (s1 >> 4) + (s2 >> 4);
    }
    // the run's last symbols, one lookup at a time
    while (rem8) {
      const uint32_t x = peek(q);
      const uint2 e = lds64(tab + 8 * lut_index(x));
      uint32_t k8 = e.y >> 24, nb = (e.y >> 20) & 15u, syms = e.x;
      if (!k8) {
        const uint32_t d = decode_long(T, x);
        if (!d) break;
        syms = d & 0xFFu;
        nb = d >> 8;
        k8 = 8;
      }
      if (k8 >= rem8) {
        out.put(syms & (rem8 >= 32 ? ~0u : (1u << rem8) - 1u), rem8);
        rem8 = 0;
        break;
      }
      out.put(syms, k8);
      rem8 -= k8;
      q += nb;
    }
    out.finish();
    if (rem8) *timeout |= 2u;  // an invalid code after the count accepted the chunk
  }
  __syncwarp();
  return true;
}

// Steps 2-5 with a value index: thread t writes values [128t, 128t + 128) of
// the chunk from the bit vidx[t] on; no boundary search, no count, no scan.
// The run must end exactly at the next entry (or the chunk's end); a thread
// whose run does not returns false.  *r0, *r1 receive the warp's region.
template <bool kSmem>
__device__ bool decode_chunk_indexed(GroupSmem &G, const DecodeTables &T, const uint32_t *words, uint32_t rel0,
                                     uint32_t nbits, uint32_t cnt, uint32_t gtid, const uint32_t *vidx,
                                     uint32_t per, uint32_t *r0, uint32_t *r1) {
  const uint32_t tab = (uint32_t)__cvta_generic_to_shared(&T.l1[0]);
  const uint32_t j0 = gtid * kIndexStride;
  const uint32_t wbase = (gtid & ~31u) * kIndexStride;
  *r0 = min(wbase, cnt);
  *r1 = min(wbase + 32 * kIndexStride, cnt);
  uint32_t start = 0, stop = 0, n = 0;
  bool bad = false;
  if (gtid < per && j0 < cnt) {
    n = min(kIndexStride, cnt - j0);
    start = __ldg(vidx + gtid);
    stop = (gtid + 1 < per && j0 + kIndexStride < cnt) ? __ldg(vidx + gtid + 1) : nbits;
    bad = start > stop || stop > nbits || stop - start < n || stop - start > 32u * n;
  }
  if (!bad && n) {
    Peek<kSmem> peek{words + ((rel0 + start) >> 5)};
    const uint32_t q0 = (rel0 + start) & 31u;
    uint32_t q = q0;
    const uint32_t qe = q0 + (stop - start);
    RunWriter out;  // runs start on multiples of 128 values: whole words
    out.init(G.exps, j0);
    uint32_t rem8 = 8 * n;
    while (rem8 > 64 && q < qe) {
      const uint32_t x = peek(q);
      const uint2 e1 = lds64(tab + 8 * lut_index(x));
      if (e1.y < (1u << 24)) {
        const uint32_t d = decode_long(T, x);
        if (!d) { bad = true; break; }
        out.put(d & 0xFFu, 8);
        rem8 -= 8;
        q += d >> 8;
        continue;
      }
      const uint32_t s1 = e1.y >> 20;
      const uint2 e2 = lds64(tab + 8 * lut_index(__funnelshift_l(0u, x, s1)));
      const uint32_t s2 = e2.y >> 20;
      out.put(e1.x, s1 >> 4);
      out.put(e2.x, s2 >> 4);
      q += (s1 & 15u) + (s2 & 15u);
      rem8 -= (s1 >> 4) + (s2 >> 4);
    }
    while (!bad && rem8 && q < qe) {
      const uint32_t x = peek(q);
      const uint2 e = lds64(tab + 8 * lut_index(x));
      uint32_t k8 = e.y >> 24, nb = (e.y >> 20) & 15u, syms = e.x;
      if (!k8) {
        const uint32_t d = decode_long(T, x);
        if (!d) { bad = true; break; }
        syms = d & 0xFFu;
        nb = d >> 8;
        k8 = 8;
      }
      if (k8 >= rem8) {
        // bits of the first rem8 / 8 codes: up to the start of the next one
        const uint32_t r = rem8 >> 3;
        if (r < (k8 >> 3)) {
          uint32_t bm = meta_starts(e.y);
          for (uint32_t i = 0; i < r; i++) bm &= bm - 1u;  // drop the first r code starts
          nb = __ffs(bm) - 1u;
        }
        out.put(syms & (rem8 >= 32 ? ~0u : (1u << rem8) - 1u), rem8);
        q += nb;
        rem8 = 0;
        break;
      }
      out.put(syms, k8);
      rem8 -= k8;
      q += nb;
    }
    out.finish();
    bad = bad || rem8 != 0 || q != qe;
  }
  return !__any_sync(0xffffffffu, bad);
}

// (sign+mantissa word, rotated exponent word) of four values -> four BF16
// values: bytes [sm, sign of sm] against [r, r] under the mask 0x807F807F.
__device__ __forceinline__ uint2 bf16_merge4(uint32_t smw, uint32_t ew) {
  constexpr uint32_t kM = 0x807F807Fu;
  const uint32_t x0 = prmt(smw, 0u, 0x9180u), r0 = prmt(ew, 0u, 0x1100u);
  const uint32_t x1 = prmt(smw, 0u, 0xB3A2u), r1 = prmt(ew, 0u, 0x3322u);
  return make_uint2((x0 & kM) | (r0 & ~kM), (x1 & kM) | (r1 & ~kM));
}

// four sign+mantissa nibbles (16 bits) and four exponent bytes -> 4 FP8 values
__device__ __forceinline__ uint32_t fp8_merge4(uint32_t nib16, uint32_t e4) {
  const uint32_t t = prmt(nib16 & 0x0F0Fu, (nib16 >> 4) & 0x0F0Fu, 0x5140u);  // one nibble per byte
  return ((t << 4) & 0x80808080u) | (t & 0x07070707u) | (e4 << 3);
}

template <int DT, bool kPlain>
__device__ __forceinline__ ChunkInfo chunk_info(const Batch &b, uint32_t g) {
  ChunkInfo ci;
  ci.item = find_item(b, g);
  const Item &I = b.item[ci.item];
  ci.c = I.first_chunk + (g - I.chunk0);
  ci.raw = 0;
  uint64_t B0, B1, Bt, i0;
  if (!kPlain && I.page_meta) {
    // page store: the page's codes start at bit 0 of its own slot
    const uint32_t slot = I.slot_ids[ci.c];
    ci.cnt = b.chunk_elems;
    const uint32_t meta = slot < I.n_slots ? I.page_meta[slot] : 0u;
    const uint64_t sm_page = DT == EH_BF16 ? b.chunk_elems : (DT == EH_FP8_E4M3 ? b.chunk_elems / 2 : 0);
    ci.sm_off = (uint64_t)slot * sm_page;
    ci.out_off = (uint64_t)ci.c * b.chunk_elems;
    if (slot < I.n_slots && (meta & EH_PAGE_RAW)) {
      const uint32_t idx = meta & ~EH_PAGE_RAW;
      ci.raw = idx + 1;
      ci.ok = idx < I.raw_cap;
      ci.nbits = 0;
      ci.lo = 0;
      ci.rel0 = 0;
      ci.fits = false;
      ci.bytes = 0;
      return ci;
    }
    B0 = (uint64_t)slot * I.slot_bytes * 8;
    B1 = B0 + meta;
    Bt = (uint64_t)I.n_slots * I.slot_bytes * 8;
    ci.ok = slot < I.n_slots && B1 - B0 >= ci.cnt && B1 - B0 <= (uint64_t)ci.cnt * 32u &&
            (B1 - B0 + 7) / 8 + 16 <= I.slot_bytes;
  } else {
    i0 = (uint64_t)ci.c * b.chunk_elems;
    ci.cnt = (uint32_t)min((uint64_t)b.chunk_elems, I.n - i0);
    ci.sm_off = DT == EH_BF16 ? i0 : (DT == EH_FP8_E4M3 ? i0 / 2 : 0);
    ci.out_off = i0 - I.elem0;
    B0 = I.off[ci.c];
    B1 = I.off[ci.c + 1];
    Bt = I.off[I.total_chunks];
    // the stream must hold every chunk's bits plus 16 readable bytes
    ci.ok = I.off[0] == 0 && B0 <= B1 && B1 <= Bt && (Bt + 7) / 8 + 16 <= I.stream_cap &&
            B1 - B0 >= ci.cnt && B1 - B0 <= (uint64_t)ci.cnt * 32u;
  }
  ci.nbits = (uint32_t)(B1 - B0);
  ci.lo = (B0 >> 3) & ~uint64_t(15);
  const uint64_t hi = (((B1 + 7) >> 3) + 16 + 15) & ~uint64_t(15);
  ci.rel0 = (uint32_t)(B0 - ci.lo * 8);
  ci.fits = ci.ok && hi - ci.lo <= (uint64_t)kGroupStage && hi <= I.stream_cap;
  ci.bytes = ci.fits ? (uint32_t)(hi - ci.lo) : 0u;
  return ci;
}

__device__ __forceinline__ void issue_stage(GroupSmem &G, const uint8_t *src, uint32_t bytes) {
  mbar_expect_tx(&G.mbar, bytes);
  bulk_g2s(G.stage, src, bytes, &G.mbar);
  G.issued++;
}

// 6. merge the exponents of values [r0, r1) of a chunk (r0 a multiple of 16)
// with their sign/mantissa bytes and store them: one warp, 16-byte stores.
// `exps` holds the exponents in output form; `raw` (page store) instead
// points at the plain exponent bytes of values [0, cnt) in global memory.
template <int DT, bool kRaw>
__device__ __forceinline__ void merge_region(const Item &I, const ChunkInfo &ci, const uint8_t *exps,
                                             const uint8_t *raw, uint32_t r0, uint32_t r1, uint32_t lane) {
  const uint32_t v0 = r0 / 16, v1 = r1 / 16;
  const uint32_t cnt = ci.cnt;
  auto exp_word4 = [&](uint32_t v) -> uint4 {
    if (!kRaw) {
      const uint32_t *p = (const uint32_t *)(exps + 16 * v + 4 * (v >> 3));  // padded rows
      return make_uint4(p[0], p[1], p[2], p[3]);
    }
    uint4 w = __ldg((const uint4 *)(raw + 16 * (uint64_t)v));
    if (DT == EH_BF16) {  // plain exponents -> output form
      w.x = ((w.x >> 1) & 0x7F7F7F7Fu) | ((w.x << 7) & 0x80808080u);
      w.y = ((w.y >> 1) & 0x7F7F7F7Fu) | ((w.y << 7) & 0x80808080u);
      w.z = ((w.z >> 1) & 0x7F7F7F7Fu) | ((w.z << 7) & 0x80808080u);
      w.w = ((w.w >> 1) & 0x7F7F7F7Fu) | ((w.w << 7) & 0x80808080u);
    }
    return w;
  };
  auto exp_byte = [&](uint32_t i) -> uint32_t {
    if (!kRaw) return exps[i + 4 * (i >> 7)];
    const uint32_t e = raw[i];
    return DT == EH_BF16 ? ((e >> 1) | ((e & 1u) << 7)) : e;
  };
  if (DT == EH_BF16) {
    const uint8_t *smp = I.sm + ci.sm_off;
    uint16_t *outp = (uint16_t *)I.out + ci.out_off;
    if (kRaw) {
      for (uint32_t v = v0 + lane; v < v1; v += 32) {
        const uint4 m = ld_nc16(smp + 16 * (uint64_t)v), e = exp_word4(v);
        const uint2 a = bf16_merge4(m.x, e.x), c = bf16_merge4(m.y, e.y);
        const uint2 d = bf16_merge4(m.z, e.z), f = bf16_merge4(m.w, e.w);
        uint4 *dst = (uint4 *)(outp + 16 * (uint64_t)v);
        dst[0] = make_uint4(a.x, a.y, c.x, c.y);
        dst[1] = make_uint4(d.x, d.y, f.x, f.y);
      }
    } else if (v0 + lane < v1) {
      // lane's vectors v0 + lane + 32k: constant strides for all three
      // pointers (in the padded exponent rows, 32 vectors are 528 bytes)
      const uint32_t vl = v0 + lane, K = (v1 - vl + 31) / 32;
      const uint4 *sp = (const uint4 *)smp + vl;
      uint4 *op = (uint4 *)outp + 2 * (uint64_t)vl;
      uint32_t ea = (uint32_t)__cvta_generic_to_shared(exps) + 16 * vl + 4 * (vl >> 3);
      uint32_t k = 0;
      for (; k + 1 < K; k += 2, sp += 64, op += 128, ea += 2 * 528) {
        const uint4 m0 = ld_nc16(sp), m1 = ld_nc16(sp + 32);
        const uint4 e0 = make_uint4(lds32(ea), lds32(ea + 4), lds32(ea + 8), lds32(ea + 12));
        const uint4 e1 = make_uint4(lds32(ea + 528), lds32(ea + 532), lds32(ea + 536), lds32(ea + 540));
        uint2 a = bf16_merge4(m0.x, e0.x), c = bf16_merge4(m0.y, e0.y);
        uint2 d = bf16_merge4(m0.z, e0.z), f = bf16_merge4(m0.w, e0.w);
        op[0] = make_uint4(a.x, a.y, c.x, c.y);
        op[1] = make_uint4(d.x, d.y, f.x, f.y);
        a = bf16_merge4(m1.x, e1.x);
        c = bf16_merge4(m1.y, e1.y);
        d = bf16_merge4(m1.z, e1.z);
        f = bf16_merge4(m1.w, e1.w);
        op[64] = make_uint4(a.x, a.y, c.x, c.y);
        op[65] = make_uint4(d.x, d.y, f.x, f.y);
      }
      if (k < K) {
        const uint4 m0 = ld_nc16(sp);
        const uint4 e0 = make_uint4(lds32(ea), lds32(ea + 4), lds32(ea + 8), lds32(ea + 12));
        const uint2 a = bf16_merge4(m0.x, e0.x), c = bf16_merge4(m0.y, e0.y);
        const uint2 d = bf16_merge4(m0.z, e0.z), f = bf16_merge4(m0.w, e0.w);
        op[0] = make_uint4(a.x, a.y, c.x, c.y);
        op[1] = make_uint4(d.x, d.y, f.x, f.y);
      }
    }
    if (r1 == cnt)
      for (uint32_t i = max(v1 * 16, r0) + lane; i < cnt; i += 32) {
        const uint32_t sm = smp[i], r = exp_byte(i);
        outp[i] = (uint16_t)(((sm & 0x80u) << 8) | ((r & 0x7Fu) << 8) | (r & 0x80u) | (sm & 0x7Fu));
      }
  } else if (DT == EH_BYTES) {
    // the decoded symbols are the output bytes
    uint8_t *outp = (uint8_t *)I.out + ci.out_off;
    for (uint32_t v = v0 + lane; v < v1; v += 32) *(uint4 *)(outp + 16 * (uint64_t)v) = exp_word4(v);
    if (r1 == cnt)
      for (uint32_t i = max(v1 * 16, r0) + lane; i < cnt; i += 32) outp[i] = (uint8_t)exp_byte(i);
  } else {
    const uint8_t *smp = I.sm + ci.sm_off;
    uint8_t *outp = (uint8_t *)I.out + ci.out_off;
    for (uint32_t b0 = v0 + lane; b0 < v1; b0 += 4 * 32) {
      uint2 m[4];
      #pragma unroll
      for (int u = 0; u < 4; u++) {
        const uint32_t v = b0 + u * 32;
        m[u] = v < v1 ? ld_nc8(smp + 8 * (uint64_t)v) : make_uint2(0, 0);
      }
      #pragma unroll
      for (int u = 0; u < 4; u++) {
        const uint32_t v = b0 + u * 32;
        if (v < v1) {
          const uint4 e = exp_word4(v);
          uint4 o;
          o.x = fp8_merge4(m[u].x & 0xFFFFu, e.x);
          o.y = fp8_merge4(m[u].x >> 16, e.y);
          o.z = fp8_merge4(m[u].y & 0xFFFFu, e.z);
          o.w = fp8_merge4(m[u].y >> 16, e.w);
          *(uint4 *)(outp + 16 * (uint64_t)v) = o;
        }
      }
    }
    if (r1 == cnt)
      for (uint32_t i = max(v1 * 16, r0) + lane; i < cnt; i += 32) {
        const uint32_t sm = (smp[i / 2] >> (4 * (i & 1))) & 0xFu, e = exp_byte(i);
        outp[i] = (uint8_t)(((sm & 8u) << 4) | (e << 3) | (sm & 7u));
      }
  }
}

// Persistent: CTA i of G decodes the contiguous chunk range
// [i*C/G, (i+1)*C/G), split into runs of one tensor (one codebook); inside a
// run the two groups take alternate chunks.  The last warp of a group to
// finish writing a chunk's exponents (and so reading its stage) starts the
// copy of the group's next chunk; every warp then merges its own region.
// kPlain: no tensor of the call is a page store or has a value index (a
// separate kernel, so that the common case carries none of their code).
template <int DT, bool kPlain>
__global__ void __launch_bounds__(kDecThreads, 1) decode_kernel(const __grid_constant__ Batch b) {
  extern __shared__ __align__(128) uint8_t smem_raw[];
  DecodeSmem &S = *reinterpret_cast<DecodeSmem *>(smem_raw);
  const uint32_t tid = threadIdx.x;
  const uint32_t grp = tid / kGroupThreads, gtid = tid % kGroupThreads, id = 1 + grp;
  const uint32_t lane = gtid & 31u;
  GroupSmem &G = S.grp[grp];
  const uint32_t g0 = (uint32_t)(((uint64_t)b.total_chunks * blockIdx.x) / gridDim.x);
  const uint32_t g1 = (uint32_t)(((uint64_t)b.total_chunks * (blockIdx.x + 1)) / gridDim.x);
  if (g0 >= g1) return;
  if (gtid == 0) {
    mbar_init(&G.mbar, 1);
    G.writers_done = 0;
    G.issued = 0;
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
  }
  if (tid == 0) S.abort_flag = 0;
  pdl_wait();  // the decode tables (and everything before them)
  __syncthreads();
  uint32_t parity = 0, timeout = 0, landed = 0;  // landed: stage copies of this group waited for
  const uint32_t max_rounds = b.fixup_rounds ? b.fixup_rounds : kGroupThreads + 3;

  for (uint32_t seg = g0; seg < g1;) {
    const Item &I = b.item[find_item(b, seg)];
    const uint32_t seg_end = min(g1, I.chunk0 + I.nchunks);
    __syncthreads();  // both groups are done with the previous tables and stages
    // the first chunk's stage copy runs while the tables are copied
    uint32_t g = seg + grp;
    ChunkInfo ci;
    ci.fits = false;
    if (g < seg_end) {
      ci = chunk_info<DT, kPlain>(b, g);
      if (ci.fits && gtid == 0) issue_stage(G, b.item[ci.item].stream + ci.lo, ci.bytes);
    }
    {
      const uint4 *src = (const uint4 *)I.lut;
      uint4 *dst = (uint4 *)&S.tabs;
      for (uint32_t i = tid; i < sizeof(DecodeTables) / 16; i += kDecThreads) dst[i] = src[i];
    }
    __syncthreads();
    const bool terr = S.tabs.err != 0;
    // Stagger the groups by one decode: group 1 starts its first chunk when
    // group 0 has decoded its own and turns to the memory-bound output, so
    // one group's output overlaps the other's decode instead of coinciding.
    // With only two chunks there is nothing to overlap afterwards, and both
    // groups start at once.
    const bool stagger = seg_end - seg >= 3;
    if (stagger && grp == 1) named_sync(kStaggerBarrier, kDecThreads);
    for (uint32_t j = 0; g < seg_end; g += kNumGroups, j ^= 1u) {
      // The group's next chunk is described once, by its first thread, in
      // the entry of this chunk's parity: every thread reads it at the start
      // of the next chunk, and the last writer of this chunk starts its stage
      // copy from it.  (The entry of the other parity may still be read by
      // the last writer of the previous chunk.)
      if (g != seg + grp) ci = G.next[j ^ 1u];
      const uint32_t cnt = ci.cnt;
      bool ok = ci.ok && !terr && !S.abort_flag;
      if (gtid == 0) {
        const uint32_t gn = g + kNumGroups;
        if (gn < seg_end) G.next[j] = chunk_info<DT, kPlain>(b, gn);
        else G.next[j].fits = false;
      }

      // Every thread waits for the chunk's stage copy itself.  The plain
      // decode's first barrier tells the group whether a copy came late;
      // every other path takes one barrier here, so that the warps of a
      // group never drift more than a chunk apart, and a chunk read from
      // global memory (no copy to wait for) cannot overwrite the end bits
      // that a slow warp of the previous chunk still reads.
      const uint32_t *vidx = (!kPlain && ok && I.vindex && !I.page_meta)
                                 ? I.vindex + (uint64_t)ci.c * (b.chunk_elems / kIndexStride)
                                 : nullptr;
      bool late = false;
      if (ci.fits) {
        late = !mbar_wait_bounded(&G.mbar, parity);
        if (!late) {
          parity ^= 1u;
          landed++;
        }
      }
      const bool raw_page = !kPlain && ci.raw;
      if (!ok || raw_page || vidx || !ci.fits) {
        if (gsync_or(id, late)) {
          if (gtid == 0) {
            set_status(b.status, kFlagTimeout);
            S.abort_flag = 1;
          }
          ok = false;
        }
      }
      uint32_t r0 = 0, r1 = 0;  // this warp's region of the chunk's values
      const uint8_t *raw = nullptr;
      if (ok && raw_page) {
        // page stored raw: the merge reads its exponent bytes from the pool
        raw = I.raw_pool + (uint64_t)(ci.raw - 1) * b.chunk_elems;
        const uint32_t per_warp = (cnt + kGroupWarps * 16 - 1) / (kGroupWarps * 16) * 16;
        r0 = min((gtid >> 5) * per_warp, cnt);
        r1 = min(r0 + per_warp, cnt);
      } else if (ok) {
        const uint32_t per = b.chunk_elems / kIndexStride;
        const uint32_t *gw = (const uint32_t *)(I.stream + ci.lo);
        if (!kPlain && vidx) {
          const bool wok = ci.fits ? decode_chunk_indexed<true>(G, S.tabs, G.stage, ci.rel0, ci.nbits, cnt, gtid,
                                                                vidx, per, &r0, &r1)
                                   : decode_chunk_indexed<false>(G, S.tabs, gw, ci.rel0, ci.nbits, cnt, gtid,
                                                                 vidx, per, &r0, &r1);
          if (!wok) {
            if (lane == 0) set_status(b.status, kFlagCorrupt);
            r1 = r0;  // nothing of this warp's region is written out
          }
        } else {
          ok = ci.fits ? decode_chunk<true>(G, S.tabs, G.stage, ci.rel0, ci.nbits, cnt, id, gtid, &timeout, &r0, &r1, late, max_rounds)
                       : decode_chunk<false>(G, S.tabs, gw, ci.rel0, ci.nbits, cnt, id, gtid, &timeout, &r0, &r1, late, max_rounds);
          if (!ok && gtid == 0) set_status(b.status, (timeout & 1u) ? kFlagTimeout | kFlagCorrupt : kFlagCorrupt);
          if (timeout & 2u) set_status(b.status, kFlagCorrupt);
        }
      } else if (gtid == 0 && !S.abort_flag) {
        set_status(b.status, kFlagCorrupt);
      }

      if (stagger && grp == 0 && g == seg) named_arrive(kStaggerBarrier, kDecThreads);
      // The stage is free once every warp of the group has written its runs:
      // the last one starts copying the group's next chunk.  (The generic
      // writes of the byte swap were fenced before the chunk's barrier.)
      __syncwarp();
      if (lane == 0) {
        __threadfence_block();
        if (atomicAdd(&G.writers_done, 1u) == kGroupWarps - 1) {
          G.writers_done = 0;
          const ChunkInfo &cn = G.next[j];
          if (cn.fits) issue_stage(G, b.item[cn.item].stream + cn.lo, cn.bytes);
        }
      }

      // 6. merge this warp's region with the sign/mantissa bytes
      if (ok && r1 > r0) {
        if (!kPlain && raw) merge_region<DT, true>(I, ci, G.exps, raw, r0, r1, lane);
        else merge_region<DT, false>(I, ci, G.exps, raw, r0, r1, lane);
      }
      // no barrier here: the next chunk's barriers order these reads of the
      // exponent buffer before it is written again
    }
    seg = seg_end;
  }
  // a copy still in flight (only after an abort) must land before the exit
  __syncthreads();
  if (gtid == 0 && G.issued != landed) mbar_wait_bounded(&G.mbar, parity);
  __syncthreads();
}

}  // namespace

cudaError_t launch_tables(const Batch &b, cudaStream_t s) {
  return launch_pdl(tables_kernel, dim3(b.k * kTabParts), dim3(256), 0, s, b);
}

cudaError_t launch_decode(const Batch &b, cudaStream_t s, int num_sms) {
  if (b.total_chunks == 0) return cudaSuccess;
  const size_t smem = sizeof(DecodeSmem) + 128;
  uint32_t grid = (uint32_t)num_sms;
  if (grid > b.total_chunks) grid = b.total_chunks;
  bool plain = true;
  for (uint32_t i = 0; i < b.k; i++) plain &= !b.item[i].page_meta && !b.item[i].vindex;
  const dim3 g(grid), t(kDecThreads);
  if (plain) {
    if (b.dtype == EH_BF16) return launch_pdl(decode_kernel<EH_BF16, true>, g, t, smem, s, b);
    if (b.dtype == EH_BYTES) return launch_pdl(decode_kernel<EH_BYTES, true>, g, t, smem, s, b);
    return launch_pdl(decode_kernel<EH_FP8_E4M3, true>, g, t, smem, s, b);
  }
  if (b.dtype == EH_BF16) return launch_pdl(decode_kernel<EH_BF16, false>, g, t, smem, s, b);
  if (b.dtype == EH_BYTES) return launch_pdl(decode_kernel<EH_BYTES, false>, g, t, smem, s, b);
  return launch_pdl(decode_kernel<EH_FP8_E4M3, false>, g, t, smem, s, b);
}

cudaError_t configure_decode() {
  const int smem = (int)(sizeof(DecodeSmem) + 128);
  const void *kernels[] = {(const void *)decode_kernel<EH_BF16, true>, (const void *)decode_kernel<EH_BYTES, true>,
                           (const void *)decode_kernel<EH_FP8_E4M3, true>, (const void *)decode_kernel<EH_BF16, false>,
                           (const void *)decode_kernel<EH_BYTES, false>, (const void *)decode_kernel<EH_FP8_E4M3, false>};
  cudaError_t e = cudaSuccess;
  for (const void *k : kernels)
    if (e == cudaSuccess) e = cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
  return e;
}

}  // namespace eh

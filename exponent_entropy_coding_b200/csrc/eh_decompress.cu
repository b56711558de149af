// eh_decompress.cu -- decompression kernels of libexphuff (sm_100a).
//
//   tables  eight CTAs per codebook: validate the code lengths and codes and
//           build the decode tables (a 12-bit first level giving, for the
//           index bits, the symbols of up to four complete codes, their bits,
//           and the number, bits and start offsets of all complete codes;
//           8-bit second-level tables for codes of 13..20 bits; canonical
//           limits for anything longer);
//   decode  persistent CTAs of two independent groups, one chunk per group
//           at a time:
//             1. the chunk's bit range is copied into shared memory with one
//                bulk asynchronous copy (cp.async.bulk + mbarrier) when it
//                fits, else read from global memory;
//             2. every thread counts the codes of its own window of the
//                chunk's bits, starting speculatively at the window start and
//                recording the code boundaries of its first 64 bits;
//             3. fix-up rounds: each thread restarts from the true end of its
//                predecessor and stops as soon as it lands on one of its
//                recorded boundaries (Huffman codes resynchronise after a few
//                codes), until no end moves;
//             4. group-wide exclusive scan of the per-thread code counts
//                gives every thread its first output index;
//             5. the threads decode again from their true starts and write
//                their exponents to shared memory;
//             6. coalesced pass: exponents merged with the sign/mantissa
//                stream and stored with 16-byte stores.
// The DFloat11 article ("方法介绍") describes compact LUTs sized for on-chip
// SRAM, a two-phase kernel coordinating where each thread reads and writes,
// and block-level decompression; here the per-thread start positions are not
// stored in the format but recovered by the self-synchronising fix-up.
#include "eh_internal.cuh"

namespace eh {
namespace {

constexpr uint32_t kMaskBits = 64;            // code starts recorded per thread
constexpr uint32_t kSpinLimit = 1u << 26;     // bounded mbarrier wait

// ---------------------------------------------------------------- tables
// kTabParts CTAs of 256 threads per codebook; each builds 1/kTabParts of the
// first level, part 0 also writes the second levels and the limits.
constexpr uint32_t kTabParts = 8;

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
  if (part == 0) T->sorted[tid] = tid < (int)nsym ? srt[tid] : (uint8_t)0;

  // first level.  Codes longer than kLutBits fill the left-justified range
  // [lim[kLutBits], lim[32]), so their prefixes are consecutive: the first
  // kNumSub of them get a second-level table.
  constexpr uint32_t kShift = 32 - kLutBits;
  const uint32_t sub0 = (uint32_t)(limL[kLutBits] >> kShift);
  constexpr uint32_t kPerPart = (1u << kLutBits) / kTabParts;
  for (uint32_t p = part * kPerPart + tid; p < (part + 1) * kPerPart; p += 256) {
    // every complete code inside the index bits: all of them for counting,
    // the first four (their symbols fill 32 bits) for writing
    uint32_t syms = 0, pos = 0, nc = 0, bnd = 0, pos4 = 0, nc4 = 0;
    while (pos < (uint32_t)kLutBits) {
      const uint32_t x = (p << kShift) << pos;  // next bits, left-justified, zero-filled
      const uint32_t L = code_length_of(x, limL);
      if (L > (uint32_t)kLutBits - pos) break;  // not complete inside the index bits
      if (nc < 4) {
        const uint32_t v = x >> (32 - L);
        syms |= (uint32_t)srt[baseL[L] + v - firstL[L]] << (8 * nc);
        pos4 = pos + L;
        nc4 = nc + 1;
      }
      bnd |= 1u << pos;
      pos += L;
      nc++;
    }
    uint32_t sub = kNoSub;
    if (nc == 0 && ((uint64_t)p << kShift) < limL[32] && p - sub0 < (uint32_t)kNumSub) sub = p - sub0;
    T->l1sym[p] = syms;
    T->l1meta[p] = pos4 | (nc4 << 4) | (bnd << 7) | (sub << 19) | (pos << 24) | (nc << 28);
  }
  if (part != 0) return;
  // second level: codes of kLutBits+1 .. kLutBits+8 bits
  for (uint32_t j = 0; j < (uint32_t)kNumSub; j++) {
    uint32_t e = 0;
    const uint32_t p = sub0 + j;
    if (((uint64_t)p << kShift) < limL[32]) {
      const uint32_t x = (p << kShift) | ((uint32_t)tid << (kShift - 8));
      for (uint32_t L = kLutBits + 1; L <= (uint32_t)kLutBits + 8; L++) {
        if ((uint64_t)x < limL[L]) {
          if (x >= (uint32_t)(limL[L - 1])) {
            const uint32_t v = x >> (32 - L);
            e = (uint32_t)srt[baseL[L] + v - firstL[L]] | (L << 8);
          }
          break;
        }
      }
    }
    T->sub[j][tid] = e;
  }
  if (tid == 0) T->err = err;
}

// ---------------------------------------------------------------- decode
// Exponent j of a chunk is kept at byte j + 4*(j/128) of the exponent buffer:
// every 128-byte row is followed by 4 pad bytes, so threads whose outputs
// start about 128 values apart write to different shared-memory banks.
constexpr uint32_t kExpBytes = kMaxChunk + 4 * (kMaxChunk / 128);
__device__ __forceinline__ uint32_t exp_slot(uint32_t j) { return j + ((j >> 7) << 2); }

// 32 stream bits starting at bit p.  Shared-memory stages are byte-swapped
// once after the copy, so their words are already MSB-first; global words are
// swapped on load.
template <bool kSmem>
struct Peek {
  const uint32_t *w;
  __device__ __forceinline__ uint32_t word(uint32_t i) const { return kSmem ? w[i] : bswap32(__ldg(w + i)); }
  __device__ __forceinline__ uint32_t operator()(uint32_t p) const {
    const uint32_t i = p >> 5;
    return __funnelshift_l(word(i + 1), word(i), p & 31);
  }
};

__device__ __forceinline__ uint32_t lut_index(uint32_t x) { return x >> (32 - kLutBits); }

// Code longer than the first-level index: second-level table, else search of
// the canonical limits.  Returns 1 and the symbol and length, or 0 for an
// invalid code.
__device__ __forceinline__ uint32_t decode_long(const DecodeTables &T, uint32_t peek, uint32_t meta,
                                                uint32_t &syms, uint32_t &nbits) {
  const uint32_t si = (meta >> 19) & 31u;
  if (si != kNoSub) {
    const uint32_t e2 = T.sub[si][(peek >> (24 - kLutBits)) & 0xFFu];
    const uint32_t l = (e2 >> 8) & 63u;
    if (l) {
      nbits = l;
      syms = e2 & 0xFFu;
      return 1;
    }
  }
  uint32_t L = kLutBits + 1;
  #pragma unroll 1
  while (L <= 32 && (uint64_t)peek >= T.lim[L]) L++;
  if (L > 32) return 0;
  const uint32_t v = L == 32 ? peek : peek >> (32 - L);
  syms = T.sorted[T.base[L] + (v - T.first[L])];
  nbits = L;
  return 1;
}

// One decode step on the next 32 bits `x`, taking only codes that start in
// the next `lim` (>= 1) bits.  Returns the number of codes taken (0: invalid
// code); their symbols (8 bits each, first in the low byte) when kSyms, the
// bits up to the end of the last code taken, and the code starts as a bitmap.
template <bool kSyms>
__device__ __forceinline__ uint32_t decode_step(const DecodeTables &T, uint32_t x, uint32_t lim,
                                                uint32_t &syms, uint32_t &nbits, uint32_t &bnd) {
  const uint32_t idx = lut_index(x);
  const uint32_t meta = T.l1meta[idx];
  // writing takes the first four codes (their symbols), counting all of them
  uint32_t k = kSyms ? (meta >> 4) & 7u : meta >> 28;
  if (k) {
    uint32_t nb = kSyms ? meta & 15u : (meta >> 24) & 15u;
    uint32_t bm = (meta >> 7) & 0xFFFu;
    if (kSyms) bm &= (1u << nb) - 1u;
    uint32_t sy = kSyms ? T.l1sym[idx] : 0u;
    if (nb > lim) {
      // codes starting at or after the limit belong to the next window
      const uint32_t keep = bm & ((1u << lim) - 1u);
      const uint32_t rest = bm >> lim;
      k = __popc(keep);
      nb = rest ? lim + __ffs(rest) - 1 : nb;
      bm = keep;
      if (kSyms && k < 4) sy &= (1u << (8 * k)) - 1u;
    }
    nbits = nb;
    bnd = bm;
    syms = sy;
    return k;
  }
  bnd = 1u;
  return decode_long(T, x, meta, syms, nbits);
}

// The decoding CTA holds two independent groups of kGroupThreads threads.
// Each group decodes its own chunk into its own exponent buffer, so one
// group's memory-bound output pass overlaps the other's decode; the decode
// tables are shared.
constexpr uint32_t kGroupThreads = 512;
constexpr uint32_t kNumGroups = kDecThreads / kGroupThreads;
constexpr uint32_t kGroupStage = 27136;  // bytes of stream staged per group

struct GroupSmem {
  alignas(128) uint32_t stage[kGroupStage / 4 + 16];  // bulk-copy target (stream bytes as stored)
  alignas(16) uint8_t exps[kExpBytes];                // decoded exponents of one chunk (padded rows)
  uint32_t ends[kGroupThreads];
  uint32_t wsum[kGroupThreads / 32];
  alignas(8) unsigned long long mbar;
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

// Named barrier shared by both groups (ids 1 and 2 are the groups' own).
constexpr uint32_t kStaggerBarrier = 3;
__device__ __forceinline__ void named_sync(uint32_t id, uint32_t n) {
  asm volatile("bar.sync %0, %1;" ::"r"(id), "r"(n) : "memory");
}
__device__ __forceinline__ void named_arrive(uint32_t id, uint32_t n) {
  asm volatile("bar.arrive %0, %1;" ::"r"(id), "r"(n) : "memory");
}

// Barriers of one group: named barrier `id` over kGroupThreads threads.
__device__ __forceinline__ void gsync(uint32_t id) {
  asm volatile("bar.sync %0, %1;" ::"r"(id), "n"(kGroupThreads) : "memory");
}
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
// over the group (*any).  Every warp reduces the warp totals itself.
__device__ __forceinline__ uint32_t group_excl_scan_or(uint32_t v, bool pred, uint32_t *wsum, uint32_t *total,
                                                       bool *any, uint32_t id, uint32_t gtid) {
  constexpr uint32_t kWarps = kGroupThreads / 32;
  const uint32_t lane = gtid & 31u, warp = gtid >> 5;
  uint32_t x = v;
  #pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const uint32_t y = __shfl_up_sync(0xffffffffu, x, o);
    if (lane >= (uint32_t)o) x += y;
  }
  if (lane == 31) wsum[warp] = x;
  *any = gsync_or(id, pred);
  const uint32_t t = lane < kWarps ? wsum[lane] : 0u;
  uint32_t pre = lane < warp ? t : 0u, all = t;
  #pragma unroll
  for (int o = 16; o; o >>= 1) {
    pre += __shfl_xor_sync(0xffffffffu, pre, o);
    all += __shfl_xor_sync(0xffffffffu, all, o);
  }
  *total = all;
  return pre + x - v;
}

// Packs decoded exponents four to a word into the exponent buffer, which
// is zeroed before each chunk.  Words are combined with OR, so the words a run
// shares with its neighbours need no special case.
template <bool kOwn = false>
struct ExpWriter {
  uint32_t *words;  // exponent buffer as words
  uint32_t wi;      // word being filled (exponents 4*wi .. 4*wi+3)
  uint32_t s;       // bits of that word filled so far (those below the run are zero)
  uint32_t acc;
  __device__ __forceinline__ void init(uint8_t *e, uint32_t j) {
    words = (uint32_t *)e;
    wi = j >> 2;
    s = 8 * (j & 3u);
    acc = 0;
  }
  // kOwn: the run owns every word it touches (it starts on a word), so the
  // words are stored, not OR-ed into a cleared buffer
  __device__ __forceinline__ void store(uint32_t v) {
    if (kOwn) words[wi + (wi >> 5)] = v;  // word wi of the padded rows
    else atomicOr(words + wi + (wi >> 5), v);
  }
  // up to four symbols, first in the low byte, zero above; k8 = 8 * count
  __device__ __forceinline__ void put(uint32_t syms, uint32_t k8) {
    const uint32_t lo = acc | (syms << s);
    const uint32_t hi = __funnelshift_l(syms, 0u, s);  // the bytes past the word; none for s = 0
    s += k8;
    if (s >= 32) {
      store(lo);
      wi++;
      acc = hi;
      s -= 32;
    } else {
      acc = lo;
    }
  }
  __device__ __forceinline__ void finish() {
    if (s) store(acc);
  }
};

// the low r8 / 8 bytes of a word (r8 a multiple of 8, at most 32)
__device__ __forceinline__ uint32_t low_bytes_mask(uint32_t r8) { return r8 >= 32 ? ~0u : (1u << r8) - 1u; }

// Steps 2-5 for one chunk whose bits are [rel0, rel0 + nbits) of `words`,
// decoded by one group.  Returns false (group-uniform) if the chunk is
// corrupt.
template <bool kSmem>
__device__ bool decode_chunk(GroupSmem &G, const DecodeTables &T, const uint32_t *words, uint32_t rel0,
                             uint32_t nbits, uint32_t cnt, uint32_t id, uint32_t gtid, uint32_t *timeout) {
  // window width: a multiple of the gcd of the code lengths, so that a
  // fixed-length code starts every window on a code boundary
  const uint32_t gq = T.gcd;
  uint32_t W = (nbits + kGroupThreads - 1) / kGroupThreads;
  W = (W + gq - 1) / gq * gq;
  const uint32_t ws = min(gtid * W, nbits), we = min(ws + W, nbits);
  Peek<kSmem> peek{words};
  // Bulk decoding runs while 2 * kLutBits bits of the window remain: two
  // first-level lookups per 32-bit peek, no window-end handling.
  constexpr uint32_t kBulk = 2 * kLutBits;

  // 2. speculative decode of the own window; record where codes start in
  //    its first kMaskBits bits
  uint32_t pos = ws, n = 0;
  uint64_t mask = 0;
  bool bad = false;
  // (a) while the recorded bits last
  while (pos + kBulk <= we && pos - ws < kMaskBits) {
    const uint32_t x = peek(rel0 + pos);
    const uint32_t off = pos - ws;
    const uint32_t m1 = T.l1meta[lut_index(x)];
    const uint32_t k1 = m1 >> 28, nb1 = (m1 >> 24) & 15u;
    if (!k1) {
      uint32_t syms, nb;
      if (!decode_long(T, x, m1, syms, nb)) { bad = true; break; }
      mask |= 1ull << off;
      pos += nb;
      n += 1;
      continue;
    }
    // a prefix with no complete code has count, bits and starts all zero
    const uint32_t m2 = T.l1meta[lut_index(x << nb1)];
    mask |= (uint64_t)((m1 >> 7) & 0xFFFu) << off;
    if (off + nb1 < kMaskBits) mask |= (uint64_t)((m2 >> 7) & 0xFFFu) << (off + nb1);
    pos += nb1 + ((m2 >> 24) & 15u);
    n += k1 + (m2 >> 28);
  }
  // (b) the rest of the window, counting only
  while (!bad && pos + kBulk <= we) {
    const uint32_t x = peek(rel0 + pos);
    const uint32_t m1 = T.l1meta[lut_index(x)];
    const uint32_t k1 = m1 >> 28, nb1 = (m1 >> 24) & 15u;
    if (!k1) {
      uint32_t syms, nb;
      if (!decode_long(T, x, m1, syms, nb)) { bad = true; break; }
      pos += nb;
      n += 1;
      continue;
    }
    const uint32_t m2 = T.l1meta[lut_index(x << nb1)];
    pos += nb1 + ((m2 >> 24) & 15u);
    n += k1 + (m2 >> 28);
  }
  // (c) the window's last bits, taking only codes that start inside it
  while (!bad && pos < we) {
    uint32_t syms, nb, bnd;
    const uint32_t k = decode_step<false>(T, peek(rel0 + pos), we - pos, syms, nb, bnd);
    if (!k) { bad = true; break; }
    const uint32_t off = pos - ws;
    if (off < kMaskBits) mask |= (uint64_t)bnd << off;
    pos += nb;
    n += k;
  }
  const uint32_t spec_end = bad ? we : pos, spec_n = n;
  const uint64_t spec_mask = bad ? 0ull : mask;
  uint32_t my_start = ws, my_end = spec_end, my_n = spec_n;
  G.ends[gtid] = my_end;
  gsync(id);

  // 3. fix-up rounds: restart from the predecessor's end until a code starts
  //    where a speculative one did (from there on the speculative decode is
  //    right)
  for (uint32_t round = 0;; round++) {
    const uint32_t pred = gtid == 0 ? 0u : G.ends[gtid - 1];
    bool changed = false;
    if (gtid > 0 && pred != my_start) {
      my_start = pred;
      uint32_t p = pred, k = 0;
      bool synced = false, bad2 = false;
      while (p < we) {
        uint32_t syms, nb, bnd;
        const uint32_t kk = decode_step<false>(T, peek(rel0 + p), we - p, syms, nb, bnd);
        if (!kk) { bad2 = true; break; }
        const uint32_t off = p - ws;
        if (off < kMaskBits) {
          const uint64_t common = ((uint64_t)bnd << off) & spec_mask;
          if (common) {
            const uint32_t q = __ffsll(common) - 1;  // offset from ws, >= off
            k += __popc(bnd & ((1u << (q - off)) - 1u));
            p = ws + q;
            synced = true;
            break;
          }
        }
        p += nb;
        k += kk;
      }
      uint32_t new_end;
      if (synced) {
        my_n = k + spec_n - __popcll(spec_mask & ((1ull << (p - ws)) - 1ull));
        new_end = spec_end;
        bad = false;
      } else {
        my_n = k;
        new_end = bad2 ? we : p;
        bad = bad2;
      }
      changed = new_end != my_end;
      my_end = new_end;
    }
    // A successor may read this end in the same round, before or after the
    // store: an older end only costs it another round, and a round in which
    // no end moved (seen by everyone after the barrier) ends the fix-up.
    if (changed) G.ends[gtid] = my_end;
    if (!gsync_or(id, changed)) break;
    if (round > kGroupThreads + 1) {  // cannot happen for consistent data
      if (gtid == 0) *timeout = 1;
      bad = true;
      break;
    }
  }

  // 4. output index of every thread's first code
  uint32_t total;
  bool anybad;
  const uint32_t o = group_excl_scan_or(my_n, bad, G.wsum, &total, &anybad, id, gtid);
  const bool ok = !anybad && total == cnt && G.ends[kGroupThreads - 1] == nbits;
  if (!ok) return false;

  // 5. decode again from the true start, writing exactly the thread's my_n
  //    exponents (a count, not the window end, stops the loop)
  ExpWriter<> out;
  out.init(G.exps, o);
  pos = gtid == 0 ? 0u : G.ends[gtid - 1];
  uint32_t rem8 = 8 * my_n;  // exponent bits still to write
  while (rem8) {
    const uint32_t x = peek(rel0 + pos);
    const uint32_t i1 = lut_index(x);
    const uint32_t m1 = T.l1meta[i1];
    const uint32_t k1 = (m1 >> 1) & 0x38u, nb1 = m1 & 15u;  // k1: 8 * codes
    if (!k1) {
      uint32_t syms, nb;
      if (!decode_long(T, x, m1, syms, nb)) break;
      pos += nb;
      out.put(syms, 8);
      rem8 -= 8;
      continue;
    }
    const uint32_t s1 = T.l1sym[i1];
    if (k1 >= rem8) {  // the last codes of the thread
      out.put(s1 & low_bytes_mask(rem8), rem8);
      break;
    }
    out.put(s1, k1);
    rem8 -= k1;
    const uint32_t i2 = lut_index(x << nb1);
    const uint32_t m2 = T.l1meta[i2];
    const uint32_t k2 = (m2 >> 1) & 0x38u, nb2 = m2 & 15u;
    if (!k2) {
      pos += nb1;
      continue;
    }
    const uint32_t s2 = T.l1sym[i2];
    if (k2 >= rem8) {
      out.put(s2 & low_bytes_mask(rem8), rem8);
      break;
    }
    out.put(s2, k2);
    rem8 -= k2;
    pos += nb1 + nb2;
  }
  out.finish();
  gsync(id);
  return true;
}

// Bits taken by the first r (1..4) of the codes that start at the set bits
// of bm (offsets from the lookup position), when the lookup holds kk >= r
// complete codes ending at bit nb.
__device__ __forceinline__ uint32_t bits_of_first(uint32_t bm, uint32_t r, uint32_t kk, uint32_t nb) {
  if (r >= kk) return nb;
  #pragma unroll
  for (int i = 0; i < 4; i++)
    if ((uint32_t)i < r) bm &= bm - 1u;  // drop the first r code starts
  return __ffs(bm) - 1u;                  // the start of code r + 1
}

// Steps 2-5 with a value index: thread t writes values [128t, 128t + 128) of
// the chunk from the bit vidx[t] on; no boundary search, no count, no scan.
// The run must end exactly at the next entry (or the chunk's end), else the
// chunk is reported corrupt.  Returns false (group-uniform) if corrupt.
template <bool kSmem>
__device__ bool decode_chunk_indexed(GroupSmem &G, const DecodeTables &T, const uint32_t *words, uint32_t rel0,
                                     uint32_t nbits, uint32_t cnt, uint32_t id, uint32_t gtid,
                                     const uint32_t *vidx, uint32_t per) {
  Peek<kSmem> peek{words};
  const uint32_t j0 = gtid * kIndexStride;
  uint32_t start = 0, stop = 0, n = 0;
  bool bad = false;
  if (gtid < per && j0 < cnt) {
    n = min(kIndexStride, cnt - j0);
    start = __ldg(vidx + gtid);
    stop = (gtid + 1 < per && j0 + kIndexStride < cnt) ? __ldg(vidx + gtid + 1) : nbits;
    bad = start > stop || stop > nbits || stop - start < n || stop - start > 32u * n;
  }
  // also orders the caller's clearing of the exponent buffer before the writes
  if (gsync_or(id, bad)) return false;

  ExpWriter<true> out;  // runs start on multiples of 128 values: whole words
  out.init(G.exps, j0);
  uint32_t pos = start, rem8 = 8 * n;
  while (rem8 && pos < stop) {
    const uint32_t x = peek(rel0 + pos);
    const uint32_t i1 = lut_index(x);
    const uint32_t m1 = T.l1meta[i1];
    const uint32_t k1 = (m1 >> 1) & 0x38u, nb1 = m1 & 15u;  // k1: 8 * codes
    if (!k1) {
      uint32_t syms, nb;
      if (!decode_long(T, x, m1, syms, nb)) { bad = true; break; }
      pos += nb;
      out.put(syms, 8);
      rem8 -= 8;
      continue;
    }
    const uint32_t s1 = T.l1sym[i1];
    if (k1 >= rem8) {  // the run's last codes
      out.put(s1 & low_bytes_mask(rem8), rem8);
      pos += bits_of_first((m1 >> 7) & 0xFFFu, rem8 >> 3, k1 >> 3, nb1);
      rem8 = 0;
      break;
    }
    out.put(s1, k1);
    rem8 -= k1;
    const uint32_t i2 = lut_index(x << nb1);
    const uint32_t m2 = T.l1meta[i2];
    const uint32_t k2 = (m2 >> 1) & 0x38u, nb2 = m2 & 15u;
    if (!k2) {
      pos += nb1;
      continue;
    }
    const uint32_t s2 = T.l1sym[i2];
    if (k2 >= rem8) {
      out.put(s2 & low_bytes_mask(rem8), rem8);
      pos += nb1 + bits_of_first((m2 >> 7) & 0xFFFu, rem8 >> 3, k2 >> 3, nb2);
      rem8 = 0;
      break;
    }
    out.put(s2, k2);
    rem8 -= k2;
    pos += nb1 + nb2;
  }
  out.finish();
  bad = bad || rem8 != 0 || pos != stop;
  return !gsync_or(id, bad);
}

// (sign+mantissa, exponent) byte pairs [s0, e0, s1, e1] -> two BF16 values
__device__ __forceinline__ uint32_t bf16_merge2(uint32_t p) {
  return (p & 0x007F007Fu) | ((p >> 1) & 0x7F807F80u) | ((p & 0x00800080u) << 8);
}

// four sign+mantissa nibbles (16 bits) and four exponent bytes -> 4 FP8 values
__device__ __forceinline__ uint32_t fp8_merge4(uint32_t nib16, uint32_t e4) {
  const uint32_t t = (nib16 & 0xFu) | ((nib16 & 0xF0u) << 4) | ((nib16 & 0xF00u) << 8) | ((nib16 & 0xF000u) << 12);
  return ((t & 0x08080808u) << 4) | ((e4 << 3) & 0x78787878u) | (t & 0x07070707u);
}

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

template <int DT>
__device__ __forceinline__ ChunkInfo chunk_info(const Batch &b, uint32_t g) {
  ChunkInfo ci;
  ci.item = find_item(b, g);
  const Item &I = b.item[ci.item];
  ci.c = I.first_chunk + (g - I.chunk0);
  ci.raw = 0;
  uint64_t B0, B1, Bt, i0;
  if (I.page_meta) {
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

__device__ __forceinline__ void issue_stage(GroupSmem &G, const Batch &b, const ChunkInfo &ci) {
  mbar_expect_tx(&G.mbar, ci.bytes);
  bulk_g2s(G.stage, b.item[ci.item].stream + ci.lo, ci.bytes, &G.mbar);
}

// Persistent: CTA i of G decodes the contiguous chunk range
// [i*C/G, (i+1)*C/G), split into runs of one tensor (one codebook); inside a
// run the two groups take alternate chunks.  Each group copies its next
// chunk's stream bits while it merges and stores the current one.
template <int DT>
__global__ void __launch_bounds__(kDecThreads, 1) decode_kernel(const __grid_constant__ Batch b) {
  extern __shared__ __align__(128) uint8_t smem_raw[];
  DecodeSmem &S = *reinterpret_cast<DecodeSmem *>(smem_raw);
  const uint32_t tid = threadIdx.x;
  const uint32_t grp = tid / kGroupThreads, gtid = tid % kGroupThreads, id = 1 + grp;
  GroupSmem &G = S.grp[grp];
  const uint32_t g0 = (uint32_t)(((uint64_t)b.total_chunks * blockIdx.x) / gridDim.x);
  const uint32_t g1 = (uint32_t)(((uint64_t)b.total_chunks * (blockIdx.x + 1)) / gridDim.x);
  if (g0 >= g1) return;
  if (gtid == 0) {
    mbar_init(&G.mbar, 1);
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
  }
  if (tid == 0) S.abort_flag = 0;
  pdl_wait();  // the decode tables (and everything before them)
  __syncthreads();
  uint32_t parity = 0, timeout = 0;
  bool pending = false;  // a stage copy of this group is in flight

  for (uint32_t seg = g0; seg < g1;) {
    const Item &I = b.item[find_item(b, seg)];
    const uint32_t seg_end = min(g1, I.chunk0 + I.nchunks);
    __syncthreads();  // both groups are done with the previous tables
    {
      const uint4 *src = (const uint4 *)I.lut;
      uint4 *dst = (uint4 *)&S.tabs;
      for (uint32_t i = tid; i < sizeof(DecodeTables) / 16; i += kDecThreads) dst[i] = src[i];
    }
    __syncthreads();
    const bool terr = S.tabs.err != 0;
    uint32_t g = seg + grp;
    ChunkInfo ci;
    ci.fits = false;
    if (g < seg_end) {
      ci = chunk_info<DT>(b, g);
      if (ci.fits && gtid == 0) issue_stage(G, b, ci);
      pending = ci.fits;
    }
    // Stagger the groups by one decode: group 1 starts its first chunk when
    // group 0 has decoded its own and turns to the memory-bound output, so
    // one group's output overlaps the other's decode instead of coinciding.
    const bool stagger = seg_end - seg >= 2;
    if (stagger && grp == 1) named_sync(kStaggerBarrier, kDecThreads);
    for (; g < seg_end; g += kNumGroups) {
      const uint32_t cnt = ci.cnt;
      bool ok = ci.ok && !terr && !S.abort_flag;

      // One barrier per chunk before the decode: after it the stage holds the
      // chunk's stream words in MSB-first order and every thread of the group
      // is done with the previous chunk's exponent buffer.
      if (ci.fits) {
        uint32_t spins = 0;
        while (!mbar_try_wait(&G.mbar, parity) && ++spins < kSpinLimit) {
        }
        const bool late = spins >= kSpinLimit;
        if (!late) {
          // stream words to MSB-first order, once, for the peeks
          for (uint32_t i = gtid; i < ci.bytes / 4; i += kGroupThreads) G.stage[i] = bswap32(G.stage[i]);
        }
        // these generic writes come before the next bulk copy into the stage
        asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
        if (gsync_or(id, late)) {
          if (gtid == 0) {
            set_status(b.status, kFlagTimeout);
            S.abort_flag = 1;
          }
          ok = false;
        } else {
          parity ^= 1u;
          pending = false;
        }
      } else {
        gsync(id);
      }
      if (ok && ci.raw) {
        // page stored raw: its exponent bytes go straight to the buffer
        const uint8_t *src = I.raw_pool + (uint64_t)(ci.raw - 1) * b.chunk_elems;
        for (uint32_t v = gtid; v < cnt / 16; v += kGroupThreads) {
          const uint4 x = __ldg((const uint4 *)src + v);
          uint32_t *d = (uint32_t *)(G.exps + exp_slot(16 * v));  // 4-byte aligned
          d[0] = x.x;
          d[1] = x.y;
          d[2] = x.z;
          d[3] = x.w;
        }
        for (uint32_t i = cnt / 16 * 16 + gtid; i < cnt; i += kGroupThreads) G.exps[exp_slot(i)] = src[i];
        gsync(id);
      } else if (ok) {
        const uint32_t per = b.chunk_elems / kIndexStride;
        const uint32_t *vidx = (I.vindex && !I.page_meta) ? I.vindex + (uint64_t)ci.c * per : nullptr;
        // the search path ORs exponent words in: clear them (ordered before the
        // writing pass by the decoder's barriers); indexed runs store whole words
        if (!vidx)
          for (uint32_t i = gtid; i < kExpBytes / 16; i += kGroupThreads) ((uint4 *)G.exps)[i] = make_uint4(0, 0, 0, 0);
        const uint32_t *gw = (const uint32_t *)(I.stream + ci.lo);
        if (vidx) {
          if (ci.fits) ok = decode_chunk_indexed<true>(G, S.tabs, G.stage, ci.rel0, ci.nbits, cnt, id, gtid, vidx, per);
          else ok = decode_chunk_indexed<false>(G, S.tabs, gw, ci.rel0, ci.nbits, cnt, id, gtid, vidx, per);
        } else if (ci.fits) {
          ok = decode_chunk<true>(G, S.tabs, G.stage, ci.rel0, ci.nbits, cnt, id, gtid, &timeout);
        } else {
          ok = decode_chunk<false>(G, S.tabs, gw, ci.rel0, ci.nbits, cnt, id, gtid, &timeout);
        }
        if (!ok && gtid == 0) set_status(b.status, timeout ? kFlagTimeout | kFlagCorrupt : kFlagCorrupt);
      } else if (gtid == 0 && !S.abort_flag) {
        set_status(b.status, kFlagCorrupt);
      }

      if (stagger && grp == 0 && g == seg) named_arrive(kStaggerBarrier, kDecThreads);
      // The stage is free: every read of it came before the decoder's last
      // barrier, and its generic writes were fenced before the chunk's first
      // barrier.  Start copying the group's next chunk.
      ChunkInfo cn;
      cn.fits = false;
      if (g + kNumGroups < seg_end && !pending && !S.abort_flag) {
        cn = chunk_info<DT>(b, g + kNumGroups);
        if (cn.fits && gtid == 0) issue_stage(G, b, cn);
        pending = cn.fits;
      } else if (g + kNumGroups < seg_end) {
        cn = chunk_info<DT>(b, g + kNumGroups);
        cn.fits = false;
      }

      // 6. merge exponents with sign/mantissa, 16-byte coalesced stores
      if (ok) {
        const uint32_t nvec = cnt / 16;
        if (DT == EH_BF16) {
          const uint8_t *smp = I.sm + ci.sm_off;
          uint16_t *outp = (uint16_t *)I.out + ci.out_off;
          for (uint32_t v0 = gtid; v0 < nvec; v0 += 4 * kGroupThreads) {
            uint4 m[4];
            #pragma unroll
            for (int u = 0; u < 4; u++) {
              const uint32_t v = v0 + u * kGroupThreads;
              m[u] = v < nvec ? ld_nc16(smp + 16 * (uint64_t)v) : make_uint4(0, 0, 0, 0);
            }
            #pragma unroll
            for (int u = 0; u < 4; u++) {
              const uint32_t v = v0 + u * kGroupThreads;
              if (v < nvec) {
                const uint32_t *ew = (const uint32_t *)(G.exps + exp_slot(16 * v));
                const uint32_t mw[4] = {m[u].x, m[u].y, m[u].z, m[u].w};
                uint32_t o[8];
                #pragma unroll
                for (int q = 0; q < 4; q++) {
                  const uint32_t e = ew[q];
                  o[2 * q] = bf16_merge2(__byte_perm(mw[q], e, 0x5140));
                  o[2 * q + 1] = bf16_merge2(__byte_perm(mw[q], e, 0x7362));
                }
                uint4 *dst = (uint4 *)(outp + 16 * (uint64_t)v);
                dst[0] = make_uint4(o[0], o[1], o[2], o[3]);
                dst[1] = make_uint4(o[4], o[5], o[6], o[7]);
              }
            }
          }
          for (uint32_t i = nvec * 16 + gtid; i < cnt; i += kGroupThreads) {
            const uint32_t sm = smp[i], e = G.exps[exp_slot(i)];
            outp[i] = (uint16_t)(((sm & 0x80u) << 8) | (e << 7) | (sm & 0x7Fu));
          }
        } else if (DT == EH_BYTES) {
          // the decoded symbols are the output bytes
          uint8_t *outp = (uint8_t *)I.out + ci.out_off;
          for (uint32_t v = gtid; v < nvec; v += kGroupThreads) {
            const uint32_t *ew = (const uint32_t *)(G.exps + exp_slot(16 * v));
            *(uint4 *)(outp + 16 * (uint64_t)v) = make_uint4(ew[0], ew[1], ew[2], ew[3]);
          }
          for (uint32_t i = nvec * 16 + gtid; i < cnt; i += kGroupThreads) outp[i] = G.exps[exp_slot(i)];
        } else {
          const uint8_t *smp = I.sm + ci.sm_off;
          uint8_t *outp = (uint8_t *)I.out + ci.out_off;
          for (uint32_t v0 = gtid; v0 < nvec; v0 += 4 * kGroupThreads) {
            uint2 m[4];
            #pragma unroll
            for (int u = 0; u < 4; u++) {
              const uint32_t v = v0 + u * kGroupThreads;
              m[u] = v < nvec ? ld_nc8(smp + 8 * (uint64_t)v) : make_uint2(0, 0);
            }
            #pragma unroll
            for (int u = 0; u < 4; u++) {
              const uint32_t v = v0 + u * kGroupThreads;
              if (v < nvec) {
                const uint32_t *ew = (const uint32_t *)(G.exps + exp_slot(16 * v));
                uint4 o;
                o.x = fp8_merge4(m[u].x & 0xFFFFu, ew[0]);
                o.y = fp8_merge4(m[u].x >> 16, ew[1]);
                o.z = fp8_merge4(m[u].y & 0xFFFFu, ew[2]);
                o.w = fp8_merge4(m[u].y >> 16, ew[3]);
                *(uint4 *)(outp + 16 * (uint64_t)v) = o;
              }
            }
          }
          for (uint32_t i = nvec * 16 + gtid; i < cnt; i += kGroupThreads) {
            const uint32_t sm = (smp[i / 2] >> (4 * (i & 1))) & 0xFu, e = G.exps[exp_slot(i)];
            outp[i] = (uint8_t)(((sm & 8u) << 4) | (e << 3) | (sm & 7u));
          }
        }
      }
      // no barrier here: the next chunk's first barrier orders these reads of
      // the exponent buffer before it is cleared or written again
      ci = cn;
    }
    seg = seg_end;
  }
  // a copy still in flight (only after an abort) must land before the exit
  if (pending) {
    uint32_t spins = 0;
    while (!mbar_try_wait(&G.mbar, parity) && ++spins < kSpinLimit) {
    }
  }
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
  if (b.dtype == EH_BF16) return launch_pdl(decode_kernel<EH_BF16>, dim3(grid), dim3(kDecThreads), smem, s, b);
  if (b.dtype == EH_BYTES) return launch_pdl(decode_kernel<EH_BYTES>, dim3(grid), dim3(kDecThreads), smem, s, b);
  return launch_pdl(decode_kernel<EH_FP8_E4M3>, dim3(grid), dim3(kDecThreads), smem, s, b);
}

cudaError_t configure_decode() {
  const int smem = (int)(sizeof(DecodeSmem) + 128);
  cudaError_t e = cudaFuncSetAttribute(decode_kernel<EH_BF16>, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
  if (e != cudaSuccess) return e;
  e = cudaFuncSetAttribute(decode_kernel<EH_BYTES>, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
  if (e != cudaSuccess) return e;
  return cudaFuncSetAttribute(decode_kernel<EH_FP8_E4M3>, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
}

}  // namespace eh

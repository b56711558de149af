// eh_decompress.cu -- decompression kernels of libexphuff (sm_100a).
//
//   tables  one CTA per codebook: validates the code lengths and codes and
//           builds the decode tables (an 8-bit first level that decodes up to
//           four short codes per lookup, 8-bit second-level tables for codes
//           of 9..16 bits, canonical limits for anything longer);
//   decode  persistent CTAs, one chunk at a time:
//             1. the chunk's bit range is copied into shared memory with one
//                bulk asynchronous copy (cp.async.bulk + mbarrier) when it
//                fits, else read from global memory;
//             2. every thread decodes speculatively from the start of its own
//                window of the chunk's bits, recording the code boundaries of
//                its first 32 bits;
//             3. fix-up rounds: each thread restarts from the true end of its
//                predecessor and stops as soon as it lands on one of its
//                recorded boundaries (Huffman codes resynchronise after a few
//                codes), until no end moves;
//             4. CTA-wide exclusive scan of the per-thread code counts gives
//                every thread its first output index;
//             5. the threads decode again and write exponents to shared memory;
//             6. coalesced pass: exponents merged with the sign/mantissa
//                stream and stored with 16-byte stores.
// The DFloat11 article ("方法介绍") describes compact LUTs sized for on-chip
// SRAM, a two-phase kernel coordinating where each thread reads and writes,
// and block-level decompression; here the per-thread start positions are not
// stored in the format but recovered by the self-synchronising fix-up.
#include "eh_internal.cuh"

namespace eh {
namespace {

constexpr uint32_t kMaskBits = 32;            // boundaries recorded per thread
constexpr uint32_t kSpinLimit = 1u << 26;     // bounded mbarrier wait

// ---------------------------------------------------------------- tables
__global__ void __launch_bounds__(256) tables_kernel(const __grid_constant__ Batch b) {
  const Item &I = b.item[blockIdx.x];
  DecodeTables *T = (DecodeTables *)I.lut;
  const int A = alphabet_of(b.dtype);
  const int tid = threadIdx.x;
  __shared__ uint32_t cntL[33], firstL[33], baseL[33];
  __shared__ uint64_t limL[33];
  __shared__ uint8_t lens[256];
  __shared__ unsigned long long kraft;
  __shared__ uint32_t err, nsub;
  __shared__ uint32_t subpre[kNumSub];
  __shared__ uint32_t wcount[8];
  __shared__ uint8_t srt[256];

  if (blockIdx.x == 0 && tid == 0) *b.status = 0u;  // this call's status starts clean
  if (tid <= 32) cntL[tid] = 0;
  if (tid == 0) { kraft = 0; err = 0; nsub = 0; }
  const uint32_t l = tid < A ? I.code_len[tid] : 0u;
  lens[tid] = (uint8_t)l;
  __syncthreads();
  if (l > 32) atomicOr(&err, 1u);
  else if (l) {
    atomicAdd(&cntL[l], 1u);
    atomicAdd(&kraft, 1ull << (32 - l));
  }
  const uint32_t nsym = __syncthreads_count(l > 0 && l <= 32);
  if (tid == 0) {
    uint64_t code = 0;
    uint32_t idx = 0, g = 0, maxlen = 0;
    for (int L = 1; L <= 32; L++) {
      firstL[L] = (uint32_t)code;
      baseL[L] = idx;
      limL[L] = (code + cntL[L]) << (32 - L);
      code = (code + cntL[L]) << 1;
      idx += cntL[L];
      if (cntL[L]) {
        uint32_t a = g, c = (uint32_t)L;
        while (c) { uint32_t t = a % c; a = c; c = t; }
        g = a;
        maxlen = (uint32_t)L;
      }
    }
    limL[0] = 0;
    firstL[0] = baseL[0] = cntL[0] = 0;
    if (kraft > (1ull << 32)) err = 1;
    if (I.n > 0 && nsym == 0) err = 1;
    T->gcd = g ? g : 1;
    T->maxlen = maxlen;
    T->nsym = nsym;
  }
  __syncthreads();
  // symbol order (length, symbol); stored codes must be the canonical ones
  if (tid < A && l && l <= 32) {
    uint32_t k = 0;
    for (int s2 = 0; s2 < tid; s2++) k += lens[s2] == l;
    srt[baseL[l] + k] = (uint8_t)tid;
    if (I.code[tid] != firstL[l] + k) atomicOr(&err, 1u);
  }
  if (tid <= 32) {
    T->first[tid] = firstL[tid];
    T->base[tid] = baseL[tid];
    T->lim[tid] = limL[tid];
  }
  __syncthreads();
  T->sorted[tid] = tid < (int)nsym ? srt[tid] : (uint8_t)0;
  const uint8_t *sorted_g = srt;
  // first level: pattern tid = next 8 bits
  uint32_t syms = 0, pos = 0, nc = 0, len0 = 0;
  while (nc < 4) {
    int found = 0;
    for (uint32_t L = 1; L + pos <= 8; L++) {
      uint32_t v = (tid >> (8 - pos - L)) & ((1u << L) - 1u);
      if (cntL[L] && v >= firstL[L] && v - firstL[L] < cntL[L]) {
        syms |= (uint32_t)sorted_g[baseL[L] + v - firstL[L]] << (8 * nc);
        if (nc == 0) len0 = L;
        pos += L;
        nc++;
        found = 1;
        break;
      }
    }
    if (!found) break;
  }
  // prefixes of codes longer than 8 bits get a second-level table (in prefix
  // order, at most kNumSub of them)
  const bool need_sub = nc == 0 && ((uint64_t)tid << 24) < limL[32];
  const uint32_t ballot = __ballot_sync(0xffffffffu, need_sub);
  if ((tid & 31) == 0) wcount[tid >> 5] = __popc(ballot);
  __syncthreads();
  uint32_t sidx = __popc(ballot & ((1u << (tid & 31)) - 1u));
  for (int w = 0; w < (tid >> 5); w++) sidx += wcount[w];
  uint32_t sub_field = 0xFFu;
  if (need_sub && sidx < (uint32_t)kNumSub) {
    sub_field = sidx;
    subpre[sidx] = tid;
    atomicMax(&nsub, sidx + 1);
  }
  T->l1[tid] = (uint64_t)syms | ((uint64_t)len0 << 32) | ((uint64_t)pos << 36) |
               ((uint64_t)nc << 40) | ((uint64_t)sub_field << 48);
  __syncthreads();
  for (uint32_t j = 0; j < (uint32_t)kNumSub; j++) {
    uint32_t e = 0;
    if (j < nsub) {
      const uint32_t v16 = (subpre[j] << 8) | (uint32_t)tid;
      for (uint32_t L = 9; L <= 16; L++) {
        uint32_t v = v16 >> (16 - L);
        if (cntL[L] && v >= firstL[L] && v - firstL[L] < cntL[L]) {
          e = (uint32_t)sorted_g[baseL[L] + v - firstL[L]] | (L << 8);
          break;
        }
      }
    }
    T->sub[j][tid] = e;
  }
  if (tid == 0) T->err = err;
}

// ---------------------------------------------------------------- decode
template <bool kSmem>
struct BitSrc {
  const uint32_t *w;  // shared memory: words already in MSB-first order
  __device__ __forceinline__ uint32_t word(uint32_t i) const {
    if (kSmem) return w[i];
    return bswap32(__ldg(w + i));
  }
  // 32 bits starting at bit p
  __device__ __forceinline__ uint32_t peek(uint32_t p) const {
    const uint32_t i = p >> 5;
    return __funnelshift_l(word(i + 1), word(i), p & 31);
  }
};

// One decode step at the bit window `peek`.  multi: consume every complete
// code inside the 8-bit first-level index (up to 4); else only the first.
// Returns the number of codes (0: invalid code), their symbols in *syms (8
// bits each) and the bits consumed in *nbits.
__device__ __forceinline__ uint32_t decode_step(const DecodeTables &T, uint32_t peek, bool multi,
                                                uint32_t *syms, uint32_t *nbits) {
  const uint64_t e = T.l1[peek >> 24];
  const uint32_t hi = (uint32_t)(e >> 32);
  const uint32_t nc = (hi >> 8) & 7u;
  if (nc) {
    if (multi) {
      *nbits = (hi >> 4) & 15u;
      *syms = (uint32_t)e;
      return nc;
    }
    *nbits = hi & 15u;
    *syms = (uint32_t)e & 0xFFu;
    return 1;
  }
  const uint32_t si = (hi >> 16) & 0xFFu;
  if (si != 0xFFu) {
    const uint32_t e2 = T.sub[si][(peek >> 16) & 0xFFu];
    const uint32_t l = (e2 >> 8) & 63u;
    if (l) {
      *nbits = l;
      *syms = e2 & 0xFFu;
      return 1;
    }
  }
  uint32_t L = 9;
  #pragma unroll 1
  while (L <= 32 && (uint64_t)peek >= T.lim[L]) L++;
  if (L > 32) return 0;
  const uint32_t v = L == 32 ? peek : peek >> (32 - L);
  *syms = T.sorted[T.base[L] + (v - T.first[L])];
  *nbits = L;
  return 1;
}

struct DecodeSmem {
  alignas(128) uint32_t stage[kStageBytes / 4 + 16];  // bulk-copy target
  alignas(16) uint8_t exps[kMaxChunk];                // decoded exponents of one chunk
  alignas(16) DecodeTables tabs;
  uint32_t ends[kThreads];
  uint32_t wsum[kThreads / 32];
  alignas(8) unsigned long long mbar;
};

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

__device__ __forceinline__ uint32_t block_excl_scan(uint32_t v, uint32_t *wsum, uint32_t *total) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  uint32_t x = v;
  #pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    uint32_t y = __shfl_up_sync(0xffffffffu, x, o);
    if (lane >= o) x += y;
  }
  if (lane == 31) wsum[warp] = x;
  __syncthreads();
  if (warp == 0) {
    uint32_t t = lane < kThreads / 32 ? wsum[lane] : 0u;
    #pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      uint32_t y = __shfl_up_sync(0xffffffffu, t, o);
      if (lane >= o) t += y;
    }
    if (lane < kThreads / 32) wsum[lane] = t;
  }
  __syncthreads();
  *total = wsum[kThreads / 32 - 1];
  return (warp ? wsum[warp - 1] : 0u) + x - v;
}

// Steps 2-5 for one chunk whose bits are [rel0, rel0 + nbits) of `src`.
// Returns false (CTA-uniform) if the chunk is corrupt.
template <bool kSmem>
__device__ bool decode_chunk(DecodeSmem &S, const BitSrc<kSmem> src, uint32_t rel0, uint32_t nbits,
                             uint32_t cnt, uint32_t *timeout) {
  const DecodeTables &T = S.tabs;
  const uint32_t tid = threadIdx.x;
  // window width: a multiple of the gcd of the code lengths, so that a
  // fixed-length code starts every window on a code boundary
  const uint32_t gq = T.gcd;
  uint32_t W = (nbits + kThreads - 1) / kThreads;
  W = (W + gq - 1) / gq * gq;
  const uint32_t ws = min(tid * W, nbits), we = min(ws + W, nbits);

  // 2. speculative decode of the own window
  uint32_t pos = ws, n = 0, mask = 0;
  bool bad = false;
  while (pos < we) {
    const uint32_t off = pos - ws;
    const bool single = off < kMaskBits || pos + 8 > we;
    uint32_t syms, nb;
    const uint32_t k = decode_step(T, src.peek(rel0 + pos), !single, &syms, &nb);
    if (!k) { bad = true; break; }
    if (off < kMaskBits) mask |= 1u << off;
    pos += nb;
    n += k;
  }
  const uint32_t spec_end = bad ? we : pos, spec_n = n;
  const uint32_t spec_mask = bad ? 0u : mask;
  uint32_t my_start = ws, my_end = spec_end, my_n = spec_n;
  S.ends[tid] = my_end;
  __syncthreads();

  // 3. fix-up rounds
  for (uint32_t round = 0;; round++) {
    const uint32_t pred = tid == 0 ? 0u : S.ends[tid - 1];
    bool changed = false;
    if (tid > 0 && pred != my_start) {
      my_start = pred;
      uint32_t p = pred, k = 0;
      bool synced = false, bad2 = false;
      while (p < we) {
        const uint32_t off = p - ws;
        if (off < kMaskBits && ((spec_mask >> off) & 1u)) { synced = true; break; }
        const bool single = off < kMaskBits || p + 8 > we;
        uint32_t syms, nb;
        const uint32_t kk = decode_step(T, src.peek(rel0 + p), !single, &syms, &nb);
        if (!kk) { bad2 = true; break; }
        p += nb;
        k += kk;
      }
      uint32_t new_end;
      if (synced) {
        my_n = k + spec_n - __popc(spec_mask & ((1u << (p - ws)) - 1u));
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
    __syncthreads();
    if (changed) S.ends[tid] = my_end;
    if (!__syncthreads_or(changed)) break;
    if (round > kThreads + 1) {  // cannot happen for consistent data
      if (tid == 0) *timeout = 1;
      bad = true;
      break;
    }
  }

  // 4. output index of every thread's first code
  uint32_t total;
  const uint32_t o = block_excl_scan(my_n, S.wsum, &total);
  const bool ok = !__syncthreads_or(bad) && total == cnt && S.ends[kThreads - 1] == nbits;
  if (!ok) return false;

  // 5. decode again from the true start, writing exponents
  uint32_t j = o;
  pos = tid == 0 ? 0u : S.ends[tid - 1];
  while (pos < we) {
    uint32_t syms, nb;
    const uint32_t k = decode_step(T, src.peek(rel0 + pos), pos + 8 <= we, &syms, &nb);
    if (!k) break;
    for (uint32_t q = 0; q < k; q++) {
      if (j + q < cnt) S.exps[j + q] = (uint8_t)(syms >> (8 * q));
    }
    j += k;
    pos += nb;
  }
  __syncthreads();
  return true;
}

// exponent bytes E and sign/mantissa bytes M (4 values) -> 4 BF16 values
__device__ __forceinline__ uint32_t bf16_merge2(uint32_t p) {
  // p = [s0, e0, s1, e1] as bytes; value = (s&0x80)<<8 | e<<7 | (s&0x7F)
  return (p & 0x007F007Fu) | ((p >> 1) & 0x7F807F80u) | ((p & 0x00800080u) << 8);
}

template <int DT>
__global__ void __launch_bounds__(kThreads, 2) decode_kernel(const __grid_constant__ Batch b) {
  extern __shared__ __align__(128) uint8_t smem_raw[];
  DecodeSmem &S = *reinterpret_cast<DecodeSmem *>(smem_raw);
  const uint32_t tid = threadIdx.x;
  if (tid == 0) {
    mbar_init(&S.mbar, 1);
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
  }
  __syncthreads();
  uint32_t parity = 0;
  int cur = -1;
  uint32_t timeout = 0;

  for (uint32_t g = blockIdx.x; g < b.total_chunks; g += gridDim.x) {
    const int it = find_item(b, g);
    const Item &I = b.item[it];
    if (it != cur) {
      __syncthreads();
      const uint4 *src = (const uint4 *)I.lut;
      uint4 *dst = (uint4 *)&S.tabs;
      for (uint32_t i = tid; i < sizeof(DecodeTables) / 16; i += kThreads) dst[i] = src[i];
      cur = it;
      __syncthreads();
    }
    if (S.tabs.err) {
      if (tid == 0) set_status(b.status, kFlagCorrupt);
      continue;
    }
    const uint32_t c = I.first_chunk + (g - I.chunk0);
    const uint64_t i0 = (uint64_t)c * b.chunk_elems;
    const uint32_t cnt = (uint32_t)min((uint64_t)b.chunk_elems, I.n - i0);
    const uint64_t B0 = I.off[c], B1 = I.off[c + 1], Bt = I.off[I.total_chunks];
    // the stream must hold every chunk's bits plus 16 readable bytes
    const bool sane = I.off[0] == 0 && B0 <= B1 && B1 <= Bt && (Bt + 7) / 8 + 16 <= I.stream_cap &&
                      B1 - B0 >= cnt && B1 - B0 <= (uint64_t)cnt * S.tabs.maxlen;
    if (!sane) {
      if (tid == 0) set_status(b.status, kFlagCorrupt);
      continue;
    }
    const uint32_t nbits = (uint32_t)(B1 - B0);
    const uint64_t lo = (B0 >> 3) & ~uint64_t(15);
    const uint64_t hi = (((B1 + 7) >> 3) + 8 + 15) & ~uint64_t(15);
    const uint32_t rel0 = (uint32_t)(B0 - lo * 8);
    bool ok;
    if (hi - lo <= (uint64_t)kStageBytes && hi <= I.stream_cap) {
      const uint32_t bytes = (uint32_t)(hi - lo);
      // order this CTA's earlier generic accesses of the stage before the
      // asynchronous copy overwrites it
      asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
      __syncthreads();
      if (tid == 0) {
        mbar_expect_tx(&S.mbar, bytes);
        bulk_g2s(S.stage, I.stream + lo, bytes, &S.mbar);
      }
      uint32_t spins = 0;
      while (!mbar_try_wait(&S.mbar, parity) && ++spins < kSpinLimit) {
      }
      if (__syncthreads_or(spins >= kSpinLimit)) {
        // the copy never completed: give it one more bounded wait, then stop
        spins = 0;
        while (!mbar_try_wait(&S.mbar, parity) && ++spins < kSpinLimit) {
        }
        if (tid == 0) set_status(b.status, kFlagTimeout);
        return;
      }
      parity ^= 1u;
      const uint32_t nw = bytes / 4;
      for (uint32_t i = tid; i < nw; i += kThreads) S.stage[i] = bswap32(S.stage[i]);
      if (tid < 2) S.stage[nw + tid] = 0u;
      __syncthreads();
      BitSrc<true> src{S.stage};
      ok = decode_chunk<true>(S, src, rel0, nbits, cnt, &timeout);
    } else {
      BitSrc<false> src{(const uint32_t *)(I.stream + lo)};
      ok = decode_chunk<false>(S, src, rel0, nbits, cnt, &timeout);
    }
    if (!ok) {
      if (tid == 0) set_status(b.status, timeout ? kFlagTimeout | kFlagCorrupt : kFlagCorrupt);
      __syncthreads();
      continue;
    }

    // 6. merge exponents with sign/mantissa, 16-byte stores
    if (DT == EH_BF16) {
      const uint8_t *smp = I.sm + i0;
      uint16_t *outp = (uint16_t *)I.out + (i0 - I.elem0);
      const uint32_t nvec = cnt / 16;
      #pragma unroll 2
      for (uint32_t v = tid; v < nvec; v += kThreads) {
        const uint4 m = __ldg((const uint4 *)smp + v);
        const uint4 e = *(const uint4 *)(S.exps + 16 * v);
        const uint32_t mw[4] = {m.x, m.y, m.z, m.w}, ew[4] = {e.x, e.y, e.z, e.w};
        uint32_t o[8];
        #pragma unroll
        for (int q = 0; q < 4; q++) {
          o[2 * q] = bf16_merge2(__byte_perm(mw[q], ew[q], 0x5140));
          o[2 * q + 1] = bf16_merge2(__byte_perm(mw[q], ew[q], 0x7362));
        }
        uint4 *dst = (uint4 *)(outp + 16 * (uint64_t)v);
        dst[0] = make_uint4(o[0], o[1], o[2], o[3]);
        dst[1] = make_uint4(o[4], o[5], o[6], o[7]);
      }
      for (uint32_t i = nvec * 16 + tid; i < cnt; i += kThreads) {
        const uint32_t s = smp[i], e = S.exps[i];
        outp[i] = (uint16_t)(((s & 0x80u) << 8) | (e << 7) | (s & 0x7Fu));
      }
    } else {
      const uint8_t *smp = I.sm + i0 / 2;
      uint8_t *outp = (uint8_t *)I.out + (i0 - I.elem0);
      const uint32_t nvec = cnt / 16;
      #pragma unroll 2
      for (uint32_t v = tid; v < nvec; v += kThreads) {
        const uint2 m = __ldg((const uint2 *)smp + v);
        const uint4 e = *(const uint4 *)(S.exps + 16 * v);
        const uint32_t mh[4] = {m.x & 0xFFFFu, m.x >> 16, m.y & 0xFFFFu, m.y >> 16};
        const uint32_t ew[4] = {e.x, e.y, e.z, e.w};
        uint32_t o[4];
        #pragma unroll
        for (int q = 0; q < 4; q++) {
          const uint32_t x = mh[q];
          const uint32_t t = (x & 0xFu) | ((x & 0xF0u) << 4) | ((x & 0xF00u) << 8) | ((x & 0xF000u) << 12);
          o[q] = ((t & 0x08080808u) << 4) | ((ew[q] << 3) & 0x78787878u) | (t & 0x07070707u);
        }
        *(uint4 *)(outp + 16 * (uint64_t)v) = make_uint4(o[0], o[1], o[2], o[3]);
      }
      for (uint32_t i = nvec * 16 + tid; i < cnt; i += kThreads) {
        const uint32_t s = (smp[i / 2] >> (4 * (i & 1))) & 0xFu, e = S.exps[i];
        outp[i] = (uint8_t)(((s & 8u) << 4) | (e << 3) | (s & 7u));
      }
    }
    __syncthreads();
  }
}

}  // namespace

cudaError_t launch_tables(const Batch &b, cudaStream_t s) {
  tables_kernel<<<b.k, 256, 0, s>>>(b);
  return cudaGetLastError();
}

cudaError_t launch_decode(const Batch &b, cudaStream_t s, int num_sms) {
  if (b.total_chunks == 0) return cudaSuccess;
  const size_t smem = sizeof(DecodeSmem) + 128;
  uint32_t grid = (uint32_t)num_sms * 2;
  if (grid > b.total_chunks) grid = b.total_chunks;
  if (b.dtype == EH_BF16) decode_kernel<EH_BF16><<<grid, kThreads, smem, s>>>(b);
  else decode_kernel<EH_FP8_E4M3><<<grid, kThreads, smem, s>>>(b);
  return cudaGetLastError();
}

cudaError_t configure_decode() {
  const int smem = (int)(sizeof(DecodeSmem) + 128);
  cudaError_t e = cudaFuncSetAttribute(decode_kernel<EH_BF16>, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
  if (e != cudaSuccess) return e;
  return cudaFuncSetAttribute(decode_kernel<EH_FP8_E4M3>, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
}

}  // namespace eh

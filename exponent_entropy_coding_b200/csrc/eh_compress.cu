// eh_compress.cu -- compression kernels of libexphuff (sm_100a).
//
// Steps, in launch order (one launch per step for a whole batch of tensors):
//   hist     count the exponent fields per chunk and per tensor (DFloat11
//            article, "方法介绍": the Huffman code is built from the exponent
//            distribution);
//   book     one CTA per tensor: code lengths (minimum-variance Huffman,
//            package-merge when the depth exceeds the limit), rank assignment,
//            canonical codes;
//   offsets  code bits per chunk from its histogram, then (last CTA) an
//            exclusive scan into the chunk bit offsets and the clearing of the
//            stream words that two chunks share;
//   encode   one CTA per chunk (256 threads when the call has a full wave
//            of such CTAs, else 512): the packed sign/mantissa array (sign and
//            mantissa stay raw), code lookup, CTA-wide exclusive scan of code
//            lengths, bit packing into a shared-memory word ring, coalesced
//            stores of whole words and atomic OR of the two edge words (and,
//            when asked for, the value index).
// Each kernel after hist is a programmatic dependent launch: it starts while
// its predecessor finishes and waits for it before reading its results.
// All of this is integer work (no dense contraction, no tensor cores); the
// histogram runs near the HBM bound, the encoder is bound by instruction
// issue.
#include "eh_internal.cuh"

namespace eh {
namespace {

__device__ __forceinline__ uint4 ld_stream(const void *p) {
  uint4 v;
  asm volatile("ld.global.nc.L1::no_allocate.v4.u32 {%0,%1,%2,%3}, [%4];"
               : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w)
               : "l"(p));
  return v;
}

// BF16 pair in one word -> the two sign+mantissa bytes (s<<7 | m7), low
// element in the low byte.
__device__ __forceinline__ uint32_t bf16x2_sm(uint32_t x) {
  return (x & 0x7Fu) | ((x >> 8) & 0x7F80u) | ((x >> 16) & 0x8000u);
}

// Four FP8 bytes in one word -> four sign+mantissa nibbles (s<<3 | m3),
// element 0 in the low nibble.
__device__ __forceinline__ uint32_t fp8x4_sm(uint32_t x) {
  uint32_t t = (x & 0x07070707u) | ((x >> 4) & 0x08080808u);
  return (t & 0xFu) | ((t >> 4) & 0xF0u) | ((t >> 8) & 0xF00u) | ((t >> 12) & 0xF000u);
}

// ---------------------------------------------------------------- hist
// Exponent counters are replicated per lane: counter (e, lane) lives at
// h[e*32 + lane], so the 32 lanes of a warp always hit 32 distinct banks and
// never the same address, however skewed the exponents are.
template <int DT>
__global__ void __launch_bounds__(kThreads, 2) hist_kernel(const __grid_constant__ Batch b) {
  constexpr int A = DT == EH_FP8_E4M3 ? 16 : 256;
  __shared__ uint32_t h[A * 32];
  pdl_trigger();
  const uint32_t g = blockIdx.x;
  const Item &I = b.item[find_item(b, g)];
  const uint32_t c = g - I.chunk0;
  const uint64_t i0 = (uint64_t)c * b.chunk_elems;
  const uint32_t cnt = (uint32_t)min((uint64_t)b.chunk_elems, I.n - i0);
  const int tid = threadIdx.x, lane = tid & 31;
  for (int i = tid; i < A * 32; i += kThreads) h[i] = 0;
  __syncthreads();
  uint32_t *hl = h + lane;
  uint8_t *hb = (uint8_t *)hl;
  if (DT == EH_BF16) {
    const uint16_t *in = (const uint16_t *)I.in + i0;
    const uint32_t nvec = cnt / 16;  // 16 values per step: 32 B in
    #pragma unroll 2
    for (uint32_t v = tid; v < nvec; v += kThreads) {
      uint4 p = ld_stream(in + 16 * (uint64_t)v);
      uint4 q = ld_stream(in + 16 * (uint64_t)v + 8);
      uint32_t w[8] = {p.x, p.y, p.z, p.w, q.x, q.y, q.z, q.w};
      #pragma unroll
      for (int j = 0; j < 8; j++) {
        // exponent e sits in bits 7..14 of each half: e << 7 is the byte
        // offset of row e (32 counters of 4 bytes) in the lane's column
        atomicAdd((uint32_t *)(hb + (w[j] & 0x7F80u)), 1u);
        atomicAdd((uint32_t *)(hb + ((w[j] >> 16) & 0x7F80u)), 1u);
      }
    }
    for (uint32_t i = nvec * 16 + tid; i < cnt; i += kThreads) atomicAdd(hl + (((in[i] >> 7) & 0xFFu) << 5), 1u);
  } else if (DT == EH_BYTES) {
    // every byte is a symbol; there is no sign/mantissa to write
    const uint8_t *in = (const uint8_t *)I.in + i0;
    const uint32_t nvec = cnt / 32;
    #pragma unroll 2
    for (uint32_t v = tid; v < nvec; v += kThreads) {
      uint4 p = ld_stream(in + 32 * (uint64_t)v);
      uint4 q = ld_stream(in + 32 * (uint64_t)v + 16);
      const uint32_t w[8] = {p.x, p.y, p.z, p.w, q.x, q.y, q.z, q.w};
      #pragma unroll
      for (int j = 0; j < 8; j++) {
        #pragma unroll
        for (int k = 0; k < 4; k++) atomicAdd(hl + (((w[j] >> (8 * k)) & 0xFFu) << 5), 1u);
      }
    }
    for (uint32_t i = nvec * 32 + tid; i < cnt; i += kThreads) atomicAdd(hl + ((uint32_t)in[i] << 5), 1u);
  } else {
    const uint8_t *in = (const uint8_t *)I.in + i0;
    const uint32_t nvec = cnt / 32;  // 32 values per step: 32 B in
    #pragma unroll 2
    for (uint32_t v = tid; v < nvec; v += kThreads) {
      uint4 p = ld_stream(in + 32 * (uint64_t)v);
      uint4 q = ld_stream(in + 32 * (uint64_t)v + 16);
      uint32_t w[8] = {p.x, p.y, p.z, p.w, q.x, q.y, q.z, q.w};
      #pragma unroll
      for (int j = 0; j < 8; j++) {
        #pragma unroll
        for (int k = 0; k < 4; k++) atomicAdd(hl + (((w[j] >> (8 * k + 3)) & 0xFu) << 5), 1u);
      }
    }
    for (uint32_t i = nvec * 32 + tid; i < cnt; i += kThreads) atomicAdd(hl + (((in[i] >> 3) & 0xFu) << 5), 1u);
  }
  __syncthreads();
  if (tid < A) {
    uint32_t s = 0;
    #pragma unroll 8
    for (int l = 0; l < 32; l++) s += h[tid * 32 + ((l + tid) & 31)];
    I.chist[(uint64_t)c * A + tid] = s;
    if (s) atomicAdd((unsigned long long *)&I.counts[tid], (unsigned long long)s);
  }
}

// ---------------------------------------------------------------- book
// One CTA of 256 threads per tensor.
__global__ void __launch_bounds__(256) book_kernel(const __grid_constant__ Batch b) {
  pdl_trigger();
  pdl_wait();  // the histogram kernel's counts
  const Item &I = b.item[blockIdx.x];
  const int A = alphabet_of(b.dtype);
  const int Lmax = (int)b.max_code_len;
  const int tid = threadIdx.x;
  __shared__ uint64_t lw[256];      // leaf weights in (count, symbol) order
  __shared__ uint64_t iw[256];      // internal node weights in creation order
  __shared__ uint16_t lpar[256], ipar[256];
  __shared__ uint8_t idep[256];
  __shared__ uint8_t len[256];
  __shared__ uint32_t nlen[33], firstc[33];
  __shared__ uint32_t xsel[33];     // package-merge: leaves selected per level
  __shared__ uint32_t maxd, nint_s;
  __shared__ uint8_t ps[256];       // present symbols, increasing
  __shared__ uint64_t pcnt[256];    // their counts, in the same order
  __shared__ uint8_t plen[256];     // their code lengths, in the same order
  __shared__ uint32_t wpres[8];

  const uint64_t c = tid < A ? I.counts[tid] : 0ull;
  len[tid] = 0;
  if (tid <= 32) nlen[tid] = 0;
  if (tid == 0) maxd = 0;
  // compact list of the present symbols (loops below run over it only)
  const uint32_t pb = __ballot_sync(0xffffffffu, c > 0);
  if ((tid & 31) == 0) wpres[tid >> 5] = __popc(pb);
  __syncthreads();
  uint32_t pidx = __popc(pb & ((1u << (tid & 31)) - 1u));
  int m = 0;
  for (int w = 0; w < 8; w++) {
    if (w < (tid >> 5)) pidx += wpres[w];
    m += wpres[w];
  }
  if (c > 0) {
    ps[pidx] = (uint8_t)tid;
    pcnt[pidx] = c;
  }
  __syncthreads();
  // rank of each present symbol in (count, symbol) order (independent loads)
  uint32_t r_asc = 0, r_desc = 0;
  if (c > 0) {
    #pragma unroll 4
    for (int j = 0; j < m; j++) {
      const uint64_t c2 = pcnt[j];
      const bool below = ps[j] < tid;
      r_asc += c2 < c || (c2 == c && below);
      r_desc += c2 > c || (c2 == c && below);
    }
    lw[r_asc] = c;
  }
  bool feasible = m <= 1 || Lmax >= 32 || (uint64_t)m <= (1ull << Lmax);
  if (!feasible) {
    if (tid == 0) set_status(b.status, kFlagInfeasible);
  }
  __syncthreads();

  uint32_t d = 0;  // raw length of the leaf with rank `tid` in (count, symbol) order
  if (m >= 2 && feasible) {
    if (tid == 0) {
      // two-queue Huffman: leaves sorted by (count, symbol), internal nodes in
      // creation order; on equal weight the leaf wins (its id is smaller).
      // The next leaf and the next internal weight are kept in registers.
      int i = 0, j = 0, nint = 0;
      uint64_t li = lw[0], ij = 0;  // ij is iw[j] while j < nint
      for (int step = 0; step < m - 1; step++) {
        uint64_t w = 0;
        #pragma unroll
        for (int pick = 0; pick < 2; pick++) {
          if (i < m && (j >= nint || li <= ij)) {
            w += li;
            lpar[i++] = (uint16_t)nint;
            li = i < m ? lw[i] : 0ull;
          } else {
            w += ij;
            ipar[j++] = (uint16_t)nint;
            ij = j < nint ? iw[j] : 0ull;
          }
        }
        iw[nint] = w;
        if (j == nint) ij = w;  // the queue was empty: the new node is next
        nint++;
      }
      nint_s = (uint32_t)nint;
    }
    __syncthreads();
    // internal node depths by pointer jumping: depth += depth(parent),
    // parent = parent(parent); the root (last node) is its own parent
    const uint32_t nint = nint_s;
    uint32_t dep = 0, par = 0;
    if (tid < nint) {
      const bool root = tid == nint - 1;
      dep = root ? 0u : 1u;
      par = root ? tid : ipar[tid];
      idep[tid] = (uint8_t)dep;
      ipar[tid] = (uint16_t)par;
    }
    __syncthreads();
    for (int round = 0; round < 8; round++) {  // 2^8 levels cover any tree of 256 leaves
      uint32_t pd = 0, pp = 0;
      if (tid < nint) {
        pd = idep[par];
        pp = ipar[par];
      }
      __syncthreads();
      if (tid < nint) {
        dep += pd;
        par = pp;
        idep[tid] = (uint8_t)dep;
        ipar[tid] = (uint16_t)par;
      }
      __syncthreads();
    }
    if (tid < m) {
      d = idep[lpar[tid]] + 1u;
      atomicMax(&maxd, d);
    }
    __syncthreads();
    if ((int)maxd > Lmax) {
      if (tid == 0) {
        // package-merge with counts only: list(level) = merge(leaves,
        // packages(level)), leaf first on equal weight; packages(level) pair
        // up consecutive items of list(level+1); list(Lmax) = leaves.
        uint64_t *pk = I.pm_scratch;  // [33][256]
        uint32_t npk[33];
        npk[Lmax] = 0;
        for (int lev = Lmax - 1; lev >= 1; lev--) {
          const uint64_t *below = pk + (uint64_t)(lev + 1) * 256;
          uint64_t *cur = pk + (uint64_t)lev * 256;
          uint32_t nb = npk[lev + 1], li = 0, pi = 0, np = 0;
          uint64_t pend = 0;
          bool have = false;
          for (uint32_t r = 0; r < (uint32_t)m + nb; r++) {
            uint64_t w;
            if (li < (uint32_t)m && (pi >= nb || lw[li] <= below[pi])) w = lw[li++];
            else w = below[pi++];
            if (have) { cur[np++] = pend + w; have = false; }
            else { pend = w; have = true; }
          }
          npk[lev] = np;
        }
        uint32_t sel = 2u * (uint32_t)m - 2u;
        for (int lev = 1; lev <= Lmax; lev++) {
          const uint64_t *cur = pk + (uint64_t)lev * 256;
          uint32_t np = npk[lev], li = 0, pi = 0;
          for (uint32_t r = 0; r < sel; r++) {
            if (li < (uint32_t)m && (pi >= np || lw[li] <= cur[pi])) li++;
            else pi++;
          }
          xsel[lev] = li;
          sel = 2u * pi;
        }
      }
      __syncthreads();
      if (tid < m) {
        d = 0;
        for (int lev = 1; lev <= Lmax; lev++) d += (uint32_t)tid < xsel[lev];
      }
    }
    if (tid < m) atomicAdd(&nlen[d], 1u);
  } else if (m == 1 && tid < m) {
    d = 1;
    atomicAdd(&nlen[1], 1u);
  }
  __syncthreads();

  // rank assignment: the r-th shortest length goes to the symbol of rank r in
  // (count descending, symbol ascending) order
  if (c > 0 && feasible) {
    const uint32_t r = r_desc;
    uint32_t cum = 0, L = 1;
    for (; L <= 32; L++) {
      cum += nlen[L];
      if (cum > r) break;
    }
    len[tid] = (uint8_t)L;
  }
  if (tid < 32) {
    // first canonical code of each length L (lane L-1): the exclusive prefix
    // of nlen[L'] << (32 - L'), shifted down by 32 - L
    const uint32_t L = tid + 1;
    const uint64_t aL = (uint64_t)nlen[L] << (32 - L);
    uint64_t inc = aL;
    #pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const uint64_t y = __shfl_up_sync(0xffffffffu, inc, o);
      if (tid >= (uint32_t)o) inc += y;
    }
    firstc[L] = (uint32_t)((inc - aL) >> (32 - L));
  }
  __syncthreads();
  if (tid < m) plen[tid] = len[ps[tid]];
  __syncthreads();
  if (tid < A) {
    uint32_t l = len[tid], code = 0;
    if (l) {
      // symbols of the same length below this one (present symbols are in
      // increasing order, so the first pidx entries are the smaller ones)
      uint32_t k = 0;
      #pragma unroll 4
      for (uint32_t j = 0; j < pidx; j++) k += plen[j] == l;
      code = firstc[l] + k;
    }
    I.code_len[tid] = (uint8_t)l;
    I.code[tid] = code;
  }
}

// ---------------------------------------------------------------- offsets
__device__ __forceinline__ uint64_t warp_sum64(uint64_t v) {
  #pragma unroll
  for (int o = 16; o; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  return v;
}

constexpr int kOffThreads = 1024;          // one warp per chunk
constexpr int kOffPerThread = 4;           // chunks per thread in the final scan
constexpr int kOffTile = kOffThreads * kOffPerThread;

__global__ void __launch_bounds__(kOffThreads) offsets_kernel(const __grid_constant__ Batch b) {
  pdl_trigger();
  pdl_wait();  // the code lengths
  const int A = alphabet_of(b.dtype);
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const uint32_t g = blockIdx.x * (kOffThreads / 32) + warp;
  if (g < b.total_chunks) {
    const Item &I = b.item[find_item(b, g)];
    const uint32_t c = g - I.chunk0;
    uint64_t bits = 0;
    for (int s = lane; s < A; s += 32) bits += (uint64_t)I.chist[(uint64_t)c * A + s] * I.code_len[s];
    bits = warp_sum64(bits);
    if (lane == 0) I.cbits[c] = bits;
  }
  __shared__ uint32_t last;
  __threadfence();
  __syncthreads();
  if (tid == 0) last = atomicAdd(b.ticket, 1u) == gridDim.x - 1;
  __syncthreads();
  if (!last) return;
  __threadfence();

  // Last CTA: one exclusive scan over the chunks of all tensors in launch
  // order; a tensor's offsets are that scan minus its value at the tensor's
  // first chunk.
  __shared__ uint64_t wtot[kOffThreads / 32];
  __shared__ uint64_t base[EH_MAX_BATCH + 1];
  __shared__ uint64_t carry_sh;
  if (tid == 0) carry_sh = 0;
  __syncthreads();
  for (uint32_t t0 = 0; t0 < b.total_chunks; t0 += kOffTile) {
    const uint32_t g0 = t0 + tid * kOffPerThread;
    uint64_t v[kOffPerThread], local = 0;
    #pragma unroll
    for (int j = 0; j < kOffPerThread; j++) {
      v[j] = 0;
      const uint32_t gg = g0 + j;
      if (gg < b.total_chunks) {
        const Item &I = b.item[find_item(b, gg)];
        v[j] = __ldcg(I.cbits + (gg - I.chunk0));
      }
      local += v[j];
    }
    uint64_t x = local;
    #pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const uint64_t y = __shfl_up_sync(0xffffffffu, x, o);
      if (lane >= o) x += y;
    }
    if (lane == 31) wtot[warp] = x;
    __syncthreads();
    if (warp == 0) {
      uint64_t t = wtot[lane];
      #pragma unroll
      for (int o = 1; o < 32; o <<= 1) {
        const uint64_t y = __shfl_up_sync(0xffffffffu, t, o);
        if (lane >= o) t += y;
      }
      wtot[lane] = t;
    }
    __syncthreads();
    const uint64_t carry = carry_sh;
    uint64_t run = carry + (warp ? wtot[warp - 1] : 0ull) + x - local;  // exclusive at g0
    uint64_t ex[kOffPerThread];
    #pragma unroll
    for (int j = 0; j < kOffPerThread; j++) {
      ex[j] = run;
      const uint32_t gg = g0 + j;
      if (gg < b.total_chunks) {
        const int it = find_item(b, gg);
        if (gg == b.item[it].chunk0) base[it] = run;
      }
      run += v[j];
    }
    __syncthreads();
    #pragma unroll
    for (int j = 0; j < kOffPerThread; j++) {
      const uint32_t gg = g0 + j;
      if (gg < b.total_chunks) {
        const int it = find_item(b, gg);
        const Item &I = b.item[it];
        const uint64_t off = ex[j] - base[it];
        I.off[gg - I.chunk0] = off;
        ((uint32_t *)I.stream)[off >> 5] = 0u;  // word shared with the previous chunk: cleared for OR
      }
    }
    __syncthreads();
    if (tid == kOffThreads - 1) carry_sh = run;
    __syncthreads();
  }
  // totals: the scan value after each tensor's last chunk
  if (tid < (int)b.k) {
    const Item &I = b.item[tid];
    uint64_t end;
    if (I.nchunks == 0) {
      end = 0;
    } else {
      // exclusive value at the next tensor's first chunk, or the grand total
      uint64_t after = carry_sh;
      for (uint32_t j = tid + 1; j < b.k; j++)
        if (b.item[j].nchunks) { after = base[j]; break; }
      end = after - base[tid];
    }
    I.off[I.nchunks] = end;
    if (end & 31) ((uint32_t *)I.stream)[end >> 5] = 0u;
    I.bits_out[0] = end;
    if (I.bits_dev) I.bits_dev[0] = end;
  }
  if (tid == 0) *b.ticket = 0u;  // ready for the next call
}

// ---------------------------------------------------------------- encode
constexpr int kEncPerThread = 16;  // values per thread per tile

// An encoding CTA of NT threads takes tiles of NT * 16 values and packs them
// into a shared ring of twice as many 32-bit words (more than one tile of
// 32-bit codes plus the partial word carried over).
template <int NT>
struct Enc {
  static constexpr int kTile = NT * kEncPerThread;
  static constexpr int kRingWords = 2 * kTile;
  static constexpr uint32_t kRingMask = kRingWords - 1;
  static constexpr int kMinBlocks = NT == 256 ? 4 : 2;  // CTAs per SM (64 registers a thread)
};
// Calls with at least a full wave of 256-thread CTAs (four per SM) use them;
// calls with fewer chunks use 512-thread CTAs, which finish a chunk sooner.
constexpr int kEncSmall = 256, kEncLarge = 512;

// Exclusive scan over the CTA with a single barrier: every warp publishes
// its total, then each thread adds up the totals of the warps before its own.
// The caller must separate two uses of `wsum` by a barrier.
template <int NT>
__device__ __forceinline__ uint32_t block_excl_scan1(uint32_t v, uint32_t *wsum, uint32_t *total) {
  constexpr int kWarps = NT / 32;
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  uint32_t x = v;
  #pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const uint32_t y = __shfl_up_sync(0xffffffffu, x, o);
    if (lane >= o) x += y;
  }
  if (lane == 31) wsum[warp] = x;
  __syncthreads();
  // lane i < kWarps holds warp i's total; prefix over lanes below `warp`
  const uint32_t t = lane < kWarps ? wsum[lane] : 0u;
  *total = __reduce_add_sync(0xffffffffu, t);  // one warp reduction each
  const uint32_t pre = __reduce_add_sync(0xffffffffu, lane < warp ? t : 0u);
  return pre + x - v;
}

template <int DT>
__device__ __forceinline__ void load_exps(const void *in, uint32_t idx, uint32_t cnt, uint4 &p, uint4 &q) {
  if (DT == EH_BF16) {
    const uint16_t *x = (const uint16_t *)in;
    if (idx + 16 <= cnt) {
      p = ld_stream(x + idx);
      q = ld_stream(x + idx + 8);
    } else {
      uint32_t w[8];
      #pragma unroll
      for (int j = 0; j < 8; j++) {
        const uint32_t a = idx + 2 * j < cnt ? x[idx + 2 * j] : 0u;
        const uint32_t b2 = idx + 2 * j + 1 < cnt ? x[idx + 2 * j + 1] : 0u;
        w[j] = a | (b2 << 16);
      }
      p = make_uint4(w[0], w[1], w[2], w[3]);
      q = make_uint4(w[4], w[5], w[6], w[7]);
    }
  } else {
    const uint8_t *x = (const uint8_t *)in;
    if (idx + 16 <= cnt) {
      p = ld_stream(x + idx);
    } else {
      uint32_t w[4] = {0, 0, 0, 0};
      #pragma unroll
      for (int j = 0; j < 16; j++)
        if (idx + j < cnt) w[j / 4] |= (uint32_t)x[idx + j] << (8 * (j & 3));
      p = make_uint4(w[0], w[1], w[2], w[3]);
    }
    q = make_uint4(0, 0, 0, 0);
  }
}

template <int DT>
__device__ __forceinline__ uint32_t exp_of(const uint4 &p, const uint4 &q, int j) {
  if (DT == EH_BF16) {
    const uint32_t w[8] = {p.x, p.y, p.z, p.w, q.x, q.y, q.z, q.w};
    return (w[j >> 1] >> ((j & 1) ? 23 : 7)) & 0xFFu;
  } else if (DT == EH_BYTES) {
    const uint32_t w[4] = {p.x, p.y, p.z, p.w};
    return (w[j >> 2] >> (8 * (j & 3))) & 0xFFu;
  } else {
    const uint32_t w[4] = {p.x, p.y, p.z, p.w};
    return (w[j >> 2] >> (8 * (j & 3) + 3)) & 0xFu;
  }
}

// (code left-aligned, length) of value j's exponent.  BF16: the exponent
// sits in bits 7..14 of each half, so (e << 3), the entry's byte offset, is
// one shift and one mask away.
template <int DT>
__device__ __forceinline__ uint2 code_of(const uint2 *tab, const uint4 &p, const uint4 &q, int j) {
  if (DT == EH_BF16) {
    const uint32_t w[8] = {p.x, p.y, p.z, p.w, q.x, q.y, q.z, q.w};
    const uint32_t off = (w[j >> 1] >> ((j & 1) ? 20 : 4)) & 0x7F8u;
    return *(const uint2 *)((const uint8_t *)tab + off);
  }
  return tab[exp_of<DT>(p, q, j)];
}

// The sign/mantissa array of values [idx, idx + 16) of a chunk (held in p, q
// as loaded by load_exps), written by the encoder beside the code packing.
// BF16: one byte per value (s << 7 | m7); FP8: one nibble (s << 3 | m3),
// value 2i in the low nibble of byte i, the high nibble of an odd tail zero.
template <int DT>
__device__ __forceinline__ void store_sm(uint8_t *smo, uint32_t idx, uint32_t cnt, const uint4 &p, const uint4 &q) {
  if (DT == EH_BF16) {
    const uint32_t w[8] = {p.x, p.y, p.z, p.w, q.x, q.y, q.z, q.w};
    if (idx + 16 <= cnt) {
      uint32_t o[4];
      #pragma unroll
      for (int j = 0; j < 4; j++) {
        // low bytes carry the mantissas, high bytes the signs (bit 7)
        const uint32_t lows = __byte_perm(w[2 * j], w[2 * j + 1], 0x6420);
        const uint32_t highs = __byte_perm(w[2 * j], w[2 * j + 1], 0x7531);
        o[j] = (lows & 0x7F7F7F7Fu) | (highs & 0x80808080u);
      }
      *(uint4 *)(smo + idx) = make_uint4(o[0], o[1], o[2], o[3]);
    } else {
      for (int j = 0; j < 16; j++)
        if (idx + j < cnt) smo[idx + j] = (uint8_t)(bf16x2_sm(w[j >> 1] >> (16 * (j & 1))) & 0xFFu);
    }
  } else if (DT == EH_FP8_E4M3) {
    if (idx + 16 <= cnt) {
      const uint32_t lo = fp8x4_sm(p.x) | (fp8x4_sm(p.y) << 16);
      const uint32_t hi = fp8x4_sm(p.z) | (fp8x4_sm(p.w) << 16);
      *(uint2 *)(smo + idx / 2) = make_uint2(lo, hi);
    } else {
      const uint32_t w[4] = {p.x, p.y, p.z, p.w};
      for (int j = 0; j < 16; j += 2) {
        if (idx + j >= cnt) break;
        const uint32_t pair = (w[j >> 2] >> (8 * (j & 3))) & 0xFFFFu;  // values j, j + 1
        uint32_t sm = fp8x4_sm(pair) & 0xFFu;
        if (idx + j + 1 >= cnt) sm &= 0xFu;
        smo[(idx + j) / 2] = (uint8_t)sm;
      }
    }
  }
}

// Ring positions are bits relative to the start of the stream word that
// holds the range's first bit (32-bit arithmetic; a range is one chunk or
// page).  Ring word k is stream word (bit0 >> 5) + k, at slot k & kRingMask.
// ring_or ORs the `nbits` (<= 32) code bits held right-aligned in `acc` in at
// relative bit `pos`.
template <int NT>
__device__ __forceinline__ void ring_or(uint32_t *ring, uint32_t pos, uint32_t acc, uint32_t nbits) {
  constexpr uint32_t kRingMask = Enc<NT>::kRingMask;
  const uint32_t s = pos & 31, w = pos >> 5;
  const uint64_t y = (uint64_t)acc << (64 - s - nbits);
  atomicOr(&ring[w & kRingMask], (uint32_t)(y >> 32));
  if (s + nbits > 32) atomicOr(&ring[(w + 1) & kRingMask], (uint32_t)y);
}

// ORs the low nbits (1..64) of (hi:lo) into the ring at relative bit pos.
template <int NT>
__device__ __forceinline__ void ring_or64(uint32_t *ring, uint32_t pos, uint32_t hi, uint32_t lo, uint32_t nbits) {
  constexpr uint32_t kRingMask = Enc<NT>::kRingMask;
  const uint32_t s = pos & 31, w = pos >> 5;
  const uint64_t L = (((uint64_t)hi << 32) | lo) << (64 - nbits);  // left-aligned
  atomicOr(&ring[w & kRingMask], (uint32_t)(L >> (32 + s)));
  if (s + nbits > 32) atomicOr(&ring[(w + 1) & kRingMask], (uint32_t)(L >> s));
  if (s + nbits > 64) atomicOr(&ring[(w + 2) & kRingMask], (uint32_t)(L << (32 - s)));
}

// Packs the codes of values [0, cnt) of `in` into stream bits [bit0, bit1)
// of gs.  The ring must be zero on entry and is zero on return.  Words that
// the range shares with its neighbours are OR-ed into (pre-cleared) stream
// words unless `exclusive`, when the range owns every word it touches.
// kIndex: the value index is written (into vindex); without it the encoding
// loop carries no index code at all.
template <int DT, int NT, bool kIndex = false>
__device__ void encode_range(const uint2 *tab, const uint8_t *in, uint32_t cnt, uint64_t bit0, uint64_t bit1,
                             uint32_t *gs, uint32_t *ring, uint32_t *wsum, bool exclusive,
                             uint32_t *vindex = nullptr, uint8_t *smo = nullptr) {
  constexpr int kEncTile = Enc<NT>::kTile;
  constexpr uint32_t kRingMask = Enc<NT>::kRingMask;
  const int tid = threadIdx.x;
  const uint64_t gw0 = bit0 >> 5;             // stream word of relative word 0
  const uint32_t r0 = (uint32_t)(bit0 & 31);  // relative bit of the range's first code
  const uint32_t rend = r0 + (uint32_t)(bit1 - bit0);
  uint32_t tile_base = r0;  // relative bit where the current tile starts
  uint32_t wdone = 0;       // first relative word not yet written out
  uint4 np, nq;
  load_exps<DT>(in, tid * kEncPerThread, cnt, np, nq);
  for (uint32_t t0 = 0; t0 < cnt; t0 += kEncTile) {
    const uint32_t idx = t0 + tid * kEncPerThread;
    const uint4 p = np, q = nq;
    if (t0 + kEncTile < cnt) load_exps<DT>(in, idx + kEncTile, cnt, np, nq);
    if (smo && idx < cnt) store_sm<DT>(smo, idx, cnt, p, q);
    // two groups of 8 codes, each concatenated in a 64-bit accumulator
    // (hi:lo) when it fits (all but pathological codes); longer groups take
    // the per-code path
    uint32_t hi[2] = {0u, 0u}, lo[2] = {0u, 0u}, tot[2] = {0u, 0u};
    if (idx + kEncPerThread <= cnt) {
      #pragma unroll
      for (int j = 0; j < kEncPerThread; j++) {
        const uint2 cl = code_of<DT>(tab, p, q, j);
        hi[j >> 3] = __funnelshift_lc(lo[j >> 3], hi[j >> 3], cl.y);
        lo[j >> 3] = __funnelshift_lc(cl.x, lo[j >> 3], cl.y);
        tot[j >> 3] += cl.y;
      }
    } else {
      #pragma unroll
      for (int j = 0; j < kEncPerThread; j++) {
        uint2 cl = code_of<DT>(tab, p, q, j);
        if (idx + j >= cnt) cl = make_uint2(0u, 0u);
        hi[j >> 3] = __funnelshift_lc(lo[j >> 3], hi[j >> 3], cl.y);
        lo[j >> 3] = __funnelshift_lc(cl.x, lo[j >> 3], cl.y);
        tot[j >> 3] += cl.y;
      }
    }
    uint32_t total;
    const uint32_t excl = block_excl_scan1<NT>(tot[0] + tot[1], wsum, &total);
    uint32_t pos = tile_base + excl;
    // value index: where every kIndexStride-th value's code starts, from the
    // range's first bit
    if (kIndex && (idx % kIndexStride) == 0 && idx < cnt) vindex[idx / kIndexStride] = pos - r0;
    #pragma unroll
    for (int h = 0; h < 2; h++) {
      if (tot[h] == 0) continue;
      if (tot[h] <= 64) {
        ring_or64<NT>(ring, pos, hi[h], lo[h], tot[h]);
      } else {
        uint32_t pp = pos;
        for (int j = 8 * h; j < 8 * h + 8; j++) {
          uint2 cl = code_of<DT>(tab, p, q, j);
          if (idx + j >= cnt || cl.y == 0) continue;
          ring_or<NT>(ring, pp, cl.x >> (32 - cl.y), cl.y);
          pp += cl.y;
        }
      }
      pos += tot[h];
    }
    __syncthreads();
    tile_base += total;
    const bool last = t0 + kEncTile >= cnt;
    const uint32_t wend = last ? (rend + 31) >> 5 : tile_base >> 5;
    for (uint32_t wi = wdone + tid; wi < wend; wi += NT) {
      const uint32_t slot = wi & kRingMask;
      const uint32_t val = bswap32(ring[slot]);
      ring[slot] = 0u;
      // the first and last words may hold bits of the neighbouring ranges
      const bool edge = !exclusive && ((wi == 0 && r0 != 0) || ((wi + 1) << 5) > rend);
      if (edge) atomicOr(gs + gw0 + wi, val);
      else gs[gw0 + wi] = val;
    }
    wdone = wend;
  }
}

template <int DT>
__device__ __forceinline__ void load_code_table(uint2 *tab, const uint8_t *code_len, const uint32_t *code) {
  constexpr int A = DT == EH_FP8_E4M3 ? 16 : 256;
  for (int s2 = threadIdx.x; s2 < A; s2 += blockDim.x) {
    const uint32_t l = code_len[s2];
    tab[s2] = make_uint2(l ? code[s2] << (32 - l) : 0u, l);
  }
}

// kIndex: some tensor of the call has a value index (a separate kernel, so
// that the common case's encoding loop has no index code).
template <int DT, int NT, bool kIndex>
__global__ void __launch_bounds__(NT, Enc<NT>::kMinBlocks) encode_kernel(const __grid_constant__ Batch b) {
  constexpr int A = DT == EH_FP8_E4M3 ? 16 : 256;
  extern __shared__ uint32_t ring[];  // Enc<NT>::kRingWords words, code bits in MSB-first order
  __shared__ uint2 tab[A];            // (code left-aligned in 32 bits, length)
  __shared__ uint32_t wsum[NT / 32];
  const uint32_t g = blockIdx.x;
  const Item &I = b.item[find_item(b, g)];
  const uint32_t c = g - I.chunk0;
  const uint64_t i0 = (uint64_t)c * b.chunk_elems;
  const uint32_t cnt = (uint32_t)min((uint64_t)b.chunk_elems, I.n - i0);
  for (int i = threadIdx.x; i < Enc<NT>::kRingWords; i += NT) ring[i] = 0u;
  pdl_wait();  // the codebook and the chunk offsets
  load_code_table<DT>(tab, I.code_len, I.code);
  const uint8_t *in = (const uint8_t *)I.in + i0 * (DT == EH_BF16 ? 2 : 1);
  __syncthreads();
  uint8_t *smo = DT == EH_BF16 ? I.sm + i0 : (DT == EH_FP8_E4M3 ? I.sm + i0 / 2 : nullptr);
  if (!kIndex || !I.vindex) {
    encode_range<DT, NT>(tab, in, cnt, I.off[c], I.off[c + 1], (uint32_t *)I.stream, ring, wsum, false, nullptr, smo);
    return;
  }
  uint32_t *vindex = I.vindex + (uint64_t)c * (b.chunk_elems / kIndexStride);
  encode_range<DT, NT, true>(tab, in, cnt, I.off[c], I.off[c + 1], (uint32_t *)I.stream, ring, wsum, false, vindex,
                             smo);
  {
    // entries past a short last chunk's end: the chunk's bit count
    const uint32_t bits = (uint32_t)(I.off[c + 1] - I.off[c]);
    for (uint32_t k = (cnt + kIndexStride - 1) / kIndexStride + threadIdx.x; k < b.chunk_elems / kIndexStride;
         k += NT)
      vindex[k] = bits;
  }
}

// ---------------------------------------------------------------- pages
// One CTA per appended K/V page: code bits of the page with the frozen
// codebook (and its sign/mantissa array), then either the codes into the
// page's own slot (every word of the slot belongs to the page) or, when they
// do not fit or an exponent has no code, the exponent bytes into the next
// free page of the raw pool.
template <int DT>
__global__ void __launch_bounds__(kThreads, 2) page_append_kernel(const __grid_constant__ PageLaunch pl) {
  constexpr int A = DT == EH_FP8_E4M3 ? 16 : 256;
  extern __shared__ uint32_t ring[];
  __shared__ uint2 tab[A];
  __shared__ uint32_t wsum[kThreads / 32];
  __shared__ uint32_t raw_idx;
  const int tid = threadIdx.x;
  const uint32_t pg = blockIdx.x;
  const uint32_t slot = pl.slot_ids[pg];
  if (slot >= pl.n_slots) {
    if (tid == 0) set_status(pl.status, kFlagCorrupt);
    return;
  }
  const uint32_t n = pl.page_elems;
  const uint8_t *in = (const uint8_t *)pl.in + (uint64_t)pg * n * (DT == EH_BF16 ? 2 : 1);
  const uint64_t sm_page = DT == EH_BF16 ? n : (DT == EH_FP8_E4M3 ? n / 2 : 0);
  uint8_t *smo = pl.sm + (uint64_t)slot * sm_page;
  load_code_table<DT>(tab, pl.code_len, pl.code);
  for (int i = tid; i < Enc<kThreads>::kRingWords; i += kThreads) ring[i] = 0u;
  __syncthreads();

  // pass 1: code bits, missing codes, sign/mantissa
  uint32_t bits = 0, missing = 0;
  for (uint32_t idx = tid * kEncPerThread; idx < n; idx += Enc<kThreads>::kTile) {
    uint4 p, q;
    load_exps<DT>(in, idx, n, p, q);
    #pragma unroll
    for (int j = 0; j < kEncPerThread; j++) {
      const uint32_t l = tab[exp_of<DT>(p, q, j)].y;
      bits += l;
      missing |= l == 0;
    }
    if (DT == EH_BF16) {
      const uint32_t w[8] = {p.x, p.y, p.z, p.w, q.x, q.y, q.z, q.w};
      uint32_t o[4];
      #pragma unroll
      for (int j = 0; j < 4; j++) o[j] = bf16x2_sm(w[2 * j]) | (bf16x2_sm(w[2 * j + 1]) << 16);
      *(uint4 *)(smo + idx) = make_uint4(o[0], o[1], o[2], o[3]);
    } else if (DT == EH_FP8_E4M3) {
      const uint32_t w[4] = {p.x, p.y, p.z, p.w};
      const uint32_t lo = fp8x4_sm(w[0]) | (fp8x4_sm(w[1]) << 16);
      const uint32_t hi = fp8x4_sm(w[2]) | (fp8x4_sm(w[3]) << 16);
      *(uint2 *)(smo + idx / 2) = make_uint2(lo, hi);
    }
  }
  uint32_t total;
  (void)block_excl_scan1<kThreads>(bits, wsum, &total);
  const bool any_missing = __syncthreads_or(missing != 0);
  const bool coded = !any_missing && (total + 7) / 8 + 16 <= pl.slot_bytes;
  if (coded) {
    const uint64_t b0 = (uint64_t)slot * pl.slot_bytes * 8;
    encode_range<DT, kThreads>(tab, in, n, b0, b0 + total, (uint32_t *)pl.slots, ring, wsum, true);
    if (tid == 0) pl.page_meta[slot] = total;
    return;
  }
  if (tid == 0) {
    raw_idx = atomicAdd(pl.raw_used, 1u);
    if (raw_idx >= pl.raw_cap) set_status(pl.status, kFlagNoRoom);
    pl.page_meta[slot] = EH_PAGE_RAW | (raw_idx < pl.raw_cap ? raw_idx : 0x7FFFFFFFu);
  }
  __syncthreads();
  if (raw_idx >= pl.raw_cap) return;
  uint8_t *dst = pl.raw_pool + (uint64_t)raw_idx * n;
  for (uint32_t idx = tid * kEncPerThread; idx < n; idx += Enc<kThreads>::kTile) {
    uint4 p, q;
    load_exps<DT>(in, idx, n, p, q);
    uint32_t o[4];
    #pragma unroll
    for (int w = 0; w < 4; w++) {
      o[w] = 0;
      #pragma unroll
      for (int k = 0; k < 4; k++) o[w] |= exp_of<DT>(p, q, 4 * w + k) << (8 * k);
    }
    *(uint4 *)(dst + idx) = make_uint4(o[0], o[1], o[2], o[3]);
  }
}

// Split append, for calls with few pages: kPageParts CTAs per page.
// Pass 1 (one CTA per part): the part's code bits and missing codes, its
// sign/mantissa bytes, and the clearing of its share of the page's slot.
// Pass 2 (one CTA per part): every part reads its page's part totals, takes
// the same coded/raw decision as the one-CTA kernel, and codes its values at
// its offset in the slot (the words it shares with the neighbouring parts by
// atomic OR into the cleared slot); a raw page is copied by its first part.
constexpr int kPageThreads = 256;
static_assert(kPageThreads == kEncSmall, "the split append's ring is sized like the small encoder's");

template <int DT>
__global__ void __launch_bounds__(kPageThreads) page_bits_kernel(const __grid_constant__ PageLaunch pl) {
  constexpr int A = DT == EH_FP8_E4M3 ? 16 : 256;
  __shared__ uint2 tab[A];
  __shared__ uint32_t wsum[kPageThreads / 32];
  pdl_trigger();
  const int tid = threadIdx.x;
  const uint32_t pg = blockIdx.x / kPageParts, part = blockIdx.x % kPageParts;
  const uint32_t slot = pl.slot_ids[pg];
  if (slot >= pl.n_slots) {
    if (tid == 0 && part == 0) set_status(pl.status, kFlagCorrupt);
    return;
  }
  const uint32_t n = pl.page_elems, pn = n / kPageParts, i0 = part * pn;
  const uint8_t *in = (const uint8_t *)pl.in + ((uint64_t)pg * n + i0) * (DT == EH_BF16 ? 2 : 1);
  const uint64_t sm_page = DT == EH_BF16 ? n : (DT == EH_FP8_E4M3 ? n / 2 : 0);
  uint8_t *smo = pl.sm + (uint64_t)slot * sm_page + (DT == EH_BF16 ? i0 : i0 / 2);
  load_code_table<DT>(tab, pl.code_len, pl.code);
  // this part's share of the slot's words, cleared for the second pass
  {
    uint32_t *sw = (uint32_t *)(pl.slots + (uint64_t)slot * pl.slot_bytes);
    const uint32_t nw = (uint32_t)(pl.slot_bytes / 4), w0 = nw * part / kPageParts, w1 = nw * (part + 1) / kPageParts;
    for (uint32_t w = w0 + tid; w < w1; w += kPageThreads) sw[w] = 0u;
  }
  __syncthreads();
  uint32_t bits = 0, missing = 0;
  for (uint32_t idx = tid * kEncPerThread; idx < pn; idx += kPageThreads * kEncPerThread) {
    uint4 p, q;
    load_exps<DT>(in, idx, pn, p, q);
    #pragma unroll
    for (int j = 0; j < kEncPerThread; j++) {
      const uint32_t l = tab[exp_of<DT>(p, q, j)].y;
      bits += l;
      missing |= l == 0;
    }
    store_sm<DT>(smo, idx, pn, p, q);
  }
  uint32_t total;
  (void)block_excl_scan1<kPageThreads>(bits, wsum, &total);
  const bool any_missing = __syncthreads_or(missing != 0);
  if (tid == 0) pl.part_bits[blockIdx.x] = total | (any_missing ? 0x80000000u : 0u);
}

template <int DT>
__global__ void __launch_bounds__(kPageThreads) page_encode_kernel(const __grid_constant__ PageLaunch pl) {
  constexpr int A = DT == EH_FP8_E4M3 ? 16 : 256;
  extern __shared__ uint32_t ring[];
  __shared__ uint2 tab[A];
  __shared__ uint32_t wsum[kPageThreads / 32];
  __shared__ uint32_t raw_idx;
  const int tid = threadIdx.x;
  const uint32_t pg = blockIdx.x / kPageParts, part = blockIdx.x % kPageParts;
  const uint32_t slot = pl.slot_ids[pg];
  if (slot >= pl.n_slots) return;
  const uint32_t n = pl.page_elems, pn = n / kPageParts, i0 = part * pn;
  load_code_table<DT>(tab, pl.code_len, pl.code);
  for (int i = tid; i < Enc<kPageThreads>::kRingWords; i += kPageThreads) ring[i] = 0u;
  pdl_wait();  // the part totals, the cleared slot
  uint32_t total = 0, before = 0;
  bool missing = false;
  #pragma unroll
  for (uint32_t k = 0; k < kPageParts; k++) {
    const uint32_t v = pl.part_bits[pg * kPageParts + k];
    missing |= (v >> 31) != 0;
    total += v & 0x7FFFFFFFu;
    if (k < part) before += v & 0x7FFFFFFFu;
  }
  const uint32_t mine = pl.part_bits[blockIdx.x] & 0x7FFFFFFFu;
  __syncthreads();
  const uint8_t *page_in = (const uint8_t *)pl.in + (uint64_t)pg * n * (DT == EH_BF16 ? 2 : 1);
  const bool coded = !missing && (total + 7) / 8 + 16 <= pl.slot_bytes;
  if (coded) {
    const uint64_t b0 = (uint64_t)slot * pl.slot_bytes * 8 + before;
    encode_range<DT, kPageThreads>(tab, page_in + (uint64_t)i0 * (DT == EH_BF16 ? 2 : 1), pn, b0, b0 + mine,
                                   (uint32_t *)pl.slots, ring, wsum, false);
    if (tid == 0 && part == 0) pl.page_meta[slot] = total;
    return;
  }
  if (part != 0) return;
  if (tid == 0) {
    raw_idx = atomicAdd(pl.raw_used, 1u);
    if (raw_idx >= pl.raw_cap) set_status(pl.status, kFlagNoRoom);
    pl.page_meta[slot] = EH_PAGE_RAW | (raw_idx < pl.raw_cap ? raw_idx : 0x7FFFFFFFu);
  }
  __syncthreads();
  if (raw_idx >= pl.raw_cap) return;
  uint8_t *dst = pl.raw_pool + (uint64_t)raw_idx * n;
  for (uint32_t idx = tid * kEncPerThread; idx < n; idx += kPageThreads * kEncPerThread) {
    uint4 p, q;
    load_exps<DT>(page_in, idx, n, p, q);
    uint32_t o[4];
    #pragma unroll
    for (int w = 0; w < 4; w++) {
      o[w] = 0;
      #pragma unroll
      for (int k = 0; k < 4; k++) o[w] |= exp_of<DT>(p, q, 4 * w + k) << (8 * k);
    }
    *(uint4 *)(dst + idx) = make_uint4(o[0], o[1], o[2], o[3]);
  }
}

}  // namespace

cudaError_t launch_hist(const Batch &b, cudaStream_t s) {
  if (b.total_chunks == 0) return cudaSuccess;
  if (b.dtype == EH_BF16) hist_kernel<EH_BF16><<<b.total_chunks, kThreads, 0, s>>>(b);
  else if (b.dtype == EH_BYTES) hist_kernel<EH_BYTES><<<b.total_chunks, kThreads, 0, s>>>(b);
  else hist_kernel<EH_FP8_E4M3><<<b.total_chunks, kThreads, 0, s>>>(b);
  return cudaGetLastError();
}

cudaError_t launch_book(const Batch &b, cudaStream_t s) {
  return launch_pdl(book_kernel, dim3(b.k), dim3(256), 0, s, b);
}

cudaError_t launch_offsets(const Batch &b, cudaStream_t s) {
  uint32_t grid = (b.total_chunks + kOffThreads / 32 - 1) / (kOffThreads / 32);
  if (grid == 0) grid = 1;  // the last CTA still writes off[0] = 0 and the bit totals
  return launch_pdl(offsets_kernel, dim3(grid), dim3(kOffThreads), 0, s, b);
}

cudaError_t configure_encode() {
  const int smem = Enc<kThreads>::kRingWords * (int)sizeof(uint32_t);
  const int small = Enc<kEncSmall>::kRingWords * (int)sizeof(uint32_t);
  const int large = Enc<kEncLarge>::kRingWords * (int)sizeof(uint32_t);
  const cudaFuncAttribute dyn = cudaFuncAttributeMaxDynamicSharedMemorySize;
  cudaError_t e = cudaSuccess;
  const void *small_k[] = {(const void *)encode_kernel<EH_BF16, kEncSmall, false>,
                           (const void *)encode_kernel<EH_BYTES, kEncSmall, false>,
                           (const void *)encode_kernel<EH_FP8_E4M3, kEncSmall, false>,
                           (const void *)encode_kernel<EH_BF16, kEncSmall, true>,
                           (const void *)encode_kernel<EH_BYTES, kEncSmall, true>,
                           (const void *)encode_kernel<EH_FP8_E4M3, kEncSmall, true>};
  const void *large_k[] = {(const void *)encode_kernel<EH_BF16, kEncLarge, false>,
                           (const void *)encode_kernel<EH_BYTES, kEncLarge, false>,
                           (const void *)encode_kernel<EH_FP8_E4M3, kEncLarge, false>,
                           (const void *)encode_kernel<EH_BF16, kEncLarge, true>,
                           (const void *)encode_kernel<EH_BYTES, kEncLarge, true>,
                           (const void *)encode_kernel<EH_FP8_E4M3, kEncLarge, true>};
  for (const void *k : small_k)
    if (e == cudaSuccess) e = cudaFuncSetAttribute(k, dyn, small);
  for (const void *k : large_k)
    if (e == cudaSuccess) e = cudaFuncSetAttribute(k, dyn, large);
  if (e != cudaSuccess) return e;
  e = cudaFuncSetAttribute(page_append_kernel<EH_BF16>, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
  if (e != cudaSuccess) return e;
  e = cudaFuncSetAttribute(page_append_kernel<EH_BYTES>, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
  if (e != cudaSuccess) return e;
  e = cudaFuncSetAttribute(page_append_kernel<EH_FP8_E4M3>, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
  if (e == cudaSuccess) e = cudaFuncSetAttribute(page_encode_kernel<EH_BF16>, dyn, small);
  if (e == cudaSuccess) e = cudaFuncSetAttribute(page_encode_kernel<EH_BYTES>, dyn, small);
  if (e == cudaSuccess) e = cudaFuncSetAttribute(page_encode_kernel<EH_FP8_E4M3>, dyn, small);
  return e;
}

cudaError_t launch_page_append(const PageLaunch &pl, cudaStream_t s) {
  if (pl.n_pages == 0) return cudaSuccess;
  if (pl.part_bits) {
    const dim3 grid(pl.n_pages * kPageParts), block(kPageThreads);
    const size_t ring = Enc<kPageThreads>::kRingWords * sizeof(uint32_t);
    if (pl.dtype == EH_BF16) page_bits_kernel<EH_BF16><<<grid, block, 0, s>>>(pl);
    else if (pl.dtype == EH_BYTES) page_bits_kernel<EH_BYTES><<<grid, block, 0, s>>>(pl);
    else page_bits_kernel<EH_FP8_E4M3><<<grid, block, 0, s>>>(pl);
    cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess) return e;
    if (pl.dtype == EH_BF16) return launch_pdl(page_encode_kernel<EH_BF16>, grid, block, ring, s, pl);
    if (pl.dtype == EH_BYTES) return launch_pdl(page_encode_kernel<EH_BYTES>, grid, block, ring, s, pl);
    return launch_pdl(page_encode_kernel<EH_FP8_E4M3>, grid, block, ring, s, pl);
  }
  const size_t smem = Enc<kThreads>::kRingWords * sizeof(uint32_t);
  if (pl.dtype == EH_BF16) page_append_kernel<EH_BF16><<<pl.n_pages, kThreads, smem, s>>>(pl);
  else if (pl.dtype == EH_BYTES) page_append_kernel<EH_BYTES><<<pl.n_pages, kThreads, smem, s>>>(pl);
  else page_append_kernel<EH_FP8_E4M3><<<pl.n_pages, kThreads, smem, s>>>(pl);
  return cudaGetLastError();
}

template <int NT, bool kIndex>
cudaError_t launch_encode_nti(const Batch &b, cudaStream_t s) {
  const size_t smem = Enc<NT>::kRingWords * sizeof(uint32_t);
  const dim3 grid(b.total_chunks), block(NT);
  if (b.dtype == EH_BF16) return launch_pdl(encode_kernel<EH_BF16, NT, kIndex>, grid, block, smem, s, b);
  if (b.dtype == EH_BYTES) return launch_pdl(encode_kernel<EH_BYTES, NT, kIndex>, grid, block, smem, s, b);
  return launch_pdl(encode_kernel<EH_FP8_E4M3, NT, kIndex>, grid, block, smem, s, b);
}

template <int NT>
cudaError_t launch_encode_nt(const Batch &b, cudaStream_t s) {
  bool index = false;
  for (uint32_t i = 0; i < b.k; i++) index |= b.item[i].vindex != nullptr;
  return index ? launch_encode_nti<NT, true>(b, s) : launch_encode_nti<NT, false>(b, s);
}

cudaError_t launch_encode(const Batch &b, cudaStream_t s) {
  if (b.total_chunks == 0) return cudaSuccess;
  int dev = 0, sms = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e == cudaSuccess) e = cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  if (e != cudaSuccess) return e;
  if (b.total_chunks >= (uint32_t)(Enc<kEncSmall>::kMinBlocks * sms)) return launch_encode_nt<kEncSmall>(b, s);
  return launch_encode_nt<kEncLarge>(b, s);
}

}  // namespace eh

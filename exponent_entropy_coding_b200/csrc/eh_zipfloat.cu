// eh_zipfloat.cu -- the ZipFloat comparison codec (BF16), sm_100a.
//
// "ZipFloat: An Ultra-fast and Lossless Floating-Point Compressor for LLM
// Inference Systems": blocks of 2048 values are coded independently (§3.1);
// each block's most frequent exponent MD fixes the dominant range
// [MD - 6, MD + 2) and every exponent is remapped to r = e - (MD - 6)
// (§3.2, Eq. 4); the low three bits of r go to three bit planes of 2048 bits
// and a non-zero high part to a 16-bit <11-bit index, 5-bit value> record
// (§3.3); sign and mantissa stay raw.  Each block's records are placed with
// one atomic reservation, as the page does for weights, so the order of the
// blocks' record ranges depends on scheduling; everything else is
// deterministic.
//
// One warp per block (the page's §3.3: a warp works on 32 rows of the bit
// matrix at a time), eight blocks per CTA of 256 threads.  The block is read
// as eight 256-value slices; in slice c lane l holds values 256c + 8l .. +7,
// so every load and store of a slice is a coalesced 16 bytes per lane, and
// the lane's eight bits of a plane are byte 32c + l of that plane.  Nothing
// but the records' reservation (one atomic per CTA) is shared between warps.
#include <cstring>

#include "eh_internal.cuh"

namespace eh {
namespace {

constexpr uint32_t kZfBlock = 2048;
constexpr uint32_t kZfWarps = 8;              // blocks per CTA
constexpr uint32_t kZfThreads = 32 * kZfWarps;
constexpr uint32_t kZfPlaneBytes = kZfBlock / 8;  // 256
constexpr uint32_t kZfSlices = kZfBlock / 256;    // 8

struct ZfArgs {
  const uint16_t *in;
  uint16_t *out;
  uint64_t n;
  uint64_t blocks;
  uint8_t *sm;
  uint32_t *meta;
  uint32_t *dense;
  uint32_t *sparse_off;
  uint16_t *sparse;
  uint64_t sparse_cap;
  uint32_t *status;   // workspace word 0
  uint32_t *counter;  // workspace word 2: records reserved so far
};

// the eight values [i, i+8) of the tensor as four words (zero past n)
__device__ __forceinline__ uint4 load8(const uint16_t *in, uint64_t i, uint64_t n) {
  if (i + 8 <= n) return __ldg((const uint4 *)(in + i));
  uint32_t w[4] = {0, 0, 0, 0};
  for (int j = 0; j < 8; j++)
    if (i + j < n) w[j / 2] |= (uint32_t)in[i + j] << (16 * (j & 1));
  return make_uint4(w[0], w[1], w[2], w[3]);
}

__device__ __forceinline__ uint32_t half_of(const uint4 &q, int j) {
  const uint32_t w = j < 2 ? q.x : j < 4 ? q.y : j < 6 ? q.z : q.w;
  return (w >> (16 * (j & 1))) & 0xFFFFu;
}

__global__ void __launch_bounds__(kZfThreads, 4) zf_compress_kernel(const __grid_constant__ ZfArgs a) {
  __shared__ uint32_t hist[kZfWarps][256];
  __shared__ __align__(16) uint8_t planes[kZfWarps][3 * kZfPlaneBytes];
  __shared__ uint16_t recs[kZfWarps][kZfBlock];
  __shared__ uint32_t s_nnz[kZfWarps], s_base[kZfWarps];
  const uint32_t lane = threadIdx.x & 31u, warp = threadIdx.x >> 5;
  const uint64_t blk = (uint64_t)blockIdx.x * kZfWarps + warp;
  const bool live = blk < a.blocks;
  const uint64_t i0 = blk * kZfBlock;
  const uint32_t count = live ? (uint32_t)min((uint64_t)kZfBlock, a.n - i0) : 0u;
  // the whole block in registers: all eight loads in flight at once
  uint4 q[kZfSlices];
  #pragma unroll
  for (uint32_t c = 0; c < kZfSlices; c++) q[c] = load8(a.in, i0 + 256 * c + 8 * lane, i0 + count);
  uint32_t *h = hist[warp];
  #pragma unroll
  for (int k = 0; k < 8; k++) h[lane + 32 * k] = 0;
  __syncwarp();

  // §3.2: MD, the most frequent exponent field of the block
  #pragma unroll
  for (uint32_t c = 0; c < kZfSlices; c++) {
    const uint32_t j0 = 256 * c + 8 * lane;
    #pragma unroll
    for (int j = 0; j < 8; j++)
      if (j0 + j < count) atomicAdd(&h[(half_of(q[c], j) >> 7) & 0xFFu], 1u);
  }
  __syncwarp();
  // (count << 8) | (255 - field): the maximum is the most frequent field, the
  // smaller field on ties; l_b = MD - 6
  uint32_t best = 0;
  #pragma unroll
  for (int k = 0; k < 8; k++) best = max(best, (h[8 * lane + k] << 8) | (255u - (8 * lane + k)));
  best = __reduce_max_sync(0xffffffffu, best);
  const uint32_t lb = ((255u - (best & 0xFFu)) + 256u - 6u) & 0xFFu;

  // Eq. 4 remap: plane bytes, raw sign/mantissa bytes, and the records,
  // staged in shared memory in element order until the block's place in
  // `sparse` is known
  uint16_t *rec = recs[warp];
  uint32_t nnz = 0;
  #pragma unroll
  for (uint32_t c = 0; c < kZfSlices; c++) {
    const uint32_t j0 = 256 * c + 8 * lane;
    uint16_t v[8];
    #pragma unroll
    for (int j = 0; j < 8; j++) v[j] = (uint16_t)half_of(q[c], j);
    uint32_t pb0 = 0, pb1 = 0, pb2 = 0, hm = 0, lo = 0, hi = 0;
    #pragma unroll
    for (int j = 0; j < 8; j++) {
      const uint32_t rj = j0 + j < count ? (((v[j] >> 7) & 0xFFu) + 256u - lb) & 0xFFu : 0u;
      pb0 |= (rj & 1u) << j;
      pb1 |= ((rj >> 1) & 1u) << j;
      pb2 |= ((rj >> 2) & 1u) << j;
      hm |= (rj >= 8u ? 1u : 0u) << j;
      const uint32_t sv = ((v[j] >> 8) & 0x80u) | (v[j] & 0x7Fu);
      if (j < 4) lo |= sv << (8 * j);
      else hi |= sv << (8 * (j - 4));
    }
    planes[warp][32 * c + lane] = (uint8_t)pb0;
    planes[warp][kZfPlaneBytes + 32 * c + lane] = (uint8_t)pb1;
    planes[warp][2 * kZfPlaneBytes + 32 * c + lane] = (uint8_t)pb2;
    if (j0 + 8 <= count) {
      *(uint2 *)(a.sm + i0 + j0) = make_uint2(lo, hi);
    } else {
      for (int j = 0; j < 8; j++)
        if (j0 + j < count) a.sm[i0 + j0 + j] = (uint8_t)(((v[j] >> 8) & 0x80u) | (v[j] & 0x7Fu));
    }
    const uint32_t mine = (uint32_t)__popc(hm);
    uint32_t x = mine;
    #pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const uint32_t y = __shfl_up_sync(0xffffffffu, x, o);
      if (lane >= (uint32_t)o) x += y;
    }
    if (hm) {
      uint32_t k = nnz + x - mine;
      #pragma unroll
      for (int j = 0; j < 8; j++) {
        if ((hm >> j) & 1u) {
          const uint32_t rj = (((v[j] >> 7) & 0xFFu) + 256u - lb) & 0xFFu;
          rec[k++] = (uint16_t)(((j0 + j) << 5) | (rj >> 3));
        }
      }
    }
    nnz += __shfl_sync(0xffffffffu, x, 31);
  }
  __syncwarp();
  // the planes: 768 bytes as 48 16-byte stores
  if (live) {
    for (uint32_t t = lane; t < 3 * kZfPlaneBytes / 16; t += 32)
      *(uint4 *)(a.dense + blk * 192 + 4 * t) = *(const uint4 *)(&planes[warp][16 * t]);
  }
  // one reservation for the CTA's blocks, in block order
  if (lane == 0) s_nnz[warp] = live ? nnz : 0u;
  __syncthreads();
  if (threadIdx.x == 0) {
    uint32_t tot = 0;
    for (uint32_t w = 0; w < kZfWarps; w++) tot += s_nnz[w];
    uint32_t base = tot ? atomicAdd(a.counter, tot) : 0u;
    if ((uint64_t)base + tot > a.sparse_cap) set_status(a.status, kFlagNoRoom);
    for (uint32_t w = 0; w < kZfWarps; w++) {
      s_base[w] = s_nnz[w] ? base : 0u;
      base += s_nnz[w];
    }
  }
  __syncthreads();
  if (!live) return;
  const uint64_t base = s_base[warp];
  if (lane == 0) {
    a.meta[blk] = lb | (nnz << 8);
    a.sparse_off[blk] = (uint32_t)base;
  }
  if (base + nnz > a.sparse_cap) return;
  for (uint32_t k = lane; k < nnz; k += 32) a.sparse[base + k] = rec[k];
}

__global__ void __launch_bounds__(kZfThreads, 4) zf_decompress_kernel(const __grid_constant__ ZfArgs a) {
  __shared__ __align__(16) uint8_t high[kZfWarps][kZfBlock];
  __shared__ __align__(16) uint8_t planes[kZfWarps][3 * kZfPlaneBytes];
  const uint32_t lane = threadIdx.x & 31u, warp = threadIdx.x >> 5;
  const uint64_t blk = (uint64_t)blockIdx.x * kZfWarps + warp;
  if (blk >= a.blocks) return;  // warp-uniform; no CTA barrier below
  const uint64_t i0 = blk * kZfBlock;
  const uint32_t count = (uint32_t)min((uint64_t)kZfBlock, a.n - i0);
  const uint32_t meta = a.meta[blk];
  const uint32_t lb = meta & 0xFFu, nnz = meta >> 8;
  const uint64_t off = a.sparse_off[blk];
  if (nnz > count || off + nnz > a.sparse_cap) {
    if (lane == 0) set_status(a.status, kFlagCorrupt);
    return;
  }
  // the block's sign/mantissa bytes: all eight loads in flight at once
  uint2 smv[kZfSlices];
  #pragma unroll
  for (uint32_t c = 0; c < kZfSlices; c++) {
    const uint32_t j0 = 256 * c + 8 * lane;
    smv[c] = j0 + 8 <= count ? __ldg((const uint2 *)(a.sm + i0 + j0)) : make_uint2(0, 0);
  }
  uint8_t *hb = high[warp];
  #pragma unroll
  for (int k = 0; k < 4; k++) *(uint4 *)(hb + 16 * (lane + 32 * k)) = make_uint4(0, 0, 0, 0);
  for (uint32_t t = lane; t < 3 * kZfPlaneBytes / 16; t += 32)
    *(uint4 *)(&planes[warp][16 * t]) = __ldg((const uint4 *)(a.dense + blk * 192 + 4 * t));
  __syncwarp();
  bool bad = false;
  for (uint32_t k = lane; k < nnz; k += 32) {
    const uint32_t rcd = a.sparse[off + k];
    if ((rcd >> 5) < count) hb[rcd >> 5] = (uint8_t)(rcd & 31u);
    else bad = true;
  }
  if (__any_sync(0xffffffffu, bad)) {
    if (lane == 0) set_status(a.status, kFlagCorrupt);
    return;
  }
  __syncwarp();
  #pragma unroll
  for (uint32_t c = 0; c < kZfSlices; c++) {
    const uint32_t j0 = 256 * c + 8 * lane;
    if (j0 >= count) break;
    const uint32_t p0 = planes[warp][32 * c + lane];
    const uint32_t p1 = planes[warp][kZfPlaneBytes + 32 * c + lane];
    const uint32_t p2 = planes[warp][2 * kZfPlaneBytes + 32 * c + lane];
    const uint2 hh = *(const uint2 *)(hb + j0);
    uint32_t e[8];
    #pragma unroll
    for (int j = 0; j < 8; j++) {
      const uint32_t hj = ((j < 4 ? hh.x : hh.y) >> (8 * (j & 3))) & 0xFFu;
      const uint32_t rj = ((p0 >> j) & 1u) | (((p1 >> j) & 1u) << 1) | (((p2 >> j) & 1u) << 2) | (hj << 3);
      e[j] = (rj + lb) & 0xFFu;  // inverse of Eq. 4
    }
    if (j0 + 8 <= count) {
      const uint2 s = smv[c];
      uint32_t o[4];
      #pragma unroll
      for (int q = 0; q < 4; q++) {
        const uint32_t sw = q < 2 ? s.x : s.y;
        const uint32_t s0 = (sw >> (16 * (q & 1))) & 0xFFu, s1 = (sw >> (16 * (q & 1) + 8)) & 0xFFu;
        const uint32_t x0 = ((s0 & 0x80u) << 8) | (e[2 * q] << 7) | (s0 & 0x7Fu);
        const uint32_t x1 = ((s1 & 0x80u) << 8) | (e[2 * q + 1] << 7) | (s1 & 0x7Fu);
        o[q] = x0 | (x1 << 16);
      }
      *(uint4 *)(a.out + i0 + j0) = make_uint4(o[0], o[1], o[2], o[3]);
    } else {
      for (int j = 0; j < 8; j++)
        if (j0 + j < count) {
          const uint32_t sv = a.sm[i0 + j0 + j];
          a.out[i0 + j0 + j] = (uint16_t)(((sv & 0x80u) << 8) | (e[j] << 7) | (sv & 0x7Fu));
        }
    }
  }
}

}  // namespace
}  // namespace eh

using namespace eh;

namespace {

bool zf_args(const eh_zf_t *c, ZfArgs *a, void *workspace, uint64_t workspace_bytes) {
  if (!c || !workspace || workspace_bytes < 256 || ((uintptr_t)workspace & 255u)) return false;
  if (c->n == 0 || c->n >= (1ull << 32)) return c->n == 0;
  const auto al16 = [](const void *p) { return p && ((uintptr_t)p & 15u) == 0; };
  if (!al16(c->sign_mant) || !al16(c->dense) || !c->meta || !c->sparse_off || !c->sparse) return false;
  std::memset(a, 0, sizeof(*a));
  a->n = c->n;
  a->blocks = (c->n + kZfBlock - 1) / kZfBlock;
  a->sm = c->sign_mant;
  a->meta = c->meta;
  a->dense = c->dense;
  a->sparse_off = c->sparse_off;
  a->sparse = c->sparse;
  a->sparse_cap = c->sparse_cap;
  a->status = (uint32_t *)workspace;
  a->counter = (uint32_t *)workspace + 2;
  return true;
}

}  // namespace

extern "C" {

eh_status eh_zf_bound(uint64_t n, uint64_t *blocks, uint64_t *sparse_cap) {
  if (!blocks || !sparse_cap || n >= (1ull << 32)) return EH_ERR_INVALID_ARG;
  *blocks = (n + kZfBlock - 1) / kZfBlock;
  *sparse_cap = n;
  return EH_OK;
}

eh_status eh_zf_compress(const void *in, eh_zf_t *out, void *workspace, uint64_t workspace_bytes, int wait,
                         void *stream) {
  ZfArgs a;
  if (!out || !zf_args(out, &a, workspace, workspace_bytes)) return EH_ERR_INVALID_ARG;
  cudaStream_t s = (cudaStream_t)stream;
  if (cudaMemsetAsync(workspace, 0, 16, s) != cudaSuccess) return EH_ERR_CUDA;
  if (out->n) {
    if (!in || ((uintptr_t)in & 15u)) return EH_ERR_INVALID_ARG;
    a.in = (const uint16_t *)in;
    const uint32_t grid = (uint32_t)((a.blocks + kZfWarps - 1) / kZfWarps);
    zf_compress_kernel<<<grid, kZfThreads, 0, s>>>(a);
    if (cudaGetLastError() != cudaSuccess) return EH_ERR_CUDA;
  }
  if (wait) {
    uint32_t h[3];
    if (cudaMemcpyAsync(h, workspace, 12, cudaMemcpyDeviceToHost, s) != cudaSuccess) return EH_ERR_CUDA;
    if (cudaStreamSynchronize(s) != cudaSuccess) return EH_ERR_CUDA;
    out->n_records = h[2];
    if (h[0] & kFlagNoRoom) return EH_ERR_NOMEM;
  }
  return EH_OK;
}

eh_status eh_zf_decompress(const eh_zf_t *c, void *out, void *workspace, uint64_t workspace_bytes, void *stream) {
  ZfArgs a;
  if (!c || !zf_args(c, &a, workspace, workspace_bytes)) return EH_ERR_INVALID_ARG;
  cudaStream_t s = (cudaStream_t)stream;
  if (cudaMemsetAsync(workspace, 0, 16, s) != cudaSuccess) return EH_ERR_CUDA;
  if (c->n) {
    if (!out || ((uintptr_t)out & 15u)) return EH_ERR_INVALID_ARG;
    a.out = (uint16_t *)out;
    const uint32_t grid = (uint32_t)((a.blocks + kZfWarps - 1) / kZfWarps);
    zf_decompress_kernel<<<grid, kZfThreads, 0, s>>>(a);
    if (cudaGetLastError() != cudaSuccess) return EH_ERR_CUDA;
  }
  return EH_OK;
}

}  // extern "C"

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
// One CTA of 256 threads per block, eight values per thread: the thread's
// eight bits of each plane form one byte of that plane (bit j = element
// 8*tid + j), so the planes are assembled in shared memory byte by byte and
// written with 16-byte stores.
#include <cstring>

#include "eh_internal.cuh"

namespace eh {
namespace {

constexpr uint32_t kZfBlock = 2048;
constexpr uint32_t kZfThreads = 256;
constexpr uint32_t kZfPlaneWords = 64;  // 2048 bits

struct ZfArgs {
  const uint16_t *in;
  uint16_t *out;
  uint64_t n;
  uint8_t *sm;
  uint32_t *meta;
  uint32_t *dense;
  uint32_t *sparse_off;
  uint16_t *sparse;
  uint64_t sparse_cap;
  uint32_t *status;   // workspace word 0
  uint32_t *counter;  // workspace word 2: records reserved so far
};

__device__ __forceinline__ uint32_t block_excl_scan256(uint32_t v, uint32_t *wsum, uint32_t *total) {
  const uint32_t lane = threadIdx.x & 31u, warp = threadIdx.x >> 5;
  uint32_t x = v;
  #pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const uint32_t y = __shfl_up_sync(0xffffffffu, x, o);
    if (lane >= (uint32_t)o) x += y;
  }
  if (lane == 31) wsum[warp] = x;
  __syncthreads();
  if (warp == 0) {
    uint32_t t = lane < kZfThreads / 32 ? wsum[lane] : 0u;
    #pragma unroll
    for (int o = 1; o < 8; o <<= 1) {
      const uint32_t y = __shfl_up_sync(0xffffffffu, t, o);
      if (lane >= (uint32_t)o) t += y;
    }
    if (lane < kZfThreads / 32) wsum[lane] = t;
  }
  __syncthreads();
  *total = wsum[kZfThreads / 32 - 1];
  return (warp ? wsum[warp - 1] : 0u) + x - v;
}

__global__ void __launch_bounds__(kZfThreads) zf_compress_kernel(const __grid_constant__ ZfArgs a) {
  __shared__ uint32_t hist[256];
  __shared__ alignas(16) uint8_t planes[3 * kZfThreads];
  __shared__ uint32_t wsum[kZfThreads / 32];
  __shared__ uint32_t s_lb, s_base;
  const uint32_t tid = threadIdx.x, lane = tid & 31u;
  const uint64_t i0 = (uint64_t)blockIdx.x * kZfBlock;
  const uint32_t count = (uint32_t)min((uint64_t)kZfBlock, a.n - i0);
  const uint32_t j0 = 8 * tid;  // first element of this thread in the block

  hist[tid] = 0;
  uint16_t v[8];
  if (j0 + 8 <= count) {
    const uint4 q = __ldg((const uint4 *)(a.in + i0 + j0));
    const uint32_t w[4] = {q.x, q.y, q.z, q.w};
    #pragma unroll
    for (int j = 0; j < 8; j++) v[j] = (uint16_t)(w[j / 2] >> (16 * (j & 1)));
  } else {
    #pragma unroll
    for (int j = 0; j < 8; j++) v[j] = j0 + j < count ? a.in[i0 + j0 + j] : (uint16_t)0;
  }
  __syncthreads();

  // §3.2: MD, the most frequent exponent field of the block.  Lanes holding
  // the same field add once (warp-aggregated); lanes past the end get a key
  // no field has.
  #pragma unroll
  for (int j = 0; j < 8; j++) {
    const bool ok = j0 + j < count;
    const uint32_t key = ok ? (v[j] >> 7) & 0xFFu : 256u + lane;
    const uint32_t same = __match_any_sync(0xffffffffu, key);
    if (ok && lane == (uint32_t)(__ffs(same) - 1)) atomicAdd(&hist[key], (uint32_t)__popc(same));
  }
  __syncthreads();
  if (tid < 32) {
    // (count << 8) | (255 - field): the maximum is the most frequent field,
    // the smaller field on ties
    uint32_t best = 0;
    #pragma unroll
    for (int k = 0; k < 8; k++) {
      const uint32_t e = tid * 8 + k;
      best = max(best, (hist[e] << 8) | (255u - e));
    }
    best = __reduce_max_sync(0xffffffffu, best);
    if (tid == 0) s_lb = ((255u - (best & 0xFFu)) + 256u - 6u) & 0xFFu;  // l_b = MD - 6
  }
  __syncthreads();
  const uint32_t lb = s_lb;

  // Eq. 4 remap; the low three bits into the planes, high parts counted
  uint32_t pb0 = 0, pb1 = 0, pb2 = 0, hi_mask = 0;
  uint8_t r[8];
  #pragma unroll
  for (int j = 0; j < 8; j++) {
    const uint32_t rj = j0 + j < count ? (((v[j] >> 7) & 0xFFu) + 256u - lb) & 0xFFu : 0u;
    r[j] = (uint8_t)rj;
    pb0 |= (rj & 1u) << j;
    pb1 |= ((rj >> 1) & 1u) << j;
    pb2 |= ((rj >> 2) & 1u) << j;
    hi_mask |= (rj >= 8u ? 1u : 0u) << j;
  }
  planes[tid] = (uint8_t)pb0;
  planes[kZfThreads + tid] = (uint8_t)pb1;
  planes[2 * kZfThreads + tid] = (uint8_t)pb2;

  uint32_t nnz;
  const uint32_t pos = block_excl_scan256((uint32_t)__popc(hi_mask), wsum, &nnz);
  if (tid == 0) {
    const uint32_t base = nnz ? atomicAdd(a.counter, nnz) : 0u;
    s_base = base;
    a.meta[blockIdx.x] = lb | (nnz << 8);
    a.sparse_off[blockIdx.x] = base;
    if ((uint64_t)base + nnz > a.sparse_cap) set_status(a.status, kFlagNoRoom);
  }
  __syncthreads();  // planes complete, base known
  if (tid < 3 * kZfThreads / 16) {
    const uint32_t p = tid / (kZfThreads / 16), q = tid % (kZfThreads / 16);
    *(uint4 *)(a.dense + (uint64_t)blockIdx.x * 3 * kZfPlaneWords + p * kZfPlaneWords + 4 * q) =
        *(const uint4 *)(planes + p * kZfThreads + 16 * q);
  }
  const uint64_t base = s_base;
  if (base + nnz <= a.sparse_cap) {
    uint32_t k = pos;
    #pragma unroll
    for (int j = 0; j < 8; j++)
      if ((hi_mask >> j) & 1u) a.sparse[base + k++] = (uint16_t)(((j0 + j) << 5) | (r[j] >> 3));
  }
  // raw sign and mantissa
  if (j0 + 8 <= count) {
    uint32_t lo = 0, hi = 0;
    #pragma unroll
    for (int j = 0; j < 8; j++) {
      const uint32_t s = ((v[j] >> 8) & 0x80u) | (v[j] & 0x7Fu);
      if (j < 4) lo |= s << (8 * j);
      else hi |= s << (8 * (j - 4));
    }
    *(uint2 *)(a.sm + i0 + j0) = make_uint2(lo, hi);
  } else {
    for (int j = 0; j < 8; j++)
      if (j0 + j < count) a.sm[i0 + j0 + j] = (uint8_t)(((v[j] >> 8) & 0x80u) | (v[j] & 0x7Fu));
  }
}

__global__ void __launch_bounds__(kZfThreads) zf_decompress_kernel(const __grid_constant__ ZfArgs a) {
  __shared__ alignas(16) uint8_t high[kZfBlock];
  __shared__ alignas(16) uint8_t planes[3 * kZfThreads];
  __shared__ uint32_t s_bad;
  const uint32_t tid = threadIdx.x;
  const uint64_t i0 = (uint64_t)blockIdx.x * kZfBlock;
  const uint32_t count = (uint32_t)min((uint64_t)kZfBlock, a.n - i0);
  const uint32_t j0 = 8 * tid;
  const uint32_t meta = a.meta[blockIdx.x];
  const uint32_t lb = meta & 0xFFu, nnz = meta >> 8;
  const uint64_t off = a.sparse_off[blockIdx.x];
  if (nnz > count || off + nnz > a.sparse_cap) {  // uniform over the CTA
    if (tid == 0) set_status(a.status, kFlagCorrupt);
    return;
  }
  if (tid == 0) s_bad = 0;
  *(uint2 *)(high + j0) = make_uint2(0, 0);
  if (tid < 3 * kZfThreads / 16) {
    const uint32_t p = tid / (kZfThreads / 16), q = tid % (kZfThreads / 16);
    *(uint4 *)(planes + p * kZfThreads + 16 * q) =
        __ldg((const uint4 *)(a.dense + (uint64_t)blockIdx.x * 3 * kZfPlaneWords + p * kZfPlaneWords + 4 * q));
  }
  __syncthreads();
  for (uint32_t k = tid; k < nnz; k += kZfThreads) {
    const uint32_t rcd = a.sparse[off + k];
    if ((rcd >> 5) < count) high[rcd >> 5] = (uint8_t)(rcd & 31u);
    else s_bad = 1;
  }
  __syncthreads();
  if (s_bad) {
    if (tid == 0) set_status(a.status, kFlagCorrupt);
    return;
  }
  const uint32_t p0 = planes[tid], p1 = planes[kZfThreads + tid], p2 = planes[2 * kZfThreads + tid];
  const uint2 h = *(const uint2 *)(high + j0);
  uint32_t e[8];
  #pragma unroll
  for (int j = 0; j < 8; j++) {
    const uint32_t hj = ((j < 4 ? h.x : h.y) >> (8 * (j & 3))) & 0xFFu;
    const uint32_t rj = ((p0 >> j) & 1u) | (((p1 >> j) & 1u) << 1) | (((p2 >> j) & 1u) << 2) | (hj << 3);
    e[j] = (rj + lb) & 0xFFu;  // inverse of Eq. 4
  }
  if (j0 + 8 <= count) {
    const uint2 s = __ldg((const uint2 *)(a.sm + i0 + j0));
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
        const uint32_t s = a.sm[i0 + j0 + j];
        a.out[i0 + j0 + j] = (uint16_t)(((s & 0x80u) << 8) | (e[j] << 7) | (s & 0x7Fu));
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
    const uint32_t B = (uint32_t)((out->n + kZfBlock - 1) / kZfBlock);
    zf_compress_kernel<<<B, kZfThreads, 0, s>>>(a);
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
    const uint32_t B = (uint32_t)((c->n + kZfBlock - 1) / kZfBlock);
    zf_decompress_kernel<<<B, kZfThreads, 0, s>>>(a);
    if (cudaGetLastError() != cudaSuccess) return EH_ERR_CUDA;
  }
  return EH_OK;
}

}  // extern "C"

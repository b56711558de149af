// eh_api.cu -- the C ABI of libexphuff (include/exphuff.h): argument checks,
// workspace layout, kernel launches and status mapping.  No allocation happens
// here: every buffer, the workspace included, belongs to the caller.
#include <atomic>
#include <cstring>
#include <mutex>

#include "eh_internal.cuh"

using namespace eh;

namespace {

constexpr int kMaxDevices = 64;

// Fix-up round limit handed to the decoder (0: its default); set only by the
// test hook eh_debug_set_fixup_rounds.
std::atomic<uint32_t> g_fixup_rounds{0};

struct DeviceInfo {
  std::once_flag once;
  int num_sms = 0;
  cudaError_t err = cudaSuccess;
};
DeviceInfo g_dev[kMaxDevices];

// SM count of the current device; configures the kernels once per device.
cudaError_t device_setup(int *num_sms) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  if (dev < 0 || dev >= kMaxDevices) return cudaErrorInvalidDevice;
  DeviceInfo &d = g_dev[dev];
  std::call_once(d.once, [&d, dev]() {
    d.err = cudaDeviceGetAttribute(&d.num_sms, cudaDevAttrMultiProcessorCount, dev);
    if (d.err == cudaSuccess) d.err = configure_decode();
    if (d.err == cudaSuccess) d.err = configure_encode();
  });
  *num_sms = d.num_sms;
  return d.err;
}

inline bool aligned16(const void *p) { return ((uintptr_t)p & 15u) == 0; }
inline uint64_t ceil_div(uint64_t a, uint64_t b) { return (a + b - 1) / b; }

bool plan_ok(const eh_plan_t *p) {
  return p && (p->dtype == EH_BF16 || p->dtype == EH_FP8_E4M3 || p->dtype == EH_BYTES) && p->chunk_elems >= 1024 &&
         p->chunk_elems <= (uint32_t)kMaxChunk && p->chunk_elems % 1024 == 0 && p->max_code_len >= 1 &&
         p->max_code_len <= EH_MAX_CODE_LEN;
}

uint64_t stream_cap_for(const eh_plan_t *p, uint64_t n) {
  return ((ceil_div(n * p->max_code_len, 8) + 15) & ~uint64_t(15)) + 16;
}

uint64_t sm_bytes_for(int dtype, uint64_t n) {
  if (dtype == EH_BYTES) return 0;
  return dtype == EH_BF16 ? n : ceil_div(n, 2);
}

// ---- compress workspace layout
//   [0, 256)                 status (u32), ticket (u32), bit totals u64[k]
//   [256, 256 + 2048k)       per-tensor exponent counts u64[256]
//   then per tensor, each 256-aligned: package-merge scratch u64[33][256],
//   per-chunk histograms u32[C][A], per-chunk bits u64[C]
constexpr uint64_t kHeader = 256;
constexpr uint64_t kCountsBytes = 256 * sizeof(uint64_t);
constexpr uint64_t kPmBytes = 33 * 256 * sizeof(uint64_t);

uint64_t compress_ws_bytes(const eh_plan_t *p, int k, const uint64_t *ns) {
  uint64_t total = align256(kHeader + (uint64_t)k * kCountsBytes);
  const uint64_t A = alphabet_of(p->dtype);
  for (int i = 0; i < k; i++) {
    const uint64_t C = ceil_div(ns[i], p->chunk_elems);
    total += align256(kPmBytes) + align256(C * A * 4) + align256(C * 8);
  }
  return total;
}

}  // namespace

extern "C" {

const char *eh_version(void) { return "libexphuff 0.1 sm_100a"; }

const char *eh_status_str(eh_status s) {
  switch (s) {
    case EH_OK: return "ok";
    case EH_ERR_INVALID_ARG: return "invalid argument";
    case EH_ERR_UNSUPPORTED: return "unsupported dtype, chunk size or code length limit";
    case EH_ERR_INFEASIBLE: return "more distinct exponents than the code length limit allows";
    case EH_ERR_CUDA: return "CUDA runtime error";
    case EH_ERR_CORRUPT: return "corrupt compressed data or codebook";
    case EH_ERR_TIMEOUT: return "a bounded wait in a kernel gave up";
    case EH_ERR_NOMEM: return "workspace too small";
  }
  return "unknown status";
}

eh_status eh_plan(eh_plan_t *plan, int32_t dtype, uint32_t chunk_elems, uint32_t max_code_len) {
  if (!plan) return EH_ERR_INVALID_ARG;
  eh_plan_t p;
  p.dtype = dtype;
  p.chunk_elems = chunk_elems ? chunk_elems : EH_DEFAULT_CHUNK_ELEMS;
  p.max_code_len = max_code_len ? max_code_len : EH_MAX_CODE_LEN;
  p.reserved = 0;
  if (!plan_ok(&p)) return EH_ERR_UNSUPPORTED;
  *plan = p;
  return EH_OK;
}

eh_status eh_compress_bound(const eh_plan_t *plan, uint64_t n, uint64_t *stream_cap, uint64_t *sm_bytes,
                            uint64_t *workspace_bytes) {
  if (!plan_ok(plan)) return EH_ERR_INVALID_ARG;
  if (n > (1ull << 40)) return EH_ERR_INVALID_ARG;
  if (stream_cap) *stream_cap = stream_cap_for(plan, n);
  if (sm_bytes) *sm_bytes = sm_bytes_for(plan->dtype, n);
  if (workspace_bytes) *workspace_bytes = compress_ws_bytes(plan, 1, &n);
  return EH_OK;
}

eh_status eh_compress_batch_workspace(const eh_plan_t *plan, int k, const uint64_t *ns,
                                      uint64_t *workspace_bytes) {
  if (!plan_ok(plan) || k < 1 || k > EH_MAX_BATCH || !ns || !workspace_bytes) return EH_ERR_INVALID_ARG;
  *workspace_bytes = compress_ws_bytes(plan, k, ns);
  return EH_OK;
}

}  // extern "C"

namespace {

// Checks the arguments of a compress call and lays out its launch
// descriptor and workspace.
eh_status prepare_compress(const eh_plan_t *plan, int k, const void *const *ins, eh_compressed_t *outs,
                           uint64_t *bits_dev, void *workspace, uint64_t workspace_bytes, Batch *bp) {
  if (!plan_ok(plan) || k < 1 || k > EH_MAX_BATCH || !ins || !outs || !workspace) return EH_ERR_INVALID_ARG;
  if (((uintptr_t)workspace & 255u) != 0 || (bits_dev && ((uintptr_t)bits_dev & 7u))) return EH_ERR_INVALID_ARG;
  uint64_t ns[EH_MAX_BATCH];
  uint64_t total_chunks = 0;
  for (int i = 0; i < k; i++) {
    const eh_compressed_t &o = outs[i];
    const uint64_t n = o.n;
    if (o.dtype != plan->dtype || n > (1ull << 40)) return EH_ERR_INVALID_ARG;
    if (!o.code_len || !o.code || !o.chunk_bit_off) return EH_ERR_INVALID_ARG;
    if (((uintptr_t)o.code & 3u) || ((uintptr_t)o.chunk_bit_off & 7u) || ((uintptr_t)o.value_index & 3u))
      return EH_ERR_INVALID_ARG;
    const bool has_sm = plan->dtype != EH_BYTES;
    if (n > 0 && (!ins[i] || !o.exp_stream || (has_sm && !o.sign_mant))) return EH_ERR_INVALID_ARG;
    if (n > 0 && (!aligned16(ins[i]) || !aligned16(o.exp_stream) || (has_sm && !aligned16(o.sign_mant))))
      return EH_ERR_INVALID_ARG;
    if (o.exp_stream_cap < stream_cap_for(plan, n) && n > 0) return EH_ERR_INVALID_ARG;
    ns[i] = n;
    total_chunks += ceil_div(n, plan->chunk_elems);
  }
  if (total_chunks > 0x7FFFFFFFull) return EH_ERR_INVALID_ARG;
  if (workspace_bytes < compress_ws_bytes(plan, k, ns)) return EH_ERR_NOMEM;

  uint8_t *ws = (uint8_t *)workspace;
  Batch &b = *bp;
  std::memset(&b, 0, sizeof(b));
  b.k = (uint32_t)k;
  b.chunk_elems = plan->chunk_elems;
  b.dtype = plan->dtype;
  b.max_code_len = plan->max_code_len;
  b.status = (uint32_t *)ws;
  b.ticket = (uint32_t *)(ws + 4);
  uint64_t *bits_ws = (uint64_t *)(ws + 8);
  const uint64_t A = alphabet_of(plan->dtype);
  uint64_t cursor = align256(kHeader + (uint64_t)k * kCountsBytes);
  uint32_t chunk0 = 0;
  for (int i = 0; i < k; i++) {
    Item &it = b.item[i];
    const eh_compressed_t &o = outs[i];
    const uint32_t C = (uint32_t)ceil_div(o.n, plan->chunk_elems);
    it.in = ins[i];
    it.n = o.n;
    it.chunk0 = chunk0;
    it.nchunks = C;
    it.first_chunk = 0;
    it.total_chunks = C;
    it.code_len = o.code_len;
    it.code = o.code;
    it.off = o.chunk_bit_off;
    it.stream = o.exp_stream;
    it.stream_cap = o.exp_stream_cap;
    it.sm = o.sign_mant;
    it.vindex = o.value_index;
    it.counts = (uint64_t *)(ws + kHeader + (uint64_t)i * kCountsBytes);
    it.bits_out = bits_ws + i;
    it.bits_dev = bits_dev ? bits_dev + i : nullptr;
    it.pm_scratch = (uint64_t *)(ws + cursor);
    cursor += align256(kPmBytes);
    it.chist = (uint32_t *)(ws + cursor);
    cursor += align256((uint64_t)C * A * 4);
    it.cbits = (uint64_t *)(ws + cursor);
    cursor += align256((uint64_t)C * 8);
    chunk0 += C;
  }
  b.total_chunks = chunk0;
  for (int i = 0; i < k; i++) outs[i].n_chunks = b.item[i].nchunks;
  return EH_OK;
}

// Codebook, offsets and encode launches, then (without bits_dev) the wait
// for the bit counts and the status.
eh_status finish_compress(const Batch &b, int k, eh_compressed_t *outs, bool wait, void *workspace,
                          cudaStream_t s) {
  if (launch_book(b, s) != cudaSuccess) return EH_ERR_CUDA;
  if (launch_offsets(b, s) != cudaSuccess) return EH_ERR_CUDA;
  if (launch_encode(b, s) != cudaSuccess) return EH_ERR_CUDA;
  if (!wait) return EH_OK;
  uint64_t host[1 + EH_MAX_BATCH];
  if (cudaMemcpyAsync(host, workspace, 8 + 8 * (uint64_t)k, cudaMemcpyDeviceToHost, s) != cudaSuccess)
    return EH_ERR_CUDA;
  if (cudaStreamSynchronize(s) != cudaSuccess) return EH_ERR_CUDA;
  const uint32_t status = (uint32_t)host[0];
  for (int i = 0; i < k; i++) outs[i].exp_stream_bits = host[1 + i];
  if (status & kFlagInfeasible) return EH_ERR_INFEASIBLE;
  if (status & kFlagTimeout) return EH_ERR_TIMEOUT;
  if (status & kFlagCorrupt) return EH_ERR_CORRUPT;
  return EH_OK;
}

}  // namespace

extern "C" {

eh_status eh_compress_batch(const eh_plan_t *plan, int k, const void *const *ins, eh_compressed_t *outs,
                            uint64_t *bits_dev, void *workspace, uint64_t workspace_bytes, void *stream) {
  Batch b;
  eh_status st = prepare_compress(plan, k, ins, outs, bits_dev, workspace, workspace_bytes, &b);
  if (st != EH_OK) return st;
  int num_sms = 0;
  if (device_setup(&num_sms) != cudaSuccess) return EH_ERR_CUDA;
  cudaStream_t s = (cudaStream_t)stream;
  if (cudaMemsetAsync(workspace, 0, kHeader + (uint64_t)k * kCountsBytes, s) != cudaSuccess) return EH_ERR_CUDA;
  if (launch_hist(b, s) != cudaSuccess) return EH_ERR_CUDA;
  return finish_compress(b, k, outs, bits_dev == nullptr, workspace, s);
}

eh_status eh_compress_shard_begin(const eh_plan_t *plan, const void *in, eh_compressed_t *out, uint64_t *counts,
                                  void *workspace, uint64_t workspace_bytes, void *stream) {
  if (!counts || ((uintptr_t)counts & 7u)) return EH_ERR_INVALID_ARG;
  const void *ins[1] = {in};
  Batch b;
  eh_status st = prepare_compress(plan, 1, ins, out, nullptr, workspace, workspace_bytes, &b);
  if (st != EH_OK) return st;
  b.item[0].counts = counts;
  int num_sms = 0;
  if (device_setup(&num_sms) != cudaSuccess) return EH_ERR_CUDA;
  cudaStream_t s = (cudaStream_t)stream;
  if (cudaMemsetAsync(workspace, 0, kHeader, s) != cudaSuccess) return EH_ERR_CUDA;
  if (cudaMemsetAsync(counts, 0, sizeof(uint64_t) * alphabet_of(plan->dtype), s) != cudaSuccess) return EH_ERR_CUDA;
  if (launch_hist(b, s) != cudaSuccess) return EH_ERR_CUDA;
  return EH_OK;
}

eh_status eh_compress_shard_finish(const eh_plan_t *plan, const void *in, eh_compressed_t *out,
                                   const uint64_t *counts, uint64_t *bits_dev, void *workspace,
                                   uint64_t workspace_bytes, void *stream) {
  if (!counts || ((uintptr_t)counts & 7u)) return EH_ERR_INVALID_ARG;
  const void *ins[1] = {in};
  Batch b;
  eh_status st = prepare_compress(plan, 1, ins, out, bits_dev, workspace, workspace_bytes, &b);
  if (st != EH_OK) return st;
  b.item[0].counts = const_cast<uint64_t *>(counts);
  int num_sms = 0;
  if (device_setup(&num_sms) != cudaSuccess) return EH_ERR_CUDA;
  return finish_compress(b, 1, out, bits_dev == nullptr, workspace, (cudaStream_t)stream);
}

eh_status eh_compress(const eh_plan_t *plan, const void *in, uint64_t n, eh_compressed_t *out, void *workspace,
                      uint64_t workspace_bytes, void *stream) {
  if (!out) return EH_ERR_INVALID_ARG;
  if (out->n != n) return EH_ERR_INVALID_ARG;
  const void *ins[1] = {in};
  return eh_compress_batch(plan, 1, ins, out, nullptr, workspace, workspace_bytes, stream);
}

eh_status eh_decompress_workspace(const eh_plan_t *plan, int k, uint64_t *workspace_bytes) {
  if (!plan_ok(plan) || k < 1 || k > EH_MAX_BATCH || !workspace_bytes) return EH_ERR_INVALID_ARG;
  *workspace_bytes = kHeader + (uint64_t)k * kLutBytes;
  return EH_OK;
}

}  // extern "C"

// Shared by the decompression entry points and the prefetcher.
eh_status eh::decompress_impl(const eh_plan_t *plan, int k, const eh_compressed_t *cs, void *const *outs,
                          const uint32_t *firsts, const uint32_t *counts, void *workspace,
                          uint64_t workspace_bytes, void *stream, uint32_t max_ctas) {
  if (!plan_ok(plan) || k < 1 || k > EH_MAX_BATCH || !cs || !outs || !workspace) return EH_ERR_INVALID_ARG;
  if (((uintptr_t)workspace & 255u) != 0) return EH_ERR_INVALID_ARG;
  if (workspace_bytes < kHeader + (uint64_t)k * kLutBytes) return EH_ERR_NOMEM;
  uint8_t *ws = (uint8_t *)workspace;
  Batch b;
  std::memset(&b, 0, sizeof(b));
  b.k = (uint32_t)k;
  b.chunk_elems = plan->chunk_elems;
  b.dtype = plan->dtype;
  b.max_code_len = plan->max_code_len;
  b.status = (uint32_t *)ws;
  b.ticket = (uint32_t *)(ws + 4);
  uint64_t chunk0 = 0;
  for (int i = 0; i < k; i++) {
    const eh_compressed_t &c = cs[i];
    if (c.dtype != plan->dtype || c.n > (1ull << 40)) return EH_ERR_INVALID_ARG;
    const uint64_t C = ceil_div(c.n, plan->chunk_elems);
    if (c.n_chunks != C) return EH_ERR_INVALID_ARG;
    const uint32_t first = firsts ? firsts[i] : 0u;
    const uint32_t count = counts ? counts[i] : (uint32_t)C;
    if ((uint64_t)first + count > C) return EH_ERR_INVALID_ARG;
    if (!c.code_len || !c.code || !c.chunk_bit_off || ((uintptr_t)c.chunk_bit_off & 7u) ||
        ((uintptr_t)c.value_index & 3u))
      return EH_ERR_INVALID_ARG;
    if (count > 0) {
      const bool has_sm = plan->dtype != EH_BYTES;
      if (!outs[i] || !c.exp_stream || (has_sm && !c.sign_mant)) return EH_ERR_INVALID_ARG;
      if (!aligned16(outs[i]) || !aligned16(c.exp_stream) || (has_sm && !aligned16(c.sign_mant)))
        return EH_ERR_INVALID_ARG;
    }
    Item &it = b.item[i];
    it.out = outs[i];
    it.n = c.n;
    it.elem0 = (uint64_t)first * plan->chunk_elems;
    it.chunk0 = (uint32_t)chunk0;
    it.nchunks = count;
    it.first_chunk = first;
    it.total_chunks = (uint32_t)C;
    it.code_len = c.code_len;
    it.code = c.code;
    it.off = c.chunk_bit_off;
    it.stream = c.exp_stream;
    it.stream_cap = c.exp_stream_cap;
    it.sm = c.sign_mant;
    it.vindex = c.value_index;
    it.lut = ws + kHeader + (uint64_t)i * kLutBytes;
    chunk0 += count;
  }
  if (chunk0 > 0x7FFFFFFFull) return EH_ERR_INVALID_ARG;
  b.total_chunks = (uint32_t)chunk0;
  b.fixup_rounds = g_fixup_rounds.load(std::memory_order_relaxed);
  int num_sms = 0;
  if (device_setup(&num_sms) != cudaSuccess) return EH_ERR_CUDA;
  cudaStream_t s = (cudaStream_t)stream;
  if (max_ctas && max_ctas < (uint32_t)num_sms) num_sms = (int)max_ctas;
  if (launch_tables(b, s) != cudaSuccess) return EH_ERR_CUDA;
  if (launch_decode(b, s, num_sms) != cudaSuccess) return EH_ERR_CUDA;
  return EH_OK;
}

extern "C" {

eh_status eh_decompress(const eh_plan_t *plan, const eh_compressed_t *c, void *out, void *workspace,
                        uint64_t workspace_bytes, void *stream) {
  void *outs[1] = {out};
  return decompress_impl(plan, 1, c, outs, nullptr, nullptr, workspace, workspace_bytes, stream, 0);
}

eh_status eh_decompress_batch(const eh_plan_t *plan, int k, const eh_compressed_t *cs, void *const *outs,
                              void *workspace, uint64_t workspace_bytes, void *stream) {
  return decompress_impl(plan, k, cs, outs, nullptr, nullptr, workspace, workspace_bytes, stream, 0);
}

eh_status eh_decompress_chunks(const eh_plan_t *plan, const eh_compressed_t *c, uint32_t first, uint32_t count,
                               void *out, void *workspace, uint64_t workspace_bytes, void *stream) {
  void *outs[1] = {out};
  return decompress_impl(plan, 1, c, outs, &first, &count, workspace, workspace_bytes, stream, 0);
}

eh_status eh_codebook_from_counts(const eh_plan_t *plan, const uint64_t *counts, uint8_t *code_len, uint32_t *code,
                                  void *workspace, uint64_t workspace_bytes, void *stream) {
  if (!plan_ok(plan) || !counts || !code_len || !code || !workspace) return EH_ERR_INVALID_ARG;
  if (((uintptr_t)workspace & 255u) || ((uintptr_t)counts & 7u) || ((uintptr_t)code & 3u)) return EH_ERR_INVALID_ARG;
  const uint64_t zero = 0;
  if (workspace_bytes < compress_ws_bytes(plan, 1, &zero)) return EH_ERR_NOMEM;
  int num_sms = 0;
  if (device_setup(&num_sms) != cudaSuccess) return EH_ERR_CUDA;
  uint8_t *ws = (uint8_t *)workspace;
  Batch b;
  std::memset(&b, 0, sizeof(b));
  b.k = 1;
  b.chunk_elems = plan->chunk_elems;
  b.dtype = plan->dtype;
  b.max_code_len = plan->max_code_len;
  b.status = (uint32_t *)ws;
  b.ticket = (uint32_t *)(ws + 4);
  Item &it = b.item[0];
  it.counts = const_cast<uint64_t *>(counts);
  it.code_len = code_len;
  it.code = code;
  it.pm_scratch = (uint64_t *)(ws + align256(kHeader + kCountsBytes));
  cudaStream_t s = (cudaStream_t)stream;
  if (cudaMemsetAsync(ws, 0, kHeader, s) != cudaSuccess) return EH_ERR_CUDA;
  if (launch_book(b, s) != cudaSuccess) return EH_ERR_CUDA;
  return EH_OK;
}

eh_status eh_pages_append(const eh_plan_t *plan, const eh_page_store_t *store, const void *in, uint32_t n_pages,
                          const uint32_t *slot_ids, void *workspace, uint64_t workspace_bytes, void *stream) {
  if (!plan_ok(plan) || !store || !workspace || workspace_bytes < kHeader) return EH_ERR_INVALID_ARG;
  if (n_pages == 0) return EH_OK;
  const bool has_sm = plan->dtype != EH_BYTES;
  if (!in || !slot_ids || !store->code_len || !store->code || !store->slots || !store->page_meta ||
      !store->raw_used || (has_sm && !store->sign_mant) || (store->raw_cap && !store->raw_pool))
    return EH_ERR_INVALID_ARG;
  if (!aligned16(in) || !aligned16(store->slots) || (has_sm && !aligned16(store->sign_mant)) ||
      (store->raw_pool && !aligned16(store->raw_pool)) || store->slot_bytes % 16 || store->slot_bytes == 0 ||
      ((uintptr_t)workspace & 255u))
    return EH_ERR_INVALID_ARG;
  int num_sms = 0;
  if (device_setup(&num_sms) != cudaSuccess) return EH_ERR_CUDA;
  PageLaunch pl;
  std::memset(&pl, 0, sizeof(pl));
  pl.in = in;
  pl.slot_ids = slot_ids;
  pl.n_pages = n_pages;
  pl.page_elems = plan->chunk_elems;
  pl.code_len = store->code_len;
  pl.code = store->code;
  pl.slots = store->slots;
  pl.slot_bytes = store->slot_bytes;
  pl.n_slots = store->n_slots;
  pl.raw_cap = store->raw_cap;
  pl.sm = store->sign_mant;
  pl.page_meta = store->page_meta;
  pl.raw_pool = store->raw_pool;
  pl.raw_used = store->raw_used;
  pl.status = (uint32_t *)workspace;
  pl.dtype = plan->dtype;
  // Calls of fewer pages than two waves of one-CTA-per-page kernels are
  // split into kPageParts CTAs per page when the workspace holds their part
  // totals (16 bytes a page).
  if (n_pages < 4u * (uint32_t)num_sms && workspace_bytes >= kHeader + 4ull * kPageParts * n_pages)
    pl.part_bits = (uint32_t *)((uint8_t *)workspace + kHeader);
  cudaStream_t s = (cudaStream_t)stream;
  if (cudaMemsetAsync(workspace, 0, 4, s) != cudaSuccess) return EH_ERR_CUDA;
  if (launch_page_append(pl, s) != cudaSuccess) return EH_ERR_CUDA;
  return EH_OK;
}

namespace {

// Arguments of a page-store read that the decoder relies on.
bool page_read_args_ok(const eh_plan_t *plan, const eh_page_store_t *store, const uint32_t *slot_ids,
                       const void *out) {
  const bool has_sm = plan->dtype != EH_BYTES;
  return out && slot_ids && store->code_len && store->code && store->slots && store->page_meta &&
         (!has_sm || store->sign_mant) && aligned16(out) && aligned16(store->slots) &&
         (!has_sm || aligned16(store->sign_mant)) && (!store->raw_pool || aligned16(store->raw_pool)) &&
         store->slot_bytes % 16 == 0 && store->slot_bytes != 0;
}

// The decoder's descriptor of a read of n_pages pages, with the decode
// tables at `lut` and the status word at `status`.
void page_read_batch(const eh_plan_t *plan, const eh_page_store_t *store, const uint32_t *slot_ids,
                     uint32_t n_pages, void *out, uint8_t *status, const void *lut, Batch *bp) {
  Batch &b = *bp;
  std::memset(&b, 0, sizeof(b));
  b.k = 1;
  b.chunk_elems = plan->chunk_elems;
  b.dtype = plan->dtype;
  b.max_code_len = plan->max_code_len;
  b.status = (uint32_t *)status;
  b.ticket = (uint32_t *)(status + 4);
  b.total_chunks = n_pages;
  Item &it = b.item[0];
  it.out = out;
  it.n = (uint64_t)n_pages * plan->chunk_elems;
  it.chunk0 = 0;
  it.nchunks = n_pages;
  it.total_chunks = n_pages;
  it.code_len = const_cast<uint8_t *>(store->code_len);
  it.code = const_cast<uint32_t *>(store->code);
  it.stream = store->slots;
  it.stream_cap = (uint64_t)store->n_slots * store->slot_bytes;
  it.sm = store->sign_mant;
  it.lut = const_cast<void *>(lut);
  it.slot_ids = slot_ids;
  it.page_meta = store->page_meta;
  it.raw_pool = store->raw_pool;
  it.slot_bytes = store->slot_bytes;
  it.n_slots = store->n_slots;
  it.raw_cap = store->raw_cap;
}

}  // namespace

eh_status eh_pages_read(const eh_plan_t *plan, const eh_page_store_t *store, const uint32_t *slot_ids,
                        uint32_t n_pages, void *out, void *workspace, uint64_t workspace_bytes, void *stream) {
  if (!plan_ok(plan) || !store || !workspace) return EH_ERR_INVALID_ARG;
  if (((uintptr_t)workspace & 255u) != 0) return EH_ERR_INVALID_ARG;
  if (workspace_bytes < kHeader + kLutBytes) return EH_ERR_NOMEM;
  if (n_pages == 0) return EH_OK;
  if (!page_read_args_ok(plan, store, slot_ids, out)) return EH_ERR_INVALID_ARG;
  uint8_t *ws = (uint8_t *)workspace;
  Batch b;
  page_read_batch(plan, store, slot_ids, n_pages, out, ws, ws + kHeader, &b);
  int num_sms = 0;
  if (device_setup(&num_sms) != cudaSuccess) return EH_ERR_CUDA;
  cudaStream_t s = (cudaStream_t)stream;
  if (launch_tables(b, s) != cudaSuccess) return EH_ERR_CUDA;
  if (launch_decode(b, s, num_sms) != cudaSuccess) return EH_ERR_CUDA;
  return EH_OK;
}

eh_status eh_pages_prepare(const eh_plan_t *plan, const eh_page_store_t *store, void *tables,
                           uint64_t tables_bytes, void *stream) {
  if (!plan_ok(plan) || !store || !store->code_len || !store->code || !tables) return EH_ERR_INVALID_ARG;
  if (((uintptr_t)tables & 255u) != 0) return EH_ERR_INVALID_ARG;
  if (tables_bytes < kHeader + kLutBytes) return EH_ERR_NOMEM;
  uint8_t *t = (uint8_t *)tables;
  Batch b;
  std::memset(&b, 0, sizeof(b));
  b.k = 1;
  b.chunk_elems = plan->chunk_elems;
  b.dtype = plan->dtype;
  b.max_code_len = plan->max_code_len;
  b.status = (uint32_t *)t;
  b.ticket = (uint32_t *)(t + 4);
  Item &it = b.item[0];
  it.n = plan->chunk_elems;  // pages hold values: a codebook without codes is invalid
  it.code_len = const_cast<uint8_t *>(store->code_len);
  it.code = const_cast<uint32_t *>(store->code);
  it.lut = t + kHeader;
  int num_sms = 0;
  if (device_setup(&num_sms) != cudaSuccess) return EH_ERR_CUDA;
  if (launch_tables(b, (cudaStream_t)stream) != cudaSuccess) return EH_ERR_CUDA;
  return EH_OK;
}

eh_status eh_pages_read_prepared(const eh_plan_t *plan, const eh_page_store_t *store, const void *tables,
                                 const uint32_t *slot_ids, uint32_t n_pages, void *out, void *workspace,
                                 uint64_t workspace_bytes, void *stream) {
  if (!plan_ok(plan) || !store || !tables || !workspace) return EH_ERR_INVALID_ARG;
  if (((uintptr_t)workspace & 255u) != 0 || ((uintptr_t)tables & 255u) != 0) return EH_ERR_INVALID_ARG;
  if (workspace_bytes < kHeader) return EH_ERR_NOMEM;
  if (n_pages == 0) return EH_OK;
  if (!page_read_args_ok(plan, store, slot_ids, out)) return EH_ERR_INVALID_ARG;
  uint8_t *ws = (uint8_t *)workspace;
  Batch b;
  page_read_batch(plan, store, slot_ids, n_pages, out, ws, (const uint8_t *)tables + kHeader, &b);
  int num_sms = 0;
  if (device_setup(&num_sms) != cudaSuccess) return EH_ERR_CUDA;
  cudaStream_t s = (cudaStream_t)stream;
  if (cudaMemsetAsync(ws, 0, 8, s) != cudaSuccess) return EH_ERR_CUDA;  // this call's status starts clean
  if (launch_decode(b, s, num_sms) != cudaSuccess) return EH_ERR_CUDA;
  return EH_OK;
}

eh_status eh_debug_set_fixup_rounds(uint32_t rounds) {
  g_fixup_rounds.store(rounds, std::memory_order_relaxed);
  return EH_OK;
}

eh_status eh_get_status(void *workspace, void *stream) {
  if (!workspace) return EH_ERR_INVALID_ARG;
  uint32_t st = 0;
  cudaStream_t s = (cudaStream_t)stream;
  if (cudaMemcpyAsync(&st, workspace, 4, cudaMemcpyDeviceToHost, s) != cudaSuccess) return EH_ERR_CUDA;
  if (cudaStreamSynchronize(s) != cudaSuccess) return EH_ERR_CUDA;
  if (st & kFlagInfeasible) return EH_ERR_INFEASIBLE;
  if (st & kFlagTimeout) return EH_ERR_TIMEOUT;
  if (st & kFlagNoRoom) return EH_ERR_NOMEM;
  if (st & kFlagCorrupt) return EH_ERR_CORRUPT;
  return EH_OK;
}

}  // extern "C"

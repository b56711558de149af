// eh_prefetch.cu -- ring of decoded-operand slots filled on a decode stream
// ahead of a consumer stream (host code; the decoding is eh_decompress's).
//
// Each slot has its own decompression workspace, so the status word of a
// slot's decode survives until the slot is submitted again, and two events:
// `ready` (recorded on the decode stream after the decode) and `released`
// (recorded on the consumer stream when the consumer is done with the slot).
// The decode stream waits for `released` before overwriting a slot and the
// consumer waits for `ready` before reading it; the host never blocks.
#include <cstdlib>
#include <cstring>
#include <new>

#include "eh_internal.cuh"

using namespace eh;

namespace {

enum SlotState { kFree = 0, kSubmitted = 1, kAcquired = 2 };

// one decompression workspace of EH_MAX_BATCH tensors per slot, 256-byte aligned
uint64_t slot_ws_bytes(const eh_plan_t *plan) {
  uint64_t b = 0;
  if (eh_decompress_workspace(plan, EH_MAX_BATCH, &b) != EH_OK) return 0;
  return (b + 255) & ~uint64_t(255);
}

uint64_t elem_bytes(int32_t dtype) { return dtype == EH_BF16 ? 2u : 1u; }

}  // namespace

struct eh_prefetch {
  eh_plan_t plan;
  int depth;
  int next;                  // slot of the next submit
  uint32_t max_ctas;
  uint64_t slot_bytes;
  uint64_t ws_bytes;         // per slot
  cudaStream_t dstream;
  void *slots[EH_PREFETCH_MAX_DEPTH];
  uint8_t *ws[EH_PREFETCH_MAX_DEPTH];
  cudaEvent_t ready[EH_PREFETCH_MAX_DEPTH];
  cudaEvent_t released[EH_PREFETCH_MAX_DEPTH];
  bool has_release[EH_PREFETCH_MAX_DEPTH];  // `released` was recorded since creation
  int state[EH_PREFETCH_MAX_DEPTH];
};

extern "C" {

eh_status eh_prefetch_workspace(const eh_plan_t *plan, int depth, uint64_t *workspace_bytes) {
  if (!plan || !workspace_bytes || depth < 1 || depth > EH_PREFETCH_MAX_DEPTH) return EH_ERR_INVALID_ARG;
  const uint64_t per = slot_ws_bytes(plan);
  if (!per) return EH_ERR_INVALID_ARG;
  *workspace_bytes = (uint64_t)depth * per;
  return EH_OK;
}

eh_status eh_prefetch_create(const eh_plan_t *plan, int depth, void *const *slots, uint64_t slot_bytes,
                             void *workspace, uint64_t workspace_bytes, void *decode_stream, uint32_t max_ctas,
                             eh_prefetch **out) {
  if (!out) return EH_ERR_INVALID_ARG;
  *out = nullptr;
  if (!plan || !slots || !workspace || depth < 1 || depth > EH_PREFETCH_MAX_DEPTH) return EH_ERR_INVALID_ARG;
  if (plan->dtype != EH_BF16 && plan->dtype != EH_FP8_E4M3 && plan->dtype != EH_BYTES) return EH_ERR_INVALID_ARG;
  if (((uintptr_t)workspace & 255u) != 0) return EH_ERR_INVALID_ARG;
  for (int i = 0; i < depth; i++)
    if (!slots[i] || ((uintptr_t)slots[i] & 255u) != 0) return EH_ERR_INVALID_ARG;
  const uint64_t per = slot_ws_bytes(plan);
  if (!per) return EH_ERR_INVALID_ARG;
  if (workspace_bytes < (uint64_t)depth * per) return EH_ERR_NOMEM;
  eh_prefetch *pf = new (std::nothrow) eh_prefetch;
  if (!pf) return EH_ERR_NOMEM;
  std::memset(pf, 0, sizeof(*pf));
  pf->plan = *plan;
  pf->depth = depth;
  pf->max_ctas = max_ctas;
  pf->slot_bytes = slot_bytes;
  pf->ws_bytes = per;
  pf->dstream = (cudaStream_t)decode_stream;
  for (int i = 0; i < depth; i++) {
    pf->slots[i] = slots[i];
    pf->ws[i] = (uint8_t *)workspace + (uint64_t)i * per;
    if (cudaEventCreateWithFlags(&pf->ready[i], cudaEventDisableTiming) != cudaSuccess ||
        cudaEventCreateWithFlags(&pf->released[i], cudaEventDisableTiming) != cudaSuccess) {
      eh_prefetch_destroy(pf);
      return EH_ERR_CUDA;
    }
  }
  *out = pf;
  return EH_OK;
}

eh_status eh_prefetch_submit(eh_prefetch *pf, int k, const eh_compressed_t *cs, uint64_t *offsets, int *slot) {
  if (!pf || !cs || !offsets || !slot || k < 1 || k > EH_MAX_BATCH) return EH_ERR_INVALID_ARG;
  const int s = pf->next;
  if (pf->state[s] != kFree) return EH_ERR_INVALID_ARG;  // not released since its last submit
  void *outs[EH_MAX_BATCH];
  uint64_t off = 0;
  for (int i = 0; i < k; i++) {
    if (cs[i].dtype != pf->plan.dtype) return EH_ERR_INVALID_ARG;
    const uint64_t bytes = cs[i].n * elem_bytes(pf->plan.dtype);
    if (off + bytes > pf->slot_bytes) return EH_ERR_NOMEM;
    offsets[i] = off;
    outs[i] = (uint8_t *)pf->slots[s] + off;
    off = (off + bytes + 255) & ~uint64_t(255);
  }
  if (pf->has_release[s] && cudaStreamWaitEvent(pf->dstream, pf->released[s], 0) != cudaSuccess)
    return EH_ERR_CUDA;
  const eh_status st = decompress_impl(&pf->plan, k, cs, outs, nullptr, nullptr, pf->ws[s], pf->ws_bytes,
                                       pf->dstream, pf->max_ctas);
  if (st != EH_OK) return st;
  if (cudaEventRecord(pf->ready[s], pf->dstream) != cudaSuccess) return EH_ERR_CUDA;
  pf->state[s] = kSubmitted;
  pf->next = (s + 1) % pf->depth;
  *slot = s;
  return EH_OK;
}

eh_status eh_prefetch_acquire(eh_prefetch *pf, int slot, void *consumer_stream) {
  if (!pf || slot < 0 || slot >= pf->depth || pf->state[slot] != kSubmitted) return EH_ERR_INVALID_ARG;
  if (cudaStreamWaitEvent((cudaStream_t)consumer_stream, pf->ready[slot], 0) != cudaSuccess) return EH_ERR_CUDA;
  pf->state[slot] = kAcquired;
  return EH_OK;
}

eh_status eh_prefetch_release(eh_prefetch *pf, int slot, void *consumer_stream) {
  if (!pf || slot < 0 || slot >= pf->depth || pf->state[slot] != kAcquired) return EH_ERR_INVALID_ARG;
  if (cudaEventRecord(pf->released[slot], (cudaStream_t)consumer_stream) != cudaSuccess) return EH_ERR_CUDA;
  pf->has_release[slot] = true;
  pf->state[slot] = kFree;
  return EH_OK;
}

eh_status eh_prefetch_status(eh_prefetch *pf, int slot) {
  if (!pf || slot < 0 || slot >= pf->depth) return EH_ERR_INVALID_ARG;
  if (pf->state[slot] == kFree && !pf->has_release[slot]) return EH_ERR_INVALID_ARG;  // never submitted
  if (cudaEventSynchronize(pf->ready[slot]) != cudaSuccess) return EH_ERR_CUDA;
  return eh_get_status(pf->ws[slot], pf->dstream);
}

eh_status eh_prefetch_destroy(eh_prefetch *pf) {
  if (!pf) return EH_OK;
  eh_status st = EH_OK;
  if (cudaStreamSynchronize(pf->dstream) != cudaSuccess) st = EH_ERR_CUDA;
  for (int i = 0; i < pf->depth; i++) {
    if (pf->ready[i]) cudaEventDestroy(pf->ready[i]);
    if (pf->released[i]) cudaEventDestroy(pf->released[i]);
  }
  delete pf;
  return st;
}

}  // extern "C"

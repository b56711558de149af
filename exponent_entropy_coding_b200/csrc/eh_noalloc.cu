// eh_noalloc.cu -- block decompression for callers that cannot allocate
// device memory.
//
// Some callers cannot call cudaMalloc (or any allocating routine) at the point
// where they need to decompress: runtimes that plan all device memory up front
// and forbid later allocations, or allocator callbacks that must not re-enter
// the allocator.  eh_decompress_batch_noalloc serves them: the decoder's
// scratch (the status word and one set of decode tables per tensor) lives in a
// file-scope device array of fixed size instead of a caller-provided
// workspace.  The caller still provides the compressed inputs and the output
// buffers.  The call reads the status back and synchronises the stream, so it
// is not meant for a stream that is being captured into a CUDA graph.
//
// The array is allocated by the CUDA runtime in every device context that
// loads this library and stays there until the process exits.  All calls
// share it: each call clears the status word before use (the table kernel
// does), and calls that overlap on the GPU (different streams, other
// threads) race on it.
#include <mutex>

#include "eh_internal.cuh"

namespace {

static_assert(eh::kLutBytes == 37888, "the header documents 37,888 bytes of decode tables per tensor");
constexpr uint64_t kNoallocBytes = 256 + (uint64_t)EH_NOALLOC_MAX_BATCH * eh::kLutBytes;

static __device__ __align__(256) uint8_t g_noalloc_scratch[kNoallocBytes];

constexpr int kMaxDevices = 64;
std::mutex g_addr_mu;
void *g_addr[kMaxDevices];  // device address of the array, per device (null: not looked up yet)

// Device address of the scratch array on the current device (the host-side
// symbol is not a device address).  Only a successful lookup is kept, so a
// transient failure is retried by the next call.
cudaError_t scratch_address(void **ptr) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  if (dev < 0 || dev >= kMaxDevices) return cudaErrorInvalidDevice;
  std::lock_guard<std::mutex> lock(g_addr_mu);
  if (!g_addr[dev]) {
    void *p = nullptr;
    e = cudaGetSymbolAddress(&p, g_noalloc_scratch);
    if (e != cudaSuccess) return e;
    g_addr[dev] = p;
  }
  *ptr = g_addr[dev];
  return cudaSuccess;
}

}  // namespace

extern "C" {

eh_status eh_decompress_batch_noalloc(const eh_plan_t *plan, int k, const eh_compressed_t *cs,
                                      void *const *outs, void *stream) {
  if (k < 1 || k > EH_NOALLOC_MAX_BATCH) return EH_ERR_INVALID_ARG;
  void *scratch = nullptr;
  if (scratch_address(&scratch) != cudaSuccess || !scratch) return EH_ERR_CUDA;
  const eh_status st = eh_decompress_batch(plan, k, cs, outs, scratch, kNoallocBytes, stream);
  if (st != EH_OK) return st;
  return eh_get_status(scratch, stream);
}

}  // extern "C"

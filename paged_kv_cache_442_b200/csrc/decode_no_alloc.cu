// pa_decode_no_alloc: paged decode for callers that cannot allocate device memory.
//
// pa_decode needs a scratch buffer for its split-K partials, and expects the caller
// to allocate it. Some callers cannot: a serving runtime that carves the whole GPU
// into fixed pools at start-up and refuses any later allocation, or a host program
// that drives this library only through its C ABI and has no handle on a CUDA
// allocator. This entry point uses scratch that the library itself owns instead:
// a file-scope device array, created when the library's device code is loaded on a
// GPU and held by every GPU that loads the library until the process exits.
//
// The array's name is only a host-side stand-in in host code, not a device address:
// the device address is looked up with cudaGetSymbolAddress, with the device current,
// and that address is what the kernels receive. The lookup is repeated on every call
// (a host-side table lookup, no stream work): after a device reset the library's
// device code is loaded again and the array may sit at another address, so a cached
// pointer could point at memory the array no longer occupies.
#include <cuda_runtime.h>

#include "pa.h"
#include "pa_internal.h"

namespace pa {
namespace {

static __device__ __align__(256) unsigned char g_decode_scratch[PA_DECODE_NO_ALLOC_SCRATCH_BYTES];

// Device address of g_decode_scratch on the current device.
cudaError_t scratch_address(void** out) {
  void* p = nullptr;
  const cudaError_t e = cudaGetSymbolAddress(&p, g_decode_scratch);
  if (e != cudaSuccess) return e;
  *out = p;
  return cudaSuccess;
}

}  // namespace
}  // namespace pa

extern "C" pa_status pa_decode_no_alloc(void* out, const void* q, const void* k_cache,
                                        const void* v_cache, pa_cache_desc cache,
                                        const int32_t* block_tables, int32_t max_blocks_per_seq,
                                        const int32_t* context_lens, int32_t num_seqs,
                                        int32_t num_q_heads, float scale, int32_t max_context_len,
                                        int32_t partition_size, void* stream) {
  if (partition_size < 0 || (partition_size % 64) != 0) return PA_ERR_INVALID_ARG;
  if (num_seqs <= 0) {
    return pa_decode(out, q, k_cache, v_cache, cache, block_tables, max_blocks_per_seq,
                     context_lens, num_seqs, num_q_heads, scale, max_context_len,
                     partition_size, nullptr, 0, stream);
  }
  // the split pa_decode would pick; fixed here so sizing and launch agree
  const int32_t P = partition_size > 0
                        ? partition_size
                        : pa_decode_default_partition(num_seqs, cache.num_kv_heads, max_context_len);
  const size_t need =
      pa_decode_workspace_size(num_seqs, num_q_heads, cache.head_dim, max_context_len, P);
  if (need > PA_DECODE_NO_ALLOC_SCRATCH_BYTES) return PA_ERR_UNSUPPORTED;
  void* scratch = nullptr;
  if (need > 0 && pa::scratch_address(&scratch) != cudaSuccess) {
    cudaGetLastError();
    return PA_ERR_CUDA;
  }
  return pa_decode(out, q, k_cache, v_cache, cache, block_tables, max_blocks_per_seq,
                   context_lens, num_seqs, num_q_heads, scale, max_context_len, P, scratch,
                   need > 0 ? static_cast<size_t>(PA_DECODE_NO_ALLOC_SCRATCH_BYTES) : 0, stream);
}

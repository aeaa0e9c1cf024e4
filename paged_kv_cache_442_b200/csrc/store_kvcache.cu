// store_kvcache: scatter this step's new K/V rows into the paged pool through the
// slot mapping (mini-vllm page, section 2 "KVCache": the block table decides where
// in the pre-allocated tensor K/V are written).
//
// HBM-bound copy: every 16-byte vector of a token's row is moved by one thread;
// consecutive threads take consecutive vectors of a row, so both the reads of
// k/v and the writes into the pool row are fully coalesced. K and V are handled
// by the same thread (two independent 16-byte transfers in flight).
#include "pa_internal.h"
#include "pa_ptx.cuh"

namespace pa {
namespace {

__global__ void __launch_bounds__(256) store_kvcache_kernel(
    const uint4* __restrict__ k, const uint4* __restrict__ v, uint4* __restrict__ k_cache,
    uint4* __restrict__ v_cache, const int32_t* __restrict__ slot_mapping, int32_t num_tokens,
    int32_t row_vecs, int64_t num_slots, unsigned* err) {
  const int64_t total = static_cast<int64_t>(num_tokens) * row_vecs;
  const int64_t stride = static_cast<int64_t>(gridDim.x) * blockDim.x;
  for (int64_t i = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x; i < total;
       i += stride) {
    const int64_t t = i / row_vecs;
    const int64_t c = i - t * row_vecs;
    const int64_t slot = __ldg(slot_mapping + t);
    if (slot < 0) continue;
    if (slot >= num_slots) {
      flag_error(err, PA_DEV_ERR_BAD_INDEX);
      continue;
    }
    const uint4 kv = __ldcs(k + i);
    const uint4 vv = __ldcs(v + i);
    __stcs(k_cache + slot * row_vecs + c, kv);
    __stcs(v_cache + slot * row_vecs + c, vv);
  }
}

}  // namespace

cudaError_t launch_store_kvcache(const void* k, const void* v, void* k_cache, void* v_cache,
                                 const pa_cache_desc& c, const int32_t* slot_mapping,
                                 int32_t num_tokens, cudaStream_t stream) {
  if (num_tokens == 0) return cudaSuccess;
  const int32_t row_vecs = c.num_kv_heads * c.head_dim * 2 / 16;
  const int64_t total = static_cast<int64_t>(num_tokens) * row_vecs;
  const int threads = 256;
  int64_t blocks = (total + threads - 1) / threads;
  const int64_t cap = static_cast<int64_t>(sm_count()) * 8;
  if (blocks > cap) blocks = cap;
  store_kvcache_kernel<<<static_cast<unsigned>(blocks), threads, 0, stream>>>(
      static_cast<const uint4*>(k), static_cast<const uint4*>(v), static_cast<uint4*>(k_cache),
      static_cast<uint4*>(v_cache), slot_mapping, num_tokens, row_vecs,
      static_cast<int64_t>(c.num_blocks) * c.block_size, device_error_word());
  return cudaGetLastError();
}

}  // namespace pa

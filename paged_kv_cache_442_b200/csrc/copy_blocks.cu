// copy_blocks: copy-on-write of shared KV blocks. Blocks are shared between sequences
// by reference count (nano vllm page, section 3.2.1); a sequence that is about to
// append into a shared block first gets a private copy, so the other sharers keep
// reading the unchanged block.
//
// HBM-bound copy: each (src, dst) pair moves one block of K and one of V
// (block_size x Hkv x D x 2 bytes each). The grid is (chunks of a block, pairs);
// consecutive threads take consecutive 16-byte vectors, and each thread keeps four
// vectors of K and four of V in flight before storing them.
#include "pa_internal.h"
#include "pa_ptx.cuh"

namespace pa {
namespace {

constexpr int kThreads = 256;
constexpr int kUnroll = 4;

__global__ void __launch_bounds__(kThreads) copy_blocks_kernel(
    uint4* __restrict__ k_cache, uint4* __restrict__ v_cache, const int32_t* __restrict__ src,
    const int32_t* __restrict__ dst, int32_t num_pairs, int64_t block_vecs, int32_t num_blocks,
    unsigned* err) {
  for (int pair = blockIdx.y; pair < num_pairs; pair += gridDim.y) {
    const int a = __ldg(src + pair);
    const int b = __ldg(dst + pair);
    if (a < 0 || a >= num_blocks || b < 0 || b >= num_blocks) {
      if (blockIdx.x == 0 && threadIdx.x == 0) flag_error(err, PA_DEV_ERR_BAD_INDEX);
      continue;
    }
    if (a == b) continue;
    const uint4* ks = k_cache + static_cast<int64_t>(a) * block_vecs;
    const uint4* vs = v_cache + static_cast<int64_t>(a) * block_vecs;
    uint4* kd = k_cache + static_cast<int64_t>(b) * block_vecs;
    uint4* vd = v_cache + static_cast<int64_t>(b) * block_vecs;
    const int64_t step = static_cast<int64_t>(gridDim.x) * kThreads * kUnroll;
    for (int64_t base = static_cast<int64_t>(blockIdx.x) * kThreads * kUnroll + threadIdx.x;
         base < block_vecs; base += step) {
      uint4 kv[kUnroll], vv[kUnroll];
#pragma unroll
      for (int u = 0; u < kUnroll; ++u) {
        const int64_t c = base + u * kThreads;
        if (c < block_vecs) {
          kv[u] = __ldcs(ks + c);
          vv[u] = __ldcs(vs + c);
        }
      }
#pragma unroll
      for (int u = 0; u < kUnroll; ++u) {
        const int64_t c = base + u * kThreads;
        if (c < block_vecs) {
          __stcs(kd + c, kv[u]);
          __stcs(vd + c, vv[u]);
        }
      }
    }
  }
}

}  // namespace

cudaError_t launch_copy_blocks(void* k_cache, void* v_cache, const pa_cache_desc& c,
                               const int32_t* src_blocks, const int32_t* dst_blocks,
                               int32_t num_pairs, cudaStream_t stream) {
  if (num_pairs == 0) return cudaSuccess;
  const int64_t block_vecs =
      static_cast<int64_t>(c.block_size) * c.num_kv_heads * c.head_dim * 2 / 16;
  const int64_t per_cta = static_cast<int64_t>(kThreads) * kUnroll;
  const int64_t gx = (block_vecs + per_cta - 1) / per_cta;
  dim3 grid(static_cast<unsigned>(gx), static_cast<unsigned>(num_pairs < 65535 ? num_pairs : 65535));
  copy_blocks_kernel<<<grid, kThreads, 0, stream>>>(
      static_cast<uint4*>(k_cache), static_cast<uint4*>(v_cache), src_blocks, dst_blocks, num_pairs,
      block_vecs, c.num_blocks, device_error_word());
  return cudaGetLastError();
}

}  // namespace pa

// store_kvcache: scatter this step's new K/V rows into the paged pool through the
// slot mapping (mini-vllm page, section 2 "KVCache": the block table decides where
// in the pre-allocated tensor K/V are written).
//
// HBM-bound copy: every 16-byte vector of a token's row is moved by one thread;
// consecutive threads take consecutive vectors of a row, so both the reads of
// k/v and the writes into the pool row are fully coalesced. K and V are handled
// by the same thread (two independent 16-byte transfers in flight).
#include <cuda_bf16.h>
#include <cuda_fp8.h>

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

// The new row of each sequence of a pa_store_decode call, written only when its slot
// is the slot of the sequence's last position (context_lens[s] - 1) as the block
// table gives it; any other slot is reported and skipped. One CTA per sequence, one
// 16-byte vector of K and one of V per thread.
__global__ void __launch_bounds__(128) store_last_rows_kernel(
    const uint4* __restrict__ k, const uint4* __restrict__ v, uint4* __restrict__ k_cache,
    uint4* __restrict__ v_cache, const int32_t* __restrict__ slot_mapping,
    const int32_t* __restrict__ block_tables, const int32_t* __restrict__ context_lens,
    int32_t max_blocks, int32_t max_context_len, int32_t bs_log2, int32_t num_blocks,
    int32_t row_vecs, unsigned* err) {
  const int s = blockIdx.x;
  const int slot = __ldg(slot_mapping + s);
  if (slot < 0) return;
  const int ctx = __ldg(context_lens + s);
  const int pos = ctx - 1;
  bool ok = ctx > 0 && ctx <= max_context_len && (pos >> bs_log2) < max_blocks;
  int id = -1;
  if (ok) id = __ldg(block_tables + static_cast<int64_t>(s) * max_blocks + (pos >> bs_log2));
  ok = ok && id >= 0 && id < num_blocks &&
       static_cast<int64_t>(slot) ==
           (static_cast<int64_t>(id) << bs_log2) + (pos & ((1 << bs_log2) - 1));
  if (!ok) {
    if (threadIdx.x == 0) flag_error(err, PA_DEV_ERR_BAD_INDEX);
    return;
  }
  for (int c = threadIdx.x; c < row_vecs; c += blockDim.x) {
    const int64_t src = static_cast<int64_t>(s) * row_vecs + c;
    const int64_t dst = static_cast<int64_t>(slot) * row_vecs + c;
    k_cache[dst] = __ldg(k + src);
    v_cache[dst] = __ldg(v + src);
  }
}

// fp8 pools: one warp per (token, kv head, K or V) row. The row's largest magnitude
// sets its scale (amax / 448, fp32); codes are e4m3(x * (448 / amax)) rounded to
// nearest even and saturated. A row whose 448 / amax is not a finite fp32 (all
// zeros, or amax below 448 / FLT_MAX) stores zero codes and scale 0.
template <int D>
__global__ void __launch_bounds__(256) store_kvcache_fp8_kernel(
    const __nv_bfloat16* __restrict__ k, const __nv_bfloat16* __restrict__ v,
    uint8_t* __restrict__ k_codes, uint8_t* __restrict__ v_codes, float* __restrict__ k_scales,
    float* __restrict__ v_scales, const int32_t* __restrict__ slot_mapping, int32_t num_tokens,
    int32_t hkv, int64_t num_slots, unsigned* err) {
  constexpr int PER = D / 32;  // values per lane
  const int lane = threadIdx.x & 31;
  const int64_t warps = (static_cast<int64_t>(gridDim.x) * blockDim.x) >> 5;
  const int64_t total = static_cast<int64_t>(num_tokens) * hkv * 2;
  for (int64_t w = (static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x) >> 5; w < total;
       w += warps) {
    const int64_t t = w / (2 * hkv);
    const int rem = static_cast<int>(w - t * 2 * hkv);
    const int g = rem >> 1;
    const bool is_v = rem & 1;
    const int64_t slot = __ldg(slot_mapping + t);
    if (slot < 0) continue;
    if (slot >= num_slots) {
      if (lane == 0) flag_error(err, PA_DEV_ERR_BAD_INDEX);
      continue;
    }
    const __nv_bfloat16* src = (is_v ? v : k) + (t * hkv + g) * D + lane * PER;
    float x[PER];
#pragma unroll
    for (int i = 0; i < PER; ++i) x[i] = __bfloat162float(src[i]);
    float amax = 0.f;
#pragma unroll
    for (int i = 0; i < PER; ++i) amax = fmaxf(amax, fabsf(x[i]));
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, o));
    float inv = __fdiv_rn(448.f, amax);
    const bool zero_row = isinf(inv);
    if (zero_row) inv = 0.f;
    // a zero row stores +0 codes (x * 0 would give -0 for negative x)
    uint32_t packed = 0;
#pragma unroll
    for (int i = 0; i < PER && !zero_row; i += 2) {
      const __nv_fp8x2_storage_t two = __nv_cvt_float2_to_fp8x2(
          make_float2(__fmul_rn(x[i], inv), __fmul_rn(x[i + 1], inv)), __NV_SATFINITE, __NV_E4M3);
      packed |= static_cast<uint32_t>(two) << (8 * i);
    }
    uint8_t* dst = (is_v ? v_codes : k_codes) + (slot * hkv + g) * D + lane * PER;
    if (PER == 4) {
      *reinterpret_cast<uint32_t*>(dst) = packed;
    } else {
      *reinterpret_cast<uint16_t*>(dst) = static_cast<uint16_t>(packed);
    }
    if (lane == 0)
      (is_v ? v_scales : k_scales)[g * num_slots + slot] = zero_row ? 0.f : __fdiv_rn(amax, 448.f);
  }
}

}  // namespace

cudaError_t launch_store_kvcache_fp8(const void* k, const void* v, void* k_codes, void* v_codes,
                                     float* k_scales, float* v_scales, const pa_cache_desc& c,
                                     const int32_t* slot_mapping, int32_t num_tokens,
                                     cudaStream_t stream) {
  if (num_tokens == 0) return cudaSuccess;
  const int64_t rows = static_cast<int64_t>(num_tokens) * c.num_kv_heads * 2;
  int64_t blocks = (rows * 32 + 255) / 256;
  const int64_t cap = static_cast<int64_t>(sm_count()) * 8;
  if (blocks > cap) blocks = cap;
  const int64_t num_slots = static_cast<int64_t>(c.num_blocks) * c.block_size;
  if (c.head_dim == 128)
    store_kvcache_fp8_kernel<128><<<static_cast<unsigned>(blocks), 256, 0, stream>>>(
        static_cast<const __nv_bfloat16*>(k), static_cast<const __nv_bfloat16*>(v),
        static_cast<uint8_t*>(k_codes), static_cast<uint8_t*>(v_codes), k_scales, v_scales,
        slot_mapping, num_tokens, c.num_kv_heads, num_slots, device_error_word());
  else
    store_kvcache_fp8_kernel<64><<<static_cast<unsigned>(blocks), 256, 0, stream>>>(
        static_cast<const __nv_bfloat16*>(k), static_cast<const __nv_bfloat16*>(v),
        static_cast<uint8_t*>(k_codes), static_cast<uint8_t*>(v_codes), k_scales, v_scales,
        slot_mapping, num_tokens, c.num_kv_heads, num_slots, device_error_word());
  return cudaGetLastError();
}

cudaError_t launch_store_last_rows(const DecodeLaunch& a, cudaStream_t stream) {
  if (a.num_seqs == 0 || !a.slot_mapping) return cudaSuccess;
  const int32_t row_vecs = a.cache.num_kv_heads * a.cache.head_dim * 2 / 16;
  store_last_rows_kernel<<<a.num_seqs, 128, 0, stream>>>(
      static_cast<const uint4*>(a.new_k), static_cast<const uint4*>(a.new_v),
      static_cast<uint4*>(const_cast<void*>(a.k_cache)),
      static_cast<uint4*>(const_cast<void*>(a.v_cache)), a.slot_mapping, a.block_tables,
      a.context_lens, a.max_blocks_per_seq, a.max_context_len,
      31 - __builtin_clz(static_cast<unsigned>(a.cache.block_size)), a.cache.num_blocks, row_vecs,
      device_error_word());
  return cudaGetLastError();
}

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

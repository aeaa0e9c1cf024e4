// Internal host-side interfaces between the C ABI layer (pa_api.cu) and the
// kernel translation units. Not part of the public ABI.
#pragma once

#include <cuda.h>
#include <cuda_runtime.h>
#include <stddef.h>
#include <stdint.h>

#include "pa.h"

namespace pa {

// Bits of the per-device error word that kernels set instead of trapping.
constexpr unsigned PA_DEV_ERR_BAD_INDEX = 1u;
constexpr unsigned PA_DEV_ERR_TIMEOUT = 2u;

// Per-device pointer to the device error word (lives in pa_api.cu).
unsigned* device_error_word();

// Bound, in ns of %globaltimer, of the waits between the roles of the tensor-core
// kernels (pa_set_wait_limit_ns; 2 s unless a test shortened it). The waits a CTA
// makes before it exits, for its own copies and MMAs still in flight, always keep
// the full 2 s.
unsigned long long wait_limit_ns();

// Number of SMs of the current device (cached).
int sm_count();

// Raise a kernel's dynamic shared-memory limit once per (kernel, device).
cudaError_t ensure_max_dynamic_smem(const void* func, int bytes);

// Encode a 3-D bf16 tensor map over a [dim2][dim1][dim0] row-major tensor.
// swizzle128: 128-byte swizzle (box_dim0 * 2 must then be <= 128).
// Any rank (<= 5), element type and size; dims innermost first; strides from dims.
bool encode_tensor_map(CUtensorMap* map, const void* base, CUtensorMapDataType dtype,
                       int elem_bytes, int rank, const uint64_t* dims, const uint32_t* box,
                       bool swizzle128);
bool encode_tensor_map_3d(CUtensorMap* map, const void* base, uint64_t dim0, uint64_t dim1,
                          uint64_t dim2, uint32_t box0, uint32_t box1, uint32_t box2,
                          bool swizzle128);

cudaError_t launch_block_hashes(const int32_t* token_ids, const int32_t* cu_tokens,
                                const int32_t* cu_blocks, int32_t num_seqs, int32_t block_size,
                                uint32_t* hashes_out, cudaStream_t stream);
cudaError_t launch_store_kvcache_fp8(const void* k, const void* v, void* k_codes, void* v_codes,
                                     float* k_scales, float* v_scales, const pa_cache_desc& c,
                                     const int32_t* slot_mapping, int32_t num_tokens,
                                     cudaStream_t stream);
cudaError_t launch_copy_blocks(void* k_cache, void* v_cache, const pa_cache_desc& c,
                               const int32_t* src_blocks, const int32_t* dst_blocks,
                               int32_t num_pairs, cudaStream_t stream);
cudaError_t launch_store_kvcache(const void* k, const void* v, void* k_cache, void* v_cache,
                                 const pa_cache_desc& c, const int32_t* slot_mapping,
                                 int32_t num_tokens, cudaStream_t stream);

struct DecodeLaunch {
  void* out;
  const void* q;
  const void* k_cache;
  const void* v_cache;
  pa_cache_desc cache;
  const int32_t* block_tables;
  int32_t max_blocks_per_seq;
  const int32_t* context_lens;
  int32_t num_seqs;
  int32_t num_q_heads;
  float scale;
  int32_t max_context_len;
  int32_t partition_size;  // resolved (> 0)
  int32_t max_parts;       // ceil(max_context_len / partition_size)
  float* ws_o;             // [B, Hq, max_parts, D] fp32 (NULL when max_parts == 1)
  float* ws_ml;            // [B, Hq, max_parts, 2] fp32
  // pa_store_decode: new rows [B, Hkv, D] stored to slot_mapping[s] (the slot of
  // position context_lens[s] - 1, or -1) before they are read; all NULL for pa_decode
  const void* new_k = nullptr;
  const void* new_v = nullptr;
  const int32_t* slot_mapping = nullptr;
  // pa_decode_fp8: k_cache / v_cache hold e4m3 codes; scales [Hkv][num_blocks * bs] fp32
  bool fp8 = false;
  const float* k_scales = nullptr;
  const float* v_scales = nullptr;
  // pa_decode_shared_prefix: positions below shared_len are shared by every sequence
  // (partition 0, attended by launch_shared_prefix); 0 = plain decode
  int32_t shared_len = 0;
};
cudaError_t launch_decode(const DecodeLaunch& a, cudaStream_t stream);
// Stores the new rows of a pa_store_decode call on its own (the paths whose decode
// kernel does not store them): checks each slot against the sequence's last position.
cudaError_t launch_store_last_rows(const DecodeLaunch& a, cudaStream_t stream);

// Persistent tcgen05 decode (head dim 128). `counters` is the workspace's counter
// region: 1 + num_seqs * num_q_heads epoch-tagged 64-bit counters.
bool decode_tc_supported(const DecodeLaunch& a);
// The shared prefix of a pa_decode_shared_prefix call, once for all sequences: output
// rows of contexts inside the prefix, partition-0 partials of the others.
cudaError_t launch_shared_prefix(const DecodeLaunch& a, const int32_t* shared_blocks,
                                 int shared_len, cudaStream_t stream);
cudaError_t launch_decode_tc(const DecodeLaunch& a, unsigned long long* counters,
                             cudaStream_t stream);

// Bytes of the counter region at the start of the decode workspace (256-aligned).
inline size_t decode_counter_bytes(int32_t num_seqs, int32_t num_q_heads) {
  const size_t b = 8 * (1 + static_cast<size_t>(num_seqs) * num_q_heads);
  return (b + 255) / 256 * 256;
}

struct PrefillLaunch {
  void* out;
  const void* q;
  const void* k_cache;
  const void* v_cache;
  pa_cache_desc cache;
  const int32_t* block_tables;
  int32_t max_blocks_per_seq;
  const int32_t* cu_seqlens_q;
  const int32_t* context_lens;
  int32_t num_seqs;
  int32_t num_q_heads;
  int32_t max_q_len;
  int32_t total_q;  // rows of q/out (cu_seqlens_q[num_seqs]) upper bound for the tensor map
  float scale;
  // pa_store_prefill: the new rows [total_q, Hkv, D] (read by the attention in place
  // of the pool) and their slots; all NULL for pa_prefill
  const void* new_k = nullptr;
  const void* new_v = nullptr;
  const int32_t* slot_mapping = nullptr;
};
cudaError_t launch_prefill(const PrefillLaunch& a, cudaStream_t stream);

}  // namespace pa

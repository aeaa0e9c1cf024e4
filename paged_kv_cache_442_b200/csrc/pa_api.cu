// C ABI of libpa.so: argument validation, scratch-space sizing, device error
// word and tensor-map encoding. Kernels live in store_kvcache.cu, decode.cu and
// prefill.cu.
#include <cuda.h>
#include <cuda_runtime.h>

#include <atomic>
#include <cmath>
#include <cstdint>
#include <mutex>
#include <set>
#include <utility>

#include "pa.h"
#include "pa_internal.h"

namespace pa {

// One word per device that loads the library: bit 0 = bad index, bit 1 = timeout.
__device__ unsigned g_device_error_word;

namespace {

constexpr int kMaxDevices = 64;
constexpr unsigned long long kDefaultWaitLimitNs = 2000000000ull;
std::atomic<int> g_debug{0};
std::atomic<unsigned long long> g_wait_limit_ns{kDefaultWaitLimitNs};
std::mutex g_mu;
int g_sm_count[kMaxDevices] = {0};
std::set<std::pair<const void*, int>> g_smem_set;  // (kernel, device) already raised

using EncodeTiledFn = CUresult (*)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*,
                                   const cuuint64_t*, const cuuint64_t*, const cuuint32_t*,
                                   const cuuint32_t*, CUtensorMapInterleave, CUtensorMapSwizzle,
                                   CUtensorMapL2promotion, CUtensorMapFloatOOBfill);
EncodeTiledFn g_encode = nullptr;

int current_device() {
  int d = 0;
  if (cudaGetDevice(&d) != cudaSuccess) return -1;
  return d;
}

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

bool is_pow2(int x) { return x > 0 && (x & (x - 1)) == 0; }

pa_status check_cache(const pa_cache_desc& c) {
  if (c.num_blocks <= 0 || c.num_kv_heads <= 0) return PA_ERR_INVALID_ARG;
  if (!is_pow2(c.block_size) || c.block_size < 16 || c.block_size > 1024) return PA_ERR_INVALID_ARG;
  if (c.head_dim != 64 && c.head_dim != 128) return PA_ERR_INVALID_ARG;
  const int64_t slots = static_cast<int64_t>(c.num_blocks) * c.block_size;
  if (slots > INT32_MAX) return PA_ERR_INVALID_ARG;
  return PA_OK;
}

pa_status finish(cudaError_t e, void* stream) {
  if (e != cudaSuccess) {
    cudaGetLastError();  // clear a sticky launch error from the runtime's slot
    return e == cudaErrorInvalidValue ? PA_ERR_INVALID_ARG : PA_ERR_CUDA;
  }
  if (g_debug.load(std::memory_order_relaxed)) return pa_check_device_errors(stream);
  return PA_OK;
}

}  // namespace

// Looked up on every call (a host-side table lookup): after a device reset the
// library's device code is loaded again and the word may sit at another address.
unsigned* device_error_word() {
  void* ptr = nullptr;
  if (cudaGetSymbolAddress(&ptr, g_device_error_word) != cudaSuccess) {
    cudaGetLastError();
    return nullptr;
  }
  return static_cast<unsigned*>(ptr);
}

unsigned long long wait_limit_ns() { return g_wait_limit_ns.load(std::memory_order_relaxed); }

int sm_count() {
  const int d = current_device();
  if (d < 0 || d >= kMaxDevices) return 148;
  std::lock_guard<std::mutex> lk(g_mu);
  if (!g_sm_count[d]) {
    int n = 0;
    if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, d) != cudaSuccess || n <= 0)
      n = 148;
    g_sm_count[d] = n;
  }
  return g_sm_count[d];
}

cudaError_t ensure_max_dynamic_smem(const void* func, int bytes) {
  const int d = current_device();
  std::lock_guard<std::mutex> lk(g_mu);
  auto key = std::make_pair(func, d);
  if (g_smem_set.count(key)) return cudaSuccess;
  cudaError_t e = cudaFuncSetAttribute(func, cudaFuncAttributeMaxDynamicSharedMemorySize, bytes);
  if (e == cudaSuccess) g_smem_set.insert(key);
  return e;
}

bool encode_tensor_map(CUtensorMap* map, const void* base, CUtensorMapDataType dtype,
                       int elem_bytes, int rank, const uint64_t* dims, const uint32_t* box,
                       bool swizzle128) {
  if (rank < 1 || rank > 5) return false;
  {
    std::lock_guard<std::mutex> lk(g_mu);
    if (!g_encode) {
      void* fn = nullptr;
      cudaDriverEntryPointQueryResult q;
      if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &fn, cudaEnableDefault, &q) !=
              cudaSuccess ||
          q != cudaDriverEntryPointSuccess || !fn)
        return false;
      g_encode = reinterpret_cast<EncodeTiledFn>(fn);
    }
  }
  cuuint64_t gdims[5], strides[4];
  cuuint32_t gbox[5], estr[5];
  uint64_t stride = static_cast<uint64_t>(elem_bytes);
  for (int i = 0; i < rank; ++i) {
    gdims[i] = dims[i];
    gbox[i] = box[i];
    estr[i] = 1;
    if (i > 0) strides[i - 1] = stride;  // bytes between consecutive indices of dim i
    stride *= dims[i];
  }
  CUresult r = g_encode(map, dtype, static_cast<cuuint32_t>(rank), const_cast<void*>(base), gdims,
                        strides, gbox, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
                        swizzle128 ? CU_TENSOR_MAP_SWIZZLE_128B : CU_TENSOR_MAP_SWIZZLE_NONE,
                        CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

bool encode_tensor_map_3d(CUtensorMap* map, const void* base, uint64_t dim0, uint64_t dim1,
                          uint64_t dim2, uint32_t box0, uint32_t box1, uint32_t box2,
                          bool swizzle128) {
  const uint64_t dims[3] = {dim0, dim1, dim2};
  const uint32_t box[3] = {box0, box1, box2};
  return encode_tensor_map(map, base, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, 3, dims, box, swizzle128);
}

namespace {

// pa_decode, and pa_store_decode when `store` carries the new rows and slots
struct StoreRows {
  const void* new_k;
  const void* new_v;
  const int32_t* slot_mapping;
};

// k_scales / v_scales: non-null for e4m3 pools (pa_decode_fp8)
pa_status decode_impl(const StoreRows* store, const float* k_scales, const float* v_scales,
                      void* out, const void* q, const void* k_cache,
                      const void* v_cache, pa_cache_desc cache, const int32_t* block_tables,
                      int32_t max_blocks_per_seq, const int32_t* context_lens, int32_t num_seqs,
                      int32_t num_q_heads, float scale, int32_t max_context_len,
                      int32_t partition_size, void* workspace, size_t workspace_bytes,
                      void* stream) {
  pa_status st = check_cache(cache);
  if (st != PA_OK) return st;
  if (num_seqs < 0 || num_q_heads <= 0 || max_blocks_per_seq <= 0 || max_context_len < 0)
    return PA_ERR_INVALID_ARG;
  if (num_q_heads % cache.num_kv_heads) return PA_ERR_INVALID_ARG;
  if (!std::isfinite(scale)) return PA_ERR_INVALID_ARG;
  if (static_cast<int64_t>(max_context_len) >
      static_cast<int64_t>(max_blocks_per_seq) * cache.block_size)
    return PA_ERR_INVALID_ARG;
  const int G = num_q_heads / cache.num_kv_heads;
  if (G != 1 && G != 2 && G != 4 && G != 8 && !(G == 16 && cache.head_dim == 128))
    return PA_ERR_UNSUPPORTED;
  if (num_seqs == 0) return PA_OK;
  if (!out || !q || !k_cache || !v_cache || !block_tables || !context_lens)
    return PA_ERR_INVALID_ARG;
  if (!aligned16(out) || !aligned16(q) || !aligned16(k_cache) || !aligned16(v_cache))
    return PA_ERR_INVALID_ARG;
  if (store && (!store->new_k || !store->new_v || !store->slot_mapping ||
                !aligned16(store->new_k) || !aligned16(store->new_v)))
    return PA_ERR_INVALID_ARG;
  const bool fp8 = k_scales != nullptr || v_scales != nullptr;
  if (fp8 && (!k_scales || !v_scales || !aligned16(k_scales) || !aligned16(v_scales)))
    return PA_ERR_INVALID_ARG;
  if (partition_size < 0 || (partition_size % 64) != 0) return PA_ERR_INVALID_ARG;
  const int P = partition_size > 0 ? partition_size
                                   : pa_decode_default_partition(num_seqs, cache.num_kv_heads,
                                                                 max_context_len);
  const int64_t parts64 = max_context_len > 0 ? (max_context_len + P - 1) / P : 1;
  // work items are counted in 24 bits, with room for one extra take per CTA
  if (parts64 * num_seqs * cache.num_kv_heads >= (1ll << 24) - 4096) return PA_ERR_UNSUPPORTED;
  const int parts = static_cast<int>(parts64);
  const size_t need =
      pa_decode_workspace_size(num_seqs, num_q_heads, cache.head_dim, max_context_len, P);
  if (!workspace || workspace_bytes < need || !aligned16(workspace)) return PA_ERR_INVALID_ARG;

  DecodeLaunch a;
  a.out = out;
  a.q = q;
  a.k_cache = k_cache;
  a.v_cache = v_cache;
  a.cache = cache;
  a.block_tables = block_tables;
  a.max_blocks_per_seq = max_blocks_per_seq;
  a.context_lens = context_lens;
  a.num_seqs = num_seqs;
  a.num_q_heads = num_q_heads;
  a.scale = scale;
  a.max_context_len = max_context_len;
  a.partition_size = P;
  a.max_parts = parts;
  const size_t cbytes = decode_counter_bytes(num_seqs, num_q_heads);
  unsigned long long* counters = static_cast<unsigned long long*>(workspace);
  float* ws = reinterpret_cast<float*>(static_cast<uint8_t*>(workspace) + cbytes);
  a.ws_o = parts > 1 ? ws : nullptr;
  a.ws_ml = parts > 1 ? ws + static_cast<size_t>(num_seqs) * num_q_heads * parts * cache.head_dim
                      : nullptr;
  const cudaStream_t s = static_cast<cudaStream_t>(stream);
  if (store) {
    a.new_k = store->new_k;
    a.new_v = store->new_v;
    a.slot_mapping = store->slot_mapping;
  }
  if (fp8) {
    // e4m3 pools have only the tensor-core path
    a.fp8 = true;
    a.k_scales = k_scales;
    a.v_scales = v_scales;
    if (!decode_tc_supported(a)) return PA_ERR_UNSUPPORTED;
  }
  // the persistent kernel stores the new rows itself; the CUDA-core path stores them
  // with a checked kernel first
  if (decode_tc_supported(a)) return finish(launch_decode_tc(a, counters, s), stream);
  if (G == 16) return PA_ERR_UNSUPPORTED;
  if (store) {
    const cudaError_t e = launch_store_last_rows(a, s);
    if (e != cudaSuccess) return finish(e, stream);
  }
  return finish(launch_decode(a, s), stream);
}

}  // namespace

}  // namespace pa

using namespace pa;

extern "C" {

int32_t pa_version(void) { return 100; }

const char* pa_status_string(pa_status s) {
  switch (s) {
    case PA_OK: return "PA_OK";
    case PA_ERR_INVALID_ARG: return "PA_ERR_INVALID_ARG";
    case PA_ERR_UNSUPPORTED: return "PA_ERR_UNSUPPORTED";
    case PA_ERR_BAD_INDEX: return "PA_ERR_BAD_INDEX";
    case PA_ERR_CUDA: return "PA_ERR_CUDA";
    case PA_ERR_TIMEOUT: return "PA_ERR_TIMEOUT";
    case PA_ERR_NO_BLOCKS: return "PA_ERR_NO_BLOCKS";
  }
  return "PA_ERR_UNKNOWN";
}

void pa_set_debug_checks(int on) { g_debug.store(on ? 1 : 0); }

void pa_set_wait_limit_ns(uint64_t ns) {
  g_wait_limit_ns.store(ns == 0 ? kDefaultWaitLimitNs : static_cast<unsigned long long>(ns));
}

pa_status pa_check_device_errors(void* stream) {
  if (cudaStreamSynchronize(static_cast<cudaStream_t>(stream)) != cudaSuccess) {
    cudaGetLastError();
    return PA_ERR_CUDA;
  }
  unsigned* w = device_error_word();
  if (!w) return PA_ERR_CUDA;
  unsigned v = 0;
  if (cudaMemcpy(&v, w, sizeof(v), cudaMemcpyDeviceToHost) != cudaSuccess) return PA_ERR_CUDA;
  if (v) {
    const unsigned zero = 0;
    if (cudaMemcpy(w, &zero, sizeof(zero), cudaMemcpyHostToDevice) != cudaSuccess)
      return PA_ERR_CUDA;
  }
  if (v & PA_DEV_ERR_TIMEOUT) return PA_ERR_TIMEOUT;
  if (v & PA_DEV_ERR_BAD_INDEX) return PA_ERR_BAD_INDEX;
  return PA_OK;
}

pa_status pa_store_kvcache(const void* k, const void* v, void* k_cache, void* v_cache,
                           pa_cache_desc cache, const int32_t* slot_mapping, int32_t num_tokens,
                           void* stream) {
  pa_status st = check_cache(cache);
  if (st != PA_OK) return st;
  if (num_tokens < 0) return PA_ERR_INVALID_ARG;
  if (num_tokens == 0) return PA_OK;
  if (!k || !v || !k_cache || !v_cache || !slot_mapping) return PA_ERR_INVALID_ARG;
  if (!aligned16(k) || !aligned16(v) || !aligned16(k_cache) || !aligned16(v_cache))
    return PA_ERR_INVALID_ARG;
  return finish(launch_store_kvcache(k, v, k_cache, v_cache, cache, slot_mapping, num_tokens,
                                     static_cast<cudaStream_t>(stream)),
                stream);
}

pa_status pa_block_hashes(const int32_t* token_ids, const int32_t* cu_tokens,
                          const int32_t* cu_blocks, int32_t num_seqs, int32_t block_size,
                          uint32_t* hashes_out, void* stream) {
  if (num_seqs < 0 || block_size <= 0) return PA_ERR_INVALID_ARG;
  if (num_seqs == 0) return PA_OK;
  if (!token_ids || !cu_tokens || !cu_blocks || !hashes_out) return PA_ERR_INVALID_ARG;
  return finish(launch_block_hashes(token_ids, cu_tokens, cu_blocks, num_seqs, block_size,
                                    hashes_out, static_cast<cudaStream_t>(stream)),
                stream);
}

pa_status pa_copy_blocks(void* k_cache, void* v_cache, pa_cache_desc cache,
                         const int32_t* src_blocks, const int32_t* dst_blocks, int32_t num_pairs,
                         void* stream) {
  pa_status st = check_cache(cache);
  if (st != PA_OK) return st;
  if (num_pairs < 0) return PA_ERR_INVALID_ARG;
  if (num_pairs == 0) return PA_OK;
  if (!k_cache || !v_cache || !src_blocks || !dst_blocks) return PA_ERR_INVALID_ARG;
  if (!aligned16(k_cache) || !aligned16(v_cache)) return PA_ERR_INVALID_ARG;
  return finish(launch_copy_blocks(k_cache, v_cache, cache, src_blocks, dst_blocks, num_pairs,
                                   static_cast<cudaStream_t>(stream)),
                stream);
}

int32_t pa_decode_default_partition(int32_t num_seqs, int32_t num_kv_heads,
                                    int32_t max_context_len) {
  // Work items are (partition, sequence, kv head) taken dynamically by one
  // persistent CTA per SM. Aim for ~16 items per SM on the upper bound of the work
  // (every sequence at max_context_len) so the last items finish close together,
  // with partitions a power of two in [256, 2048] positions (tiles are 128).
  const int64_t work = static_cast<int64_t>(num_seqs > 0 ? num_seqs : 1) *
                       (num_kv_heads > 0 ? num_kv_heads : 1) *
                       (max_context_len > 0 ? max_context_len : 1);
  const int64_t per_item = work / (static_cast<int64_t>(sm_count()) * 16);
  int P = 256;
  while (P < 2048 && P < per_item) P *= 2;
  return P;
}

size_t pa_decode_workspace_size(int32_t num_seqs, int32_t num_q_heads, int32_t head_dim,
                                int32_t max_context_len, int32_t partition_size) {
  // [epoch-tagged counters][partials o: B*Hq*parts*D fp32][partials (m, l): B*Hq*parts*2]
  if (num_seqs <= 0 || num_q_heads <= 0 || head_dim <= 0) return 0;
  if (partition_size <= 0) return 0;
  const size_t counters = decode_counter_bytes(num_seqs, num_q_heads);
  const int64_t parts =
      max_context_len > 0 ? (max_context_len + partition_size - 1) / partition_size : 1;
  if (parts <= 1) return counters;
  return counters +
         static_cast<size_t>(num_seqs) * num_q_heads * parts * (head_dim + 2) * sizeof(float);
}


pa_status pa_decode(void* out, const void* q, const void* k_cache, const void* v_cache,
                    pa_cache_desc cache, const int32_t* block_tables, int32_t max_blocks_per_seq,
                    const int32_t* context_lens, int32_t num_seqs, int32_t num_q_heads,
                    float scale, int32_t max_context_len, int32_t partition_size, void* workspace,
                    size_t workspace_bytes, void* stream) {
  return decode_impl(nullptr, nullptr, nullptr, out, q, k_cache, v_cache, cache, block_tables,
                     max_blocks_per_seq,
                     context_lens, num_seqs, num_q_heads, scale, max_context_len, partition_size,
                     workspace, workspace_bytes, stream);
}

size_t pa_decode_shared_prefix_workspace_size(int32_t num_seqs, int32_t num_q_heads,
                                              int32_t head_dim, int32_t max_context_len,
                                              int32_t shared_len, int32_t partition_size) {
  // pa_decode's layout with one more partition (the shared prefix's) in front
  if (num_seqs <= 0 || num_q_heads <= 0 || head_dim <= 0 || partition_size <= 0 ||
      shared_len < 0)
    return 0;
  const size_t counters = decode_counter_bytes(num_seqs, num_q_heads);
  const int64_t rest = max_context_len > shared_len ? max_context_len - shared_len : 0;
  const int64_t parts = 1 + (rest + partition_size - 1) / partition_size;
  return counters +
         static_cast<size_t>(num_seqs) * num_q_heads * parts * (head_dim + 2) * sizeof(float);
}

pa_status pa_decode_shared_prefix(void* out, const void* q, const void* k_cache,
                                  const void* v_cache, pa_cache_desc cache,
                                  const int32_t* block_tables, int32_t max_blocks_per_seq,
                                  const int32_t* context_lens, int32_t num_seqs,
                                  int32_t num_q_heads, float scale, int32_t max_context_len,
                                  const int32_t* shared_blocks, int32_t shared_len,
                                  int32_t partition_size, void* workspace,
                                  size_t workspace_bytes, void* stream) {
  if (shared_len == 0)
    return pa_decode(out, q, k_cache, v_cache, cache, block_tables, max_blocks_per_seq,
                     context_lens, num_seqs, num_q_heads, scale, max_context_len, partition_size,
                     workspace, workspace_bytes, stream);
  pa_status st = check_cache(cache);
  if (st != PA_OK) return st;
  if (num_seqs < 0 || num_q_heads <= 0 || max_blocks_per_seq <= 0 || max_context_len < 0 ||
      shared_len < 0)
    return PA_ERR_INVALID_ARG;
  if (num_q_heads % cache.num_kv_heads || !std::isfinite(scale)) return PA_ERR_INVALID_ARG;
  if (static_cast<int64_t>(max_context_len) >
          static_cast<int64_t>(max_blocks_per_seq) * cache.block_size ||
      static_cast<int64_t>(shared_len) >
          static_cast<int64_t>(max_blocks_per_seq) * cache.block_size)
    return PA_ERR_INVALID_ARG;
  const int G = num_q_heads / cache.num_kv_heads;
  if (cache.head_dim != 128 || (G != 1 && G != 2 && G != 4 && G != 8 && G != 16) ||
      shared_len % 128 != 0)
    return PA_ERR_UNSUPPORTED;
  if (num_seqs == 0) return PA_OK;
  if (!out || !q || !k_cache || !v_cache || !block_tables || !context_lens || !shared_blocks)
    return PA_ERR_INVALID_ARG;
  if (!aligned16(out) || !aligned16(q) || !aligned16(k_cache) || !aligned16(v_cache))
    return PA_ERR_INVALID_ARG;
  if (partition_size < 0 || (partition_size % 128) != 0 || partition_size > 2048)
    return partition_size < 0 || partition_size % 64 ? PA_ERR_INVALID_ARG : PA_ERR_UNSUPPORTED;
  const int32_t rest = max_context_len > shared_len ? max_context_len - shared_len : 0;
  const int P = partition_size > 0
                    ? partition_size
                    : pa_decode_default_partition(num_seqs, cache.num_kv_heads, rest > 0 ? rest : 1);
  const int64_t parts64 = 1 + (static_cast<int64_t>(rest) + P - 1) / P;
  if (parts64 * num_seqs * cache.num_kv_heads >= (1ll << 24) - 4096) return PA_ERR_UNSUPPORTED;
  const size_t need = pa_decode_shared_prefix_workspace_size(num_seqs, num_q_heads, cache.head_dim,
                                                             max_context_len, shared_len, P);
  if (!workspace || workspace_bytes < need || !aligned16(workspace)) return PA_ERR_INVALID_ARG;
  DecodeLaunch a;
  a.out = out;
  a.q = q;
  a.k_cache = k_cache;
  a.v_cache = v_cache;
  a.cache = cache;
  a.block_tables = block_tables;
  a.max_blocks_per_seq = max_blocks_per_seq;
  a.context_lens = context_lens;
  a.num_seqs = num_seqs;
  a.num_q_heads = num_q_heads;
  a.scale = scale;
  a.max_context_len = max_context_len;
  a.partition_size = P;
  a.max_parts = static_cast<int>(parts64);
  a.shared_len = shared_len;
  const size_t cbytes = decode_counter_bytes(num_seqs, num_q_heads);
  unsigned long long* counters = static_cast<unsigned long long*>(workspace);
  float* ws = reinterpret_cast<float*>(static_cast<uint8_t*>(workspace) + cbytes);
  a.ws_o = ws;
  a.ws_ml = ws + static_cast<size_t>(num_seqs) * num_q_heads * a.max_parts * cache.head_dim;
  const cudaStream_t s = static_cast<cudaStream_t>(stream);
  cudaError_t e = launch_shared_prefix(a, shared_blocks, shared_len, s);
  if (e == cudaSuccess && rest > 0) e = launch_decode_tc(a, counters, s);
  return finish(e, stream);
}

pa_status pa_store_decode(const void* new_k, const void* new_v, const int32_t* slot_mapping,
                          void* out, const void* q, void* k_cache, void* v_cache,
                          pa_cache_desc cache, const int32_t* block_tables,
                          int32_t max_blocks_per_seq, const int32_t* context_lens,
                          int32_t num_seqs, int32_t num_q_heads, float scale,
                          int32_t max_context_len, int32_t partition_size, void* workspace,
                          size_t workspace_bytes, void* stream) {
  const StoreRows rows{new_k, new_v, slot_mapping};
  return decode_impl(&rows, nullptr, nullptr, out, q, k_cache, v_cache, cache, block_tables,
                     max_blocks_per_seq,
                     context_lens, num_seqs, num_q_heads, scale, max_context_len, partition_size,
                     workspace, workspace_bytes, stream);
}

pa_status pa_store_kvcache_fp8(const void* k, const void* v, void* k_codes, void* v_codes,
                               float* k_scales, float* v_scales, pa_cache_desc cache,
                               const int32_t* slot_mapping, int32_t num_tokens, void* stream) {
  pa_status st = check_cache(cache);
  if (st != PA_OK) return st;
  if (num_tokens < 0) return PA_ERR_INVALID_ARG;
  if (num_tokens == 0) return PA_OK;
  if (!k || !v || !k_codes || !v_codes || !k_scales || !v_scales || !slot_mapping)
    return PA_ERR_INVALID_ARG;
  if (!aligned16(k) || !aligned16(v) || !aligned16(k_codes) || !aligned16(v_codes) ||
      !aligned16(k_scales) || !aligned16(v_scales))
    return PA_ERR_INVALID_ARG;
  return finish(launch_store_kvcache_fp8(k, v, k_codes, v_codes, k_scales, v_scales, cache,
                                         slot_mapping, num_tokens,
                                         static_cast<cudaStream_t>(stream)),
                stream);
}

pa_status pa_decode_fp8(void* out, const void* q, const void* k_codes, const void* v_codes,
                        const float* k_scales, const float* v_scales, pa_cache_desc cache,
                        const int32_t* block_tables, int32_t max_blocks_per_seq,
                        const int32_t* context_lens, int32_t num_seqs, int32_t num_q_heads,
                        float scale, int32_t max_context_len, int32_t partition_size,
                        void* workspace, size_t workspace_bytes, void* stream) {
  if (!k_scales || !v_scales) return PA_ERR_INVALID_ARG;
  return decode_impl(nullptr, k_scales, v_scales, out, q, k_codes, v_codes, cache, block_tables,
                     max_blocks_per_seq, context_lens, num_seqs, num_q_heads, scale,
                     max_context_len, partition_size, workspace, workspace_bytes, stream);
}

namespace {
pa_status prefill_impl(const StoreRows* store, void* out, const void* q, const void* k_cache,
                       const void* v_cache, pa_cache_desc cache, const int32_t* block_tables,
                       int32_t max_blocks_per_seq, const int32_t* cu_seqlens_q,
                       const int32_t* context_lens, int32_t num_seqs, int32_t num_q_heads,
                       int32_t total_q, int32_t max_q_len, float scale, void* stream) {
  pa_status st = check_cache(cache);
  if (st != PA_OK) return st;
  if (num_seqs < 0 || num_q_heads <= 0 || max_blocks_per_seq <= 0 || total_q < 0 ||
      max_q_len < 0)
    return PA_ERR_INVALID_ARG;
  if (num_q_heads % cache.num_kv_heads) return PA_ERR_INVALID_ARG;
  if (!std::isfinite(scale)) return PA_ERR_INVALID_ARG;
  if (cache.head_dim != 128) return PA_ERR_UNSUPPORTED;
  if (num_seqs == 0 || total_q == 0 || max_q_len == 0) return PA_OK;
  if (!out || !q || !k_cache || !v_cache || !block_tables || !cu_seqlens_q || !context_lens)
    return PA_ERR_INVALID_ARG;
  if (!aligned16(out) || !aligned16(q) || !aligned16(k_cache) || !aligned16(v_cache))
    return PA_ERR_INVALID_ARG;
  if (store && (!store->new_k || !store->new_v || !store->slot_mapping ||
                !aligned16(store->new_k) || !aligned16(store->new_v)))
    return PA_ERR_INVALID_ARG;
  PrefillLaunch a;
  a.out = out;
  a.q = q;
  a.k_cache = k_cache;
  a.v_cache = v_cache;
  a.cache = cache;
  a.block_tables = block_tables;
  a.max_blocks_per_seq = max_blocks_per_seq;
  a.cu_seqlens_q = cu_seqlens_q;
  a.context_lens = context_lens;
  a.num_seqs = num_seqs;
  a.num_q_heads = num_q_heads;
  a.max_q_len = max_q_len;
  a.total_q = total_q;
  a.scale = scale;
  if (store) {
    a.new_k = store->new_k;
    a.new_v = store->new_v;
    a.slot_mapping = store->slot_mapping;
  }
  return finish(launch_prefill(a, static_cast<cudaStream_t>(stream)), stream);
}
}  // namespace

pa_status pa_prefill(void* out, const void* q, const void* k_cache, const void* v_cache,
                     pa_cache_desc cache, const int32_t* block_tables, int32_t max_blocks_per_seq,
                     const int32_t* cu_seqlens_q, const int32_t* context_lens, int32_t num_seqs,
                     int32_t num_q_heads, int32_t total_q, int32_t max_q_len, float scale,
                     void* stream) {
  return prefill_impl(nullptr, out, q, k_cache, v_cache, cache, block_tables, max_blocks_per_seq,
                      cu_seqlens_q, context_lens, num_seqs, num_q_heads, total_q, max_q_len, scale,
                      stream);
}

pa_status pa_store_prefill(const void* new_k, const void* new_v, const int32_t* slot_mapping,
                           void* out, const void* q, void* k_cache, void* v_cache,
                           pa_cache_desc cache, const int32_t* block_tables,
                           int32_t max_blocks_per_seq, const int32_t* cu_seqlens_q,
                           const int32_t* context_lens, int32_t num_seqs, int32_t num_q_heads,
                           int32_t total_q, int32_t max_q_len, float scale, void* stream) {
  const StoreRows rows{new_k, new_v, slot_mapping};
  return prefill_impl(&rows, out, q, k_cache, v_cache, cache, block_tables, max_blocks_per_seq,
                      cu_seqlens_q, context_lens, num_seqs, num_q_heads, total_q, max_q_len, scale,
                      stream);
}

}  // extern "C"

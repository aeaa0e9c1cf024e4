/*
 * pa.h — C ABI of the B200 paged KV-cache library (libpa.so).
 *
 * The library keeps the keys and values of every sequence in a pre-allocated
 * pool of fixed-size blocks and reaches them through per-sequence block tables
 * (nano vllm KV-cache practice page, section 3.2.1 "Block设计" and section 3.1
 * "Sequence管理": each Sequence owns a block_table; mini-vllm page, section 2
 * "KVCache": the block table decides where in the pre-allocated GPU tensor K/V
 * are read and written).
 *
 * Conventions shared by every entry point
 * ---------------------------------------
 *  - All pointers are DEVICE pointers into memory the caller owns (allocated
 *    by the caller, e.g. through PyTorch). The library allocates no device
 *    memory and keeps no per-call state; scratch space is passed in.
 *  - bf16 tensors are dense, row-major, 16-byte aligned.
 *  - Pool layout (k_cache, v_cache): [num_blocks, block_size, num_kv_heads,
 *    head_dim] bf16. Logical position p of sequence s lives in pool row
 *        block_tables[s * max_blocks_per_seq + p / block_size] * block_size
 *        + p % block_size,
 *    a row being num_kv_heads * head_dim contiguous bf16 values.
 *  - block_tables: int32 [num_seqs, max_blocks_per_seq], unused entries -1.
 *  - context_lens: int32 [num_seqs], the number of positions of each sequence
 *    INCLUDING the tokens written in the current step.
 *  - Grouped-query attention: query head h reads kv head
 *    h / (num_q_heads / num_kv_heads).
 *  - Scores are scale * dot(q, k); softmax over the visible positions; the
 *    result is rounded once to bf16 (nearest even). Accumulation is fp32.
 *  - Calls are asynchronous on `stream` (a cudaStream_t; NULL = legacy
 *    default stream) and do not synchronise, except when debug checks are on
 *    (see pa_set_debug_checks).
 *
 * Errors
 * ------
 *  - Arguments are validated on the host before any launch; a bad argument
 *    returns PA_ERR_INVALID_ARG and launches nothing. Supported sizes:
 *    head_dim 64 or 128 for the store, copy and decode entry points, 128 only
 *    for pa_prefill, pa_store_prefill and pa_decode_fp8 (other head dims
 *    return PA_ERR_UNSUPPORTED there); block_size a power of two in
 *    [16, 1024]; num_q_heads a multiple of num_kv_heads.
 *  - A valid but unimplemented combination returns PA_ERR_UNSUPPORTED.
 *  - A failed launch returns PA_ERR_CUDA.
 *  - Device-side index checks never trap: an out-of-range block id or slot is
 *    recorded in a device error word and the access is redirected to row 0 of
 *    the pool (store: the write is skipped). The error word is read (and
 *    cleared) by pa_check_device_errors, which returns PA_ERR_BAD_INDEX, or
 *    PA_ERR_TIMEOUT if a bounded wait inside a kernel gave up.
 */
#ifndef PA_H_
#define PA_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
  PA_OK = 0,
  PA_ERR_INVALID_ARG = 1,
  PA_ERR_UNSUPPORTED = 2,
  PA_ERR_BAD_INDEX = 3,
  PA_ERR_CUDA = 4,
  PA_ERR_TIMEOUT = 5,
  PA_ERR_NO_BLOCKS = 6  /* block manager: the pool has no free block left */
} pa_status;

/* Shape of the paged pool (both k_cache and v_cache have this shape). */
typedef struct {
  int32_t num_blocks;   /* physical blocks in the pool                     */
  int32_t block_size;   /* token positions per block (power of two)        */
  int32_t num_kv_heads; /* Hkv                                             */
  int32_t head_dim;     /* D: 64 or 128                                    */
} pa_cache_desc;

/*
 * pa_store_kvcache — write the K/V rows of this step's new tokens into the pool.
 *
 * Defines: k_cache[slot_mapping[t]] = k[t] and v_cache[slot_mapping[t]] = v[t]
 * for every t with slot_mapping[t] >= 0 (mini-vllm page, section 2: the block
 * table decides where K/V are written; the caller turns (sequence, position)
 * into a pool row ("slot") with the row formula above).
 *
 *   k, v          [num_tokens, Hkv, D] bf16, read only.
 *   k_cache,
 *   v_cache       pool, written in place (only the mapped rows change).
 *   slot_mapping  int32 [num_tokens]; -1 skips the token. Two tokens mapped to
 *                 one slot is a caller error (the surviving row is unspecified).
 *   num_tokens    >= 0; 0 is a no-op.
 * A slot >= num_blocks * block_size is skipped and flags PA_ERR_BAD_INDEX.
 */
pa_status pa_store_kvcache(const void* k, const void* v, void* k_cache, void* v_cache,
                           pa_cache_desc cache, const int32_t* slot_mapping,
                           int32_t num_tokens, void* stream);

/*
 * Host block manager (no device memory, no CUDA calls): which physical block of the
 * pool each block of a request lives in, and which blocks requests share (nano vllm
 * page, section 3.2: Block = id, reference count, hash, token ids; BlockManager
 * reuses a full block whose chained hash is registered and whose tokens match, else
 * takes a free block and registers it; section 4.2: rolling hash h = h * 31 + token
 * mod 2^32 seeded with the previous block's hash; mini-vllm page, section 1: the
 * BlockAllocator hands out blocks and takes them back). Readings: a trailing partial
 * block whose prefix chain matched reuses a cached full block it is a prefix of; free
 * blocks are taken in the order given at creation; a freed block forgets its hash.
 * All pointers are host pointers. A manager is not thread-safe: calls on one manager
 * must not overlap.
 */
typedef struct pa_block_manager pa_block_manager;

/* num_blocks blocks of block_size positions; free_order: int32 [num_blocks], a
 * permutation of the pool giving the order free blocks are taken (NULL = 0, 1, ...).
 * Returns NULL for bad sizes or a free_order that is not a permutation. */
pa_block_manager* pa_bm_create(int32_t num_blocks, int32_t block_size, const int32_t* free_order);
void pa_bm_destroy(pa_block_manager* bm);

/* The block table of one request: token_ids int32 [num_tokens] (non-negative);
 * table_out int32 [ceil(num_tokens / block_size)]. block_hashes: NULL (hashes are
 * computed here) or uint32 [num_tokens / block_size], the chained hash of each full
 * block as pa_block_hashes computes it. PA_ERR_NO_BLOCKS when the pool runs out: the
 * request then holds no block (the blocks it had taken go back to the free list). */
pa_status pa_bm_allocate(pa_block_manager* bm, const int32_t* token_ids, int32_t num_tokens,
                         const uint32_t* block_hashes, int32_t* table_out);

/* pa_bm_allocate for a batch of requests in one call, in order (a scheduler admitting
 * a step's prefills). token_ids: the requests back to back; cu_tokens int32
 * [num_seqs + 1] (cu_tokens[0] = 0) their offsets. block_hashes: NULL, or each
 * request's full-block hashes back to back at offsets cu_blocks [num_seqs + 1]
 * (cu_blocks[s+1] - cu_blocks[s] = length_s / block_size). tables_out: every request's
 * table back to back, ceil(length_s / block_size) entries each. *num_done: the number
 * of requests allocated. When the pool runs out at request s, the call returns
 * PA_ERR_NO_BLOCKS with *num_done = s: requests 0..s-1 keep their blocks (free them,
 * or run them), request s holds nothing. Bad offsets and negative token ids return
 * PA_ERR_INVALID_ARG before any block is taken. */
pa_status pa_bm_allocate_batch(pa_block_manager* bm, const int32_t* token_ids,
                               const int32_t* cu_tokens, int32_t num_seqs,
                               const uint32_t* block_hashes, const int32_t* cu_blocks,
                               int32_t* tables_out, int32_t* num_done);

/* A finished request: one reference dropped per entry; blocks reaching zero go back to
 * the free list. An id outside the pool or a block released more often than it is held
 * returns PA_ERR_INVALID_ARG and changes nothing. */
pa_status pa_bm_free(pa_block_manager* bm, const int32_t* table, int32_t num_entries);

/* Decode append of token_id at position pos (the sequence's current length) of a
 * request whose table has *num_entries entries (room for capacity). Writes the slot
 * (block * block_size + pos % block_size) to slot_out. A position that starts a block
 * appends a fresh block to the table. A block other requests also hold is replaced by
 * a private copy: the table entry changes and *copy_src -> *copy_dst is the copy the
 * step must make first (pa_copy_blocks); otherwise both are -1. A private block still
 * registered under a hash leaves the hash map before it is written. */
pa_status pa_bm_append(pa_block_manager* bm, int32_t* table, int32_t* num_entries, int32_t capacity,
                       int32_t pos, int32_t token_id, int32_t* slot_out, int32_t* copy_src,
                       int32_t* copy_dst);

/* Blocks with a reference count above zero (-1 for a NULL manager). */
int32_t pa_bm_num_used(const pa_block_manager* bm);
/* Reference count of every block: out int32 [num_blocks]. */
pa_status pa_bm_ref_counts(const pa_block_manager* bm, int32_t* out);

/*
 * pa_block_hashes — the chained hash of every full block of a batch of token
 * sequences on the GPU (the hash of nano vllm page, section 4.2, as above; the first
 * block of a sequence is seeded with 0), for pa_bm_allocate. Device pointers:
 *   token_ids   int32 [cu_tokens[num_seqs]], the sequences back to back;
 *   cu_tokens   int32 [num_seqs + 1], token offsets;
 *   cu_blocks   int32 [num_seqs + 1], offsets of each sequence's full blocks in
 *               hashes_out (cu_blocks[s+1] - cu_blocks[s] = length_s / block_size);
 *   hashes_out  uint32 [cu_blocks[num_seqs]].
 * One warp per sequence: each lane hashes whole blocks on its own, then the lanes
 * chain them with a scan (the chained hash of a prefix is a polynomial in 31).
 * Offsets that disagree (a block count other than length_s / block_size) are
 * clamped to the sequence's own tokens, so nothing is read past them; the hashes
 * past the clamp are not written, and the mismatch is reported as PA_ERR_BAD_INDEX
 * (debug checks / pa_check_device_errors).
 */
pa_status pa_block_hashes(const int32_t* token_ids, const int32_t* cu_tokens,
                          const int32_t* cu_blocks, int32_t num_seqs, int32_t block_size,
                          uint32_t* hashes_out, void* stream);

/*
 * pa_copy_blocks — copy-on-write of shared blocks. Blocks are shared between
 * sequences by reference count (nano vllm page, section 3.2.1); the page does not
 * say what happens when a sequence writes into a shared block, and the reading
 * taken here is that the writer first gets a private copy, so the other sharers
 * keep reading the unchanged block. For every i, block dst_blocks[i] of both pools
 * becomes a copy of block src_blocks[i] (all block_size x Hkv x D values of K and
 * of V).
 *
 *   src_blocks, dst_blocks  int32 [num_pairs], device. Destinations must be
 *                  distinct and must not also be sources in the same call (the
 *                  pairs are copied in no particular order). A pair with an id
 *                  outside the pool is skipped and reported as PA_ERR_BAD_INDEX
 *                  (debug checks / pa_check_device_errors); src == dst is a no-op.
 * Moves 4 x block_size x Hkv x D x 2 bytes per pair (read and write, K and V).
 */
pa_status pa_copy_blocks(void* k_cache, void* v_cache, pa_cache_desc cache,
                         const int32_t* src_blocks, const int32_t* dst_blocks, int32_t num_pairs,
                         void* stream);

/*
 * Decode split size. The context of every sequence is cut into partitions of
 * partition_size positions (a multiple of 64); each (sequence, kv head,
 * partition) is processed independently and the partials are merged at the end
 * (inside the persistent kernel on the tensor-core path, by a second kernel on
 * the CUDA-core path). pa_decode_default_partition returns the size pa_decode picks when
 * given partition_size = 0 (depends on the batch, heads, max context and the
 * device's SM count of the current device).
 */
int32_t pa_decode_default_partition(int32_t num_seqs, int32_t num_kv_heads,
                                    int32_t max_context_len);

/*
 * Bytes of scratch pa_decode needs for these sizes (> 0 whenever num_seqs > 0):
 * a 256-byte-aligned region of 1 + num_seqs * num_q_heads 64-bit work/arrival
 * counters, then, when the context is split into more than one partition, the
 * fp32 partials [num_seqs, Hq, parts, D] and their (max, sum) pairs
 * [num_seqs, Hq, parts, 2].
 */
size_t pa_decode_workspace_size(int32_t num_seqs, int32_t num_q_heads, int32_t head_dim,
                                int32_t max_context_len, int32_t partition_size);

/*
 * pa_decode — one query token per sequence attends over its whole paged
 * context (mini-vllm page, "性能评估与基准测试": in the decode phase only the one
 * new token is computed; its K/V must already be stored, so context_lens[s]
 * counts it).
 *
 *   out            [num_seqs, Hq, D] bf16, written.
 *   q              [num_seqs, Hq, D] bf16.
 *   block_tables   int32 [num_seqs, max_blocks_per_seq].
 *   context_lens   int32 [num_seqs]; a sequence with length <= 0 gets zeros.
 *   scale          softmax scale (1/sqrt(D) for standard attention).
 *   max_context_len  host upper bound of context_lens (sizes the split); a
 *                  larger device value is clipped to it and flags
 *                  PA_ERR_BAD_INDEX.
 *   partition_size 0 = automatic, else a multiple of 64.
 *   workspace      device scratch of at least pa_decode_workspace_size(...)
 *                  bytes for the partition size used; its contents on entry do
 *                  not matter (its counters carry a tag unique to each call, so
 *                  leftovers of earlier calls never count). Calls that overlap
 *                  on the GPU must use different workspaces.
 *                  CUDA graphs: the tag is drawn on the host when the call is
 *                  made, so a captured call replays with its capture's tag. Clear
 *                  the workspace's leading counter block (the 256-byte-rounded
 *                  8 * (1 + num_seqs * num_q_heads) bytes) before each replay, e.g.
 *                  with a memset node ahead of it in the same graph; a replay is
 *                  then exactly a fresh call. The same holds for pa_store_decode
 *                  and pa_decode_fp8. pa_decode_no_alloc's scratch belongs to the
 *                  library and cannot be cleared by the caller: do not capture it.
 * Supported: Hq / Hkv in {1, 2, 4, 8} (and 16 when head_dim is 128).
 * head_dim 128 runs the persistent tcgen05 kernel (partition_size a multiple
 * of 128, at most 2048; other sizes run the CUDA-core kernel); head_dim 64 runs
 * the CUDA-core kernel.
 */
pa_status pa_decode(void* out, const void* q, const void* k_cache, const void* v_cache,
                    pa_cache_desc cache, const int32_t* block_tables,
                    int32_t max_blocks_per_seq, const int32_t* context_lens, int32_t num_seqs,
                    int32_t num_q_heads, float scale, int32_t max_context_len,
                    int32_t partition_size, void* workspace, size_t workspace_bytes,
                    void* stream);

/*
 * pa_store_decode — one decode step of a layer in one call: store this step's
 * new K/V row of every sequence, then attend (nano vllm page, section 3.1: the
 * new token's slot is the next position of the sequence's last block; mini-vllm
 * page, section 2: K/V are written where the block table points, then read
 * through it). The result, and the pool afterwards, equal pa_store_kvcache
 * followed by pa_decode with the same arguments.
 *
 *   new_k, new_v   [num_seqs, Hkv, D] bf16: the new token's K and V rows.
 *   slot_mapping   int32 [num_seqs]: -1 = store nothing for that sequence, else
 *                  the slot of position context_lens[s] - 1 of sequence s
 *                  (block_tables[s][(ctx-1) / bs] * bs + (ctx-1) % bs). Any other
 *                  value is not stored and is reported as PA_ERR_BAD_INDEX (debug
 *                  checks / pa_check_device_errors): the row is written by the
 *                  part of the kernel that reads that position, just before it
 *                  reads it, so a slot elsewhere could be read before it is written.
 *                  The slot must not be read by another sequence of the same call
 *                  (a block shared by several sequences is copied before it is
 *                  appended to).
 *   other arguments as pa_decode.
 * On the tensor-core path (head dim 128, partition size a multiple of 128 up to
 * 2048) the store happens inside the decode kernel: one launch per step. Other
 * shapes launch a checked store kernel and then the decode kernels.
 */
pa_status pa_store_decode(const void* new_k, const void* new_v, const int32_t* slot_mapping,
                          void* out, const void* q, void* k_cache, void* v_cache,
                          pa_cache_desc cache, const int32_t* block_tables,
                          int32_t max_blocks_per_seq, const int32_t* context_lens,
                          int32_t num_seqs, int32_t num_q_heads, float scale,
                          int32_t max_context_len, int32_t partition_size, void* workspace,
                          size_t workspace_bytes, void* stream);

/*
 * pa_decode_shared_prefix — pa_decode for a batch whose sequences all start with the
 * same shared_len positions held in the same physical blocks (nano vllm page, section
 * 3.2.2: requests with a common prompt share reference-counted blocks; the block
 * manager that handed them out knows how long the common part is). The shared
 * prefix is attended once for all sequences: one dense tensor-core pass per kv head
 * over every sequence's query rows (each row sees min(context_lens[s], shared_len)
 * of the prefix), whose result is the output row of a context that ends inside the
 * prefix and the first split-K partial of a longer one; the persistent decode then
 * reads only the positions past the prefix and merges. Two launches on `stream`.
 *
 *   shared_blocks  int32 [shared_len / block_size], device: the physical blocks of
 *                  the shared prefix. Every sequence's block table must hold them at
 *                  the prefix positions it uses (b * block_size < context_lens[s]); a
 *                  difference is reported as PA_ERR_BAD_INDEX. The prefix is read
 *                  through shared_blocks.
 *   shared_len     a multiple of 128 (0 = pa_decode).
 *   workspace      at least pa_decode_shared_prefix_workspace_size(...) bytes for the
 *                  partition size used (partition_size 0 = automatic, sized on the
 *                  positions past the prefix).
 *   other arguments as pa_decode. Supported: head_dim 128, Hq / Hkv in {1, 2, 4, 8,
 *   16}, partition_size a multiple of 128 up to 2048; else PA_ERR_UNSUPPORTED.
 * The result equals pa_decode's within the same rounding (the positions are summed in
 * another grouping); CUDA graphs: as pa_decode (clear the counter block).
 */
size_t pa_decode_shared_prefix_workspace_size(int32_t num_seqs, int32_t num_q_heads,
                                              int32_t head_dim, int32_t max_context_len,
                                              int32_t shared_len, int32_t partition_size);
pa_status pa_decode_shared_prefix(void* out, const void* q, const void* k_cache,
                                  const void* v_cache, pa_cache_desc cache,
                                  const int32_t* block_tables, int32_t max_blocks_per_seq,
                                  const int32_t* context_lens, int32_t num_seqs,
                                  int32_t num_q_heads, float scale, int32_t max_context_len,
                                  const int32_t* shared_blocks, int32_t shared_len,
                                  int32_t partition_size, void* workspace,
                                  size_t workspace_bytes, void* stream);

/*
 * pa_decode_no_alloc — pa_decode for callers that cannot allocate device memory.
 * (The pages have no counterpart: this is an interface convenience, not a step of
 * the method.)
 *
 * Some callers have no way to provide pa_decode's workspace: a serving runtime
 * that carves the GPU into fixed pools at start-up and allows no allocation
 * afterwards, or a host program that drives this library only through its C ABI
 * without access to a CUDA allocator. This entry point takes the same arguments
 * as pa_decode minus the workspace, and uses instead a scratch array of
 * PA_DECODE_NO_ALLOC_SCRATCH_BYTES that the library owns: a device array that
 * every GPU loading the library holds until the process exits. It allocates
 * nothing and calls no allocator. The caller still passes inputs and outputs.
 *
 *  - Every call looks up the array's device address (cudaGetSymbolAddress,
 *    with the device current; a host-side lookup, so a device reset never leaves
 *    a stale address behind). The first call on a device may load the library's
 *    device code; make that first call before any stream capture.
 *  - Sizes whose split-K scratch (pa_decode_workspace_size for the partition
 *    used) exceeds PA_DECODE_NO_ALLOC_SCRATCH_BYTES are rejected with
 *    PA_ERR_UNSUPPORTED and nothing is launched; pass a larger partition_size
 *    or use pa_decode.
 *  - Every call on a device shares the one array and it keeps the last call's
 *    contents; nothing in it has to start at zero (each partial is written
 *    before it is read, and the counters carry a tag unique to each call).
 *    Calls that overlap on the GPU (e.g. on two streams without ordering
 *    between them) race on the array: order them.
 */
#define PA_DECODE_NO_ALLOC_SCRATCH_BYTES (8u * 1024u * 1024u)
pa_status pa_decode_no_alloc(void* out, const void* q, const void* k_cache, const void* v_cache,
                             pa_cache_desc cache, const int32_t* block_tables,
                             int32_t max_blocks_per_seq, const int32_t* context_lens,
                             int32_t num_seqs, int32_t num_q_heads, float scale,
                             int32_t max_context_len, int32_t partition_size, void* stream);

/*
 * fp8 (e4m3) KV cache. The nano vllm KV-cache practice page lists quantisation
 * support among its extensions (section 5.3 "扩展建议") and the Nano-vLLM
 * architecture page names quantised compression as a further direction (section 7
 * "总结与展望"); neither fixes a format, so the readings taken here are:
 *  - values are OCP fp8 e4m3 codes (bias 7, no infinities, largest finite 448);
 *  - every (pool row, kv head) pair of D values has its own fp32 scale, chosen when
 *    the row is written (a decode step writes one row of a block at a time, so a
 *    per-block scale could not be fixed before the block is full);
 *  - a row x is quantised in fp32: amax = max |x|; amax == 0 gives codes 0 and
 *    scale 0; else code_i = e4m3(x_i * (448 / amax)), rounded to nearest even and
 *    saturated to +-448, and scale = amax / 448 (both divisions rounded to nearest);
 *  - a stored value reads back as e4m3(code) * scale.
 * Pools: codes uint8 [num_blocks, block_size, Hkv, D] (the bf16 pool's row
 * layout with one byte per value); scales fp32 [Hkv, num_blocks * block_size]
 * (kv head major: the scales of one kv head's consecutive pool rows are
 * contiguous). Halves the bytes a decode step reads.
 */

/*
 * pa_store_kvcache_fp8 — pa_store_kvcache into e4m3 pools: row slot_mapping[t] of
 * k_codes / v_codes receives the quantised k[t] / v[t] and k_scales / v_scales
 * [g][slot_mapping[t]] the scale of kv head g's row. k, v: [num_tokens, Hkv, D]
 * bf16. Skipped and bad slots as in pa_store_kvcache. head_dim 64 or 128.
 */
pa_status pa_store_kvcache_fp8(const void* k, const void* v, void* k_codes, void* v_codes,
                               float* k_scales, float* v_scales, pa_cache_desc cache,
                               const int32_t* slot_mapping, int32_t num_tokens, void* stream);

/*
 * pa_decode_fp8 — pa_decode over e4m3 pools: the attention of the values the
 * pools hold (code * scale). The tensor cores read the stored codes directly
 * (e4m3 x e4m3 products, fp32 accumulation); no code is converted. Each row's K
 * scale multiplies that position's score, and each row's V scale its probability,
 * in fp32. q reaches the tensor cores as three e4m3 terms (about 2^-13 relative
 * per element: a score's error is multiplied by the score's size in the exponent,
 * so peaked softmaxes need q this exact) and the probabilities as two (a high term
 * and the scaled remainder: about 2^-8 relative per element). Arguments as pa_decode, with the pools replaced by codes
 * and scales (16-byte aligned). Values whose products overflow fp32 are out of
 * range (as for pa_decode).
 * Supported: head_dim 128, Hq / Hkv in {1, 2, 4, 8, 16}, partition_size (given or
 * automatic) a multiple of 128 up to 2048; anything else returns
 * PA_ERR_UNSUPPORTED (there is no CUDA-core fp8 path).
 */
pa_status pa_decode_fp8(void* out, const void* q, const void* k_codes, const void* v_codes,
                        const float* k_scales, const float* v_scales, pa_cache_desc cache,
                        const int32_t* block_tables, int32_t max_blocks_per_seq,
                        const int32_t* context_lens, int32_t num_seqs, int32_t num_q_heads,
                        float scale, int32_t max_context_len, int32_t partition_size,
                        void* workspace, size_t workspace_bytes, void* stream);

/*
 * pa_prefill — causal attention of a chunk of new tokens appended to each
 * sequence's cached prefix (nano vllm page, section 3.1: num_cached_tokens of a
 * Sequence are reused; mini-vllm page, section 1: blocks are allocated for the
 * prefill). The new tokens' K/V must already be in the pool
 * (pa_store_kvcache), so every K/V read goes through the block table.
 *
 *   out, q         [total_q, Hq, D] bf16 (varlen: sequence s owns rows
 *                  cu_seqlens_q[s] .. cu_seqlens_q[s+1]-1).
 *   total_q        rows of q and out (= cu_seqlens_q[num_seqs]); q is never
 *                  read past it.
 *   cu_seqlens_q   int32 [num_seqs + 1], non-decreasing, cu_seqlens_q[0] = 0.
 *   context_lens   int32 [num_seqs]; new token i of sequence s sits at position
 *                  context_lens[s] - n_new + i and sees positions 0..that one.
 *                  Requires n_new <= context_lens[s].
 *   max_q_len      host upper bound of the new tokens of one sequence.
 * Uses the tcgen05 tensor cores; head_dim must be 128.
 */
pa_status pa_prefill(void* out, const void* q, const void* k_cache, const void* v_cache,
                     pa_cache_desc cache, const int32_t* block_tables,
                     int32_t max_blocks_per_seq, const int32_t* cu_seqlens_q,
                     const int32_t* context_lens, int32_t num_seqs, int32_t num_q_heads,
                     int32_t total_q, int32_t max_q_len, float scale, void* stream);

/*
 * pa_store_prefill — one chunked-prefill step of a layer in one call: store the new
 * tokens' K/V rows, then attend (nano vllm page, section 3.1: the new tokens follow
 * the num_cached_tokens of a Sequence in its blocks; mini-vllm page, section 2: K/V are
 * written where the block table points, then read through it). The result, and the
 * pool afterwards, equal pa_store_kvcache followed by pa_prefill with the same
 * arguments.
 *
 *   new_k, new_v   [total_q, Hkv, D] bf16: the K and V rows of the new tokens, in the
 *                  token order of q (sequence s owns rows cu_seqlens_q[s] ..).
 *   slot_mapping   int32 [total_q]: the slot of each new token, which must be the slot
 *                  the block table gives for its position (context_lens[s] - n_new + i
 *                  for new token i of sequence s), or -1 (not stored). Any other value
 *                  is not stored and is reported as PA_ERR_BAD_INDEX (debug checks /
 *                  pa_check_device_errors).
 *   other arguments as pa_prefill.
 * The attention reads the new tokens' rows from new_k / new_v directly (the bits the
 * store writes), so the launch has no ordering between its store and its reads; the
 * rows reach the pool in the same launch. A slot of -1 therefore still attends to the
 * row in new_k / new_v (store then prefill would read the pool's old row there).
 */
pa_status pa_store_prefill(const void* new_k, const void* new_v, const int32_t* slot_mapping,
                           void* out, const void* q, void* k_cache, void* v_cache,
                           pa_cache_desc cache, const int32_t* block_tables,
                           int32_t max_blocks_per_seq, const int32_t* cu_seqlens_q,
                           const int32_t* context_lens, int32_t num_seqs, int32_t num_q_heads,
                           int32_t total_q, int32_t max_q_len, float scale, void* stream);

/*
 * Debug mode: when on, every entry point synchronises its stream after the
 * launch and returns the device error status (see pa_check_device_errors).
 */
void pa_set_debug_checks(int on);

/*
 * Test hook: the time limit, in nanoseconds, of the waits between the cooperating
 * roles (data movement, tensor-core issue, softmax, epilogue) inside the
 * tensor-core kernels of later calls; 0 restores the default of 2 s. A wait that
 * runs out records PA_ERR_TIMEOUT in the device error word and the kernel winds
 * down: every role leaves its loop, each CTA still waits (with the full 2 s limit)
 * for the copies and tensor-core operations it has started, frees its tensor
 * memory and returns, so the context stays usable and the next call is a normal
 * one. Outputs of a call that timed out are unspecified. Exists so that tests can
 * make a wait run out without a fault; a serving process leaves it alone.
 */
void pa_set_wait_limit_ns(uint64_t ns);

/*
 * Synchronise `stream`, read and clear this device's error word.
 * Returns PA_OK, PA_ERR_BAD_INDEX, PA_ERR_TIMEOUT or PA_ERR_CUDA.
 */
pa_status pa_check_device_errors(void* stream);

/* Human-readable name of a status (static string). */
const char* pa_status_string(pa_status s);

/* Library ABI version (major * 100 + minor). */
int32_t pa_version(void);

#ifdef __cplusplus
}
#endif

#endif /* PA_H_ */

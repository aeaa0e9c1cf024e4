// Paged decode attention on the tcgen05 tensor cores (head dim 128), persistent.
//
// One query token per sequence attends over its paged context (mini-vllm page,
// "性能评估与基准测试": decode computes only the new token; KVCache reads K/V where
// the block table points, section 2). The work is HBM-bound: every K/V byte is read
// once per step. The tensor cores only take the G-query GEMV of each kv head off the
// CUDA cores:  S^T = K Q^T  (M = 128 positions, N = 16 padded query heads, K = 128
// head dims) and  O^T += V^T P^T  (M = 128 head dims, N = 16, K = 128 positions),
// both with fp32 accumulators in tensor memory.
//
// Grid: one CTA per SM looping over work items (partition p, sequence s, kv head g)
// taken from a counter in the workspace, so load balances dynamically and the TMA
// ring never drains between items. Roles (352 threads):
//   warp 10 scheduler: takes the next item from the counter, skips empty partitions
//           (writing zero rows for empty contexts) and reads the item's block ids, one
//           item ahead of the producer;
//   warp 4  producer: loads q (one box per item) and the K and V tiles
//           of 128 positions through the block table (one TMA box per physical
//           block) into two 3-deep rings of 32 KB slots. A K slot frees as soon as
//           its score MMA is done and a V slot when its value MMA is done, so both
//           streams run about two tiles ahead of the consumers (the fetch latency,
//           ~1.4 us per tile, must overlap; a shared K+V slot held until the value MMA
//           left one tile in flight);
//   warp 5  tensor-core issuer: owns the TMEM allocation; for tile j it issues S^T(j)
//           and then O^T += V^T P^T for tile j-1, and the last tile's value MMA of an
//           item right away so the item's epilogue never waits on the next item;
//   warps 0-3  softmax: thread r owns position r of a tile (TMEM lane r): per-head
//           tile max across the 128 positions, exp2 against a per-item reference max,
//           P^T to shared memory as bf16. O^T is rescaled in TMEM only when a tile's
//           max exceeds the reference by more than 2^8 (so probabilities stay <= 256,
//           exact in fp32 and bf16 range) — the only step that waits for the previous
//           value MMA. At the end of an item they post (m, l) and move on;
//   warps 6-9  epilogue: thread d owns output dim d (TMEM lane d) of the item's O^T
//           (one of three accumulators, so the epilogue of item k overlaps items k+1
//           and k+2) and writes the output row (single partition) or the partial
//           (m, l, o); the CTA completing the last partition of a (sequence, kv head)
//           merges them (split-K merge in the same kernel).
// Counters in the workspace carry a per-call tag, so an earlier call's leftovers never
// count: the workspace needs no clearing between calls.
//
// fp8 variant (pa_decode_fp8): the pools hold e4m3 codes with one fp32 scale per
// (position, kv head) row. The producer loads a tile's codes into the upper half of
// its 32 KB ring slot and the tile's scales (one box per block, each on a 128-byte
// boundary) into a small area of the slot's own; converter warps (11-18 for up to 4
// query heads per kv head, two threads per row; 11-14 for 8, one thread per row)
// dequantise it in place: one of them waits for the bytes while the rest sleep in a
// named barrier, each thread reads its share of a row's 128 codes and the row's scale
// into registers, and after a warp sync (a row's upper-half bf16 covers only its own
// codes) writes the row as bf16 (code * scale, rounded once) into both swizzled
// halves. The score, softmax, value and merge stages are the bf16 ones, unchanged.
#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <cuda_fp8.h>

#include <atomic>
#include <ctime>

#include "pa_internal.h"
#include "pa_ptx.cuh"

namespace pa {
namespace {

constexpr int TM = 128;        // positions per tile
constexpr int HD = 128;        // head dim
constexpr int NQ = 16;         // MMA N: query heads of one kv head, padded
constexpr int NK = 3;          // K ring depth (a slot frees when its score MMA is done)
constexpr int NV = 3;          // V ring depth (a slot frees when its value MMA is done)
constexpr int NS = 4;          // S^T buffers in TMEM
constexpr int NP = 4;          // P^T buffers in shared memory
constexpr int QN = 2;          // item queue depth (producer -> issuer, softmax)
constexpr int QS = 2;          // scheduler queue depth: one item prepared ahead (deeper
                               // queues reserve work early and unbalance the tail)
constexpr int NO = 3;          // O^T accumulators in TMEM (one per item in flight)
constexpr int kThreads = 352;  // softmax 0-3, producer 4, issuer 5, epilogue 6-9, scheduler 10
constexpr int kConvWarp0 = 11;   // fp8 pools: converter warps follow the scheduler
// fp8: 8 converter warps (two threads per row of a tile) where the other roles fit in
// the registers that leaves (608 threads: up to 4 query heads per kv head), else 4
template <int G>
constexpr int conv_warps() { return G <= 4 ? 8 : 4; }
template <int G, bool F8>
constexpr int tc_threads() { return kThreads + (F8 ? 32 * conv_warps<G>() : 0); }
constexpr float kRescaleLog2 = 8.f;  // rescale O only when the max grows by more than this
constexpr int kRegion = TM * 128;            // 64 head dims x 128 positions (16 KB)
constexpr int kTileBytes = 2 * kRegion;      // one K or V tile (32 KB)
constexpr int kQRegion = NQ * 128;           // 16 rows x 64 elements (2 KB)
constexpr int kQBytes = 2 * kQRegion;
constexpr int kPBytes = 2 * kQRegion;        // P^T: 16 heads x 128 positions, bf16
constexpr int kMaxIds = 2048 / 16 + 2;       // block ids of one item (partition <= 2048)

constexpr int align_up(int x, int a) { return (x + a - 1) / a * a; }

// every region starts on a 16-byte boundary (1024 for the swizzled operand tiles);
// the static_asserts below keep it that way when depths change
constexpr int kOffK = 0;
constexpr int kOffV = kOffK + NK * kTileBytes;
constexpr int kOffQ = kOffV + NV * kTileBytes;
constexpr int kOffP = kOffQ + QN * kQBytes;
constexpr int kOffRed = kOffP + NP * kPBytes;                     // [3][4 warps][NQ] floats
constexpr int kOffIds = align_up(kOffRed + 3 * 4 * NQ * 4, 16);
constexpr int kOffSched = align_up(kOffIds + QS * kMaxIds * 4, 16);  // [QS] descriptors
constexpr int kOffSchedFb = align_up(kOffSched + QS * 32, 16);       // [QS] first blocks
constexpr int kOffDesc = align_up(kOffSchedFb + QS * 4, 16);         // [QN] item descriptors
constexpr int kOffEpi = align_up(kOffDesc + QN * 32, 16);            // [NO] hand-offs
constexpr int kEpiBytes = 32 + 2 * NQ * 4;                           // descriptor, m, l
constexpr int kOffBar = align_up(kOffEpi + NO * kEpiBytes, 16);
constexpr int kNumBars = 2 * NK + 2 * NV + 2 * QN + 2 * NS + 2 * NP + 4 * NO + 2 * QS + NK + NV;
constexpr int kOffMisc = align_up(kOffBar + 8 * kNumBars, 16);
constexpr int kSmemBytes = kOffMisc + 64 + 1024;
// fp8 only: each K / V ring slot's row scales are staged in a 1 KB area of their own
// (one 128-byte-aligned box per block; block size >= 16 gives at most 8 boxes), so
// converting a slot in place never overwrites scales another thread still has to read
constexpr int kSclBytes = 1024;
constexpr int kOffScl = align_up(kOffMisc + 64, 1024);
constexpr int kSmemBytesF8 = kOffScl + (NK + NV) * kSclBytes + 1024;
static_assert(kSmemBytesF8 <= 227 * 1024, "shared memory per CTA (fp8)");
static_assert(kOffK % 1024 == 0 && kOffV % 1024 == 0 && kOffQ % 1024 == 0 && kOffP % 1024 == 0,
              "128-byte-swizzled TMA / MMA operands need 1024-byte alignment");
static_assert(kTileBytes % 1024 == 0 && kQBytes % 1024 == 0 && kPBytes % 1024 == 0, "tile sizes");
static_assert(kOffBar % 8 == 0, "mbarriers need 8-byte alignment");
static_assert(kOffSched % 16 == 0 && kOffDesc % 16 == 0 && kOffEpi % 16 == 0 && kEpiBytes % 16 == 0,
              "descriptor slots");
static_assert(kSmemBytes <= 227 * 1024, "shared memory per CTA");
constexpr float kLog2e = 1.4426950408889634f;
constexpr uint32_t kTmemCols = 128;  // S[NS] at 16*i; O[NO] at 64 + 16*i
constexpr uint32_t kTmemO = 64;
static_assert(kTmemO + 16 * NO <= kTmemCols, "tensor memory columns");

constexpr unsigned kCountBits = 24;
constexpr unsigned long long kCountMask = (1ull << kCountBits) - 1;

struct TcParams {
  __nv_bfloat16* out;
  const int32_t* block_tables;
  const int32_t* context_lens;
  unsigned long long* counters;  // [0]: work counter, [1 + s*Hq + g*G]: arrivals of (s, g)
  float* ws_o;                   // [B, Hq, max_parts, D]
  float* ws_ml;                  // [B, Hq, max_parts, 2]
  unsigned* err;
  unsigned long long tag;        // per-call epoch (< 2^40, never 0)
  int num_seqs;
  int num_kv_heads;
  int max_blocks;
  int num_blocks;
  int bs_log2;
  int partition_size;  // multiple of 128, <= 2048
  int max_parts;
  int max_context_len;
  unsigned total_items;
  float scale_log2;
  // fused store (pa_store_decode), else all NULL: row s of new_k / new_v goes to the
  // slot slot_mapping[s], which must be the slot of the sequence's last position
  const uint4* new_k;        // [B, Hkv, D] bf16, 16 vectors per head
  const uint4* new_v;
  const int32_t* slot_mapping;
  uint4* k_rows;             // the pools, as rows of Hkv x 16 vectors
  uint4* v_rows;
};

struct ItemDesc {
  int s, g, p, t0, n, ntiles, nparts, stop;
};

// Add one to an epoch-tagged counter and return the count before the add; a counter
// carrying another epoch's tag counts as zero. The tag is installed first (count 0):
// a thread that reads a stale tag swaps in (tag, 0), and stops as soon as it sees this
// call's tag, whoever installed it. After that only atomicAdds touch the counter, and
// they keep the tag, so the common case is one atomicAdd with no retries even with one
// producer per SM on one address. Bounded number of attempts.
__device__ __forceinline__ unsigned tagged_fetch_add(unsigned long long* ctr,
                                                     unsigned long long tag, unsigned* err,
                                                     bool* ok) {
  unsigned long long v = *reinterpret_cast<volatile unsigned long long*>(ctr);
  int it = 0;
  while ((v >> kCountBits) != tag) {
    if (++it > 4096) {
      flag_error(err, PA_DEV_ERR_TIMEOUT);
      *ok = false;
      return 0;
    }
    const unsigned long long prev = atomicCAS(ctr, v, tag << kCountBits);
    v = (prev == v) ? (tag << kCountBits) : prev;
  }
  const unsigned long long old = atomicAdd(ctr, 1ull);
  if ((old >> kCountBits) != tag) {  // the count ran into the tag bits
    flag_error(err, PA_DEV_ERR_TIMEOUT);
    *ok = false;
    return 0;
  }
  *ok = true;
  return static_cast<unsigned>(old & kCountMask);
}

// Same contract as tagged_fetch_add for a counter that only a few threads ever touch
// (the arrivals of one sequence's partitions): add first, and only if the tag was
// stale try to restart the count under this call's tag. With so few contenders this
// is one atomic in the common case. Bounded number of attempts.
__device__ __forceinline__ unsigned tagged_arrive(unsigned long long* ctr, unsigned long long tag,
                                                  unsigned* err, bool* ok) {
  for (int it = 0; it < 4096; ++it) {
    const unsigned long long old = atomicAdd(ctr, 1ull);
    if ((old >> kCountBits) == tag) {
      *ok = true;
      return static_cast<unsigned>(old & kCountMask);
    }
    if (atomicCAS(ctr, old + 1, (tag << kCountBits) | 1ull) == old + 1) {
      *ok = true;
      return 0u;
    }
  }
  flag_error(err, PA_DEV_ERR_TIMEOUT);
  *ok = false;
  return 0;
}

// bounded wait that also gives up once another role has given up
__device__ __forceinline__ bool wait_or_abort(uint64_t* bar, unsigned parity, unsigned* err,
                                              volatile int* abort_flag) {
  if (mbar_try_wait(bar, parity)) return true;
  const unsigned long long t0 = globaltimer_ns();
  while (true) {
    if (mbar_try_wait(bar, parity)) return true;
    if (*abort_flag) return false;
    if (globaltimer_ns() - t0 > kWaitLimitNs) {
      flag_error(err, PA_DEV_ERR_TIMEOUT);
      *abort_flag = 1;
      return false;
    }
  }
}

__device__ __forceinline__ void named_bar_sync(int id, int n) {
  asm volatile("bar.sync %0, %1;" ::"r"(id), "r"(n) : "memory");
}

// named barrier that also ORs a flag over the participating threads
__device__ __forceinline__ bool bar_or(int id, int n, bool v) {
  unsigned r;
  asm volatile(
      "{\n\t.reg .pred q, p;\n\t"
      "setp.ne.u32 q, %1, 0;\n\t"
      "bar.red.or.pred p, %2, %3, q;\n\t"
      "selp.u32 %0, 1, 0, p;\n\t}"
      : "=r"(r)
      : "r"(v ? 1u : 0u), "r"(id), "r"(n)
      : "memory");
  return r != 0;
}

// 16 consecutive fp32 columns of this thread's TMEM lane.
__device__ __forceinline__ void tmem_ld16(uint32_t taddr, float (&v)[16]) {
  uint32_t r[16];
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x16.b32 "
      "{%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15}, [%16];"
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]),
        "=r"(r[7]), "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]),
        "=r"(r[14]), "=r"(r[15])
      : "r"(taddr)
      : "memory");
#pragma unroll
  for (int i = 0; i < 16; ++i) v[i] = __uint_as_float(r[i]);
}

// 2-D tiled tensor load global -> shared (the fp8 scales: [Hkv][slots] fp32).
__device__ __forceinline__ void tma_load_2d(void* smem_dst, const CUtensorMap* map, uint64_t* bar,
                                            int c0, int c1) {
  asm volatile(
      "cp.async.bulk.tensor.2d.shared::cluster.global.mbarrier::complete_tx::bytes"
      " [%0], [%1, {%3, %4}], [%2];" ::"r"(smem_u32(smem_dst)),
      "l"(reinterpret_cast<uint64_t>(map)), "r"(smem_u32(bar)), "r"(c0), "r"(c1)
      : "memory");
}

// 16 e4m3 codes (one uint4, code i in byte i) times a scale -> 16 bf16 values as two
// uint4 (values 0-7, 8-15; element i in the low half of word i/2 ... as bf16 pairs).
// e4m3 -> f16 is exact, so code * scale is rounded once (fp32 product, then to bf16).
// Each step runs over all eight pairs before the next, so the eight chains overlap.
__device__ __forceinline__ void dequant16(const uint4 raw, float2 scale2, uint4& lo, uint4& hi) {
  const uint32_t w[4] = {raw.x, raw.y, raw.z, raw.w};
  __half2_raw h[8];
#pragma unroll
  for (int i = 0; i < 8; ++i)
    h[i] = __nv_cvt_fp8x2_to_halfraw2(
        static_cast<__nv_fp8x2_storage_t>((w[i >> 1] >> ((i & 1) * 16)) & 0xFFFFu), __NV_E4M3);
  float2 f[8];
#pragma unroll
  for (int i = 0; i < 8; ++i) f[i] = __half22float2(*reinterpret_cast<const __half2*>(&h[i]));
#pragma unroll
  for (int i = 0; i < 8; ++i) f[i] = __fmul2_rn(f[i], scale2);
  uint32_t out[8];
#pragma unroll
  for (int i = 0; i < 8; ++i) out[i] = pack_bf16x2(f[i].x, f[i].y);
  lo = make_uint4(out[0], out[1], out[2], out[3]);
  hi = make_uint4(out[4], out[5], out[6], out[7]);
}

__device__ __forceinline__ void tmem_st16(uint32_t taddr, const float (&v)[16]) {
  asm volatile(
      "tcgen05.st.sync.aligned.32x32b.x16.b32 [%0], "
      "{%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,%16};" ::"r"(taddr),
      "r"(__float_as_uint(v[0])), "r"(__float_as_uint(v[1])), "r"(__float_as_uint(v[2])),
      "r"(__float_as_uint(v[3])), "r"(__float_as_uint(v[4])), "r"(__float_as_uint(v[5])),
      "r"(__float_as_uint(v[6])), "r"(__float_as_uint(v[7])), "r"(__float_as_uint(v[8])),
      "r"(__float_as_uint(v[9])), "r"(__float_as_uint(v[10])), "r"(__float_as_uint(v[11])),
      "r"(__float_as_uint(v[12])), "r"(__float_as_uint(v[13])), "r"(__float_as_uint(v[14])),
      "r"(__float_as_uint(v[15]))
      : "memory");
}

template <int G, bool F8>
__global__ void __launch_bounds__(tc_threads<G, F8>(), 1) decode_tc_kernel(
    const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
    const __grid_constant__ CUtensorMap tmV, const __grid_constant__ CUtensorMap tmSK,
    const __grid_constant__ CUtensorMap tmSV, const TcParams p) {
  static_assert(G >= 1 && G <= NQ, "query heads per kv head");
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
  const int tid = threadIdx.x;
  const int warp = tid >> 5;
  const int lane = tid & 31;
  const int Hq = p.num_kv_heads * G;
  const int bs = 1 << p.bs_log2;

  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + kOffBar);
  uint64_t* k_full = bars;                     // [NK] TMA -> issuer
  uint64_t* k_empty = k_full + NK;             // [NK] score MMA done -> producer
  uint64_t* v_full = k_empty + NK;             // [NV] TMA -> issuer (+ softmax)
  uint64_t* v_empty = v_full + NV;             // [NV] value MMA done -> producer
  uint64_t* item_full = v_empty + NV;          // [QN] descriptor + q landed
  uint64_t* item_empty = item_full + QN;       // [QN] score MMAs done + descriptor read
  uint64_t* s_full = item_empty + QN;          // [NS] score MMA done -> softmax
  uint64_t* s_free = s_full + NS;              // [NS] softmax read S -> issuer
  uint64_t* p_full = s_free + NS;              // [NP] P^T written -> issuer
  uint64_t* pv_done = p_full + NP;             // [NP] value MMA of that P buffer done
  uint64_t* o_full = pv_done + NP;             // [NO] last value MMA of an item done
  uint64_t* o_free = o_full + NO;              // [NO] epilogue read O^T -> issuer
  uint64_t* epi_full = o_free + NO;            // [NO] softmax hand-off -> epilogue
  uint64_t* epi_empty = epi_full + NO;         // [NO] epilogue read the hand-off
  uint64_t* sched_full = epi_empty + NO;       // [QS] scheduler -> producer
  uint64_t* sched_empty = sched_full + QS;     // [QS] producer done with a queued item
  uint64_t* kst_full = sched_empty + QS;       // [NK] fp8: codes + scales of K landed
  uint64_t* vst_full = kst_full + NK;          // [NV] fp8: codes + scales of V landed
  ItemDesc* sched_desc = reinterpret_cast<ItemDesc*>(smem + kOffSched);
  int* sched_fb = reinterpret_cast<int*>(smem + kOffSchedFb);
  ItemDesc* descs = reinterpret_cast<ItemDesc*>(smem + kOffDesc);
  int* ids = reinterpret_cast<int*>(smem + kOffIds);
  float* red = reinterpret_cast<float*>(smem + kOffRed);
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + kOffMisc);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + kOffMisc + 8);
  volatile int* last_flag = reinterpret_cast<volatile int*>(smem + kOffMisc + 16);
  volatile int* conv_stop = reinterpret_cast<volatile int*>(smem + kOffMisc + 32);  // [NK], fp8

  // zero the Q slots and P^T buffers: rows >= G are never written and stay zero
  for (int i = tid; i < (QN * kQBytes + NP * kPBytes) / 16; i += blockDim.x)
    reinterpret_cast<uint4*>(smem + kOffQ)[i] = make_uint4(0, 0, 0, 0);
  fence_proxy_async_smem();
  if (tid == 0) {
    // fp8: a ring slot is full once every converter warp has written its rows
    for (int i = 0; i < NK; ++i) {
      mbar_init(&k_full[i], F8 ? conv_warps<G>() : 1);
      mbar_init(&k_empty[i], 1);
      mbar_init(&kst_full[i], 1);
      conv_stop[i] = 0;
    }
    for (int i = 0; i < NV; ++i) {
      mbar_init(&v_full[i], F8 ? conv_warps<G>() : 1);
      mbar_init(&v_empty[i], 1);
      mbar_init(&vst_full[i], 1);
    }
    for (int i = 0; i < QN; ++i) {
      mbar_init(&item_full[i], 1);
      mbar_init(&item_empty[i], 2);
    }
    for (int i = 0; i < NS; ++i) {
      mbar_init(&s_full[i], 1);
      mbar_init(&s_free[i], 4);
    }
    for (int i = 0; i < NP; ++i) {
      mbar_init(&p_full[i], 4);
      mbar_init(&pv_done[i], 1);
    }
    for (int i = 0; i < NO; ++i) {
      mbar_init(&o_full[i], 1);
      mbar_init(&o_free[i], 4);
      mbar_init(&epi_full[i], 1);
      mbar_init(&epi_empty[i], 1);
    }
    for (int i = 0; i < QS; ++i) {
      mbar_init(&sched_full[i], 1);
      mbar_init(&sched_empty[i], 1);
    }
    *abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == 5) {
    tmem_alloc(tmem_slot, kTmemCols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;

  // lane 0 waits, the warp follows its verdict (keeps the warp's control flow uniform)
  auto wwait = [&](uint64_t* bar, unsigned parity) -> bool {
    int okw = 0;
    if (lane == 0) okw = wait_or_abort(bar, parity, p.err, abort_flag) ? 1 : 0;
    return __shfl_sync(0xffffffffu, okw, 0) != 0;
  };

  if (warp == 4) {
    // ======================================================== producer warp
    if (lane == 0) {
      prefetch_tensormap(&tmQ);
      prefetch_tensormap(&tmK);
      prefetch_tensormap(&tmV);
      if (F8) {
        prefetch_tensormap(&tmSK);
        prefetch_tensormap(&tmSV);
      }
    }
    const int rows = bs < TM ? bs : TM;
    const int nbox = TM / rows;
    // fp8: each box's scales start on a 128-byte boundary of the slot
    const int sstride = rows * 4 < 128 ? 128 : rows * 4;
    int q = 0;       // items taken from the scheduler queue
    int k = 0;       // items published to the issuer / softmax
    unsigned j = 0;  // tiles issued
    while (true) {
      const int ss = q % QS;
      if (!wwait(&sched_full[ss], (q / QS) & 1)) break;
      const ItemDesc cur = sched_desc[ss];
      const int first_blk = sched_fb[ss];
      const int* idc = ids + ss * kMaxIds;
      const int slot = k % QN;
      if (k >= QN && !wwait(&item_empty[slot], ((k / QN) - 1) & 1)) break;
      if (cur.stop) {
        if (lane == 0) {
          descs[slot] = cur;
          mbar_arrive(&item_full[slot]);
        }
        if (F8) {
          // the converters follow the tile sequence: mark the next K slot as the end
          const int ks = j % NK;
          if (j < NK || wwait(&k_empty[ks], ((j / NK) - 1) & 1)) {
            if (lane == 0) {
              conv_stop[ks] = 1;
              mbar_arrive(&kst_full[ks]);
            }
          }
        }
        break;
      }
      const int g = cur.g, t0 = cur.t0, ntiles = cur.ntiles;
      if (p.slot_mapping != nullptr && cur.p == cur.nparts - 1) {
        // pa_store_decode: this item reads the sequence's last position, so it writes
        // that position's new row for its kv head first (lanes 0-15: the 16 vectors
        // of K, lanes 16-31: V), then makes the writes visible to its TMA loads.
        // Only the slot the block table gives for that position is accepted.
        const int pos = t0 + cur.n - 1;
        const int bi = (pos >> p.bs_log2) - first_blk;
        const int64_t expect =
            static_cast<int64_t>(bi < kMaxIds ? idc[bi] : 0) * bs + (pos & (bs - 1));
        const int dst_slot = __ldg(p.slot_mapping + cur.s);
        if (dst_slot >= 0) {
          if (dst_slot != expect) {
            if (lane == 0) flag_error(p.err, PA_DEV_ERR_BAD_INDEX);
          } else {
            const int64_t src = (static_cast<int64_t>(cur.s) * p.num_kv_heads + g) * 16 + (lane & 15);
            const int64_t dst = (static_cast<int64_t>(dst_slot) * p.num_kv_heads + g) * 16 + (lane & 15);
            if (lane < 16)
              p.k_rows[dst] = __ldg(p.new_k + src);
            else
              p.v_rows[dst] = __ldg(p.new_v + src);
            fence_proxy_async_global();
          }
        }
        __syncwarp();
      }
      if (lane == 0) {
        descs[slot] = cur;
        mbar_arrive_expect_tx(&item_full[slot], 2 * G * 128);
        uint8_t* qdst = smem + kOffQ + slot * kQBytes;
        tma_load_3d(qdst, &tmQ, &item_full[slot], 0, g * G, cur.s);
        tma_load_3d(qdst + kQRegion, &tmQ, &item_full[slot], 64, g * G, cur.s);
      }
      bool alive = true;
      for (int i = 0; i < ntiles; ++i, ++j) {
        // K of tile j: its slot frees when the score MMA of tile j - NK is done
        const int ks = j % NK;
        if (j >= NK && !wwait(&k_empty[ks], ((j / NK) - 1) & 1)) {
          alive = false;
          break;
        }
        if (lane == 0) {
          uint8_t* kdst = smem + kOffK + ks * kTileBytes;
          if (F8) {
            // codes into the upper half of the slot, scales into the slot's scale area
            mbar_arrive_expect_tx(&kst_full[ks], kRegion + TM * 4);
            for (int b = 0; b < nbox; ++b) {
              const int pos = t0 + i * TM + b * rows;
              const int bi = (pos >> p.bs_log2) - first_blk;
              const int row = (bi < kMaxIds ? idc[bi] : 0) * bs + (pos & (bs - 1));
              tma_load_3d(kdst + kRegion + b * rows * 128, &tmK, &kst_full[ks], 0, g, row);
              tma_load_2d(smem + kOffScl + ks * kSclBytes + b * sstride, &tmSK, &kst_full[ks],
                          row, g);
            }
          } else {
            mbar_arrive_expect_tx(&k_full[ks], kTileBytes);
            for (int b = 0; b < nbox; ++b) {
              const int pos = t0 + i * TM + b * rows;
              const int bi = (pos >> p.bs_log2) - first_blk;
              const int row = (bi < kMaxIds ? idc[bi] : 0) * bs + (pos & (bs - 1));
              tma_load_3d(kdst + b * rows * 128, &tmK, &k_full[ks], 0, g, row);
              tma_load_3d(kdst + kRegion + b * rows * 128, &tmK, &k_full[ks], 64, g, row);
            }
          }
        }
        __syncwarp();
        // V of tile j: its slot frees when the value MMA of tile j - NV is done
        const int vs = j % NV;
        if (j >= NV && !wwait(&v_empty[vs], ((j / NV) - 1) & 1)) {
          alive = false;
          break;
        }
        if (lane == 0) {
          uint8_t* vdst = smem + kOffV + vs * kTileBytes;
          if (F8) {
            mbar_arrive_expect_tx(&vst_full[vs], kRegion + TM * 4);
            for (int b = 0; b < nbox; ++b) {
              const int pos = t0 + i * TM + b * rows;
              const int bi = (pos >> p.bs_log2) - first_blk;
              const int row = (bi < kMaxIds ? idc[bi] : 0) * bs + (pos & (bs - 1));
              tma_load_3d(vdst + kRegion + b * rows * 128, &tmV, &vst_full[vs], 0, g, row);
              tma_load_2d(smem + kOffScl + (NK + vs) * kSclBytes + b * sstride, &tmSV,
                          &vst_full[vs], row, g);
            }
          } else {
            mbar_arrive_expect_tx(&v_full[vs], kTileBytes);
            for (int b = 0; b < nbox; ++b) {
              const int pos = t0 + i * TM + b * rows;
              const int bi = (pos >> p.bs_log2) - first_blk;
              const int row = (bi < kMaxIds ? idc[bi] : 0) * bs + (pos & (bs - 1));
              tma_load_3d(vdst + b * rows * 128, &tmV, &v_full[vs], 0, g, row);
              tma_load_3d(vdst + kRegion + b * rows * 128, &tmV, &v_full[vs], 64, g, row);
            }
          }
        }
        __syncwarp();
      }
      if (!alive) break;
      if (lane == 0) mbar_arrive(&sched_empty[ss]);  // this item's block ids are no longer needed
      ++k;
      ++q;
    }
  } else if (warp == 10) {
    // ======================================================== scheduler warp
    // Takes items (the CTA's first is its own index, later ones come from the tagged
    // counter), skips empty partitions, reads the context length and the item's
    // block ids, and queues them for the producer QS deep, so none of these dependent
    // global reads sit on the TMA producer's path.
    int q = 0;
    bool first_take = true;
    while (true) {
      const int slot = q % QS;
      if (q >= QS && !wwait(&sched_empty[slot], ((q / QS) - 1) & 1)) break;
      ItemDesc d;
      int first_blk = 0;
      while (true) {
        unsigned idx = 0;
        bool ok = true;
        if (first_take) {
          idx = blockIdx.x;
          first_take = false;
        } else {
          if (lane == 0) idx = tagged_fetch_add(p.counters, p.tag, p.err, &ok) + gridDim.x;
          idx = __shfl_sync(0xffffffffu, idx, 0);
          ok = __shfl_sync(0xffffffffu, ok ? 1 : 0, 0) != 0;
        }
        if (*abort_flag) ok = false;
        if (!ok || idx >= p.total_items) {
          d.stop = 1;
          d.ntiles = 0;
          break;
        }
        const int g = idx % p.num_kv_heads;
        const unsigned rr = idx / p.num_kv_heads;
        const int s = rr % p.num_seqs;
        const int part = rr / p.num_seqs;
        int ctx = __ldg(p.context_lens + s);
        if (ctx > p.max_context_len) {
          if (lane == 0 && part == 0) flag_error(p.err, PA_DEV_ERR_BAD_INDEX);
          ctx = p.max_context_len;
        }
        if (part * p.partition_size >= ctx) {
          if (part == 0) {  // empty context: a zero output row
            for (int i = lane; i < G * HD; i += 32)
              p.out[(static_cast<int64_t>(s) * Hq + g * G) * HD + i] = __float2bfloat16(0.f);
            // and no last position to store a new row at
            if (p.slot_mapping != nullptr && lane == 0 && __ldg(p.slot_mapping + s) >= 0)
              flag_error(p.err, PA_DEV_ERR_BAD_INDEX);
          }
          continue;
        }
        const int t0 = part * p.partition_size;
        const int n = min(ctx - t0, p.partition_size);
        const int ntiles = (n + TM - 1) / TM;
        first_blk = t0 >> p.bs_log2;
        const int nb = ((t0 + ntiles * TM - 1) >> p.bs_log2) - first_blk + 1;
        int* idb = ids + slot * kMaxIds;
        for (int i = lane; i < nb && i < kMaxIds; i += 32) {
          const int b = first_blk + i;
          int id = b < p.max_blocks
                       ? __ldg(p.block_tables + static_cast<int64_t>(s) * p.max_blocks + b)
                       : -1;
          if (id < 0 || id >= p.num_blocks) {
            if ((b << p.bs_log2) < ctx) flag_error(p.err, PA_DEV_ERR_BAD_INDEX);
            id = 0;  // in-bounds stand-in; positions past ctx are masked
          }
          idb[i] = id;
        }
        d.s = s; d.g = g; d.p = part; d.t0 = t0; d.n = n; d.ntiles = ntiles;
        d.nparts = (ctx + p.partition_size - 1) / p.partition_size;
        d.stop = 0;
        break;
      }
      __syncwarp();  // the block ids are in shared memory before lane 0 publishes
      if (lane == 0) {
        sched_desc[slot] = d;
        sched_fb[slot] = first_blk;
        mbar_arrive(&sched_full[slot]);
      }
      if (d.stop) break;
      ++q;
    }
  } else if (warp == 5) {
    // ======================================================== tensor-core issuer
    if (lane == 0) {
      constexpr uint32_t idS = idesc_bf16_f32(TM, NQ, 0, 0);  // K: K-major, Q^T: K-major
      constexpr uint32_t idO = idesc_bf16_f32(HD, NQ, 1, 0);  // V^T: MN-major, P^T: K-major
      const uint32_t sP = smem_u32(smem + kOffP);
      unsigned j = 0;  // tiles whose score MMA was issued
      // O^T(obuf) += V^T(t) P^T(t); `first` overwrites instead of accumulating
      auto pv = [&](unsigned t, bool first, int obuf, int item) -> bool {
        const int b = t % NP;
        const int vs = t % NV;
        if (!wait_or_abort(&p_full[b], (t / NP) & 1, p.err, abort_flag) ||
            !wait_or_abort(&v_full[vs], (t / NV) & 1, p.err, abort_flag))
          return false;
        // the first value MMA of an item overwrites O(obuf): the epilogue of the item
        // that used this accumulator NO items ago must have read it
        if (first && item >= NO &&
            !wait_or_abort(&o_free[obuf], ((item / NO) - 1) & 1, p.err, abort_flag))
          return false;
        tc_fence_after();
        const uint32_t sV = smem_u32(smem + kOffV + vs * kTileBytes);
        const uint32_t sPt = sP + b * kPBytes;
        const uint32_t dO = tmem + kTmemO + obuf * 16;
#pragma unroll
        for (int kk = 0; kk < TM / 16; ++kk) {
          const uint64_t a = smem_desc_sw128(sV + kk * 16 * 128, kRegion, 1024);
          const uint64_t bdesc = smem_desc_sw128(sPt + (kk >> 2) * kQRegion + (kk & 3) * 32, 16, 1024);
          tc_mma_f16_ss(dO, a, bdesc, idO, (first && kk == 0) ? 0u : 1u);
        }
        tc_commit(&pv_done[b]);
        tc_commit(&v_empty[vs]);
        return true;
      };
      int k = 0;
      bool ok = true;
      while (ok) {
        const int slot = k % QN;
        if (!wait_or_abort(&item_full[slot], (k / QN) & 1, p.err, abort_flag)) break;
        const ItemDesc d = descs[slot];
        if (d.stop) break;
        const uint32_t sQ = smem_u32(smem + kOffQ + slot * kQBytes);
        const int obuf = k % NO;
        for (int i = 0; i < d.ntiles; ++i, ++j) {
          const int ks = j % NK;
          const int sb = j % NS;
          if (!wait_or_abort(&k_full[ks], (j / NK) & 1, p.err, abort_flag) ||
              (j >= NS && !wait_or_abort(&s_free[sb], ((j / NS) - 1) & 1, p.err, abort_flag))) {
            ok = false;
            break;
          }
          tc_fence_after();
          const uint32_t sK = smem_u32(smem + kOffK + ks * kTileBytes);
#pragma unroll
          for (int kk = 0; kk < HD / 16; ++kk) {
            const uint32_t ko = (kk >> 2) * kRegion + (kk & 3) * 32;
            const uint32_t qo = (kk >> 2) * kQRegion + (kk & 3) * 32;
            tc_mma_f16_ss(tmem + sb * 16, smem_desc_sw128(sK + ko, 16, 1024),
                          smem_desc_sw128(sQ + qo, 16, 1024), idS, kk > 0 ? 1u : 0u);
          }
          tc_commit(&s_full[sb]);
          tc_commit(&k_empty[ks]);                              // K slot reusable
          if (i == d.ntiles - 1) tc_commit(&item_empty[slot]);  // Q slot reusable
          // the value MMA of the previous tile of this item follows this score MMA
          if (i > 0 && !pv(j - 1, i == 1, obuf, k)) {
            ok = false;
            break;
          }
        }
        // the last tile's value MMA right away, so the item's epilogue need not wait
        // for the next item's tiles
        if (!ok || !pv(j - 1, d.ntiles == 1, obuf, k)) break;
        tc_commit(&o_full[obuf]);  // O(obuf) complete once the MMAs so far are done
        ++k;
      }
    }
  } else if (warp < 4) {
    // ======================================================== softmax warps 0-3
    // Control flow stays uniform across the 128 threads: a wait that fails (time
    // limit, or another role gave up) only marks `failed`; the group leaves together
    // at an item boundary through a barrier vote, so no thread can strand the others
    // at a named barrier.
    const int r = tid;  // position within a tile = TMEM lane
    const uint32_t lane_off = static_cast<uint32_t>(warp * 32) << 16;
    int k = 0;
    unsigned j = 0;
    while (true) {
      const int slot = k % QN;
      bool failed = !wait_or_abort(&item_full[slot], (k / QN) & 1, p.err, abort_flag);
      const ItemDesc d = descs[slot];
      if (bar_or(1, 128, failed)) break;  // every thread has read the descriptor
      if (tid == 0) mbar_arrive(&item_empty[slot]);
      if (d.stop) {
        if (tid == 0) {  // tell the epilogue warps, once they have read slot k % NO
          const int b = k % NO;
          if (k < NO || wait_or_abort(&epi_empty[b], ((k / NO) - 1) & 1, p.err, abort_flag)) {
            reinterpret_cast<ItemDesc*>(smem + kOffEpi + b * kEpiBytes)->stop = 1;
            mbar_arrive(&epi_full[b]);
          }
        }
        break;
      }
      const int obuf = k % NO;
      float m[G], lp[G];
#pragma unroll
      for (int h = 0; h < G; ++h) {
        m[h] = -INFINITY;
        lp[h] = 0.f;
      }
      for (int i = 0; i < d.ntiles; ++i, ++j) {
        const int sb = j % NS;
        failed |= !wait_or_abort(&s_full[sb], (j / NS) & 1, p.err, abort_flag);
        tc_fence_after();
        float sv[16];
        tmem_ld16(tmem + sb * 16 + lane_off, sv);
        tc_wait_ld();
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(&s_free[sb]);
        const bool valid = i * TM + r < d.n;
        // per-head max over the tile: warp shuffles, then across the 4 warps
        float* rb = red + (j & 1) * 4 * NQ;
        float x[G];
#pragma unroll
        for (int h = 0; h < G; ++h) {
          x[h] = valid ? sv[h] * p.scale_log2 : -INFINITY;
          float v = x[h];
#pragma unroll
          for (int o = 16; o > 0; o >>= 1) v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, o));
          if (lane == 0) rb[warp * NQ + h] = v;
        }
        named_bar_sync(1, 128);
        bool rescale = false;
        float alpha[G];
#pragma unroll
        for (int h = 0; h < G; ++h) {
          const float mx = fmaxf(fmaxf(rb[h], rb[NQ + h]), fmaxf(rb[2 * NQ + h], rb[3 * NQ + h]));
          alpha[h] = 1.f;
          if (i == 0) {
            m[h] = mx;  // reference max of this item (every tile has a valid position)
          } else if (mx > m[h] + kRescaleLog2) {
            alpha[h] = ex2_approx(m[h] - mx);
            m[h] = mx;
            rescale = true;
          }
          const float pr = valid ? ex2_approx(x[h] - m[h]) : 0.f;
          lp[h] = lp[h] * alpha[h] + pr;
          x[h] = pr;
        }
        // this P^T buffer was last read by the value MMA of tile j - NP
        const int pb = j % NP;
        if (j >= NP) failed |= !wait_or_abort(&pv_done[pb], ((j / NP) - 1) & 1, p.err, abort_flag);
        uint8_t* pt = smem + kOffP + pb * kPBytes + (r >> 6) * kQRegion;
#pragma unroll
        for (int h = 0; h < G; ++h) {
          const int chunk = ((r & 63) >> 3) ^ (h & 7);
          *reinterpret_cast<__nv_bfloat16*>(pt + h * 128 + chunk * 16 + (r & 7) * 2) =
              __float2bfloat16_rn(x[h]);
        }
        if (i == d.ntiles - 1 && d.n - i * TM < TM) {
          // V rows past the partition's end may hold anything (even NaN); P is 0 there
          // but 0 * NaN is NaN: clear them before the tensor core reads the tile
          const int vs = j % NV;
          failed |= !wait_or_abort(&v_full[vs], (j / NV) & 1, p.err, abort_flag);
          if (!valid) {
            uint8_t* v = smem + kOffV + vs * kTileBytes + r * 128;
#pragma unroll
            for (int c = 0; c < 8; ++c) {
              *reinterpret_cast<uint4*>(v + c * 16) = make_uint4(0, 0, 0, 0);
              *reinterpret_cast<uint4*>(v + kRegion + c * 16) = make_uint4(0, 0, 0, 0);
            }
          }
        }
        if (rescale) {  // uniform across the group: every thread saw the same tile max
          // O holds the value MMAs up to tile j-1: wait for the last of them
          const unsigned t = j - 1;
          failed |= !wait_or_abort(&pv_done[t % NP], (t / NP) & 1, p.err, abort_flag);
          tc_fence_after();
          float o[16];
          tmem_ld16(tmem + kTmemO + obuf * 16 + lane_off, o);
          tc_wait_ld();
#pragma unroll
          for (int h = 0; h < G; ++h) o[h] *= alpha[h];
          tmem_st16(tmem + kTmemO + obuf * 16 + lane_off, o);
          tc_wait_st();
        }
        fence_proxy_async_smem();
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(&p_full[pb]);
      }
      // hand the item to the epilogue warps: l per head (the per-position shares summed
      // over the 128 threads) and the reference max; O^T stays in TMEM
      float* lb = red + 2 * 4 * NQ;
#pragma unroll
      for (int h = 0; h < G; ++h) {
        float v = lp[h];
#pragma unroll
        for (int off = 16; off > 0; off >>= 1) v += __shfl_xor_sync(0xffffffffu, v, off);
        if (lane == 0) lb[warp * NQ + h] = v;
      }
      named_bar_sync(1, 128);
      if (tid == 0) {
        const int b = k % NO;
        if (k >= NO) failed |= !wait_or_abort(&epi_empty[b], ((k / NO) - 1) & 1, p.err, abort_flag);
        if (!failed) {
          uint8_t* es = smem + kOffEpi + b * kEpiBytes;
          *reinterpret_cast<ItemDesc*>(es) = d;
          float* em = reinterpret_cast<float*>(es + 32);
#pragma unroll
          for (int h = 0; h < G; ++h) {
            em[h] = m[h];
            em[NQ + h] = lb[h] + lb[NQ + h] + lb[2 * NQ + h] + lb[3 * NQ + h];
          }
          mbar_arrive(&epi_full[b]);
        }
      }
      if (bar_or(1, 128, failed)) break;
      ++k;
    }
  } else if (warp < 10) {
    // ======================================================== epilogue warps 6-9
    // warp w reads TMEM lanes 32*(w%4)..+31: thread dl owns output dim dl of the item.
    // Same uniform-exit rule as the softmax group (barrier 2).
    const int dl = ((warp & 3) << 5) | lane;
    const uint32_t lane_off = static_cast<uint32_t>((warp & 3) * 32) << 16;
    const bool leader = (tid == 6 * 32);
    int k = 0;
    while (true) {
      const int b = k % NO;
      bool failed = !wait_or_abort(&epi_full[b], (k / NO) & 1, p.err, abort_flag);
      const uint8_t* es = smem + kOffEpi + b * kEpiBytes;
      const ItemDesc d = *reinterpret_cast<const ItemDesc*>(es);
      float m[G], L[G];
#pragma unroll
      for (int h = 0; h < G; ++h) {
        m[h] = reinterpret_cast<const float*>(es + 32)[h];
        L[h] = reinterpret_cast<const float*>(es + 32)[NQ + h];
      }
      if (bar_or(2, 128, failed)) break;  // every epilogue thread has read the hand-off
      if (leader) mbar_arrive(&epi_empty[b]);
      if (d.stop) break;
      failed |= !wait_or_abort(&o_full[b], (k / NO) & 1, p.err, abort_flag);
      tc_fence_after();
      float o[16];
      tmem_ld16(tmem + kTmemO + b * 16 + lane_off, o);
      tc_wait_ld();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&o_free[b]);
      const int64_t row0 = static_cast<int64_t>(d.s) * Hq + d.g * G;
      if (d.nparts == 1) {
        if (!failed) {
#pragma unroll
          for (int h = 0; h < G; ++h) p.out[(row0 + h) * HD + dl] = __float2bfloat16_rn(o[h] / L[h]);
        }
      } else {
#pragma unroll
        for (int h = 0; h < G; ++h) {
          const int64_t pr = (row0 + h) * p.max_parts + d.p;
          p.ws_o[pr * HD + dl] = o[h];
          if (dl == 0) {
            p.ws_ml[pr * 2 + 0] = m[h];
            p.ws_ml[pr * 2 + 1] = L[h];
          }
        }
        // the partial written by all 128 threads, then one release by the leader:
        // barrier (CTA order) + fence (device scope) + arrival
        named_bar_sync(2, 128);
        if (leader) {
          __threadfence();
          bool okc = true;
          const unsigned before = tagged_arrive(p.counters + 1 + row0, p.tag, p.err, &okc);
          *last_flag = okc && (before == static_cast<unsigned>(d.nparts - 1));
          __threadfence();
        }
        named_bar_sync(2, 128);
        if (*last_flag) {
          // this CTA completed the last partition of (s, g): merge all of them
#pragma unroll
          for (int h = 0; h < G; ++h) {
            const int64_t base = (row0 + h) * p.max_parts;
            float M = -INFINITY;
            for (int q = 0; q < d.nparts; ++q) M = fmaxf(M, __ldcg(p.ws_ml + (base + q) * 2));
            float Ls = 0.f, acc = 0.f;
            for (int q = 0; q < d.nparts; ++q) {
              const float f = ex2_approx(__ldcg(p.ws_ml + (base + q) * 2) - M);
              Ls += __ldcg(p.ws_ml + (base + q) * 2 + 1) * f;
              acc += __ldcg(p.ws_o + (base + q) * HD + dl) * f;
            }
            p.out[(row0 + h) * HD + dl] = __float2bfloat16_rn(acc / Ls);
          }
        }
      }
      if (bar_or(2, 128, failed)) break;  // also orders last_flag's reuse
      ++k;
    }
  } else if (F8) {
    // ======================================================== converter warps 11..
    // Follow the tile sequence of the producer; PPR threads (adjacent lanes) share row
    // r of each K and V tile and dequantise it in place, CPT 16-byte chunks of codes
    // each. One thread polls the staging barrier while the others sleep in a named
    // barrier (spinning warps would take issue slots from the MMA and TMA threads);
    // the vote there also carries abort and end-of-tiles. A row's upper-half bf16
    // covers only that row's codes, so a warp-level sync orders reads before writes.
    constexpr int NCT = 32 * conv_warps<G>();
    constexpr int PPR = NCT / TM;
    constexpr int CPT = 8 / PPR;
    const int t = tid - kConvWarp0 * 32;
    const int r = t / PPR;
    const int part = t % PPR;
    const int sw = r & 7;
    const int rot = r & (CPT - 1);
    // where the producer put row r's scale: box r / rows, 128-byte aligned boxes
    const int rows = bs < TM ? bs : TM;
    const int soff = (r / rows) * (rows * 4 < 128 ? 128 : rows * 4) + (r % rows) * 4;
    // stop_slot: the K ring slot whose end-of-tiles mark to honour, or -1 (V tiles)
    auto convert = [&](uint8_t* slot, const uint8_t* scl, uint64_t* staged, unsigned parity,
                       uint64_t* full, int stop_slot) -> bool {
      bool quit = false;
      if (t == 0) {
        quit = !wait_or_abort(staged, parity, p.err, abort_flag) ||
               (stop_slot >= 0 && conv_stop[stop_slot] != 0);
      }
      if (bar_or(3, NCT, quit)) return false;
      // the phase is complete (the slot cannot refill before this tile is consumed):
      // each thread's own test of it orders the TMA's bytes before its reads
      if (!mbar_try_wait(staged, parity)) flag_error(p.err, PA_DEV_ERR_TIMEOUT);
      uint4 raw[CPT];
      // code chunk part * CPT + (c ^ rot) of the row in step c: the 8 threads of a
      // quarter warp read 8 different 16-byte bank groups (rows are 128 bytes apart)
      const uint4* src = reinterpret_cast<const uint4*>(slot + kRegion + r * 128);
#pragma unroll
      for (int c = 0; c < CPT; ++c) raw[c] = src[part * CPT + (c ^ rot)];
      const float scv = *reinterpret_cast<const float*>(scl + soff);
      const float2 sc2 = make_float2(scv, scv);
      __syncwarp();
#pragma unroll
      for (int c = 0; c < CPT; ++c) {
        uint4 lo, hi;
        dequant16(raw[c], sc2, lo, hi);
        // dims 16k..16k+15 = 16-byte bf16 chunks 2k (lo) and 2k+1 (hi) of the row;
        // chunk q lies in half q / 8 at position (q % 8) ^ (r % 8) (128-byte swizzle).
        // The two threads of a row write their chunk pairs in opposite orders, so for
        // every step the quarter warp's 8 positions are distinct.
        const int kc = part * CPT + (c ^ rot);
#pragma unroll
        for (int h = 0; h < 2; ++h) {
          const int q = 2 * kc + (h ^ (PPR == 2 ? part : 0));
          uint4* dst = reinterpret_cast<uint4*>(slot + (q >> 3) * kRegion + r * 128 +
                                                (((q & 7) ^ sw) << 4));
          *dst = (q & 1) ? hi : lo;
        }
      }
      fence_proxy_async_smem();
      __syncwarp();
      if (lane == 0) mbar_arrive(full);
      return true;
    };
    // K(0), V(0), K(1), ... through one call site (keeps the unrolled conversion's
    // code once in the instruction cache)
#pragma unroll 1
    for (unsigned i = 0;; ++i) {
      const unsigned j = i >> 1;
      const bool is_v = i & 1;
      const int rs = is_v ? j % NV : j % NK;
      const unsigned ph = is_v ? (j / NV) & 1 : (j / NK) & 1;
      uint8_t* slot = smem + (is_v ? kOffV : kOffK) + rs * kTileBytes;
      const uint8_t* scl = smem + kOffScl + (is_v ? NK + rs : rs) * kSclBytes;
      if (!convert(slot, scl, is_v ? &vst_full[rs] : &kst_full[rs], ph,
                   is_v ? &v_full[rs] : &k_full[rs], is_v ? -1 : rs))
        break;
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 5) {
    tc_fence_after();
    tmem_dealloc(tmem, kTmemCols);
  }
}

unsigned long long next_tag() {
  // per-process random start: a workspace left by another process (or by an earlier
  // call of this one) never carries the current call's tag
  static std::atomic<unsigned long long> counter{[] {
    unsigned long long t = static_cast<unsigned long long>(time(nullptr)) * 0x9E3779B97F4A7C15ull;
    t ^= static_cast<unsigned long long>(clock()) * 0xC2B2AE3D27D4EB4Full;
    return t;
  }()};
  unsigned long long v;
  do {
    v = counter.fetch_add(1) & ((1ull << 40) - 1);
  } while (v == 0);
  return v;
}

template <int G, bool F8>
cudaError_t launch_tc_t(const DecodeLaunch& a, const TcParams& p, cudaStream_t stream) {
  const int bs = a.cache.block_size;
  const int rows = bs < TM ? bs : TM;
  const uint64_t slots = static_cast<uint64_t>(a.cache.num_blocks) * bs;
  const uint64_t hkv = static_cast<uint64_t>(a.cache.num_kv_heads);
  CUtensorMap tmQ, tmK, tmV, tmSK, tmSV;
  if (!encode_tensor_map_3d(&tmQ, a.q, HD, a.num_q_heads, a.num_seqs, 64, G, 1, true))
    return cudaErrorInvalidValue;
  if (F8) {
    // codes [slots][Hkv][D] bytes, one 128-byte row per box row, no swizzle;
    // scales [Hkv][slots] fp32, a run of `rows` positions of one kv head per box
    const uint64_t cd[3] = {HD, hkv, slots};
    const uint32_t cb[3] = {HD, 1, static_cast<uint32_t>(rows)};
    const uint64_t sd[2] = {slots, hkv};
    const uint32_t sb[2] = {static_cast<uint32_t>(rows), 1};
    if (!encode_tensor_map(&tmK, a.k_cache, CU_TENSOR_MAP_DATA_TYPE_UINT8, 1, 3, cd, cb, false) ||
        !encode_tensor_map(&tmV, a.v_cache, CU_TENSOR_MAP_DATA_TYPE_UINT8, 1, 3, cd, cb, false) ||
        !encode_tensor_map(&tmSK, a.k_scales, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 4, 2, sd, sb, false) ||
        !encode_tensor_map(&tmSV, a.v_scales, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 4, 2, sd, sb, false))
      return cudaErrorInvalidValue;
  } else {
    if (!encode_tensor_map_3d(&tmK, a.k_cache, HD, hkv, slots, 64, 1, rows, true) ||
        !encode_tensor_map_3d(&tmV, a.v_cache, HD, hkv, slots, 64, 1, rows, true))
      return cudaErrorInvalidValue;
    tmSK = tmQ;  // unused by the bf16 kernel
    tmSV = tmQ;
  }
  constexpr int smem_bytes = F8 ? kSmemBytesF8 : kSmemBytes;
  cudaError_t e = ensure_max_dynamic_smem(reinterpret_cast<const void*>(decode_tc_kernel<G, F8>),
                                          smem_bytes);
  if (e != cudaSuccess) return e;
  int grid = sm_count();
  if (static_cast<unsigned>(grid) > p.total_items) grid = static_cast<int>(p.total_items);
  if (grid < 1) grid = 1;
  decode_tc_kernel<G, F8><<<grid, tc_threads<G, F8>(), smem_bytes, stream>>>(
      tmQ, tmK, tmV, tmSK, tmSV, p);
  return cudaGetLastError();
}

}  // namespace

bool decode_tc_supported(const DecodeLaunch& a) {
  const int G = a.num_q_heads / a.cache.num_kv_heads;
  // fp8 pools add four or eight converter warps: up to 8 query heads per kv head
  const bool g_ok = a.fp8 ? (G == 1 || G == 2 || G == 4 || G == 8)
                          : (G == 1 || G == 2 || G == 4 || G == 8 || G == 16);
  // fp8 scale boxes start at slot index (block id * block size): a multiple of four
  // fp32 (16 bytes) only when the block size is
  const bool bs_ok = !a.fp8 || a.cache.block_size % 4 == 0;
  return a.cache.head_dim == HD && g_ok && bs_ok && a.partition_size % TM == 0 &&
         a.partition_size <= 2048;
}

cudaError_t launch_decode_tc(const DecodeLaunch& a, unsigned long long* counters,
                             cudaStream_t stream) {
  TcParams p;
  p.out = static_cast<__nv_bfloat16*>(a.out);
  p.block_tables = a.block_tables;
  p.context_lens = a.context_lens;
  p.counters = counters;
  p.ws_o = a.ws_o;
  p.ws_ml = a.ws_ml;
  p.err = device_error_word();
  p.tag = next_tag();
  p.num_seqs = a.num_seqs;
  p.num_kv_heads = a.cache.num_kv_heads;
  p.max_blocks = a.max_blocks_per_seq;
  p.num_blocks = a.cache.num_blocks;
  p.bs_log2 = 31 - __builtin_clz(static_cast<unsigned>(a.cache.block_size));
  p.partition_size = a.partition_size;
  p.max_parts = a.max_parts;
  p.max_context_len = a.max_context_len;
  p.total_items = static_cast<unsigned>(a.max_parts) * a.num_seqs * a.cache.num_kv_heads;
  p.scale_log2 = a.scale * kLog2e;
  p.new_k = static_cast<const uint4*>(a.new_k);
  p.new_v = static_cast<const uint4*>(a.new_v);
  p.slot_mapping = a.slot_mapping;
  p.k_rows = static_cast<uint4*>(const_cast<void*>(a.k_cache));
  p.v_rows = static_cast<uint4*>(const_cast<void*>(a.v_cache));
  if (a.fp8) {
    switch (a.num_q_heads / a.cache.num_kv_heads) {
      case 1: return launch_tc_t<1, true>(a, p, stream);
      case 2: return launch_tc_t<2, true>(a, p, stream);
      case 4: return launch_tc_t<4, true>(a, p, stream);
      case 8: return launch_tc_t<8, true>(a, p, stream);
      default: return cudaErrorInvalidValue;
    }
  }
  switch (a.num_q_heads / a.cache.num_kv_heads) {
    case 1: return launch_tc_t<1, false>(a, p, stream);
    case 2: return launch_tc_t<2, false>(a, p, stream);
    case 4: return launch_tc_t<4, false>(a, p, stream);
    case 8: return launch_tc_t<8, false>(a, p, stream);
    case 16: return launch_tc_t<16, false>(a, p, stream);
    default: return cudaErrorInvalidValue;
  }
}

}  // namespace pa

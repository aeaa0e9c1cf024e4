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
//   warp 4  producer: loads q (bf16: one box per item) and the K and V tiles of 128
//           positions through the block table (one TMA box per physical block) into a
//           K ring and a V ring; the whole warp waits and computes the coordinates, an
//           elected lane issues each load. A K slot frees as soon as its score MMA is
//           done and a V slot when its value MMA is done, so both streams run several
//           tiles ahead of the consumers (the fetch latency, ~1.4 us per tile, must
//           overlap);
//   warp 5  tensor-core issuer: owns the TMEM allocation; an event loop over two
//           cursors: the value MMA O^T += V^T P^T of the oldest scored tile whenever its
//           P, V and accumulator are ready (the softmax and the V ring wait on it),
//           else the score MMA S^T of the next tile, up to four tiles ahead and across
//           item boundaries, whenever its item, K tile and S buffer are ready. In the
//           kernel an issue group with its waits and commits takes the warp several
//           hundred cycles, so the order matters: value first keeps V slots and P
//           buffers turning over, and scoring ahead lets the next item's first tile be
//           ready when the softmax gets there;
//   warps 0-3  softmax (and 11-14 for e4m3 with up to 8 heads per kv head, taking the
//           second 128-position half of each tile): thread r owns position r of its
//           128 positions of a tile (TMEM lane r): per-head
//           tile max across the 128 positions, exp2 against a per-item reference max,
//           P^T to shared memory. O^T is rescaled in TMEM only when a tile's max
//           exceeds the reference by more than 2^8 (so probabilities stay <= 256,
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
// e4m3 pools (pa_decode_fp8): the tensor cores read the codes as they are stored
// (tcgen05.mma kind::f8f6f4: K tiles K-major, V tiles as the MN-major A operand of
// the value product, both 128-byte-swizzled by TMA), so no code is ever converted.
// Each row's scale is applied where its index is a free dimension of the product:
//   * a K row scale multiplies that position's score column in the softmax;
//   * a V row scale multiplies that position's probability before P^T is written:
//     P'_j = 2^(x_j + log2 s_v,j - R), with R a per-item, per-head reference kept so
//     that P' <= 2^6 (O^T is rescaled when a tile would exceed that, as for the max);
//     l keeps summing 2^(x_j - m) in fp32, and the output is O^T 2^(R - m) / l;
//   * q (bf16) becomes three e4m3 terms with one fp32 scale per head, hi = e4m3(q/s),
//     mid = e4m3(q/s - hi), lo = e4m3(q/s - hi - mid), written by the scheduler warp;
//     the three terms are the 48 rows of one B operand, so one product gives
//     [K hi^T | K mid^T | K lo^T] and the softmax adds the three column groups (about
//     2^-13 relative error on a typical q element: a score error is multiplied by the
//     score's size in the exponent, so peaked softmaxes need q this exact; K's codes
//     are exact);
//   * P' becomes hi = e4m3(P') and lo = e4m3(128 (P' - hi)), the 32 rows of one B
//     operand, so one product fills two side-by-side O^T accumulators combined as
//     O_hi + O_lo / 128 (about 2^-8 relative on P', and an absolute floor near 2^-17,
//     so small probabilities keep their precision).
// Per 128 positions that is 4 + 4 MMA instructions (K = 32 bytes each) instead of 20;
// an e4m3 tile is 256 positions (32 KB, as a bf16 tile of 128).
// Before a CTA ends, its producer waits for every copy it started and its issuer for
// every MMA it issued (with the full time limit, even when the roles gave up early),
// so no asynchronous write outlives the CTA's shared and tensor memory.
#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <cuda_fp8.h>

#include <atomic>
#include <cfloat>
#include <ctime>

#include "pa_internal.h"
#include "pa_ptx.cuh"

namespace pa {
namespace {

constexpr int TM = 128;        // positions per product (the MMAs' M) and per bf16 tile
constexpr int HD = 128;        // head dim
constexpr int NQ = 16;         // MMA N: query heads of one kv head, padded
constexpr int NS = 4;          // S^T buffers in TMEM
constexpr int NP = 4;          // P^T buffers in shared memory
constexpr int QN = 2;          // item queue depth (producer -> issuer, softmax)
constexpr int QS = 2;          // scheduler queue depth: one item prepared ahead (deeper
                               // queues reserve work early and unbalance the tail)
constexpr int NO = 3;          // O^T accumulators in TMEM (one per item in flight)
constexpr int kThreads = 352;  // softmax 0-3, producer 4, issuer 5, epilogue 6-9, scheduler 10
constexpr float kRescaleLog2 = 8.f;  // rescale when the max grows by more than this
constexpr int kQRegion = NQ * 128;           // 16 rows x 128 bytes (2 KB)
constexpr int kQTerms = 3;                   // e4m3: q as hi + mid + lo terms
constexpr int kPChunk = 2 * kQRegion;        // bf16: P^T 16 x 128; e4m3: hi, lo terms of 128 positions
constexpr int kMaxIds = 2048 / 16 + 2;       // block ids of one item (partition <= 2048)
// e4m3: one tile's 256 row scales: one box per physical block, each box on a 128-byte
// boundary (a tensor copy's shared-memory destination must be 128-byte aligned), so 16
// boxes of 16 scales (block size 16) take 2 KB
constexpr int kSclBytes = 2048;
constexpr int kEpiBytes = 32 + 3 * NQ * 4;   // descriptor, m, l, e4m3 output factor
// e4m3 value path: P' <= 2^kPBoundLog2 (a rescale brings the bound to 2^kPTargetLog2),
// so its low term, scaled by kPLoScale, stays inside e4m3's range (|128 (P' - hi)| <=
// 128 * 2 = 256 < 448)
constexpr float kPBoundLog2 = 6.f;
constexpr float kPTargetLog2 = 1.f;
constexpr float kPLoScale = 128.f;

constexpr int align_up(int x, int a) { return (x + a - 1) / a * a; }

// Shared-memory layout and ring depths of the bf16 (F8 = false) and e4m3 kernels.
// Every region starts on a 16-byte boundary (1024 for the swizzled operand tiles);
// the static_asserts below keep it that way when depths change.
template <bool F8>
struct Cfg {
  // A tile is 128 positions of bf16 rows (256 bytes each) or 256 positions of e4m3 rows
  // (128 bytes each): 32 KB either way. Every tile costs the kernel's roles about the
  // same time whatever it holds, so e4m3 tiles of 128 positions (16 KB) left the e4m3
  // decode at half the bf16 decode's bandwidth.
  static constexpr int TT = F8 ? 2 * TM : TM;                 // positions per tile
  static constexpr int kSub = TT / TM;                         // products of 128 positions
  static constexpr int kRegion = TM * 128;                    // 128 rows x 128 bytes
  static constexpr int kTileBytes = 2 * kRegion;              // one K or V tile
  static constexpr int NK = F8 ? 2 : 3;  // K ring (a slot frees when its score MMA is done)
  static constexpr int NV = 3;           // V ring (a slot frees when its value MMA is done)
  static constexpr int NSC = F8 ? 4 : 1;  // e4m3: K-scale ring (freed by the softmax); unused for bf16
  static constexpr int kPBytes = kSub * kPChunk;  // one P^T buffer
  static constexpr int kQBytes = (F8 ? kQTerms : 2) * kQRegion;  // bf16: two 64-dim halves
  static constexpr int kOffK = 0;
  static constexpr int kOffV = kOffK + NK * kTileBytes;
  static constexpr int kOffQ = kOffV + NV * kTileBytes;
  static constexpr int kOffP = kOffQ + QN * kQBytes;
  static constexpr int kOffRed = kOffP + NP * kPBytes;  // [3][8 warps][NQ] + [2][8] floats
  static constexpr int kRedFloats = 3 * 8 * NQ + 2 * 8;  // up to 8 softmax warps
  static constexpr int kOffQs = align_up(kOffRed + kRedFloats * 4, 16);  // [QN][NQ] q scales
  static constexpr int kOffIds = align_up(kOffQs + QN * NQ * 4, 16);
  static constexpr int kOffSched = align_up(kOffIds + QS * kMaxIds * 4, 16);  // [QS] descriptors
  static constexpr int kOffSchedFb = align_up(kOffSched + QS * 32, 16);       // [QS] first blocks
  static constexpr int kOffDesc = align_up(kOffSchedFb + QS * 4, 16);         // [QN] item descriptors
  static constexpr int kOffEpi = align_up(kOffDesc + QN * 32, 16);            // [NO] hand-offs
  static constexpr int kOffBar = align_up(kOffEpi + NO * kEpiBytes, 16);
  static constexpr int kNumBars = 2 * NK + 2 * NV + 2 * QN + 2 * NS + 2 * NP + 4 * NO + 2 * QS +
                                  1 + (F8 ? 2 * NSC + NV + QN : 0);
  static constexpr int kOffMisc = align_up(kOffBar + 8 * kNumBars, 16);
  // e4m3: the K-scale ring [NSC] and each V slot's scales [NV], kSclBytes each
  static constexpr int kOffScl = align_up(kOffMisc + 64, 1024);
  static constexpr int kSmemBytes = (F8 ? kOffScl + (NSC + NV) * kSclBytes : kOffMisc + 64) + 1024;
  // TMEM columns. bf16: S^T[NS] 16 columns each, then O^T[NO] 16 each. e4m3: S^T[NS] 96
  // columns each (per 128 positions, the hi, mid and lo q terms' products side by side:
  // one MMA with the three terms stacked as N = 48; two such for a tile), then O^T[NO]
  // 32 each (P's hi and lo terms stacked as N = 32: the hi accumulator, then the lo one)
  static constexpr uint32_t kSCols = F8 ? kSub * NQ * kQTerms : NQ;
  static constexpr uint32_t kOCols = F8 ? 2 * NQ : NQ;
  static constexpr uint32_t kTmemO = NS * kSCols;
  static constexpr uint32_t kTmemCols = F8 ? 512 : 128;
  static_assert(kSmemBytes <= 227 * 1024, "shared memory per CTA");
  static_assert(kOffK % 1024 == 0 && kOffV % 1024 == 0 && kOffQ % 1024 == 0 && kOffP % 1024 == 0,
                "128-byte-swizzled TMA / MMA operands need 1024-byte alignment");
  static_assert(kTileBytes % 1024 == 0 && kQBytes % 1024 == 0 && kPBytes % 1024 == 0, "tile sizes");
  static_assert(kOffBar % 8 == 0, "mbarriers need 8-byte alignment");
  static_assert(kOffSched % 16 == 0 && kOffDesc % 16 == 0 && kOffEpi % 16 == 0 && kEpiBytes % 16 == 0,
                "descriptor slots");
  static_assert(kTmemO + kOCols * NO <= kTmemCols, "tensor memory columns");
};
constexpr float kLog2e = 1.4426950408889634f;

constexpr unsigned kCountBits = 24;
constexpr unsigned long long kCountMask = (1ull << kCountBits) - 1;

struct TcParams {
  __nv_bfloat16* out;
  const __nv_bfloat16* q;        // [B, Hq, D] (read by the scheduler for e4m3 pools)
  const int32_t* block_tables;
  const int32_t* context_lens;
  unsigned long long* counters;  // [0]: work counter, [1 + s*Hq + g*G]: arrivals of (s, g)
  float* ws_o;                   // [B, Hq, max_parts, D]
  float* ws_ml;                  // [B, Hq, max_parts, 2]
  unsigned* err;
  unsigned long long tag;        // per-call epoch (< 2^40, never 0)
  unsigned long long wait_ns;    // bound of the waits between roles
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
  // shared-prefix decode: positions below shared_len were attended by the prefix kernel
  // (partition 0 of every longer context, already in the workspace); this kernel's
  // partitions start at shared_len and are numbered from 1. 0 = plain decode.
  int shared_len;
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

// N consecutive fp32 columns of this thread's TMEM lane (N = 1, 2, 4, 8 or 16; the
// score columns a softmax thread needs are the group's G heads).
template <int N>
__device__ __forceinline__ void tmem_ld_cols(uint32_t taddr, float (&v)[N]) {
  static_assert(N == 1 || N == 2 || N == 4 || N == 8 || N == 16, "tcgen05.ld column count");
  uint32_t r[16];
  if constexpr (N == 1) {
    asm volatile("tcgen05.ld.sync.aligned.32x32b.x1.b32 {%0}, [%1];" : "=r"(r[0]) : "r"(taddr) : "memory");
  } else if constexpr (N == 2) {
    asm volatile("tcgen05.ld.sync.aligned.32x32b.x2.b32 {%0,%1}, [%2];"
                 : "=r"(r[0]), "=r"(r[1]) : "r"(taddr) : "memory");
  } else if constexpr (N == 4) {
    asm volatile("tcgen05.ld.sync.aligned.32x32b.x4.b32 {%0,%1,%2,%3}, [%4];"
                 : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]) : "r"(taddr) : "memory");
  } else if constexpr (N == 8) {
    asm volatile("tcgen05.ld.sync.aligned.32x32b.x8.b32 {%0,%1,%2,%3,%4,%5,%6,%7}, [%8];"
                 : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]),
                   "=r"(r[6]), "=r"(r[7])
                 : "r"(taddr)
                 : "memory");
  } else {
    float t[16];
    tmem_ld16(taddr, t);
#pragma unroll
    for (int i = 0; i < 16; ++i) r[i] = __float_as_uint(t[i]);
  }
#pragma unroll
  for (int i = 0; i < N; ++i) v[i] = __uint_as_float(r[i]);
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


// Two values -> their e4m3 codes (round to nearest even, saturated to +-448), packed
// with a in the low byte, and the values those codes stand for.
__device__ __forceinline__ uint32_t e4m3x2(float a, float b, float2& back) {
  const __nv_fp8x2_storage_t c =
      __nv_cvt_float2_to_fp8x2(make_float2(a, b), __NV_SATFINITE, __NV_E4M3);
  const __half2_raw h = __nv_cvt_fp8x2_to_halfraw2(c, __NV_E4M3);
  back = __half22float2(*reinterpret_cast<const __half2*>(&h));
  return static_cast<uint32_t>(c);
}

// hi / lo e4m3 terms of two values: hi = e4m3(v), lo = e4m3(lo_scale * (v - hi)),
// as two packed byte pairs (value a in the low byte of each).
__device__ __forceinline__ void split_e4m3x2(float a, float b, float lo_scale, uint32_t& hi,
                                             uint32_t& lo) {
  float2 h, unused;
  hi = e4m3x2(a, b, h);
  lo = e4m3x2((a - h.x) * lo_scale, (b - h.y) * lo_scale, unused);
}

// Softmax groups: for e4m3 with up to 8 heads per kv head, two groups of four warps take
// the two 128-position halves of a tile side by side (one position per thread, 480
// threads, 128 registers each); otherwise one group takes the whole tile.
template <int G, bool F8>
constexpr int kSoftGroups = (F8 && G <= 8) ? 2 : 1;
template <int G, bool F8>
constexpr int kThreadsOf = kSoftGroups<G, F8> == 2 ? 480 : kThreads;

template <int G, bool F8>
__global__ void __launch_bounds__(kThreadsOf<G, F8>, 1) decode_tc_kernel(
    const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
    const __grid_constant__ CUtensorMap tmV, const __grid_constant__ CUtensorMap tmSK,
    const __grid_constant__ CUtensorMap tmSV, const TcParams p) {
  static_assert(G >= 1 && G <= NQ, "query heads per kv head");
  using C = Cfg<F8>;
  constexpr int NK = C::NK, NV = C::NV, NSC = C::NSC;
  constexpr int SG = kSoftGroups<G, F8>;
  constexpr int kSoftThreads = 128 * SG;
  static_assert(SG == 1 || C::kSub == SG, "two softmax groups take one half of a tile each");
  constexpr int kRegion = C::kRegion, kTileBytes = C::kTileBytes;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
  const int tid = threadIdx.x;
  const int warp = tid >> 5;
  const int lane = tid & 31;
  const int Hq = p.num_kv_heads * G;
  const int bs = 1 << p.bs_log2;
  const unsigned long long wl = p.wait_ns;

  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + C::kOffBar);
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
  uint64_t* mma_drain = sched_empty + QS;      // [1] every MMA of the issuer finished
  uint64_t* ksc_full = mma_drain + 1;          // [NSC] e4m3: K scales of a tile landed
  uint64_t* ksc_empty = ksc_full + NSC;        // [NSC] e4m3: softmax read them
  uint64_t* vsc_full = ksc_empty + NSC;        // [NV] e4m3: V scales of a tile landed
  uint64_t* q_ready = vsc_full + NV;           // [QN] e4m3: the item's q terms written
  ItemDesc* sched_desc = reinterpret_cast<ItemDesc*>(smem + C::kOffSched);
  int* sched_fb = reinterpret_cast<int*>(smem + C::kOffSchedFb);
  ItemDesc* descs = reinterpret_cast<ItemDesc*>(smem + C::kOffDesc);
  int* ids = reinterpret_cast<int*>(smem + C::kOffIds);
  float* red = reinterpret_cast<float*>(smem + C::kOffRed);
  float* qscale = reinterpret_cast<float*>(smem + C::kOffQs);  // [QN][NQ] e4m3 q scales
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + C::kOffMisc);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + C::kOffMisc + 8);
  volatile int* last_flag = reinterpret_cast<volatile int*>(smem + C::kOffMisc + 16);
  // e4m3: where a tile's row scales sit (box r / rows, each box on a 128-byte boundary:
  // a tensor copy's shared-memory destination must be 128-byte aligned)
  const int srows = bs < C::TT ? bs : C::TT;
  const int sstride = srows * 4 < 128 ? 128 : srows * 4;

  // The scheduler's first item is the CTA's own index: its context length, block ids
  // and (e4m3) q are read here, before the set-up barrier, so that their latency
  // overlaps the set-up instead of delaying the first tile
  constexpr int kPreIds = (kMaxIds + 31) / 32;
  int pre_ctx = 0;
  int pre_id[kPreIds];
  uint2 pre_q[F8 ? G : 1];
  if (warp == 10 && blockIdx.x < p.total_items) {
    const int s = (blockIdx.x / p.num_kv_heads) % p.num_seqs;
    const int part = (blockIdx.x / p.num_kv_heads) / p.num_seqs;
    pre_ctx = __ldg(p.context_lens + s);
    const int fb = (p.shared_len + part * p.partition_size) >> p.bs_log2;
#pragma unroll
    for (int k = 0; k < kPreIds; ++k) {
      const int b = fb + lane + 32 * k;
      pre_id[k] = (lane + 32 * k < kMaxIds && b < p.max_blocks)
                      ? __ldg(p.block_tables + static_cast<int64_t>(s) * p.max_blocks + b)
                      : -1;
    }
    if constexpr (F8) {
      const uint2* src = reinterpret_cast<const uint2*>(
          p.q + (static_cast<int64_t>(s) * Hq + (blockIdx.x % p.num_kv_heads) * G) * HD);
#pragma unroll
      for (int h = 0; h < G; ++h) pre_q[h] = __ldg(src + h * (HD / 4) + lane);
    }
  }

  // zero the Q slots and P^T buffers: rows >= G are never written and stay zero
  for (int i = tid; i < (QN * C::kQBytes + NP * C::kPBytes) / 16; i += blockDim.x)
    reinterpret_cast<uint4*>(smem + C::kOffQ)[i] = make_uint4(0, 0, 0, 0);
  fence_proxy_async_smem();
  if (tid == 0) {
    for (int i = 0; i < NK; ++i) {
      mbar_init(&k_full[i], 1);
      mbar_init(&k_empty[i], 1);
    }
    for (int i = 0; i < NV; ++i) {
      mbar_init(&v_full[i], 1);
      mbar_init(&v_empty[i], 1);
      if (F8) mbar_init(&vsc_full[i], 1);
    }
    for (int i = 0; F8 && i < NSC; ++i) {
      mbar_init(&ksc_full[i], 1);
      mbar_init(&ksc_empty[i], 4 * SG);
    }
    for (int i = 0; F8 && i < QN; ++i) mbar_init(&q_ready[i], 1);
    for (int i = 0; i < QN; ++i) {
      mbar_init(&item_full[i], 1);
      mbar_init(&item_empty[i], 2);
    }
    for (int i = 0; i < NS; ++i) {
      mbar_init(&s_full[i], 1);
      mbar_init(&s_free[i], 4 * SG);
    }
    for (int i = 0; i < NP; ++i) {
      mbar_init(&p_full[i], 4 * SG);
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
    mbar_init(mma_drain, 1);
    *abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == 5) {
    tmem_alloc(tmem_slot, C::kTmemCols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  if (warp == 4 && lane == 0) {
    prefetch_tensormap(&tmK);
    prefetch_tensormap(&tmV);
    if (F8) {
      prefetch_tensormap(&tmSK);
      prefetch_tensormap(&tmSV);
    } else {
      prefetch_tensormap(&tmQ);
    }
  }

  // lane 0 waits, the warp follows its verdict (keeps the warp's control flow uniform)
  auto wwait = [&](uint64_t* bar, unsigned parity) -> bool {
    int okw = 0;
    if (lane == 0) okw = wait_or_abort(bar, parity, p.err, abort_flag, wl) ? 1 : 0;
    return __shfl_sync(0xffffffffu, okw, 0) != 0;
  };

  if (warp == 4) {
    // ======================================================== producer warp
    const int rows = srows;
    const int nbox = C::TT / rows;
    int q = 0;        // items taken from the scheduler queue
    int k = 0;        // items published to the issuer / softmax
    int kq = 0;       // q loads started (bf16)
    int npub = 0;     // items published to the item slots (the final stop included)
    unsigned jk = 0;  // K tiles whose loads were started
    unsigned jv = 0;  // V tiles whose loads were started
    auto row_of = [&](const int* idc, int first_blk, int pos) {
      const int bi = (pos >> p.bs_log2) - first_blk;
      return (bi < kMaxIds ? idc[bi] : 0) * bs + (pos & (bs - 1));
    };
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
        ++npub;
        break;
      }
      const int g = cur.g, t0 = cur.t0, ntiles = cur.ntiles;
      if (!F8 && p.slot_mapping != nullptr && cur.p == cur.nparts - 1) {
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
        if (F8) {
          mbar_arrive(&item_full[slot]);  // the q terms were written by the scheduler
        } else {
          mbar_arrive_expect_tx(&item_full[slot], 2 * G * 128);
          uint8_t* qdst = smem + C::kOffQ + slot * C::kQBytes;
          tma_load_3d(qdst, &tmQ, &item_full[slot], 0, g * G, cur.s);
          tma_load_3d(qdst + kQRegion, &tmQ, &item_full[slot], 64, g * G, cur.s);
        }
      }
      if (!F8) kq = k + 1;
      ++npub;
      bool alive = true;
      __syncwarp();  // converged: the loop's loads are elected from the whole warp
      // The whole warp runs the tile loop (waits and coordinates warp-uniform); one
      // elected lane issues each load. A lane-0 branch with broadcast verdicts cost this
      // warp ~2000 cycles a tile, more than an e4m3 tile's share of the DRAM time.
#pragma unroll 1
      for (int i = 0; i < ntiles; ++i) {
        // K of tile jk: its slot frees when the score MMA of tile jk - NK is done
        const int ks = jk % NK;
        if (jk >= NK && !warp_wait_or_abort(&k_empty[ks], ((jk / NK) - 1) & 1, p.err, abort_flag, wl)) {
          alive = false;
          break;
        }
        const int kl = F8 ? jk % NSC : 0;
        if (F8 && jk >= NSC &&
            !warp_wait_or_abort(&ksc_empty[kl], ((jk / NSC) - 1) & 1, p.err, abort_flag, wl)) {
          alive = false;
          break;
        }
        {
          uint8_t* kdst = smem + C::kOffK + ks * kTileBytes;
          mbar_arrive_expect_tx_w(&k_full[ks], kTileBytes);
          if (F8) mbar_arrive_expect_tx_w(&ksc_full[kl], C::TT * 4);
#pragma unroll 1
          for (int b = 0; b < nbox; ++b) {
            const int row = row_of(idc, first_blk, t0 + i * C::TT + b * rows);
            if (F8) {
              tma_load_3d_w(kdst + b * rows * 128, &tmK, &k_full[ks], 0, g, row);
              tma_load_2d_w(smem + C::kOffScl + kl * kSclBytes + b * sstride, &tmSK, &ksc_full[kl],
                            row, g);
            } else {
              tma_load_3d_w(kdst + b * rows * 128, &tmK, &k_full[ks], 0, g, row);
              tma_load_3d_w(kdst + kRegion + b * rows * 128, &tmK, &k_full[ks], 64, g, row);
            }
          }
        }
        ++jk;
        // V of tile jv: its slot frees when the value MMA of tile jv - NV is done
        const int vs = jv % NV;
        if (jv >= NV && !warp_wait_or_abort(&v_empty[vs], ((jv / NV) - 1) & 1, p.err, abort_flag, wl)) {
          alive = false;
          break;
        }
        {
          uint8_t* vdst = smem + C::kOffV + vs * kTileBytes;
          mbar_arrive_expect_tx_w(&v_full[vs], kTileBytes);
          if (F8) mbar_arrive_expect_tx_w(&vsc_full[vs], C::TT * 4);
#pragma unroll 1
          for (int b = 0; b < nbox; ++b) {
            const int row = row_of(idc, first_blk, t0 + i * C::TT + b * rows);
            if (F8) {
              tma_load_3d_w(vdst + b * rows * 128, &tmV, &v_full[vs], 0, g, row);
              tma_load_2d_w(smem + C::kOffScl + (NSC + vs) * kSclBytes + b * sstride, &tmSV,
                            &vsc_full[vs], row, g);
            } else {
              tma_load_3d_w(vdst + b * rows * 128, &tmV, &v_full[vs], 0, g, row);
              tma_load_3d_w(vdst + kRegion + b * rows * 128, &tmV, &v_full[vs], 64, g, row);
            }
          }
        }
        ++jv;
      }
      if (!alive) break;
      if (lane == 0) mbar_arrive(&sched_empty[ss]);  // this item's block ids are no longer needed
      ++k;
      ++q;
    }
    // Before the CTA ends, every copy this warp started must have landed. Per slot
    // only its last load can still be in flight (the one before it was consumed), so
    // waiting for the last phase of each slot is enough; on the normal path these
    // completed long ago. Full time limit: these copies always complete.
    if (lane == 0) {
#pragma unroll 1
      for (unsigned t = jk > static_cast<unsigned>(NK) ? jk - NK : 0; t < jk; ++t)
        mbar_wait(&k_full[t % NK], (t / NK) & 1, p.err);
#pragma unroll 1
      for (unsigned t = jv > static_cast<unsigned>(NV) ? jv - NV : 0; t < jv; ++t)
        mbar_wait(&v_full[t % NV], (t / NV) & 1, p.err);
      if (F8) {
#pragma unroll 1
        for (unsigned t = jk > static_cast<unsigned>(NSC) ? jk - NSC : 0; t < jk; ++t)
          mbar_wait(&ksc_full[t % NSC], (t / NSC) & 1, p.err);
#pragma unroll 1
        for (unsigned t = jv > static_cast<unsigned>(NV) ? jv - NV : 0; t < jv; ++t)
          mbar_wait(&vsc_full[t % NV], (t / NV) & 1, p.err);
      } else {
        // a q load whose slot took a later item has landed (the slot was handed on only
        // after the issuer had waited for it); only the others are waited for here
#pragma unroll 1
        for (int t = kq > QN ? kq - QN : 0; t < kq; ++t)
          if (t + QN >= npub) mbar_wait(&item_full[t % QN], (t / QN) & 1, p.err);
      }
    }
  } else if (warp == 10) {
    // ======================================================== scheduler warp
    // Takes items (the CTA's first is its own index, later ones come from the tagged
    // counter), skips empty partitions, reads the context length and the item's
    // block ids, and queues them for the producer QS deep, so none of these dependent
    // global reads sit on the TMA producer's path. For e4m3 pools it also writes the
    // item's q as three e4m3 terms into the item's Q slot.
    int q = 0;
    bool first_take = true;
    while (true) {
      const int slot = q % QS;
      if (q >= QS && !wwait(&sched_empty[slot], ((q / QS) - 1) & 1)) break;
      ItemDesc d;
      int first_blk = 0;
      bool used_pre = false;  // this item's inputs were read before the set-up barrier
      while (true) {
        unsigned idx = 0;
        bool ok = true;
        const bool pre = first_take;
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
        int ctx = pre ? pre_ctx : __ldg(p.context_lens + s);
        if (ctx > p.max_context_len) {
          if (lane == 0 && part == 0) flag_error(p.err, PA_DEV_ERR_BAD_INDEX);
          ctx = p.max_context_len;
        }
        const int t0 = p.shared_len + part * p.partition_size;
        if (t0 >= ctx) {
          if (part == 0 && p.shared_len == 0) {  // empty context: a zero output row
#pragma unroll 1
            for (int i = lane; i < G * HD; i += 32)
              p.out[(static_cast<int64_t>(s) * Hq + g * G) * HD + i] = __float2bfloat16(0.f);
            // and no last position to store a new row at
            if (p.slot_mapping != nullptr && lane == 0 && __ldg(p.slot_mapping + s) >= 0)
              flag_error(p.err, PA_DEV_ERR_BAD_INDEX);
          }
          continue;
        }
        const int n = min(ctx - t0, p.partition_size);
        const int ntiles = (n + C::TT - 1) / C::TT;
        first_blk = t0 >> p.bs_log2;
        const int nb = ((t0 + ntiles * C::TT - 1) >> p.bs_log2) - first_blk + 1;
        int* idb = ids + slot * kMaxIds;
        auto put_id = [&](int i, int id) {
          if (id < 0 || id >= p.num_blocks) {
            if (((first_blk + i) << p.bs_log2) < ctx) flag_error(p.err, PA_DEV_ERR_BAD_INDEX);
            id = 0;  // in-bounds stand-in; positions past ctx are masked
          }
          idb[i] = id;
        };
        if (pre) {
#pragma unroll
          for (int k = 0; k < kPreIds; ++k)
            if (lane + 32 * k < nb && lane + 32 * k < kMaxIds) put_id(lane + 32 * k, pre_id[k]);
        } else {
#pragma unroll 1
          for (int i = lane; i < nb && i < kMaxIds; i += 32) {
            const int b = first_blk + i;
            put_id(i, b < p.max_blocks
                          ? __ldg(p.block_tables + static_cast<int64_t>(s) * p.max_blocks + b)
                          : -1);
          }
        }
        used_pre = pre;
        const int shared = p.shared_len > 0 ? 1 : 0;
        d.s = s; d.g = g; d.p = part + shared; d.t0 = t0; d.n = n; d.ntiles = ntiles;
        d.nparts = shared + (ctx - p.shared_len + p.partition_size - 1) / p.partition_size;
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
      if (F8) {
        // q of the item's G heads as e4m3 terms, after the item is published (the
        // producer starts its tiles meanwhile); this scheduler item is the producer's
        // item q, in Q slot q % QN, whose previous item's score MMAs must be done. Per
        // head s = amax / 448, y = q * 448 / amax; lane L holds dims 4L..4L+3 and writes
        // them, 4 bytes per term, into row h of the 128-byte-swizzled slot.
        const int qs = q % QN;
        if (q >= QN && !wwait(&item_empty[qs], ((q / QN) - 1) & 1)) break;
        uint8_t* qd = smem + C::kOffQ + qs * C::kQBytes;
        const uint2* src = reinterpret_cast<const uint2*>(
            p.q + (static_cast<int64_t>(d.s) * Hq + d.g * G) * HD);
#pragma unroll
        for (int h = 0; h < G; ++h) {
          const uint2 raw = used_pre ? pre_q[h] : __ldg(src + h * (HD / 4) + lane);
          const float f0 = bf16lo_to_f32(raw.x), f1 = bf16hi_to_f32(raw.x);
          const float f2 = bf16lo_to_f32(raw.y), f3 = bf16hi_to_f32(raw.y);
          float amax = fmaxf(fmaxf(fabsf(f0), fabsf(f1)), fmaxf(fabsf(f2), fabsf(f3)));
#pragma unroll
          for (int o = 16; o > 0; o >>= 1) amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, o));
          float inv = 448.f / amax;
          if (!(inv <= FLT_MAX)) inv = 0.f;  // all zero (or tiny): codes 0, scale 0
          // three terms: each is the e4m3 rounding of what the terms before it left
          float y[4] = {f0 * inv, f1 * inv, f2 * inv, f3 * inv};
          const int off = h * 128 + ((((lane >> 2) ^ h) & 7) << 4) + (lane & 3) * 4;
#pragma unroll
          for (int term = 0; term < kQTerms; ++term) {
            float2 b01, b23;
            const uint32_t c01 = e4m3x2(y[0], y[1], b01);
            const uint32_t c23 = e4m3x2(y[2], y[3], b23);
            *reinterpret_cast<uint32_t*>(qd + term * kQRegion + off) = c01 | (c23 << 16);
            y[0] -= b01.x;
            y[1] -= b01.y;
            y[2] -= b23.x;
            y[3] -= b23.y;
          }
          if (lane == 0) qscale[qs * NQ + h] = inv > 0.f ? amax / 448.f : 0.f;
        }
        fence_proxy_async_smem();
        __syncwarp();
        if (lane == 0) mbar_arrive(&q_ready[qs]);
      }
      ++q;
    }
  } else if (warp == 5) {
    // ======================================================== tensor-core issuer
    // the whole warp runs this loop (its descriptors stay warp-uniform); one elected lane
    // issues each MMA and commit
    {
      // bf16: K K-major, Q^T K-major; V^T MN-major, P^T K-major (same for e4m3, with the
      // q terms stacked as N = 48 and P's two terms as N = 32)
      constexpr uint32_t idS = F8 ? idesc_e4m3_f32(TM, NQ * kQTerms, 0, 0) : idesc_bf16_f32(TM, NQ, 0, 0);
      constexpr uint32_t idO = F8 ? idesc_e4m3_f32(HD, 2 * NQ, 1, 0) : idesc_bf16_f32(HD, NQ, 1, 0);
      const uint32_t sP = smem_u32(smem + C::kOffP);
      // Two cursors over the CTA's tiles: the score cursor (item ks, tile is, CTA tile
      // js) runs up to kLookahead tiles ahead of the value cursor (item kp, tile ip, CTA
      // tile jp). Both advance only on non-blocking tests of their barriers.
      constexpr unsigned kLookahead = NS;
      int ks = 0, is = 0, s_nt = 0;
      unsigned js = 0;
      bool s_in = false, s_end = false;  // the score cursor holds an item / saw the stop item
      uint32_t sQ = 0;
      int nt_ring[8];  // tile counts of the items between the two cursors
      int kp = 0, ip = 0;
      unsigned jp = 0;
      // the score cursor enters its next item (false: not published yet, or the stop item)
      auto s_enter = [&]() -> bool {
        const int slot = ks % QN;
        const unsigned ph = (ks / QN) & 1;
        if (!__all_sync(0xffffffffu, mbar_test_wait(&item_full[slot], ph))) return false;
        const ItemDesc d = descs[slot];
        if (d.stop) { s_end = true; return false; }
        // e4m3: the scheduler writes the item's q terms after publishing the item
        if (F8 && !__all_sync(0xffffffffu, mbar_test_wait(&q_ready[slot], ph))) return false;
        s_nt = d.ntiles;
        nt_ring[ks & 7] = s_nt;
        sQ = smem_u32(smem + C::kOffQ + slot * C::kQBytes);
        is = 0;
        s_in = true;
        return true;
      };
      // S^T(js) (false: its item, K tile or S buffer is not ready)
      auto score = [&]() -> bool {
        if (!s_in && (s_end || !s_enter())) return false;
        const int kslot = js % NK;
        const int sb = js % NS;
        if (!__all_sync(0xffffffffu, mbar_test_wait(&k_full[kslot], (js / NK) & 1) &&
                                         (js < NS || mbar_test_wait(&s_free[sb], ((js / NS) - 1) & 1))))
          return false;
        tc_fence_after();
        const uint64_t aK = smem_desc_sw128(smem_u32(smem + C::kOffK + kslot * kTileBytes), 16, 1024);
        const uint64_t bQ = smem_desc_sw128(sQ, 16, 1024);
        if (F8) {
          // per 128 positions, [K hi^T | K mid^T | K lo^T] in one product: the three q
          // terms are the 48 rows of one B operand; 32 head dims (bytes) of each row per
          // instruction; positions 128 h .. 128 h + 127 (rows of the tile 16 KB apart)
          // into columns 48 h .. 48 h + 47 of the S buffer
#pragma unroll
          for (int h = 0; h < C::kSub; ++h)
#pragma unroll
            for (int kk = 0; kk < HD / 32; ++kk)
              tc_mma_f8_ss(tmem + sb * C::kSCols + h * NQ * kQTerms,
                           desc_advance(aK, h * kRegion + kk * 32), desc_advance(bQ, kk * 32), idS,
                           kk > 0 ? 1u : 0u);
        } else {
#pragma unroll
          for (int kk = 0; kk < HD / 16; ++kk)
            tc_mma_f16_ss(tmem + sb * C::kSCols, desc_advance(aK, (kk >> 2) * kRegion + (kk & 3) * 32),
                          desc_advance(bQ, (kk >> 2) * kQRegion + (kk & 3) * 32), idS,
                          kk > 0 ? 1u : 0u);
        }
        tc_commit(&s_full[sb]);
        tc_commit(&k_empty[kslot]);  // K slot reusable
        ++js;
        if (++is == s_nt) {
          tc_commit(&item_empty[ks % QN]);  // Q slot reusable
          s_in = false;
          ++ks;
        }
        return true;
      };
      // O^T(obuf) += V^T(t) P^T(t); `first` overwrites instead of accumulating
      // (false: P, V or the accumulator is not ready yet)
      auto pv = [&](unsigned t, bool first, int obuf, int item) -> bool {
        const int b = t % NP;
        const int vs = t % NV;
        // the first value MMA of an item overwrites O(obuf): the epilogue of the item
        // that used this accumulator NO items ago must have read it
        if (!__all_sync(0xffffffffu, mbar_test_wait(&p_full[b], (t / NP) & 1) &&
                                         mbar_test_wait(&v_full[vs], (t / NV) & 1) &&
                                         (!first || item < NO ||
                                          mbar_test_wait(&o_free[obuf], ((item / NO) - 1) & 1))))
          return false;
        tc_fence_after();
        // one descriptor per operand, stepped by constant offsets (see desc_advance)
        const uint64_t aV = smem_desc_sw128(smem_u32(smem + C::kOffV + vs * kTileBytes),
                                            kRegion, 1024);
        const uint64_t bP = smem_desc_sw128(sP + b * C::kPBytes, 16, 1024);
        const uint32_t dO = tmem + C::kTmemO + obuf * C::kOCols;
        if (F8) {
          // 32 positions (4 rows of 8-row swizzle atoms) per instruction; P's hi and lo
          // terms are one B operand of 32 rows (per 128 positions: a chunk of P^T), so
          // O_hi and O_lo come out side by side
#pragma unroll
          for (int kk = 0; kk < C::TT / 32; ++kk)
            tc_mma_f8_ss(dO, desc_advance(aV, kk * 32 * 128),
                         desc_advance(bP, (kk >> 2) * kPChunk + (kk & 3) * 32), idO,
                         (first && kk == 0) ? 0u : 1u);
        } else {
#pragma unroll
          for (int kk = 0; kk < TM / 16; ++kk)
            tc_mma_f16_ss(dO, desc_advance(aV, kk * 16 * 128),
                          desc_advance(bP, (kk >> 2) * kQRegion + (kk & 3) * 32), idO,
                          (first && kk == 0) ? 0u : 1u);
        }
        tc_commit(&pv_done[b]);
        tc_commit(&v_empty[vs]);
        return true;
      };
      // Event loop: a value MMA whenever its P, V and accumulator are ready (the
      // softmax and the V ring wait on it), else a score MMA up to kLookahead tiles
      // ahead whenever its item, K tile and S buffer are ready; when nothing is, wait
      // briefly on the barrier most likely to complete next. The idle time is bounded.
      unsigned long long idle_since = 0;
      while (true) {
        bool progressed = false;
        if (jp < js && pv(jp, ip == 0, kp % NO, kp)) {
          ++jp;
          if (++ip == nt_ring[kp & 7]) {
            tc_commit(&o_full[kp % NO]);  // O complete once the MMAs so far are done
            ip = 0;
            ++kp;
          }
          progressed = true;
        } else if (js < jp + kLookahead && ks - kp < 7 && score()) {
          progressed = true;
        }
        if (jp == js && s_end) break;  // every item done
        if (progressed) {
          idle_since = 0;
          continue;
        }
        if (jp < js)
          mbar_try_wait(&p_full[jp % NP], (jp / NP) & 1);
        else if (s_in)
          mbar_try_wait(&k_full[js % NK], (js / NK) & 1);
        else
          mbar_try_wait(&item_full[ks % QN], (ks / QN) & 1);
        const unsigned long long now = globaltimer_ns();
        if (idle_since == 0) idle_since = now;
        const bool give_up = *abort_flag || now - idle_since > wl;
        if (__any_sync(0xffffffffu, give_up)) {
          if (!*abort_flag) {
            if (lane == 0) flag_error(p.err, PA_DEV_ERR_TIMEOUT);
            *abort_flag = 1;
          }
          break;
        }
      }
      // every MMA this thread issued has finished before TMEM and shared memory go away
      tc_commit(mma_drain);
      mbar_wait(mma_drain, 0, p.err);
    }
  } else if (warp < 4 || (SG == 2 && warp >= 11)) {
    // ======================================================== softmax warps 0-3 (+ 11-14)
    // Control flow stays uniform across the softmax threads: a wait that fails (time
    // limit, or another role gave up) only marks `failed`; the group leaves together
    // at an item boundary through a barrier vote, so no thread can strand the others
    // at a named barrier.
    const int sg = warp < 4 ? 0 : 1;         // softmax group
    const int quad = warp & 3;               // TMEM lane quadrant of this warp
    const int wi = sg * 4 + quad;            // this warp's slot in the exchange buffers
    const int r = quad * 32 + lane;          // position within a 128-position product = TMEM lane
    const uint32_t lane_off = static_cast<uint32_t>(quad * 32) << 16;
    // the tile's 128-position products this thread takes: its group's half with two
    // groups, else every one
    constexpr int PT = SG == 2 ? 1 : C::kSub;
    auto sub_of = [&](int t) { return SG == 2 ? sg : t; };
    // e4m3: byte offsets of this thread's positions' scales within a tile's scale area
    int soff[PT];
#pragma unroll
    for (int t = 0; t < PT; ++t) {
      const int pos = sub_of(t) * TM + r;
      soff[t] = (pos / srows) * sstride + (pos % srows) * 4;
    }
    int k = 0;
    unsigned j = 0;  // tiles of this CTA done
    while (true) {
      const int slot = k % QN;
      bool failed = !wait_or_abort(&item_full[slot], (k / QN) & 1, p.err, abort_flag, wl);
      const ItemDesc d = descs[slot];
      // e4m3: the item's per-head q scales, written with its q terms
      if (F8 && !d.stop)
        failed |= !wait_or_abort(&q_ready[slot], (k / QN) & 1, p.err, abort_flag, wl);
      float qsg[G];
#pragma unroll
      for (int h = 0; h < G; ++h) qsg[h] = F8 ? qscale[slot * NQ + h] : 1.f;
      if (bar_or(1, kSoftThreads, failed)) break;  // every thread has read the descriptor
      if (tid == 0) mbar_arrive(&item_empty[slot]);
      if (d.stop) {
        if (tid == 0) {  // tell the epilogue warps, once they have read slot k % NO
          const int b = k % NO;
          if (k < NO ||
              wait_or_abort(&epi_empty[b], ((k / NO) - 1) & 1, p.err, abort_flag, wl)) {
            reinterpret_cast<ItemDesc*>(smem + C::kOffEpi + b * kEpiBytes)->stop = 1;
            mbar_arrive(&epi_full[b]);
          }
        }
        break;
      }
      const int obuf = k % NO;
      float m[G], lp[G], R[G];
#pragma unroll
      for (int h = 0; h < G; ++h) {
        m[h] = -INFINITY;
        lp[h] = 0.f;
        R[h] = -INFINITY;  // e4m3: O's reference, unset until a tile has a non-zero V scale
      }
      // A tile is kSub products of 128 positions: thread r owns position r of the ones
      // it takes (see sub_of)
      constexpr int SUB = PT;
      for (int i = 0; i < d.ntiles; ++i, ++j) {
        const int sb = j % NS;
        bool valid[SUB];
#pragma unroll
        for (int u = 0; u < SUB; ++u) valid[u] = i * C::TT + sub_of(u) * TM + r < d.n;
        // e4m3: the tile's K and V row scales first: they land with the tiles, well
        // before the score MMA is done, so their waits and reads overlap it
        float skr[SUB], svr[SUB];  // svr: this position's V scale (0 past the partition)
#pragma unroll
        for (int u = 0; u < SUB; ++u) {
          skr[u] = 1.f;
          svr[u] = 0.f;
        }
        if constexpr (F8) {
          const int kl = j % NSC;
          failed |= !wait_or_abort(&ksc_full[kl], (j / NSC) & 1, p.err, abort_flag, wl);
#pragma unroll
          for (int u = 0; u < SUB; ++u)
            skr[u] = *reinterpret_cast<const float*>(smem + C::kOffScl + kl * kSclBytes + soff[u]);
          __syncwarp();
          if (lane == 0) mbar_arrive(&ksc_empty[kl]);
          const int vs = j % NV;
          failed |= !wait_or_abort(&vsc_full[vs], (j / NV) & 1, p.err, abort_flag, wl);
#pragma unroll
          for (int u = 0; u < SUB; ++u)
            if (valid[u])
              svr[u] = *reinterpret_cast<const float*>(smem + C::kOffScl + (NSC + vs) * kSclBytes +
                                                       soff[u]);
        }
        failed |= !wait_or_abort(&s_full[sb], (j / NS) & 1, p.err, abort_flag, wl);
        tc_fence_after();
        float sv[SUB][G];
#pragma unroll
        for (int u = 0; u < SUB; ++u) {
          const uint32_t ts = tmem + sb * C::kSCols + sub_of(u) * NQ * kQTerms + lane_off;
          tmem_ld_cols<G>(ts, sv[u]);
          if constexpr (F8) {
            // S = products with the hi, mid and lo q terms, summed
            float s1[G], s2[G];
            tmem_ld_cols<G>(ts + NQ, s1);
            tmem_ld_cols<G>(ts + 2 * NQ, s2);
            tc_wait_ld();
#pragma unroll
            for (int h = 0; h < G; ++h) sv[u][h] = (sv[u][h] + s1[h]) + s2[h];
          }
        }
        tc_wait_ld();
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(&s_free[sb]);
        float x[SUB][G];
#pragma unroll
        for (int u = 0; u < SUB; ++u) {
          if constexpr (F8) {
            const float fr = p.scale_log2 * skr[u];
#pragma unroll
            for (int h = 0; h < G; ++h) x[u][h] = valid[u] ? sv[u][h] * (fr * qsg[h]) : -INFINITY;
          } else {
#pragma unroll
            for (int h = 0; h < G; ++h) x[u][h] = valid[u] ? sv[u][h] * p.scale_log2 : -INFINITY;
          }
        }
        // per-head max over the tile: warp shuffles, then across the 4 warps
        float* rb = red + (j & 1) * 8 * NQ;
#pragma unroll
        for (int h = 0; h < G; ++h) {
          float v = x[0][h];
#pragma unroll
          for (int u = 1; u < SUB; ++u) v = fmaxf(v, x[u][h]);
#pragma unroll
          for (int o = 16; o > 0; o >>= 1) v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, o));
          if (lane == 0) rb[wi * NQ + h] = v;
        }
        float* svb = red + 3 * 8 * NQ + (j & 1) * 8;  // e4m3: the tile's largest V scale
        if (F8) {
          float v = svr[0];
#pragma unroll
          for (int u = 1; u < SUB; ++u) v = fmaxf(v, svr[u]);
#pragma unroll
          for (int o = 16; o > 0; o >>= 1) v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, o));
          if (lane == 0) svb[wi] = v;
        }
        named_bar_sync(1, kSoftThreads);
        bool rescale = false;
        auto tile_max = [&](int h) {
          float v = rb[h];
#pragma unroll
          for (int w = 1; w < 4 * SG; ++w) v = fmaxf(v, rb[w * NQ + h]);
          return v;
        };
        float alpha[G];
        float pp[SUB][G];  // P' (e4m3) or P (bf16) of this thread's positions per head
        if constexpr (F8) {
          // bound of P' over the tile: 2^(max x + log2 max s_v - R)
          float smax = svb[0];
#pragma unroll
          for (int w = 1; w < 4 * SG; ++w) smax = fmaxf(smax, svb[w]);
          const float lsm = lg2_approx(smax);
          float lsv[SUB];
#pragma unroll
          for (int u = 0; u < SUB; ++u) lsv[u] = lg2_approx(svr[u]);  // -inf for s_v = 0
#pragma unroll
          for (int h = 0; h < G; ++h) {
            const float mx = tile_max(h);
            // l's reference (the row sum stays fp32, only its range matters)
            if (i == 0) {
              m[h] = mx;
            } else if (mx > m[h] + kRescaleLog2) {
              lp[h] *= ex2_approx(m[h] - mx);
              m[h] = mx;
            }
#pragma unroll
            for (int u = 0; u < SUB; ++u) lp[h] += valid[u] ? ex2_approx(x[u][h] - m[h]) : 0.f;
            // O's reference: set by the first tile with a non-zero V scale (O is exactly
            // 0 before it), raised when the bound would pass 2^kPBoundLog2
            alpha[h] = 1.f;
            const float bnd = mx + lsm;
            if (R[h] == -INFINITY) {
              if (bnd > -INFINITY) R[h] = bnd - kPTargetLog2;
            } else if (bnd > R[h] + kPBoundLog2) {
              const float rn = bnd - kPTargetLog2;
              alpha[h] = ex2_approx(R[h] - rn);
              R[h] = rn;
              rescale = true;
            }
#pragma unroll
            for (int u = 0; u < SUB; ++u)
              pp[u][h] = (valid[u] && R[h] > -INFINITY) ? ex2_approx(x[u][h] + lsv[u] - R[h]) : 0.f;
          }
        } else {
#pragma unroll
          for (int h = 0; h < G; ++h) {
            const float mx = tile_max(h);
            alpha[h] = 1.f;
            if (i == 0) {
              m[h] = mx;  // reference max of this item (every tile has a valid position)
            } else if (mx > m[h] + kRescaleLog2) {
              alpha[h] = ex2_approx(m[h] - mx);
              m[h] = mx;
              rescale = true;
            }
            float ps = 0.f;
#pragma unroll
            for (int u = 0; u < SUB; ++u) {
              pp[u][h] = valid[u] ? ex2_approx(x[u][h] - m[h]) : 0.f;
              ps += pp[u][h];
            }
            lp[h] = lp[h] * alpha[h] + ps;
          }
        }
        // this P^T buffer was last read by the value MMA of tile j - NP
        const int pb = j % NP;
        if (j >= NP)
          failed |= !wait_or_abort(&pv_done[pb], ((j / NP) - 1) & 1, p.err, abort_flag, wl);
        if constexpr (F8) {
          // row h of P^T (K-major, 128 positions = 128 bytes per chunk, 128-byte
          // swizzle): byte r of chunk u; the lo terms kQRegion after the hi ones
#pragma unroll
          for (int u = 0; u < SUB; ++u) {
            uint8_t* pt = smem + C::kOffP + pb * C::kPBytes + sub_of(u) * kPChunk;
#pragma unroll
            for (int h = 0; h < G; h += 2) {
              uint32_t hi, lo;
              split_e4m3x2(pp[u][h], h + 1 < G ? pp[u][h + 1] : 0.f, kPLoScale, hi, lo);
#pragma unroll
              for (int e = 0; e < 2 && h + e < G; ++e) {
                const int hh = h + e;
                const int off = hh * 128 + ((((r >> 4) ^ hh) & 7) << 4) + (r & 15);
                pt[off] = static_cast<uint8_t>(hi >> (8 * e));
                pt[kQRegion + off] = static_cast<uint8_t>(lo >> (8 * e));
              }
            }
          }
        } else {
          uint8_t* pt = smem + C::kOffP + pb * C::kPBytes + (r >> 6) * kQRegion;
#pragma unroll
          for (int h = 0; h < G; ++h) {
            const int chunk = ((r & 63) >> 3) ^ (h & 7);
            *reinterpret_cast<__nv_bfloat16*>(pt + h * 128 + chunk * 16 + (r & 7) * 2) =
                __float2bfloat16_rn(pp[0][h]);
          }
        }
        if (i == d.ntiles - 1 && d.n - i * C::TT < C::TT) {
          // V rows past the partition's end may hold anything (even NaN); P is 0 there
          // but 0 * NaN is NaN: clear them before the tensor core reads the tile
          const int vs = j % NV;
          failed |= !wait_or_abort(&v_full[vs], (j / NV) & 1, p.err, abort_flag, wl);
#pragma unroll
          for (int u = 0; u < SUB; ++u) {
            if (!valid[u]) {
              // e4m3: row u * 128 + r of 128 bytes; bf16: row r in both 64-dim halves
              uint8_t* v = smem + C::kOffV + vs * kTileBytes + (sub_of(u) * TM + r) * 128;
#pragma unroll
              for (int c = 0; c < 8; ++c) {
                *reinterpret_cast<uint4*>(v + c * 16) = make_uint4(0, 0, 0, 0);
                if (!F8) *reinterpret_cast<uint4*>(v + kRegion + c * 16) = make_uint4(0, 0, 0, 0);
              }
            }
          }
        }
        // uniform across the groups (every thread saw the same tile max); group 0's
        // warps cover all 128 TMEM lanes of O, so it rescales alone
        if (sg == 0 && rescale) {
          // O holds the value MMAs up to tile j-1: wait for the last of them
          const unsigned t = j - 1;
          failed |= !wait_or_abort(&pv_done[t % NP], (t / NP) & 1, p.err, abort_flag, wl);
          tc_fence_after();
          float o[16];
          tmem_ld16(tmem + C::kTmemO + obuf * C::kOCols + lane_off, o);
          tc_wait_ld();
#pragma unroll
          for (int h = 0; h < G; ++h) o[h] *= alpha[h];
          tmem_st16(tmem + C::kTmemO + obuf * C::kOCols + lane_off, o);
          if (F8) {  // the lo accumulator, next to the hi one
            tmem_ld16(tmem + C::kTmemO + obuf * C::kOCols + NQ + lane_off, o);
            tc_wait_ld();
#pragma unroll
            for (int h = 0; h < G; ++h) o[h] *= alpha[h];
            tmem_st16(tmem + C::kTmemO + obuf * C::kOCols + NQ + lane_off, o);
          }
          tc_wait_st();
        }
        fence_proxy_async_smem();
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(&p_full[pb]);
      }
      // hand the item to the epilogue warps: l per head (the per-position shares summed
      // over the 128 threads), the reference max and, for e4m3, O's factor 2^(R - m);
      // O^T stays in TMEM
      float* lb = red + 2 * 8 * NQ;
#pragma unroll
      for (int h = 0; h < G; ++h) {
        float v = lp[h];
#pragma unroll
        for (int off = 16; off > 0; off >>= 1) v += __shfl_xor_sync(0xffffffffu, v, off);
        if (lane == 0) lb[wi * NQ + h] = v;
      }
      named_bar_sync(1, kSoftThreads);
      if (tid == 0) {
        const int b = k % NO;
        if (k >= NO)
          failed |= !wait_or_abort(&epi_empty[b], ((k / NO) - 1) & 1, p.err, abort_flag, wl);
        if (!failed) {
          uint8_t* es = smem + C::kOffEpi + b * kEpiBytes;
          *reinterpret_cast<ItemDesc*>(es) = d;
          float* em = reinterpret_cast<float*>(es + 32);
#pragma unroll
          for (int h = 0; h < G; ++h) {
            em[h] = m[h];
            float L = 0.f;
            for (int w = 0; w < 4 * SG; ++w) L += lb[w * NQ + h];
            em[NQ + h] = L;
            em[2 * NQ + h] = (F8 && R[h] > -INFINITY) ? ex2_approx(R[h] - m[h]) : (F8 ? 0.f : 1.f);
          }
          mbar_arrive(&epi_full[b]);
        }
      }
      if (bar_or(1, kSoftThreads, failed)) break;
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
      bool failed = !wait_or_abort(&epi_full[b], (k / NO) & 1, p.err, abort_flag, wl);
      const uint8_t* es = smem + C::kOffEpi + b * kEpiBytes;
      const ItemDesc d = *reinterpret_cast<const ItemDesc*>(es);
      float m[G], L[G], fac[G];
#pragma unroll
      for (int h = 0; h < G; ++h) {
        m[h] = reinterpret_cast<const float*>(es + 32)[h];
        L[h] = reinterpret_cast<const float*>(es + 32)[NQ + h];
        fac[h] = reinterpret_cast<const float*>(es + 32)[2 * NQ + h];
      }
      if (bar_or(2, 128, failed)) break;  // every epilogue thread has read the hand-off
      if (leader) mbar_arrive(&epi_empty[b]);
      if (d.stop) break;
      failed |= !wait_or_abort(&o_full[b], (k / NO) & 1, p.err, abort_flag, wl);
      tc_fence_after();
      float o[16];
      tmem_ld16(tmem + C::kTmemO + b * C::kOCols + lane_off, o);
      if (F8) {
        float olo[16];
        tmem_ld16(tmem + C::kTmemO + b * C::kOCols + NQ + lane_off, olo);
        tc_wait_ld();
#pragma unroll
        for (int h = 0; h < G; ++h) o[h] = fmaf(olo[h], 1.f / kPLoScale, o[h]) * fac[h];
      } else {
        tc_wait_ld();
      }
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
          // this kernel's partitions of (s, g) (the shared prefix's one came earlier)
          const int arrivals = d.nparts - (p.shared_len > 0 ? 1 : 0);
          *last_flag = okc && (before == static_cast<unsigned>(arrivals - 1));
          __threadfence();
        }
        named_bar_sync(2, 128);
        if (*last_flag) {
          // this CTA completed the last partition of (s, g): merge all of them. Each
          // head's partials are read eight partitions at a time in one pass (m, l and
          // this thread's o element together, an online max across the chunks), and no
          // output is stored before every head's loads, so the loads of all heads can be
          // in flight together: one round trip per chunk, not two per head and chunk
          constexpr int CH = 8;
          float res[G];
#pragma unroll
          for (int h = 0; h < G; ++h) {
            const int64_t base = (row0 + h) * p.max_parts;
            const int np = d.nparts;
            float M = -INFINITY, Ls = 0.f, acc = 0.f;
#pragma unroll 1
            for (int q0 = 0; q0 < np; q0 += CH) {
              float2 ml[CH];
              float oo[CH];
#pragma unroll
              for (int i = 0; i < CH; ++i) {
                const bool in = q0 + i < np;
                ml[i] = in ? __ldcg(reinterpret_cast<const float2*>(p.ws_ml) + base + q0 + i)
                           : make_float2(-INFINITY, 0.f);
                oo[i] = in ? __ldcg(p.ws_o + (base + q0 + i) * HD + dl) : 0.f;
              }
              float Mc = M;
#pragma unroll
              for (int i = 0; i < CH; ++i) Mc = fmaxf(Mc, ml[i].x);
              // every partition has a finite max (it holds at least one position)
              const float r = ex2_approx(M - Mc);  // 0 on the first chunk (M = -inf)
              Ls *= r;
              acc *= r;
#pragma unroll
              for (int i = 0; i < CH; ++i) {
                const float f = ex2_approx(ml[i].x - Mc);
                Ls += ml[i].y * f;
                acc += oo[i] * f;
              }
              M = Mc;
            }
            res[h] = acc / Ls;
          }
#pragma unroll
          for (int h = 0; h < G; ++h) p.out[(row0 + h) * HD + dl] = __float2bfloat16_rn(res[h]);
        }
      }
      if (bar_or(2, 128, failed)) break;  // also orders last_flag's reuse
      ++k;
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 5) {
    tc_fence_after();
    tmem_dealloc(tmem, C::kTmemCols);
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
  const int rows = bs < Cfg<F8>::TT ? bs : Cfg<F8>::TT;  // positions per TMA box
  const uint64_t slots = static_cast<uint64_t>(a.cache.num_blocks) * bs;
  const uint64_t hkv = static_cast<uint64_t>(a.cache.num_kv_heads);
  CUtensorMap tmQ, tmK, tmV, tmSK, tmSV;
  if (!encode_tensor_map_3d(&tmQ, a.q, HD, a.num_q_heads, a.num_seqs, 64, G, 1, true))
    return cudaErrorInvalidValue;
  if (F8) {
    // codes [slots][Hkv][D] bytes, 128-byte rows, 128-byte swizzle (the MMA operand
    // layout); scales [Hkv][slots] fp32, a run of `rows` positions of one kv head per box
    const uint64_t cd[3] = {HD, hkv, slots};
    const uint32_t cb[3] = {HD, 1, static_cast<uint32_t>(rows)};
    const uint64_t sd[2] = {slots, hkv};
    const uint32_t sb[2] = {static_cast<uint32_t>(rows), 1};
    if (!encode_tensor_map(&tmK, a.k_cache, CU_TENSOR_MAP_DATA_TYPE_UINT8, 1, 3, cd, cb, true) ||
        !encode_tensor_map(&tmV, a.v_cache, CU_TENSOR_MAP_DATA_TYPE_UINT8, 1, 3, cd, cb, true) ||
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
  constexpr int smem_bytes = Cfg<F8>::kSmemBytes;
  cudaError_t e = ensure_max_dynamic_smem(reinterpret_cast<const void*>(decode_tc_kernel<G, F8>),
                                          smem_bytes);
  if (e != cudaSuccess) return e;
  int grid = sm_count();
  if (static_cast<unsigned>(grid) > p.total_items) grid = static_cast<int>(p.total_items);
  if (grid < 1) grid = 1;
  decode_tc_kernel<G, F8><<<grid, kThreadsOf<G, F8>, smem_bytes, stream>>>(tmQ, tmK, tmV, tmSK,
                                                                          tmSV, p);
  return cudaGetLastError();
}

}  // namespace

bool decode_tc_supported(const DecodeLaunch& a) {
  const int G = a.num_q_heads / a.cache.num_kv_heads;
  const bool g_ok = G == 1 || G == 2 || G == 4 || G == 8 || G == 16;
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
  p.q = static_cast<const __nv_bfloat16*>(a.q);
  p.block_tables = a.block_tables;
  p.context_lens = a.context_lens;
  p.counters = counters;
  p.ws_o = a.ws_o;
  p.ws_ml = a.ws_ml;
  p.err = device_error_word();
  p.tag = next_tag();
  p.wait_ns = wait_limit_ns();
  p.num_seqs = a.num_seqs;
  p.num_kv_heads = a.cache.num_kv_heads;
  p.max_blocks = a.max_blocks_per_seq;
  p.num_blocks = a.cache.num_blocks;
  p.bs_log2 = 31 - __builtin_clz(static_cast<unsigned>(a.cache.block_size));
  p.partition_size = a.partition_size;
  p.max_parts = a.max_parts;
  p.max_context_len = a.max_context_len;
  p.shared_len = a.shared_len;
  p.total_items = static_cast<unsigned>(a.max_parts - (a.shared_len > 0 ? 1 : 0)) * a.num_seqs *
                  a.cache.num_kv_heads;
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
      case 16: return launch_tc_t<16, true>(a, p, stream);
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

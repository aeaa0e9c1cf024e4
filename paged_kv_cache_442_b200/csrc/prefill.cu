// Causal paged prefill on the tcgen05 tensor cores: a chunk of new tokens of each
// sequence attends to the sequence's cached prefix plus itself (nano vllm page,
// section 3.1: num_cached_tokens of a Sequence are reused; mini-vllm page,
// section 1: blocks are allocated for the prefill; all K/V are read through the
// block table, section 2).
//
// One CTA = 128 query rows of one (sequence, query head). Per KV tile of 128
// positions:  S = Q K^T  (tcgen05.mma, M=128 N=128 K=128, fp32 in TMEM)
//             softmax on S, P written back to TMEM as bf16
//             O += P V    (tcgen05.mma with A = P read from TMEM, B = V from shared
//                          memory, accumulator in TMEM)
// Roles (320 threads):
//   warps 0-7  softmax + epilogue. Warp w reads TMEM lanes 32(w%4).. (its 32 query
//              rows) and the column half w/4 of each tile, so every row is shared by
//              two warps on the same SM sub-partition: two warps per scheduler hide
//              each other's latencies, and each thread keeps 64 scores in registers.
//              The two halves agree on the row max through shared memory.
//   warp 8     TMA producer: Q once, then K and V tiles gathered block by block
//              through the block table into two 3-deep rings (K runs two tiles ahead
//              of V; a K slot frees when its score MMA is done, a V slot when its
//              value MMA is done).
//   warp 9     owns the TMEM allocation and issues the MMAs from one thread.
// S and P are double-buffered in TMEM, and O is rescaled only when a row's running
// max grows by more than 2^8 (probabilities stay <= 256: in range for bf16). The
// tensor core runs its queue in order, so S(j+2) is issued as soon as the softmax has
// read S(j), ahead of O += P(j) V(j): the next scores never queue behind a value MMA
// that waited for the softmax, and the exp2 work overlaps both MMAs. P never touches
// shared memory, whose bandwidth the score MMA and the TMA writes use.
// Shared-memory operands use the 128-byte swizzled K-major layout (Q, K) and the
// MN-major layout (V, whose head dim is contiguous), both produced directly by TMA.
#include <cuda_bf16.h>

#include "pa_internal.h"
#include "pa_ptx.cuh"

namespace pa {
namespace {

constexpr int BM = 128;          // query rows per CTA
constexpr int BN = 128;          // KV positions per tile
constexpr int HD = 128;          // head dim
constexpr int kSoftmaxWarps = 8;
constexpr int kProducerWarp = 8;
constexpr int kIssuerWarp = 9;
constexpr int kThreads = 320;
constexpr int NK = 3;            // K ring depth
constexpr int NV = 3;            // V ring depth
constexpr int kKAhead = 2;       // K loads run this many tiles ahead of V loads
constexpr int kRegion = BM * 128;  // one 64-column half of a 128x128 bf16 tile (16 KB)
constexpr int kTileBytes = 2 * kRegion;
// Small objects first (8-byte aligned at the start of dynamic shared memory), then
// the 1024-byte-aligned operand tiles.
constexpr int kNumBars = 2 + 2 * NK + 2 * NV + 4 * 2;  // q, drain, K/V rings, s/p/pv pairs
constexpr int kOffXch = 8 * kNumBars;                  // [2 halves][128 rows] fp32
constexpr int kOffMisc = kOffXch + 2 * BM * 4;         // tmem address, abort flag
constexpr int kSmallBytes = kOffMisc + 16;
constexpr int kOffQ = 0;                               // within the aligned region
constexpr int kOffK = kOffQ + kTileBytes;
constexpr int kOffV = kOffK + NK * kTileBytes;
constexpr int kDataBytes = kOffV + NV * kTileBytes;
constexpr int kSmemBytes = kSmallBytes + 1023 + kDataBytes;  // worst-case alignment pad
static_assert(kOffK % 1024 == 0 && kOffV % 1024 == 0,
              "128-byte-swizzled TMA / MMA operands need 1024-byte alignment");
static_assert(kOffXch % 8 == 0 && kOffMisc % 8 == 0, "mbarriers / words alignment");
static_assert(kSmemBytes <= 227 * 1024, "shared memory per CTA");
constexpr float kLog2e = 1.4426950408889634f;
constexpr float kRescaleLog2 = 8.f;   // rescale O only past this growth of the row max
constexpr uint32_t kTmemCols = 512;   // S[0] 0-127, S[1] 128-255, O 256-383, P[0] 384-447, P[1] 448-511
constexpr uint32_t kTmemO = 256;
constexpr uint32_t kTmemP = 384;      // P: 128 bf16 per row = 64 columns

struct PrefillParams {
  __nv_bfloat16* out;
  const int32_t* block_tables;
  const int32_t* cu_seqlens_q;
  const int32_t* context_lens;
  unsigned* err;
  int max_blocks;
  int num_blocks;
  int bs_log2;
  int num_q_heads;
  int group;  // Hq / Hkv
  int total_q;
  int max_q_len;
  float scale_log2;
};

// bounded wait that also gives up when another role has already given up
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

// named barrier over the two softmax warps that share a group of 32 rows
__device__ __forceinline__ void pair_sync(int id) {
  asm volatile("bar.sync %0, 64;" ::"r"(id) : "memory");
}

// kPosScale: scale > 0, so the row max can be taken on the raw scores and the scale
// folded into the exponent's FMA; otherwise (scale <= 0) the scores are scaled first.
template <bool kPosScale>
__global__ void __launch_bounds__(kThreads, 1) prefill_kernel(
    const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
    const __grid_constant__ CUtensorMap tmV, const PrefillParams p) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* small = smem_raw;
  uint8_t* smem = reinterpret_cast<uint8_t*>(
      (reinterpret_cast<uintptr_t>(smem_raw + kSmallBytes) + 1023) &
      ~static_cast<uintptr_t>(1023));

  const int tid = threadIdx.x;
  const int warp = tid >> 5;
  const int lane = tid & 31;
  const int qt = blockIdx.x;
  const int h = blockIdx.y;
  const int s = blockIdx.z;
  const int g = h / p.group;

  const int q0 = __ldg(p.cu_seqlens_q + s);
  const int n_new = __ldg(p.cu_seqlens_q + s + 1) - q0;
  const int ctx = __ldg(p.context_lens + s);
  if (qt * BM >= n_new) return;
  if (n_new > ctx || q0 < 0 || q0 + n_new > p.total_q || n_new > p.max_q_len) {
    // caller broke a precondition: compute nothing, write nothing
    if (tid == 0) flag_error(p.err, PA_DEV_ERR_BAD_INDEX);
    return;
  }
  const int first = ctx - n_new;                          // position of the first new token
  const int rows_valid = min(BM, n_new - qt * BM);
  const int pos_max = first + qt * BM + rows_valid - 1;   // last visible position in the tile
  const int ntiles = pos_max / BN + 1;
  const int bs = 1 << p.bs_log2;

  uint64_t* bars = reinterpret_cast<uint64_t*>(small);
  uint64_t* bar_q = bars;
  uint64_t* mma_drain = bars + 1;
  uint64_t* k_full = bars + 2;               // [NK] each
  uint64_t* k_empty = k_full + NK;
  uint64_t* v_full = k_empty + NK;           // [NV] each
  uint64_t* v_empty = v_full + NV;
  uint64_t* s_full = v_empty + NV;           // [2] each
  uint64_t* s_free = s_full + 2;
  uint64_t* p_full = s_free + 2;
  uint64_t* pv_done = p_full + 2;
  float* xch = reinterpret_cast<float*>(small + kOffXch);
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(small + kOffMisc);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(small + kOffMisc + 8);

  if (tid == 0) {
    mbar_init(bar_q, 1);
    mbar_init(mma_drain, 1);
    for (int i = 0; i < NK; ++i) {
      mbar_init(&k_full[i], 1);
      mbar_init(&k_empty[i], 1);
    }
    for (int i = 0; i < NV; ++i) {
      mbar_init(&v_full[i], 1);
      mbar_init(&v_empty[i], 1);
    }
    for (int i = 0; i < 2; ++i) {
      mbar_init(&s_full[i], 1);
      mbar_init(&s_free[i], kSoftmaxWarps);   // one arrival per softmax warp
      mbar_init(&p_full[i], kSoftmaxWarps);
      mbar_init(&pv_done[i], 1);
    }
    *abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == kIssuerWarp) {
    tmem_alloc(tmem_slot, kTmemCols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  const uint32_t tO = tmem + kTmemO;

  if (warp == kProducerWarp) {
    // ------------------------------------------------------------ TMA producer
    // lane 0 waits and issues; the verdict of each wait is broadcast so the warp
    // leaves the loop together
    auto wwait = [&](uint64_t* bar, unsigned parity) -> bool {
      int okw = 0;
      if (lane == 0) okw = wait_or_abort(bar, parity, p.err, abort_flag) ? 1 : 0;
      return __shfl_sync(0xffffffffu, okw, 0) != 0;
    };
    const int rows = bs < BN ? bs : BN;
    const int nbox = BN / rows;
    const uint64_t keep = policy_evict_last();  // K/V tiles are re-read by G heads and q tiles
    auto block_row = [&](int pos) {
      const int bi = pos >> p.bs_log2;
      int id = bi < p.max_blocks
                   ? __ldg(p.block_tables + static_cast<int64_t>(s) * p.max_blocks + bi)
                   : -1;
      if (id < 0 || id >= p.num_blocks) {
        if (pos < ctx) flag_error(p.err, PA_DEV_ERR_BAD_INDEX);
        id = 0;  // in-bounds stand-in; positions past the context are masked
      }
      return id * bs + (pos & (bs - 1));
    };
    auto load_tile = [&](const CUtensorMap* map, uint8_t* dst, uint64_t* bar, int j) {
      mbar_arrive_expect_tx(bar, kTileBytes);
      for (int c = 0; c < nbox; ++c) {
        const int row = block_row(j * BN + c * rows);
        tma_load_3d_hint(dst + c * rows * 128, map, bar, 0, g, row, keep);
        tma_load_3d_hint(dst + kRegion + c * rows * 128, map, bar, 64, g, row, keep);
      }
    };
    if (lane == 0) {
      prefetch_tensormap(&tmQ);
      prefetch_tensormap(&tmK);
      prefetch_tensormap(&tmV);
      const int qrow = q0 + qt * BM;
      mbar_arrive_expect_tx(bar_q, kTileBytes);
      tma_load_3d(smem + kOffQ, &tmQ, bar_q, 0, h, qrow);
      tma_load_3d(smem + kOffQ + kRegion, &tmQ, bar_q, 64, h, qrow);
    }
    int k_issued = 0, v_issued = 0;
    for (int step = 0; step < ntiles + kKAhead; ++step) {
      const int kj = step;            // K(kj) is needed early: by the score MMA
      const int vj = step - kKAhead;  // V(vj) only once the softmax of vj is done
      if (kj < ntiles) {
        const int ks = kj % NK;
        if (kj >= NK && !wwait(&k_empty[ks], ((kj / NK) - 1) & 1)) break;
        if (lane == 0) load_tile(&tmK, smem + kOffK + ks * kTileBytes, &k_full[ks], kj);
        k_issued = kj + 1;
      }
      if (vj >= 0 && vj < ntiles) {
        const int vs = vj % NV;
        if (vj >= NV && !wwait(&v_empty[vs], ((vj / NV) - 1) & 1)) break;
        if (lane == 0) load_tile(&tmV, smem + kOffV + vs * kTileBytes, &v_full[vs], vj);
        v_issued = vj + 1;
      }
    }
    // Before the CTA ends, every copy this warp started must have landed. Per slot
    // only the last load can still be in flight (the one before it was consumed),
    // so waiting for those is enough; on the normal path they completed long ago.
    if (lane == 0) {
      mbar_wait(bar_q, 0, p.err);
      for (int t = k_issued - NK > 0 ? k_issued - NK : 0; t < k_issued; ++t)
        mbar_wait(&k_full[t % NK], (t / NK) & 1, p.err);
      for (int t = v_issued - NV > 0 ? v_issued - NV : 0; t < v_issued; ++t)
        mbar_wait(&v_full[t % NV], (t / NV) & 1, p.err);
    }
  } else if (warp == kIssuerWarp) {
    // ------------------------------------------------------------ MMA issuer
    if (lane == 0) {
      constexpr uint32_t idS = idesc_bf16_f32(BM, BN, 0, 0);  // Q K-major, K K-major
      constexpr uint32_t idO = idesc_bf16_f32(BM, HD, 0, 1);  // P (TMEM), V MN-major
      const uint32_t sQ = smem_u32(smem + kOffQ);
      // S(j) into TMEM buffer j & 1, once K(j) has landed and the softmax has read
      // S(j-2) out of that buffer
      auto score = [&](int j) -> bool {
        const int b = j & 1;
        const int ks = j % NK;
        if (!wait_or_abort(&k_full[ks], (j / NK) & 1, p.err, abort_flag) ||
            (j >= 2 && !wait_or_abort(&s_free[b], ((j >> 1) - 1) & 1, p.err, abort_flag)))
          return false;
        tc_fence_after();
        const uint32_t sK = smem_u32(smem + kOffK + ks * kTileBytes);
#pragma unroll
        for (int kk = 0; kk < HD / 16; ++kk) {
          const uint32_t off = (kk >> 2) * kRegion + (kk & 3) * 32;
          tc_mma_f16_ss(tmem + b * 128, smem_desc_sw128(sQ + off, 16, 1024),
                        smem_desc_sw128(sK + off, 16, 1024), idS, kk > 0 ? 1u : 0u);
        }
        tc_commit(&s_full[b]);
        tc_commit(&k_empty[ks]);
        return true;
      };
      // O += P(t) V(t), once the softmax has written P(t) and V(t) has landed
      auto pv = [&](int t) -> bool {
        const int b = t & 1;
        const int vs = t % NV;
        if (!wait_or_abort(&p_full[b], (t >> 1) & 1, p.err, abort_flag) ||
            !wait_or_abort(&v_full[vs], (t / NV) & 1, p.err, abort_flag))
          return false;
        tc_fence_after();
        const uint32_t tP = tmem + kTmemP + b * (BN / 2);
        const uint32_t sV = smem_u32(smem + kOffV + vs * kTileBytes);
#pragma unroll
        for (int kk = 0; kk < BN / 16; ++kk) {
          // 16 kv positions per step = 8 packed columns of P
          const uint64_t bd = smem_desc_sw128(sV + kk * 16 * 128, kRegion, 1024);
          tc_mma_f16_ts(tO, tP + kk * 8, bd, idO, (t > 0 || kk > 0) ? 1u : 0u);
        }
        tc_commit(&pv_done[b]);
        tc_commit(&v_empty[vs]);
        return true;
      };
      bool ok = wait_or_abort(bar_q, 0, p.err, abort_flag);
      if (ok) ok = score(0);
      if (ok && ntiles > 1) ok = score(1);
      for (int j = 0; ok && j < ntiles; ++j) {
        if (j + 2 < ntiles) ok = score(j + 2);
        if (ok) ok = pv(j);
      }
      // every MMA this thread issued has finished before TMEM and shared memory go away
      tc_commit(mma_drain);
      mbar_wait(mma_drain, 0, p.err);
    }
  } else {
    // ------------------------------------------------------------ softmax warps
    // Every lane runs every step (the tcgen05 loads and stores are warp-collective,
    // and the pair barriers count both warps): a failed wait only marks `failed`.
    constexpr int HC = BN / 2;                // columns per half
    const int quad = warp & 3;
    const int half = warp >> 2;
    const int r = quad * 32 + lane;           // query row within the tile == TMEM lane
    const int pos_r = first + qt * BM + (r < rows_valid ? r : rows_valid - 1);
    const uint32_t lane_off = static_cast<uint32_t>(quad * 32) << 16;
    const int pair_bar = 1 + quad;
    float* my_x = xch + half * BM + r;
    const float* other_x = xch + (half ^ 1) * BM + r;
    float m = -INFINITY;
    float l = 0.f;                            // this half's share of the row sum
    bool failed = false;
    for (int j = 0; j < ntiles; ++j) {
      const int b = j & 1;
      failed |= !wait_or_abort(&s_full[b], (j >> 1) & 1, p.err, abort_flag);
      tc_fence_after();
      float sv[HC];
#pragma unroll
      for (int c = 0; c < HC / 32; ++c) {
        float t32[32];
        tmem_ld32(tmem + b * 128 + half * HC + lane_off + c * 32, t32);
#pragma unroll
        for (int i = 0; i < 32; ++i) sv[c * 32 + i] = t32[i];
      }
      tc_wait_ld();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&s_free[b]);

      const int kv0 = j * BN + half * HC;
      const int lim = pos_r - kv0;  // columns past lim are in this row's future: masked
      float hmx;
      if constexpr (kPosScale) {
        if (lim < HC - 1) {
#pragma unroll
          for (int c = 0; c < HC; ++c) sv[c] = c > lim ? -INFINITY : sv[c];
        }
        // max of the raw scores (the scale is positive), four independent chains
        float a0 = -INFINITY, a1 = -INFINITY, a2 = -INFINITY, a3 = -INFINITY;
#pragma unroll
        for (int c = 0; c < HC; c += 8) {
          a0 = fmax3(a0, sv[c + 0], sv[c + 1]);
          a1 = fmax3(a1, sv[c + 2], sv[c + 3]);
          a2 = fmax3(a2, sv[c + 4], sv[c + 5]);
          a3 = fmax3(a3, sv[c + 6], sv[c + 7]);
        }
        hmx = fmax3(a0, a1, fmaxf(a2, a3));
      } else {
#pragma unroll
        for (int c = 0; c < HC; ++c) sv[c] = c > lim ? -INFINITY : sv[c] * p.scale_log2;
        hmx = -INFINITY;
#pragma unroll
        for (int c = 0; c < HC; ++c) hmx = fmaxf(hmx, sv[c]);
      }
      // the two halves of the row swap their maxima: write, sync, read, sync (the
      // second sync keeps the next tile's write behind this read)
      *my_x = hmx;
      pair_sync(pair_bar);
      const float omx = *other_x;
      pair_sync(pair_bar);
      const float mx = kPosScale ? fmaxf(hmx, omx) * p.scale_log2 : fmaxf(hmx, omx);
      // reference max: the first tile's (position 0 is visible to every row), raised
      // only when a later tile exceeds it by more than 2^8; both halves compute the
      // same value from the same inputs
      float alpha = 1.f;
      bool rescale = false;
      if (j == 0) {
        m = mx;
      } else if (mx > m + kRescaleLog2) {
        alpha = ex2_approx(m - mx);
        m = mx;
        rescale = true;
      }
      // p = 2^(s * scale_log2 - m), two lanes of fp32 per instruction
      const float sc = kPosScale ? p.scale_log2 : 1.f;
      const float2 sc2 = make_float2(sc, sc);
      const float2 nm2 = make_float2(-m, -m);
      float2 acc[4] = {make_float2(0.f, 0.f), make_float2(0.f, 0.f), make_float2(0.f, 0.f),
                       make_float2(0.f, 0.f)};
      uint32_t pk[HC / 2];
#pragma unroll
      for (int c = 0; c < HC; c += 2) {
        const float2 x = __ffma2_rn(make_float2(sv[c], sv[c + 1]), sc2, nm2);
        const float2 e = make_float2(ex2_approx(x.x), ex2_approx(x.y));
        acc[(c >> 1) & 3] = __fadd2_rn(acc[(c >> 1) & 3], e);
        pk[c >> 1] = pack_bf16x2(e.x, e.y);
      }
      const float rs = ((acc[0].x + acc[0].y) + (acc[1].x + acc[1].y)) +
                       ((acc[2].x + acc[2].y) + (acc[3].x + acc[3].y));
      l = l * alpha + rs;

      // P buffer b was last read by the value MMA of tile j-2
      if (j >= 2) failed |= !wait_or_abort(&pv_done[b], ((j >> 1) - 1) & 1, p.err, abort_flag);
      tc_fence_after();
      if (__any_sync(0xffffffffu, rescale)) {
        // O holds the value MMAs up to tile j-1: wait for the last one, then rescale
        // this half's columns (rows that do not need it multiply by 1)
        const int t = j - 1;
        failed |= !wait_or_abort(&pv_done[t & 1], (t >> 1) & 1, p.err, abort_flag);
        tc_fence_after();
#pragma unroll
        for (int c = 0; c < HC / 32; ++c) {
          float o[32];
          tmem_ld32(tO + half * HC + lane_off + c * 32, o);
          tc_wait_ld();
#pragma unroll
          for (int i = 0; i < 32; ++i) o[i] *= alpha;
          tmem_st32(tO + half * HC + lane_off + c * 32, o);
        }
      }
      if (j == ntiles - 1 && ctx - j * BN < BN) {
        // rows past the context in the last V tile may hold anything (even NaN);
        // P is 0 there but 0 * NaN is NaN, so clear them before the value MMA.
        // Thread (quad, lane, half) clears head-dim half `half` of V row r.
        const int vs = j % NV;
        failed |= !wait_or_abort(&v_full[vs], (j / NV) & 1, p.err, abort_flag);
        if (r >= ctx - j * BN) {
          uint8_t* v = smem + kOffV + vs * kTileBytes + half * kRegion + r * 128;
          const uint4 z = make_uint4(0, 0, 0, 0);
#pragma unroll
          for (int c = 0; c < 8; ++c) *reinterpret_cast<uint4*>(v + c * 16) = z;
        }
        fence_proxy_async_smem();
      }
      // this half of the P row -> TMEM: 32 columns of packed bf16 pairs (the A-operand
      // layout: row in the lane, consecutive kv positions in consecutive half-words)
      tmem_st32_bits(tmem + kTmemP + b * (BN / 2) + half * (HC / 2) + lane_off, pk);
      tc_wait_st();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&p_full[b]);
    }
    const int t = ntiles - 1;
    failed |= !wait_or_abort(&pv_done[t & 1], (t >> 1) & 1, p.err, abort_flag);
    tc_fence_after();
    // row sum = both halves' shares (the exchange slots are free: the last read of
    // them is behind the final pair barrier of the loop)
    *my_x = l;
    pair_sync(pair_bar);
    const float inv_l = 1.f / (l + *other_x);
    const bool store = r < rows_valid && !failed;
    __nv_bfloat16* orow =
        p.out + (static_cast<int64_t>(q0 + qt * BM + r) * p.num_q_heads + h) * HD + half * HC;
#pragma unroll
    for (int c = 0; c < HC / 32; ++c) {
      float o[32];
      tmem_ld32(tO + half * HC + lane_off + c * 32, o);
      tc_wait_ld();
      if (store) {
#pragma unroll
        for (int v4 = 0; v4 < 4; ++v4) {
          uint4 w;
          w.x = pack_bf16x2(o[v4 * 8 + 0] * inv_l, o[v4 * 8 + 1] * inv_l);
          w.y = pack_bf16x2(o[v4 * 8 + 2] * inv_l, o[v4 * 8 + 3] * inv_l);
          w.z = pack_bf16x2(o[v4 * 8 + 4] * inv_l, o[v4 * 8 + 5] * inv_l);
          w.w = pack_bf16x2(o[v4 * 8 + 6] * inv_l, o[v4 * 8 + 7] * inv_l);
          *reinterpret_cast<uint4*>(orow + c * 32 + v4 * 8) = w;
        }
      }
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == kIssuerWarp) {
    tc_fence_after();
    tmem_dealloc(tmem, kTmemCols);
  }
}

}  // namespace

cudaError_t launch_prefill(const PrefillLaunch& a, cudaStream_t stream) {
  if (a.cache.head_dim != HD) return cudaErrorInvalidValue;
  const int bs = a.cache.block_size;
  const int rows = bs < BN ? bs : BN;
  const uint64_t slots = static_cast<uint64_t>(a.cache.num_blocks) * bs;
  CUtensorMap tmQ, tmK, tmV;
  if (!encode_tensor_map_3d(&tmQ, a.q, HD, a.num_q_heads, a.total_q > 0 ? a.total_q : 1, 64, 1,
                            BM, true) ||
      !encode_tensor_map_3d(&tmK, a.k_cache, HD, a.cache.num_kv_heads, slots, 64, 1, rows, true) ||
      !encode_tensor_map_3d(&tmV, a.v_cache, HD, a.cache.num_kv_heads, slots, 64, 1, rows, true))
    return cudaErrorInvalidValue;
  PrefillParams p;
  p.out = static_cast<__nv_bfloat16*>(a.out);
  p.block_tables = a.block_tables;
  p.cu_seqlens_q = a.cu_seqlens_q;
  p.context_lens = a.context_lens;
  p.err = device_error_word();
  p.max_blocks = a.max_blocks_per_seq;
  p.num_blocks = a.cache.num_blocks;
  p.bs_log2 = 31 - __builtin_clz(static_cast<unsigned>(bs));
  p.num_q_heads = a.num_q_heads;
  p.group = a.num_q_heads / a.cache.num_kv_heads;
  p.total_q = a.total_q;
  p.max_q_len = a.max_q_len;
  p.scale_log2 = a.scale * kLog2e;
  const bool pos = a.scale > 0.f;
  const void* fn = pos ? reinterpret_cast<const void*>(prefill_kernel<true>)
                       : reinterpret_cast<const void*>(prefill_kernel<false>);
  cudaError_t e = ensure_max_dynamic_smem(fn, kSmemBytes);
  if (e != cudaSuccess) return e;
  dim3 grid((a.max_q_len + BM - 1) / BM, a.num_q_heads, a.num_seqs);
  if (grid.x == 0 || a.num_seqs == 0) return cudaSuccess;
  if (pos)
    prefill_kernel<true><<<grid, kThreads, kSmemBytes, stream>>>(tmQ, tmK, tmV, p);
  else
    prefill_kernel<false><<<grid, kThreads, kSmemBytes, stream>>>(tmQ, tmK, tmV, p);
  return cudaGetLastError();
}

}  // namespace pa

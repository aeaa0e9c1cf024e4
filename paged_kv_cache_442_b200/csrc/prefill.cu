// Causal paged prefill on the tcgen05 tensor cores: a chunk of new tokens of each
// sequence attends to the sequence's cached prefix plus itself (nano vllm page,
// section 3.1: num_cached_tokens of a Sequence are reused; mini-vllm page,
// section 1: blocks are allocated for the prefill; all K/V are read through the
// block table, section 2).
//
// One CTA = two units of 128 query rows that read the same K/V: two query heads of
// one kv head over the same 128 new tokens (when the group has an even number of
// heads), else two consecutive 128-token tiles of one head. Per KV tile of 128
// positions and unit u:
//   S_u = Q_u K^T   (tcgen05.mma, M=128 N=128 K=128, fp32 in TMEM)
//   softmax of S_u, P_u written back to TMEM as bf16 over S_u's own columns
//   O_u += P_u V    (tcgen05.mma with A = P_u read from TMEM, B = V from shared
//                    memory, accumulator in TMEM)
// The tensor core alternates between the units: while the softmax of one unit runs,
// it executes the other unit's value and score products, so its queue is fed from two
// independent chains. Issue order per tile: PV_0(j), S_0(j+1), PV_1(j), S_1(j+1);
// S_u(j+1) overwrites P_u(j) only after PV_u(j) has read it (the tensor core runs its
// queue in order), and S_u(j+1) being done implies PV_u(j) is done, so the softmax of
// tile j+1 may rescale O_u right away.
// Roles (320 threads; 352 when the call also stores the new rows):
//   warps 0-3   softmax of unit 0, warps 4-7 softmax of unit 1: thread r owns query
//               row r (TMEM lane r) and the whole 128-column row of S, so the row max
//               needs no exchange between threads; O is rescaled only when a row's
//               running max grows by more than 2^8 (probabilities stay <= 256);
//   warp 8      TMA producer: both Q tiles once, then K and V tiles gathered block by
//               block through the block table into two rings;
//   warp 9      owns the TMEM allocation (all 512 columns: S_0/P_0, S_1/P_1, O_0, O_1)
//               and issues the MMAs from one thread;
//   warp 10     (store + prefill only) copies new K/V rows into the pool.
// Store + prefill (pa_store_prefill): the new tokens' K/V rows are read from the
// caller's k / v tensors (the bits the store writes), never from the pool, so no CTA
// depends on another CTA's store. The tile holding the first new position, when that
// position is not tile-aligned, is loaded from the pool and its new rows overwritten
// from k / v by the producer before the tensor core reads it. The CTA of each
// (sequence, query tile, kv head) that holds the group's first query head writes that
// tile's new rows to their slots.
// Shared-memory operands use the 128-byte swizzled K-major layout (Q, K) and the
// MN-major layout (V, whose head dim is contiguous), both produced directly by TMA.
#include <cuda_bf16.h>

#include "pa_internal.h"
#include "pa_ptx.cuh"

namespace pa {
namespace {

constexpr int BM = 128;          // query rows per unit
constexpr int BN = 128;          // KV positions per tile
constexpr int HD = 128;          // head dim
constexpr int kProducerWarp = 8;
constexpr int kIssuerWarp = 9;
constexpr int kStoreWarp = 10;
constexpr int NK = 2;            // K ring depth (a slot frees when both units' score MMAs are done)
constexpr int NV = 2;            // V ring depth (a slot frees when both units' value MMAs are done)
constexpr int kRegion = BM * 128;  // one 64-column half of a 128x128 bf16 tile (16 KB)
constexpr int kTileBytes = 2 * kRegion;
// Small objects first (8-byte aligned at the start of dynamic shared memory), then
// the 1024-byte-aligned operand tiles.
constexpr int kNumBars = 3 + 2 * NK + 2 * NV + 3 * 2;  // q, drain, patch, K/V rings, s/p/pv per unit
constexpr int kOffMisc = 8 * kNumBars;                 // tmem address, abort flag
constexpr int kSmallBytes = kOffMisc + 16;
constexpr int kOffQ = 0;                               // within the aligned region: Q_0, Q_1
constexpr int kOffK = kOffQ + 2 * kTileBytes;
constexpr int kOffV = kOffK + NK * kTileBytes;
constexpr int kDataBytes = kOffV + NV * kTileBytes;
constexpr int kSmemBytes = kSmallBytes + 1023 + kDataBytes;  // worst-case alignment pad
static_assert(kOffK % 1024 == 0 && kOffV % 1024 == 0,
              "128-byte-swizzled TMA / MMA operands need 1024-byte alignment");
static_assert(kOffMisc % 8 == 0, "mbarriers / words alignment");
static_assert(kSmemBytes <= 227 * 1024, "shared memory per CTA");
constexpr float kLog2e = 1.4426950408889634f;
constexpr float kRescaleLog2 = 8.f;   // rescale O only past this growth of the row max
constexpr uint32_t kTmemCols = 512;   // S_0/P_0 0-127, S_1/P_1 128-255, O_0 256-383, O_1 384-511
constexpr uint32_t kTmemO = 256;

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
  int num_kv_heads;
  int group;        // Hq / Hkv
  int head_pairs;   // units are two heads of a group (group even), else two q tiles
  int total_q;
  int max_q_len;
  float scale_log2;
  unsigned long long wait_ns;  // bound of the waits between roles
  // store + prefill: the new rows [total_q, Hkv, D] and their slots, else NULL
  const uint4* new_k;
  const uint4* new_v;
  const int32_t* slot_mapping;
  uint4* k_rows;    // the pools, as rows of Hkv x 16 vectors
  uint4* v_rows;
};

// One unit's place in the batch: its query tile, head, visible range and tile count.
struct Unit {
  int qt, h, rows_valid, pos_max, ntiles;
};

// kPosScale: scale > 0, so the row max can be taken on the raw scores and the scale
// folded into the exponent's FMA; otherwise (scale <= 0) the scores are scaled first.
// kStore: pa_store_prefill (new rows read from k / v and written to the pool).
template <bool kPosScale, bool kStore>
__global__ void __launch_bounds__(kStore ? 352 : 320, 1) prefill_kernel(
    const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
    const __grid_constant__ CUtensorMap tmV, const __grid_constant__ CUtensorMap tmKn,
    const __grid_constant__ CUtensorMap tmVn, const PrefillParams p) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* small = smem_raw;
  uint8_t* smem = reinterpret_cast<uint8_t*>(
      (reinterpret_cast<uintptr_t>(smem_raw + kSmallBytes) + 1023) &
      ~static_cast<uintptr_t>(1023));

  const int tid = threadIdx.x;
  const int warp = tid >> 5;
  const int lane = tid & 31;
  const int s = blockIdx.z;

  const int q0 = __ldg(p.cu_seqlens_q + s);
  const int n_new = __ldg(p.cu_seqlens_q + s + 1) - q0;
  const int ctx = __ldg(p.context_lens + s);
  if (n_new > ctx || q0 < 0 || q0 + n_new > p.total_q || n_new > p.max_q_len) {
    // caller broke a precondition: compute nothing, write nothing
    if (tid == 0 && blockIdx.x == 0 && blockIdx.y == 0) flag_error(p.err, PA_DEV_ERR_BAD_INDEX);
    return;
  }
  const int first = ctx - n_new;  // position of the first new token
  auto make_unit = [&](int u) {
    Unit x;
    x.qt = p.head_pairs ? static_cast<int>(blockIdx.x) : 2 * static_cast<int>(blockIdx.x) + u;
    x.h = p.head_pairs ? 2 * static_cast<int>(blockIdx.y) + u : static_cast<int>(blockIdx.y);
    x.rows_valid = min(BM, n_new - x.qt * BM);
    x.pos_max = first + x.qt * BM + x.rows_valid - 1;
    x.ntiles = x.rows_valid > 0 ? x.pos_max / BN + 1 : 0;
    return x;
  };
  const Unit u0 = make_unit(0), u1 = make_unit(1);
  const int nt0 = u0.ntiles, nt1 = u1.ntiles;
  // unit 0 is active whenever unit 1 is; nothing to do when it is not (CTA-uniform)
  if (nt0 == 0) return;
  const int g = u0.h / p.group;  // both units read kv head g
  const int nmax = max(nt0, nt1);
  const int bs = 1 << p.bs_log2;

  uint64_t* bars = reinterpret_cast<uint64_t*>(small);
  uint64_t* bar_q = bars;
  uint64_t* mma_drain = bars + 1;
  uint64_t* patch = bars + 2;                // store + prefill: the straddling tile's pool rows
  uint64_t* k_full = bars + 3;               // [NK] each
  uint64_t* k_empty = k_full + NK;
  uint64_t* v_full = k_empty + NK;           // [NV] each
  uint64_t* v_empty = v_full + NV;
  uint64_t* s_full = v_empty + NV;           // [2 units] each
  uint64_t* p_full = s_full + 2;
  uint64_t* pv_done = p_full + 2;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(small + kOffMisc);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(small + kOffMisc + 8);

  if (tid == 0) {
    mbar_init(bar_q, 1);
    mbar_init(mma_drain, 1);
    mbar_init(patch, 1);
    for (int i = 0; i < NK; ++i) {
      mbar_init(&k_full[i], 1);
      mbar_init(&k_empty[i], 1);
    }
    for (int i = 0; i < NV; ++i) {
      mbar_init(&v_full[i], 1);
      mbar_init(&v_empty[i], 1);
    }
    for (int u = 0; u < 2; ++u) {
      mbar_init(&s_full[u], 1);
      mbar_init(&p_full[u], 4);   // one arrival per softmax warp of the unit
      mbar_init(&pv_done[u], 1);
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

  if (warp == kProducerWarp) {
    // ------------------------------------------------------------ TMA producer
    // lane 0 waits and issues; the verdict of each wait is broadcast so the warp
    // leaves the loop together
    auto wwait = [&](uint64_t* bar, unsigned parity) -> bool {
      int okw = 0;
      if (lane == 0) okw = wait_or_abort(bar, parity, p.err, abort_flag, p.wait_ns) ? 1 : 0;
      return __shfl_sync(0xffffffffu, okw, 0) != 0;
    };
    const int rows = bs < BN ? bs : BN;
    const int nbox = BN / rows;
    const uint64_t keep = policy_evict_last();  // K/V tiles are re-read by other CTAs
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
    // tile j of K or V into `dst`: boxes of the pool through the block table; for
    // store + prefill, a tile that starts at or after the first new position comes
    // from the new rows (one box of 128 consecutive rows of k / v per head-dim half)
    auto load_tile = [&](const CUtensorMap* map, const CUtensorMap* nmap, uint8_t* dst,
                         uint64_t* bar, int j) {
      mbar_arrive_expect_tx(bar, kTileBytes);
      if (kStore && j * BN >= first) {
        const int row = q0 + (j * BN - first);
        tma_load_3d_hint(dst, nmap, bar, 0, g, row, keep);
        tma_load_3d_hint(dst + kRegion, nmap, bar, 64, g, row, keep);
        return;
      }
#pragma unroll 1
      for (int c = 0; c < nbox; ++c) {
        const int row = block_row(j * BN + c * rows);
        tma_load_3d_hint(dst + c * rows * 128, map, bar, 0, g, row, keep);
        tma_load_3d_hint(dst + kRegion + c * rows * 128, map, bar, 64, g, row, keep);
      }
    };
    // store + prefill, the tile holding the first new position when it starts before
    // it: the pool's rows, then its new rows (from `first` on) from k / v, written into
    // the swizzled tile by the warp, then the consumers' barrier
    const int jst = (kStore && (first % BN) != 0 && first / BN < nmax) ? first / BN : -1;
    int patch_started = 0, patch_done = 0;
    auto load_straddling = [&](const CUtensorMap* map, const uint4* src, uint8_t* dst,
                               uint64_t* bar) -> bool {
      if (lane == 0) {
        mbar_arrive_expect_tx(patch, kTileBytes);
#pragma unroll 1
        for (int c = 0; c < nbox; ++c) {
          const int row = block_row(jst * BN + c * rows);
          tma_load_3d(dst + c * rows * 128, map, patch, 0, g, row);
          tma_load_3d(dst + kRegion + c * rows * 128, map, patch, 64, g, row);
        }
      }
      ++patch_started;
      if (!wwait(patch, (patch_started - 1) & 1)) return false;
      ++patch_done;
      // row r >= r0 of the tile is new row r - r0 of the sequence: 16 vectors each
      const int r0 = first - jst * BN;
      const int nr = min(BN - r0, n_new);
#pragma unroll 1
      for (int i = lane; i < nr * 16; i += 32) {
        const int r = r0 + (i >> 4), c = i & 15;  // 16-byte chunk c holds dims 8c..8c+7
        const uint4 v =
            __ldg(src + (static_cast<int64_t>(q0 + r - r0) * p.num_kv_heads + g) * 16 + c);
        uint8_t* d = dst + (c >> 3) * kRegion + r * 128 + (((c & 7) ^ (r & 7)) << 4);
        *reinterpret_cast<uint4*>(d) = v;
      }
      fence_proxy_async_smem();
      __syncwarp();
      if (lane == 0) mbar_arrive(bar);
      return true;
    };
    if (lane == 0) {
      prefetch_tensormap(&tmQ);
      prefetch_tensormap(&tmK);
      prefetch_tensormap(&tmV);
      mbar_arrive_expect_tx(bar_q, (nt1 > 0 ? 2 : 1) * kTileBytes);
      for (int u = 0; u < 2; ++u) {
        const Unit x = u ? u1 : u0;
        if (x.ntiles == 0) continue;
        const int qrow = q0 + x.qt * BM;
        tma_load_3d(smem + kOffQ + u * kTileBytes, &tmQ, bar_q, 0, x.h, qrow);
        tma_load_3d(smem + kOffQ + u * kTileBytes + kRegion, &tmQ, bar_q, 64, x.h, qrow);
      }
    }
    int k_issued = 0, v_issued = 0;
#pragma unroll 1
    for (int j = 0; j < nmax; ++j) {
      const int ks = j % NK;
      if (j >= NK && !wwait(&k_empty[ks], ((j / NK) - 1) & 1)) break;
      if (j == jst) {
        if (!load_straddling(&tmK, p.new_k, smem + kOffK + ks * kTileBytes, &k_full[ks])) break;
      } else if (lane == 0) {
        load_tile(&tmK, &tmKn, smem + kOffK + ks * kTileBytes, &k_full[ks], j);
      }
      k_issued = j + 1;
      const int vs = j % NV;
      if (j >= NV && !wwait(&v_empty[vs], ((j / NV) - 1) & 1)) break;
      if (j == jst) {
        if (!load_straddling(&tmV, p.new_v, smem + kOffV + vs * kTileBytes, &v_full[vs])) break;
      } else if (lane == 0) {
        load_tile(&tmV, &tmVn, smem + kOffV + vs * kTileBytes, &v_full[vs], j);
      }
      v_issued = j + 1;
    }
    // Before the CTA ends, every copy this warp started must have landed. Per slot
    // only the last load can still be in flight (the one before it was consumed),
    // so waiting for those is enough; on the normal path they completed long ago.
    if (lane == 0) {
      mbar_wait(bar_q, 0, p.err);
#pragma unroll 1
      for (int t = k_issued - NK > 0 ? k_issued - NK : 0; t < k_issued; ++t)
        mbar_wait(&k_full[t % NK], (t / NK) & 1, p.err);
#pragma unroll 1
      for (int t = v_issued - NV > 0 ? v_issued - NV : 0; t < v_issued; ++t)
        mbar_wait(&v_full[t % NV], (t / NV) & 1, p.err);
      // a straddling tile's pool copy whose wait gave up may still be in flight
      if (patch_started > patch_done) mbar_wait(patch, (patch_started - 1) & 1, p.err);
    }
  } else if (warp == kIssuerWarp) {
    // ------------------------------------------------------------ MMA issuer
    // the whole warp runs this loop (its descriptors stay warp-uniform); one elected lane
    // issues each MMA and commit
    {
      constexpr uint32_t idS = idesc_bf16_f32(BM, BN, 0, 0);  // Q K-major, K K-major
      constexpr uint32_t idO = idesc_bf16_f32(BM, HD, 0, 1);  // P (TMEM), V MN-major
      // S_u(j) over S_u's columns once K(j) has landed (S_u(j-1) was read and P_u(j-1)
      // consumed by the value MMA queued before it); K(j) frees after its last reader
      auto score = [&](int u, int j) -> bool {
        const int ks = j % NK;
        if (!warp_wait_or_abort(&k_full[ks], (j / NK) & 1, p.err, abort_flag, p.wait_ns))
          return false;
        tc_fence_after();
        // one descriptor per operand, stepped by constant offsets (see desc_advance)
        const uint64_t aQ = smem_desc_sw128(smem_u32(smem + kOffQ + u * kTileBytes), 16, 1024);
        const uint64_t bK = smem_desc_sw128(smem_u32(smem + kOffK + ks * kTileBytes), 16, 1024);
#pragma unroll
        for (int kk = 0; kk < HD / 16; ++kk) {
          const uint32_t off = (kk >> 2) * kRegion + (kk & 3) * 32;
          tc_mma_f16_ss(tmem + u * 128, desc_advance(aQ, off), desc_advance(bK, off), idS,
                        kk > 0 ? 1u : 0u);
        }
        tc_commit(&s_full[u]);
        if (u == 1 || j >= nt1) tc_commit(&k_empty[ks]);
        return true;
      };
      // O_u += P_u(t) V(t), once the softmax has written P_u(t) and V(t) has landed
      auto pv = [&](int u, int t) -> bool {
        const int vs = t % NV;
        if (!warp_wait_or_abort(&p_full[u], t & 1, p.err, abort_flag, p.wait_ns) ||
            !warp_wait_or_abort(&v_full[vs], (t / NV) & 1, p.err, abort_flag, p.wait_ns))
          return false;
        tc_fence_after();
        const uint32_t tP = tmem + u * 128;
        const uint64_t bV = smem_desc_sw128(smem_u32(smem + kOffV + vs * kTileBytes), kRegion, 1024);
#pragma unroll
        for (int kk = 0; kk < BN / 16; ++kk)  // 16 kv positions per step = 8 packed columns of P
          tc_mma_f16_ts(tmem + kTmemO + u * 128, tP + kk * 8, desc_advance(bV, kk * 16 * 128), idO,
                        (t > 0 || kk > 0) ? 1u : 0u);
        tc_commit(&pv_done[u]);
        if (u == 1 || t >= nt1) tc_commit(&v_empty[vs]);
        return true;
      };
      bool ok = warp_wait_or_abort(bar_q, 0, p.err, abort_flag, p.wait_ns);
      if (ok) ok = score(0, 0);
      if (ok && nt1 > 0) ok = score(1, 0);
      for (int j = 0; ok && j < nmax; ++j) {
        if (j < nt0) {
          ok = pv(0, j);
          if (ok && j + 1 < nt0) ok = score(0, j + 1);
        }
        if (ok && j < nt1) {
          ok = pv(1, j);
          if (ok && j + 1 < nt1) ok = score(1, j + 1);
        }
      }
      // every MMA this thread issued has finished before TMEM and shared memory go away
      tc_commit(mma_drain);
      mbar_wait(mma_drain, 0, p.err);
    }
  } else if (warp < 8) {
    // ------------------------------------------------------------ softmax warps
    // Every lane runs every step (the tcgen05 loads and stores are warp-collective): a
    // failed wait only marks `failed`.
    const int u = warp >> 2;
    const Unit me = make_unit(u);
    const int quad = warp & 3;
    const int r = quad * 32 + lane;           // query row within the tile == TMEM lane
    const uint32_t lane_off = static_cast<uint32_t>(quad * 32) << 16;
    const uint32_t tS = tmem + u * 128 + lane_off;
    const uint32_t tO = tmem + kTmemO + u * 128 + lane_off;
    const int pos_r = first + me.qt * BM + (r < me.rows_valid ? r : me.rows_valid - 1);
    float m = -INFINITY;
    float l = 0.f;
    bool failed = false;
    for (int j = 0; j < me.ntiles; ++j) {
      failed |= !wait_or_abort(&s_full[u], j & 1, p.err, abort_flag, p.wait_ns);
      tc_fence_after();
      float sv[BN];
#pragma unroll
      for (int c = 0; c < BN / 32; ++c) {
        float t32[32];
        tmem_ld32(tS + c * 32, t32);
#pragma unroll
        for (int i = 0; i < 32; ++i) sv[c * 32 + i] = t32[i];
      }
      tc_wait_ld();
      const int lim = pos_r - j * BN;  // columns past lim are in this row's future: masked
      float mx;
      if constexpr (kPosScale) {
        if (lim < BN - 1) {
#pragma unroll
          for (int c = 0; c < BN; ++c) sv[c] = c > lim ? -INFINITY : sv[c];
        }
        // max of the raw scores (the scale is positive), four independent chains
        float a0 = -INFINITY, a1 = -INFINITY, a2 = -INFINITY, a3 = -INFINITY;
#pragma unroll
        for (int c = 0; c < BN; c += 8) {
          a0 = fmax3(a0, sv[c + 0], sv[c + 1]);
          a1 = fmax3(a1, sv[c + 2], sv[c + 3]);
          a2 = fmax3(a2, sv[c + 4], sv[c + 5]);
          a3 = fmax3(a3, sv[c + 6], sv[c + 7]);
        }
        mx = fmax3(a0, a1, fmaxf(a2, a3)) * p.scale_log2;
      } else {
#pragma unroll
        for (int c = 0; c < BN; ++c) sv[c] = c > lim ? -INFINITY : sv[c] * p.scale_log2;
        mx = -INFINITY;
#pragma unroll
        for (int c = 0; c < BN; ++c) mx = fmaxf(mx, sv[c]);
      }
      // reference max: the first tile's (position 0 is visible to every row), raised
      // only when a later tile exceeds it by more than 2^8
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
      float2 acc[2] = {make_float2(0.f, 0.f), make_float2(0.f, 0.f)};
      // 16 columns at a time: their P (8 packed columns) goes straight to TMEM, over S
      // columns already read (P column c' holds S columns 2c' and 2c'+1)
#pragma unroll
      for (int cb = 0; cb < BN; cb += 16) {
        uint32_t pk[8];
#pragma unroll
        for (int c = cb; c < cb + 16; c += 2) {
          const float2 x = __ffma2_rn(make_float2(sv[c], sv[c + 1]), sc2, nm2);
          const float2 e = make_float2(ex2_approx(x.x), ex2_approx(x.y));
          acc[(c >> 1) & 1] = __fadd2_rn(acc[(c >> 1) & 1], e);
          pk[(c - cb) >> 1] = pack_bf16x2(e.x, e.y);
        }
        tmem_st8_bits(tS + (cb >> 1), pk);
      }
      const float rs = (acc[0].x + acc[0].y) + (acc[1].x + acc[1].y);
      l = l * alpha + rs;
      if (__any_sync(0xffffffffu, rescale)) {
        // O_u holds the value MMAs up to tile j-1, all done (S_u(j), queued after them,
        // is): rescale this warp's rows (rows that do not need it multiply by 1)
#pragma unroll
        for (int c = 0; c < HD / 32; ++c) {
          float o[32];
          tmem_ld32(tO + c * 32, o);
          tc_wait_ld();
#pragma unroll
          for (int i = 0; i < 32; ++i) o[i] *= alpha;
          tmem_st32(tO + c * 32, o);
        }
      }
      if (j == me.ntiles - 1 && ctx - j * BN < BN) {
        // rows past the context in the last V tile may hold anything (even NaN);
        // P is 0 there but 0 * NaN is NaN, so clear them before the value MMA. Every
        // unit that reads this tile has it as its last one and clears the rows itself
        // before it signals (the other unit's clearing writes zeros over zeros).
        const int vs = j % NV;
        failed |= !wait_or_abort(&v_full[vs], (j / NV) & 1, p.err, abort_flag, p.wait_ns);
        if (r >= ctx - j * BN) {
          uint8_t* v = smem + kOffV + vs * kTileBytes + r * 128;
          const uint4 z = make_uint4(0, 0, 0, 0);
#pragma unroll
          for (int c = 0; c < 8; ++c) {
            *reinterpret_cast<uint4*>(v + c * 16) = z;
            *reinterpret_cast<uint4*>(v + kRegion + c * 16) = z;
          }
        }
        fence_proxy_async_smem();
      }
      // P_u is over S_u's first 64 columns (the A-operand layout: row in the lane,
      // consecutive kv positions in consecutive half-words)
      tc_wait_st();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&p_full[u]);
    }
    if (me.ntiles > 0) {
      const int t = me.ntiles - 1;
      failed |= !wait_or_abort(&pv_done[u], t & 1, p.err, abort_flag, p.wait_ns);
      tc_fence_after();
      const float inv_l = 1.f / l;
      const bool store = r < me.rows_valid && !failed;
      __nv_bfloat16* orow =
          p.out + (static_cast<int64_t>(q0 + me.qt * BM + r) * p.num_q_heads + me.h) * HD;
#pragma unroll
      for (int c = 0; c < HD / 32; ++c) {
        float o[32];
        tmem_ld32(tO + c * 32, o);
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
  } else if (kStore && warp == kStoreWarp) {
    // ------------------------------------------------------------ new-row store
    // The CTA holding the group's first query head stores, for kv head g, the new rows
    // of its query tile(s) to their slots. slot_mapping[t] must be the slot the block
    // table gives for token t's position (or -1: not stored); any other slot is
    // reported and not written. The attention itself used the rows of k / v.
    if (u0.h % p.group == 0) {
      for (int u = 0; u < 2; ++u) {
        const Unit x = u ? u1 : u0;
        if (x.ntiles == 0 || (p.head_pairs && u == 1)) continue;
        for (int i = lane; i < x.rows_valid * 2; i += 32) {
          const int rr = i >> 1;
          const int t = q0 + x.qt * BM + rr;   // token row of k / v
          const int pos = first + x.qt * BM + rr;
          const int slot = __ldg(p.slot_mapping + t);
          if (slot < 0) continue;
          const int bi = pos >> p.bs_log2;
          const int id = bi < p.max_blocks
                             ? __ldg(p.block_tables + static_cast<int64_t>(s) * p.max_blocks + bi)
                             : -1;
          if (id < 0 || id >= p.num_blocks ||
              static_cast<int64_t>(slot) != static_cast<int64_t>(id) * bs + (pos & (bs - 1))) {
            flag_error(p.err, PA_DEV_ERR_BAD_INDEX);
            continue;
          }
          const uint4* src = (i & 1) ? p.new_v : p.new_k;
          uint4* dst = (i & 1) ? p.v_rows : p.k_rows;
          const int64_t so = (static_cast<int64_t>(t) * p.num_kv_heads + g) * 16;
          const int64_t d = (static_cast<int64_t>(slot) * p.num_kv_heads + g) * 16;
#pragma unroll
          for (int c = 0; c < 16; ++c) dst[d + c] = __ldg(src + so + c);
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

template <bool kPosScale, bool kStore>
cudaError_t launch_t(const CUtensorMap* maps, const PrefillParams& p, dim3 grid,
                     cudaStream_t stream) {
  const void* fn = reinterpret_cast<const void*>(prefill_kernel<kPosScale, kStore>);
  cudaError_t e = ensure_max_dynamic_smem(fn, kSmemBytes);
  if (e != cudaSuccess) return e;
  prefill_kernel<kPosScale, kStore><<<grid, kStore ? 352 : 320, kSmemBytes, stream>>>(
      maps[0], maps[1], maps[2], maps[3], maps[4], p);
  return cudaGetLastError();
}

}  // namespace

cudaError_t launch_prefill(const PrefillLaunch& a, cudaStream_t stream) {
  if (a.cache.head_dim != HD) return cudaErrorInvalidValue;
  const int bs = a.cache.block_size;
  const int rows = bs < BN ? bs : BN;
  const uint64_t slots = static_cast<uint64_t>(a.cache.num_blocks) * bs;
  const bool store = a.new_k != nullptr;
  CUtensorMap maps[5];  // Q, K pool, V pool, new K rows, new V rows
  const uint64_t tq = a.total_q > 0 ? a.total_q : 1;
  if (!encode_tensor_map_3d(&maps[0], a.q, HD, a.num_q_heads, tq, 64, 1, BM, true) ||
      !encode_tensor_map_3d(&maps[1], a.k_cache, HD, a.cache.num_kv_heads, slots, 64, 1, rows, true) ||
      !encode_tensor_map_3d(&maps[2], a.v_cache, HD, a.cache.num_kv_heads, slots, 64, 1, rows, true))
    return cudaErrorInvalidValue;
  if (store) {
    // the new rows [total_q, Hkv, D]: one box of 128 consecutive rows per tile half
    if (!encode_tensor_map_3d(&maps[3], a.new_k, HD, a.cache.num_kv_heads, tq, 64, 1, BN, true) ||
        !encode_tensor_map_3d(&maps[4], a.new_v, HD, a.cache.num_kv_heads, tq, 64, 1, BN, true))
      return cudaErrorInvalidValue;
  } else {
    maps[3] = maps[1];  // unused
    maps[4] = maps[2];
  }
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
  p.num_kv_heads = a.cache.num_kv_heads;
  p.group = a.num_q_heads / a.cache.num_kv_heads;
  p.head_pairs = (p.group % 2) == 0 ? 1 : 0;
  p.total_q = a.total_q;
  p.max_q_len = a.max_q_len;
  p.scale_log2 = a.scale * kLog2e;
  p.wait_ns = wait_limit_ns();
  p.new_k = static_cast<const uint4*>(a.new_k);
  p.new_v = static_cast<const uint4*>(a.new_v);
  p.slot_mapping = a.slot_mapping;
  p.k_rows = static_cast<uint4*>(const_cast<void*>(a.k_cache));
  p.v_rows = static_cast<uint4*>(const_cast<void*>(a.v_cache));
  const int qtiles = (a.max_q_len + BM - 1) / BM;
  dim3 grid(p.head_pairs ? qtiles : (qtiles + 1) / 2,
            p.head_pairs ? a.num_q_heads / 2 : a.num_q_heads, a.num_seqs);
  if (grid.x == 0 || a.num_seqs == 0) return cudaSuccess;
  const bool pos = a.scale > 0.f;
  if (pos) return store ? launch_t<true, true>(maps, p, grid, stream)
                        : launch_t<true, false>(maps, p, grid, stream);
  return store ? launch_t<false, true>(maps, p, grid, stream)
               : launch_t<false, false>(maps, p, grid, stream);
}

}  // namespace pa

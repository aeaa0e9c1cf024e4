// Decode over a prefix that every sequence of the batch shares, attended once for all
// of its sharers (nano vllm page, section 3.2.2: requests whose prompts start alike
// share reference-counted blocks, e.g. a common system prompt; the page reports
// 40-60% less memory from it).
//
// When the first shared_len positions of every sequence map to the same physical
// blocks, the decode of those positions is one dense product per kv head: the query
// rows of all sequences (G heads each) against the same keys and values. This kernel
// computes it on the tensor cores, 128 query rows (128 / G sequences x G heads) per
// CTA, 128 shared positions per tile:
//   S = Q K^T (tcgen05.mma, fp32 in TMEM), softmax in registers (thread r owns query
//   row r), P written back over S as bf16, O += P V (A = P from TMEM).
// Row (s, h) sees positions 0 .. min(context_lens[s], shared_len) - 1. Its result is
// the output row when the whole context lies in the shared prefix, else the partial
// (m, l, o) of partition 0 of the split-K decode (the same record and reference as the
// decode kernel's partitions), which the persistent decode over the remaining
// positions merges in.
// Each CTA takes two such tiles of 128 query rows (units 0 and 1, consecutive rows of
// one kv head) that read the same shared tiles (one tile when two per CTA would leave
// SMs idle), and the tensor core alternates between them: issue order PV_0(j), S_0(j+1), PV_1(j), S_1(j+1), so one unit's softmax runs
// while the other unit's products execute (P_u is written over S_u in TMEM, and
// S_u(j+1) done implies PV_u(j) done).
// Roles (320 threads): warps 0-3 / 4-7 softmax + output of unit 0 / 1, warp 8 TMA
// producer (both Q tiles, then K and V of the shared blocks in two-deep rings),
// warp 9 TMEM owner (all 512 columns: S_0/P_0, S_1/P_1, O_0, O_1) and MMA issuer. The
// softmax warps first check every sequence of the CTA's rows against the shared blocks
// (while the first tiles load).
#include <cuda_bf16.h>

#include "pa_internal.h"
#include "pa_ptx.cuh"

namespace pa {
namespace {

constexpr int BM = 128;          // query rows per CTA
constexpr int BN = 128;          // shared positions per tile
constexpr int HD = 128;
constexpr int kThreads = 320;
constexpr int kProducerWarp = 8;
constexpr int kIssuerWarp = 9;
constexpr int NK = 2;
constexpr int NV = 2;
constexpr int kRegion = BM * 128;
constexpr int kTileBytes = 2 * kRegion;
constexpr int kNumBars = 2 + 2 * NK + 2 * NV + 3 * 2;  // q, drain, K/V rings, s/p/pv per unit
constexpr int kOffMisc = 8 * kNumBars;
constexpr int kSmallBytes = kOffMisc + 16;
constexpr int kOffQ = 0;                         // Q_0, Q_1
constexpr int kOffK = kOffQ + 2 * kTileBytes;
constexpr int kOffV = kOffK + NK * kTileBytes;
constexpr int kDataBytes = kOffV + NV * kTileBytes;
constexpr int kSmemBytes = kSmallBytes + 1023 + kDataBytes;
static_assert(kSmemBytes <= 227 * 1024, "shared memory per CTA");
static_assert(kOffK % 1024 == 0 && kOffV % 1024 == 0, "swizzled operands need 1024-byte alignment");
constexpr float kLog2e = 1.4426950408889634f;
constexpr float kRescaleLog2 = 8.f;
constexpr uint32_t kTmemCols = 512;  // S_0/P_0 0-127, S_1/P_1 128-255, O_0 256-383, O_1 384-511
constexpr uint32_t kTmemO = 256;

struct PrefixParams {
  __nv_bfloat16* out;          // [B, Hq, D]
  const int32_t* block_tables;
  const int32_t* shared_blocks;  // [shared_len / block_size]: the prefix's physical blocks
  const int32_t* context_lens;
  float* ws_o;                 // [B, Hq, max_parts, D]: partition 0 written here
  float* ws_ml;                // [B, Hq, max_parts, 2]
  unsigned* err;
  int num_seqs;
  int num_q_heads;
  int group;
  int max_blocks;
  int num_blocks;
  int bs_log2;
  int shared_len;              // multiple of 128
  int units;                   // 128-row units per CTA: 2, or 1 when two would leave SMs idle
  int max_parts;
  int max_context_len;
  float scale_log2;
  unsigned long long wait_ns;
};

__global__ void __launch_bounds__(kThreads, 1) shared_prefix_kernel(
    const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
    const __grid_constant__ CUtensorMap tmV, const PrefixParams p) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* small = smem_raw;
  uint8_t* smem = reinterpret_cast<uint8_t*>(
      (reinterpret_cast<uintptr_t>(smem_raw + kSmallBytes) + 1023) &
      ~static_cast<uintptr_t>(1023));
  const int tid = threadIdx.x;
  const int warp = tid >> 5;
  const int lane = tid & 31;
  const int G = p.group;
  const int spt = BM / G;                        // sequences per unit
  const int s0 = blockIdx.x * p.units * spt;     // first sequence of the CTA (unit 0)
  const bool two = p.units == 2 && s0 + spt < p.num_seqs;  // unit 1 has rows of real sequences
  const int g = blockIdx.y;
  const int ntiles = p.shared_len / BN;
  const int bs = 1 << p.bs_log2;

  uint64_t* bars = reinterpret_cast<uint64_t*>(small);
  uint64_t* bar_q = bars;
  uint64_t* mma_drain = bars + 1;
  uint64_t* k_full = bars + 2;
  uint64_t* k_empty = k_full + NK;
  uint64_t* v_full = k_empty + NK;
  uint64_t* v_empty = v_full + NV;
  uint64_t* s_full = v_empty + NV;   // [2 units] each
  uint64_t* p_full = s_full + 2;
  uint64_t* pv_done = p_full + 2;
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
    for (int u = 0; u < 2; ++u) {
      mbar_init(&s_full[u], 1);
      mbar_init(&p_full[u], 4);
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
    auto wwait = [&](uint64_t* bar, unsigned parity) -> bool {
      int okw = 0;
      if (lane == 0) okw = wait_or_abort(bar, parity, p.err, abort_flag, p.wait_ns) ? 1 : 0;
      return __shfl_sync(0xffffffffu, okw, 0) != 0;
    };
    const int rows = bs < BN ? bs : BN;
    const int nbox = BN / rows;
    const uint64_t keep = policy_evict_last();  // the prefix is read by every CTA of g
    auto load_tile = [&](const CUtensorMap* map, uint8_t* dst, uint64_t* bar, int j) {
      mbar_arrive_expect_tx(bar, kTileBytes);
#pragma unroll 1
      for (int c = 0; c < nbox; ++c) {
        const int pos = j * BN + c * rows;
        int id = __ldg(p.shared_blocks + (pos >> p.bs_log2));
        if (id < 0 || id >= p.num_blocks) {
          flag_error(p.err, PA_DEV_ERR_BAD_INDEX);
          id = 0;
        }
        const int row = id * bs + (pos & (bs - 1));
        tma_load_3d_hint(dst + c * rows * 128, map, bar, 0, g, row, keep);
        tma_load_3d_hint(dst + kRegion + c * rows * 128, map, bar, 64, g, row, keep);
      }
    };
    if (lane == 0) {
      prefetch_tensormap(&tmQ);
      prefetch_tensormap(&tmK);
      prefetch_tensormap(&tmV);
      // Q: G heads x 128/G sequences per box, rows in (sequence, head) order
      mbar_arrive_expect_tx(bar_q, (two ? 2 : 1) * kTileBytes);
      for (int u = 0; u < (two ? 2 : 1); ++u) {
        tma_load_3d(smem + kOffQ + u * kTileBytes, &tmQ, bar_q, 0, g * G, s0 + u * spt);
        tma_load_3d(smem + kOffQ + u * kTileBytes + kRegion, &tmQ, bar_q, 64, g * G, s0 + u * spt);
      }
    }
    int k_issued = 0, v_issued = 0;
#pragma unroll 1
    for (int j = 0; j < ntiles; ++j) {
      const int ks = j % NK;
      if (j >= NK && !wwait(&k_empty[ks], ((j / NK) - 1) & 1)) break;
      if (lane == 0) load_tile(&tmK, smem + kOffK + ks * kTileBytes, &k_full[ks], j);
      k_issued = j + 1;
      const int vs = j % NV;
      if (j >= NV && !wwait(&v_empty[vs], ((j / NV) - 1) & 1)) break;
      if (lane == 0) load_tile(&tmV, smem + kOffV + vs * kTileBytes, &v_full[vs], j);
      v_issued = j + 1;
    }
    if (lane == 0) {
      mbar_wait(bar_q, 0, p.err);
#pragma unroll 1
      for (int t = k_issued - NK > 0 ? k_issued - NK : 0; t < k_issued; ++t)
        mbar_wait(&k_full[t % NK], (t / NK) & 1, p.err);
#pragma unroll 1
      for (int t = v_issued - NV > 0 ? v_issued - NV : 0; t < v_issued; ++t)
        mbar_wait(&v_full[t % NV], (t / NV) & 1, p.err);
    }
  } else if (warp == kIssuerWarp) {
    // ------------------------------------------------------------ MMA issuer
    // the whole warp runs this loop (its descriptors stay warp-uniform); one elected lane
    // issues each MMA and commit
    {
      constexpr uint32_t idS = idesc_bf16_f32(BM, BN, 0, 0);
      constexpr uint32_t idO = idesc_bf16_f32(BM, HD, 0, 1);
      const int nu = two ? 2 : 1;
      auto score = [&](int u, int j) -> bool {
        const int ks = j % NK;
        if (!warp_wait_or_abort(&k_full[ks], (j / NK) & 1, p.err, abort_flag, p.wait_ns)) return false;
        tc_fence_after();
        const uint64_t aQ = smem_desc_sw128(smem_u32(smem + kOffQ + u * kTileBytes), 16, 1024);
        const uint64_t bK = smem_desc_sw128(smem_u32(smem + kOffK + ks * kTileBytes), 16, 1024);
#pragma unroll
        for (int kk = 0; kk < HD / 16; ++kk) {
          const uint32_t off = (kk >> 2) * kRegion + (kk & 3) * 32;
          tc_mma_f16_ss(tmem + u * 128, desc_advance(aQ, off), desc_advance(bK, off), idS,
                        kk > 0 ? 1u : 0u);
        }
        tc_commit(&s_full[u]);
        if (u == nu - 1) tc_commit(&k_empty[ks]);  // K(j) frees after its last reader
        return true;
      };
      auto pv = [&](int u, int t) -> bool {
        const int vs = t % NV;
        if (!warp_wait_or_abort(&p_full[u], t & 1, p.err, abort_flag, p.wait_ns) ||
            !warp_wait_or_abort(&v_full[vs], (t / NV) & 1, p.err, abort_flag, p.wait_ns))
          return false;
        tc_fence_after();
        const uint64_t bV = smem_desc_sw128(smem_u32(smem + kOffV + vs * kTileBytes), kRegion, 1024);
#pragma unroll
        for (int kk = 0; kk < BN / 16; ++kk)
          tc_mma_f16_ts(tmem + kTmemO + u * 128, tmem + u * 128 + kk * 8,
                        desc_advance(bV, kk * 16 * 128), idO, (t > 0 || kk > 0) ? 1u : 0u);
        tc_commit(&pv_done[u]);
        if (u == nu - 1) tc_commit(&v_empty[vs]);
        return true;
      };
      bool ok = warp_wait_or_abort(bar_q, 0, p.err, abort_flag, p.wait_ns);
#pragma unroll 1
      for (int u = 0; ok && u < nu; ++u) ok = score(u, 0);
#pragma unroll 1
      for (int j = 0; ok && j < ntiles; ++j) {
        for (int u = 0; ok && u < nu; ++u) {
          ok = pv(u, j);
          if (ok && j + 1 < ntiles) ok = score(u, j + 1);
        }
      }
      tc_commit(mma_drain);
      mbar_wait(mma_drain, 0, p.err);
    }
  } else if (warp < 8) {
    // ------------------------------------------------------------ softmax + output
    // First, while the first tiles load: every sequence of the CTA must hold the shared
    // blocks at the prefix positions it uses (the caller's statement of what is
    // shared); a difference is reported. (256 threads: these dependent global reads
    // would hold up the producer's first loads by tens of microseconds.)
    {
      const int nsb = p.shared_len >> p.bs_log2;
#pragma unroll 1
      for (int i = tid; i < p.units * spt * nsb; i += 8 * 32) {
        const int s = s0 + i / nsb, b = i % nsb;
        if (s >= p.num_seqs || (b << p.bs_log2) >= __ldg(p.context_lens + s)) continue;
        const int id = __ldg(p.block_tables + static_cast<int64_t>(s) * p.max_blocks + b);
        if (id != __ldg(p.shared_blocks + b)) flag_error(p.err, PA_DEV_ERR_BAD_INDEX);
      }
    }
    const int u = warp >> 2;
    if (u == 0 || two) {
    const int r = tid & 127;                            // query row == TMEM lane
    const uint32_t lane_off = static_cast<uint32_t>((warp & 3) * 32) << 16;
    const uint32_t tS = tmem + u * 128 + lane_off;
    const uint32_t tO = tmem + kTmemO + u * 128 + lane_off;
    const int s = s0 + u * spt + r / G;
    const int h = g * G + r % G;
    int ctx = s < p.num_seqs ? __ldg(p.context_lens + s) : 0;
    if (ctx > p.max_context_len) {
      flag_error(p.err, PA_DEV_ERR_BAD_INDEX);
      ctx = p.max_context_len;
    }
    const int vis = ctx < p.shared_len ? (ctx > 0 ? ctx : 0) : p.shared_len;
    float m = -INFINITY, l = 0.f;
    bool failed = false;
#pragma unroll 1
    for (int j = 0; j < ntiles; ++j) {
      failed |= !wait_or_abort(&s_full[u], j & 1, p.err, abort_flag, p.wait_ns);
      tc_fence_after();
      float sv[BN];
#pragma unroll
      for (int c = 0; c < BN / 32; ++c) {
        float t32[32];
        tmem_ld32(tS + c * 32, t32);
#pragma unroll
        for (int i = 0; i < 32; ++i) sv[c * 32 + i] = t32[i] * p.scale_log2;
      }
      tc_wait_ld();
      const int lim = vis - 1 - j * BN;  // columns past lim are not this row's positions
      if (lim < BN - 1) {
#pragma unroll
        for (int c = 0; c < BN; ++c) sv[c] = c > lim ? -INFINITY : sv[c];
      }
      float mx = -INFINITY;
#pragma unroll
      for (int c = 0; c < BN; c += 2) mx = fmax3(mx, sv[c], sv[c + 1]);
      float alpha = 1.f;
      bool rescale = false;
      if (m == -INFINITY) {
        m = mx;                 // first tile with a visible position (or none yet)
      } else if (mx > m + kRescaleLog2) {
        alpha = ex2_approx(m - mx);
        m = mx;
        rescale = true;
      }
      const float mref = m == -INFINITY ? 0.f : m;   // no visible position yet: p = 0
      float2 acc = make_float2(0.f, 0.f);
#pragma unroll
      for (int cb = 0; cb < BN; cb += 16) {
        uint32_t pk[8];
#pragma unroll
        for (int c = cb; c < cb + 16; c += 2) {
          const float2 e = make_float2(ex2_approx(sv[c] - mref), ex2_approx(sv[c + 1] - mref));
          acc = __fadd2_rn(acc, e);
          pk[(c - cb) >> 1] = pack_bf16x2(e.x, e.y);
        }
        tmem_st8_bits(tS + (cb >> 1), pk);
      }
      l = l * alpha + (acc.x + acc.y);
      if (__any_sync(0xffffffffu, rescale)) {
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
      tc_wait_st();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&p_full[u]);
    }
    failed |= !wait_or_abort(&pv_done[u], (ntiles - 1) & 1, p.err, abort_flag, p.wait_ns);
    tc_fence_after();
    const bool mine = s < p.num_seqs && !failed;
    const bool whole = ctx <= p.shared_len;          // the context ends inside the prefix
    const int64_t row = static_cast<int64_t>(s) * p.num_q_heads + h;
    const float inv_l = l > 0.f ? 1.f / l : 0.f;
#pragma unroll
    for (int c = 0; c < HD / 32; ++c) {
      float o[32];
      tmem_ld32(tO + c * 32, o);
      tc_wait_ld();
      if (!mine) continue;
      if (whole) {
        __nv_bfloat16* orow = p.out + row * HD + c * 32;
#pragma unroll
        for (int v4 = 0; v4 < 4; ++v4) {
          uint4 w;
          w.x = pack_bf16x2(o[v4 * 8 + 0] * inv_l, o[v4 * 8 + 1] * inv_l);
          w.y = pack_bf16x2(o[v4 * 8 + 2] * inv_l, o[v4 * 8 + 3] * inv_l);
          w.z = pack_bf16x2(o[v4 * 8 + 4] * inv_l, o[v4 * 8 + 5] * inv_l);
          w.w = pack_bf16x2(o[v4 * 8 + 6] * inv_l, o[v4 * 8 + 7] * inv_l);
          *reinterpret_cast<uint4*>(orow + v4 * 8) = w;
        }
      } else {
        float4* dst = reinterpret_cast<float4*>(p.ws_o + (row * p.max_parts) * HD + c * 32);
#pragma unroll
        for (int v4 = 0; v4 < 8; ++v4)
          dst[v4] = make_float4(o[v4 * 4], o[v4 * 4 + 1], o[v4 * 4 + 2], o[v4 * 4 + 3]);
      }
    }
    if (mine && !whole) {
      p.ws_ml[row * p.max_parts * 2 + 0] = m;
      p.ws_ml[row * p.max_parts * 2 + 1] = l;
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

cudaError_t launch_shared_prefix(const DecodeLaunch& a, const int32_t* shared_blocks,
                                 int shared_len, cudaStream_t stream) {
  const int G = a.num_q_heads / a.cache.num_kv_heads;
  const int bs = a.cache.block_size;
  const int rows = bs < BN ? bs : BN;
  const uint64_t slots = static_cast<uint64_t>(a.cache.num_blocks) * bs;
  CUtensorMap tmQ, tmK, tmV;
  if (!encode_tensor_map_3d(&tmQ, a.q, HD, a.num_q_heads, a.num_seqs, 64, G, BM / G, true) ||
      !encode_tensor_map_3d(&tmK, a.k_cache, HD, a.cache.num_kv_heads, slots, 64, 1, rows, true) ||
      !encode_tensor_map_3d(&tmV, a.v_cache, HD, a.cache.num_kv_heads, slots, 64, 1, rows, true))
    return cudaErrorInvalidValue;
  PrefixParams p;
  p.out = static_cast<__nv_bfloat16*>(a.out);
  p.block_tables = a.block_tables;
  p.shared_blocks = shared_blocks;
  p.context_lens = a.context_lens;
  p.ws_o = a.ws_o;
  p.ws_ml = a.ws_ml;
  p.err = device_error_word();
  p.num_seqs = a.num_seqs;
  p.num_q_heads = a.num_q_heads;
  p.group = G;
  p.max_blocks = a.max_blocks_per_seq;
  p.num_blocks = a.cache.num_blocks;
  p.bs_log2 = 31 - __builtin_clz(static_cast<unsigned>(bs));
  p.shared_len = shared_len;
  p.max_parts = a.max_parts;
  p.max_context_len = a.max_context_len;
  p.scale_log2 = a.scale * kLog2e;
  p.wait_ns = wait_limit_ns();
  cudaError_t e = ensure_max_dynamic_smem(reinterpret_cast<const void*>(shared_prefix_kernel),
                                          kSmemBytes);
  if (e != cudaSuccess) return e;
  // sequences per 128-row unit; two units per CTA (one unit's softmax overlaps the
  // other's products) unless that leaves SMs idle, then one (more SMs beat the overlap)
  const int spt = BM / G;
  const int tiles = (a.num_seqs + spt - 1) / spt;
  p.units = ((tiles + 1) / 2) * a.cache.num_kv_heads < sm_count() ? 1 : 2;
  dim3 grid((a.num_seqs + p.units * spt - 1) / (p.units * spt), a.cache.num_kv_heads);
  shared_prefix_kernel<<<grid, kThreads, kSmemBytes, stream>>>(tmQ, tmK, tmV, p);
  return cudaGetLastError();
}

}  // namespace pa

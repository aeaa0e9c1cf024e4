// Causal paged prefill on the tcgen05 tensor cores: a chunk of new tokens of each
// sequence attends to the sequence's cached prefix plus itself (nano vllm page,
// section 3.1: num_cached_tokens of a Sequence are reused; mini-vllm page,
// section 1: blocks are allocated for the prefill; all K/V are read through the
// block table, section 2).
//
// One CTA = 128 query rows of one (sequence, query head). Per KV tile of 128
// positions:  S = Q K^T  (tcgen05.mma, M=128 N=128 K=128, fp32 in TMEM)
//             softmax on S, one thread per query row (row max / sum stay in the
//             thread; no shuffles), P written to shared memory as bf16
//             O += P V    (tcgen05.mma, accumulator in TMEM, rescaled in place when
//                          the running max moves)
// Roles (192 threads): warps 0-3 softmax + epilogue (warp w owns TMEM lanes
// 32w..32w+31), warp 4 issues TMA loads (Q once, K/V tiles double-buffered and
// gathered block by block through the block table), warp 5 owns the TMEM
// allocation and issues the MMAs from one thread. S(j+1) is issued before PV(j),
// so the tensor core works on the next scores while the softmax runs.
// Operands use the 128-byte swizzled K-major layout (Q, K, P) and the MN-major
// layout (V, whose head dim is contiguous), both produced directly by TMA.
#include <cuda_bf16.h>

#include "pa_internal.h"
#include "pa_ptx.cuh"

namespace pa {
namespace {

constexpr int BM = 128;          // query rows per CTA
constexpr int BN = 128;          // KV positions per tile
constexpr int HD = 128;          // head dim
constexpr int kThreads = 192;
constexpr int kRegion = BM * 128;  // one 64-column half of a 128x128 bf16 tile (16 KB)
constexpr int kTileBytes = 2 * kRegion;
constexpr int kOffQ = 0;
constexpr int kOffK = kOffQ + kTileBytes;       // 2 stages
constexpr int kOffV = kOffK + 2 * kTileBytes;   // 2 stages
constexpr int kOffP = kOffV + 2 * kTileBytes;
constexpr int kOffBar = kOffP + kTileBytes;
constexpr int kNumBars = 12;
constexpr int kOffMisc = kOffBar + 8 * kNumBars;
constexpr int kSmemBytes = kOffMisc + 64 + 1024;  // + slack to align the base to 1 KB
static_assert(kOffQ % 1024 == 0 && kOffK % 1024 == 0 && kOffV % 1024 == 0 && kOffP % 1024 == 0,
              "128-byte-swizzled TMA / MMA operands need 1024-byte alignment");
static_assert(kOffBar % 8 == 0, "mbarriers need 8-byte alignment");
static_assert(kSmemBytes <= 227 * 1024, "shared memory per CTA");
constexpr float kLog2e = 1.4426950408889634f;
constexpr uint32_t kTmemCols = 256;               // S: cols 0-127, O: cols 128-255

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

__global__ void __launch_bounds__(kThreads, 1) prefill_kernel(
    const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
    const __grid_constant__ CUtensorMap tmV, const PrefillParams p) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));

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
  const int first = ctx - n_new;                       // position of the first new token
  const int rows_valid = min(BM, n_new - qt * BM);
  const int pos_max = first + qt * BM + rows_valid - 1;  // last visible position in the tile
  const int ntiles = pos_max / BN + 1;
  const int bs = 1 << p.bs_log2;

  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + kOffBar);
  uint64_t* bar_q = bars + 0;
  uint64_t* bar_kfull = bars + 1;    // [2]
  uint64_t* bar_vfull = bars + 3;    // [2]
  uint64_t* bar_kvempty = bars + 5;  // [2]
  uint64_t* bar_sfull = bars + 7;
  uint64_t* bar_sfree = bars + 8;
  uint64_t* bar_pfull = bars + 9;
  uint64_t* bar_pvdone = bars + 10;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + kOffMisc);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + kOffMisc + 8);

  if (tid == 0) {
    mbar_init(bar_q, 1);
    for (int i = 0; i < 2; ++i) {
      mbar_init(&bar_kfull[i], 1);
      mbar_init(&bar_vfull[i], 1);
      mbar_init(&bar_kvempty[i], 1);
    }
    mbar_init(bar_sfull, 1);
    mbar_init(bar_sfree, BM);
    mbar_init(bar_pfull, BM);
    mbar_init(bar_pvdone, 1);
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
  const uint32_t tS = tmem;
  const uint32_t tO = tmem + 128;

  if (warp == 4) {
    // ------------------------------------------------------------ TMA producer
    if (lane == 0) {
      prefetch_tensormap(&tmQ);
      prefetch_tensormap(&tmK);
      prefetch_tensormap(&tmV);
      const int qrow = q0 + qt * BM;
      mbar_arrive_expect_tx(bar_q, kTileBytes);
      tma_load_3d(smem + kOffQ, &tmQ, bar_q, 0, h, qrow);
      tma_load_3d(smem + kOffQ + kRegion, &tmQ, bar_q, 64, h, qrow);
      const int rows = bs < BN ? bs : BN;
      const int nbox = BN / rows;
      const uint64_t keep = policy_evict_last();  // K/V tiles are re-read by G heads / q tiles
      for (int j = 0; j < ntiles; ++j) {
        const int st = j & 1;
        if (j >= 2 && !wait_or_abort(&bar_kvempty[st], ((j >> 1) - 1) & 1, p.err, abort_flag))
          break;
        uint8_t* kdst = smem + kOffK + st * kTileBytes;
        uint8_t* vdst = smem + kOffV + st * kTileBytes;
        mbar_arrive_expect_tx(&bar_kfull[st], kTileBytes);
        mbar_arrive_expect_tx(&bar_vfull[st], kTileBytes);
        for (int b = 0; b < nbox; ++b) {
          const int pos = j * BN + b * rows;
          const int bi = pos >> p.bs_log2;
          int id = bi < p.max_blocks
                       ? __ldg(p.block_tables + static_cast<int64_t>(s) * p.max_blocks + bi)
                       : -1;
          if (id < 0 || id >= p.num_blocks) {
            if (pos < ctx) flag_error(p.err, PA_DEV_ERR_BAD_INDEX);
            id = 0;
          }
          const int row = id * bs + (pos & (bs - 1));
          tma_load_3d_hint(kdst + b * rows * 128, &tmK, &bar_kfull[st], 0, g, row, keep);
          tma_load_3d_hint(kdst + kRegion + b * rows * 128, &tmK, &bar_kfull[st], 64, g, row, keep);
          tma_load_3d_hint(vdst + b * rows * 128, &tmV, &bar_vfull[st], 0, g, row, keep);
          tma_load_3d_hint(vdst + kRegion + b * rows * 128, &tmV, &bar_vfull[st], 64, g, row, keep);
        }
      }
    }
  } else if (warp == 5) {
    // ------------------------------------------------------------ MMA issuer
    if (lane == 0) {
      constexpr uint32_t idS = idesc_bf16_f32(BM, BN, 0, 0);  // Q K-major, K K-major
      constexpr uint32_t idO = idesc_bf16_f32(BM, HD, 0, 1);  // P K-major, V MN-major
      const uint32_t sQ = smem_u32(smem + kOffQ);
      const uint32_t sP = smem_u32(smem + kOffP);
      auto pv = [&](int i) -> bool {
        if (!wait_or_abort(bar_pfull, i & 1, p.err, abort_flag)) return false;
        if (!wait_or_abort(&bar_vfull[i & 1], (i >> 1) & 1, p.err, abort_flag)) return false;
        tc_fence_after();
        const uint32_t sV = smem_u32(smem + kOffV + (i & 1) * kTileBytes);
#pragma unroll
        for (int kk = 0; kk < BN / 16; ++kk) {
          const uint64_t a = smem_desc_sw128(sP + (kk >> 2) * kRegion + (kk & 3) * 32, 16, 1024);
          const uint64_t b = smem_desc_sw128(sV + kk * 16 * 128, kRegion, 1024);
          tc_mma_f16_ss(tO, a, b, idO, (i > 0 || kk > 0) ? 1u : 0u);
        }
        tc_commit(bar_pvdone);
        tc_commit(&bar_kvempty[i & 1]);
        return true;
      };
      bool ok = wait_or_abort(bar_q, 0, p.err, abort_flag);
      for (int j = 0; ok && j < ntiles; ++j) {
        const int st = j & 1;
        if (!wait_or_abort(&bar_kfull[st], (j >> 1) & 1, p.err, abort_flag)) break;
        if (j > 0 && !wait_or_abort(bar_sfree, (j - 1) & 1, p.err, abort_flag)) break;
        tc_fence_after();
        const uint32_t sK = smem_u32(smem + kOffK + st * kTileBytes);
#pragma unroll
        for (int kk = 0; kk < HD / 16; ++kk) {
          const uint32_t off = (kk >> 2) * kRegion + (kk & 3) * 32;
          const uint64_t a = smem_desc_sw128(sQ + off, 16, 1024);
          const uint64_t b = smem_desc_sw128(sK + off, 16, 1024);
          tc_mma_f16_ss(tS, a, b, idS, kk > 0 ? 1u : 0u);
        }
        tc_commit(bar_sfull);
        if (j > 0 && !pv(j - 1)) {
          ok = false;
          break;
        }
      }
      if (ok && !*abort_flag) pv(ntiles - 1);
    }
  } else {
    // ------------------------------------------------------------ softmax warps
    const int r = tid;  // query row within the tile == TMEM lane
    const int pos_r = first + qt * BM + (r < rows_valid ? r : rows_valid - 1);
    const uint32_t lane_off = static_cast<uint32_t>(warp * 32) << 16;
    uint8_t* sProw = smem + kOffP + r * 128;
    const int sw = r & 7;
    float m = -INFINITY;
    float l = 0.f;
    bool ok = true;
    for (int j = 0; j < ntiles; ++j) {
      if (!wait_or_abort(bar_sfull, j & 1, p.err, abort_flag)) {
        ok = false;
        break;
      }
      tc_fence_after();
      float sv[BN];
#pragma unroll
      for (int c = 0; c < BN / 32; ++c) {
        float t[32];
        tmem_ld32(tS + lane_off + c * 32, t);
#pragma unroll
        for (int i = 0; i < 32; ++i) sv[c * 32 + i] = t[i];
      }
      tc_wait_ld();
      tc_fence_before();
      mbar_arrive(bar_sfree);

      const int kv0 = j * BN;
      const bool need_mask = kv0 + BN - 1 > pos_r;
      float mx = -INFINITY;
#pragma unroll
      for (int c = 0; c < BN; ++c) {
        float x = sv[c] * p.scale_log2;
        if (need_mask && kv0 + c > pos_r) x = -INFINITY;
        sv[c] = x;
        mx = fmaxf(mx, x);
      }
      const float m_new = fmaxf(m, mx);  // finite: position 0 is visible in tile 0
      const float alpha = ex2_approx(m - m_new);
      float rs = 0.f;
      uint32_t pk[BN / 2];
#pragma unroll
      for (int c = 0; c < BN; c += 2) {
        const float p0 = ex2_approx(sv[c] - m_new);
        const float p1 = ex2_approx(sv[c + 1] - m_new);
        rs += p0 + p1;
        pk[c / 2] = pack_bf16x2(p0, p1);
      }
      l = l * alpha + rs;
      m = m_new;

      if (j > 0) {
        if (!wait_or_abort(bar_pvdone, (j - 1) & 1, p.err, abort_flag)) {
          ok = false;
          break;
        }
        tc_fence_after();
        if (__any_sync(0xffffffffu, alpha < 1.f)) {
#pragma unroll
          for (int c = 0; c < HD / 32; ++c) {
            float t[32];
            tmem_ld32(tO + lane_off + c * 32, t);
            tc_wait_ld();
#pragma unroll
            for (int i = 0; i < 32; ++i) t[i] *= alpha;
            tmem_st32(tO + lane_off + c * 32, t);
          }
          tc_wait_st();
        }
      }
      if (j == ntiles - 1 && ctx - kv0 < BN) {
        // rows past the context in the last V tile may hold anything (even NaN);
        // P is 0 there but 0 * NaN is NaN, so clear them before PV reads the tile
        if (!wait_or_abort(&bar_vfull[j & 1], (j >> 1) & 1, p.err, abort_flag)) {
          ok = false;
          break;
        }
        if (r >= ctx - kv0) {
          uint8_t* v = smem + kOffV + (j & 1) * kTileBytes + r * 128;
          const uint4 z = make_uint4(0, 0, 0, 0);
#pragma unroll
          for (int c = 0; c < 8; ++c) {
            *reinterpret_cast<uint4*>(v + c * 16) = z;
            *reinterpret_cast<uint4*>(v + kRegion + c * 16) = z;
          }
        }
      }
      // P row -> shared memory, 128-byte swizzle: chunk c of the row goes to c ^ (row & 7)
#pragma unroll
      for (int c = 0; c < 16; ++c) {
        const int region = c >> 3;
        const int cc = c & 7;
        uint4 w = make_uint4(pk[c * 4 + 0], pk[c * 4 + 1], pk[c * 4 + 2], pk[c * 4 + 3]);
        *reinterpret_cast<uint4*>(sProw + region * kRegion + ((cc ^ sw) << 4)) = w;
      }
      fence_proxy_async_smem();
      tc_fence_before();
      mbar_arrive(bar_pfull);
    }
    if (ok && wait_or_abort(bar_pvdone, (ntiles - 1) & 1, p.err, abort_flag)) {
      tc_fence_after();
      const float inv_l = 1.f / l;
      const bool store = r < rows_valid;
      __nv_bfloat16* orow =
          p.out + (static_cast<int64_t>(q0 + qt * BM + r) * p.num_q_heads + h) * HD;
#pragma unroll
      for (int c = 0; c < HD / 32; ++c) {
        float t[32];
        tmem_ld32(tO + lane_off + c * 32, t);
        tc_wait_ld();
        if (store) {
#pragma unroll
          for (int v4 = 0; v4 < 4; ++v4) {
            uint4 w;
            w.x = pack_bf16x2(t[v4 * 8 + 0] * inv_l, t[v4 * 8 + 1] * inv_l);
            w.y = pack_bf16x2(t[v4 * 8 + 2] * inv_l, t[v4 * 8 + 3] * inv_l);
            w.z = pack_bf16x2(t[v4 * 8 + 4] * inv_l, t[v4 * 8 + 5] * inv_l);
            w.w = pack_bf16x2(t[v4 * 8 + 6] * inv_l, t[v4 * 8 + 7] * inv_l);
            *reinterpret_cast<uint4*>(orow + c * 32 + v4 * 8) = w;
          }
        }
      }
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 5) {
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
  cudaError_t e = ensure_max_dynamic_smem(reinterpret_cast<const void*>(prefill_kernel), kSmemBytes);
  if (e != cudaSuccess) return e;
  dim3 grid((a.max_q_len + BM - 1) / BM, a.num_q_heads, a.num_seqs);
  if (grid.x == 0 || a.num_seqs == 0) return cudaSuccess;
  prefill_kernel<<<grid, kThreads, kSmemBytes, stream>>>(tmQ, tmK, tmV, p);
  return cudaGetLastError();
}

}  // namespace pa

// Paged decode attention: one query token per sequence attends over its whole
// paged context (mini-vllm page, "性能评估与基准测试": decode computes only the new
// token; KVCache reads K/V where the block table says, section 2).
//
// Work decomposition (split-K over the context):
//   one CTA per (sequence s, kv head g, partition p of `partition_size` positions).
//   The CTA handles the G = Hq/Hkv query heads that share kv head g, so every K/V
//   byte is read from HBM exactly once per decode step.
// Data movement:
//   K and V tiles of TILE positions ([TILE, D] bf16 each) are copied by TMA from the
//   pool (viewed as a 3-D tensor [slots][Hkv][D]) into an NSTAGE-deep shared-memory
//   ring; one box per physical block touched, so tiles follow the block table.
// Arithmetic (CUDA cores, fp32; the work is a skinny GEMV per head group and is
// HBM-bound, so it stays off the tensor cores):
//   QK: 8 lanes per position, each lane a 16-element slice of the head dim held
//       against its q slice in registers (packed fp32x2 FMA); the 8 partial dot
//       products are combined with a reduce-scatter over warp shuffles so that each
//       lane ends with one (position, head) score.
//   softmax: each warp keeps its own running max / sum per head (online softmax),
//       in the log2 domain (q is pre-scaled by scale * log2 e).
//   PV: each lane owns D/32 output dims of every head; probabilities are broadcast
//       from a per-warp shared buffer.
//   The 4 warps' (max, sum, unnormalised output) are merged at the end; a single
//   partition writes bf16 output directly, otherwise the partial goes to the
//   workspace and the reduce kernel merges partitions.
#include <cuda_bf16.h>

#include "pa_internal.h"
#include "pa_ptx.cuh"

namespace pa {
namespace {

constexpr int kThreads = 128;  // 4 warps
constexpr float kLog2e = 1.4426950408889634f;

struct DecodeParams {
  const __nv_bfloat16* q;
  __nv_bfloat16* out;
  const int32_t* block_tables;
  const int32_t* context_lens;
  float* ws_o;
  float* ws_ml;
  unsigned* err;
  int max_blocks;
  int num_blocks;
  int bs_log2;
  int num_kv_heads;
  int partition_size;
  int max_parts;
  int max_context_len;
  int max_table_entries;  // capacity of the per-CTA block-id buffer
  float scale_log2;       // scale * log2(e)
};

template <int G>
struct HeadSel {
  // log2(G): the head held by a lane after the reduce-scatter is sub >> (3 - log2 G)
  static constexpr int kLog = (G == 1) ? 0 : (G == 2) ? 1 : (G == 4) ? 2 : 3;
  static constexpr int kShift = 3 - kLog;
};

// Halve the set of `n` values held by each lane: lanes with bit `off` set keep the
// upper half, the others the lower half; each kept value gains its partner's.
template <int N>
__device__ __forceinline__ void halve(float* a, bool up, int off) {
  constexpr int h = N / 2;
#pragma unroll
  for (int j = 0; j < h; ++j) {
    const float send = up ? a[j] : a[h + j];
    const float keep = up ? a[h + j] : a[j];
    a[j] = keep + __shfl_xor_sync(0xffffffffu, send, off);
  }
}

// Reduce-scatter of G partial dot products across the 8 lanes of a position group:
// afterwards lane `sub` holds the full sum for head sub >> (3 - log2 G).
template <int G>
__device__ __forceinline__ float reduce_scatter8(float (&a)[G], int sub) {
  if constexpr (G >= 2) {
    halve<G>(a, (sub & 4) != 0, 4);
  } else {
    a[0] += __shfl_xor_sync(0xffffffffu, a[0], 4);
  }
  constexpr int c2 = (G >= 2) ? G / 2 : 1;
  if constexpr (c2 >= 2) {
    halve<c2>(a, (sub & 2) != 0, 2);
  } else {
    a[0] += __shfl_xor_sync(0xffffffffu, a[0], 2);
  }
  constexpr int c3 = (c2 >= 2) ? c2 / 2 : 1;
  if constexpr (c3 >= 2) {
    halve<c3>(a, (sub & 1) != 0, 1);
  } else {
    a[0] += __shfl_xor_sync(0xffffffffu, a[0], 1);
  }
  return a[0];
}

template <int D, int G, int TILE, int NSTAGE>
struct DecodeSmem {
  static constexpr int kTileBytes = TILE * D * 2;           // one K (or V) tile
  static constexpr int kStageBytes = 2 * kTileBytes;        // K + V
  static constexpr int kRingBytes = NSTAGE * kStageBytes;
  static constexpr int kTokPerWarp = TILE / 4;              // positions per warp per tile
  static constexpr int kBarOff = kRingBytes;
  static constexpr int kPbufOff = kBarOff + 8 * NSTAGE;
  static constexpr int kPbufBytes = 4 * kTokPerWarp * G * 4;
  static constexpr int kAbufOff = kPbufOff + kPbufBytes;
  static constexpr int kMLOff = kAbufOff + 4 * G * 4;
  static constexpr int kIdsOff = kMLOff + 2 * 4 * G * 4;
  static_assert(4 * G * D * 4 <= kRingBytes, "merge buffer must fit in the ring");
  static_assert(kTileBytes % 128 == 0 && kStageBytes % 128 == 0, "TMA destinations: 128 B");
  static_assert(kBarOff % 8 == 0, "mbarriers need 8-byte alignment");
  static_assert(kPbufOff % 4 == 0 && kAbufOff % 4 == 0 && kMLOff % 4 == 0 && kIdsOff % 4 == 0,
                "float / int buffers");
  // + 1 KB so the ring can start on a 1 KB boundary whatever the base alignment
  static int bytes(int max_table_entries) { return kIdsOff + 4 * max_table_entries + 1024; }
};

template <int D, int G, int TILE, int NSTAGE>
__global__ void __launch_bounds__(kThreads) decode_kernel(const __grid_constant__ CUtensorMap tmK,
                                                          const __grid_constant__ CUtensorMap tmV,
                                                          const DecodeParams p) {
  using L = DecodeSmem<D, G, TILE, NSTAGE>;
  constexpr int NCH = D / 64;       // 8-element K chunks per lane in QK
  constexpr int DPL = D / 32;       // output dims per lane in PV
  constexpr int ITERS = TILE / 16;  // QK iterations per tile per warp (4 positions each)
  static_assert(TILE % 16 == 0, "TILE must be a multiple of 16");

  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + L::kBarOff);
  float* pbuf = reinterpret_cast<float*>(smem + L::kPbufOff);
  float* abuf = reinterpret_cast<float*>(smem + L::kAbufOff);
  float* mlbuf = reinterpret_cast<float*>(smem + L::kMLOff);
  int* blk_ids = reinterpret_cast<int*>(smem + L::kIdsOff);

  const int tid = threadIdx.x;
  const int lane = tid & 31;
  const int warp = tid >> 5;
  const int sub = lane & 7;
  const int tg = lane >> 3;
  const int part = blockIdx.x;
  const int g = blockIdx.y;
  const int s = blockIdx.z;
  const int Hq = p.num_kv_heads * G;
  const int bs = 1 << p.bs_log2;

  int ctx = __ldg(p.context_lens + s);
  if (ctx > p.max_context_len) {
    if (tid == 0 && part == 0) flag_error(p.err, PA_DEV_ERR_BAD_INDEX);
    ctx = p.max_context_len;
  }
  const int P = p.partition_size;
  const int nparts = ctx > 0 ? (ctx + P - 1) / P : 0;
  if (ctx <= 0) {
    if (part == 0) {
      for (int i = tid; i < G * D; i += kThreads)
        p.out[(static_cast<int64_t>(s) * Hq + g * G) * D + i] = __float2bfloat16(0.f);
    }
    return;
  }
  if (part >= nparts) return;
  const int t0 = part * P;
  const int n = min(ctx, t0 + P) - t0;
  const int ntiles = (n + TILE - 1) / TILE;

  // ---- block ids of the physical blocks this partition touches ---------------
  const int first_blk = t0 >> p.bs_log2;
  const int last_pos = t0 + ntiles * TILE - 1;
  const int nb = (last_pos >> p.bs_log2) - first_blk + 1;
  for (int i = tid; i < nb; i += kThreads) {
    const int b = first_blk + i;
    int id = -1;
    if (b < p.max_blocks) id = __ldg(p.block_tables + static_cast<int64_t>(s) * p.max_blocks + b);
    if (id < 0 || id >= p.num_blocks) {
      if ((b << p.bs_log2) < ctx) flag_error(p.err, PA_DEV_ERR_BAD_INDEX);
      id = 0;  // in-bounds stand-in; positions past ctx are never used
    }
    if (i < p.max_table_entries) blk_ids[i] = id;
  }
  if (tid == 0) {
    prefetch_tensormap(&tmK);
    prefetch_tensormap(&tmV);
#pragma unroll
    for (int st = 0; st < NSTAGE; ++st) mbar_init(&full[st], 1);
    fence_mbar_init();
  }
  __syncthreads();

  const int rows = bs < TILE ? bs : TILE;
  const int nbox = TILE / rows;
  auto issue = [&](int i) {
    const int st = i % NSTAGE;
    uint8_t* kdst = smem + st * L::kStageBytes;
    uint8_t* vdst = kdst + L::kTileBytes;
    mbar_arrive_expect_tx(&full[st], L::kStageBytes);
    const int tile_start = t0 + i * TILE;
    for (int b = 0; b < nbox; ++b) {
      const int pos = tile_start + b * rows;
      const int row = blk_ids[(pos >> p.bs_log2) - first_blk] * bs + (pos & (bs - 1));
      tma_load_3d(kdst + b * rows * D * 2, &tmK, &full[st], 0, g, row);
      tma_load_3d(vdst + b * rows * D * 2, &tmV, &full[st], 0, g, row);
    }
  };
  if (tid == 0) {
    const int pre = ntiles < NSTAGE ? ntiles : NSTAGE;
    for (int i = 0; i < pre; ++i) issue(i);
  }

  // ---- q slice in registers, pre-scaled into the log2 domain --------------------
  float2 q2[G][NCH * 4];
  {
    const __nv_bfloat16* qs = p.q + (static_cast<int64_t>(s) * Hq + g * G) * D;
#pragma unroll
    for (int h = 0; h < G; ++h) {
#pragma unroll
      for (int c = 0; c < NCH; ++c) {
        const uint4 w = *reinterpret_cast<const uint4*>(qs + h * D + c * 64 + sub * 8);
        const uint32_t ww[4] = {w.x, w.y, w.z, w.w};
#pragma unroll
        for (int e = 0; e < 4; ++e)
          q2[h][c * 4 + e] = make_float2(bf16lo_to_f32(ww[e]) * p.scale_log2,
                                         bf16hi_to_f32(ww[e]) * p.scale_log2);
      }
    }
  }

  const int myhead = sub >> HeadSel<G>::kShift;
  float m_run = -INFINITY;  // running max of this lane's head (log2 domain)
  float l_run = 0.f;        // this lane's share of the running sum
  float2 o2[G][DPL / 2 > 0 ? DPL / 2 : 1];
#pragma unroll
  for (int h = 0; h < G; ++h)
#pragma unroll
    for (int e = 0; e < (DPL / 2 > 0 ? DPL / 2 : 1); ++e) o2[h][e] = make_float2(0.f, 0.f);

  float* my_pbuf = pbuf + warp * L::kTokPerWarp * G;
  float* my_abuf = abuf + warp * G;
  bool alive = true;

  for (int i = 0; i < ntiles; ++i) {
    const int st = i % NSTAGE;
    const bool ok = mbar_wait(&full[st], (i / NSTAGE) & 1, p.err);
    const __nv_bfloat16* Ks = reinterpret_cast<const __nv_bfloat16*>(smem + st * L::kStageBytes);
    const __nv_bfloat16* Vs = Ks + TILE * D;
    const int nvalid = min(TILE, n - i * TILE);

    // ---- scores -------------------------------------------------------------
    float sc[ITERS];
#pragma unroll
    for (int it = 0; it < ITERS; ++it) {
      const int tok = it * 16 + warp * 4 + tg;
      float2 acc2[G];
#pragma unroll
      for (int h = 0; h < G; ++h) acc2[h] = make_float2(0.f, 0.f);
#pragma unroll
      for (int c = 0; c < NCH; ++c) {
        const uint4 w = *reinterpret_cast<const uint4*>(Ks + tok * D + c * 64 + sub * 8);
        const uint32_t ww[4] = {w.x, w.y, w.z, w.w};
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          const float2 kk = make_float2(bf16lo_to_f32(ww[e]), bf16hi_to_f32(ww[e]));
#pragma unroll
          for (int h = 0; h < G; ++h) acc2[h] = __ffma2_rn(q2[h][c * 4 + e], kk, acc2[h]);
        }
      }
      float a[G];
#pragma unroll
      for (int h = 0; h < G; ++h) a[h] = acc2[h].x + acc2[h].y;
      const float v = reduce_scatter8<G>(a, sub);
      sc[it] = tok < nvalid ? v : -INFINITY;
    }

    // ---- online softmax (per warp, per head) ---------------------------------
    float mx = sc[0];
#pragma unroll
    for (int it = 1; it < ITERS; ++it) mx = fmaxf(mx, sc[it]);
    mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 8));
    mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 16));
    const float m_new = fmaxf(m_run, mx);
    const bool live = m_new != -INFINITY;
    const float alpha = live ? ex2_approx(m_run - m_new) : 1.f;
    float psum = 0.f;
#pragma unroll
    for (int it = 0; it < ITERS; ++it) {
      const float pv = (live && sc[it] != -INFINITY) ? ex2_approx(sc[it] - m_new) : 0.f;
      psum += pv;
      my_pbuf[(it * 4 + tg) * G + myhead] = pv;
    }
    l_run = l_run * alpha + psum;
    m_run = m_new;
    if (tg == 0) my_abuf[myhead] = alpha;
    __syncwarp();

    // ---- rescale and accumulate P V -----------------------------------------
#pragma unroll
    for (int h = 0; h < G; ++h) {
      const float a_h = my_abuf[h];
      const float2 aa = make_float2(a_h, a_h);
#pragma unroll
      for (int e = 0; e < (DPL / 2 > 0 ? DPL / 2 : 1); ++e) o2[h][e] = __fmul2_rn(o2[h][e], aa);
    }
#pragma unroll
    for (int it = 0; it < ITERS; ++it) {
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        const int tok = it * 16 + warp * 4 + j;
        if (tok < nvalid) {
          float pr[G];
#pragma unroll
          for (int h = 0; h < G; ++h) pr[h] = my_pbuf[(it * 4 + j) * G + h];
          if constexpr (DPL == 4) {
            const uint2 w = *reinterpret_cast<const uint2*>(Vs + tok * D + lane * 4);
            const float2 v0 = make_float2(bf16lo_to_f32(w.x), bf16hi_to_f32(w.x));
            const float2 v1 = make_float2(bf16lo_to_f32(w.y), bf16hi_to_f32(w.y));
#pragma unroll
            for (int h = 0; h < G; ++h) {
              const float2 pp = make_float2(pr[h], pr[h]);
              o2[h][0] = __ffma2_rn(pp, v0, o2[h][0]);
              o2[h][1] = __ffma2_rn(pp, v1, o2[h][1]);
            }
          } else {
            const uint32_t w = *reinterpret_cast<const uint32_t*>(Vs + tok * D + lane * 2);
            const float2 v0 = make_float2(bf16lo_to_f32(w), bf16hi_to_f32(w));
#pragma unroll
            for (int h = 0; h < G; ++h) {
              const float2 pp = make_float2(pr[h], pr[h]);
              o2[h][0] = __ffma2_rn(pp, v0, o2[h][0]);
            }
          }
        }
      }
    }

    // every warp is done with stage `st` (and with its p buffer) -> refill it
    alive = __syncthreads_and(ok) != 0;
    if (!alive) break;
    if (tid == 0 && i + NSTAGE < ntiles) issue(i + NSTAGE);
  }

  if (!alive) {
    // a wait timed out: drain (bounded) whatever this CTA still has in flight, then leave
    if (tid == 0) {
      for (int st = 0; st < NSTAGE; ++st) mbar_wait(&full[st], 0, nullptr);
    }
    return;
  }

  // ---- merge the 4 warps (ring buffer is free: every issued tile was consumed) ----
  float lsum = l_run;
  lsum += __shfl_xor_sync(0xffffffffu, lsum, 8);
  lsum += __shfl_xor_sync(0xffffffffu, lsum, 16);
  float* ow = reinterpret_cast<float*>(smem);  // [4][G][D]
  float* mw = mlbuf;                           // [4][G]
  float* lw = mlbuf + 4 * G;                   // [4][G]
#pragma unroll
  for (int h = 0; h < G; ++h) {
#pragma unroll
    for (int e = 0; e < (DPL / 2 > 0 ? DPL / 2 : 1); ++e) {
      float* dst = ow + (warp * G + h) * D + lane * DPL + 2 * e;
      if constexpr (DPL >= 2) {
        dst[0] = o2[h][e].x;
        dst[1] = o2[h][e].y;
      }
    }
  }
  if (tg == 0) {
    mw[warp * G + myhead] = m_run;
    lw[warp * G + myhead] = lsum;
  }
  __syncthreads();

  const bool single = nparts == 1;
  for (int idx = tid; idx < G * D; idx += kThreads) {
    const int h = idx / D;
    const int d = idx - h * D;
    float M = mw[h];
#pragma unroll
    for (int w = 1; w < 4; ++w) M = fmaxf(M, mw[w * G + h]);
    float Lsum = 0.f, acc = 0.f;
#pragma unroll
    for (int w = 0; w < 4; ++w) {
      const float mwv = mw[w * G + h];
      const float f = mwv == -INFINITY ? 0.f : ex2_approx(mwv - M);
      Lsum += lw[w * G + h] * f;
      acc += ow[(w * G + h) * D + d] * f;
    }
    const int64_t row = static_cast<int64_t>(s) * Hq + g * G + h;
    if (single) {
      p.out[row * D + d] = __float2bfloat16(acc / Lsum);
    } else {
      const int64_t pr = row * p.max_parts + part;
      p.ws_o[pr * D + d] = acc;
      if (d == 0) {
        p.ws_ml[pr * 2 + 0] = M;
        p.ws_ml[pr * 2 + 1] = Lsum;
      }
    }
  }
}

// Merge partitions: M = max_p m_p, L = sum_p l_p 2^(m_p - M),
// out = sum_p 2^(m_p - M) o_p / L (all in the log2 domain of the main kernel).
__global__ void decode_reduce_kernel(const float* __restrict__ ws_o, const float* __restrict__ ws_ml,
                                     const int32_t* __restrict__ context_lens,
                                     __nv_bfloat16* __restrict__ out, int D, int Hq,
                                     int partition_size, int max_parts, int max_context_len) {
  const int h = blockIdx.x;
  const int s = blockIdx.y;
  int ctx = __ldg(context_lens + s);
  if (ctx > max_context_len) ctx = max_context_len;
  const int nparts = ctx > 0 ? (ctx + partition_size - 1) / partition_size : 0;
  if (nparts <= 1) return;
  const int64_t row = static_cast<int64_t>(s) * Hq + h;
  const float* ml = ws_ml + row * max_parts * 2;
  const float* o = ws_o + row * max_parts * D;
  float M = -INFINITY;
  for (int q = 0; q < nparts; ++q) M = fmaxf(M, ml[2 * q]);
  for (int d = threadIdx.x; d < D; d += blockDim.x) {
    float Lsum = 0.f, acc = 0.f;
    for (int q = 0; q < nparts; ++q) {
      const float f = ex2_approx(ml[2 * q] - M);
      Lsum += ml[2 * q + 1] * f;
      acc += o[static_cast<int64_t>(q) * D + d] * f;
    }
    out[row * D + d] = __float2bfloat16(acc / Lsum);
  }
}

template <int D, int G, int TILE, int NSTAGE>
cudaError_t launch_decode_t(const DecodeLaunch& a, cudaStream_t stream) {
  using L = DecodeSmem<D, G, TILE, NSTAGE>;
  const int bs = a.cache.block_size;
  const int rows = bs < TILE ? bs : TILE;
  CUtensorMap tmK, tmV;
  const uint64_t slots = static_cast<uint64_t>(a.cache.num_blocks) * bs;
  if (!encode_tensor_map_3d(&tmK, a.k_cache, D, a.cache.num_kv_heads, slots, D, 1, rows, false) ||
      !encode_tensor_map_3d(&tmV, a.v_cache, D, a.cache.num_kv_heads, slots, D, 1, rows, false))
    return cudaErrorInvalidValue;

  DecodeParams p;
  p.q = static_cast<const __nv_bfloat16*>(a.q);
  p.out = static_cast<__nv_bfloat16*>(a.out);
  p.block_tables = a.block_tables;
  p.context_lens = a.context_lens;
  p.ws_o = a.ws_o;
  p.ws_ml = a.ws_ml;
  p.err = device_error_word();
  p.max_blocks = a.max_blocks_per_seq;
  p.num_blocks = a.cache.num_blocks;
  p.bs_log2 = 31 - __builtin_clz(static_cast<unsigned>(bs));
  p.num_kv_heads = a.cache.num_kv_heads;
  p.partition_size = a.partition_size;
  p.max_parts = a.max_parts;
  p.max_context_len = a.max_context_len;
  p.max_table_entries = (a.partition_size + TILE - 1) / rows + 2;
  p.scale_log2 = a.scale * kLog2e;

  const int smem = L::bytes(p.max_table_entries);
  if (smem > 200 * 1024) return cudaErrorInvalidValue;
  cudaError_t e0 = ensure_max_dynamic_smem(
      reinterpret_cast<const void*>(decode_kernel<D, G, TILE, NSTAGE>), 200 * 1024);
  if (e0 != cudaSuccess) return e0;
  dim3 grid(a.max_parts, a.cache.num_kv_heads, a.num_seqs);
  decode_kernel<D, G, TILE, NSTAGE><<<grid, kThreads, smem, stream>>>(tmK, tmV, p);
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  if (a.max_parts > 1) {
    dim3 rgrid(a.num_q_heads, a.num_seqs);
    decode_reduce_kernel<<<rgrid, D, 0, stream>>>(a.ws_o, a.ws_ml, a.context_lens,
                                                  static_cast<__nv_bfloat16*>(a.out), D,
                                                  a.num_q_heads, a.partition_size, a.max_parts,
                                                  a.max_context_len);
    e = cudaGetLastError();
  }
  return e;
}

constexpr int kTile = 64;
constexpr int kStages = 3;

template <int D>
cudaError_t dispatch_g(const DecodeLaunch& a, int G, cudaStream_t stream) {
  switch (G) {
    case 1: return launch_decode_t<D, 1, kTile, kStages>(a, stream);
    case 2: return launch_decode_t<D, 2, kTile, kStages>(a, stream);
    case 4: return launch_decode_t<D, 4, kTile, kStages>(a, stream);
    case 8: return launch_decode_t<D, 8, kTile, kStages>(a, stream);
    default: return cudaErrorInvalidValue;
  }
}

}  // namespace

cudaError_t launch_decode(const DecodeLaunch& a, cudaStream_t stream) {
  const int G = a.num_q_heads / a.cache.num_kv_heads;
  if (a.cache.head_dim == 128) return dispatch_g<128>(a, G, stream);
  if (a.cache.head_dim == 64) return dispatch_g<64>(a, G, stream);
  return cudaErrorInvalidValue;
}

}  // namespace pa

// Chained block hashes of a batch of token sequences, for the host block manager's
// prefix lookup (nano vllm page, section 4.2: a block is hashed with
// h = h * 31 + token mod 2^32, seeded with the previous block's hash, so a block's hash
// stands for its whole prefix; the first block is seeded with 0).
//
// One warp per sequence. The hash of block b chained on its prefix is
//   H_b = H_{b-1} * 31^bs + h_b,   h_b = the block's own hash seeded with 0,
// so the lanes first hash whole blocks independently, then chain them: lane l folds a
// contiguous run of blocks into (value, 31^(bs * run length)), a warp scan composes the
// runs (earlier run A then later run B: (A.value * B.mult + B.value, A.mult * B.mult)),
// and each lane rewrites its run with the prefix that precedes it. All arithmetic is
// unsigned 32-bit, i.e. mod 2^32 like the page's mask.
#include "pa_internal.h"
#include "pa_ptx.cuh"

namespace pa {
namespace {

__device__ __forceinline__ uint32_t pow31(uint32_t e) {
  uint32_t r = 1u, b = 31u;
  while (e) {
    if (e & 1u) r *= b;
    b *= b;
    e >>= 1;
  }
  return r;
}

__global__ void __launch_bounds__(128) block_hash_kernel(const int32_t* __restrict__ tokens,
                                                         const int32_t* __restrict__ cu_tokens,
                                                         const int32_t* __restrict__ cu_blocks,
                                                         int32_t num_seqs, int32_t bs,
                                                         uint32_t* __restrict__ out,
                                                         unsigned* err) {
  const int s = static_cast<int>((blockIdx.x * blockDim.x + threadIdx.x) >> 5);
  const int lane = threadIdx.x & 31;
  if (s >= num_seqs) return;  // uniform per warp
  const int64_t t0 = __ldg(cu_tokens + s);
  const int64_t ntok = static_cast<int64_t>(__ldg(cu_tokens + s + 1)) - t0;
  const int32_t first = __ldg(cu_blocks + s);
  int nb = __ldg(cu_blocks + s + 1) - first;
  // the block offsets must agree with the token offsets: a sequence has exactly
  // ntok / bs full blocks. A count past that would read beyond the sequence's tokens;
  // it is clamped (the extra output entries are left as they are) and reported.
  const int64_t nb_max = (t0 >= 0 && ntok > 0) ? ntok / bs : 0;
  if (nb < 0 || nb > nb_max || first < 0) {
    if (lane == 0) flag_error(err, PA_DEV_ERR_BAD_INDEX);
    nb = first < 0 ? 0 : static_cast<int>(nb < 0 ? 0 : nb_max);
  }
  if (nb == 0) return;  // uniform per warp
  uint32_t* o = out + first;
  // 1) each block's own hash (seed 0)
  for (int b = lane; b < nb; b += 32) {
    const int32_t* t = tokens + t0 + static_cast<int64_t>(b) * bs;
    uint32_t h = 0u;
    for (int i = 0; i < bs; ++i) h = h * 31u + static_cast<uint32_t>(__ldg(t + i));
    o[b] = h;
  }
  __syncwarp();
  // 2) chain the blocks: lane l owns the run [b0, b1)
  const uint32_t M = pow31(static_cast<uint32_t>(bs));
  const int run = (nb + 31) / 32;
  const int b0 = min(nb, lane * run), b1 = min(nb, b0 + run);
  uint32_t v = 0u, mult = 1u;
  for (int b = b0; b < b1; ++b) {
    v = v * M + o[b];
    mult *= M;
  }
  for (int d = 1; d < 32; d <<= 1) {  // inclusive scan, earlier runs on the left
    const uint32_t pv = __shfl_up_sync(0xffffffffu, v, d);
    const uint32_t pm = __shfl_up_sync(0xffffffffu, mult, d);
    if (lane >= d) {
      v = pv * mult + v;
      mult = pm * mult;
    }
  }
  uint32_t x = __shfl_up_sync(0xffffffffu, v, 1);  // chained hash before block b0
  if (lane == 0) x = 0u;
  for (int b = b0; b < b1; ++b) {
    x = x * M + o[b];
    o[b] = x;
  }
}

}  // namespace

cudaError_t launch_block_hashes(const int32_t* token_ids, const int32_t* cu_tokens,
                                const int32_t* cu_blocks, int32_t num_seqs, int32_t block_size,
                                uint32_t* hashes_out, cudaStream_t stream) {
  if (num_seqs == 0) return cudaSuccess;
  const int threads = 128;
  const int64_t blocks = (static_cast<int64_t>(num_seqs) * 32 + threads - 1) / threads;
  block_hash_kernel<<<static_cast<unsigned>(blocks), threads, 0, stream>>>(
      token_ids, cu_tokens, cu_blocks, num_seqs, block_size, hashes_out, device_error_word());
  return cudaGetLastError();
}

}  // namespace pa

// Merge of sequence-sharded decode partials.
//
// Each shard of a sequence-sharded decode step (several devices, each holding
// a range of every sequence's cached tokens) produces per query row the
// attention over its own keys, normalised, and the base-2 log-sum-exp of
// their scores.  The merge is the log-sum-exp combine of split-K decoding
// ("Flash Decoding: split-K for long-context decode", ferrum-sampler 0.7.0
// README, Key Optimizations): out = sum_s w_s o_s / sum_s w_s with
// w_s = 2^(lse_s - max_s lse_s); shards with lse = -inf weigh nothing.
//
// One warp per row (b, i, h); lane j fetches the log-sum-exp of shards j,
// j + 32, ...; each lane owns D / 32 consecutive dimensions and reads four
// shard rows at a time.
#include <cuda_bf16.h>

#include "kvd_device.cuh"
#include "kvd_internal.h"
#include "kvd_launch.h"

namespace kvd {
namespace {

template <int D>
__global__ void __launch_bounds__(256) merge_shards_kernel(MergeArgs a) {
  grid_dep_wait();
  grid_dep_launch();
  constexpr int PER = D >= 32 ? D / 32 : 1;
  constexpr int LANES = D >= 32 ? 32 : D;
  const long long row = ((long long)blockIdx.x * blockDim.x + threadIdx.x) >> 5;
  const int lane = threadIdx.x & 31;
  if (row >= a.rows) return;
  const int S = a.shards;
  float M = -INFINITY;
  for (int s = lane; s < S; s += 32) M = fmaxf(M, a.part_lse[(size_t)s * a.rows + row]);
#pragma unroll
  for (int m = 16; m >= 1; m >>= 1) M = fmaxf(M, __shfl_xor_sync(0xffffffffu, M, m));
  const float Ms = (M == -INFINITY) ? 0.f : M;
  const size_t stride = (size_t)a.rows * D;
  const float* base = a.part_o + (size_t)row * D + (size_t)lane * PER;
  float acc[PER];
#pragma unroll
  for (int e = 0; e < PER; ++e) acc[e] = 0.f;
  float L = 0.f;
  for (int s0 = 0; s0 < S; s0 += 32) {
    const int s = s0 + lane;
    const float ls = s < S ? a.part_lse[(size_t)s * a.rows + row] : -INFINITY;
    const float w = (ls == -INFINITY) ? 0.f : fast_exp2(ls - Ms);
    L += w;
    const int m = min(32, S - s0);
    for (int k = 0; k < m; k += 4) {
      float wk[4];
      float x[4][PER];
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        const int kk = min(k + i, m - 1);   // past the end: reload a valid row, weight 0
        wk[i] = __shfl_sync(0xffffffffu, w, kk);
        if (k + i >= m) wk[i] = 0.f;
        const float* src = base + (size_t)(s0 + kk) * stride;
#pragma unroll
        for (int e = 0; e < PER; ++e) x[i][e] = lane < LANES ? src[e] : 0.f;
      }
#pragma unroll
      for (int i = 0; i < 4; ++i)
#pragma unroll
        for (int e = 0; e < PER; ++e) acc[e] += (wk[i] != 0.f) ? wk[i] * x[i][e] : 0.f;
    }
  }
#pragma unroll
  for (int m = 16; m >= 1; m >>= 1) L += __shfl_xor_sync(0xffffffffu, L, m);
  if (lane >= LANES) return;
  const float inv = (L > 0.f) ? 1.f / L : 0.f;
  const size_t ob = (size_t)row * D + (size_t)lane * PER;
#pragma unroll
  for (int e = 0; e < PER; ++e) {
    const float o = acc[e] * inv;
    if (a.out_bf16) reinterpret_cast<__nv_bfloat16*>(a.out)[ob + e] = __float2bfloat16_rn(o);
    else reinterpret_cast<float*>(a.out)[ob + e] = o;
  }
}

}  // namespace

cudaError_t launch_merge_shards(const MergeArgs& a, cudaStream_t st) {
  const dim3 grid((unsigned)((a.rows * 32 + 255) / 256));
  switch (a.D) {
    case 16: return launch_pdl(merge_shards_kernel<16>, grid, dim3(256), 0, st, a);
    case 32: return launch_pdl(merge_shards_kernel<32>, grid, dim3(256), 0, st, a);
    case 64: return launch_pdl(merge_shards_kernel<64>, grid, dim3(256), 0, st, a);
    case 128: return launch_pdl(merge_shards_kernel<128>, grid, dim3(256), 0, st, a);
    case 256: return launch_pdl(merge_shards_kernel<256>, grid, dim3(256), 0, st, a);
    default: return cudaErrorNotSupported;
  }
}

}  // namespace kvd

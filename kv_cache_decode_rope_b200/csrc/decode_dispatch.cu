// Host dispatch of the split-KV decode over storage type and cache layout.
#include "kvd_internal.h"

namespace kvd {

cudaError_t launch_decode_bf16_contig(const DecodeArgs& a, cudaStream_t st);
cudaError_t launch_decode_bf16_paged(const DecodeArgs& a, cudaStream_t st);
cudaError_t launch_decode_f32_contig(const DecodeArgs& a, cudaStream_t st);
cudaError_t launch_decode_f32_paged(const DecodeArgs& a, cudaStream_t st);

cudaError_t launch_decode_tc(const DecodeArgs& a, cudaStream_t st);

bool use_tensor_cores(int D, int bf16, int R) { return bf16 && D == 128 && R >= kTcMinRows; }

bool decode_supported(int D, int bf16, int R) {
  if (R < 1) return false;
  if (use_tensor_cores(D, bf16, R)) return R <= kMaxRows;
  if (R > kMaxRowsCore) return false;
  if (D == 16 || D == 32 || D == 64 || D == 128) return true;
  return D == 256 && bf16;
}

// CTAs of the decode launch: one per SM for the tensor-core kernel (its
// shared memory fills an SM), two per SM for the CUDA-core kernel, never
// more than one 64-token stage of work per CTA below that.
int decode_grid(int B, int Hkv, int max_kv_len, int num_sms, int D, int bf16, int R) {
  const long long chunks = (long long)B * Hkv * ((max_kv_len + kChunk - 1) / kChunk);
  long long g = (chunks + 3) / 4;  // at least one 64-token stage per CTA
  const long long cap = (long long)(use_tensor_cores(D, bf16, R) ? 1 : 2) * num_sms;
  if (g > cap) g = cap;
  if (g > kMaxGrid) g = kMaxGrid;
  if (g < 1) g = 1;
  return (int)g;
}

// Virtual chunks charged per unit in the work split (the cost of a unit
// boundary, in 16-token chunks of streaming): about four 128-token stages for
// the tensor-core kernel (q load, pipeline drain and refill, epilogue; a sweep
// of 16..64 on the MTP-verify and continuous-batching workloads put the best
// at 32-40), 8 for the CUDA-core kernel, whose CTAs each stream at half an
// SM's bandwidth.
constexpr int kSegCostTc = 32;
constexpr int kSegCostCore = 8;

cudaError_t launch_decode(const DecodeArgs& args, int bf16, cudaStream_t st) {
  DecodeArgs a = args;
  if (use_tensor_cores(a.D, bf16, a.R)) {
    a.seg_cost = kSegCostTc;
    const cudaError_t e = launch_decode_tc(a, st);
    // very large batches do not fit the tensor-core kernel's shared memory:
    // units of up to 64 rows then run on the CUDA-core kernel
    if (e != cudaErrorNotSupported || a.R > kMaxRowsCore) return e;
  }
  a.seg_cost = kSegCostCore;
  if (a.block_table)
    return bf16 ? launch_decode_bf16_paged(a, st) : launch_decode_f32_paged(a, st);
  return bf16 ? launch_decode_bf16_contig(a, st) : launch_decode_f32_contig(a, st);
}

}  // namespace kvd

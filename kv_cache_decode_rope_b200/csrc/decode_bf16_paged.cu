// Instantiates the split-KV decode kernels for __nv_bfloat16 storage, paged cache.
#include "decode_split.cuh"

namespace kvd {
cudaError_t launch_decode_bf16_paged(const DecodeArgs& a, cudaStream_t st) {
  return launch_decode_t<__nv_bfloat16, true>(a, st);
}
}  // namespace kvd

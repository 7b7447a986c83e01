// Instantiates the split-KV decode kernels for __nv_bfloat16 storage, contiguous cache.
#include "decode_split.cuh"

namespace kvd {
cudaError_t launch_decode_bf16_contig(const DecodeArgs& a, cudaStream_t st) {
  return launch_decode_t<__nv_bfloat16, false>(a, st);
}
}  // namespace kvd

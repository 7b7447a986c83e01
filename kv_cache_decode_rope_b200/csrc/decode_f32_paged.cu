// Instantiates the split-KV decode kernels for float storage, paged cache.
#include "decode_split.cuh"

namespace kvd {
cudaError_t launch_decode_f32_paged(const DecodeArgs& a, cudaStream_t st) {
  return launch_decode_t<float, true>(a, st);
}
}  // namespace kvd

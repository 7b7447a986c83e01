// Instantiates the split-KV decode kernels for float storage, contiguous cache.
#include "decode_split.cuh"

namespace kvd {
cudaError_t launch_decode_f32_contig(const DecodeArgs& a, cudaStream_t st) {
  return launch_decode_t<float, false>(a, st);
}
}  // namespace kvd

// Kernel launches with programmatic dependent launch (PDL).
//
// Every kernel of the library is launched with programmatic stream
// serialization: it may begin while the kernel before it on the stream is
// still running, once that kernel has allowed it (griddepcontrol
// .launch_dependents, which every kernel here executes early).  Each kernel
// first does the set-up that reads only seq_lens and block_table (shared-memory
// clearing, barrier and tensor-memory set-up, the per-sequence length scan,
// rotary tables), then executes griddepcontrol.wait, which returns once the
// previous kernel has completed and its writes are visible, before it reads q,
// k/v, the caches or the workspace or writes anything.  A previous kernel that
// does not allow early launch simply runs to completion first.
#pragma once

#include <cuda_runtime.h>

namespace kvd {

template <typename... KArgs, typename... Args>
cudaError_t launch_pdl(void (*kern)(KArgs...), dim3 grid, dim3 block, size_t smem, cudaStream_t st,
                       Args... args) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = smem;
  cfg.stream = st;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, kern, args...);
}

}  // namespace kvd

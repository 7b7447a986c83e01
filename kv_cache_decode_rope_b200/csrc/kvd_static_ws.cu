// decode_attention_static: decode attention whose split scratch lives in a
// fixed array inside the library instead of a caller-provided workspace.
//
// Some callers cannot allocate device memory at the point of the call.
// Examples: a host framework that owns every byte of device memory and hands
// out none after start-up; a latency-critical path where an allocation would
// synchronise the device; a foreign-function caller that has no device
// allocator at all.  For them this entry point takes the same inputs and
// outputs as decode_attention / decode_attention_paged.  It keeps the split
// partials in `g_decode_scratch`, a file-scope device array of
// KVD_STATIC_WORKSPACE_BYTES that every GPU which loads the library holds
// until the process exits.  Nothing here calls cudaMalloc, cudaFree or any
// allocating routine.
#include <cuda_runtime.h>

#include <cstdint>
#include <mutex>

#include "../../include/kvdecode.h"
#include "kvd_internal.h"

namespace kvd {
namespace {

// The scratch itself.  In host code this name is only a stand-in for the
// symbol; the device address comes from cudaGetSymbolAddress below.
static __device__ __align__(256) unsigned char g_decode_scratch[KVD_STATIC_WORKSPACE_BYTES];

constexpr int kMaxDevices = 64;
std::mutex g_scratch_mu;
// Per device: the context of the last address lookup and the address there.
// A device address belongs to one context; after a device reset, or with
// another context current, the array is looked up again.
struct ScratchAddr {
  unsigned long long ctx;
  void* ptr;
};
ScratchAddr g_scratch[kMaxDevices] = {};

// Device address of the scratch array in the current context.  The first
// call on a device (or in a new context) asks the runtime for it with that
// device current; later calls reuse it.
int scratch_for_current_context(void** ptr) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return KVD_ERR_CUDA;
  std::lock_guard<std::mutex> lock(g_scratch_mu);
  const unsigned long long ctx = current_context_id();
  if (ctx != 0 && g_scratch[dev].ctx == ctx && g_scratch[dev].ptr) {
    *ptr = g_scratch[dev].ptr;
    return KVD_OK;
  }
  void* p = nullptr;
  if (cudaGetSymbolAddress(&p, g_decode_scratch) != cudaSuccess || !p) return KVD_ERR_CUDA;
  // the lookup made a context current if none was: record that one
  g_scratch[dev].ctx = current_context_id();
  g_scratch[dev].ptr = p;
  *ptr = p;
  return KVD_OK;
}

size_t align256(size_t x) { return (x + 255) / 256 * 256; }

}  // namespace
}  // namespace kvd

using namespace kvd;

extern "C" int decode_attention_static(const kvd_params* p, const void* q, const void* k_cache,
                                       const void* v_cache, const int32_t* seq_lens,
                                       const int32_t* block_table, void* out, void* stream) {
  // the same checks, in the same order, as decode_attention / _paged
  bool nothing = false;
  int rc = check_decode(p, q, k_cache, v_cache, seq_lens, block_table, out, &nothing);
  if (rc != KVD_OK || nothing) return rc;

  void* scratch = nullptr;
  rc = scratch_for_current_context(&scratch);
  if (rc != KVD_OK) return rc;
  int dev = 0;
  const int sms = num_sms_current(&dev);
  if (sms <= 0) return KVD_ERR_CUDA;

  // Carve the scratch for the grid this call launches: one partial slot per
  // (CTA, unit) pair the work split can produce, i.e. grid + units slots.
  DecodeArgs a = decode_args(p, q, k_cache, v_cache, seq_lens, block_table, out, sms);
  const size_t U = (size_t)p->batch * p->num_kv_heads;
  const size_t slots = (size_t)a.grid + U;
  const size_t lse_off = 0;
  const size_t o_off = align256(lse_off + slots * (size_t)a.R * sizeof(float));
  const size_t need = align256(o_off + slots * (size_t)a.R * a.D * sizeof(float));
  if (need > (size_t)KVD_STATIC_WORKSPACE_BYTES) return KVD_ERR_WORKSPACE;

  unsigned char* ws = static_cast<unsigned char*>(scratch);
  a.part_o = reinterpret_cast<float*>(ws + o_off);
  a.part_lse = reinterpret_cast<float*>(ws + lse_off);
  const cudaError_t e = launch_decode(a, p->dtype == KVD_BF16, static_cast<cudaStream_t>(stream));
  if (e == cudaErrorNotSupported) return KVD_ERR_UNSUPPORTED;
  return e == cudaSuccess ? KVD_OK : KVD_ERR_CUDA;
}

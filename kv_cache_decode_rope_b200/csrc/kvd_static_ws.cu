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

#include <cmath>
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
void* g_scratch_ptr[kMaxDevices] = {};
int g_scratch_sms[kMaxDevices] = {};

// Device address of the scratch array and SM count on the current device,
// looked up once per device (the first call on a device does this set-up).
int scratch_for_current_device(void** ptr, int* sms) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return KVD_ERR_CUDA;
  std::lock_guard<std::mutex> lock(g_scratch_mu);
  if (!g_scratch_ptr[dev]) {
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_decode_scratch) != cudaSuccess || !p) return KVD_ERR_CUDA;
    int n = 0;
    if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || n <= 0)
      return KVD_ERR_CUDA;
    g_scratch_ptr[dev] = p;
    g_scratch_sms[dev] = n;
  }
  *ptr = g_scratch_ptr[dev];
  *sms = g_scratch_sms[dev];
  return KVD_OK;
}

size_t align256(size_t x) { return (x + 255) / 256 * 256; }

}  // namespace
}  // namespace kvd

using namespace kvd;

extern "C" int decode_attention_static(const kvd_params* p, const void* q, const void* k_cache,
                                       const void* v_cache, const int32_t* seq_lens,
                                       const int32_t* block_table, void* out, void* stream) {
  if (!p) return KVD_ERR_INVALID_ARG;
  if (p->batch < 0 || p->q_len < 0 || p->num_heads < 1 || p->num_kv_heads < 1 ||
      p->num_heads % p->num_kv_heads != 0)
    return KVD_ERR_INVALID_ARG;
  if (p->dtype != KVD_F32 && p->dtype != KVD_BF16) return KVD_ERR_INVALID_ARG;
  if (p->out_dtype != KVD_F32 && p->out_dtype != KVD_BF16) return KVD_ERR_INVALID_ARG;
  if (!std::isfinite(p->scale)) return KVD_ERR_INVALID_ARG;
  const bool paged = block_table != nullptr;
  if (paged) {
    if (p->page_size < kChunk || p->page_size % kChunk != 0) return KVD_ERR_UNSUPPORTED;
    if (p->num_pages < 1 || p->max_pages_per_seq < 1) return KVD_ERR_INVALID_ARG;
  } else if (p->max_seq_len < 1) {
    return KVD_ERR_INVALID_ARG;
  }
  if (p->batch == 0 || p->q_len == 0) return KVD_OK;
  if (p->max_kv_len < 1) return KVD_ERR_INVALID_ARG;
  if (p->batch > kMaxBatch) return KVD_ERR_UNSUPPORTED;
  const int g = p->num_heads / p->num_kv_heads;
  const long long R = (long long)g * p->q_len;
  if (R > kMaxRows || !decode_supported(p->head_dim, p->dtype == KVD_BF16, (int)R))
    return KVD_ERR_UNSUPPORTED;
  if (!q || !k_cache || !v_cache || !seq_lens || !out) return KVD_ERR_INVALID_ARG;
  const auto mis = [](const void* x) { return (reinterpret_cast<uintptr_t>(x) & 15u) != 0; };
  if (mis(q) || mis(k_cache) || mis(v_cache) || mis(out)) return KVD_ERR_INVALID_ARG;

  void* scratch = nullptr;
  int sms = 0;
  const int rc = scratch_for_current_device(&scratch, &sms);
  if (rc != KVD_OK) return rc;

  // Carve the scratch for the grid this call launches: one partial slot per
  // (CTA, unit) pair the work split can produce, i.e. grid + units slots.
  const int grid = decode_grid(p->batch, p->num_kv_heads, p->max_kv_len, sms, p->head_dim,
                             p->dtype == KVD_BF16, (int)R);
  const size_t U = (size_t)p->batch * p->num_kv_heads;
  const size_t slots = (size_t)grid + U;
  const size_t lse_off = 0;
  const size_t o_off = align256(lse_off + slots * (size_t)R * sizeof(float));
  const size_t need = align256(o_off + slots * (size_t)R * p->head_dim * sizeof(float));
  if (need > (size_t)KVD_STATIC_WORKSPACE_BYTES) return KVD_ERR_WORKSPACE;

  unsigned char* ws = static_cast<unsigned char*>(scratch);
  DecodeArgs a{};
  a.q = q;
  a.k_cache = k_cache;
  a.v_cache = v_cache;
  a.seq_lens = seq_lens;
  a.block_table = block_table;
  a.out = out;
  a.part_o = reinterpret_cast<float*>(ws + o_off);
  a.part_lse = reinterpret_cast<float*>(ws + lse_off);
  a.status = p->status;
  a.B = p->batch;
  a.T = p->q_len;
  a.Hq = p->num_heads;
  a.Hkv = p->num_kv_heads;
  a.g = g;
  a.R = (int)R;
  a.D = p->head_dim;
  a.max_seq_len = p->max_seq_len;
  a.page_size = p->page_size;
  a.num_pages = p->num_pages;
  a.max_pages_per_seq = p->max_pages_per_seq;
  const long long cap =
      paged ? (long long)p->max_pages_per_seq * p->page_size : (long long)p->max_seq_len;
  a.cap_tokens = (int)(cap > INT32_MAX ? INT32_MAX : cap);
  a.qscale = p->scale * 1.4426950408889634f;
  a.out_bf16 = p->out_dtype == KVD_BF16;
  a.grid = grid;
  const cudaError_t e = launch_decode(a, p->dtype == KVD_BF16, static_cast<cudaStream_t>(stream));
  if (e == cudaErrorNotSupported) return KVD_ERR_UNSUPPORTED;
  return e == cudaSuccess ? KVD_OK : KVD_ERR_CUDA;
}

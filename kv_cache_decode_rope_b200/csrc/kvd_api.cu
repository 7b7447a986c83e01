// C-ABI entry points (include/kvdecode.h): argument checks, workspace
// carve-up, grid sizing, launches.  No allocation, no synchronisation.
#include <cuda.h>
#include <cudaTypedefs.h>
#include <cuda_runtime.h>

#include <atomic>
#include <cmath>
#include <cstdint>
#include <mutex>

#include "../../include/kvdecode.h"
#include "kvd_internal.h"

namespace kvd {

namespace {

constexpr size_t kAlign = 256;
size_t align_up(size_t x) { return (x + kAlign - 1) / kAlign * kAlign; }

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

bool head_dim_ok(int D, int dtype) {
  if (D == 16 || D == 32 || D == 64 || D == 128) return true;
  return D == 256 && dtype == KVD_BF16;
}

// Checks shared by every call; returns KVD_OK or a negative status.
int check_common(const kvd_params* p) {
  if (!p) return KVD_ERR_INVALID_ARG;
  if (p->batch < 0 || p->q_len < 0) return KVD_ERR_INVALID_ARG;
  if (p->num_heads < 1 || p->num_kv_heads < 1) return KVD_ERR_INVALID_ARG;
  if (p->num_heads % p->num_kv_heads != 0) return KVD_ERR_INVALID_ARG;
  if (p->dtype != KVD_F32 && p->dtype != KVD_BF16) return KVD_ERR_INVALID_ARG;
  if (!head_dim_ok(p->head_dim, p->dtype)) return KVD_ERR_UNSUPPORTED;
  return KVD_OK;
}

int check_cache(const kvd_params* p, bool paged) {
  if (paged) {
    if (p->page_size < kChunk || p->page_size % kChunk != 0) return KVD_ERR_UNSUPPORTED;
    if (p->num_pages < 1 || p->max_pages_per_seq < 1) return KVD_ERR_INVALID_ARG;
  } else {
    if (p->max_seq_len < 1) return KVD_ERR_INVALID_ARG;
  }
  return KVD_OK;
}

std::atomic<int> g_num_sms[64];

// Checks and argument set-up of a decode call with a caller workspace;
// *nothing = true when there is no work (empty batch or no new tokens).  No
// CUDA call except device queries.
int prepare_decode(const kvd_params* p, const void* q, const void* k_cache, const void* v_cache,
                   const int32_t* seq_lens, const int32_t* block_table, void* out,
                   void* workspace, size_t workspace_bytes, DecodeArgs* args, bool* nothing) {
  const int rc = check_decode(p, q, k_cache, v_cache, seq_lens, block_table, out, nothing);
  if (rc != KVD_OK || *nothing) return rc;
  const size_t need = kvd_workspace_size(p);
  if (!workspace || workspace_bytes < need || !aligned16(workspace)) return KVD_ERR_WORKSPACE;

  int dev = 0;
  const int sms = num_sms_current(&dev);
  if (sms <= 0) return KVD_ERR_CUDA;

  DecodeArgs a = decode_args(p, q, k_cache, v_cache, seq_lens, block_table, out, sms);
  const WorkspaceLayout wl = workspace_layout(p->batch, p->num_kv_heads, a.R, p->head_dim);
  unsigned char* ws = static_cast<unsigned char*>(workspace);
  a.part_o = reinterpret_cast<float*>(ws + wl.part_o_off);
  a.part_lse = reinterpret_cast<float*>(ws + wl.part_lse_off);
  *args = a;
  return KVD_OK;
}

int run_decode(const kvd_params* p, const DecodeArgs& a, void* stream) {
  const cudaError_t e = launch_decode(a, p->dtype == KVD_BF16, static_cast<cudaStream_t>(stream));
  if (e == cudaErrorNotSupported) return KVD_ERR_UNSUPPORTED;
  return e == cudaSuccess ? KVD_OK : KVD_ERR_CUDA;
}

int decode_common(const kvd_params* p, const void* q, const void* k_cache, const void* v_cache,
                  const int32_t* seq_lens, const int32_t* block_table, void* out,
                  void* workspace, size_t workspace_bytes, void* stream) {
  DecodeArgs a{};
  bool nothing = false;
  const int rc = prepare_decode(p, q, k_cache, v_cache, seq_lens, block_table, out, workspace,
                                workspace_bytes, &a, &nothing);
  if (rc != KVD_OK || nothing) return rc;
  return run_decode(p, a, stream);
}

// Checks and argument set-up of an append call (as prepare_decode).
int prepare_append(const kvd_params* p, void* q, const void* k_new, const void* v_new,
                   void* k_cache, void* v_cache, const int32_t* seq_lens,
                   const int32_t* block_table, AppendArgs* args, bool* nothing,
                   bool rotate_only = false) {
  *nothing = false;
  int rc = check_common(p);
  if (rc != KVD_OK) return rc;
  const bool paged = block_table != nullptr;
  rc = check_cache(p, paged);
  if (rc != KVD_OK) return rc;
  if (!std::isfinite(p->rope_base) || p->rope_base <= 0.f) return KVD_ERR_INVALID_ARG;
  if (p->rope_interleaved != 0 && p->rope_interleaved != 1) return KVD_ERR_INVALID_ARG;
  const int rot = p->rotary_dim == 0 ? p->head_dim : p->rotary_dim;
  if (rot < 16 || rot > p->head_dim || rot % 16 != 0) return KVD_ERR_UNSUPPORTED;
  if (p->batch == 0 || p->q_len == 0) {
    *nothing = true;
    return KVD_OK;
  }
  if ((long long)p->batch * p->q_len > INT32_MAX) return KVD_ERR_UNSUPPORTED;
  if (!q || !seq_lens || !aligned16(q)) return KVD_ERR_INVALID_ARG;
  if (!rotate_only) {
    if (!k_new || !v_new || !k_cache || !v_cache) return KVD_ERR_INVALID_ARG;
    if (!aligned16(k_new) || !aligned16(v_new) || !aligned16(k_cache) || !aligned16(v_cache))
      return KVD_ERR_INVALID_ARG;
  } else {
    k_new = v_new = nullptr;
    k_cache = v_cache = nullptr;
  }
  AppendArgs a{};
  a.q = q;
  a.k_new = k_new;
  a.v_new = v_new;
  a.k_cache = k_cache;
  a.v_cache = v_cache;
  a.seq_lens = seq_lens;
  a.block_table = block_table;
  a.status = p->status;
  a.B = p->batch;
  a.T = p->q_len;
  a.Hq = p->num_heads;
  a.Hkv = p->num_kv_heads;
  a.D = p->head_dim;
  a.max_seq_len = p->max_seq_len;
  a.page_size = p->page_size;
  a.num_pages = p->num_pages;
  a.max_pages_per_seq = p->max_pages_per_seq;
  a.rope_base = (double)p->rope_base;
  a.interleaved = p->rope_interleaved;
  a.rot = rot;
  *args = a;
  return KVD_OK;
}

int run_append(const kvd_params* p, const AppendArgs& a, void* stream) {
  const cudaError_t e = launch_append(a, p->dtype == KVD_BF16, static_cast<cudaStream_t>(stream));
  if (e == cudaErrorNotSupported) return KVD_ERR_UNSUPPORTED;
  return e == cudaSuccess ? KVD_OK : KVD_ERR_CUDA;
}

}  // namespace

int num_sms_current(int* dev_out) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return -1;
  *dev_out = dev;
  if (dev >= 0 && dev < 64) {
    const int cached = g_num_sms[dev].load();
    if (cached > 0) return cached;
  }
  int n = 0;
  if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess) return -1;
  if (dev >= 0 && dev < 64) g_num_sms[dev].store(n);
  return n;
}

int check_decode(const kvd_params* p, const void* q, const void* k_cache, const void* v_cache,
                 const int32_t* seq_lens, const int32_t* block_table, const void* out,
                 bool* nothing) {
  *nothing = false;
  int rc = check_common(p);
  if (rc != KVD_OK) return rc;
  const bool paged = block_table != nullptr;
  rc = check_cache(p, paged);
  if (rc != KVD_OK) return rc;
  if (p->out_dtype != KVD_F32 && p->out_dtype != KVD_BF16) return KVD_ERR_INVALID_ARG;
  if (!std::isfinite(p->scale)) return KVD_ERR_INVALID_ARG;
  if (p->batch == 0 || p->q_len == 0) {  // nothing to attend
    *nothing = true;
    return KVD_OK;
  }
  if (p->max_kv_len < 1) return KVD_ERR_INVALID_ARG;
  if (p->batch > kMaxBatch) return KVD_ERR_UNSUPPORTED;
  const int g = p->num_heads / p->num_kv_heads;
  const long long R = (long long)g * p->q_len;
  if (!decode_supported(p->head_dim, p->dtype == KVD_BF16, (int)(R > kMaxRows ? kMaxRows + 1 : R)))
    return KVD_ERR_UNSUPPORTED;
  if (!q || !k_cache || !v_cache || !seq_lens || !out) return KVD_ERR_INVALID_ARG;
  if (!aligned16(q) || !aligned16(k_cache) || !aligned16(v_cache) || !aligned16(out))
    return KVD_ERR_INVALID_ARG;
  return KVD_OK;
}

DecodeArgs decode_args(const kvd_params* p, const void* q, const void* k_cache, const void* v_cache,
                       const int32_t* seq_lens, const int32_t* block_table, void* out, int sms) {
  const bool paged = block_table != nullptr;
  const int g = p->num_heads / p->num_kv_heads;
  const int R = g * p->q_len;
  DecodeArgs a{};
  a.q = q;
  a.k_cache = k_cache;
  a.v_cache = v_cache;
  a.seq_lens = seq_lens;
  a.block_table = block_table;
  a.out = out;
  a.status = p->status;
  a.B = p->batch;
  a.T = p->q_len;
  a.Hq = p->num_heads;
  a.Hkv = p->num_kv_heads;
  a.g = g;
  a.R = R;
  a.D = p->head_dim;
  a.max_seq_len = p->max_seq_len;
  a.page_size = p->page_size;
  a.num_pages = p->num_pages;
  a.max_pages_per_seq = p->max_pages_per_seq;
  const long long cap =
      paged ? (long long)p->max_pages_per_seq * p->page_size : (long long)p->max_seq_len;
  a.cap_tokens = (int)(cap > INT32_MAX ? INT32_MAX : cap);
  a.qscale = p->scale * 1.4426950408889634f;  // log2(e): softmax evaluated with exp2
  a.out_bf16 = p->out_dtype == KVD_BF16;
  a.grid = decode_grid(p->batch, p->num_kv_heads, p->max_kv_len, sms, p->head_dim,
                       p->dtype == KVD_BF16, R);
  return a;
}

unsigned long long current_context_id() {
  static PFN_cuCtxGetCurrent_v4000 get_current = nullptr;
  static PFN_cuCtxGetId_v12000 get_id = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* f = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuCtxGetCurrent", &f, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      get_current = reinterpret_cast<PFN_cuCtxGetCurrent_v4000>(f);
    f = nullptr;
    if (cudaGetDriverEntryPoint("cuCtxGetId", &f, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      get_id = reinterpret_cast<PFN_cuCtxGetId_v12000>(f);
  });
  if (!get_current || !get_id) return 0;
  CUcontext c = nullptr;
  if (get_current(&c) != CUDA_SUCCESS || !c) return 0;
  unsigned long long id = 0;
  if (get_id(c, &id) != CUDA_SUCCESS) return 0;
  return id + 1;   // 0 stays "no context"
}

cudaError_t smem_opt_in(const void* func, int bytes, PerContextOnce& once) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  const bool tracked = dev >= 0 && dev < 64;
  const unsigned long long id = current_context_id();
  if (tracked && id != 0 && once.ctx[dev].load() == id) return cudaSuccess;
  e = cudaFuncSetAttribute(func, cudaFuncAttributeMaxDynamicSharedMemorySize, bytes);
  if (e != cudaSuccess) return e;
  // the runtime call made a context current if none was
  if (tracked) once.ctx[dev].store(current_context_id());
  return cudaSuccess;
}

WorkspaceLayout workspace_layout(int B, int Hkv, int R, int D) {
  WorkspaceLayout w{};
  const size_t U = (size_t)B * Hkv;
  const size_t slots = (size_t)kMaxGrid + U;
  w.part_lse_off = 0;
  w.part_o_off = align_up(w.part_lse_off + slots * R * sizeof(float));
  w.total = align_up(w.part_o_off + slots * R * D * sizeof(float));
  return w;
}

}  // namespace kvd

using namespace kvd;

extern "C" {

int kv_append_rope(const kvd_params* p, void* q, const void* k_new, const void* v_new,
                   void* k_cache, void* v_cache, const int32_t* seq_lens,
                   const int32_t* block_table, void* stream) {
  AppendArgs a{};
  bool nothing = false;
  const int rc = prepare_append(p, q, k_new, v_new, k_cache, v_cache, seq_lens, block_table, &a,
                                &nothing);
  if (rc != KVD_OK || nothing) return rc;
  return run_append(p, a, stream);
}

int kvd_decode_step(const kvd_params* p, void* q, const void* k_new, const void* v_new,
                    void* k_cache, void* v_cache, const int32_t* seq_lens,
                    const int32_t* block_table, void* out, void* workspace,
                    size_t workspace_bytes, void* stream) {
  if (!p) return KVD_ERR_INVALID_ARG;
  AppendArgs aa{};
  DecodeArgs da{};
  bool none_a = false, none_d = false;
  int rc = prepare_append(p, q, k_new, v_new, k_cache, v_cache, seq_lens, block_table, &aa, &none_a);
  if (rc != KVD_OK) return rc;
  rc = prepare_decode(p, q, k_cache, v_cache, seq_lens, block_table, out, workspace,
                      workspace_bytes, &da, &none_d);
  if (rc != KVD_OK || none_a) return rc;
  rc = run_append(p, aa, stream);
  if (rc != KVD_OK || none_d) return rc;
  return run_decode(p, da, stream);
}

int kv_append_rope_cow(const kvd_params* p, void* q, const void* k_new, const void* v_new,
                       void* k_cache, void* v_cache, const int32_t* seq_lens,
                       const int32_t* block_table, const int32_t* cow_src, void* stream) {
  if (!block_table || !cow_src) return KVD_ERR_INVALID_ARG;
  AppendArgs a{};
  bool nothing = false;
  const int rc = prepare_append(p, q, k_new, v_new, k_cache, v_cache, seq_lens, block_table, &a,
                                &nothing);
  if (rc != KVD_OK || nothing) return rc;
  a.cow_src = cow_src;
  return run_append(p, a, stream);
}

int kv_append_rope_shard(const kvd_params* p, void* q, const void* k_new, const void* v_new,
                         void* k_cache, void* v_cache, const int32_t* seq_lens,
                         const int32_t* shard_start, const int32_t* block_table, void* stream) {
  if (!shard_start) return KVD_ERR_INVALID_ARG;
  const bool rotate_only = k_cache == nullptr && v_cache == nullptr;
  AppendArgs a{};
  bool nothing = false;
  const int rc = prepare_append(p, q, k_new, v_new, k_cache, v_cache, seq_lens, block_table, &a,
                                &nothing, rotate_only);
  if (rc != KVD_OK || nothing) return rc;
  a.shard_start = shard_start;
  return run_append(p, a, stream);
}

int decode_attention_shard(const kvd_params* p, const void* q, const void* k_cache,
                           const void* v_cache, const int32_t* seq_lens,
                           const int32_t* shard_start, const int32_t* shard_lens,
                           const int32_t* block_table, float* out, float* out_lse,
                           void* workspace, size_t workspace_bytes, void* stream) {
  if (!p || !shard_start || !shard_lens || !out_lse) return KVD_ERR_INVALID_ARG;
  if (p->out_dtype != KVD_F32) return KVD_ERR_INVALID_ARG;   // partials are fp32
  DecodeArgs a{};
  bool nothing = false;
  const int rc = prepare_decode(p, q, k_cache, v_cache, seq_lens, block_table, out, workspace,
                                workspace_bytes, &a, &nothing);
  if (rc != KVD_OK || nothing) return rc;
  a.shard_start = shard_start;
  a.shard_lens = shard_lens;
  a.out_lse = out_lse;
  return run_decode(p, a, stream);
}

int kvd_merge_partials(const kvd_params* p, const float* part_o, const float* part_lse,
                       int num_shards, void* out, void* stream) {
  int rc = check_common(p);
  if (rc != KVD_OK) return rc;
  if (p->out_dtype != KVD_F32 && p->out_dtype != KVD_BF16) return KVD_ERR_INVALID_ARG;
  if (num_shards < 1) return KVD_ERR_INVALID_ARG;
  const long long rows = (long long)p->batch * p->q_len * p->num_heads;
  if (rows == 0) return KVD_OK;
  if (!part_o || !part_lse || !out) return KVD_ERR_INVALID_ARG;
  if ((reinterpret_cast<uintptr_t>(part_o) & 3u) || (reinterpret_cast<uintptr_t>(part_lse) & 3u) ||
      !aligned16(out))
    return KVD_ERR_INVALID_ARG;
  if (rows * 32 > (long long)INT32_MAX * 8) return KVD_ERR_UNSUPPORTED;
  MergeArgs a{};
  a.part_o = part_o;
  a.part_lse = part_lse;
  a.out = out;
  a.rows = rows;
  a.shards = num_shards;
  a.D = p->head_dim;
  a.out_bf16 = p->out_dtype == KVD_BF16;
  const cudaError_t e = launch_merge_shards(a, static_cast<cudaStream_t>(stream));
  if (e == cudaErrorNotSupported) return KVD_ERR_UNSUPPORTED;
  return e == cudaSuccess ? KVD_OK : KVD_ERR_CUDA;
}

int decode_attention(const kvd_params* p, const void* q, const void* k_cache,
                     const void* v_cache, const int32_t* seq_lens, void* out,
                     void* workspace, size_t workspace_bytes, void* stream) {
  return decode_common(p, q, k_cache, v_cache, seq_lens, nullptr, out, workspace,
                       workspace_bytes, stream);
}

int decode_attention_paged(const kvd_params* p, const void* q, const void* k_cache,
                           const void* v_cache, const int32_t* seq_lens,
                           const int32_t* block_table, void* out, void* workspace,
                           size_t workspace_bytes, void* stream) {
  if (!block_table) return KVD_ERR_INVALID_ARG;
  return decode_common(p, q, k_cache, v_cache, seq_lens, block_table, out, workspace,
                       workspace_bytes, stream);
}

size_t kvd_workspace_size(const kvd_params* p) {
  if (check_common(p) != KVD_OK) return 0;
  const long long R = (long long)(p->num_heads / p->num_kv_heads) * p->q_len;
  if (R < 1 || R > kMaxRows || p->batch < 1 || p->batch > kMaxBatch) return 0;
  return workspace_layout(p->batch, p->num_kv_heads, (int)R, p->head_dim).total;
}

const char* kvd_status_string(int status) {
  switch (status) {
    case KVD_OK: return "ok";
    case KVD_ERR_INVALID_ARG: return "invalid argument";
    case KVD_ERR_UNSUPPORTED: return "unsupported configuration";
    case KVD_ERR_WORKSPACE: return "workspace missing or too small";
    case KVD_ERR_CUDA: return "CUDA launch or device error";
    default: return "unknown status";
  }
}

int kvd_version(void) { return 100; }

}  // extern "C"

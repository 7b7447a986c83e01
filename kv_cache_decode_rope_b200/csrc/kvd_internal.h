// Internal launch interface between the C-ABI layer (kvd_api.cu) and the
// kernel translation units.  Not part of the public ABI.
#pragma once

#include <cuda_runtime.h>
#include <stddef.h>
#include <stdint.h>

#include <atomic>

#include "../../include/kvdecode.h"

namespace kvd {

constexpr int kChunk = 16;        // tokens per work quantum (one page of 16, or a slice of one)
constexpr int kMaxGrid = 1024;    // upper bound on decode CTAs; sizes the workspace
constexpr int kMaxRows = 128;     // g * q_len rows per (sequence, kv head): tensor-core path
constexpr int kMaxRowsCore = 64;  // ... on the CUDA-core path
constexpr int kTcMinRows = 8;     // rows from which QK^T / PV run on the tensor cores
constexpr int kMaxBatch = 8192;   // sequences per call (per-CTA length scan lives in shared memory)

struct AppendArgs {
  void* q;
  const void* k_new;
  const void* v_new;
  void* k_cache;
  void* v_cache;
  const int32_t* seq_lens;
  const int32_t* block_table;  // null: contiguous
  int* status;
  int B, T, Hq, Hkv, D;
  int max_seq_len;
  int page_size, num_pages, max_pages_per_seq;
  double rope_base;
  int interleaved;   // pairs (2j, 2j + 1) instead of (j, j + rot / 2)
  int rot;           // rotated width (a multiple of 16, <= D)
  // Sequence-sharded mode: k and v of position p go to local slot
  // p - shard_start[b] (null: slot p); null caches rotate q only.
  const int32_t* shard_start;
  // Copy on write of shared boundary pages (paged only): before its new
  // tokens land, sequence b with cow_src[b] >= 0 gets slots 0 .. L_b % P - 1
  // of page cow_src[b] copied into page block_table[b][L_b / P].
  const int32_t* cow_src;
};

struct DecodeArgs {
  const void* q;
  const void* k_cache;
  const void* v_cache;
  const int32_t* seq_lens;
  const int32_t* block_table;  // null: contiguous
  void* out;
  float* part_o;      // [slots, R, D]
  float* part_lse;    // [slots, R]
  int* status;
  int B, T, Hq, Hkv, g, R, D;
  int max_seq_len;                       // contiguous capacity
  int page_size, num_pages, max_pages_per_seq;
  int cap_tokens;                        // capacity per sequence in tokens
  float qscale;                          // scale * log2(e)
  int out_bf16;
  int grid;                              // decode CTAs
  int seg_cost;                          // virtual chunks charged per unit (set by the launch)
  // Sequence-sharded mode (all null otherwise): this cache holds the tokens at
  // global positions shard_start[b] .. + shard_lens[b] - 1 of sequence b; the
  // output is fp32 o in `out` plus the base-2 log-sum-exp of each row in out_lse.
  const int32_t* shard_start;
  const int32_t* shard_lens;
  float* out_lse;
};

// Merge of sequence-sharded partials (kvd_merge_partials).
struct MergeArgs {
  const float* part_o;    // [shards, rows, D]
  const float* part_lse;  // [shards, rows], base 2
  void* out;              // [rows, D]
  long long rows;         // B * T * Hq
  int shards, D, out_bf16;
};
cudaError_t launch_merge_shards(const MergeArgs& a, cudaStream_t st);

// Workspace carve-up, shared by kvd_workspace_size and the launch.
struct WorkspaceLayout {
  size_t part_lse_off, part_o_off, total;
};
WorkspaceLayout workspace_layout(int B, int Hkv, int R, int D);

// Host checks of a decode call, in the order every decode entry point applies
// them; no CUDA call.  Sets *nothing when there is no work (empty batch or no
// new tokens), after the checks that do not depend on the work.
int check_decode(const kvd_params* p, const void* q, const void* k_cache, const void* v_cache,
                 const int32_t* seq_lens, const int32_t* block_table, const void* out,
                 bool* nothing);
// Launch arguments of a checked decode call for `sms` SMs (grid included),
// except the split partials part_o / part_lse, which the caller points at its
// scratch.
DecodeArgs decode_args(const kvd_params* p, const void* q, const void* k_cache, const void* v_cache,
                       const int32_t* seq_lens, const int32_t* block_table, void* out, int sms);
// SM count of the current device (cached per device); -1 on a CUDA error.
int num_sms_current(int* dev_out);

// Unique id of the CUDA context current on the calling thread (never reused
// by a later context, e.g. after cudaDeviceReset), or 0 when there is none or
// the driver cannot tell.
unsigned long long current_context_id();

// One-time set-up of one kernel, per device ordinal: the context id under
// which it was last done.  A new context (a device reset, a driver-API
// context) gets the set-up again.
struct PerContextOnce {
  std::atomic<unsigned long long> ctx[64] = {};
};
// Raise func's dynamic shared-memory limit to `bytes`, once per context.
cudaError_t smem_opt_in(const void* func, int bytes, PerContextOnce& once);

cudaError_t launch_append(const AppendArgs& a, int bf16, cudaStream_t st);
// Returns cudaErrorNotSupported when no kernel is compiled for the shape.
cudaError_t launch_decode(const DecodeArgs& a, int bf16, cudaStream_t st);
bool use_tensor_cores(int D, int bf16, int R);
int decode_grid(int B, int Hkv, int max_kv_len, int num_sms, int D, int bf16, int R);
bool decode_supported(int D, int bf16, int R);

}  // namespace kvd

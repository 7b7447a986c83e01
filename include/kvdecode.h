/*
 * kvdecode.h -- C ABI of the KV-cache decode-step library (sm_100a).
 *
 * One autoregressive decode step of a transformer attention layer:
 *   1. kv_append_rope: rotate the new tokens' q and k with RoPE at their
 *      absolute positions and append k and v to the layer's KV cache;
 *   2. decode_attention / decode_attention_paged: attend every new query
 *      token, with grouped-query heads, against the whole cache.
 * The result equals the last rows of a full, non-cached causal attention over
 * the prefix (ferric-core 0.1.0, examples/generate.rs: module doc comment and
 * the exactness check in `run`).
 *
 * Conventions shared by every entry point
 * ---------------------------------------
 * - All tensor pointers are DEVICE pointers owned by the caller.  The library
 *   allocates nothing, keeps no per-call state, never synchronises the
 *   stream, and may be called from several host threads at once.
 * - `stream` is a cudaStream_t passed as void* (NULL = legacy default stream).
 * - Host-side argument checks run before any launch; a failed check returns a
 *   negative kvd_status and launches nothing.  A launch failure returns
 *   KVD_ERR_CUDA (details via cudaGetLastError in the caller's runtime).
 * - Problems only the device can see (a block-table entry outside
 *   [0, num_pages), a length beyond the cache capacity, a pipeline wait that
 *   ran out of its time limit) skip the affected access and OR a
 *   KVD_FLAG_* bit into *params->status when that pointer is non-NULL.  No
 *   kernel traps or asserts.
 * - Stream order with programmatic dependent launch: every kernel of the
 *   library may begin while the kernel before it on the stream finishes,
 *   when that kernel allows early launch (the library's own kernels do).
 *   Before waiting for it, a kernel reads only seq_lens, block_table and
 *   (sequence-sharded calls) shard_start / shard_lens, and may OR a flag
 *   into the status word; q, k_new, v_new, the caches, out and the
 *   workspace are touched only after that kernel has completed.  So a
 *   preceding kernel that allows early launch must not write those index
 *   arrays; any other preceding work is fully ordered as usual.
 *
 * Notation: B = batch, T = q_len (new tokens per sequence), Hq / Hkv = query /
 * key-value heads, g = Hq / Hkv, D = head_dim, L_b = seq_lens[b] = tokens
 * already cached for sequence b BEFORE the step.  New token i of sequence b
 * sits at absolute position L_b + i and attends positions 0 .. L_b + i.
 * Query head h reads kv head h / g.
 *
 * Layouts (row-major, innermost last):
 *   q, out          [B, T, Hq, D]
 *   k_new, v_new    [B, T, Hkv, D]
 *   contiguous cache  k_cache, v_cache [B, Hkv, max_seq_len, D]
 *   paged cache       k_cache, v_cache [num_pages, Hkv, page_size, D]
 *   block_table     [B, max_pages_per_seq] int32: logical page j of sequence b
 *                   (positions j*page_size .. ) lives in physical page
 *                   block_table[b*max_pages_per_seq + j]
 *   seq_lens        [B] int32
 * Every pointer must be 16-byte aligned.
 */
#ifndef KVDECODE_H
#define KVDECODE_H

#include <stddef.h>
#include <stdint.h>

#if defined(__GNUC__)
#define KVD_API __attribute__((visibility("default")))
#else
#define KVD_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

typedef enum kvd_status {
  KVD_OK = 0,
  KVD_ERR_INVALID_ARG = -1, /* null pointer, bad size, bad alignment        */
  KVD_ERR_UNSUPPORTED = -2, /* valid request outside the compiled kernels   */
  KVD_ERR_WORKSPACE = -3,   /* workspace NULL or smaller than required      */
  KVD_ERR_CUDA = -4         /* launch failure or no usable device           */
} kvd_status;

typedef enum kvd_dtype {
  KVD_F32 = 0,
  KVD_BF16 = 1
} kvd_dtype;

/* Bits OR-ed into *kvd_params.status by the device. */
#define KVD_FLAG_PAGE_OUT_OF_RANGE 0x1 /* block-table entry outside [0, num_pages) */
#define KVD_FLAG_CAPACITY 0x2          /* L_b + T beyond the cache capacity        */
#define KVD_FLAG_WAIT_TIMEOUT 0x4      /* a pipeline wait hit its iteration limit  */

/* Parameters shared by all entry points.  Fields a call does not use are
 * ignored (e.g. rope_base by the attention calls, paging fields by the
 * contiguous calls). */
typedef struct kvd_params {
  int batch;             /* B >= 1                                                    */
  int num_heads;         /* Hq >= 1                                                   */
  int num_kv_heads;      /* Hkv >= 1, Hq % Hkv == 0                                   */
  int head_dim;          /* D: 16, 32, 64, 128 or 256                                 */
  int q_len;             /* T >= 1 new tokens per sequence                            */
  float scale;           /* softmax scale applied to q.k (e.g. 1/sqrt(D))             */
  float rope_base;       /* RoPE base (e.g. 10000); kv_append_rope only               */
  int dtype;             /* kvd_dtype of q, k_new, v_new and both caches              */
  int out_dtype;         /* kvd_dtype of out                                          */
  int max_seq_len;       /* contiguous: token capacity per (sequence, kv head)        */
  int page_size;         /* paged: tokens per page, a positive multiple of 16         */
  int num_pages;         /* paged: pages in the pool                                  */
  int max_pages_per_seq; /* paged: block_table row stride                             */
  int max_kv_len;        /* attention: host upper bound on L_b + T over the batch     */
  int* status;           /* optional device int, OR-ed with KVD_FLAG_* bits; may be 0 */
  int rope_interleaved;  /* kv_append_rope: 0 = pairs (j, j + r/2), 1 = pairs (2j, 2j+1) */
  int rotary_dim;        /* kv_append_rope: rotated width r (0 = head_dim); a multiple of
                            16 <= head_dim; elements r .. D-1 are not rotated           */
} kvd_params;

/*
 * kv_append_rope -- RoPE on the new tokens and KV-cache append.
 *
 * Defined by ferric-core 0.1.0, examples/generate.rs, `step_gpu`: the new
 * token's q and k are rotated with `rope_off_t` at the absolute position, v is
 * not rotated, and k and v are appended to the cache (`kc.extend`,
 * `vc.extend`).  Batched with a per-sequence position as in the
 * ferrum-sampler 0.7.0 README, "Key Optimizations" ("Batched RoPE: per-item
 * positions in single kernel launch").
 *
 * RoPE reading (the pages do not fix the pairing): with r = rotary_dim (0
 * means D), the pairs (j, j + r/2) for j < r/2 are rotated by angle
 * (L_b+i) * rope_base^(-2j/r):
 *   (a, b) -> (a cos - b sin, a sin + b cos);
 * rope_interleaved = 1 pairs (2j, 2j+1) instead (the ferrox-models index
 * exports a `RopeLayout` type without defining its members; these are the two
 * common layouts).  Elements r .. D-1 of q and k are not rotated.  The angle
 * and the rotation are evaluated in fp64 and rounded once to dtype (round to
 * nearest even).  KVD_ERR_UNSUPPORTED if rotary_dim is not 0 or a multiple of
 * 16 in [16, D]; KVD_ERR_INVALID_ARG if rope_interleaved is not 0 or 1.
 *
 * q        in/out [B,T,Hq,D]: rotated in place.
 * k_new    in [B,T,Hkv,D]; v_new in [B,T,Hkv,D] (not modified).
 * k_cache, v_cache: receive rotated k and v at position L_b + i; no other slot
 *          is written.
 * block_table: NULL selects the contiguous layout (max_seq_len used);
 *          otherwise the paged layout (page_size, num_pages,
 *          max_pages_per_seq used).  The caller must have mapped every page
 *          that positions L_b .. L_b+T-1 fall in.
 * seq_lens: read only; the caller advances it after the step.
 * Returns KVD_OK or a negative kvd_status.
 */
KVD_API int kv_append_rope(const kvd_params* p, void* q, const void* k_new, const void* v_new,
                   void* k_cache, void* v_cache, const int32_t* seq_lens,
                   const int32_t* block_table, void* stream);

/*
 * decode_attention -- grouped-query attention of the T new query tokens
 * against the contiguous cache.
 *
 * Defined by ferric-core 0.1.0, examples/generate.rs, `step_gpu`
 * (`mha_decode_t(q1, kc, vc, h, h, dh, s)`: single-query attention over all
 * cached tokens, with separate q-head and kv-head counts) and `cpu::mha_causal`
 * in `layer_cpu` (causal softmax attention).  Long contexts are split over
 * several CTAs and merged by log-sum-exp, the split-K scheme named
 * "Flash Decoding" in the ferrum-sampler 0.7.0 README, "Key Optimizations".
 *
 * q        in [B,T,Hq,D], already rotated (kv_append_rope writes it).
 * k_cache, v_cache in [B,Hkv,max_seq_len,D]: positions 0 .. L_b+T-1 are read.
 * seq_lens in [B]: L_b (tokens before the step); the new tokens are the last T
 *          of the L_b+T attended positions, with a causal mask among them.
 * out      out [B,T,Hq,D] in out_dtype:
 *          out = sum_t softmax_t(scale * q.k_t) v_t over the visible t.
 * workspace: caller-owned device scratch of at least
 *          kvd_workspace_size(p) bytes (split partials); contents need no
 *          initialisation and are overwritten.  Two calls that run at the
 *          same time must not share a workspace.
 * Requires max_kv_len >= L_b + T for every b (the grid is sized from it).
 */
KVD_API int decode_attention(const kvd_params* p, const void* q, const void* k_cache,
                     const void* v_cache, const int32_t* seq_lens, void* out,
                     void* workspace, size_t workspace_bytes, void* stream);

/*
 * decode_attention_paged -- decode_attention over the paged cache.
 *
 * Block-table indirection into a shared page pool, as in the ferrum-sampler
 * 0.7.0 README, "Key Optimizations" ("Paged KV attention: GPU block pool with
 * block-table indirection").  Same arguments and result as decode_attention;
 * k_cache/v_cache are [num_pages, Hkv, page_size, D] and block_table maps
 * logical pages to physical pages.
 */
KVD_API int decode_attention_paged(const kvd_params* p, const void* q, const void* k_cache,
                           const void* v_cache, const int32_t* seq_lens,
                           const int32_t* block_table, void* out, void* workspace,
                           size_t workspace_bytes, void* stream);

/*
 * kvd_workspace_size -- bytes of workspace decode_attention[_paged] needs for
 * these parameters (depends on batch, heads, q_len, head_dim; not on the
 * device).  Returns 0 if the parameters are invalid.
 */
KVD_API size_t kvd_workspace_size(const kvd_params* p);

/*
 * kvd_decode_step -- one layer's whole decode step: kv_append_rope, then
 * decode_attention (block_table == NULL) or decode_attention_paged.
 *
 * The loop of ferric-core 0.1.0, examples/generate.rs, `step_gpu` (rope the
 * new tokens, extend the caches, attend) in one call, so that a step of every
 * layer can be captured into a CUDA graph call by call; the ferrum-sampler
 * 0.7.0 README ("Performance") replays decode steps from CUDA graphs.
 *
 * Arguments as kv_append_rope followed by decode_attention[_paged] on the same
 * q (rotated in place by the append), caches, seq_lens and block_table.  Both
 * sets of checks run before anything is launched: any failed check returns
 * its status and launches nothing.  seq_lens is not advanced: the caller adds
 * q_len before the next step.
 */
KVD_API int kvd_decode_step(const kvd_params* p, void* q, const void* k_new, const void* v_new,
                            void* k_cache, void* v_cache, const int32_t* seq_lens,
                            const int32_t* block_table, void* out, void* workspace,
                            size_t workspace_bytes, void* stream);

/*
 * kv_append_rope_cow -- kv_append_rope on a paged cache whose sequences may
 * share prefix pages, with copy on write of the shared boundary page.
 *
 * Sequences that start with the same tokens can point their block-table rows
 * at the same physical pages (the ferrox-models index's `prefix_cache`: reuse
 * the KV state of a shared leading subsequence instead of recomputing it);
 * decode_attention_paged reads such pages like any other.  A page that is
 * shared and only partly filled cannot take a sequence's new tokens: the
 * caller (who owns page allocation) gives the sequence a fresh page in
 * block_table[b][L_b / page_size] and passes the shared page's id in
 * cow_src[b].  Before the new tokens land, slots 0 .. L_b % page_size - 1 of
 * every kv head of page cow_src[b] are copied, k and v, into the fresh page;
 * the shared page is not modified.  cow_src[b] < 0, or L_b a multiple of
 * page_size, means no copy.  Otherwise as kv_append_rope (paged only); page ids
 * outside [0, num_pages) skip the copy and flag KVD_FLAG_PAGE_OUT_OF_RANGE.
 * cow_src in [B] int32, device memory; block_table required.
 */
KVD_API int kv_append_rope_cow(const kvd_params* p, void* q, const void* k_new, const void* v_new,
                               void* k_cache, void* v_cache, const int32_t* seq_lens,
                               const int32_t* block_table, const int32_t* cow_src, void* stream);

/*
 * Sequence-sharded decode (context parallelism): several devices each hold a
 * range of every sequence's cached tokens, compute the attention of the new
 * query tokens over their own range, exchange the per-row results and merge
 * them.  This is the split-K of "Flash Decoding" (ferrum-sampler 0.7.0 README,
 * "Key Optimizations") with the key ranges on different devices; ferrite's
 * context-parallel decode is the same idea.
 *
 * A shard's cache holds, for sequence b, the tokens at global positions
 * shard_start[b] .. shard_start[b] + shard_lens[b] - 1 as its local tokens
 * 0 .. shard_lens[b] - 1, in either layout (max_seq_len / the block table
 * describe the local cache).  seq_lens[b] stays the GLOBAL count of tokens
 * before the step: new token i sits at global position seq_lens[b] + i.
 */

/*
 * kv_append_rope_shard -- kv_append_rope for a shard: q and k of new token i
 * are rotated at the global position seq_lens[b] + i; k and v are stored at the
 * local slot seq_lens[b] + i - shard_start[b] when that slot lies inside the
 * local cache; positions outside the shard's range are not stored (and not
 * flagged: another shard holds them).  With k_cache == v_cache == NULL
 * only q is rotated (k_new, v_new are then ignored): the shards that do not
 * store the new tokens still need the rotated q.
 */
KVD_API int kv_append_rope_shard(const kvd_params* p, void* q, const void* k_new,
                                 const void* v_new, void* k_cache, void* v_cache,
                                 const int32_t* seq_lens, const int32_t* shard_start,
                                 const int32_t* block_table, void* stream);

/*
 * decode_attention_shard -- one shard's part of a sequence-sharded decode.
 *
 * q        in [B,T,Hq,D], rotated.  New token i sees the local tokens whose
 *          global position is at most seq_lens[b] + i (causal among drafts).
 * shard_start, shard_lens in [B] int32 (device): the shard's token range of
 *          each sequence; shard_lens[b] may be 0.
 * block_table: NULL for the contiguous layout [B,Hkv,max_seq_len,D].
 * out      out [B,T,Hq,D] fp32 (out_dtype must be KVD_F32): the attention
 *          over this shard's visible tokens, normalised (0 if none).
 * out_lse  out [B,T,Hq] fp32: log2 of the sum over those tokens of
 *          exp(scale * q.k) (-inf if none).
 * workspace: as decode_attention.  max_kv_len bounds shard_lens[b] (sizes the
 *          grid).  Merging every shard's (out, out_lse) with
 *          kvd_merge_partials gives decode_attention over the whole sequence.
 */
KVD_API int decode_attention_shard(const kvd_params* p, const void* q, const void* k_cache,
                                   const void* v_cache, const int32_t* seq_lens,
                                   const int32_t* shard_start, const int32_t* shard_lens,
                                   const int32_t* block_table, float* out, float* out_lse,
                                   void* workspace, size_t workspace_bytes, void* stream);

/*
 * kvd_merge_partials -- merge S shards' results into the attention output.
 *
 * part_o   in [S,B,T,Hq,D] fp32, part_lse in [S,B,T,Hq] fp32 (base 2), stacked
 *          in any shard order (device memory).
 * out      out [B,T,Hq,D] in out_dtype:
 *          sum_s w_s part_o[s] / sum_s w_s, w_s = 2^(part_lse[s] - max_s part_lse);
 *          shards with lse = -inf weigh nothing (all -inf: 0).
 * Uses batch, q_len, num_heads, head_dim and out_dtype of p.
 */
KVD_API int kvd_merge_partials(const kvd_params* p, const float* part_o, const float* part_lse,
                               int num_shards, void* out, void* stream);

/*
 * decode_attention_static -- decode_attention / decode_attention_paged for
 * callers that cannot allocate device memory.
 *
 * The pages have no counterpart of this call; it exists for callers that have
 * no way to provide a workspace: code running inside a host framework that
 * owns all device memory and hands none out after start-up, a latency-
 * critical path where an allocation would synchronise the device, or a
 * foreign-function caller without a device allocator.
 *
 * Same inputs, outputs and result as decode_attention (block_table == NULL)
 * or decode_attention_paged (block_table != NULL).  Instead of a caller
 * workspace it uses a scratch array of KVD_STATIC_WORKSPACE_BYTES compiled
 * into the library: every GPU that loads the library holds that array until
 * the process exits.  The call allocates nothing.
 * - The first call on a device looks up the array's device address and the
 *   SM count (once per device, with that device current); make that first
 *   call before any stream capture.  The address belongs to the context that
 *   was current at the lookup: a call made with another context current
 *   (after cudaDeviceReset, or under a driver-API context) looks it up again
 *   for that context, so such a call, too, should come before any capture.
 * - All calls on a device share the one array and it keeps the last call's
 *   contents; no part of it needs clearing (every word a call reads is
 *   written earlier in the same call).  Calls that overlap on the GPU (other
 *   streams, other host threads) race on it: serialise them.
 * - Returns KVD_ERR_WORKSPACE when the problem needs more scratch than the
 *   array holds (about (2 * SMs + B * Hkv) * g * q_len * (head_dim + 1) * 4
 *   bytes); every other check, and its order, is that of decode_attention.
 */
#define KVD_STATIC_WORKSPACE_BYTES (16u << 20)
KVD_API int decode_attention_static(const kvd_params* p, const void* q, const void* k_cache,
                                    const void* v_cache, const int32_t* seq_lens,
                                    const int32_t* block_table, void* out, void* stream);

/* kvd_status_string -- static, human-readable text for a kvd_status value. */
KVD_API const char* kvd_status_string(int status);

/* kvd_version -- library version as 10000*major + 100*minor + patch. */
KVD_API int kvd_version(void);

#ifdef __cplusplus
}
#endif

#endif /* KVDECODE_H */

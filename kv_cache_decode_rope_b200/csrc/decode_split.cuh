// Kernels B and C: split-KV flash decode over a contiguous or paged KV cache,
// and the log-sum-exp merge of the splits.
//
// What is computed: ferric-core 0.1.0, examples/generate.rs, `step_gpu`
// (`mha_decode_t`: the new query attends every cached token) with the causal
// rule of `cpu::mha_causal` among several new tokens, grouped-query heads as
// in ferrox-models' `decoder` (q head h reads kv head h / g).  Work is split
// along the cache ("Flash Decoding: split-K for long-context decode", and one
// launch for all batch items, "Batched attention kernel", ferrum-sampler 0.7.0
// README, Key Optimizations) and merged by log-sum-exp.
//
// B200 design (not the pages' design; they describe other hardware):
// * Work quantum = 16 cached tokens of one (sequence, kv head) "unit".  The
//   chunks of all units are laid end to end and cut into `grid` equal ranges,
//   one per CTA, so ragged batches balance exactly and every SM streams the
//   same number of bytes.  Grid = a multiple of the SM count.
// * One CTA owns all g*q_len query rows of a unit, so each K/V byte leaves
//   HBM once.  A producer warp streams K and V stages (64 tokens of D=128
//   bf16 = 16 KB each) into shared memory with 1-D bulk copies (one per
//   page-slice for the paged layout) into a 3-deep mbarrier ring.
// * Consumer warps: each lane owns 16 bytes of a token row (8 bf16 dims) and
//   the matching slice of every query row, held in fp32 registers.  q.k partial
//   sums over the lane's dims are reduced across the lanes of a token with a
//   "transpose-reduce" (each shuffle level halves the values a lane keeps), so
//   one shuffle per score replaces log2(lanes) per score.  Packed fp32 FMA
//   (two lanes of work per instruction) does both contractions.  Online softmax
//   in base 2 with the scale folded into q.
// * A CTA whose range covers a whole unit writes `out`; otherwise it writes a
//   normalised partial (o, lse) to the workspace slot (cta + unit), and
//   kernel C merges the partials of each unit.
#pragma once

#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include <atomic>

#include "kvd_device.cuh"
#include "kvd_internal.h"
#include "kvd_launch.h"

namespace kvd {
namespace {

__host__ __device__ constexpr int ilog2(int x) { return x <= 1 ? 0 : 1 + ilog2(x / 2); }
__host__ __device__ constexpr int cmin(int a, int b) { return a < b ? a : b; }
__host__ __device__ constexpr int cmax(int a, int b) { return a > b ? a : b; }

template <typename T, int D>
struct Geo {
  static constexpr int ES = (int)sizeof(T);
  static constexpr int EPV = 16 / ES;             // elements per lane vector
  static constexpr int NP = EPV / 2;              // fp32 pairs per vector
  static constexpr int LPT = D / EPV;             // lanes per token row
  static constexpr int TPP = 32 / LPT;            // tokens per warp pass
  static constexpr int TOKEN_BYTES = D * ES;
  static constexpr int STAGE_TOKENS = cmax(kChunk, cmin(128, 16384 / TOKEN_BYTES));
  static constexpr int STAGE_CHUNKS = STAGE_TOKENS / kChunk;
  static constexpr int STAGE_BYTES = STAGE_TOKENS * TOKEN_BYTES;
  static constexpr int NSTAGES = 3;
  static_assert(LPT >= 1 && LPT <= 32, "a token row must fit one warp");
};

// Shared-memory carve-up (bytes), identical on host and device.
template <typename T, int D, int RPW, int NTW>
struct Smem {
  using G = Geo<T, D>;
  static constexpr int TW_TOKENS = G::STAGE_TOKENS / NTW;
  static constexpr int TB = cmin(cmin(32 / RPW, TW_TOKENS / G::TPP), G::LPT);
  static constexpr int P_FLOATS = TB * G::TPP * RPW;  // p buffer per warp
  __host__ __device__ static size_t stages() { return (size_t)2 * G::NSTAGES * G::STAGE_BYTES; }
  __host__ __device__ static size_t bars_off() { return stages(); }
  __host__ __device__ static size_t p_off() { return bars_off() + 2 * G::NSTAGES * 8; }
  __host__ __device__ static size_t comb_off(int ncw) { return p_off() + (size_t)ncw * P_FLOATS * 4; }
  __host__ __device__ static size_t ml_off(int ncw) { return comb_off(ncw) + (size_t)ncw * RPW * D * 4; }
  // one group's region (stage rings to merge scratch), 1 KB aligned
  __host__ __device__ static size_t group_bytes(int ncw) {
    return (ml_off(ncw) + (size_t)ncw * RPW * 2 * 4 + 1023) / 1024 * 1024;
  }
  // after the groups: the per-sequence chunk prefix [B + 1], one int per warp
  // of the block for its scan, then N_b per sequence [B]
  __host__ __device__ static size_t prefix_off(int ncw, int groups) { return groups * group_bytes(ncw); }
  __host__ __device__ static size_t total(int ncw, int B, int groups) {
    return prefix_off(ncw, groups) + (size_t)(2 * B + 1 + 32) * 4;
  }
};

struct SegState {
  int b, hk;         // unit
  int k0;            // first chunk of the unit in this CTA's range
  long long x;       // global chunk index of k0
};

// Per-sequence attended length N_b = L_b + T, clamped to the capacity.  In
// sequence-sharded mode: the tokens this shard holds, shard_lens[b].
__device__ __forceinline__ int attended_len(const DecodeArgs& a, int b, bool flag) {
  if (a.shard_lens) {
    long long n = a.shard_lens[b];
    if (n < 0 || n > a.cap_tokens) {
      if (flag && a.status) atomicOr(a.status, KVD_FLAG_CAPACITY);
      n = n < 0 ? 0 : (long long)a.cap_tokens;
    }
    return (int)n;
  }
  long long L = a.seq_lens[b];
  long long N = L + a.T;
  if (L < 0 || N > a.cap_tokens) {
    if (flag && a.status) atomicOr(a.status, KVD_FLAG_CAPACITY);
    N = L < 0 ? a.T : (long long)a.cap_tokens;
    if (N > a.cap_tokens) N = a.cap_tokens;
  }
  return (int)N;
}

// Local position of the first new token of sequence b: token t (local) is
// visible to new token i iff t < mask_base + i + 1.
__device__ __forceinline__ int mask_base(const DecodeArgs& a, int b, int Nb) {
  if (a.shard_start) return (int)max(-2147483647ll, (long long)a.seq_lens[b] - a.shard_start[b]);
  return Nb - a.T;
}

// Chunks of a sequence's unit: at least one, so that a shard holding no token
// of a sequence still writes its (empty) result.
__device__ __forceinline__ int unit_chunks(int Nb) { return max(1, (Nb + kChunk - 1) / kChunk); }

// The work split.  Each unit (sequence b, kv head) occupies seg_cost virtual
// chunks followed by its ceil(N_b / 16) real chunks in one index space, units
// in order (b, then kv head); CTA c takes the slice [total c / grid,
// total (c + 1) / grid).  The virtual chunks charge every unit boundary a
// fixed cost, so a CTA whose slice crosses many short units gets fewer real
// chunks.  Virtual chunks are never loaded.
//
// Block-wide exclusive scan of weighted chunks per sequence: sPrefix[b] = sum
// over b' < b of (max(1, ceil(N_b' / 16)) + seg_cost), sPrefix[B] = total.  All threads of the block
// call it; `scratch` holds one int per warp; `flag`: report lengths beyond
// the capacity in the status word; `sNb` (optional): receives N_b per
// sequence.  Ends with __syncthreads.
__device__ __forceinline__ void chunk_prefix_scan(const DecodeArgs& a, int* sPrefix, int* scratch,
                                                  bool flag, int* sNb = nullptr) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int nthr = blockDim.x;
  const int per = (a.B + nthr - 1) / nthr;
  const int lo = threadIdx.x * per;
  const int hi = min(a.B, lo + per);
  int tsum = 0;
  for (int b = lo; b < hi; ++b)
    tsum += unit_chunks(attended_len(a, b, flag)) + a.seg_cost;
  int incl = tsum;
#pragma unroll
  for (int m = 1; m < 32; m <<= 1) {
    const int v = __shfl_up_sync(0xffffffffu, incl, m);
    if (lane >= m) incl += v;
  }
  if (lane == 31) scratch[warp] = incl;
  __syncthreads();
  int woff = 0;
  for (int w = 0; w < warp; ++w) woff += scratch[w];
  int run = woff + incl - tsum;
  for (int b = lo; b < hi; ++b) {
    sPrefix[b] = run;
    const int nb = attended_len(a, b, false);
    if (sNb) sNb[b] = nb;
    run += unit_chunks(nb) + a.seg_cost;
  }
  if (hi == a.B && lo < hi) sPrefix[a.B] = run;
  __syncthreads();
}

// The unit (sequence b, kv head hk) and weighted chunk within it of global index x:
// largest b with Hkv * prefix[b] <= x, then the head and chunk inside b.
__device__ __forceinline__ SegState locate_chunk(const DecodeArgs& a, const int* sPrefix, long long x) {
  int lo = 0, hi = a.B - 1;
  while (lo < hi) {
    const int mid = (lo + hi + 1) >> 1;
    if ((long long)a.Hkv * sPrefix[mid] <= x) lo = mid; else hi = mid - 1;
  }
  SegState st;
  st.b = lo;
  const int nb = sPrefix[lo + 1] - sPrefix[lo];
  const long long r = x - (long long)a.Hkv * sPrefix[lo];
  st.hk = (int)(r / nb);
  st.k0 = (int)(r % nb);
  st.x = x;
  return st;
}

// A CTA's share of the unit at `c` (slice ending at x1): real chunks
// [k0, kend) of the unit's nb; empty when kend <= k0 (the slice ends inside
// the unit's virtual chunks).
struct Seg {
  int nb, k0, kend;
  long long next_x;  // weighted index where the next unit's share starts
  __device__ bool empty() const { return kend <= k0; }
  __device__ bool whole() const { return k0 == 0 && kend == nb; }
};
__device__ __forceinline__ Seg seg_of(const DecodeArgs& a, const int* sPrefix, const SegState& c,
                                      long long x1) {
  const int ext = sPrefix[c.b + 1] - sPrefix[c.b];
  const int kend_ext = (int)min((long long)ext, c.k0 + (x1 - c.x));
  Seg s;
  s.nb = ext - a.seg_cost;
  s.k0 = max(c.k0 - a.seg_cost, 0);
  s.kend = kend_ext - a.seg_cost;
  s.next_x = c.x + (kend_ext - c.k0);
  return s;
}
__device__ __forceinline__ void next_unit(const DecodeArgs& a, SegState& c, const Seg& s) {
  c.x = s.next_x;
  c.k0 = 0;
  if (++c.hk == a.Hkv) { c.hk = 0; ++c.b; }
}
// Does the slice reach real chunks of the unit after the one ending at next_x?
__device__ __forceinline__ bool next_has_work(const DecodeArgs& a, const Seg& s, long long x1) {
  return x1 - s.next_x > a.seg_cost;
}

// GROUPS = 2: one block holds two independent producer + consumer groups,
// each playing one CTA of the split (block b plays CTAs 2b and 2b + 1) with its
// own rings, barriers and named barrier.  Two separate blocks on one SM do not
// progress at the same rate (the one placed first is favoured and ends ~15%
// earlier, leaving the SM half used for the rest); two groups of one block do.
template <typename T, int D, int RPW, int NTW, bool PAGED, int GROUPS>
__global__ void __launch_bounds__(GROUPS == 2 ? 320 : (NTW == 1 ? 288 : 160))
    decode_kernel(DecodeArgs a, int nrg) {
  using G = Geo<T, D>;
  using S = Smem<T, D, RPW, NTW>;
  using VT = VecTraits<T>;
  constexpr int EPV = G::EPV, NP = G::NP, LPT = G::LPT, TPP = G::TPP;
  constexpr int TB = S::TB;
  constexpr int NV = TB * RPW;  // q.k partial sums per lane per block
  constexpr int TW_TOKENS = S::TW_TOKENS;
  constexpr int NBLK = TW_TOKENS / (TB * TPP);
  constexpr int LOG_LPT = ilog2(LPT);
  constexpr int KLEV = cmin(LOG_LPT, ilog2(NV));  // transposing shuffle levels
  constexpr int NOWN = NV >> KLEV;                 // scores a lane ends with
  constexpr int SHIFT = LOG_LPT - KLEV;            // low lane bits that only replicate
  static_assert(NV * TPP * NBLK * NTW == RPW * G::STAGE_TOKENS, "block tiling");
  static_assert(NOWN <= RPW, "each lane's scores must belong to distinct rows");

  extern __shared__ __align__(1024) unsigned char smem_all[];
  const int ncw = nrg * NTW;                 // consumer warps
  const int gthreads = (ncw + 1) * 32;       // threads of one group
  const int grp = GROUPS == 2 ? (int)threadIdx.x / gthreads : 0;
  const int tid = (int)threadIdx.x - grp * gthreads;
  const int warp = tid >> 5;
  const int lane = tid & 31;
  const int vcta = (int)blockIdx.x * GROUPS + grp;   // the CTA of the split this group plays
  const int bar = 1 + grp;                           // the group's named barrier
  unsigned char* smem = smem_all + (size_t)grp * S::group_bytes(ncw);
  T* sK = reinterpret_cast<T*>(smem);
  T* sV = reinterpret_cast<T*>(smem + (size_t)G::NSTAGES * G::STAGE_BYTES);
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + S::bars_off());
  uint64_t* empty = full + G::NSTAGES;
  float* sP = reinterpret_cast<float*>(smem + S::p_off());
  float* sComb = reinterpret_cast<float*>(smem + S::comb_off(ncw));
  float* sML = reinterpret_cast<float*>(smem + S::ml_off(ncw));
  int* sPrefix = reinterpret_cast<int*>(smem_all + S::prefix_off(ncw, GROUPS));

  // ---- prologue: clear stages, barriers, per-sequence chunk prefix --------
  // the lengths' first round trip overlaps the clearing
  if ((int)threadIdx.x < a.B) prefetch_l1(a.shard_lens ? a.shard_lens + threadIdx.x : a.seq_lens + threadIdx.x);
  {
    // V rows past a partial stage meet zero weights, so they must be finite:
    // the V ring starts from zeros.  K rows there only feed masked scores.
    uint4* z = reinterpret_cast<uint4*>(sV);
    const int n16 = (int)(S::stages() / 32);
    for (int k = tid; k < n16; k += gthreads) z[k] = make_uint4(0, 0, 0, 0);
  }
  if (tid == 0) {
    for (int s = 0; s < G::NSTAGES; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], ncw);
    }
  }
  int* sNb = sPrefix + a.B + 1 + 32;   // attended lengths, read once here
  chunk_prefix_scan(a, sPrefix, sPrefix + a.B + 1, blockIdx.x == 0, sNb);
  fence_barrier_init();
  fence_proxy_async_smem();
  __syncthreads();
  grid_dep_wait();      // q, the caches and the workspace are ready
  grid_dep_launch();

  const long long total = (long long)a.Hkv * sPrefix[a.B];
  if (vcta >= a.grid) return;  // the second group of an odd grid's last block
  const long long x0 = total * vcta / a.grid;
  const long long x1 = total * (vcta + 1) / a.grid;
  if (x0 >= x1) return;  // empty range: no copies issued, nothing to write

  const SegState st = locate_chunk(a, sPrefix, x0);

  if (warp == ncw) {
    // ======================= producer warp ===============================
    int s = 0;
    bool failed = false;
    const uint64_t pol = l2_evict_first();   // the cache is read once
    SegState p = st;
    for (; p.x < x1 && !failed; next_unit(a, p, seg_of(a, sPrefix, p, x1))) {
      const Seg sg = seg_of(a, sPrefix, p, x1);
      if (sg.empty()) continue;
      const int Nb = sNb[p.b];
      const int kend = sg.kend;
      // page ids of the sequence, two 32-chunk windows: the second is loaded
      // 32 chunks ahead of its use so the block-table latency stays off the issue path
      auto page_of = [&](int ch) -> int {
        if (ch >= kend) return -1;
        return a.block_table[(size_t)p.b * a.max_pages_per_seq + (ch * kChunk) / a.page_size];
      };
      int wbase = sg.k0, win0 = -1, win1 = -1;
      if constexpr (PAGED) {
        win0 = page_of(wbase + lane);
        win1 = page_of(wbase + 32 + lane);
      }
      for (int kk = sg.k0; kk < kend; kk += G::STAGE_CHUNKS, ++s) {
        if constexpr (PAGED) {
          if (kk - wbase >= 32) {
            wbase += 32;
            win0 = win1;
            win1 = page_of(wbase + 32 + lane);
          }
        }
        const int slot = s % G::NSTAGES;
        const uint32_t par = (uint32_t)(s / G::NSTAGES) & 1u;
        // one lane waits, the warp follows its verdict (keeps the warp converged)
        int ok = 1;
        if (lane == 0) ok = mbar_wait(&empty[slot], par ^ 1u, a.status) ? 1 : 0;
        ok = __shfl_sync(0xffffffffu, ok, 0);
        if (!ok) { failed = true; break; }
        const int nck = min(G::STAGE_CHUNKS, kend - kk);
        const int t0 = kk * kChunk;
        T* dK = sK + (size_t)slot * G::STAGE_TOKENS * D;
        T* dV = sV + (size_t)slot * G::STAGE_TOKENS * D;
        if constexpr (!PAGED) {
          const int ntok = min(nck * kChunk, Nb - t0);   // <= 0: a shard without tokens here
          const uint32_t bytes = ntok > 0 ? (uint32_t)ntok * G::TOKEN_BYTES : 0u;
          if (lane == 0) {
            mbar_arrive_expect_tx(&full[slot], 2 * bytes);
            if (bytes) {
              const size_t off = (((size_t)p.b * a.Hkv + p.hk) * a.max_seq_len + t0) * D;
              bulk_g2s_hint(dK, reinterpret_cast<const T*>(a.k_cache) + off, bytes, &full[slot], pol);
              bulk_g2s_hint(dV, reinterpret_cast<const T*>(a.v_cache) + off, bytes, &full[slot], pol);
            }
          }
        } else {
          // lane c < nck copies chunk c of the stage (16 tokens inside one page)
          uint32_t bytes = 0;
          size_t off = 0;
          const int page =
              __shfl_sync(0xffffffffu, win0, kk - wbase + min(lane, G::STAGE_CHUNKS - 1));
          const int tc = t0 + lane * kChunk;
          if (lane < nck && tc < Nb) {
            const int ntok = min(kChunk, Nb - tc);
            if (page >= 0 && page < a.num_pages) {
              bytes = (uint32_t)ntok * G::TOKEN_BYTES;
              off = (((size_t)page * a.Hkv + p.hk) * a.page_size + (tc % a.page_size)) * D;
            } else if (a.status) {
              atomicOr(a.status, KVD_FLAG_PAGE_OUT_OF_RANGE);
            }
          }
          uint32_t tot = bytes;
#pragma unroll
          for (int m = 16; m >= 1; m >>= 1) tot += __shfl_xor_sync(0xffffffffu, tot, m);
          if (lane == 0) mbar_arrive_expect_tx(&full[slot], 2 * tot);
          __syncwarp();
          if (bytes) {
            bulk_g2s_hint(dK + (size_t)lane * kChunk * D, reinterpret_cast<const T*>(a.k_cache) + off,
                          bytes, &full[slot], pol);
            bulk_g2s_hint(dV + (size_t)lane * kChunk * D, reinterpret_cast<const T*>(a.v_cache) + off,
                          bytes, &full[slot], pol);
          }
        }
        __syncwarp();
      }
    }
    // drain: every issued copy lands before the CTA may exit
    if (lane == 0) {
      for (int k = max(0, s - G::NSTAGES); k < s; ++k)
        if (!mbar_wait(&full[k % G::NSTAGES], (uint32_t)(k / G::NSTAGES) & 1u, a.status)) break;
    }
    return;
  }

  // ========================= consumer warps ==============================
  const int rg = warp / NTW;             // row group
  const int tw = warp % NTW;             // token slice of each stage
  const int hg = lane / LPT;             // token within a warp pass
  const int lg = lane % LPT;             // 16-byte slice of the head dim
  const int ncons = ncw * 32;
  // rows of this lane's own scores (fixed for the kernel)
  int own_row[NOWN];
#pragma unroll
  for (int i = 0; i < NOWN; ++i) own_row[i] = (i + NOWN * (lg >> SHIFT)) % RPW;
  int own_tok[NOWN];  // token index within a block (0..TB-1) of own score i
#pragma unroll
  for (int i = 0; i < NOWN; ++i) own_tok[i] = (i + NOWN * (lg >> SHIFT)) / RPW;
  float* myP = sP + warp * S::P_FLOATS;

  // this lane's 16-byte slice of q row r of unit (b, hk) (null past the rows)
  auto q_ptr = [&](int b, int hk, int r) -> const uint4* {
    const int rglob = rg * RPW + r;
    if (rglob >= a.R) return nullptr;
    const int i = rglob / a.g;
    const int h = hk * a.g + rglob % a.g;
    return reinterpret_cast<const uint4*>(reinterpret_cast<const T*>(a.q) +
                                          (((size_t)b * a.T + i) * a.Hq + h) * D + lg * EPV);
  };

  int s = 0;
  bool failed = false;
  SegState c = st;
  for (; c.x < x1; next_unit(a, c, seg_of(a, sPrefix, c, x1))) {
    const Seg sg = seg_of(a, sPrefix, c, x1);
    if (sg.empty()) continue;
    const int Nb = sNb[c.b];
    const int Lb = mask_base(a, c.b, Nb);  // local position of the first new token (may be <= 0)
    const int kend = sg.kend;
    const int u = c.b * a.Hkv + c.hk;

    // -- segment init: q rows of this warp, pre-scaled for exp2
    float2 q2[RPW][NP];
    float2 o2[RPW][NP];
    float m_all[RPW];
    float m_own[NOWN], l_own[NOWN];
    int vis_own[NOWN];  // visible token count of own rows
#pragma unroll
    for (int r = 0; r < RPW; ++r) {
      m_all[r] = -INFINITY;
      const uint4* qp = q_ptr(c.b, c.hk, r);
      const uint4 qv = qp ? *qp : make_uint4(0u, 0u, 0u, 0u);
      float2 f[NP];
      VT::unpack(qv, f);
#pragma unroll
      for (int e = 0; e < NP; ++e) {
        o2[r][e] = make_float2(0.f, 0.f);
        q2[r][e] = make_float2(f[e].x * a.qscale, f[e].y * a.qscale);
      }
    }
    // the unit after this one, if this slice reaches it: its q is prefetched
    // into L1 during this segment's last stage, so that the load at the
    // segment change does not wait on HBM under full load
    const bool prefetch_next = next_has_work(a, sg, x1);
    const int nx_hk = (c.hk + 1 == a.Hkv) ? 0 : c.hk + 1;
    const int nx_b = (c.hk + 1 == a.Hkv) ? c.b + 1 : c.b;
#pragma unroll
    for (int i = 0; i < NOWN; ++i) {
      m_own[i] = -INFINITY;
      l_own[i] = 0.f;
      const int rglob = rg * RPW + own_row[i];
      vis_own[i] = (rglob < a.R) ? Lb + rglob / a.g + 1 : Nb;
    }

    for (int kk = sg.k0; kk < kend; kk += G::STAGE_CHUNKS, ++s) {
      const int slot = s % G::NSTAGES;
      const uint32_t par = (uint32_t)(s / G::NSTAGES) & 1u;
      if (prefetch_next && kk + G::STAGE_CHUNKS >= kend) {
#pragma unroll
        for (int r = 0; r < RPW; ++r) {
          const uint4* qp = q_ptr(nx_b, nx_hk, r);
          if (qp) prefetch_l1(qp);
        }
      }
      if (!failed && !mbar_wait(&full[slot], par, a.status)) failed = true;
      const int t0 = kk * kChunk;
      const int nvalid = min(min(G::STAGE_CHUNKS, kend - kk) * kChunk, Nb - t0);
      // masking is needed when the stage is short or reaches the new tokens
      const bool tail = (nvalid < G::STAGE_TOKENS) || (t0 + G::STAGE_TOKENS > Lb + 1);
      const T* Ks = sK + (size_t)slot * G::STAGE_TOKENS * D;
      const T* Vs = sV + (size_t)slot * G::STAGE_TOKENS * D;

#pragma unroll 1
      for (int blk = 0; blk < NBLK; ++blk) {
        const int tbase = tw * TW_TOKENS + blk * TB * TPP;  // first token of the block in the stage
        // ---- scores: partial dot products over this lane's dims
        float sc[NV];
#pragma unroll
        for (int j = 0; j < TB; ++j) {
          const int t = tbase + j * TPP + hg;
          float2 kf[NP];
          VT::unpack(*reinterpret_cast<const uint4*>(Ks + (size_t)t * D + lg * EPV), kf);
#pragma unroll
          for (int r = 0; r < RPW; ++r) {
            float2 acc = fmul2(q2[r][0], kf[0]);
#pragma unroll
            for (int e = 1; e < NP; ++e) acc = ffma2(q2[r][e], kf[e], acc);
            sc[j * RPW + r] = acc.x + acc.y;
          }
        }
        // ---- transpose-reduce across the LPT lanes of a token
        {
          int n = NV;
#pragma unroll
          for (int lev = 0; lev < LOG_LPT; ++lev) {
            const int m = LPT >> (lev + 1);
            if (lev < KLEV) {
              const bool upper = (lane & m) != 0;
              const int half = NV >> (lev + 1);
#pragma unroll
              for (int i2 = 0; i2 < half; ++i2) {
                const float lo_v = sc[i2], hi_v = sc[i2 + half];
                const float send = upper ? lo_v : hi_v;
                const float keep = upper ? hi_v : lo_v;
                sc[i2] = keep + __shfl_xor_sync(0xffffffffu, send, m);
              }
            } else {
              sc[0] += __shfl_xor_sync(0xffffffffu, sc[0], m);
            }
          }
          (void)n;
        }
        // ---- mask
        if (tail) {
#pragma unroll
          for (int i = 0; i < NOWN; ++i) {
            const int t = tbase + own_tok[i] * TPP + hg;
            if (t >= nvalid || t0 + t >= vis_own[i]) sc[i] = -INFINITY;
          }
        }
        // ---- block max per own row, across lanes holding the same row
        float bm[NOWN];
#pragma unroll
        for (int i = 0; i < NOWN; ++i) bm[i] = sc[i];
#pragma unroll
        for (int m = 1; m < 32; m <<= 1) {
          bool same_row;
          if (m >= LPT) same_row = true;
          else if (m < (1 << SHIFT)) same_row = false;  // replica lanes hold equal values
          else same_row = ((NOWN * (m >> SHIFT)) % RPW) == 0;
          if (same_row) {
#pragma unroll
            for (int i = 0; i < NOWN; ++i) bm[i] = fmaxf(bm[i], __shfl_xor_sync(0xffffffffu, bm[i], m));
          }
        }
        // ---- every row's block max to every lane; rescale accumulators
#pragma unroll
        for (int r = 0; r < RPW; ++r) {
          const float bmr = __shfl_sync(0xffffffffu, bm[r % NOWN], (r / NOWN) << SHIFT);
          const float mn = fmaxf(m_all[r], bmr);
          const float ms = (mn == -INFINITY) ? 0.f : mn;
          const float alpha = fast_exp2(m_all[r] - ms);
          m_all[r] = mn;
          const float2 al = make_float2(alpha, alpha);
#pragma unroll
          for (int e = 0; e < NP; ++e) o2[r][e] = fmul2(o2[r][e], al);
        }
        // ---- probabilities of own scores
#pragma unroll
        for (int i = 0; i < NOWN; ++i) {
          const float mn = fmaxf(m_own[i], bm[i]);
          const float ms = (mn == -INFINITY) ? 0.f : mn;
          const float pr = fast_exp2(sc[i] - ms);
          l_own[i] = l_own[i] * fast_exp2(m_own[i] - ms) + pr;
          m_own[i] = mn;
          myP[(own_tok[i] * TPP + hg) * RPW + own_row[i]] = pr;
        }
        __syncwarp();
        // ---- o += p v
#pragma unroll
        for (int j = 0; j < TB; ++j) {
          const int t = tbase + j * TPP + hg;
          float2 vf[NP];
          VT::unpack(*reinterpret_cast<const uint4*>(Vs + (size_t)t * D + lg * EPV), vf);
          const float* pj = myP + (j * TPP + hg) * RPW;
          float pv[RPW];
          if constexpr (RPW % 4 == 0) {
#pragma unroll
            for (int r4 = 0; r4 < RPW; r4 += 4) {
              const float4 v4 = *reinterpret_cast<const float4*>(pj + r4);
              pv[r4] = v4.x; pv[r4 + 1] = v4.y; pv[r4 + 2] = v4.z; pv[r4 + 3] = v4.w;
            }
          } else {
#pragma unroll
            for (int r = 0; r < RPW; ++r) pv[r] = pj[r];
          }
#pragma unroll
          for (int r = 0; r < RPW; ++r) {
            const float2 pp = make_float2(pv[r], pv[r]);
#pragma unroll
            for (int e = 0; e < NP; ++e) o2[r][e] = ffma2(pp, vf[e], o2[r][e]);
          }
        }
        __syncwarp();
      }
      if (lane == 0) mbar_arrive(&empty[slot]);
    }

    // -- segment end: reduce within the warp, then across token slices
#pragma unroll
    for (int m = 1; m < 32; m <<= 1) {
      bool same_row;
      if (m >= LPT) same_row = true;
      else if (m < (1 << SHIFT)) same_row = false;
      else same_row = ((NOWN * (m >> SHIFT)) % RPW) == 0;
      if (same_row) {
#pragma unroll
        for (int i = 0; i < NOWN; ++i) l_own[i] += __shfl_xor_sync(0xffffffffu, l_own[i], m);
      }
    }
#pragma unroll
    for (int m = LPT; m < 32; m <<= 1) {
#pragma unroll
      for (int r = 0; r < RPW; ++r)
#pragma unroll
        for (int e = 0; e < NP; ++e) {
          o2[r][e].x += __shfl_xor_sync(0xffffffffu, o2[r][e].x, m);
          o2[r][e].y += __shfl_xor_sync(0xffffffffu, o2[r][e].y, m);
        }
    }
    if (lane < LPT) {
#pragma unroll
      for (int r = 0; r < RPW; ++r) {
        float* dst = sComb + ((size_t)warp * RPW + r) * D + lg * EPV;
#pragma unroll
        for (int e = 0; e < NP; ++e) { dst[2 * e] = o2[r][e].x; dst[2 * e + 1] = o2[r][e].y; }
      }
      if ((lg & ((1 << SHIFT) - 1)) == 0) {
#pragma unroll
        for (int i = 0; i < NOWN; ++i) {
          if (own_tok[i] == 0) {
            sML[((size_t)warp * RPW + own_row[i]) * 2 + 1] = l_own[i];
          }
        }
      }
    }
    if (lane == 0) {
#pragma unroll
      for (int r = 0; r < RPW; ++r) sML[((size_t)warp * RPW + r) * 2] = m_all[r];
    }
    named_bar_sync(bar, ncons);

    const bool whole = sg.whole();
    const long long slot_idx = (long long)vcta + u;
    for (int e = tid; e < nrg * RPW * D; e += ncons) {
      const int rgi = e / (RPW * D);
      const int r = (e / D) % RPW;
      const int d = e % D;
      const int rglob = rgi * RPW + r;
      if (rglob >= a.R) continue;
      float M = -INFINITY;
      for (int w = 0; w < NTW; ++w) M = fmaxf(M, sML[((size_t)(rgi * NTW + w) * RPW + r) * 2]);
      const float Ms = (M == -INFINITY) ? 0.f : M;
      float L = 0.f, O = 0.f;
      for (int w = 0; w < NTW; ++w) {
        const int ww = rgi * NTW + w;
        const float wt = fast_exp2(sML[((size_t)ww * RPW + r) * 2] - Ms);
        L += wt * sML[((size_t)ww * RPW + r) * 2 + 1];
        O += wt * sComb[((size_t)ww * RPW + r) * D + d];
      }
      const float o = (L > 0.f) ? O / L : 0.f;
      if (whole) {
        const int i = rglob / a.g;
        const int h = c.hk * a.g + rglob % a.g;
        const size_t row = ((size_t)c.b * a.T + i) * a.Hq + h;
        const size_t oi = row * D + d;
        if (a.out_bf16) reinterpret_cast<__nv_bfloat16*>(a.out)[oi] = __float2bfloat16_rn(o);
        else reinterpret_cast<float*>(a.out)[oi] = o;
        if (a.out_lse && d == 0) a.out_lse[row] = (L > 0.f) ? Ms + fast_log2(L) : -INFINITY;
      } else {
        // partials stay in L2 for the merge (evict_last)
        const uint64_t keep = l2_evict_last();
        st_hint(a.part_o + ((size_t)slot_idx * a.R + rglob) * D + d, o, keep);
        if (d == 0)
          st_hint(a.part_lse + (size_t)slot_idx * a.R + rglob, (L > 0.f) ? Ms + fast_log2(L) : -INFINITY, keep);
      }
    }
    named_bar_sync(bar, ncons);
  }
}

// CTA holding global weighted chunk x of a split over `total` chunks: the
// largest c with floor(total c / grid) <= x.
__device__ __forceinline__ int cta_of_chunk(long long x, long long total, int grid) {
  return (int)(((x + 1) * grid - 1) / total);
}

// Kernel C: one warp per (unit, row) merges the partials of units split over
// several CTAs: out = sum_s 2^(lse_s - LSE) o_s with LSE = log2 sum_s 2^lse_s.
// The CTAs that share a unit follow from the split itself, which every block
// recomputes from the sequence lengths before the decode kernel finishes, so
// after the wait only the partials are read: lane j fetches the log-sum-exp
// of partial j while every lane fetches its D / 32 dimensions of the first
// four partial rows, all in one round trip; longer splits continue four
// partial rows at a time.
template <int D>
__global__ void __launch_bounds__(256) combine_kernel(DecodeArgs a) {
  extern __shared__ int sPrefix[];   // [B + 1] chunk prefix, then one int per warp
  chunk_prefix_scan(a, sPrefix, sPrefix + a.B + 1, false);
  grid_dep_wait();      // the partials of the decode kernel
  grid_dep_launch();
  constexpr int PER = D >= 32 ? D / 32 : 1;   // dimensions per lane
  constexpr int LANES = D >= 32 ? 32 : D;     // lanes that hold dimensions
  const long long wid = ((long long)blockIdx.x * blockDim.x + threadIdx.x) >> 5;
  const int lane = threadIdx.x & 31;
  const long long U = (long long)a.B * a.Hkv;
  if (wid >= U * a.R) return;
  const int u = (int)(wid / a.R);
  const int r = (int)(wid % a.R);
  const int b = u / a.Hkv, hk = u % a.Hkv;
  // the unit's real chunks in the weighted index space, and their CTAs
  const long long total = (long long)a.Hkv * sPrefix[a.B];
  const int ext = sPrefix[b + 1] - sPrefix[b];
  const long long first = (long long)a.Hkv * sPrefix[b] + (long long)hk * ext + a.seg_cost;
  const long long last = (long long)a.Hkv * sPrefix[b] + (long long)(hk + 1) * ext - 1;
  const int c0 = cta_of_chunk(first, total, a.grid);
  const int c1 = cta_of_chunk(last, total, a.grid);
  if (c0 >= c1) return;  // one CTA covered the unit and wrote out directly
  const int n = c1 - c0 + 1;
  // CTAs whose chunk range came out empty wrote no partial: weight 0
  const bool all_full = total >= a.grid;
  auto lse_of = [&](int j) -> float {
    const int c = c0 + j;
    if (!all_full && total * c / a.grid >= total * (c + 1) / a.grid) return -INFINITY;
    return a.part_lse[((size_t)c + u) * a.R + r];
  };

  const size_t stride = (size_t)a.R * D;  // between the partial rows of consecutive CTAs
  const float* base = a.part_o + ((size_t)(c0 + u) * a.R + r) * D + (size_t)lane * PER;
  auto load_row = [&](int j, float* x) {
    const float* src = base + (size_t)j * stride;
    if (lane < LANES) {
      if constexpr (PER % 4 == 0) {
#pragma unroll
        for (int e = 0; e < PER; e += 4) {
          const float4 v = *reinterpret_cast<const float4*>(src + e);
          x[e] = v.x; x[e + 1] = v.y; x[e + 2] = v.z; x[e + 3] = v.w;
        }
      } else if constexpr (PER == 2) {
        const float2 v = *reinterpret_cast<const float2*>(src);
        x[0] = v.x; x[1] = v.y;
      } else {
        x[0] = src[0];
      }
    } else {
#pragma unroll
      for (int e = 0; e < PER; ++e) x[e] = 0.f;
    }
  };
  // first round trip: the first (up to) four partial rows and every partial's lse
  float x[4][PER];
#pragma unroll
  for (int i = 0; i < 4; ++i) load_row(min(i, n - 1), x[i]);
  const int nl = (n + 31) / 32;   // lse values per lane
  // lse of partial lane (kept: the weights of the first 32 partials need no reload)
  const float l0 = (lane < n) ? lse_of(lane) : -INFINITY;
  float M = l0;
  for (int t = 1; t < nl; ++t)
    if (t * 32 + lane < n) M = fmaxf(M, lse_of(t * 32 + lane));
#pragma unroll
  for (int m = 16; m >= 1; m >>= 1) M = fmaxf(M, __shfl_xor_sync(0xffffffffu, M, m));
  const float Ms = (M == -INFINITY) ? 0.f : M;
  float L = 0.f;
  float acc[PER];
#pragma unroll
  for (int e = 0; e < PER; ++e) acc[e] = 0.f;
  for (int t = 0; t < nl; ++t) {
    const float lt = (t == 0) ? l0 : (t * 32 + lane < n) ? lse_of(t * 32 + lane) : -INFINITY;
    const float w = (lt == -INFINITY) ? 0.f : fast_exp2(lt - Ms);
    L += w;
    const int m = min(32, n - t * 32);
    for (int k = 0; k < m; k += 4) {
      if (t > 0 || k > 0) {
#pragma unroll
        for (int i = 0; i < 4; ++i) load_row(t * 32 + min(k + i, m - 1), x[i]);
      }
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        float wk = __shfl_sync(0xffffffffu, w, min(k + i, m - 1));
        if (k + i >= m) wk = 0.f;   // past the end: a valid row reloaded, weight 0
#pragma unroll
        for (int e = 0; e < PER; ++e) acc[e] += (wk != 0.f) ? wk * x[i][e] : 0.f;
      }
    }
  }
#pragma unroll
  for (int m = 16; m >= 1; m >>= 1) L += __shfl_xor_sync(0xffffffffu, L, m);
  if (lane >= LANES) return;
  const int i = r / a.g;
  const int h = hk * a.g + r % a.g;
  const size_t orow = ((size_t)b * a.T + i) * a.Hq + h;
  const size_t ob = orow * D + (size_t)lane * PER;
  const float inv = (L > 0.f) ? 1.f / L : 0.f;
  if (a.out_lse && lane == 0) a.out_lse[orow] = (L > 0.f) ? Ms + fast_log2(L) : -INFINITY;
  float o[PER];
#pragma unroll
  for (int e = 0; e < PER; ++e) o[e] = acc[e] * inv;
  if (a.out_bf16) {
    __nv_bfloat16* dst = reinterpret_cast<__nv_bfloat16*>(a.out) + ob;
    if constexpr (PER == 8) {
      *reinterpret_cast<uint4*>(dst) = make_uint4(pack_bf16(o[0], o[1]), pack_bf16(o[2], o[3]),
                                                  pack_bf16(o[4], o[5]), pack_bf16(o[6], o[7]));
    } else if constexpr (PER == 4) {
      *reinterpret_cast<uint2*>(dst) = make_uint2(pack_bf16(o[0], o[1]), pack_bf16(o[2], o[3]));
    } else if constexpr (PER == 2) {
      *reinterpret_cast<uint32_t*>(dst) = pack_bf16(o[0], o[1]);
    } else {
      dst[0] = __float2bfloat16_rn(o[0]);
    }
  } else {
    float* dst = reinterpret_cast<float*>(a.out) + ob;
    if constexpr (PER % 4 == 0) {
#pragma unroll
      for (int e = 0; e < PER; e += 4)
        *reinterpret_cast<float4*>(dst + e) = make_float4(o[e], o[e + 1], o[e + 2], o[e + 3]);
    } else if constexpr (PER == 2) {
      *reinterpret_cast<float2*>(dst) = make_float2(o[0], o[1]);
    } else {
      dst[0] = o[0];
    }
  }
}

// Dynamic shared memory of the merge kernel: the chunk prefix and the scan's
// per-warp scratch.
inline size_t combine_smem(int B) { return (size_t)(B + 1 + 8) * sizeof(int); }

// ---------------------------------------------------------------- host side
inline int d_index(int D) {
  return D == 16 ? 0 : D == 32 ? 1 : D == 64 ? 2 : D == 128 ? 3 : D == 256 ? 4 : -1;
}

// Per (D, row config): the contexts in which the shared-memory opt-in was set.
template <typename T, bool PAGED>
PerContextOnce& smem_attr_once(int di, int cfg) {
  static PerContextOnce once[5][12];
  return once[di][cfg];
}

// One launch of the split kernel with `groups` CTAs of the split per block
// (2 when the configuration is one of two CTAs per SM and both groups' shared
// memory fits a block, else 1).
template <typename T, int D, int RPW, int NTW, bool PAGED, int GROUPS>
cudaError_t launch_groups(const DecodeArgs& a, int nrg, int cfg_idx, cudaStream_t st) {
  using S = Smem<T, D, RPW, NTW>;
  const int ncw = nrg * NTW;
  const size_t smem = S::total(ncw, a.B, GROUPS);
  if (smem > 227 * 1024) return cudaErrorNotSupported;
  auto kern = decode_kernel<T, D, RPW, NTW, PAGED, GROUPS>;
  cudaError_t e = smem_opt_in(reinterpret_cast<const void*>(kern), 227 * 1024,
                              smem_attr_once<T, PAGED>(d_index(D), cfg_idx + (GROUPS == 2 ? 6 : 0)));
  if (e != cudaSuccess) return e;
  e = launch_pdl(kern, dim3((a.grid + GROUPS - 1) / GROUPS), dim3(GROUPS * (ncw + 1) * 32), smem,
                 st, a, nrg);
  if (e != cudaSuccess) return e;
  const long long warps = (long long)a.B * a.Hkv * a.R;
  const int cblocks = (int)((warps * 32 + 255) / 256);
  return launch_pdl(combine_kernel<D>, dim3(cblocks), dim3(256), combine_smem(a.B), st, a);
}

// Configurations of up to 4 rows run two CTAs of the split per block while
// both groups' shared memory fits (the per-sequence prefix grows with B).
template <typename T, int D, int RPW, bool PAGED>
cudaError_t launch_paired(const DecodeArgs& a, int cfg_idx, cudaStream_t st) {
  const cudaError_t e = launch_groups<T, D, RPW, 4, PAGED, 2>(a, 1, cfg_idx, st);
  if (e != cudaErrorNotSupported) return e;
  return launch_groups<T, D, RPW, 4, PAGED, 1>(a, 1, cfg_idx, st);
}

template <typename T, int D, bool PAGED>
cudaError_t launch_rows(const DecodeArgs& a, cudaStream_t st) {
  if (a.R <= 1) return launch_paired<T, D, 1, PAGED>(a, 0, st);
  if (a.R <= 2) return launch_paired<T, D, 2, PAGED>(a, 1, st);
  if (a.R <= 4) return launch_paired<T, D, 4, PAGED>(a, 2, st);
  if (a.R <= 8) return launch_groups<T, D, 8, 4, PAGED, 1>(a, 1, 3, st);
  if (a.R <= 16) return launch_groups<T, D, 8, 2, PAGED, 1>(a, 2, 4, st);
  if (a.R <= kMaxRows) return launch_groups<T, D, 8, 1, PAGED, 1>(a, (a.R + 7) / 8, 5, st);
  return cudaErrorNotSupported;
}

}  // namespace

template <typename T, bool PAGED>
cudaError_t launch_decode_t(const DecodeArgs& a, cudaStream_t st) {
  switch (a.D) {
    case 16: return launch_rows<T, 16, PAGED>(a, st);
    case 32: return launch_rows<T, 32, PAGED>(a, st);
    case 64: return launch_rows<T, 64, PAGED>(a, st);
    case 128: return launch_rows<T, 128, PAGED>(a, st);
    case 256:
      if constexpr (sizeof(T) == 2) return launch_rows<T, 256, PAGED>(a, st);
      else return cudaErrorNotSupported;
    default: return cudaErrorNotSupported;
  }
}

}  // namespace kvd

// Tensor-core split-KV decode for bf16, head_dim 128: used when a
// (sequence, kv head) unit has enough query rows (g * q_len) for the QK^T
// and PV products to be dense contractions (multi-token verification, wide
// GQA groups).
//
// What is computed is the same as the CUDA-core kernel (decode_split.cuh):
// ferric-core 0.1.0, examples/generate.rs, `step_gpu` / `mha_decode_t` with
// the causal rule of `cpu::mha_causal` among the new tokens, split along the
// cache ("Flash Decoding", ferrum-sampler 0.7.0 README, Key Optimizations)
// and merged by log-sum-exp in kernel C.
//
// One CTA per SM, 10 warps:
// * warp 8 (TMA): 2-D tensor loads of 16-token K and V boxes (two 64-dim
//   halves each, 128-byte swizzle) into a ring of 64-token stages; page ids
//   come from a prefetched window of the block table;
// * warp 9 (MMA): one thread issues S = Q K^T (M = 64 or 128 query rows,
//   N = 64 tokens, K = 128 dims) into a double-buffered TMEM tile, then
//   O_h += P_h V_h for the two token halves h of the stage into two TMEM
//   accumulators; P is passed as bf16 high part + bf16 residual (two passes
//   over V), which keeps the probabilities to ~16 significant bits;
// * warps 0-7 (softmax): warpgroup h (warps 4h .. 4h+3) owns tokens
//   32h .. 32h+31 of every stage; thread (warp, lane) owns one query row of
//   the unit (rows spread over the four TMEM sub-partitions).  It reads its S
//   row from TMEM, masks, keeps a reference max raised only when the running
//   max grows by more than 2^8 (then its O row is rescaled in TMEM), and
//   writes its probabilities into a swizzled shared tile for the PV product.
//   At a unit boundary the two halves are merged by log-sum-exp and the
//   output (or a normalised partial) is written.
// The work split over units and CTAs is the one of the CUDA-core kernel, so
// the same merge kernel finishes split units.
#include <cuda.h>
#include <cudaTypedefs.h>

#include <mutex>

#include "decode_split.cuh"
#include "kvd_tc.cuh"

namespace kvd {
namespace {

constexpr int TC_D = 128;
constexpr int TC_STAGE = 64;                      // tokens per stage
constexpr int TC_HALF = TC_STAGE / 2;             // tokens per softmax warpgroup
constexpr int TC_CHUNKS = TC_STAGE / kChunk;      // 16-token boxes per stage
constexpr int TC_THREADS = 320;                   // 8 softmax warps + TMA + MMA
constexpr int TC_SOFTMAX_THREADS = 256;
constexpr int WARP_TMA = 8, WARP_MMA = 9;
constexpr uint32_t TC_TMEM_COLS = 512;            // S0 | S1 | O_0 | O_1
constexpr uint32_t COL_S = 0, COL_O = 128;
constexpr float kRescaleThreshold = 8.0f;         // log2 units

// M = MMA rows (query rows of a unit, padded): 64 or 128.
template <int M>
struct TcSmem {
  static constexpr int NS = M == 128 ? 3 : 4;          // ring depth (shared memory bound)
  static constexpr int HALF_Q = M * 128;               // M rows x 64 dims
  static constexpr int Q = 0;                          // 2 halves
  static constexpr int KV = Q + 2 * HALF_Q;            // ring
  static constexpr int K_HALF = TC_STAGE * 128;        // 8 KB: 64 tokens x 64 dims
  static constexpr int STAGE = 4 * K_HALF;             // K (2 halves) + V (2 halves)
  static constexpr int P = KV + NS * STAGE;            // 2 buffers x (hi, lo) x [M rows x 64 tokens]
  static constexpr int P_BUF = M * 128;
  static constexpr int BAR = P + 4 * P_BUF;
  static constexpr int NBAR = 2 * NS + 10;
  static constexpr int TMEM_SLOT = BAR + NBAR * 8;
  static constexpr int ML = TMEM_SLOT + 16;            // [2][M] x (m, l) for the epilogue merge
  static constexpr int SCRATCH = ML + 2 * M * 8;       // one int per warp for the scan
  static constexpr int PREFIX = SCRATCH + 64;
  static size_t bytes(int B) { return (size_t)PREFIX + (size_t)(B + 1) * 4 + 1024; }
};

template <bool PAGED, int M>
__global__ void __launch_bounds__(TC_THREADS, 1)
    decode_tc_kernel(const DecodeArgs a, const __grid_constant__ CUtensorMap tmk,
                     const __grid_constant__ CUtensorMap tmv) {
  using S = TcSmem<M>;
  extern __shared__ unsigned char smem_raw[];
  unsigned char* smem = smem_raw + ((1024u - (smem_u32(smem_raw) & 1023u)) & 1023u);
  unsigned char* sQ = smem + S::Q;
  unsigned char* sKV = smem + S::KV;
  unsigned char* sP = smem + S::P;
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + S::BAR);
  uint64_t* full = bars;                  // TMA -> MMA (+ softmax on short stages)
  uint64_t* empty = bars + S::NS;         // PV done -> TMA
  uint64_t* s_full = bars + 2 * S::NS;    // QK done -> softmax
  uint64_t* s_free = s_full + 2;          // S read -> MMA
  uint64_t* p_full = s_free + 2;          // P written -> MMA
  uint64_t* p_free = p_full + 2;          // PV done -> softmax
  uint64_t* q_full = p_free + 2;          // Q written -> MMA
  uint64_t* mma_done = q_full + 1;        // all issued MMAs complete (exit)
  uint32_t* sTmem = reinterpret_cast<uint32_t*>(smem + S::TMEM_SLOT);
  float2* sML = reinterpret_cast<float2*>(smem + S::ML);
  int* sScratch = reinterpret_cast<int*>(smem + S::SCRATCH);
  int* sPrefix = reinterpret_cast<int*>(smem + S::PREFIX);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;

  {  // stale ring contents must be finite: start from zeros
    uint4* z = reinterpret_cast<uint4*>(sKV);
    for (int k = threadIdx.x; k < S::NS * S::STAGE / 16; k += blockDim.x)
      z[k] = make_uint4(0, 0, 0, 0);
  }
  if (threadIdx.x == 0) {
    for (int s = 0; s < S::NS; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], 1);
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(&s_full[b], 1);
      mbar_init(&s_free[b], 8);
      mbar_init(&p_full[b], 8);
      mbar_init(&p_free[b], 1);
    }
    mbar_init(q_full, 8);
    mbar_init(mma_done, 1);
  }
  if (warp == WARP_MMA) {
    tmem_alloc(sTmem, TC_TMEM_COLS);
    tmem_relinquish();
  }
  if (warp == WARP_TMA && lane == 0) {
    prefetch_tensormap(&tmk);
    prefetch_tensormap(&tmv);
  }
  chunk_prefix_scan(a, sPrefix, sScratch);
  fence_barrier_init();
  fence_proxy_async_smem();
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *sTmem;

  const long long total = (long long)a.Hkv * sPrefix[a.B];
  if (blockIdx.x == 0 && threadIdx.x == 0) *a.total_chunks = total;
  const long long x0 = total * blockIdx.x / a.grid;
  const long long x1 = total * (blockIdx.x + 1) / a.grid;

  if (x0 < x1) {
    const SegState st = locate_chunk(a, sPrefix, x0);
    if (warp == WARP_TMA) {
      // ============================ TMA warp ===============================
      int g = 0;
      bool failed = false;
      SegState c = st;
      // page id of chunk `ch` of sequence b (paged layout), -1 past `kend`
      auto page_of = [&](int b, int ch, int kend) -> int {
        if (ch >= kend) return -1;
        return a.block_table[(size_t)b * a.max_pages_per_seq + (ch * kChunk) / a.page_size];
      };
      while (c.x < x1 && !failed) {
        const int nb = sPrefix[c.b + 1] - sPrefix[c.b];
        const int kend = (int)min((long long)nb, c.k0 + (x1 - c.x));
        // two 32-chunk windows of page ids, the second one loaded 8 stages ahead of use
        int wbase = c.k0, win0 = -1, win1 = -1;
        if (PAGED) {
          win0 = page_of(c.b, wbase + lane, kend);
          win1 = page_of(c.b, wbase + 32 + lane, kend);
        }
        for (int kk = c.k0; kk < kend; kk += TC_CHUNKS, ++g) {
          if (PAGED && kk - wbase >= 32) {
            wbase += 32;
            win0 = win1;
            win1 = page_of(c.b, wbase + 32 + lane, kend);
          }
          const int slot = g % S::NS;
          int ok = 1;
          if (lane == 0) ok = mbar_wait(&empty[slot], ((uint32_t)(g / S::NS) & 1u) ^ 1u, a.status);
          ok = __shfl_sync(0xffffffffu, ok, 0);
          if (!ok) { failed = true; break; }
          const int nck = min(TC_CHUNKS, kend - kk);
          int page = -1;
          if (PAGED) page = __shfl_sync(0xffffffffu, win0, kk - wbase + min(lane, TC_CHUNKS - 1));
          int row = -1;
          if (lane < nck) {
            const int tc = (kk + lane) * kChunk;
            if (!PAGED) {
              row = (int)(((long long)c.b * a.Hkv + c.hk) * a.max_seq_len + tc);
            } else if (page >= 0 && page < a.num_pages) {
              row = (int)(((long long)page * a.Hkv + c.hk) * a.page_size + tc % a.page_size);
            } else if (a.status) {
              atomicOr(a.status, KVD_FLAG_PAGE_OUT_OF_RANGE);
            }
          }
          uint32_t bytes = row >= 0 ? 4u * kChunk * 128u : 0u;  // K and V, two halves each
#pragma unroll
          for (int m = 16; m >= 1; m >>= 1) bytes += __shfl_xor_sync(0xffffffffu, bytes, m);
          if (lane == 0) mbar_arrive_expect_tx(&full[slot], bytes);
          __syncwarp();
          if (row >= 0) {
            unsigned char* dk = sKV + slot * S::STAGE + lane * kChunk * 128;
            unsigned char* dv = dk + 2 * S::K_HALF;
            tma_load_2d(dk, &tmk, 0, row, &full[slot]);
            tma_load_2d(dk + S::K_HALF, &tmk, 64, row, &full[slot]);
            tma_load_2d(dv, &tmv, 0, row, &full[slot]);
            tma_load_2d(dv + S::K_HALF, &tmv, 64, row, &full[slot]);
          }
          __syncwarp();
        }
        c.x += kend - c.k0;
        c.k0 = 0;
        if (++c.hk == a.Hkv) { c.hk = 0; ++c.b; }
      }
      if (lane == 0) {  // every issued copy lands before the CTA may exit
        for (int k = max(0, g - S::NS); k < g; ++k)
          if (!mbar_wait(&full[k % S::NS], (uint32_t)(k / S::NS) & 1u, a.status)) break;
      }
    } else if (warp == WARP_MMA) {
      // ============================ MMA warp ===============================
      if (lane == 0) {
        constexpr uint32_t idesc_qk = idesc_bf16_f32(M, TC_STAGE, false);
        constexpr uint32_t idesc_pv = idesc_bf16_f32(M, TC_D, true);
        // descriptors of the tile bases; a byte offset b inside a tile adds b >> 4
        const uint64_t dq = sw128_desc(smem_u32(sQ), 16, 1024);
        const uint64_t dkv = sw128_desc(smem_u32(sKV), 16, 1024);
        const uint64_t dp = sw128_desc(smem_u32(sP), 16, 1024);
        const uint64_t dv = sw128_desc(smem_u32(sKV), S::K_HALF, 1024);
        int g = 0, seg = 0;
        bool failed = false;
        // S = Q K^T for global stage gg into S buffer gg % 2
        auto issue_qk = [&](int gg) -> bool {
          const int slot = gg % S::NS;
          if (!mbar_wait(&full[slot], (uint32_t)(gg / S::NS) & 1u, a.status)) return false;
          if (!mbar_wait(&s_free[gg & 1], ((uint32_t)(gg >> 1) & 1u) ^ 1u, a.status)) return false;
          tc_fence_after();
          const uint32_t kofs = (uint32_t)slot * S::STAGE;
#pragma unroll
          for (int ks = 0; ks < TC_D / 16; ++ks) {
            const uint32_t off = (uint32_t)(ks & 3) * 32u;  // 16 dims = 32 bytes inside the row
            tc_mma_bf16(tmem + COL_S + (uint32_t)(gg & 1) * TC_STAGE,
                        dq + (((ks >> 2) * S::HALF_Q + off) >> 4),
                        dkv + ((kofs + (ks >> 2) * S::K_HALF + off) >> 4), idesc_qk, ks > 0);
          }
          tc_commit(&s_full[gg & 1]);
          return true;
        };
        SegState c = st;
        while (c.x < x1 && !failed) {
          const int nb = sPrefix[c.b + 1] - sPrefix[c.b];
          const int kend = (int)min((long long)nb, c.k0 + (x1 - c.x));
          const int n = (kend - c.k0 + TC_CHUNKS - 1) / TC_CHUNKS;
          if (!mbar_wait(q_full, (uint32_t)seg & 1u, a.status)) { failed = true; break; }
          tc_fence_after();
          if (!issue_qk(g)) { failed = true; break; }
          for (int k = 0; k < n; ++k) {
            const int gg = g + k;
            if (k + 1 < n && !issue_qk(gg + 1)) { failed = true; break; }
            if (!mbar_wait(&p_full[gg & 1], (uint32_t)(gg >> 1) & 1u, a.status)) { failed = true; break; }
            tc_fence_after();
            const uint32_t vofs = (uint32_t)(gg % S::NS) * S::STAGE + 2 * S::K_HALF;
            // token half h of the stage goes to accumulator O_h; P = P_hi + P_lo
#pragma unroll
            for (int h = 0; h < 2; ++h)
#pragma unroll
              for (int part = 0; part < 2; ++part) {
                const uint32_t pofs = (uint32_t)((gg & 1) * 2 + part) * S::P_BUF;
#pragma unroll
                for (int ks = 2 * h; ks < 2 * h + 2; ++ks)
                  tc_mma_bf16(tmem + COL_O + (uint32_t)h * TC_D, dp + ((pofs + ks * 32u) >> 4),
                              dv + ((vofs + ks * 2048u) >> 4), idesc_pv,
                              (k > 0 || part > 0 || ks > 2 * h) ? 1u : 0u);
              }
            tc_commit(&empty[gg % S::NS]);
            tc_commit(&p_free[gg & 1]);
          }
          g += n;
          ++seg;
          c.x += kend - c.k0;
          c.k0 = 0;
          if (++c.hk == a.Hkv) { c.hk = 0; ++c.b; }
        }
        // every MMA this thread issued completes before the CTA frees TMEM
        tc_commit(mma_done);
        mbar_wait(mma_done, 0, a.status);
      }
      __syncwarp();
    } else {
      // ========================= softmax warps 0-7 =========================
      // Sub-partition sp = warp % 4 reaches TMEM lanes 32 sp .. 32 sp + 31.
      // M = 128: lane l there is tile row 32 sp + l; M = 64: lanes 0-15 hold
      // tile rows 16 sp + l.  Tile row p holds query row qr = 4 l + sp, so the
      // real rows of a small group spread over all four sub-partitions.
      constexpr int RPT = M / 4;                            // tile rows per sub-partition
      const int sp = warp & 3;
      const int hw = warp >> 2;                              // token half of the stage
      const bool lane_row = lane < RPT;
      const int p = sp * RPT + lane;                         // tile row (if lane_row)
      const int qr = 4 * lane + sp;
      const int tid = threadIdx.x;                           // 0 .. 255
      const uint32_t t_lane = tmem + ((uint32_t)(sp * 32) << 16);
      const uint32_t col_o = COL_O + (uint32_t)hw * TC_D;
      const bool row_ok = lane_row && qr < a.R;
      const bool warp_rows = sp < a.R;                       // any real row in this warp
      const int di = row_ok ? qr / a.g : 0;                  // new-token index of the row
      int g = 0, seg = 0;
      bool failed = false;
      SegState c = st;
      while (c.x < x1) {
        const int nb = sPrefix[c.b + 1] - sPrefix[c.b];
        const int Nb = attended_len(a, c.b, false);
        const int Lb = Nb - a.T;
        const int kend = (int)min((long long)nb, c.k0 + (x1 - c.x));
        const int n = (kend - c.k0 + TC_CHUNKS - 1) / TC_CHUNKS;
        const int u = c.b * a.Hkv + c.hk;
        const int vis = row_ok ? Lb + di + 1 : 0;            // visible tokens of this row

        // -- query row qr, dims 64 hw .. 64 hw + 63, into tile row p (zeros for padding)
        if (lane_row) {
          const int h = c.hk * a.g + (row_ok ? qr % a.g : 0);
          const uint4* src = reinterpret_cast<const uint4*>(
              reinterpret_cast<const __nv_bfloat16*>(a.q) + (((size_t)c.b * a.T + di) * a.Hq + h) * TC_D);
#pragma unroll
          for (int ch = 0; ch < 8; ++ch) {
            const uint4 v = row_ok ? src[hw * 8 + ch] : make_uint4(0, 0, 0, 0);
            *reinterpret_cast<uint4*>(sQ + hw * S::HALF_Q + p * 128 + ((ch ^ (p & 7)) << 4)) = v;
          }
        }
        fence_proxy_async_smem();
        __syncwarp();
        if (lane == 0) mbar_arrive(q_full);

        float m = -INFINITY, l = 0.f;
        for (int k = 0; k < n; ++k) {
          const int gg = g + k;
          const int slot = gg % S::NS;
          const int t0 = (c.k0 + k * TC_CHUNKS) * kChunk;
          const int nvalid = min(min(TC_CHUNKS, kend - c.k0 - k * TC_CHUNKS) * kChunk, Nb - t0);
          const bool tail = (nvalid < TC_STAGE) || (t0 + TC_STAGE > Lb + 1);
          if (!failed && !mbar_wait(&s_full[gg & 1], (uint32_t)(gg >> 1) & 1u, a.status)) failed = true;
          tc_fence_after();
          float x[TC_HALF];
          {
            uint32_t sr[32];
            tmem_ld32(t_lane + COL_S + (uint32_t)(gg & 1) * TC_STAGE + hw * TC_HALF, sr);
            tmem_ld_wait();
#pragma unroll
            for (int j = 0; j < TC_HALF; ++j) x[j] = __uint_as_float(sr[j]) * a.qscale;
          }
          tc_fence_before();
          __syncwarp();
          if (lane == 0) mbar_arrive(&s_free[gg & 1]);

          float mx4[4] = {-INFINITY, -INFINITY, -INFINITY, -INFINITY};
#pragma unroll
          for (int j = 0; j < TC_HALF; ++j) {
            const int tj = hw * TC_HALF + j;                 // token of the stage
            if (!row_ok || (tail && (tj >= nvalid || t0 + tj >= vis))) x[j] = -INFINITY;
            mx4[j & 3] = fmaxf(mx4[j & 3], x[j]);
          }
          const float mx = fmaxf(fmaxf(mx4[0], mx4[1]), fmaxf(mx4[2], mx4[3]));
          float alpha = 1.f;
          bool rescale = false;
          if (mx > m + kRescaleThreshold) {   // raise the reference max only on a large jump
            if (m != -INFINITY) {
              alpha = fast_exp2(m - mx);
              rescale = true;
            }
            m = mx;
            l *= alpha;
          }
          uint32_t pk[TC_HALF / 2], pl[TC_HALF / 2];   // bf16 pairs: high part, residual
          if (warp_rows) {
            float ps4[4] = {0.f, 0.f, 0.f, 0.f};
            const float mref = (m == -INFINITY) ? 0.f : m;
#pragma unroll
            for (int j = 0; j < TC_HALF; j += 2) {
              const float p0 = fast_exp2(x[j] - mref), p1 = fast_exp2(x[j + 1] - mref);
              ps4[(j >> 1) & 3] += p0 + p1;
              const uint32_t hi = pack_bf16x2(p0, p1);
              pk[j / 2] = hi;
              pl[j / 2] = pack_bf16x2(p0 - __uint_as_float(hi << 16), p1 - __uint_as_float(hi & 0xffff0000u));
            }
            l += (ps4[0] + ps4[1]) + (ps4[2] + ps4[3]);
          } else {
#pragma unroll
            for (int j = 0; j < TC_HALF / 2; ++j) { pk[j] = 0u; pl[j] = 0u; }
          }

          // P buffer (gg & 1) is free once PV(gg - 2) completed
          if (!failed && !mbar_wait(&p_free[gg & 1], ((uint32_t)(gg >> 1) & 1u) ^ 1u, a.status)) failed = true;
          if (__any_sync(0xffffffffu, rescale)) {
            // O_hw must hold PV(gg - 1) before it is scaled in place
            if (!failed && !mbar_wait(&p_free[(gg - 1) & 1], (uint32_t)((gg - 1) >> 1) & 1u, a.status))
              failed = true;
            tc_fence_after();
#pragma unroll
            for (int cb = 0; cb < TC_D / 32; ++cb) {
              uint32_t o[32];
              tmem_ld32(t_lane + col_o + cb * 32, o);
              tmem_ld_wait();
#pragma unroll
              for (int j = 0; j < 32; ++j) o[j] = __float_as_uint(__uint_as_float(o[j]) * alpha);
              tmem_st32(t_lane + col_o + cb * 32, o);
            }
            tmem_st_wait();
          }
          if (lane_row) {
            // tokens 32 hw .. 32 hw + 31 = 16-byte chunks 4 hw .. 4 hw + 3 of the row
            unsigned char* prow = sP + ((gg & 1) * 2) * S::P_BUF + p * 128;
#pragma unroll
            for (int ch = 0; ch < 4; ++ch) {
              const int cc = hw * 4 + ch;
              *reinterpret_cast<uint4*>(prow + ((cc ^ (p & 7)) << 4)) =
                  make_uint4(pk[4 * ch], pk[4 * ch + 1], pk[4 * ch + 2], pk[4 * ch + 3]);
              *reinterpret_cast<uint4*>(prow + S::P_BUF + ((cc ^ (p & 7)) << 4)) =
                  make_uint4(pl[4 * ch], pl[4 * ch + 1], pl[4 * ch + 2], pl[4 * ch + 3]);
            }
          }
          if (nvalid < TC_STAGE) {
            // rows past the valid tokens hold whatever the cache held there: zero them in V
            if (!failed && !mbar_wait(&full[slot], (uint32_t)(gg / S::NS) & 1u, a.status)) failed = true;
            unsigned char* vbase = sKV + slot * S::STAGE + 2 * S::K_HALF;
            const int nz = (TC_STAGE - nvalid) * 8;  // 16-byte pieces per half
            for (int e = tid; e < 2 * nz; e += TC_SOFTMAX_THREADS) {
              const int hh = e / nz, q = e % nz;
              *reinterpret_cast<uint4*>(vbase + hh * S::K_HALF + nvalid * 128 + q * 16) =
                  make_uint4(0, 0, 0, 0);
            }
          }
          fence_proxy_async_smem();
          tc_fence_before();
          __syncwarp();
          if (lane == 0) mbar_arrive(&p_full[gg & 1]);
        }

        // -- unit segment done: merge the two token halves, write the row
        const int gl = g + n - 1;
        if (!failed && !mbar_wait(&p_free[gl & 1], (uint32_t)(gl >> 1) & 1u, a.status)) failed = true;
        tc_fence_after();
        if (lane_row) sML[hw * M + p] = make_float2(m, l);
        named_bar_sync(1, TC_SOFTMAX_THREADS);
        float2 mo = make_float2(-INFINITY, 0.f);
        if (lane_row) mo = sML[(1 - hw) * M + p];
        const float m0 = hw == 0 ? m : mo.x, l0 = hw == 0 ? l : mo.y;
        const float m1 = hw == 0 ? mo.x : m, l1 = hw == 0 ? mo.y : l;
        const float mm = fmaxf(m0, m1);
        const float ms = (mm == -INFINITY) ? 0.f : mm;
        const float w0 = fast_exp2(m0 - ms), w1 = fast_exp2(m1 - ms);
        const float L = w0 * l0 + w1 * l1;
        const float inv = (L > 0.f) ? 1.f / L : 0.f;
        const float s0 = w0 * inv, s1 = w1 * inv;
        const bool whole = (c.k0 == 0) && (kend == nb);
        const long long slot_idx = (long long)blockIdx.x + u;
        const int h = c.hk * a.g + (row_ok ? qr % a.g : 0);
        // warpgroup hw writes dims 64 hw .. 64 hw + 63 of the row
#pragma unroll
        for (int cb = 0; cb < 2; ++cb) {
          const int d0 = hw * 64 + cb * 32;
          uint32_t o0[32], o1[32];
          tmem_ld32(t_lane + COL_O + d0, o0);
          tmem_ld32(t_lane + COL_O + TC_D + d0, o1);
          tmem_ld_wait();
          float ov[32];
#pragma unroll
          for (int j = 0; j < 32; ++j) ov[j] = __uint_as_float(o0[j]) * s0 + __uint_as_float(o1[j]) * s1;
          if (row_ok) {
            if (whole) {
              const size_t ob = (((size_t)c.b * a.T + di) * a.Hq + h) * TC_D + d0;
              if (a.out_bf16) {
                uint4* dst = reinterpret_cast<uint4*>(reinterpret_cast<__nv_bfloat16*>(a.out) + ob);
#pragma unroll
                for (int q4 = 0; q4 < 4; ++q4)
                  dst[q4] = make_uint4(pack_bf16x2(ov[8 * q4], ov[8 * q4 + 1]), pack_bf16x2(ov[8 * q4 + 2], ov[8 * q4 + 3]),
                                       pack_bf16x2(ov[8 * q4 + 4], ov[8 * q4 + 5]), pack_bf16x2(ov[8 * q4 + 6], ov[8 * q4 + 7]));
              } else {
                float4* dst = reinterpret_cast<float4*>(reinterpret_cast<float*>(a.out) + ob);
#pragma unroll
                for (int q4 = 0; q4 < 8; ++q4)
                  dst[q4] = make_float4(ov[4 * q4], ov[4 * q4 + 1], ov[4 * q4 + 2], ov[4 * q4 + 3]);
              }
            } else {
              float4* dst = reinterpret_cast<float4*>(a.part_o + ((size_t)slot_idx * a.R + qr) * TC_D + d0);
#pragma unroll
              for (int q4 = 0; q4 < 8; ++q4)
                dst[q4] = make_float4(ov[4 * q4], ov[4 * q4 + 1], ov[4 * q4 + 2], ov[4 * q4 + 3]);
            }
          }
        }
        if (row_ok && !whole && hw == 0)
          a.part_lse[(size_t)slot_idx * a.R + qr] = (L > 0.f) ? ms + fast_log2(L) : -INFINITY;
        if (threadIdx.x == 0) {
          if (c.k0 == 0) a.unit_ctas[u].x = blockIdx.x;
          if (kend == nb) a.unit_ctas[u].y = blockIdx.x;
        }
        tc_fence_before();  // the O reads above precede the next segment's first PV
        named_bar_sync(1, TC_SOFTMAX_THREADS);   // sML is reused by the next segment

        g += n;
        ++seg;
        c.x += kend - c.k0;
        c.k0 = 0;
        if (++c.hk == a.Hkv) { c.hk = 0; ++c.b; }
      }
    }
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == WARP_MMA) tmem_dealloc(tmem, TC_TMEM_COLS);
}

// ---------------------------------------------------------------- host side
PFN_cuTensorMapEncodeTiled_v12000 encode_fn() {
  static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(p);
  });
  return fn;
}

// 2-D map over the cache seen as [rows, 128] bf16; box = 16 rows x 64 dims,
// 128-byte swizzle (the MMA operand layout).
bool make_map(CUtensorMap* map, const void* base, unsigned long long rows) {
  auto fn = encode_fn();
  if (!fn) return false;
  cuuint64_t dims[2] = {(cuuint64_t)TC_D, (cuuint64_t)rows};
  cuuint64_t strides[1] = {(cuuint64_t)TC_D * 2};
  cuuint32_t box[2] = {64, (cuuint32_t)kChunk};
  cuuint32_t estr[2] = {1, 1};
  const CUresult r = fn(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(base), dims,
                        strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
                        CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                        CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

template <bool PAGED, int M>
cudaError_t launch_tc(const DecodeArgs& a, cudaStream_t st) {
  const unsigned long long rows =
      PAGED ? (unsigned long long)a.num_pages * a.Hkv * a.page_size
            : (unsigned long long)a.B * a.Hkv * a.max_seq_len;
  if (rows >= (1ull << 31)) return cudaErrorNotSupported;  // TMA row coordinate is int32
  CUtensorMap mk, mv;
  if (!make_map(&mk, a.k_cache, rows) || !make_map(&mv, a.v_cache, rows)) return cudaErrorNotSupported;
  const size_t smem = TcSmem<M>::bytes(a.B);
  if (smem > 227 * 1024) return cudaErrorNotSupported;
  static std::atomic<unsigned long long> attr_done{0};
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  const unsigned long long bit = 1ull << (dev & 63);
  if (!(attr_done.load() & bit)) {
    e = cudaFuncSetAttribute(decode_tc_kernel<PAGED, M>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             227 * 1024);
    if (e != cudaSuccess) return e;
    attr_done.fetch_or(bit);
  }
  decode_tc_kernel<PAGED, M><<<a.grid, TC_THREADS, smem, st>>>(a, mk, mv);
  e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  const long long warps = (long long)a.B * a.Hkv * a.R;
  combine_kernel<TC_D><<<(int)((warps * 32 + 255) / 256), 256, 0, st>>>(a);
  return cudaGetLastError();
}

}  // namespace

cudaError_t launch_decode_tc(const DecodeArgs& a, cudaStream_t st) {
  if (a.R <= 64) return a.block_table ? launch_tc<true, 64>(a, st) : launch_tc<false, 64>(a, st);
  return a.block_table ? launch_tc<true, 128>(a, st) : launch_tc<false, 128>(a, st);
}

}  // namespace kvd

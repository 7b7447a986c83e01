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
// One CTA per SM, 6 warps:
// * warp 4 (TMA): 2-D tensor loads of 16-token K and V boxes (two 64-dim
//   halves each, 128-byte swizzle) into a 4-stage ring of 64-token stages;
// * warp 5 (MMA): one thread issues S = Q K^T (M = 128 query rows padded,
//   N = 64 tokens, K = 128 dims) into a double-buffered TMEM tile, then
//   O += P V (M = 128, N = 128 dims, K = 64 tokens) into a TMEM accumulator;
// * warps 0-3 (softmax): thread r owns query row r: reads its S row from
//   TMEM, masks, keeps a running max that is only raised when it grows by
//   more than 2^8 (the accumulator is rescaled in TMEM only then), writes its
//   probabilities as bf16 into a swizzled shared tile for the PV product, and
//   at a unit boundary reads its O row back and writes the output or a
//   normalised partial (o, lse).
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
constexpr int TC_CHUNKS = TC_STAGE / kChunk;      // 16-token boxes per stage
constexpr int TC_NS = 4;                          // ring depth
constexpr int TC_ROWS = 128;                      // MMA M (query rows, padded)
constexpr int TC_THREADS = 192;
constexpr uint32_t TC_TMEM_COLS = 256;            // S0 | S1 | O
constexpr uint32_t COL_S = 0, COL_O = 128;
constexpr float kRescaleThreshold = 8.0f;         // log2 units

struct TcSmem {
  static constexpr int HALF_Q = TC_ROWS * 128;        // 16 KB: 128 rows x 64 dims
  static constexpr int Q = 0;                          // 2 halves
  static constexpr int KV = Q + 2 * HALF_Q;            // ring
  static constexpr int K_HALF = TC_STAGE * 128;        // 8 KB: 64 tokens x 64 dims
  static constexpr int STAGE = 4 * K_HALF;             // K (2 halves) + V (2 halves)
  static constexpr int P = KV + TC_NS * STAGE;         // 2 x [128 rows x 64 tokens]
  static constexpr int P_BUF = TC_ROWS * 128;
  static constexpr int BAR = P + 2 * P_BUF;
  static constexpr int NBAR = 2 * TC_NS + 10;
  static constexpr int TMEM_SLOT = BAR + NBAR * 8;
  static constexpr int SCRATCH = TMEM_SLOT + 16;       // 8 ints for the scan
  static constexpr int PREFIX = SCRATCH + 32;
  static size_t bytes(int B) { return (size_t)PREFIX + (size_t)(B + 1) * 4 + 1024; }
};

template <bool PAGED>
__global__ void __launch_bounds__(TC_THREADS, 1)
    decode_tc_kernel(const DecodeArgs a, const __grid_constant__ CUtensorMap tmk,
                     const __grid_constant__ CUtensorMap tmv) {
  extern __shared__ unsigned char smem_raw[];
  unsigned char* smem = smem_raw + ((1024u - (smem_u32(smem_raw) & 1023u)) & 1023u);
  unsigned char* sQ = smem + TcSmem::Q;
  unsigned char* sKV = smem + TcSmem::KV;
  unsigned char* sP = smem + TcSmem::P;
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + TcSmem::BAR);
  uint64_t* full = bars;                  // TMA -> MMA (+ softmax on tail stages)
  uint64_t* empty = bars + TC_NS;         // PV done -> TMA
  uint64_t* s_full = bars + 2 * TC_NS;    // QK done -> softmax
  uint64_t* s_free = s_full + 2;          // S read -> MMA
  uint64_t* p_full = s_free + 2;          // P written -> MMA
  uint64_t* p_free = p_full + 2;          // PV done -> softmax
  uint64_t* q_full = p_free + 2;          // Q written -> MMA
  uint64_t* mma_done = q_full + 1;        // all issued MMAs complete (exit)
  uint32_t* sTmem = reinterpret_cast<uint32_t*>(smem + TcSmem::TMEM_SLOT);
  int* sScratch = reinterpret_cast<int*>(smem + TcSmem::SCRATCH);
  int* sPrefix = reinterpret_cast<int*>(smem + TcSmem::PREFIX);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;

  {  // stale ring contents must be finite: start from zeros
    uint4* z = reinterpret_cast<uint4*>(sKV);
    for (int k = threadIdx.x; k < TC_NS * TcSmem::STAGE / 16; k += blockDim.x)
      z[k] = make_uint4(0, 0, 0, 0);
  }
  if (threadIdx.x == 0) {
    for (int s = 0; s < TC_NS; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], 1);
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(&s_full[b], 1);
      mbar_init(&s_free[b], 4);
      mbar_init(&p_full[b], 4);
      mbar_init(&p_free[b], 1);
    }
    mbar_init(q_full, 4);
    mbar_init(mma_done, 1);
  }
  if (warp == 5) {
    tmem_alloc(sTmem, TC_TMEM_COLS);
    tmem_relinquish();
  }
  if (warp == 4 && lane == 0) {
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
    if (warp == 4) {
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
          const int slot = g % TC_NS;
          int ok = 1;
          if (lane == 0) ok = mbar_wait(&empty[slot], ((uint32_t)(g / TC_NS) & 1u) ^ 1u, a.status);
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
            unsigned char* dk = sKV + slot * TcSmem::STAGE + lane * kChunk * 128;
            unsigned char* dv = dk + 2 * TcSmem::K_HALF;
            tma_load_2d(dk, &tmk, 0, row, &full[slot]);
            tma_load_2d(dk + TcSmem::K_HALF, &tmk, 64, row, &full[slot]);
            tma_load_2d(dv, &tmv, 0, row, &full[slot]);
            tma_load_2d(dv + TcSmem::K_HALF, &tmv, 64, row, &full[slot]);
          }
          __syncwarp();
        }
        c.x += kend - c.k0;
        c.k0 = 0;
        if (++c.hk == a.Hkv) { c.hk = 0; ++c.b; }
      }
      if (lane == 0) {  // every issued copy lands before the CTA may exit
        for (int k = max(0, g - TC_NS); k < g; ++k)
          if (!mbar_wait(&full[k % TC_NS], (uint32_t)(k / TC_NS) & 1u, a.status)) break;
      }
    } else if (warp == 5) {
      // ============================ MMA warp ===============================
      if (lane == 0) {
        constexpr uint32_t idesc_qk = idesc_bf16_f32(TC_ROWS, TC_STAGE, false);
        constexpr uint32_t idesc_pv = idesc_bf16_f32(TC_ROWS, TC_D, true);
        const uint32_t q_addr = smem_u32(sQ);
        const uint32_t kv_addr = smem_u32(sKV);
        const uint32_t p_addr = smem_u32(sP);
        int g = 0, seg = 0;
        bool failed = false;
        // S = Q K^T for global stage gg into S buffer gg % 2
        auto issue_qk = [&](int gg) -> bool {
          const int slot = gg % TC_NS;
          if (!mbar_wait(&full[slot], (uint32_t)(gg / TC_NS) & 1u, a.status)) return false;
          if (!mbar_wait(&s_free[gg & 1], ((uint32_t)(gg >> 1) & 1u) ^ 1u, a.status)) return false;
          tc_fence_after();
          const uint32_t k_addr = kv_addr + slot * TcSmem::STAGE;
#pragma unroll
          for (int ks = 0; ks < TC_D / 16; ++ks) {
            const uint32_t off = (uint32_t)(ks & 3) * 32u;  // 16 dims = 32 bytes inside the row
            const uint64_t ad = sw128_desc(q_addr + (ks >> 2) * TcSmem::HALF_Q + off, 16, 1024);
            const uint64_t bd = sw128_desc(k_addr + (ks >> 2) * TcSmem::K_HALF + off, 16, 1024);
            tc_mma_bf16(tmem + COL_S + (uint32_t)(gg & 1) * TC_STAGE, ad, bd, idesc_qk, ks > 0);
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
            const uint32_t v_addr = kv_addr + (gg % TC_NS) * TcSmem::STAGE + 2 * TcSmem::K_HALF;
            const uint32_t pb = p_addr + (uint32_t)(gg & 1) * TcSmem::P_BUF;
#pragma unroll
            for (int ks = 0; ks < TC_STAGE / 16; ++ks) {
              const uint64_t ad = sw128_desc(pb + ks * 32u, 16, 1024);
              const uint64_t bd = sw128_desc(v_addr + ks * 2048u, TcSmem::K_HALF, 1024);
              tc_mma_bf16(tmem + COL_O, ad, bd, idesc_pv, (k > 0 || ks > 0) ? 1u : 0u);
            }
            tc_commit(&empty[gg % TC_NS]);
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
      // ========================= softmax warps 0-3 =========================
      // Tile row (= TMEM lane) p = 32 * warp + lane holds query row qr = 4 * lane + warp,
      // so the real rows of a small group spread over all four warps / schedulers.
      const int p = warp * 32 + lane;
      const int qr = 4 * lane + warp;
      const uint32_t t_lane = tmem + ((uint32_t)(warp * 32) << 16);
      const bool row_ok = qr < a.R;
      const bool warp_rows = warp < a.R;                    // any real row in this warp
      const int di = row_ok ? qr / a.g : 0;                 // new-token index of the row
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
        const int vis = row_ok ? Lb + di + 1 : 0;           // visible tokens of this row

        // -- query row qr into tile row p of the swizzled K-major tile (zeros for padding)
        {
          const int h = c.hk * a.g + (row_ok ? qr % a.g : 0);
          const uint4* src = reinterpret_cast<const uint4*>(
              reinterpret_cast<const __nv_bfloat16*>(a.q) + (((size_t)c.b * a.T + di) * a.Hq + h) * TC_D);
#pragma unroll
          for (int hh = 0; hh < 2; ++hh)
#pragma unroll
            for (int ch = 0; ch < 8; ++ch) {
              const uint4 v = row_ok ? src[hh * 8 + ch] : make_uint4(0, 0, 0, 0);
              *reinterpret_cast<uint4*>(sQ + hh * TcSmem::HALF_Q + p * 128 + ((ch ^ (p & 7)) << 4)) = v;
            }
        }
        fence_proxy_async_smem();
        __syncwarp();
        if (lane == 0) mbar_arrive(q_full);

        float m = -INFINITY, l = 0.f;
        for (int k = 0; k < n; ++k) {
          const int gg = g + k;
          const int slot = gg % TC_NS;
          const int t0 = (c.k0 + k * TC_CHUNKS) * kChunk;
          const int nvalid = min(min(TC_CHUNKS, kend - c.k0 - k * TC_CHUNKS) * kChunk, Nb - t0);
          const bool tail = (nvalid < TC_STAGE) || (t0 + TC_STAGE > Lb + 1);
          if (!failed && !mbar_wait(&s_full[gg & 1], (uint32_t)(gg >> 1) & 1u, a.status)) failed = true;
          tc_fence_after();
          float x[TC_STAGE];
          {
            uint32_t s0[32], s1[32];
            tmem_ld32(t_lane + COL_S + (uint32_t)(gg & 1) * TC_STAGE, s0);
            tmem_ld32(t_lane + COL_S + (uint32_t)(gg & 1) * TC_STAGE + 32, s1);
            tmem_ld_wait();
#pragma unroll
            for (int j = 0; j < 32; ++j) {
              x[j] = __uint_as_float(s0[j]) * a.qscale;
              x[j + 32] = __uint_as_float(s1[j]) * a.qscale;
            }
          }
          tc_fence_before();
          __syncwarp();
          if (lane == 0) mbar_arrive(&s_free[gg & 1]);

          float mx4[4] = {-INFINITY, -INFINITY, -INFINITY, -INFINITY};
#pragma unroll
          for (int j = 0; j < TC_STAGE; ++j) {
            if (!row_ok || (tail && (j >= nvalid || t0 + j >= vis))) x[j] = -INFINITY;
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
          uint32_t pk[TC_STAGE / 2];
          if (warp_rows) {
            float ps4[4] = {0.f, 0.f, 0.f, 0.f};
            const float mref = (m == -INFINITY) ? 0.f : m;
#pragma unroll
            for (int j = 0; j < TC_STAGE; j += 2) {
              const float p0 = fast_exp2(x[j] - mref), p1 = fast_exp2(x[j + 1] - mref);
              ps4[(j >> 1) & 3] += p0 + p1;
              pk[j / 2] = pack_bf16x2(p0, p1);
            }
            l += (ps4[0] + ps4[1]) + (ps4[2] + ps4[3]);
          } else {
#pragma unroll
            for (int j = 0; j < TC_STAGE / 2; ++j) pk[j] = 0u;
          }

          // P buffer (gg & 1) is free once PV(gg - 2) completed
          if (!failed && !mbar_wait(&p_free[gg & 1], ((uint32_t)(gg >> 1) & 1u) ^ 1u, a.status)) failed = true;
          if (__any_sync(0xffffffffu, rescale)) {
            // O must hold PV(gg - 1) before it is scaled in place
            if (!failed && !mbar_wait(&p_free[(gg - 1) & 1], (uint32_t)((gg - 1) >> 1) & 1u, a.status))
              failed = true;
            tc_fence_after();
#pragma unroll
            for (int cb = 0; cb < TC_D / 32; ++cb) {
              uint32_t o[32];
              tmem_ld32(t_lane + COL_O + cb * 32, o);
              tmem_ld_wait();
#pragma unroll
              for (int j = 0; j < 32; ++j) o[j] = __float_as_uint(__uint_as_float(o[j]) * alpha);
              tmem_st32(t_lane + COL_O + cb * 32, o);
            }
            tmem_st_wait();
          }
          {
            unsigned char* prow = sP + (gg & 1) * TcSmem::P_BUF + p * 128;
#pragma unroll
            for (int ch = 0; ch < 8; ++ch)
              *reinterpret_cast<uint4*>(prow + ((ch ^ (p & 7)) << 4)) =
                  make_uint4(pk[4 * ch], pk[4 * ch + 1], pk[4 * ch + 2], pk[4 * ch + 3]);
          }
          if (nvalid < TC_STAGE) {
            // rows past the valid tokens hold whatever the cache held there: zero them in V
            if (!failed && !mbar_wait(&full[slot], (uint32_t)(gg / TC_NS) & 1u, a.status)) failed = true;
            unsigned char* vbase = sKV + slot * TcSmem::STAGE + 2 * TcSmem::K_HALF;
            const int nz = (TC_STAGE - nvalid) * 8;  // 16-byte pieces per half
            for (int e = p; e < 2 * nz; e += 128) {
              const int hh = e / nz, q = e % nz;
              *reinterpret_cast<uint4*>(vbase + hh * TcSmem::K_HALF + nvalid * 128 + q * 16) =
                  make_uint4(0, 0, 0, 0);
            }
          }
          fence_proxy_async_smem();
          tc_fence_before();
          __syncwarp();
          if (lane == 0) mbar_arrive(&p_full[gg & 1]);
        }

        // -- unit segment done: O row out
        const int gl = g + n - 1;
        if (!failed && !mbar_wait(&p_free[gl & 1], (uint32_t)(gl >> 1) & 1u, a.status)) failed = true;
        tc_fence_after();
        const bool whole = (c.k0 == 0) && (kend == nb);
        const float inv = (l > 0.f) ? 1.f / l : 0.f;
        const long long slot_idx = (long long)blockIdx.x + u;
        const int h = c.hk * a.g + (row_ok ? qr % a.g : 0);
#pragma unroll
        for (int cb = 0; cb < TC_D / 32; ++cb) {
          uint32_t o[32];
          tmem_ld32(t_lane + COL_O + cb * 32, o);
          tmem_ld_wait();
          if (row_ok) {
            if (whole) {
              const size_t ob = (((size_t)c.b * a.T + di) * a.Hq + h) * TC_D + cb * 32;
              if (a.out_bf16) {
                uint4* dst = reinterpret_cast<uint4*>(reinterpret_cast<__nv_bfloat16*>(a.out) + ob);
#pragma unroll
                for (int q4 = 0; q4 < 4; ++q4) {
                  uint32_t w[4];
#pragma unroll
                  for (int e = 0; e < 4; ++e)
                    w[e] = pack_bf16x2(__uint_as_float(o[q4 * 8 + 2 * e]) * inv,
                                       __uint_as_float(o[q4 * 8 + 2 * e + 1]) * inv);
                  dst[q4] = make_uint4(w[0], w[1], w[2], w[3]);
                }
              } else {
                float4* dst = reinterpret_cast<float4*>(reinterpret_cast<float*>(a.out) + ob);
#pragma unroll
                for (int q4 = 0; q4 < 8; ++q4)
                  dst[q4] = make_float4(__uint_as_float(o[4 * q4]) * inv, __uint_as_float(o[4 * q4 + 1]) * inv,
                                        __uint_as_float(o[4 * q4 + 2]) * inv, __uint_as_float(o[4 * q4 + 3]) * inv);
              }
            } else {
              float4* dst = reinterpret_cast<float4*>(a.part_o + ((size_t)slot_idx * a.R + qr) * TC_D + cb * 32);
#pragma unroll
              for (int q4 = 0; q4 < 8; ++q4)
                dst[q4] = make_float4(__uint_as_float(o[4 * q4]) * inv, __uint_as_float(o[4 * q4 + 1]) * inv,
                                      __uint_as_float(o[4 * q4 + 2]) * inv, __uint_as_float(o[4 * q4 + 3]) * inv);
            }
          }
        }
        if (row_ok && !whole)
          a.part_lse[(size_t)slot_idx * a.R + qr] = (l > 0.f) ? m + fast_log2(l) : -INFINITY;
        if (threadIdx.x == 0) {
          if (c.k0 == 0) a.unit_ctas[u].x = blockIdx.x;
          if (kend == nb) a.unit_ctas[u].y = blockIdx.x;
        }
        tc_fence_before();  // the O reads above precede the next segment's first PV

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
  if (warp == 5) tmem_dealloc(tmem, TC_TMEM_COLS);
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

template <bool PAGED>
cudaError_t launch_tc(const DecodeArgs& a, cudaStream_t st) {
  const unsigned long long rows =
      PAGED ? (unsigned long long)a.num_pages * a.Hkv * a.page_size
            : (unsigned long long)a.B * a.Hkv * a.max_seq_len;
  if (rows >= (1ull << 31)) return cudaErrorNotSupported;  // TMA row coordinate is int32
  CUtensorMap mk, mv;
  if (!make_map(&mk, a.k_cache, rows) || !make_map(&mv, a.v_cache, rows)) return cudaErrorNotSupported;
  const size_t smem = TcSmem::bytes(a.B);
  if (smem > 227 * 1024) return cudaErrorNotSupported;
  static std::atomic<unsigned long long> attr_done{0};
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  const unsigned long long bit = 1ull << (dev & 63);
  if (!(attr_done.load() & bit)) {
    e = cudaFuncSetAttribute(decode_tc_kernel<PAGED>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             227 * 1024);
    if (e != cudaSuccess) return e;
    attr_done.fetch_or(bit);
  }
  decode_tc_kernel<PAGED><<<a.grid, TC_THREADS, smem, st>>>(a, mk, mv);
  e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  const long long warps = (long long)a.B * a.Hkv * a.R;
  combine_kernel<TC_D><<<(int)((warps * 32 + 255) / 256), 256, 0, st>>>(a);
  return cudaGetLastError();
}

}  // namespace

cudaError_t launch_decode_tc(const DecodeArgs& a, cudaStream_t st) {
  return a.block_table ? launch_tc<true>(a, st) : launch_tc<false>(a, st);
}

}  // namespace kvd

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
// One CTA per SM, 12 warps, each with one role:
// * warps 8 and 11 (loaders): 2-D tensor loads of 16-token K (warp 8) and V
//   (warp 11) boxes, two 64-dim halves each with a 128-byte swizzle, into two
//   separate rings.  A K stage is released as soon as its QK product is done,
//   so K runs several stages ahead; a V stage lives until its PV product is
//   done.  Page ids come from a prefetched window of the block table.
// * warp 9 (QK issuer): one thread issues S = Q K^T (M = MQ, N = tokens of
//   the stage, K = 128 dims) into a double-buffered TMEM tile.
// * warp 10 (PV issuer): one thread issues O_h += P_h V_h for the two token
//   halves h of the stage into two TMEM accumulators, as soon as each half of
//   P is written; it never waits on the next stage's keys.
//   P is passed as a bf16 high part (the top 16 bits of the fp32 value) plus
//   the exact remainder rounded to the nearest bf16, which keeps each
//   probability to within 2^-15 relative.
//   With MQ = 64 the two parts are stacked into the 128 rows of one M = 128
//   product (an M = 64 MMA runs at half the rate of an M = 128 one), and the
//   epilogue adds the two output rows; with MQ = 128 they are two passes.
// * warps 0-7 (softmax): warpgroup h owns token half h of every stage; each
//   thread owns 32 scores of one query row per stage (with MQ = 64 two threads
//   share a row through the 16-lane TMEM loads, so every lane works).  Rows
//   are spread over the four TMEM sub-partitions.  A thread masks, keeps a
//   reference max raised only when the running max grows by more than 2^8
//   (its O row is then rescaled in TMEM), and writes its probabilities into a
//   swizzled shared tile for the PV product.  At a unit boundary the two
//   halves are merged by log-sum-exp and the output (or a normalised partial)
//   is written.
// Units of up to 64 query rows use MQ = 64 and 128-token stages; larger units
// MQ = 128 and 64-token stages.  Every tcgen05.mma costs at least ~45 cycles,
// so the stage sizes keep the instruction count per token low.
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
constexpr int TC_THREADS = 384;                   // 8 softmax warps + 4 single-role warps
constexpr int TC_SOFTMAX_THREADS = 256;
constexpr int WARP_KLOAD = 8, WARP_QK = 9, WARP_PV = 10, WARP_VLOAD = 11;
constexpr uint32_t TC_TMEM_COLS = 512;            // S0 | S1 | O_0 | O_1
constexpr float kRescaleThreshold = 8.0f;         // log2 units

// MQ = rows of the QK tile (query rows of a unit, padded): 64 or 128.
template <int MQ>
struct TcCfg {
  // MQ = 64: two threads share a score row (16-lane TMEM shapes) and the high
  // and residual parts of P are stacked into the 128 rows of one PV product.
  static constexpr bool STACK = MQ == 64;
  static constexpr int ST = STACK ? 128 : 64;          // tokens per stage
  static constexpr int CH = ST / kChunk;               // 16-token boxes per stage
  static constexpr int HALF = ST / 2;                  // tokens per softmax warpgroup
  static constexpr int NK = STACK ? 3 : 4;             // K ring depth
  static constexpr int NV = STACK ? 3 : 4;             // V ring depth
  static constexpr int HALF_Q = MQ * 128;              // MQ rows x 64 dims
  static constexpr int DHALF = ST * 128;               // one 64-dim half of a K or V stage
  static constexpr int KVSTAGE = 2 * DHALF;
  static constexpr int Q = 0;                          // 2 dim halves
  static constexpr int KR = Q + 2 * HALF_Q;            // K ring
  static constexpr int VR = KR + NK * KVSTAGE;         // V ring
  static constexpr int P = VR + NV * KVSTAGE;
  // P: with STACK it lives in tensor memory (the columns of the S buffer it
  // was computed from); otherwise two 128-row x 128-byte shared tiles [high,
  // residual], token half h in bytes [64 h, 64 h + 64) of a row.
  static constexpr int P_TILE = 128 * 128;
  static constexpr int BAR = P + (STACK ? 0 : 2 * P_TILE);
  static constexpr int NBAR = 2 * NK + 2 * NV + 2 + 2 + 2 + 2 + 1 + 2;
  static constexpr int TMEM_SLOT = BAR + NBAR * 8;
  static constexpr int ML = TMEM_SLOT + 16;            // [2 halves][MQ] (m, l) for the merge
  static constexpr int SCRATCH = ML + 2 * MQ * 8;      // one int per warp for the scan
  static constexpr int PREFIX = SCRATCH + 64;
  static constexpr uint32_t COL_S = 0;                 // S buffers: 2 x ST columns
  static constexpr uint32_t COL_O = 2 * ST;            // O_h at COL_O + 128 h
  static size_t bytes(int B) { return (size_t)PREFIX + (size_t)(B + 1) * 4 + 1024; }
};

// One loader warp: 16-token boxes (two 64-dim halves each) of K or V for
// every stage of the CTA's chunk range, into a ring of NSLOT stages.
template <bool PAGED, int ST, int NSLOT>
__device__ __forceinline__ void tc_loader(const DecodeArgs& a, const int* sPrefix, SegState c,
                                          long long x1, const CUtensorMap* tm, unsigned char* ring,
                                          uint64_t* fullb, uint64_t* emptyb) {
  constexpr int CH = ST / kChunk, DHALF = ST * 128;
  const int lane = threadIdx.x & 31;
  int g = 0;
  bool failed = false;
  bool waited = false;   // programmatic-dependency wait done (before the first copy)
  const uint64_t pol = l2_evict_first();   // the cache is read once
  // page id of chunk `ch` of sequence b (paged layout), -1 past `kend`
  auto page_of = [&](int b, int ch, int kend) -> int {
    if (ch >= kend) return -1;
    return a.block_table[(size_t)b * a.max_pages_per_seq + (ch * kChunk) / a.page_size];
  };
  for (; c.x < x1 && !failed; next_unit(a, c, seg_of(a, sPrefix, c, x1))) {
    const Seg sg = seg_of(a, sPrefix, c, x1);
    if (sg.empty()) continue;
    const int kend = sg.kend;
    // a shard holding no token of the sequence still has one (empty) chunk:
    // it is not loaded; outside sharded mode every chunk holds tokens
    const int Nb = a.shard_lens ? attended_len(a, c.b, false) : INT_MAX;
    // two 32-chunk windows of page ids, the second one loaded ahead of its use
    int wbase = sg.k0, win0 = -1, win1 = -1;
    if (PAGED) {
      win0 = page_of(c.b, wbase + lane, kend);
      win1 = page_of(c.b, wbase + 32 + lane, kend);
    }
    for (int kk = sg.k0; kk < kend; kk += CH, ++g) {
      if (PAGED && kk - wbase >= 32) {
        wbase += 32;
        win0 = win1;
        win1 = page_of(c.b, wbase + 32 + lane, kend);
      }
      const int slot = g % NSLOT;
      int ok = 1;
      if (lane == 0) ok = mbar_wait(&emptyb[slot], ((uint32_t)(g / NSLOT) & 1u) ^ 1u, a.status);
      ok = __shfl_sync(0xffffffffu, ok, 0);
      if (!ok) { failed = true; break; }
      if (!waited) {   // the caches are read only once the previous kernel is done
        grid_dep_wait();
        waited = true;
      }
      const int nck = min(CH, kend - kk);
      int page = -1;
      if (PAGED) page = __shfl_sync(0xffffffffu, win0, kk - wbase + min(lane, CH - 1));
      int row = -1;
      if (lane < nck && (kk + lane) * kChunk < Nb) {
        const int tc = (kk + lane) * kChunk;
        if (!PAGED) {
          row = (int)(((long long)c.b * a.Hkv + c.hk) * a.max_seq_len + tc);
        } else if (page >= 0 && page < a.num_pages) {
          row = (int)(((long long)page * a.Hkv + c.hk) * a.page_size + tc % a.page_size);
        } else if (a.status) {
          atomicOr(a.status, KVD_FLAG_PAGE_OUT_OF_RANGE);
        }
      }
      uint32_t bytes = row >= 0 ? 2u * kChunk * 128u : 0u;
#pragma unroll
      for (int m = 16; m >= 1; m >>= 1) bytes += __shfl_xor_sync(0xffffffffu, bytes, m);
      if (lane == 0) mbar_arrive_expect_tx(&fullb[slot], bytes);
      __syncwarp();
      if (row >= 0) {
        unsigned char* dst = ring + slot * (2 * DHALF) + lane * kChunk * 128;
        tma_load_2d_hint(dst, tm, 0, row, &fullb[slot], pol);
        tma_load_2d_hint(dst + DHALF, tm, 64, row, &fullb[slot], pol);
      }
      __syncwarp();
    }
  }
  if (lane == 0) {  // every issued copy lands before the CTA may exit
    for (int k = max(0, g - NSLOT); k < g; ++k)
      if (!mbar_wait(&fullb[k % NSLOT], (uint32_t)(k / NSLOT) & 1u, a.status)) break;
  }
  __syncwarp();
}

template <bool PAGED, int MQ>
__global__ void __launch_bounds__(TC_THREADS, 1)
    decode_tc_kernel(const DecodeArgs a, const __grid_constant__ CUtensorMap tmk,
                     const __grid_constant__ CUtensorMap tmv) {
  using C = TcCfg<MQ>;
  constexpr int ST = C::ST, CH = C::CH, HALF = C::HALF, NK = C::NK, NV = C::NV;
  extern __shared__ unsigned char smem_raw[];
  unsigned char* smem = smem_raw + ((1024u - (smem_u32(smem_raw) & 1023u)) & 1023u);
  unsigned char* sQ = smem + C::Q;
  unsigned char* sK = smem + C::KR;
  unsigned char* sV = smem + C::VR;
  unsigned char* sP = smem + C::P;
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + C::BAR);
  uint64_t* k_full = bars;                // K loader -> QK issuer
  uint64_t* k_empty = k_full + NK;        // QK done -> K loader
  uint64_t* v_full = k_empty + NK;        // V loader -> PV issuer (+ softmax on short stages)
  uint64_t* v_empty = v_full + NV;        // PV done -> V loader
  uint64_t* s_full = v_empty + NV;        // QK done -> softmax            [S buffer]
  uint64_t* s_free = s_full + 2;          // S buffer reusable -> QK issuer [S buffer]
  uint64_t* p_full = s_free + 2;          // P half written -> PV issuer   [token half]
  uint64_t* p_free = p_full + 2;          // PV of a half done -> softmax  [token half]
  uint64_t* q_full = p_free + 2;          // Q written -> QK issuer
  uint64_t* mma_done = q_full + 1;        // [QK, PV] issued MMAs complete (exit)
  uint32_t* sTmem = reinterpret_cast<uint32_t*>(smem + C::TMEM_SLOT);
  float2* sML = reinterpret_cast<float2*>(smem + C::ML);
  int* sScratch = reinterpret_cast<int*>(smem + C::SCRATCH);
  int* sPrefix = reinterpret_cast<int*>(smem + C::PREFIX);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;

  // the lengths' first round trip overlaps the clearing
  if ((int)threadIdx.x < a.B) prefetch_l1(a.shard_lens ? a.shard_lens + threadIdx.x : a.seq_lens + threadIdx.x);
  {  // V rows past a partial stage meet zero weights, so they must be finite:
     // the V ring starts from zeros.  K rows there only feed masked scores (and
     // padding rows, whose output is never written).
    uint4* z = reinterpret_cast<uint4*>(sV);
    for (int k = threadIdx.x; k < NV * C::KVSTAGE / 16; k += blockDim.x)
      z[k] = make_uint4(0, 0, 0, 0);
  }
  if (threadIdx.x == 0) {
    for (int s = 0; s < NK; ++s) {
      mbar_init(&k_full[s], 1);
      mbar_init(&k_empty[s], 1);
    }
    for (int s = 0; s < NV; ++s) {
      mbar_init(&v_full[s], 1);
      mbar_init(&v_empty[s], 1);
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(&s_full[b], 1);
      // STACK: P overwrites S in tensor memory, so the buffer is free once the
      // PV product of its stage is done (one commit); otherwise once the 8
      // softmax warps have read S
      mbar_init(&s_free[b], C::STACK ? 1 : 8);
      mbar_init(&p_full[b], 4);
      mbar_init(&p_free[b], 1);
      mbar_init(&mma_done[b], 1);
    }
    mbar_init(q_full, 8);
  }
  if (warp == WARP_QK) {
    tmem_alloc(sTmem, TC_TMEM_COLS);
    tmem_relinquish();
  }
  if (warp == WARP_KLOAD && lane == 0) prefetch_tensormap(&tmk);
  if (warp == WARP_VLOAD && lane == 0) prefetch_tensormap(&tmv);
  chunk_prefix_scan(a, sPrefix, sScratch, blockIdx.x == 0);
  fence_barrier_init();
  fence_proxy_async_smem();
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *sTmem;
  grid_dep_launch();
  // Each role waits for the previous kernel (griddepcontrol.wait) itself, just
  // before its first access to q, the caches or the outputs: the loaders
  // before their first copy (their first block-table reads go out before it),
  // the softmax warps before the q load.  The two MMA issuers touch only
  // shared and tensor memory and never wait.

  const long long total = (long long)a.Hkv * sPrefix[a.B];
  const long long x0 = total * blockIdx.x / a.grid;
  const long long x1 = total * (blockIdx.x + 1) / a.grid;

  if (x0 < x1) {
    const SegState st = locate_chunk(a, sPrefix, x0);
    if (warp == WARP_KLOAD) {
      tc_loader<PAGED, ST, NK>(a, sPrefix, st, x1, &tmk, sK, k_full, k_empty);
    } else if (warp == WARP_VLOAD) {
      tc_loader<PAGED, ST, NV>(a, sPrefix, st, x1, &tmv, sV, v_full, v_empty);
    } else if (warp == WARP_QK) {
      // ====================== QK issuer: S = Q K^T =========================
      if (lane == 0) {
        constexpr uint32_t idesc_qk = idesc_bf16_f32(MQ, ST, false);
        // descriptors of the tile bases; a byte offset b inside a tile adds b >> 4
        const uint64_t dq = sw128_desc(smem_u32(sQ), 16, 1024);
        const uint64_t dk = sw128_desc(smem_u32(sK), 16, 1024);
        int g = 0, seg = 0;
        bool failed = false;
        SegState c = st;
        for (; c.x < x1 && !failed; next_unit(a, c, seg_of(a, sPrefix, c, x1))) {
          const Seg sg = seg_of(a, sPrefix, c, x1);
          if (sg.empty()) continue;
          const int n = (sg.kend - sg.k0 + CH - 1) / CH;
          if (!mbar_wait(q_full, (uint32_t)seg & 1u, a.status)) { failed = true; break; }
          for (int k = 0; k < n; ++k) {
            const int gg = g + k;
            const int slot = gg % NK;
            if (!mbar_wait(&k_full[slot], (uint32_t)(gg / NK) & 1u, a.status) ||
                !mbar_wait(&s_free[gg & 1], ((uint32_t)(gg >> 1) & 1u) ^ 1u, a.status)) {
              failed = true;
              break;
            }
            tc_fence_after();
            const uint32_t kofs = (uint32_t)slot * C::KVSTAGE;
#pragma unroll
            for (int ks = 0; ks < TC_D / 16; ++ks) {
              const uint32_t off = (uint32_t)(ks & 3) * 32u;  // 16 dims = 32 bytes inside the row
              tc_mma_bf16(tmem + C::COL_S + (uint32_t)(gg & 1) * ST,
                          dq + (((ks >> 2) * C::HALF_Q + off) >> 4),
                          dk + ((kofs + (ks >> 2) * C::DHALF + off) >> 4), idesc_qk, ks > 0);
            }
            tc_commit(&k_empty[slot]);
            tc_commit(&s_full[gg & 1]);
          }
          g += n;
          ++seg;
        }
        // every MMA this thread issued completes before the CTA frees TMEM
        tc_commit(&mma_done[0]);
        mbar_wait(&mma_done[0], 0, a.status);
      }
      __syncwarp();
    } else if (warp == WARP_PV) {
      // ===================== PV issuer: O_h += P_h V_h =====================
      if (lane == 0) {
        constexpr uint32_t idesc_pv = idesc_bf16_f32(128, TC_D, true);
        const uint64_t dp = sw128_desc(smem_u32(sP), 16, 1024);
        const uint64_t dv = sw128_desc(smem_u32(sV), C::DHALF, 1024);
        int g = 0;
        bool failed = false;
        SegState c = st;
        for (; c.x < x1 && !failed; next_unit(a, c, seg_of(a, sPrefix, c, x1))) {
          const Seg sg = seg_of(a, sPrefix, c, x1);
          if (sg.empty()) continue;
          const int n = (sg.kend - sg.k0 + CH - 1) / CH;
          for (int k = 0; k < n && !failed; ++k) {
            const int gg = g + k;
            const int slot = gg % NV;
            if (!mbar_wait(&v_full[slot], (uint32_t)(gg / NV) & 1u, a.status)) { failed = true; break; }
            const uint32_t vofs = (uint32_t)slot * C::KVSTAGE;
#pragma unroll
            for (int h = 0; h < 2; ++h) {
              if (!mbar_wait(&p_full[h], (uint32_t)gg & 1u, a.status)) { failed = true; break; }
              tc_fence_after();
              if constexpr (C::STACK) {
                // rows [high; residual] of P_h (tensor memory, 32 columns of S
                // buffer gg % 2 from column 64 h) against the 64 tokens of half h
#pragma unroll
                for (int ks = 0; ks < HALF / 16; ++ks) {
                  const int t = h * HALF + ks * 16;
                  tc_mma_bf16_ta(tmem + C::COL_O + (uint32_t)h * TC_D,
                                 tmem + C::COL_S + (uint32_t)(gg & 1) * ST + (uint32_t)(h * 64 + ks * 8),
                                 dv + ((vofs + t * 128) >> 4), idesc_pv, (k > 0 || ks > 0) ? 1u : 0u);
                }
              } else {
#pragma unroll
                for (int part = 0; part < 2; ++part)
#pragma unroll
                  for (int ks = 0; ks < HALF / 16; ++ks) {
                    const int t = h * HALF + ks * 16;
                    tc_mma_bf16(tmem + C::COL_O + (uint32_t)h * TC_D,
                                dp + (((uint32_t)part * C::P_TILE + (t / 16) * 32) >> 4),
                                dv + ((vofs + t * 128) >> 4), idesc_pv,
                                (k > 0 || part > 0 || ks > 0) ? 1u : 0u);
                  }
              }
              tc_commit(&p_free[h]);
            }
            tc_commit(&v_empty[slot]);
            if constexpr (C::STACK) tc_commit(&s_free[gg & 1]);   // P(gg) read: the S buffer is free
          }
          g += n;
        }
        tc_commit(&mma_done[1]);
        mbar_wait(&mma_done[1], 0, a.status);
      }
      __syncwarp();
    } else {
      // ========================= softmax warps 0-7 =========================
      // Sub-partition sp = warp % 4 reaches TMEM lanes 32 sp .. 32 sp + 31.
      // MQ = 128: tile row p = 32 sp + lane sits in lane `lane` of S and O.
      // MQ = 64: tile row p = 16 sp + (lane % 16) sits in S lane lane % 16 and
      // threads lane and lane + 16 share it (columns [0, 32) and [32, 64) of
      // the half); in O, lane `lane` of the sub-partition holds the high part
      // (lane < 16) or the residual part (lane >= 16) of that row.  Tile row p
      // holds query row qr = 4 (p % RPT) + sp, spreading the rows of a small
      // group over the four sub-partitions.
      constexpr int RPT = MQ / 4;                            // tile rows per sub-partition
      const int sp = warp & 3;
      const int hw = warp >> 2;                              // token half of the stage
      const int rl = C::STACK ? (lane & 15) : lane;          // row within the sub-partition
      const int cs = C::STACK ? (lane >> 4) : 0;             // column sub-half (pairs)
      const int p = sp * RPT + rl;                           // tile row
      const int qr = 4 * rl + sp;                            // query row
      const int tok0 = hw * HALF + cs * 32;                  // first of this thread's 32 tokens
      const int tid = threadIdx.x;                           // 0 .. 255
      const uint32_t t_lane = tmem + ((uint32_t)(sp * 32) << 16);
      const uint32_t col_o = C::COL_O + (uint32_t)hw * TC_D;
      const bool row_ok = qr < a.R;
      const bool warp_rows = sp < a.R;                       // any real row in this warp
      const int di = row_ok ? qr / a.g : 0;                  // new-token index of the row
      // MQ = 128: this thread's row of the shared P tiles and its first 16-byte
      // chunk there (MQ = 64 keeps P in tensor memory)
      unsigned char* p_hi = sP + p * 128;
      unsigned char* p_lo = p_hi + C::P_TILE;
      const int pch0 = (tok0 % 64) / 8;
      // Scores enter the exponent as fma(q . k, qs, -m).  With qs > 0 the
      // reference comes from the largest raw product, with qs < 0 from the
      // smallest; masked tokens take the raw value that the scale maps to -inf.
      // A zero scale becomes a tiny positive one: the same all-ones weights,
      // while masked tokens still map to -inf.
      const bool qneg = a.qscale < 0.f;
      const float qs = qneg ? a.qscale : fmaxf(a.qscale, 1e-30f);
      const uint32_t mask_raw = __float_as_uint(qneg ? INFINITY : -INFINITY);
      // q rows of unit (b, hk) into the Q tile: tile row p, dim half hw, 16-byte
      // chunks 4 cs .. 4 cs + 3 (pairs) or all 8; padding rows read as zeros
      auto issue_q = [&](int b, int hk) {
        const int h = hk * a.g + (row_ok ? qr % a.g : 0);
        const uint4* src = reinterpret_cast<const uint4*>(
            reinterpret_cast<const __nv_bfloat16*>(a.q) + (((size_t)b * a.T + di) * a.Hq + h) * TC_D);
        constexpr int NCH = C::STACK ? 4 : 8;
#pragma unroll
        for (int k8 = 0; k8 < NCH; ++k8) {
          const int ch = cs * 4 + k8;
          cp_async16(sQ + hw * C::HALF_Q + p * 128 + ((ch ^ (p & 7)) << 4), src + hw * 8 + ch,
                     row_ok ? 16u : 0u);
        }
      };
      // the copies have landed: hand the tile to the QK issuer
      auto publish_q = [&]() {
        cp_async_wait_all();
        fence_proxy_async_smem();
        __syncwarp();
        if (lane == 0) mbar_arrive(q_full);
      };
      grid_dep_wait();      // q and the outputs: only after the previous kernel
      issue_q(st.b, st.hk);
      publish_q();
      int Nb_cur = attended_len(a, st.b, false);
      int g = 0;
      bool failed = false;
      SegState c = st;
      for (; c.x < x1; next_unit(a, c, seg_of(a, sPrefix, c, x1))) {
        const Seg sg = seg_of(a, sPrefix, c, x1);
        if (sg.empty()) continue;
        const int Nb = Nb_cur;
        const int Lb = mask_base(a, c.b, Nb);
        const int kend = sg.kend;
        const int n = (kend - sg.k0 + CH - 1) / CH;
        const int u = c.b * a.Hkv + c.hk;
        const int vis = row_ok ? Lb + di + 1 : 0;            // visible tokens of this row

        // the next unit of this CTA's range, whose q is fetched during the last
        // stage of this one (the Q tile is free once that stage's QK is done)
        const bool has_next = next_has_work(a, sg, x1);
        const int nx_hk = (c.hk + 1 == a.Hkv) ? 0 : c.hk + 1;
        const int nx_b = (c.hk + 1 == a.Hkv) ? c.b + 1 : c.b;
        // length of the next unit's sequence, loaded now and used after this unit
        if (has_next && nx_b != c.b) Nb_cur = attended_len(a, nx_b, false);

        float m = -INFINITY, l = 0.f;
        for (int k = 0; k < n; ++k) {
          const int gg = g + k;
          const int t0 = (sg.k0 + k * CH) * kChunk;
          const int nvalid = min(min(CH, kend - sg.k0 - k * CH) * kChunk, Nb - t0);
          const bool tail = (nvalid < ST) || (t0 + ST > Lb + 1);
          if (!failed && !mbar_wait(&s_full[gg & 1], (uint32_t)(gg >> 1) & 1u, a.status)) failed = true;
          tc_fence_after();
          const bool last = k == n - 1;
          if (last && has_next) issue_q(nx_b, nx_hk);
          uint32_t sr[32];   // raw scores q . k of this thread's 32 tokens
          {
            const uint32_t sa = t_lane + C::COL_S + (uint32_t)(gg & 1) * ST + hw * HALF;
            if constexpr (C::STACK) tmem_ld16x2_32(sa, sr);
            else tmem_ld32(sa, sr);
            tmem_ld_wait();
          }
          tc_fence_before();
          __syncwarp();
          if constexpr (!C::STACK) {
            if (lane == 0) mbar_arrive(&s_free[gg & 1]);
          }

          // Masking only on the stages that hold a causal edge, the end of the
          // cache or a partial chunk (the same for every thread).  Outside them
          // padding rows keep their finite scores: a padding row only feeds its
          // own O row, which is never written out.
          if (tail) {
#pragma unroll
            for (int j = 0; j < 32; ++j) {
              const int tj = tok0 + j;                       // token of the stage
              if (!row_ok || tj >= nvalid || t0 + tj >= vis) sr[j] = mask_raw;
            }
          }
          float mx;   // raw product that the scale maps to the largest score
          {
            float t16[16];
            if (!qneg) {
#pragma unroll
              for (int j = 0; j < 16; ++j) t16[j] = fmaxf(__uint_as_float(sr[j]), __uint_as_float(sr[j + 16]));
#pragma unroll
              for (int w = 8; w >= 1; w >>= 1)
#pragma unroll
                for (int j = 0; j < w; ++j) t16[j] = fmaxf(t16[j], t16[j + w]);
            } else {
#pragma unroll
              for (int j = 0; j < 16; ++j) t16[j] = fminf(__uint_as_float(sr[j]), __uint_as_float(sr[j + 16]));
#pragma unroll
              for (int w = 8; w >= 1; w >>= 1)
#pragma unroll
                for (int j = 0; j < w; ++j) t16[j] = fminf(t16[j], t16[j + w]);
            }
            mx = t16[0];
          }
          if constexpr (C::STACK) {
            const float o = __shfl_xor_sync(0xffffffffu, mx, 16);
            mx = qneg ? fminf(mx, o) : fmaxf(mx, o);
          }
          mx *= qs;                                          // the largest scaled score
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
          uint32_t pk[16], pl[16];   // bf16 pairs: high part (top 16 bits), residual (rounded)
          if (warp_rows) {
            const float mref = (m == -INFINITY) ? 0.f : m;
            const float2 qs2 = make_float2(qs, qs), nm2 = make_float2(-mref, -mref);
            float2 sum2 = make_float2(0.f, 0.f);
#pragma unroll
            for (int j = 0; j < 16; ++j) {
              const float2 e = __ffma2_rn(make_float2(__uint_as_float(sr[2 * j]), __uint_as_float(sr[2 * j + 1])),
                                          qs2, nm2);
              const float2 pp = make_float2(fast_exp2(e.x), fast_exp2(e.y));
              sum2 = __fadd2_rn(sum2, pp);
              const uint32_t b0 = __float_as_uint(pp.x), b1 = __float_as_uint(pp.y);
              const float2 hi = make_float2(__uint_as_float(b0 & 0xffff0000u), __uint_as_float(b1 & 0xffff0000u));
              const float2 lo = __ffma2_rn(hi, make_float2(-1.f, -1.f), pp);   // exact: pp - hi
              pk[j] = hi16x2(b0, b1);
              pl[j] = pack_bf16x2(lo.x, lo.y);   // residual rounded to nearest
            }
            l += sum2.x + sum2.y;
          } else {
#pragma unroll
            for (int j = 0; j < 16; ++j) { pk[j] = 0u; pl[j] = 0u; }
          }

          // PV(gg - 1) of this half completed: O_hw holds every earlier stage,
          // the shared P tile (MQ = 128) is free, and the PV issuer has taken
          // phase gg - 1 of p_full[hw], so this stage's arrival cannot run two
          // phases ahead of its wait
          if (!failed && !mbar_wait(&p_free[hw], (uint32_t)(gg - 1) & 1u, a.status)) failed = true;
          const bool any_rescale = __any_sync(0xffffffffu, rescale);
          if (any_rescale) {
            tc_fence_after();
#pragma unroll
            for (int cb = 0; cb < TC_D; cb += 16) {
              uint32_t o[16];
              tmem_ld32x32b_16(t_lane + col_o + cb, o);
              tmem_ld_wait();
#pragma unroll
              for (int j = 0; j < 16; ++j) o[j] = __float_as_uint(__uint_as_float(o[j]) * alpha);
              tmem_st32x32b_16(t_lane + col_o + cb, o);
            }
            tmem_st_wait();
          }
          if constexpr (C::STACK) {
            // P_hw into tensor memory over the S values just read: thread cs = 0
            // writes the high row (lane 32 sp + rl), cs = 1 the residual row
            // (lane 32 sp + 16 + rl), each over all 64 tokens of the half, so
            // the pair trades the 32 tokens of the part the other one writes
            uint32_t pr[32];
#pragma unroll
            for (int j = 0; j < 16; ++j) {
              const uint32_t got = __shfl_xor_sync(0xffffffffu, cs ? pk[j] : pl[j], 16);
              pr[j] = cs ? got : pk[j];          // tokens 2j, 2j + 1
              pr[16 + j] = cs ? pl[j] : got;     // tokens 32 + 2j, 33 + 2j
            }
            tmem_st32(t_lane + C::COL_S + (uint32_t)(gg & 1) * ST + (uint32_t)hw * 64, pr);
            tmem_st_wait();
          } else {
#pragma unroll
            for (int ch = 0; ch < 4; ++ch) {
              const int sw = ((pch0 + ch) ^ (rl & 7)) << 4;
              *reinterpret_cast<uint4*>(p_hi + sw) =
                  make_uint4(pk[4 * ch], pk[4 * ch + 1], pk[4 * ch + 2], pk[4 * ch + 3]);
              *reinterpret_cast<uint4*>(p_lo + sw) =
                  make_uint4(pl[4 * ch], pl[4 * ch + 1], pl[4 * ch + 2], pl[4 * ch + 3]);
            }
          }
          if (nvalid < ST) {
            // V rows past the valid tokens hold whatever the cache (or an older
            // stage) held there: zero this half's share of them
            const int vslot = gg % NV;
            if (!failed && !mbar_wait(&v_full[vslot], (uint32_t)(gg / NV) & 1u, a.status)) failed = true;
            unsigned char* vbase = sV + vslot * C::KVSTAGE;
            const int z0 = max(nvalid, hw * HALF), z1 = (hw + 1) * HALF;
            const int nz = max(0, z1 - z0) * 8;               // 16-byte pieces per dim half
            const int ltid = tid & 127;
            for (int e = ltid; e < 2 * nz; e += 128) {
              const int hh = e / nz, q = e % nz;
              *reinterpret_cast<uint4*>(vbase + hh * C::DHALF + z0 * 128 + q * 16) =
                  make_uint4(0, 0, 0, 0);
            }
          }
          fence_proxy_async_smem();
          tc_fence_before();
          __syncwarp();
          if (lane == 0) mbar_arrive(&p_full[hw]);
          if (last && has_next) publish_q();
        }

        // -- unit segment done: merge the two token halves, write the row
        const int gl = g + n - 1;
        if (!failed && (!mbar_wait(&p_free[0], (uint32_t)gl & 1u, a.status) ||
                        !mbar_wait(&p_free[1], (uint32_t)gl & 1u, a.status)))
          failed = true;
        tc_fence_after();
        if constexpr (C::STACK) l += __shfl_xor_sync(0xffffffffu, l, 16);
        if (cs == 0) sML[hw * MQ + p] = make_float2(m, l);
        named_bar_sync(1, TC_SOFTMAX_THREADS);
        const float2 h0 = sML[p], h1 = sML[MQ + p];
        const float mm = fmaxf(h0.x, h1.x);
        const float ms = (mm == -INFINITY) ? 0.f : mm;
        const float w0 = fast_exp2(h0.x - ms), w1 = fast_exp2(h1.x - ms);
        const float L = w0 * h0.y + w1 * h1.y;
        const float inv = (L > 0.f) ? 1.f / L : 0.f;
        const float s0 = w0 * inv, s1 = w1 * inv;
        const bool whole = sg.whole();
        const long long slot_idx = (long long)blockIdx.x + u;
        const int h = c.hk * a.g + (row_ok ? qr % a.g : 0);
        float* orow = whole ? nullptr : a.part_o + ((size_t)slot_idx * a.R + qr) * TC_D;
        const size_t ob = (((size_t)c.b * a.T + di) * a.Hq + h) * TC_D;
        // dimensions [64 hw, 64 hw + 64) of the row, 16 at a time; with MQ = 64
        // the high and residual lanes are summed and each thread of the pair
        // writes 8 of the 16
#pragma unroll
        for (int k4 = 0; k4 < 4; ++k4) {
          const uint32_t cc = (uint32_t)(64 * hw + 16 * k4);
          uint32_t o0[16], o1[16];
          tmem_ld32x32b_16(t_lane + C::COL_O + cc, o0);
          tmem_ld32x32b_16(t_lane + C::COL_O + TC_D + cc, o1);
          tmem_ld_wait();
          constexpr int NVAL = C::STACK ? 8 : 16;
          float ov[NVAL];
          int dbase;
          if constexpr (C::STACK) {
#pragma unroll
            for (int j = 0; j < 8; ++j) {
              // this thread keeps columns 8 cs + j and hands the other 8 to its partner
              const float mine0 = __uint_as_float(o0[j]) * s0 + __uint_as_float(o1[j]) * s1;
              const float mine1 = __uint_as_float(o0[8 + j]) * s0 + __uint_as_float(o1[8 + j]) * s1;
              const float give = cs ? mine0 : mine1;
              const float keep = cs ? mine1 : mine0;
              ov[j] = keep + __shfl_xor_sync(0xffffffffu, give, 16);
            }
            dbase = (int)cc + 8 * cs;
          } else {
#pragma unroll
            for (int j = 0; j < 16; ++j) ov[j] = __uint_as_float(o0[j]) * s0 + __uint_as_float(o1[j]) * s1;
            dbase = (int)cc;
          }
          if (row_ok) {
            if (whole) {
              if (a.out_bf16) {
                uint4* dst = reinterpret_cast<uint4*>(reinterpret_cast<__nv_bfloat16*>(a.out) + ob + dbase);
#pragma unroll
                for (int q4 = 0; q4 < NVAL / 8; ++q4)
                  dst[q4] = make_uint4(pack_bf16x2(ov[8 * q4], ov[8 * q4 + 1]), pack_bf16x2(ov[8 * q4 + 2], ov[8 * q4 + 3]),
                                       pack_bf16x2(ov[8 * q4 + 4], ov[8 * q4 + 5]), pack_bf16x2(ov[8 * q4 + 6], ov[8 * q4 + 7]));
              } else {
                float4* dst = reinterpret_cast<float4*>(reinterpret_cast<float*>(a.out) + ob + dbase);
#pragma unroll
                for (int q4 = 0; q4 < NVAL / 4; ++q4)
                  dst[q4] = make_float4(ov[4 * q4], ov[4 * q4 + 1], ov[4 * q4 + 2], ov[4 * q4 + 3]);
              }
            } else {   // partials stay in L2 for the merge (evict_last)
              const uint64_t keep = l2_evict_last();
#pragma unroll
              for (int q4 = 0; q4 < NVAL / 4; ++q4)
                st_hint4(orow + dbase + 4 * q4, make_float4(ov[4 * q4], ov[4 * q4 + 1], ov[4 * q4 + 2], ov[4 * q4 + 3]),
                         keep);
            }
          }
        }
        if (row_ok && hw == 0 && cs == 0) {
          const float lse = (L > 0.f) ? ms + fast_log2(L) : -INFINITY;
          if (!whole) st_hint(a.part_lse + (size_t)slot_idx * a.R + qr, lse, l2_evict_last());
          else if (a.out_lse) a.out_lse[ob / TC_D] = lse;
        }
        tc_fence_before();  // the O reads above precede the next segment's first PV
        named_bar_sync(1, TC_SOFTMAX_THREADS);   // sML is reused by the next segment

        g += n;
      }
    }
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == WARP_QK) tmem_dealloc(tmem, TC_TMEM_COLS);
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
  const size_t smem = TcCfg<M>::bytes(a.B);
  if (smem > 227 * 1024) return cudaErrorNotSupported;
  static PerContextOnce attr_once;
  cudaError_t e = smem_opt_in(reinterpret_cast<const void*>(decode_tc_kernel<PAGED, M>), 227 * 1024,
                              attr_once);
  if (e != cudaSuccess) return e;
  e = launch_pdl(decode_tc_kernel<PAGED, M>, dim3(a.grid), dim3(TC_THREADS), smem, st, a, mk, mv);
  if (e != cudaSuccess) return e;
  const long long warps = (long long)a.B * a.Hkv * a.R;
  return launch_pdl(combine_kernel<TC_D>, dim3((int)((warps * 32 + 255) / 256)), dim3(256),
                    combine_smem(a.B), st, a);
}

}  // namespace

cudaError_t launch_decode_tc(const DecodeArgs& a, cudaStream_t st) {
  if (a.R <= 64) return a.block_table ? launch_tc<true, 64>(a, st) : launch_tc<false, 64>(a, st);
  return a.block_table ? launch_tc<true, 128>(a, st) : launch_tc<false, 128>(a, st);
}

}  // namespace kvd

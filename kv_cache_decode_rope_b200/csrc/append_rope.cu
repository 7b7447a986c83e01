// Kernel A: RoPE on the new tokens + KV-cache append (contiguous or paged).
//
// ferric-core 0.1.0, examples/generate.rs, `step_gpu`: the new token's q and k
// are rotated at the absolute position (`rope_off_t`), v is not, and k and v
// are appended to the per-layer cache (`kc.extend`, `vc.extend`).  As in the
// ferrum-sampler 0.7.0 README ("Batched RoPE: per-item positions in single
// kernel launch") every sequence of the batch carries its own position.
//
// Work is spread as warps over all SMs: the items of one new token (b, i) --
// the 16-byte pieces of its q heads to rotate, of its k heads to rotate or
// copy, and of its v heads to copy -- are cut into groups of 32, one per
// warp.  A lane first asks for the sequence length (the only index read before
// the programmatic-dependency wait) and evaluates the inverse frequencies
// base^(-2j/r) of its pairs (r = rotated width, D unless a partial rotary
// width is asked for) while it is in flight; after the wait it issues the
// loads of its q/k/v pieces at once, so both round trips overlap.  While
// those loads are in flight the warp evaluates, in fp64, the r/2 angles
// pos * base^(-2j/r) and their sine and cosine (rope_sincos) into a table of
// its own (a warp-level sync, no block barrier): positions reach 1e5+, where
// an fp32 angle would be off by ~1e-2 rad.  Each lane then rotates the pairs
// of its piece in fp64,
// rounding once to the storage type: EPV half-split pairs (j, j + r/2) from
// two pieces, or EPV/2 interleaved pairs (2j, 2j + 1) from one.  Pieces past r
// are copied unrotated (k), or left in place (q), and v is copied.  q is
// rotated in place; k and v go to the slot of position seq_lens[b] + i.
#include <cuda_bf16.h>

#include "kvd_device.cuh"
#include "kvd_internal.h"
#include "kvd_launch.h"

namespace kvd {
namespace {

template <typename T>
struct Conv;
template <>
struct Conv<float> {
  __device__ static double to_d(float x) { return (double)x; }
  __device__ static float from_d(double x) { return __double2float_rn(x); }
};
template <>
struct Conv<__nv_bfloat16> {
  __device__ static double to_d(__nv_bfloat16 x) { return (double)__bfloat162float(x); }
  __device__ static __nv_bfloat16 from_d(double x) { return __double2bfloat16(x); }
};

constexpr int kAppendWarps = 4;   // warps per block

// sin and cos of an fp64 angle |x| < 2^31 (position x inverse frequency).
// Cody-Waite reduction by pi/2 (Cody & Waite, "Software Manual for the
// Elementary Functions", 1980): k = rint(x 2/pi), r = x - k (P1 + P2 + P3)
// with pi/2 split into three doubles.  P1 and P2 carry 22 significant bits, so
// for |k| < 2^31 the first two steps are exact, and P1 + P2 + P3 is pi/2 to
// 5e-32 relative.  The split was derived from pi by Machin's formula
// (pi = 16 atan(1/5) - 4 atan(1/239)) in exact rational arithmetic.  Then the
// Taylor series of sin and cos on |r| <= pi/4 (+ rounding of k), whose first
// omitted terms, r^21 / 21! and r^22 / 22!, are below 1e-21, and the quadrant
// k mod 4 selects the signs.  Every step is fp64; the result is within a few
// fp64 ulps of the exact sine and cosine of the fp64 angle.
__device__ __forceinline__ void rope_sincos(double x, double* sn, double* cs) {
  constexpr double kTwoOverPi = 0x1.45f306dc9c883p-1;
  constexpr double kP1 = 0x1.921fb00000000p+0;
  constexpr double kP2 = 0x1.5110b00000000p-22;
  constexpr double kP3 = 0x1.18469898cc517p-44;
  const double k = rint(x * kTwoOverPi);
  double r = fma(-k, kP1, x);
  r = fma(-k, kP2, r);
  r = fma(-k, kP3, r);
  const double r2 = r * r;
  // sin r = r + r^3 (-1/3! + r^2 (1/5! - r^2 (1/7! - ...))), to r^19
  double ps = -1.0 / 121645100408832000.0;            // -1/19!
  ps = fma(ps, r2, 1.0 / 355687428096000.0);          //  1/17!
  ps = fma(ps, r2, -1.0 / 1307674368000.0);           // -1/15!
  ps = fma(ps, r2, 1.0 / 6227020800.0);               //  1/13!
  ps = fma(ps, r2, -1.0 / 39916800.0);                // -1/11!
  ps = fma(ps, r2, 1.0 / 362880.0);                   //  1/9!
  ps = fma(ps, r2, -1.0 / 5040.0);                    // -1/7!
  ps = fma(ps, r2, 1.0 / 120.0);                      //  1/5!
  ps = fma(ps, r2, -1.0 / 6.0);                       // -1/3!
  const double s_r = fma(ps * r2, r, r);
  // cos r = 1 + r^2 (-1/2! + r^2 (1/4! - ...)), to r^20
  double pc = 1.0 / 2432902008176640000.0;            //  1/20!
  pc = fma(pc, r2, -1.0 / 6402373705728000.0);        // -1/18!
  pc = fma(pc, r2, 1.0 / 20922789888000.0);           //  1/16!
  pc = fma(pc, r2, -1.0 / 87178291200.0);             // -1/14!
  pc = fma(pc, r2, 1.0 / 479001600.0);                //  1/12!
  pc = fma(pc, r2, -1.0 / 3628800.0);                 // -1/10!
  pc = fma(pc, r2, 1.0 / 40320.0);                    //  1/8!
  pc = fma(pc, r2, -1.0 / 720.0);                     // -1/6!
  pc = fma(pc, r2, 1.0 / 24.0);                       //  1/4!
  pc = fma(pc, r2, -0.5);                             // -1/2!
  const double c_r = fma(pc, r2, 1.0);
  // x = k pi/2 + r: rotate (cos r, sin r) by k quarter turns
  const int q = (int)((long long)k & 3);
  const double sv = (q & 1) ? c_r : s_r;
  const double cv = (q & 1) ? s_r : c_r;
  *sn = (q & 2) ? -sv : sv;
  *cs = ((q + 1) & 2) ? -cv : cv;
}

template <typename T, int D>
__global__ void __launch_bounds__(kAppendWarps * 32) append_rope_kernel(AppendArgs a, int warps_per_token) {
  constexpr int EPV = 16 / (int)sizeof(T);  // elements per 16-byte vector
  constexpr int HALF = D / 2;
  constexpr int VPR = D / EPV;              // 16-byte vectors per head row
  static_assert(HALF % EPV == 0, "half head must hold whole vectors");

  __shared__ double s_tab[kAppendWarps][HALF][2];   // per warp: cos, sin of pair j

  grid_dep_launch();
  const int lane = threadIdx.x & 31;
  const int wib = threadIdx.x >> 5;
  const long long gw = (long long)blockIdx.x * kAppendWarps + wib;
  const long long tok = gw / warps_per_token;
  if (tok >= (long long)a.B * a.T) return;   // past the last token (no barrier below spans warps)
  const int wt = (int)(gw % warps_per_token);  // warp within the token
  const int b = (int)(tok / a.T);
  const int i = (int)(tok % a.T);

  // the index arrays are read before the wait (they are not written by the
  // kernel before this one); the loads complete while the wait and the q/k/v
  // loads below are pending
  const int Lraw = a.seq_lens[b];
  const int sstart = a.shard_start ? a.shard_start[b] : 0;
  // inverse frequencies base^(-2j/r) of the lane's pairs j = lane + 32 m,
  // independent of the position: evaluated while the length load is in
  // flight (pow, accurate to the last bits: at positions near 2^30 an error
  // of 1e-15 in the frequency would move the angle by 1e-6 rad)
  constexpr int NPL = (HALF + 31) / 32;        // pairs per lane (at most)
  const int RH = a.rot / 2;                     // rotated pairs per head row
  double inv_freq[NPL];
#pragma unroll
  for (int m = 0; m < NPL; ++m)
    inv_freq[m] = pow(a.rope_base, -2.0 * (double)(lane + 32 * m) / (double)a.rot);
  // everything else (q, k/v, the caches, the status word) only after the
  // previous kernel has finished
  grid_dep_wait();

  const bool store = a.k_cache != nullptr;      // no caches: rotate q only
  // per head row: RI rotation pieces, then (k only) PI pieces copied as they are
  const int RI = a.interleaved ? a.rot / EPV : RH / EPV;
  const int PI = (D - a.rot) / EPV;
  const int n_q = a.Hq * RI;
  const int n_rot = n_q + (store ? a.Hkv * (RI + PI) : 0);
  const int n_v = store ? a.Hkv * VPR : 0;
  const int w = wt * 32 + lane;                 // this lane's item

  // ---- issue this lane's loads (addresses do not depend on the position)
  int kind = 3;        // 0 q rotation, 1 k rotation, 2 k copy, 3 v copy, 4 none
  int head = 0, it = 0;
  const T* src = nullptr;
  if (w < n_q) {
    kind = 0;
    head = w / RI;
    it = w % RI;
    src = reinterpret_cast<const T*>(a.q) + (tok * a.Hq + head) * D;
  } else if (w < n_rot) {
    const int w1 = w - n_q;
    head = w1 / (RI + PI);
    it = w1 % (RI + PI);
    kind = it < RI ? 1 : 2;
    src = reinterpret_cast<const T*>(a.k_new) + (tok * a.Hkv + head) * D;
  } else if (w < n_rot + n_v) {
    const int w2 = w - n_rot;
    head = w2 / VPR;
    it = w2 % VPR;
    src = reinterpret_cast<const T*>(a.v_new) + (tok * a.Hkv + head) * D;
  } else {
    kind = 4;
  }
  // element offsets of the (up to) two 16-byte pieces
  int e0 = 0, e1 = -1;
  if (kind <= 1) {
    if (!a.interleaved) { e0 = it * EPV; e1 = RH + it * EPV; }
    else e0 = it * EPV;
  } else if (kind == 2) {
    e0 = a.rot + (it - RI) * EPV;
  } else if (kind == 3) {
    e0 = it * EPV;
  }
  uint4 ua = make_uint4(0, 0, 0, 0), ub = make_uint4(0, 0, 0, 0);
  if (kind != 4) ua = *reinterpret_cast<const uint4*>(src + e0);
  if (kind <= 1 && e1 >= 0) ub = *reinterpret_cast<const uint4*>(src + e1);

  // ---- where position pos of sequence b lives (its local slot in a shard of
  // a sequence-sharded cache); slot_base < 0 if it is outside the cache
  const long long pos = (long long)Lraw + i;
  const long long lpos = a.shard_start ? pos - sstart : pos;
  long long slot_base = -1;  // element offset of (kv head 0, lpos); heads are head_stride apart
  long long head_stride = 0;
  if (store && lpos >= 0) {
    if (a.block_table == nullptr) {
      if (lpos < a.max_seq_len) {
        slot_base = ((long long)b * a.Hkv * a.max_seq_len + lpos) * D;
        head_stride = (long long)a.max_seq_len * D;
      }
    } else {
      const long long lp = lpos / a.page_size;
      if (lp < a.max_pages_per_seq) {
        const int page = a.block_table[(long long)b * a.max_pages_per_seq + lp];
        if (page >= 0 && page < a.num_pages) {
          slot_base = ((long long)page * a.Hkv * a.page_size + lpos % a.page_size) * D;
          head_stride = (long long)a.page_size * D;
        } else if (wt == 0 && lane == 0 && a.status) {
          atomicOr(a.status, KVD_FLAG_PAGE_OUT_OF_RANGE);
        }
      }
    }
    // a shard stores only the positions inside its own range: elsewhere
    // skipping is the normal case, not an error
    if (slot_base < 0 && !a.shard_start && wt == 0 && lane == 0 && a.status)
      atomicOr(a.status, KVD_FLAG_CAPACITY);
  }

  // ---- the warp's rotation table (only warps holding rotation items)
  double (*tab)[2] = s_tab[wib];
  if (wt * 32 < n_rot) {
#pragma unroll
    for (int m = 0; m < NPL; ++m) {   // independent chains: they overlap
      const int j = lane + 32 * m;
      if (j < RH) {
        double sn, cs;
        rope_sincos((double)pos * inv_freq[m], &sn, &cs);
        tab[j][0] = cs;
        tab[j][1] = sn;
      }
    }
    __syncwarp();
  }

  // ---- copy on write of a shared boundary page: the warps of the first new
  // token copy the slots before L_b into the sequence's own page (the new
  // tokens go to later slots of that page, so the two never touch the same
  // bytes)
  if (a.cow_src && i == 0 && store) {
    const int csrc = a.cow_src[b];
    const int n = (int)(pos % a.page_size);
    if (csrc >= 0 && n > 0) {
      const long long lp = pos / a.page_size;
      const int dst = lp < a.max_pages_per_seq ? a.block_table[(long long)b * a.max_pages_per_seq + lp] : -1;
      if (csrc < a.num_pages && dst >= 0 && dst < a.num_pages) {
        const int per_tensor = a.Hkv * n * VPR;   // 16-byte pieces of one tensor
        for (int e = w; e < 2 * per_tensor; e += warps_per_token * 32) {
          const int which = e / per_tensor, r = e % per_tensor;
          const int hk = r / (n * VPR), slot = (r / VPR) % n, part = (r % VPR) * EPV;
          T* cache = reinterpret_cast<T*>(which ? a.v_cache : a.k_cache);
          const long long so = (((long long)csrc * a.Hkv + hk) * a.page_size + slot) * D + part;
          const long long doff = (((long long)dst * a.Hkv + hk) * a.page_size + slot) * D + part;
          *reinterpret_cast<uint4*>(cache + doff) = *reinterpret_cast<const uint4*>(cache + so);
        }
      } else if (wt == 0 && lane == 0 && a.status) {
        atomicOr(a.status, KVD_FLAG_PAGE_OUT_OF_RANGE);
      }
    }
  }

  // ---- rotate / copy and store
  if (kind == 4) return;
  T* dst;
  if (kind == 0) {
    dst = reinterpret_cast<T*>(a.q) + (tok * a.Hq + head) * D;
  } else {
    if (slot_base < 0) return;
    dst = reinterpret_cast<T*>(kind == 3 ? a.v_cache : a.k_cache) + slot_base + head * head_stride;
  }
  if (kind >= 2) {   // unrotated tail of k, or v
    *reinterpret_cast<uint4*>(dst + e0) = ua;
    return;
  }
  // explicit roundings: a*c - b*s and a*s + b*c, each product rounded
  if (!a.interleaved) {
    const int j0 = it * EPV;
    const T* xa = reinterpret_cast<const T*>(&ua);
    const T* xb = reinterpret_cast<const T*>(&ub);
    uint4 ra, rb;
    T* ya = reinterpret_cast<T*>(&ra);
    T* yb = reinterpret_cast<T*>(&rb);
#pragma unroll
    for (int e = 0; e < EPV; ++e) {
      const double c = tab[j0 + e][0], sn = tab[j0 + e][1];
      const double va = Conv<T>::to_d(xa[e]), vb = Conv<T>::to_d(xb[e]);
      ya[e] = Conv<T>::from_d(__dsub_rn(__dmul_rn(va, c), __dmul_rn(vb, sn)));
      yb[e] = Conv<T>::from_d(__dadd_rn(__dmul_rn(va, sn), __dmul_rn(vb, c)));
    }
    *reinterpret_cast<uint4*>(dst + e0) = ra;
    *reinterpret_cast<uint4*>(dst + e1) = rb;
  } else {
    const T* x = reinterpret_cast<const T*>(&ua);
    uint4 ru;
    T* y = reinterpret_cast<T*>(&ru);
#pragma unroll
    for (int e = 0; e < EPV; e += 2) {
      const int j = e0 / 2 + e / 2;
      const double c = tab[j][0], sn = tab[j][1];
      const double va = Conv<T>::to_d(x[e]), vb = Conv<T>::to_d(x[e + 1]);
      y[e] = Conv<T>::from_d(__dsub_rn(__dmul_rn(va, c), __dmul_rn(vb, sn)));
      y[e + 1] = Conv<T>::from_d(__dadd_rn(__dmul_rn(va, sn), __dmul_rn(vb, c)));
    }
    *reinterpret_cast<uint4*>(dst + e0) = ru;
  }
}

template <typename T>
cudaError_t launch_t(const AppendArgs& a, cudaStream_t st) {
  constexpr int EPV = 16 / (int)sizeof(T);
  const bool store = a.k_cache != nullptr;
  const int RI = a.interleaved ? a.rot / EPV : a.rot / 2 / EPV;
  const int PI = (a.D - a.rot) / EPV;
  const long long items = (long long)a.Hq * RI + (store ? (long long)a.Hkv * (RI + PI + a.D / EPV) : 0);
  const int wpt = (int)((items + 31) / 32);            // warps per token
  const long long warps = (long long)a.B * a.T * wpt;
  const long long blocks = (warps + kAppendWarps - 1) / kAppendWarps;
  if (blocks > 0x7fffffffLL) return cudaErrorNotSupported;
  const dim3 grid((unsigned)blocks), block(kAppendWarps * 32);
  switch (a.D) {
    case 16: return launch_pdl(append_rope_kernel<T, 16>, grid, block, 0, st, a, wpt);
    case 32: return launch_pdl(append_rope_kernel<T, 32>, grid, block, 0, st, a, wpt);
    case 64: return launch_pdl(append_rope_kernel<T, 64>, grid, block, 0, st, a, wpt);
    case 128: return launch_pdl(append_rope_kernel<T, 128>, grid, block, 0, st, a, wpt);
    case 256: return launch_pdl(append_rope_kernel<T, 256>, grid, block, 0, st, a, wpt);
    default: return cudaErrorNotSupported;
  }
}

}  // namespace

cudaError_t launch_append(const AppendArgs& a, int bf16, cudaStream_t st) {
  return bf16 ? launch_t<__nv_bfloat16>(a, st) : launch_t<float>(a, st);
}

}  // namespace kvd

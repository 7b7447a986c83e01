// Kernel A: RoPE on the new tokens + KV-cache append (contiguous or paged).
//
// ferric-core 0.1.0, examples/generate.rs, `step_gpu`: the new token's q and k
// are rotated at the absolute position (`rope_off_t`), v is not, and k and v
// are appended to the per-layer cache (`kc.extend`, `vc.extend`).  As in the
// ferrum-sampler 0.7.0 README ("Batched RoPE: per-item positions in single
// kernel launch") every sequence of the batch carries its own position.
//
// One CTA per new token (b, i).  The CTA first evaluates the r/2 rotation
// angles pos * base^(-2j/r) (r = rotated width, D unless a partial rotary
// width is asked for) and their sine/cosine in fp64 into shared memory
// (positions reach 1e5+, where an fp32 angle would be off by ~1e-2 rad).  Each
// thread then rotates the pairs held by 16-byte pieces of one head row, in
// fp64, rounding once to the storage type: EPV half-split pairs (j, j + r/2)
// from two pieces, or EPV/2 interleaved pairs (2j, 2j + 1) from one.  Pieces
// past r are copied unrotated (k), or left in place (q), and v is copied.  q
// is rotated in place; k and v go to the slot of position seq_lens[b] + i.
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

template <typename T, int D>
__global__ void __launch_bounds__(512) append_rope_kernel(AppendArgs a) {
  constexpr int EPV = 16 / (int)sizeof(T);  // elements per 16-byte vector
  constexpr int HALF = D / 2;
  constexpr int VPR = D / EPV;              // 16-byte vectors per head row
  static_assert(HALF % EPV == 0, "half head must hold whole vectors");

  __shared__ double s_cos[HALF];
  __shared__ double s_sin[HALF];

  grid_dep_launch();
  const int b = blockIdx.x / a.T;
  const int i = blockIdx.x % a.T;
  const long long pos = (long long)a.seq_lens[b] + i;

  const int RH = a.rot / 2;                 // rotated pairs per head row
  for (int j = threadIdx.x; j < RH; j += blockDim.x) {
    const double inv_freq = pow(a.rope_base, -2.0 * (double)j / (double)a.rot);
    double s, c;
    sincos((double)pos * inv_freq, &s, &c);
    s_cos[j] = c;
    s_sin[j] = s;
  }
  // everything above read only seq_lens: wait for the previous kernel before
  // touching q, k/v, the caches or the status word
  grid_dep_wait();

  // Where position `pos` of sequence b lives (its local slot in a shard of a
  // sequence-sharded cache); -1 if it is outside the cache.
  const bool store = a.k_cache != nullptr;      // no caches: rotate q only
  const long long lpos = a.shard_start ? pos - a.shard_start[b] : pos;
  long long slot_base = -1;  // element offset of (kv head 0, lpos); heads are `head_stride` apart
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
        } else if (threadIdx.x == 0 && a.status) {
          atomicOr(a.status, KVD_FLAG_PAGE_OUT_OF_RANGE);
        }
      }
    }
    // a shard stores only the positions inside its own range: elsewhere
    // skipping is the normal case, not an error
    if (slot_base < 0 && !a.shard_start && threadIdx.x == 0 && a.status)
      atomicOr(a.status, KVD_FLAG_CAPACITY);
  }
  __syncthreads();

  // copy on write of a shared boundary page: the first token's CTA copies the
  // slots before L_b into the sequence's own page (the new tokens go to later
  // slots of that page, so the two never touch the same bytes)
  if (a.cow_src && i == 0 && store) {
    const int src = a.cow_src[b];
    const long long L = pos;
    const int n = (int)(L % a.page_size);
    if (src >= 0 && n > 0) {
      const long long lp = L / a.page_size;
      const int dst = lp < a.max_pages_per_seq ? a.block_table[(long long)b * a.max_pages_per_seq + lp] : -1;
      if (src < a.num_pages && dst >= 0 && dst < a.num_pages) {
        const int per_tensor = a.Hkv * n * VPR;   // 16-byte pieces of one tensor
        for (int e = threadIdx.x; e < 2 * per_tensor; e += blockDim.x) {
          const int which = e / per_tensor, r = e % per_tensor;
          const int hk = r / (n * VPR), slot = (r / VPR) % n, part = (r % VPR) * EPV;
          T* cache = reinterpret_cast<T*>(which ? a.v_cache : a.k_cache);
          const long long so = (((long long)src * a.Hkv + hk) * a.page_size + slot) * D + part;
          const long long doff = (((long long)dst * a.Hkv + hk) * a.page_size + slot) * D + part;
          *reinterpret_cast<uint4*>(cache + doff) = *reinterpret_cast<const uint4*>(cache + so);
        }
      } else if (threadIdx.x == 0 && a.status) {
        atomicOr(a.status, KVD_FLAG_PAGE_OUT_OF_RANGE);
      }
    }
  }

  const long long tok = (long long)b * a.T + i;
  // per head row: RI rotation pieces, then (k only) PI pieces copied as they are
  const int RI = a.interleaved ? a.rot / EPV : RH / EPV;
  const int PI = (D - a.rot) / EPV;
  const int n_q = a.Hq * RI;
  const int n_rot = n_q + (store ? a.Hkv * (RI + PI) : 0);
  const int n_v = store ? a.Hkv * VPR : 0;
  for (int w = threadIdx.x; w < n_rot + n_v; w += blockDim.x) {
    if (w < n_rot) {
      int it;
      const T* src;
      T* dst;
      if (w < n_q) {
        const int row = w / RI;
        it = w % RI;
        T* qrow = reinterpret_cast<T*>(a.q) + (tok * a.Hq + row) * D;
        src = qrow;
        dst = qrow;
      } else {
        const int w1 = w - n_q;
        const int hk = w1 / (RI + PI);
        it = w1 % (RI + PI);
        src = reinterpret_cast<const T*>(a.k_new) + (tok * a.Hkv + hk) * D;
        if (slot_base < 0) continue;
        dst = reinterpret_cast<T*>(a.k_cache) + slot_base + hk * head_stride;
      }
      if (it >= RI) {  // unrotated tail of k
        const int e0 = a.rot + (it - RI) * EPV;
        *reinterpret_cast<uint4*>(dst + e0) = *reinterpret_cast<const uint4*>(src + e0);
        continue;
      }
      // explicit roundings: a*c - b*s and a*s + b*c, each product rounded
      if (!a.interleaved) {
        const int j0 = it * EPV;
        const uint4 ua = *reinterpret_cast<const uint4*>(src + j0);
        const uint4 ub = *reinterpret_cast<const uint4*>(src + RH + j0);
        const T* xa = reinterpret_cast<const T*>(&ua);
        const T* xb = reinterpret_cast<const T*>(&ub);
        uint4 ra, rb;
        T* ya = reinterpret_cast<T*>(&ra);
        T* yb = reinterpret_cast<T*>(&rb);
#pragma unroll
        for (int e = 0; e < EPV; ++e) {
          const double c = s_cos[j0 + e], s = s_sin[j0 + e];
          const double va = Conv<T>::to_d(xa[e]), vb = Conv<T>::to_d(xb[e]);
          ya[e] = Conv<T>::from_d(__dsub_rn(__dmul_rn(va, c), __dmul_rn(vb, s)));
          yb[e] = Conv<T>::from_d(__dadd_rn(__dmul_rn(va, s), __dmul_rn(vb, c)));
        }
        *reinterpret_cast<uint4*>(dst + j0) = ra;
        *reinterpret_cast<uint4*>(dst + RH + j0) = rb;
      } else {
        const int e0 = it * EPV;  // elements e0 .. e0 + EPV - 1: pairs e0/2 ..
        const uint4 u = *reinterpret_cast<const uint4*>(src + e0);
        const T* x = reinterpret_cast<const T*>(&u);
        uint4 ru;
        T* y = reinterpret_cast<T*>(&ru);
#pragma unroll
        for (int e = 0; e < EPV; e += 2) {
          const int j = e0 / 2 + e / 2;
          const double c = s_cos[j], s = s_sin[j];
          const double va = Conv<T>::to_d(x[e]), vb = Conv<T>::to_d(x[e + 1]);
          y[e] = Conv<T>::from_d(__dsub_rn(__dmul_rn(va, c), __dmul_rn(vb, s)));
          y[e + 1] = Conv<T>::from_d(__dadd_rn(__dmul_rn(va, s), __dmul_rn(vb, c)));
        }
        *reinterpret_cast<uint4*>(dst + e0) = ru;
      }
    } else {
      if (slot_base < 0) continue;
      const int w2 = w - n_rot;
      const int hk = w2 / VPR;
      const int part = (w2 % VPR) * EPV;
      const T* src = reinterpret_cast<const T*>(a.v_new) + (tok * a.Hkv + hk) * D + part;
      T* dst = reinterpret_cast<T*>(a.v_cache) + slot_base + hk * head_stride + part;
      *reinterpret_cast<uint4*>(dst) = *reinterpret_cast<const uint4*>(src);
    }
  }
}

template <typename T>
cudaError_t launch_t(const AppendArgs& a, cudaStream_t st) {
  const int grid = a.B * a.T;
  // one 16-byte item per thread where the heads allow (up to 512 threads), so
  // that every load of the token goes out in the first round trip
  const int work = (a.Hq + a.Hkv) * a.D / 2 + a.Hkv * a.D;  // upper bound on items
  int threads = 32;
  while (threads < 512 && threads < work / (16 / (int)sizeof(T))) threads *= 2;
  switch (a.D) {
    case 16: return launch_pdl(append_rope_kernel<T, 16>, dim3(grid), dim3(threads), 0, st, a);
    case 32: return launch_pdl(append_rope_kernel<T, 32>, dim3(grid), dim3(threads), 0, st, a);
    case 64: return launch_pdl(append_rope_kernel<T, 64>, dim3(grid), dim3(threads), 0, st, a);
    case 128: return launch_pdl(append_rope_kernel<T, 128>, dim3(grid), dim3(threads), 0, st, a);
    case 256: return launch_pdl(append_rope_kernel<T, 256>, dim3(grid), dim3(threads), 0, st, a);
    default: return cudaErrorNotSupported;
  }
}

}  // namespace

cudaError_t launch_append(const AppendArgs& a, int bf16, cudaStream_t st) {
  return bf16 ? launch_t<__nv_bfloat16>(a, st) : launch_t<float>(a, st);
}

}  // namespace kvd

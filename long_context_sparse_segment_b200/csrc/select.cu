// pbs_select_blocks: the key blocks each query block computes.
//
// "Sparser Block-Sparse Attention via Token Permutation", gist.science
// summary, "Methodik" 4 ("Block-Auswahl": block importance by mean pooling
// over the permuted keys); sciencestack.ai Figure 1 caption (every block of
// the query's own, on-diagonal segment is computed; earlier-segment blocks
// may be skipped); skillmd.com "Implementation Steps" (a fraction of the
// blocks, at least one).
//
// All decisions are taken in fp64 from fp64 block sums (exact for bf16
// rows), so that they are reproducible. One CTA per (batch, query head,
// query block):
//   a_J = sigma * qbar . kbar_J for the admissible J (one warp per J);
//   THRESHOLD: softmax over the admissible blocks, own-segment mass first,
//     then earlier blocks by descending a (ties: lower J) until mass >= tau;
//   TOPK_FRAC: the best max(0, k - own) earlier blocks, k = max(1,
//     floor(f * (I + 1)));
// then the kept flags are compacted into an ascending list.
#include <math.h>

#include "common.cuh"
#include "internal.h"

namespace pbs {
namespace {

constexpr int kThreads = 256;
constexpr int kWarps = kThreads / 32;

__host__ __device__ int next_pow2(int x) {
  int p = 1;
  while (p < x) p <<= 1;
  return p;
}

struct SelSmem {
  static size_t bytes(int nb, int d, int p2) {
    return (size_t)d * 8 + (size_t)nb * 8 * 2 + (size_t)p2 * 12 + (size_t)nb + 64 * 8;
  }
};

__device__ double block_reduce_sum(double v, double *scratch) {
#pragma unroll
  for (int o = 16; o; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  __syncthreads();
  if (lane == 0) scratch[warp] = v;
  __syncthreads();
  double s = 0.0;
  for (int w = 0; w < kWarps; ++w) s += scratch[w];
  return s;
}

__device__ double block_reduce_max(double v, double *scratch) {
#pragma unroll
  for (int o = 16; o; o >>= 1) v = fmax(v, __shfl_xor_sync(0xffffffffu, v, o));
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  __syncthreads();
  if (lane == 0) scratch[warp] = v;
  __syncthreads();
  double s = -INFINITY;
  for (int w = 0; w < kWarps; ++w) s = fmax(s, scratch[w]);
  return s;
}

// Sort (key ascending, then index ascending) for p2 entries in shared memory.
__device__ void bitonic_pairs(unsigned long long *key, int *idx, int p2) {
  for (int size = 2; size <= p2; size <<= 1) {
    for (int stride = size >> 1; stride > 0; stride >>= 1) {
      for (int i = threadIdx.x; i < p2 / 2; i += kThreads) {
        const int lo = 2 * i - (i & (stride - 1));
        const int hi = lo + stride;
        const bool asc = (lo & size) == 0;
        const unsigned long long ka = key[lo], kb = key[hi];
        const int ia = idx[lo], ib = idx[hi];
        const bool gt = ka > kb || (ka == kb && ia > ib);
        if (gt == asc) {
          key[lo] = kb;
          key[hi] = ka;
          idx[lo] = ib;
          idx[hi] = ia;
        }
      }
      __syncthreads();
    }
  }
}

__global__ void __launch_bounds__(kThreads)
    select_kernel(const double *__restrict__ qsum, const double *__restrict__ ksum, Dims dm,
                  int mode, float param, double sigma, int32_t *__restrict__ idx_out,
                  int32_t *__restrict__ cnt_out, uint8_t *__restrict__ mask_out) {
  extern __shared__ __align__(16) unsigned char smem[];
  const int nb = dm.nb, D = dm.d;
  const int I = blockIdx.x, bg = blockIdx.y;
  const int b = bg / dm.hq, g = bg % dm.hq, h = g / dm.G;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int seg = I / dm.spb;
  const int f0 = seg * dm.spb;                 // own segment: [f0, adm)
  const int adm = min(nb, f0 + dm.spb);        // admissible: [0, adm)
  const int p2 = next_pow2(f0 > 0 ? f0 : 1);

  double *qbar = reinterpret_cast<double *>(smem);
  double *a = qbar + D;
  double *pi = a + nb;
  unsigned long long *skey = reinterpret_cast<unsigned long long *>(pi + nb);
  int *sidx = reinterpret_cast<int *>(skey + p2);
  unsigned char *flag = reinterpret_cast<unsigned char *>(sidx + p2);
  double *scratch = reinterpret_cast<double *>(
      (reinterpret_cast<uintptr_t>(flag + nb) + 15) & ~(uintptr_t)15);
  __shared__ int s_taken;
  __shared__ int s_wsum[kWarps];

  for (int J = tid; J < nb; J += kThreads) flag[J] = 0;
  const bool scored = mode == PBS_SEL_THRESHOLD || mode == PBS_SEL_TOPK_FRAC;
  int taken = 0;
  if (scored) {
    const double inv_b = 1.0 / (double)dm.B;
    for (int t = tid; t < D; t += kThreads)
      qbar[t] = qsum[((size_t)bg * nb + I) * D + t] * inv_b;
    __syncthreads();
    const double *kb = ksum + (size_t)(b * dm.hkv + h) * nb * D;
    for (int J = warp; J < adm; J += kWarps) {
      double s = 0.0;
      for (int t = lane; t < D; t += 32) s = fma(qbar[t], kb[(size_t)J * D + t] * inv_b, s);
#pragma unroll
      for (int o = 16; o; o >>= 1) s += __shfl_xor_sync(0xffffffffu, s, o);
      if (lane == 0) a[J] = sigma * s;
    }
    __syncthreads();
    if (f0 > 0) {
      for (int i = tid; i < p2; i += kThreads) {
        skey[i] = i < f0 ? ~f64_order_key(a[i]) : ~0ull;
        sidx[i] = i < f0 ? i : 0x7fffffff;
      }
      __syncthreads();
    }
    if (mode == PBS_SEL_THRESHOLD) {
      double mx = -INFINITY;
      for (int J = tid; J < adm; J += kThreads) mx = fmax(mx, a[J]);
      mx = block_reduce_max(mx, scratch);
      double z = 0.0;
      for (int J = tid; J < adm; J += kThreads) {
        const double e = exp(a[J] - mx);
        pi[J] = e;
        z += e;
      }
      z = block_reduce_sum(z, scratch);
      for (int J = tid; J < adm; J += kThreads) pi[J] = pi[J] / z;
      __syncthreads();
      double own = 0.0;
      for (int J = f0 + tid; J < adm; J += kThreads) own += pi[J];
      own = block_reduce_sum(own, scratch);
      const double tau = (double)param;
      if (own < tau && f0 > 0) {
        bitonic_pairs(skey, sidx, p2);
        if (tid == 0) {
          double m = own;
          int t = 0;
          while (t < f0 && m < tau) m += pi[sidx[t++]];
          s_taken = t;
        }
        __syncthreads();
        taken = s_taken;
      }
    } else {
      const int k_i = max(1, (int)floor((double)param * (double)(I + 1)));
      taken = min(f0, max(0, k_i - (adm - f0)));
      if (taken > 0) bitonic_pairs(skey, sidx, p2);
    }
    for (int t = tid; t < taken; t += kThreads) flag[sidx[t]] = 1;
    for (int J = f0 + tid; J < adm; J += kThreads) flag[J] = 1;
  } else {
    const int last = mode == PBS_SEL_ALL ? adm : I + 1;
    for (int J = tid; J < last; J += kThreads) flag[J] = 1;
  }
  __syncthreads();

  // Compact the kept flags into an ascending list.
  const size_t row = (size_t)bg * nb + I;
  int32_t *out = idx_out + row * nb;
  int running = 0;
  for (int base = 0; base < nb; base += kThreads) {
    const int J = base + tid;
    const bool f = J < nb && flag[J];
    const unsigned bal = __ballot_sync(0xffffffffu, f);
    if (lane == 0) s_wsum[warp] = __popc(bal);
    __syncthreads();
    int off = running;
    int tot = 0;
    for (int w = 0; w < kWarps; ++w) {
      if (w < warp) off += s_wsum[w];
      tot += s_wsum[w];
    }
    if (f) out[off + __popc(bal & ((1u << lane) - 1u))] = J;
    if (mask_out && J < nb) mask_out[row * nb + J] = f ? 1 : 0;
    running += tot;
    __syncthreads();
  }
  if (tid == 0) cnt_out[row] = running;
}

}  // namespace

size_t select_ws_bytes(const Dims &dm, bool need_kbar) {
  size_t q = (size_t)dm.b * dm.hq * dm.nb * dm.d * sizeof(double);
  size_t k = need_kbar ? (size_t)dm.b * dm.hkv * dm.nb * dm.d * sizeof(double) : 0;
  return q + k;
}

cudaError_t launch_select(const Dims &dm, const double *qsum, const double *ksum, int mode,
                          float param, double sigma, int32_t *idx, int32_t *cnt, uint8_t *mask,
                          int *err, cudaStream_t st) {
  (void)err;
  const int p2max = next_pow2(dm.nb);
  const size_t smem = SelSmem::bytes(dm.nb, dm.d, p2max);
  cudaError_t e =
      cudaFuncSetAttribute(select_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return e;
  select_kernel<<<dim3(dm.nb, dm.b * dm.hq), kThreads, smem, st>>>(qsum, ksum, dm, mode, param,
                                                                   sigma, idx, cnt, mask);
  return cudaGetLastError();
}

}  // namespace pbs

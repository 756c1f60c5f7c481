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
// rows). One CTA per (batch, query head, R consecutive query blocks), one
// warp per query block:
//   the pooled key blocks are staged through shared memory in chunks of 32
//   and shared by the R rows; lane l of warp w computes a_{I_w, J} for
//   J = chunk start + l as a sequential fp64 dot product;
//   THRESHOLD: softmax over the admissible blocks, own-segment mass first,
//     then earlier blocks in descending a (ties: lower J) until the mass
//     reaches tau: a warp-level bitonic sort, then a fixed-order warp
//     prefix walk finds the cut;
//   TOPK_FRAC: the first max(0, k - own) earlier blocks of the same sort,
//     k = max(1, floor(f * (I + 1)));
// then the warp compacts the kept flags into the ascending list.
#include <math.h>

#include "common.cuh"
#include "internal.h"

namespace pbs {
namespace {

constexpr int kChunk = 32;  // key blocks per staged chunk
constexpr int kMaxD = 128;
constexpr int kPad = kMaxD + 1;  // doubles per staged row: spreads banks
constexpr size_t kSmemBudget = 200 * 1024;
constexpr int kSelThreads = 256;  // 8 warps: up to 8 rows, the rest help staging

__host__ __device__ int next_pow2(int x) {
  int p = 1;
  while (p < x) p <<= 1;
  return p;
}

// bytes of dynamic shared memory for R rows per CTA
size_t sel_smem(int rows, int nb) {
  const int p2 = next_pow2(nb);
  return (size_t)kChunk * kPad * 8 + (size_t)rows * kMaxD * 8 +
         (size_t)rows * p2 * (8 + 2) + (size_t)rows * nb + 64;
}

int sel_rows(int nb) {
  int r = 8;
  while (r > 1 && sel_smem(r, nb) > kSmemBudget) r >>= 1;
  return r;
}

__device__ __forceinline__ double f64_from_order_key(unsigned long long u) {
  return __longlong_as_double((long long)((u & 0x8000000000000000ull) ? (u ^ 0x8000000000000000ull)
                                                                       : ~u));
}

__device__ __forceinline__ double warp_sum_d(double v) {
#pragma unroll
  for (int o = 16; o; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  return v;
}
__device__ __forceinline__ double warp_max_d(double v) {
#pragma unroll
  for (int o = 16; o; o >>= 1) v = fmax(v, __shfl_xor_sync(0xffffffffu, v, o));
  return v;
}

// Ascending sort of P (a power of two) (key, idx) pairs by one warp.
__device__ void warp_bitonic(unsigned long long *key, unsigned short *idx, int p2, int lane) {
  for (int size = 2; size <= p2; size <<= 1) {
    for (int stride = size >> 1; stride > 0; stride >>= 1) {
      for (int i = lane; i < p2 / 2; i += 32) {
        const int lo = 2 * i - (i & (stride - 1));
        const int hi = lo + stride;
        const bool asc = (lo & size) == 0;
        const unsigned long long ka = key[lo], kb = key[hi];
        const unsigned short ia = idx[lo], ib = idx[hi];
        const bool gt = ka > kb || (ka == kb && ia > ib);
        if (gt == asc) {
          key[lo] = kb;
          key[hi] = ka;
          idx[lo] = ib;
          idx[hi] = ia;
        }
      }
      __syncwarp();
    }
  }
}

template <int D>
__global__ void __launch_bounds__(kSelThreads)
    select_kernel(const double *__restrict__ qsum, const double *__restrict__ ksum, Dims dm,
                  int mode, float param, double sigma, int rows, int32_t *__restrict__ idx_out,
                  int32_t *__restrict__ cnt_out, uint8_t *__restrict__ mask_out) {
  extern __shared__ __align__(16) unsigned char smem[];
  const int nb = dm.nb, p2n = next_pow2(nb);
  double *kb = reinterpret_cast<double *>(smem);                     // [kChunk][kPad]
  double *qb = kb + kChunk * kPad;                                   // [rows][kMaxD]
  unsigned long long *keys = reinterpret_cast<unsigned long long *>(qb + rows * kMaxD);
  unsigned short *ids = reinterpret_cast<unsigned short *>(keys + (size_t)rows * p2n);
  unsigned char *flags = reinterpret_cast<unsigned char *>(ids + (size_t)rows * p2n);

  const int tid = threadIdx.x, w = tid >> 5, lane = tid & 31;
  const int bg = blockIdx.y, b = bg / dm.hq, g = bg % dm.hq;
  const int kv = b * dm.hkv + g / dm.G;
  const int I = blockIdx.x * rows + w;
  const bool valid = w < rows && I < nb;  // warps past `rows` only help staging
  const int seg = valid ? I / dm.spb : 0;
  const int f0 = seg * dm.spb;                  // own segment: [f0, adm)
  const int adm = valid ? min(nb, f0 + dm.spb) : 0;
  unsigned long long *key = keys + (size_t)w * p2n;
  unsigned short *id = ids + (size_t)w * p2n;
  unsigned char *flag = flags + (size_t)w * nb;
  const bool scored = mode == PBS_SEL_THRESHOLD || mode == PBS_SEL_TOPK_FRAC;
  const double inv_b = 1.0 / (double)dm.B;

  if (scored) {
    if (valid)
      for (int t = lane; t < D; t += 32) qb[w * kMaxD + t] = qsum[((size_t)bg * nb + I) * D + t] * inv_b;
    const int last = min(nb - 1, blockIdx.x * rows + rows - 1);
    const int max_adm = min(nb, (last / dm.spb + 1) * dm.spb);
    const double *kbase = ksum + (size_t)kv * nb * D;
    // Each thread holds its share of the next chunk in registers, so that the
    // global loads of chunk c+1 are in flight while chunk c is used.
    constexpr int NL = kChunk * D / kSelThreads;
    double pre[NL];
    auto fetch = [&](int c0) {
#pragma unroll
      for (int k = 0; k < NL; ++k) {
        const int e = tid + k * kSelThreads, J = c0 + e / D;
        pre[k] = J < nb ? kbase[(size_t)J * D + e % D] : 0.0;
      }
    };
    fetch(0);
    for (int c0 = 0; c0 < max_adm; c0 += kChunk) {
      __syncthreads();
#pragma unroll
      for (int k = 0; k < NL; ++k) {
        const int e = tid + k * kSelThreads;
        kb[(e / D) * kPad + e % D] = pre[k] * inv_b;
      }
      __syncthreads();
      if (c0 + kChunk < max_adm) fetch(c0 + kChunk);
      const int J = c0 + lane;
      if (J < adm) {
        const double *qr = qb + w * kMaxD;
        const double *kr = kb + lane * kPad;
        // eight interleaved partial sums (t mod 8), added pairwise at the end
        double p[8] = {0, 0, 0, 0, 0, 0, 0, 0};
        for (int t = 0; t < D; t += 8)
#pragma unroll
          for (int u = 0; u < 8; ++u) p[u] = fma(qr[t + u], kr[t + u], p[u]);
        const double s = ((p[0] + p[1]) + (p[2] + p[3])) + ((p[4] + p[5]) + (p[6] + p[7]));
        key[J] = f64_order_key(sigma * s);
      }
    }
  }
  __syncwarp();
  if (!valid) return;  // whole warp: no block-wide barrier follows

  int taken = 0;  // earlier-segment blocks kept, taken from the sorted order
  if (scored && f0 > 0) {
    const int p2 = next_pow2(f0);
    double amax = -INFINITY;
    if (mode == PBS_SEL_THRESHOLD) {
      for (int J = lane; J < adm; J += 32) amax = fmax(amax, f64_from_order_key(key[J]));
      amax = warp_max_d(amax);
    }
    double z = 0.0, own = 0.0;
    if (mode == PBS_SEL_THRESHOLD) {
      for (int J = lane; J < adm; J += 32) {
        const double e = exp(f64_from_order_key(key[J]) - amax);
        z += e;
        if (J >= f0) own += e;
      }
      z = warp_sum_d(z);
      own = warp_sum_d(own) / z;
    }
    const double tau = (double)param;
    bool need_sort;
    if (mode == PBS_SEL_THRESHOLD) {
      need_sort = own < tau;
    } else {
      const int k_i = max(1, (int)floor((double)param * (double)(I + 1)));
      taken = min(f0, max(0, k_i - (adm - f0)));
      need_sort = taken > 0;
    }
    if (need_sort) {
      __syncwarp();
      // descending a, ties to the lower J: ascending (~order key, J)
      for (int e = lane; e < p2; e += 32) {
        key[e] = e < f0 ? ~key[e] : ~0ull;
        id[e] = e < f0 ? (unsigned short)e : (unsigned short)0xffff;
      }
      __syncwarp();
      warp_bitonic(key, id, p2, lane);
      if (mode == PBS_SEL_THRESHOLD) {
        // smallest prefix whose mass brings the kept mass to tau
        const int chunk = (f0 + 31) / 32;
        const int e0 = lane * chunk, e1 = min(f0, e0 + chunk);
        double part = 0.0;
        for (int e = e0; e < e1; ++e) part += exp(f64_from_order_key(~key[e]) - amax) / z;
        double incl = part;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
          const double v = __shfl_up_sync(0xffffffffu, incl, o);
          if (lane >= o) incl += v;
        }
        double run = own + (incl - part);
        int hit = 0x7fffffff;
        for (int e = e0; e < e1; ++e) {
          run += exp(f64_from_order_key(~key[e]) - amax) / z;
          if (run >= tau) {
            hit = e;
            break;
          }
        }
#pragma unroll
        for (int o = 16; o; o >>= 1) hit = min(hit, __shfl_xor_sync(0xffffffffu, hit, o));
        taken = hit == 0x7fffffff ? f0 : hit + 1;
      }
    }
  }

  // kept flags, then the ascending list
  for (int J = lane; J < nb; J += 32) flag[J] = 0;
  __syncwarp();
  if (scored) {
    for (int e = lane; e < taken; e += 32) flag[id[e]] = 1;
    for (int J = f0 + lane; J < adm; J += 32) flag[J] = 1;
  } else {
    const int last = mode == PBS_SEL_ALL ? adm : I + 1;
    for (int J = lane; J < last; J += 32) flag[J] = 1;
  }
  __syncwarp();
  const size_t row = (size_t)bg * nb + I;
  int32_t *out = idx_out + row * nb;
  int running = 0;
  for (int base = 0; base < nb; base += 32) {
    const int J = base + lane;
    const bool f = J < nb && flag[J];
    const unsigned bal = __ballot_sync(0xffffffffu, f);
    if (f) out[running + __popc(bal & ((1u << lane) - 1u))] = J;
    if (mask_out && J < nb) mask_out[row * nb + J] = f ? 1 : 0;
    running += __popc(bal);
  }
  if (lane == 0) cnt_out[row] = running;
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
  if (dm.nb > 65535) return cudaErrorInvalidValue;
  const int rows = sel_rows(dm.nb);
  const size_t smem = sel_smem(rows, dm.nb);
  if (smem > 227 * 1024) return cudaErrorInvalidValue;
  auto kern = dm.d == 64 ? select_kernel<64> : select_kernel<128>;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return e;
  dim3 grid((dm.nb + rows - 1) / rows, dm.b * dm.hq);
  kern<<<grid, kSelThreads, smem, st>>>(qsum, ksum, dm, mode, param, sigma, rows, idx, cnt, mask);
  return cudaGetLastError();
}

}  // namespace pbs

// pbs_permute and pbs_unpermute: the segment-local key order, the gathers it
// drives, and the inverse permutation of the output rows.
//
// "Sparser Block-Sparse Attention via Token Permutation", gist.science
// summary, "Methodik" 2 (permute only inside contiguous segments of S keys,
// keep the segment order) and 3 ("Sortierung": descending global
// importance inside each segment); sciencestack.ai Lemma 3.1 (keys and
// values move together); skillmd.com "Implementation Steps" (the output is
// put back in place with the inverse permutation).
//
// Two launches per call:
//   segsort: one CTA per (batch, KV head, segment) sorts the segment's
//            importances in shared memory (bitonic network on 64-bit keys:
//            high word = descending-importance key, low word = index, so
//            equal importances keep the lower index first) -> kpos;
//   gather:  one CTA per (batch, KV head, key block) moves the block's K and
//            V rows (and the G query heads' Q rows in permuted-query mode)
//            with 16-byte loads and stores, and sums the block's permuted
//            key rows in fp64 for the pooled block scores.
// The sort output is tiny (4 bytes per key); splitting it from the gather
// lets the gather use every SM even when there are few segments.
#include "common.cuh"
#include "internal.h"

namespace pbs {
namespace {

using bf16 = __nv_bfloat16;

constexpr int kSortThreads = 1024;
constexpr int kGatherThreads = 256;

__global__ void __launch_bounds__(kSortThreads)
    segsort_kernel(const float *__restrict__ imp, int32_t *__restrict__ kpos, Dims dm, int p2) {
  extern __shared__ unsigned long long keys[];
  const int s0 = blockIdx.x * dm.S;
  const int len = min(dm.S, dm.n - s0);
  const size_t base = (size_t)blockIdx.y * dm.n + s0;
  const int tid = threadIdx.x;
  for (int i = tid; i < p2; i += kSortThreads) {
    unsigned long long key = ~0ull;
    if (i < len) {
      uint32_t desc = ~f32_order_key(imp[base + i]);
      key = ((unsigned long long)desc << 32) | (uint32_t)i;
    }
    keys[i] = key;
  }
  __syncthreads();
  for (int size = 2; size <= p2; size <<= 1) {
    for (int stride = size >> 1; stride > 0; stride >>= 1) {
      for (int i = tid; i < p2 / 2; i += kSortThreads) {
        const int lo = 2 * i - (i & (stride - 1));
        const int hi = lo + stride;
        const bool asc = (lo & size) == 0;
        unsigned long long a = keys[lo], b = keys[hi];
        if ((a > b) == asc) {
          keys[lo] = b;
          keys[hi] = a;
        }
      }
      __syncthreads();
    }
  }
  for (int i = tid; i < len; i += kSortThreads)
    kpos[base + i] = s0 + (int32_t)(uint32_t)(keys[i] & 0xffffffffull);
}

__device__ __forceinline__ void add_bf16x8(double acc[8], uint4 v) {
  const __nv_bfloat162 *h = reinterpret_cast<const __nv_bfloat162 *>(&v);
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    float2 f = __bfloat1622float2(h[i]);
    acc[2 * i] += (double)f.x;
    acc[2 * i + 1] += (double)f.y;
  }
}

// Reduce the per-thread fp64 column sums of a block over its row lanes and
// write them: red has kGatherThreads * 8 doubles.
template <int D>
__device__ __forceinline__ void reduce_block_sums(double acc[8], double *red, double *out) {
  constexpr int CPR = D / 8, RL = kGatherThreads / CPR;
  const int tid = threadIdx.x, c = tid % CPR, rl = tid / CPR;
#pragma unroll
  for (int i = 0; i < 8; ++i) red[rl * D + c * 8 + i] = acc[i];
  __syncthreads();
  if (tid < D) {
    double s = 0.0;
    for (int r = 0; r < RL; ++r) s += red[r * D + tid];
    out[tid] = s;
  }
}

template <int D>
__global__ void __launch_bounds__(kGatherThreads)
    gather_kernel(const int32_t *__restrict__ kpos, const bf16 *__restrict__ k,
                  const bf16 *__restrict__ v, const bf16 *__restrict__ q, bf16 *__restrict__ kp,
                  bf16 *__restrict__ vp, bf16 *__restrict__ qp, double *__restrict__ kbar,
                  Dims dm, int *err) {
  __shared__ double red[kGatherThreads * 8];
  constexpr int CPR = D / 8, RL = kGatherThreads / CPR;
  const int J = blockIdx.x, bh = blockIdx.y;
  const int b = bh / dm.hkv, h = bh % dm.hkv;
  const int tid = threadIdx.x, c = tid % CPR, rl = tid / CPR;
  const int seg0 = (J / dm.spb) * dm.S;
  const int seg1 = min(seg0 + dm.S, dm.n);
  const size_t row0 = (size_t)bh * dm.n;
  double acc[8] = {0, 0, 0, 0, 0, 0, 0, 0};
  for (int p = J * dm.B + rl; p < (J + 1) * dm.B; p += RL) {
    int src = kpos[row0 + p];
    if (src < seg0 || src >= seg1) {
      report(err, PBS_ERR_DEVICE_ASSERT);
      src = p;
    }
    const uint4 kv = __ldg(reinterpret_cast<const uint4 *>(k + (row0 + src) * D) + c);
    if (kp) {  // K', V' written, or only the order and the block sums
      const uint4 vv = __ldg(reinterpret_cast<const uint4 *>(v + (row0 + src) * D) + c);
      reinterpret_cast<uint4 *>(kp + (row0 + p) * D)[c] = kv;
      reinterpret_cast<uint4 *>(vp + (row0 + p) * D)[c] = vv;
    }
    add_bf16x8(acc, kv);
    if (q) {
      for (int gl = 0; gl < dm.G; ++gl) {
        const size_t qrow = (size_t)(b * dm.hq + h * dm.G + gl) * dm.n;
        const uint4 qv = __ldg(reinterpret_cast<const uint4 *>(q + (qrow + src) * D) + c);
        reinterpret_cast<uint4 *>(qp + (qrow + p) * D)[c] = qv;
      }
    }
  }
  if (kbar) reduce_block_sums<D>(acc, red, kbar + ((size_t)bh * dm.nb + J) * D);
}

template <int D>
__global__ void __launch_bounds__(kGatherThreads)
    blocksum_kernel(const bf16 *__restrict__ x, double *__restrict__ out, Dims dm) {
  __shared__ double red[kGatherThreads * 8];
  constexpr int CPR = D / 8, RL = kGatherThreads / CPR;
  const int J = blockIdx.x, hd = blockIdx.y;
  const int tid = threadIdx.x, c = tid % CPR, rl = tid / CPR;
  const size_t row0 = (size_t)hd * dm.n;
  double acc[8] = {0, 0, 0, 0, 0, 0, 0, 0};
  for (int p = J * dm.B + rl; p < (J + 1) * dm.B; p += RL)
    add_bf16x8(acc, __ldg(reinterpret_cast<const uint4 *>(x + (row0 + p) * D) + c));
  reduce_block_sums<D>(acc, red, out + ((size_t)hd * dm.nb + J) * D);
}

template <int D>
__global__ void unpermute_kernel(const bf16 *__restrict__ op, const int32_t *__restrict__ qpos,
                                 bf16 *__restrict__ out, Dims dm, size_t total_chunks,
                                 int *err) {
  constexpr int CPR = D / 8;
  for (size_t i = blockIdx.x * (size_t)blockDim.x + threadIdx.x; i < total_chunks;
       i += (size_t)gridDim.x * blockDim.x) {
    const size_t row = i / CPR;  // over b * hq * n
    const int c = (int)(i % CPR);
    const int p = (int)(row % dm.n);
    const size_t bg = row / dm.n;
    const int b = (int)(bg / dm.hq), g = (int)(bg % dm.hq);
    const int dst = qpos[((size_t)b * dm.hkv + g / dm.G) * dm.n + p];
    if (dst < 0 || dst >= dm.n) {
      report(err, PBS_ERR_DEVICE_ASSERT);
      continue;
    }
    reinterpret_cast<uint4 *>(out + (bg * dm.n + dst) * D)[c] =
        __ldg(reinterpret_cast<const uint4 *>(op + row * D) + c);
  }
}

int next_pow2(int x) {
  int p = 1;
  while (p < x) p <<= 1;
  return p;
}

}  // namespace

cudaError_t launch_segsort(const Dims &dm, const float *imp, int32_t *kpos, int *err,
                           cudaStream_t st) {
  (void)err;
  const int p2 = next_pow2(dm.S);
  const size_t smem = (size_t)p2 * 8;
  cudaError_t e =
      cudaFuncSetAttribute(segsort_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return e;
  segsort_kernel<<<dim3(dm.nseg, dm.b * dm.hkv), kSortThreads, smem, st>>>(imp, kpos, dm, p2);
  return cudaGetLastError();
}

cudaError_t launch_gather(const Dims &dm, const int32_t *kpos, const void *k, const void *v,
                          const void *q, void *kp, void *vp, void *qp, double *kbar, int *err,
                          cudaStream_t st) {
  dim3 grid(dm.nb, dm.b * dm.hkv);
  if (dm.d == 64)
    gather_kernel<64><<<grid, kGatherThreads, 0, st>>>(
        kpos, (const bf16 *)k, (const bf16 *)v, (const bf16 *)q, (bf16 *)kp, (bf16 *)vp,
        (bf16 *)qp, kbar, dm, err);
  else
    gather_kernel<128><<<grid, kGatherThreads, 0, st>>>(
        kpos, (const bf16 *)k, (const bf16 *)v, (const bf16 *)q, (bf16 *)kp, (bf16 *)vp,
        (bf16 *)qp, kbar, dm, err);
  return cudaGetLastError();
}

cudaError_t launch_blocksum(const Dims &dm, int heads, const void *x, double *out,
                            cudaStream_t st) {
  dim3 grid(dm.nb, heads);
  if (dm.d == 64)
    blocksum_kernel<64><<<grid, kGatherThreads, 0, st>>>((const bf16 *)x, out, dm);
  else
    blocksum_kernel<128><<<grid, kGatherThreads, 0, st>>>((const bf16 *)x, out, dm);
  return cudaGetLastError();
}

cudaError_t launch_unpermute(const Dims &dm, const void *op, const int32_t *qpos, void *out,
                             int *err, cudaStream_t st) {
  const size_t total = (size_t)dm.b * dm.hq * dm.n * (dm.d / 8);
  const int threads = 256;
  size_t blocks = (total + threads - 1) / threads;
  if (blocks > 148 * 16) blocks = 148 * 16;
  if (dm.d == 64)
    unpermute_kernel<64><<<(int)blocks, threads, 0, st>>>((const bf16 *)op, qpos, (bf16 *)out,
                                                          dm, total, err);
  else
    unpermute_kernel<128><<<(int)blocks, threads, 0, st>>>((const bf16 *)op, qpos, (bf16 *)out,
                                                           dm, total, err);
  return cudaGetLastError();
}

}  // namespace pbs

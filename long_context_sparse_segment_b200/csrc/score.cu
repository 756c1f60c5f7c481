// pbs_score: global key importance from the last query block.
//
// "Sparser Block-Sparse Attention via Token Permutation", gist.science
// summary, "Methodik" 3 ("Proxy-Bewertung"): the importance of every key is
// the mean attention probability that the last query block gives it.
//
// For each (batch, KV head) there are R = G*B probe rows (the last B rows of
// the G query heads of the group) and n keys. The softmax of each probe row
// runs over all n keys, so two passes over K are needed:
//   pass 1: per row, running max and sum of exp2 over the key chunks a CTA
//           owns -> partial (m, l) per (row, CTA);
//   combine: per row, global (M, 1/L);
//   pass 2: per key chunk, p = exp2(s - M) / L summed over the R rows ->
//           imp. A chunk belongs to exactly one CTA, so no atomics are used
//           and the result is deterministic.
// Logits are kept in the log2 domain: s = (q . k) * sigma * log2(e).
#include <math.h>
#include <stdlib.h>
#include <string.h>

#include "common.cuh"
#include "internal.h"

namespace pbs {
namespace {

using bf16 = __nv_bfloat16;

constexpr int kChunk = 128;  // keys per chunk
constexpr int kWarps = 8;
constexpr int kThreads = kWarps * 32;
constexpr int kMaxRowTiles = 4;  // per warp: R <= 16 * 8 * 4 = 512

int score_splits(const Dims &dm) {
  int bh = dm.b * dm.hkv;
  int nchunk = (dm.n + kChunk - 1) / kChunk;
  int s = (2 * 148 + bh - 1) / bh;
  if (s > nchunk) s = nchunk;
  return s < 1 ? 1 : s;
}

template <int D>
size_t score_smem(int R) {
  return (size_t)R * D * 2 + (size_t)kChunk * D * 2 + (size_t)kWarps * kChunk * 4;
}

template <int D>
__global__ void __launch_bounds__(kThreads, 1)
    score_kernel(const bf16 *__restrict__ q, const bf16 *__restrict__ k, float *__restrict__ imp,
                 float2 *__restrict__ partial, const float2 *__restrict__ stats, Dims dm,
                 float sl2, int pass, int nsplit) {
  extern __shared__ __align__(128) uint8_t smem[];
  const int R = dm.G * dm.B;
  bf16 *Qs = reinterpret_cast<bf16 *>(smem);
  bf16 *Ks = Qs + (size_t)R * D;
  float *red = reinterpret_cast<float *>(Ks + kChunk * D);

  const int bh = blockIdx.y, b = bh / dm.hkv, h = bh % dm.hkv;
  const int split = blockIdx.x;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int nchunk = (dm.n + kChunk - 1) / kChunk;
  constexpr int RC = D / 8;  // 16-byte chunks per row

  for (int i = tid; i < R * RC; i += kThreads) {
    int r = i / RC, c = i % RC;
    int gl = r / dm.B, row = dm.n - dm.B + r % dm.B;
    const bf16 *src = q + ((size_t)(b * dm.hq + h * dm.G + gl) * dm.n + row) * D + c * 8;
    cp_async16(&Qs[swz<D>(r, c * 8)], src);
  }
  cp_async_commit();

  // Per-thread rows: tile t covers rows rt*16 + lane/4 (+8).
  float m_run[kMaxRowTiles][2], l_run[kMaxRowTiles][2];
#pragma unroll
  for (int t = 0; t < kMaxRowTiles; ++t) {
#pragma unroll
    for (int e = 0; e < 2; ++e) {
      m_run[t][e] = -INFINITY;
      l_run[t][e] = 0.f;
      int rt = warp + t * kWarps;
      if (pass == 1 && rt * 16 < R) {
        float2 st = stats[(size_t)bh * R + rt * 16 + (lane >> 2) + e * 8];
        m_run[t][e] = st.x;
        l_run[t][e] = st.y;  // 1 / L in pass 2
      }
    }
  }

  const bf16 *kbase = k + (size_t)bh * dm.n * D;
  for (int c = split; c < nchunk; c += nsplit) {
    const int key0 = c * kChunk;
    __syncthreads();
    for (int i = tid; i < kChunk * RC; i += kThreads) {
      int j = i / RC, cc = i % RC;
      bf16 *dst = &Ks[swz<D>(j, cc * 8)];
      if (key0 + j < dm.n)
        cp_async16(dst, kbase + (size_t)(key0 + j) * D + cc * 8);
      else
        *reinterpret_cast<uint4 *>(dst) = make_uint4(0, 0, 0, 0);
    }
    cp_async_commit();
    cp_async_wait<0>();
    __syncthreads();

    const bool edge = key0 + kChunk > dm.n - dm.B;  // causal mask / tail may apply
    float colsum[16][2];
#pragma unroll
    for (int j = 0; j < 16; ++j) colsum[j][0] = colsum[j][1] = 0.f;

#pragma unroll
    for (int t = 0; t < kMaxRowTiles; ++t) {
      const int rt = warp + t * kWarps;
      if (rt * 16 >= R) break;
      float acc[16][4];
#pragma unroll
      for (int j = 0; j < 16; ++j) acc[j][0] = acc[j][1] = acc[j][2] = acc[j][3] = 0.f;
#pragma unroll
      for (int ks = 0; ks < D / 16; ++ks) {
        uint32_t a[4];
        ldsm_x4(a, &Qs[swz<D>(rt * 16 + (lane & 7) + ((lane >> 3) & 1) * 8,
                              ks * 16 + (lane >> 4) * 8)]);
#pragma unroll
        for (int np = 0; np < 8; ++np) {
          uint32_t bb[4];
          ldsm_x4(bb, &Ks[swz<D>(np * 16 + (lane & 7) + (lane >> 4) * 8,
                                 ks * 16 + ((lane >> 3) & 1) * 8)]);
          mma_16816(acc[2 * np], a, bb[0], bb[1]);
          mma_16816(acc[2 * np + 1], a, bb[2], bb[3]);
        }
      }
      // scale to log2 units and mask
#pragma unroll
      for (int e = 0; e < 2; ++e) {
        const int r = rt * 16 + (lane >> 2) + e * 8;
        const int pos = dm.n - dm.B + r % dm.B;
#pragma unroll
        for (int j = 0; j < 16; ++j)
#pragma unroll
          for (int u = 0; u < 2; ++u) {
            float s = acc[j][e * 2 + u] * sl2;
            if (edge) {
              int key = key0 + j * 8 + 2 * (lane & 3) + u;
              if (key > pos || key >= dm.n) s = -INFINITY;
            }
            acc[j][e * 2 + u] = s;
          }
      }
      if (pass == 0) {
#pragma unroll
        for (int e = 0; e < 2; ++e) {
          float mx = -INFINITY;
#pragma unroll
          for (int j = 0; j < 16; ++j) mx = fmaxf(mx, fmaxf(acc[j][e * 2], acc[j][e * 2 + 1]));
          mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 1));
          mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 2));
          const float mnew = fmaxf(m_run[t][e], mx);
          const float mu = mnew == -INFINITY ? 0.f : mnew;  // all masked so far
          float sum = 0.f;
#pragma unroll
          for (int j = 0; j < 16; ++j)
            sum += exp2f(acc[j][e * 2] - mu) + exp2f(acc[j][e * 2 + 1] - mu);
          sum += __shfl_xor_sync(0xffffffffu, sum, 1);
          sum += __shfl_xor_sync(0xffffffffu, sum, 2);
          l_run[t][e] = l_run[t][e] * exp2f(m_run[t][e] - mu) + sum;
          m_run[t][e] = mnew;
        }
      } else {
#pragma unroll
        for (int e = 0; e < 2; ++e)
#pragma unroll
          for (int j = 0; j < 16; ++j)
#pragma unroll
            for (int u = 0; u < 2; ++u)
              colsum[j][u] += exp2f(acc[j][e * 2 + u] - m_run[t][e]) * l_run[t][e];
      }
    }
    if (pass == 1) {
#pragma unroll
      for (int j = 0; j < 16; ++j)
#pragma unroll
        for (int u = 0; u < 2; ++u) {
          float v = colsum[j][u];
          v += __shfl_xor_sync(0xffffffffu, v, 4);
          v += __shfl_xor_sync(0xffffffffu, v, 8);
          v += __shfl_xor_sync(0xffffffffu, v, 16);
          if (lane < 4) red[warp * kChunk + j * 8 + 2 * lane + u] = v;
        }
      __syncthreads();
      if (tid < kChunk && key0 + tid < dm.n) {
        float s = 0.f;
        for (int w = 0; w < kWarps; ++w) s += red[w * kChunk + tid];
        imp[(size_t)bh * dm.n + key0 + tid] = s / (float)R;
      }
    }
  }

  if (pass == 0 && (lane & 3) == 0) {
#pragma unroll
    for (int t = 0; t < kMaxRowTiles; ++t) {
      const int rt = warp + t * kWarps;
      if (rt * 16 >= R) break;
#pragma unroll
      for (int e = 0; e < 2; ++e) {
        int r = rt * 16 + (lane >> 2) + e * 8;
        partial[((size_t)bh * nsplit + split) * R + r] = make_float2(m_run[t][e], l_run[t][e]);
      }
    }
  }
}

__global__ void score_combine(const float2 *__restrict__ partial, float2 *__restrict__ stats,
                              int R, int nsplit, int total) {
  int i = blockIdx.x * blockDim.x + threadIdx.x;
  if (i >= total) return;
  int bh = i / R, r = i % R;
  const float2 *p = partial + (size_t)bh * nsplit * R + r;
  float M = -INFINITY;
  for (int s = 0; s < nsplit; ++s) M = fmaxf(M, p[(size_t)s * R].x);
  float L = 0.f;
  for (int s = 0; s < nsplit; ++s) {
    float2 v = p[(size_t)s * R];
    if (v.x != -INFINITY) L += v.y * exp2f(v.x - M);
  }
  stats[i] = make_float2(M, 1.0f / L);
}

template <int D>
cudaError_t run(const Dims &dm, const void *q, const void *k, float *imp, float sigma, void *ws,
                cudaStream_t st) {
  const int R = dm.G * dm.B;
  const int nsplit = score_splits(dm);
  const int bh = dm.b * dm.hkv;
  float2 *partial = reinterpret_cast<float2 *>(ws);
  float2 *stats = partial + (size_t)bh * nsplit * R;
  size_t smem = score_smem<D>(R);
  cudaError_t e = cudaFuncSetAttribute(score_kernel<D>,
                                       cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return e;
  dim3 grid(nsplit, bh);
  const float sl2 = sigma * kLog2e;
  score_kernel<D><<<grid, kThreads, smem, st>>>((const bf16 *)q, (const bf16 *)k, imp, partial,
                                                 stats, dm, sl2, 0, nsplit);
  int total = bh * R;
  score_combine<<<(total + 255) / 256, 256, 0, st>>>(partial, stats, R, nsplit, total);
  score_kernel<D><<<grid, kThreads, smem, st>>>((const bf16 *)q, (const bf16 *)k, imp, partial,
                                                 stats, dm, sl2, 1, nsplit);
  return cudaGetLastError();
}

}  // namespace

size_t score_ws_bytes(const Dims &dm) {
  const size_t R = (size_t)dm.G * dm.B;
  const size_t bh = (size_t)dm.b * dm.hkv;
  const size_t mma = (bh * score_splits(dm) * R + bh * R) * sizeof(float2);
  const size_t tc = score_tc_supported(dm) ? score_tc_ws_bytes(dm) : 0;
  return mma > tc ? mma : tc;
}

bool score_supported(const Dims &dm) {
  const int R = dm.G * dm.B;
  return R % 16 == 0 && R <= 16 * kWarps * kMaxRowTiles &&
         (dm.d == 64 ? score_smem<64>(R) : score_smem<128>(R)) <= 227 * 1024;
}

// The tcgen05 kernel serves G*B in {128, 256, 384, 512}; the warp-MMA
// kernel every other supported shape. PBS_SCORE=mma selects the warp-MMA
// kernel for every shape (a diagnostic switch for comparing the two).
cudaError_t launch_score(const Dims &dm, const void *q, const void *k, float *imp, float sigma,
                         void *ws, int *err, cudaStream_t st) {
  const char *sel = getenv("PBS_SCORE");
  if (score_tc_supported(dm) && !(sel && strcmp(sel, "mma") == 0))
    return launch_score_tc(dm, q, k, imp, sigma, ws, err, st);
  if (dm.d == 64) return run<64>(dm, q, k, imp, sigma, ws, st);
  return run<128>(dm, q, k, imp, sigma, ws, st);
}

}  // namespace pbs

// Block-sparse causal attention over the permuted keys, on the legacy warp
// MMA path (mma.sync m16n8k16). This is the reference kernel of the library:
// simple enough to check by reading, used by the tests as a second GPU
// implementation of the forward and as the fallback for shapes the tcgen05
// kernel does not cover.
//
// "Sparser Block-Sparse Attention via Token Permutation", sciencestack.ai
// Figure 1 caption (causality is kept across segments; blocks of the
// on-diagonal segment are computed with a per-element mask) and gist.science
// summary, "Methodik" 4 (the permuted FlashAttention kernel).
//
// One CTA per (batch, query head, query block) walks the block's ascending
// list of kept key blocks. Each warp owns 16 query rows. K'/V' tiles and
// their carried positions are double-buffered in shared memory with
// cp.async. Inside the query's own segment the mask is kpos[p] <= qpos[i];
// earlier-segment blocks are fully visible. Online softmax in the log2
// domain; the row sum is reduced across the quad at the end.
#include <math.h>
#include <stdlib.h>
#include <string.h>

#include "common.cuh"
#include "internal.h"

namespace pbs {
namespace {

using bf16 = __nv_bfloat16;

template <int D, int BB>
struct MmaCfg {
  static constexpr int kWarps = BB / 16;
  static constexpr int kThreads = kWarps * 32;
  static constexpr size_t kTile = (size_t)BB * D;  // elements
  static constexpr size_t smem = (kTile + 4 * kTile) * 2 + 2 * BB * 4;
};

template <int D, int BB>
__device__ __forceinline__ void load_tile(bf16 *dst, const bf16 *src, int tid) {
  constexpr int RC = D / 8;
  for (int i = tid; i < BB * RC; i += MmaCfg<D, BB>::kThreads) {
    const int r = i / RC, c = i % RC;
    cp_async16(&dst[swz<D>(r, c * 8)], src + (size_t)r * D + c * 8);
  }
}

// The same tile with row r read from row pos[r] of `base` (the carried key
// positions of block J: the permutation applied on the fly). A position
// outside the block's segment [seg0, seg0 + span) is reported and replaced by
// the key's own index p0 + r.
template <int D, int BB>
__device__ __forceinline__ void load_tile_rows(bf16 *dst, const bf16 *base,
                                               const int32_t *__restrict__ pos, int p0, int seg0,
                                               int span, int tid, int *err) {
  constexpr int RC = D / 8;
  for (int i = tid; i < BB * RC; i += MmaCfg<D, BB>::kThreads) {
    const int r = i / RC, c = i % RC;
    int src = __ldg(pos + r);
    if ((unsigned)(src - seg0) >= (unsigned)span) {
      report(err, PBS_ERR_DEVICE_ASSERT);
      src = p0 + r;
    }
    cp_async16(&dst[swz<D>(r, c * 8)], base + (size_t)src * D + c * 8);
  }
}

// gather != 0: kp and vp are the natural K and V, read through kpos.
template <int D, int BB>
__global__ void __launch_bounds__(MmaCfg<D, BB>::kThreads, 1)
    attn_mma_kernel(const bf16 *__restrict__ q, const bf16 *__restrict__ kp,
                    const bf16 *__restrict__ vp, const int32_t *__restrict__ kpos,
                    const int32_t *__restrict__ qpos, const int32_t *__restrict__ blk_idx,
                    const int32_t *__restrict__ blk_cnt, bf16 *__restrict__ out,
                    float *__restrict__ lse, Dims dm, float sl2, int *err, int scatter,
                    int gather) {
  using C = MmaCfg<D, BB>;
  extern __shared__ __align__(128) uint8_t smem[];
  bf16 *Qs = reinterpret_cast<bf16 *>(smem);
  bf16 *Ks = Qs + C::kTile;           // [2][BB][D]
  bf16 *Vs = Ks + 2 * C::kTile;       // [2][BB][D]
  int32_t *Ps = reinterpret_cast<int32_t *>(Vs + 2 * C::kTile);  // [2][BB]

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int heads = dm.b * dm.hq;
  const int I = dm.nb - 1 - (int)(blockIdx.x / heads);  // heavy query blocks first
  const int bg = (int)(blockIdx.x % heads);
  const int b = bg / dm.hq, g = bg % dm.hq;
  const int bh = b * dm.hkv + g / dm.G;
  const size_t qrow0 = (size_t)bg * dm.n + (size_t)I * BB;
  const size_t krow0 = (size_t)bh * dm.n;
  int count = blk_cnt[(size_t)bg * dm.nb + I];
  if (count < 0 || count > dm.nb) {
    report(err, PBS_ERR_DEVICE_ASSERT);
    count = 0;
  }
  const int32_t *list = blk_idx + ((size_t)bg * dm.nb + I) * dm.nb;
  const int segI = I / dm.spb;

  load_tile<D, BB>(Qs, q + qrow0 * D, tid);
  cp_async_commit();

  auto prefetch = [&](int it, int stage) {
    int J = list[it];
    if (J < 0 || J >= dm.nb) {
      report(err, PBS_ERR_DEVICE_ASSERT);
      J = 0;
    }
    if (gather) {
      const int32_t *pos = kpos + krow0 + (size_t)J * BB;
      const int seg0 = (J / dm.spb) * dm.S;
      const int span = min(dm.S, dm.n - seg0);  // the last segment may be short
      load_tile_rows<D, BB>(Ks + stage * C::kTile, kp + krow0 * D, pos, J * BB, seg0, span, tid,
                            err);
      load_tile_rows<D, BB>(Vs + stage * C::kTile, vp + krow0 * D, pos, J * BB, seg0, span, tid,
                            err);
    } else {
      load_tile<D, BB>(Ks + stage * C::kTile, kp + (krow0 + (size_t)J * BB) * D, tid);
      load_tile<D, BB>(Vs + stage * C::kTile, vp + (krow0 + (size_t)J * BB) * D, tid);
    }
    for (int i = tid; i < BB / 4; i += C::kThreads) {
      if (kpos)
        cp_async16(&Ps[stage * BB + i * 4], kpos + krow0 + (size_t)J * BB + i * 4);
      else
        *reinterpret_cast<int4 *>(&Ps[stage * BB + i * 4]) =
            make_int4(J * BB + i * 4, J * BB + i * 4 + 1, J * BB + i * 4 + 2, J * BB + i * 4 + 3);
    }
    cp_async_commit();
  };
  if (count > 0) prefetch(0, 0);

  if (count > 0)
    cp_async_wait<1>();
  else
    cp_async_wait<0>();
  __syncthreads();
  uint32_t qf[D / 16][4];
#pragma unroll
  for (int ks = 0; ks < D / 16; ++ks)
    ldsm_x4(qf[ks], &Qs[swz<D>(warp * 16 + (lane & 7) + ((lane >> 3) & 1) * 8,
                               ks * 16 + (lane >> 4) * 8)]);

  int qp[2];
#pragma unroll
  for (int e = 0; e < 2; ++e) {
    const int r = I * BB + warp * 16 + (lane >> 2) + e * 8;
    qp[e] = qpos ? qpos[krow0 + r] : r;
  }
  float m[2] = {-INFINITY, -INFINITY}, l[2] = {0.f, 0.f};
  float o[D / 8][4];
#pragma unroll
  for (int j = 0; j < D / 8; ++j) o[j][0] = o[j][1] = o[j][2] = o[j][3] = 0.f;

  for (int it = 0; it < count; ++it) {
    const int stage = it & 1;
    if (it + 1 < count) {
      prefetch(it + 1, stage ^ 1);
      cp_async_wait<1>();
    } else {
      cp_async_wait<0>();
    }
    __syncthreads();
    const bf16 *Kt = Ks + stage * C::kTile;
    const bf16 *Vt = Vs + stage * C::kTile;
    const int32_t *Pt = Ps + stage * BB;
    const bool diag = list[it] / dm.spb == segI;

    float s[BB / 8][4];
#pragma unroll
    for (int j = 0; j < BB / 8; ++j) s[j][0] = s[j][1] = s[j][2] = s[j][3] = 0.f;
#pragma unroll
    for (int ks = 0; ks < D / 16; ++ks) {
#pragma unroll
      for (int np = 0; np < BB / 16; ++np) {
        uint32_t bb[4];
        ldsm_x4(bb, &Kt[swz<D>(np * 16 + (lane & 7) + (lane >> 4) * 8,
                               ks * 16 + ((lane >> 3) & 1) * 8)]);
        mma_16816(s[2 * np], qf[ks], bb[0], bb[1]);
        mma_16816(s[2 * np + 1], qf[ks], bb[2], bb[3]);
      }
    }
    float alpha[2];
#pragma unroll
    for (int e = 0; e < 2; ++e) {
      float mx = -INFINITY;
#pragma unroll
      for (int j = 0; j < BB / 8; ++j)
#pragma unroll
        for (int u = 0; u < 2; ++u) {
          float x = s[j][e * 2 + u] * sl2;
          if (diag && Pt[j * 8 + 2 * (lane & 3) + u] > qp[e]) x = -INFINITY;
          s[j][e * 2 + u] = x;
          mx = fmaxf(mx, x);
        }
      mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 1));
      mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 2));
      const float mnew = fmaxf(m[e], mx);
      const float mu = mnew == -INFINITY ? 0.f : mnew;
      alpha[e] = exp2f(m[e] - mu);
      float rs = 0.f;
#pragma unroll
      for (int j = 0; j < BB / 8; ++j)
#pragma unroll
        for (int u = 0; u < 2; ++u) {
          const float p = exp2f(s[j][e * 2 + u] - mu);
          s[j][e * 2 + u] = p;
          rs += p;
        }
      l[e] = l[e] * alpha[e] + rs;
      m[e] = mnew;
    }
#pragma unroll
    for (int j = 0; j < D / 8; ++j) {
      o[j][0] *= alpha[0];
      o[j][1] *= alpha[0];
      o[j][2] *= alpha[1];
      o[j][3] *= alpha[1];
    }
#pragma unroll
    for (int kk = 0; kk < BB / 16; ++kk) {
      uint32_t a[4];
      a[0] = pack_bf16(s[2 * kk][0], s[2 * kk][1]);
      a[1] = pack_bf16(s[2 * kk][2], s[2 * kk][3]);
      a[2] = pack_bf16(s[2 * kk + 1][0], s[2 * kk + 1][1]);
      a[3] = pack_bf16(s[2 * kk + 1][2], s[2 * kk + 1][3]);
#pragma unroll
      for (int np = 0; np < D / 16; ++np) {
        uint32_t bb[4];
        ldsm_x4_t(bb, &Vt[swz<D>(kk * 16 + (lane & 7) + ((lane >> 3) & 1) * 8,
                                 np * 16 + (lane >> 4) * 8)]);
        mma_16816(o[2 * np], a, bb[0], bb[1]);
        mma_16816(o[2 * np + 1], a, bb[2], bb[3]);
      }
    }
    __syncthreads();
  }

#pragma unroll
  for (int e = 0; e < 2; ++e) {
    l[e] += __shfl_xor_sync(0xffffffffu, l[e], 1);
    l[e] += __shfl_xor_sync(0xffffffffu, l[e], 2);
  }
#pragma unroll
  for (int e = 0; e < 2; ++e) {
    const int r = warp * 16 + (lane >> 2) + e * 8;
    const float inv = l[e] > 0.f ? 1.f / l[e] : 0.f;
    // the row goes to its place in the given order, or with `scatter` to its
    // query's original position (the inverse permutation, fused)
    size_t orow_i = qrow0 + r;
    if (scatter) {
      if (qp[e] < 0 || qp[e] >= dm.n) {
        report(err, PBS_ERR_DEVICE_ASSERT);
        continue;
      }
      orow_i = (size_t)bg * dm.n + qp[e];
    }
    bf16 *orow = out + orow_i * D;
#pragma unroll
    for (int j = 0; j < D / 8; ++j)
      *reinterpret_cast<uint32_t *>(orow + j * 8 + 2 * (lane & 3)) =
          pack_bf16(o[j][e * 2] * inv, o[j][e * 2 + 1] * inv);
    if (lse && (lane & 3) == 0)
      lse[orow_i] = l[e] > 0.f ? (m[e] + log2f(l[e])) * kLn2 : -INFINITY;
  }
}

template <int D, int BB>
cudaError_t run(const Dims &dm, const void *q, const void *kp, const void *vp,
                const int32_t *kpos, const int32_t *qpos, const int32_t *idx, const int32_t *cnt,
                void *out, float *lse, float sigma, int *err, bool scatter, bool gather,
                cudaStream_t st) {
  using C = MmaCfg<D, BB>;
  if (gather && !kpos) return cudaErrorInvalidValue;
  cudaError_t e = cudaFuncSetAttribute(attn_mma_kernel<D, BB>,
                                       cudaFuncAttributeMaxDynamicSharedMemorySize, (int)C::smem);
  if (e != cudaSuccess) return e;
  const unsigned grid = (unsigned)dm.b * dm.hq * dm.nb;
  attn_mma_kernel<D, BB><<<grid, C::kThreads, C::smem, st>>>(
      (const bf16 *)q, (const bf16 *)kp, (const bf16 *)vp, kpos, qpos, idx, cnt, (bf16 *)out,
      lse, dm, sigma * kLog2e, err, scatter ? 1 : 0, gather ? 1 : 0);
  return cudaGetLastError();
}

}  // namespace

cudaError_t launch_attn_mma(const Dims &dm, const void *q, const void *kp, const void *vp,
                            const int32_t *kpos, const int32_t *qpos, const int32_t *idx,
                            const int32_t *cnt, void *out, float *lse, float sigma, int *err,
                            bool scatter, bool gather, cudaStream_t st) {
  if (dm.d == 64 && dm.B == 64)
    return run<64, 64>(dm, q, kp, vp, kpos, qpos, idx, cnt, out, lse, sigma, err, scatter,
                       gather, st);
  if (dm.d == 64 && dm.B == 128)
    return run<64, 128>(dm, q, kp, vp, kpos, qpos, idx, cnt, out, lse, sigma, err, scatter,
                        gather, st);
  if (dm.d == 128 && dm.B == 64)
    return run<128, 64>(dm, q, kp, vp, kpos, qpos, idx, cnt, out, lse, sigma, err, scatter,
                        gather, st);
  return run<128, 128>(dm, q, kp, vp, kpos, qpos, idx, cnt, out, lse, sigma, err, scatter,
                       gather, st);
}

}  // namespace pbs

namespace pbs {

// The tensor-core (tcgen05) kernels serve d = 64 or 128: for B = 128 by
// default the one with two query tiles per CTA, PBS_FORWARD=tc1 the one with
// one tile per CTA; for B = 64 the two-tile kernel whose tiles pair two
// query blocks (attn_tc64.cu). The warp-MMA kernel serves every shape under
// PBS_FORWARD=mma (diagnostic switches for comparing the kernels). A
// two-tile kernel refuses to launch
// (cudaErrorInvalidConfiguration) unless it was compiled at the register
// count its register split assumes; the one-tile kernel (B = 128) or the
// warp-MMA kernel (B = 64) then runs instead.
// PBS_FAULT_INJECT=timeout makes the tcgen05 kernels skip their first K'
// load, so that their bounded waits run out and they report
// PBS_ERR_TIMEOUT (used by the failure-detection test). With `gather` (keys
// read through kpos) the one-tile kernel is not used: the warp-MMA kernel
// serves what the two-tile kernel does not.
cudaError_t launch_attn(const Dims &dm, const void *q, const void *kp, const void *vp,
                        const int32_t *kpos, const int32_t *qpos, const int32_t *idx,
                        const int32_t *cnt, void *out, float *lse, float sigma, int *err,
                        bool scatter, bool gather, cudaStream_t st) {
  const char *fwd = getenv("PBS_FORWARD");
  const bool force_mma = fwd && strcmp(fwd, "mma") == 0;
  const bool force_tc1 = fwd && strcmp(fwd, "tc1") == 0;
  const char *fi = getenv("PBS_FAULT_INJECT");
  const int fault = (fi && strcmp(fi, "timeout") == 0) ? 1 : 0;
  if (attn_tc64_supported(dm) && !force_mma) {
    OutSet one{};
    one.p[0] = out, one.n = 1, one.hq_total = dm.hq, one.head_offset = 0;
    const cudaError_t e = launch_attn_tc64(dm, q, kp, vp, kpos, qpos, idx, cnt, one, lse, sigma,
                                           err, fault, scatter, gather, st);
    if (e != cudaErrorInvalidConfiguration) return e;
  }
  if (attn_tc_supported(dm) && !force_mma) {
    if (!force_tc1 || gather) {
      OutSet one{};
      one.p[0] = out, one.n = 1, one.hq_total = dm.hq, one.head_offset = 0;
      const cudaError_t e =
          launch_attn_tc2(dm, q, kp, vp, kpos, qpos, idx, cnt, one, lse, sigma, err, fault,
                          scatter, gather, st);
      if (e != cudaErrorInvalidConfiguration) return e;
    }
    if (!gather)
      return launch_attn_tc(dm, q, kp, vp, kpos, qpos, idx, cnt, out, lse, sigma, err, fault,
                            scatter, st);
  }
  return launch_attn_mma(dm, q, kp, vp, kpos, qpos, idx, cnt, out, lse, sigma, err, scatter,
                         gather, st);
}

}  // namespace pbs

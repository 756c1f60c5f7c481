// Block-sparse causal attention over the permuted keys on the sm_100a
// tensor cores (tcgen05 MMA, TMEM accumulators, TMA tile loads).
//
// "Sparser Block-Sparse Attention via Token Permutation", sciencestack.ai
// Figure 1 caption (inter-segment causality is kept; the blocks of the
// on-diagonal segment are computed with a per-element mask, inter-segment
// blocks are fully visible or skipped) and gist.science summary, "Methodik"
// 4 (a permuted FlashAttention kernel walks the kept blocks).
//
// One CTA per (batch, query head, 128-row query block), 256 threads:
//   warp 0, one thread   TMA: the Q tile once, then K' tiles of the kept
//                        blocks into a KS-deep ring;
//   warp 2, one thread   TMA: V' tiles into a VS-deep ring;
//   warp 1, one thread   tcgen05.mma issue: S_j = Q K_j^T into one of two
//                        TMEM S buffers, then O += P_{j-1} V_{j-1} with P
//                        read from TMEM (it overwrites S_{j-1} as bf16);
//   warps 4-7            softmax, one query row per thread (TMEM lane):
//                        mask (the block's carried original key positions
//                        read from global memory for on-diagonal-segment
//                        blocks), row max, exp2, P to TMEM, lazy rescale
//                        of O, final normalisation and store.
// S_{j+1} is computed while the softmax works on S_j. The running max is
// only moved when it grows by more than 2^8, so O is rescaled rarely.
// Every mbarrier wait is bounded; on expiry the CTA records PBS_ERR_TIMEOUT,
// drains what it issued, frees TMEM and exits.
#include <math.h>
#include <stdlib.h>
#include <string.h>

#include <mutex>

#include "common.cuh"
#include "internal.h"
#include "tc.cuh"

namespace pbs {
namespace {

using bf16 = __nv_bfloat16;
using namespace tc;

constexpr int kBM = 128;  // query rows per tile (MMA M)
constexpr int kBN = 128;  // keys per block
constexpr int KS = 3;     // K' ring depth
constexpr int VS = 2;     // V' ring depth
constexpr int kThreads = 256;
constexpr float kRescaleLog2 = 8.0f;  // move the running max only past 2^8

template <int D>
struct Cfg {
  static constexpr int H = D / 64;                          // 128-byte atoms per row
  static constexpr uint32_t TILE = (uint32_t)kBM * D * 2;  // bytes per 128-row tile
  static constexpr uint32_t HALF = (uint32_t)kBM * 128;    // bytes per 64-column half
  static constexpr size_t smem = 1024 + (size_t)TILE * (1 + KS + VS) + 256;
};

struct Bars {
  uint64_t q_full, k_full[KS], k_empty[KS], v_full[VS], v_empty[VS], s_full[2], p_full[2],
      o_ready, mma_done;
};

template <int D>
__global__ void __launch_bounds__(kThreads, 1)
    attn_tc_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
                   const __grid_constant__ CUtensorMap tmV, const int32_t *__restrict__ kpos,
                   const int32_t *__restrict__ qpos, const int32_t *__restrict__ blk_idx,
                   const int32_t *__restrict__ blk_cnt, bf16 *__restrict__ out,
                   float *__restrict__ lse, Dims dm, float sl2, int *err, int fault) {
  using C = Cfg<D>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t *base = reinterpret_cast<uint8_t *>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~(uintptr_t)1023);
  uint8_t *sQ = base;
  uint8_t *sK = sQ + C::TILE;
  uint8_t *sV = sK + KS * C::TILE;
  Bars *bar = reinterpret_cast<Bars *>(sV + VS * C::TILE);
  uint32_t *s_tmem = reinterpret_cast<uint32_t *>(bar + 1);
  volatile int *s_abort = reinterpret_cast<volatile int *>(s_tmem + 1);

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int heads = dm.b * dm.hq;
  const int I = dm.nb - 1 - (int)(blockIdx.x / heads);  // heavy query blocks first
  const int bg = (int)(blockIdx.x % heads);
  const int b = bg / dm.hq, g = bg % dm.hq;
  const int bh = b * dm.hkv + g / dm.G;
  const int32_t *list = blk_idx + ((size_t)bg * dm.nb + I) * dm.nb;
  int count = blk_cnt[(size_t)bg * dm.nb + I];
  if (count < 0 || count > dm.nb) {
    if (tid == 0) report(err, PBS_ERR_DEVICE_ASSERT);
    count = 0;
  }

  if (tid == 0) {
    mbar_init(&bar->q_full, 1);
    for (int s = 0; s < KS; ++s) {
      mbar_init(&bar->k_full[s], 1);
      mbar_init(&bar->k_empty[s], 1);
    }
    for (int s = 0; s < VS; ++s) {
      mbar_init(&bar->v_full[s], 1);
      mbar_init(&bar->v_empty[s], 1);
    }
    for (int s = 0; s < 2; ++s) {
      mbar_init(&bar->s_full[s], 1);
      mbar_init(&bar->p_full[s], 128);
    }
    mbar_init(&bar->o_ready, 1);
    mbar_init(&bar->mma_done, 1);
    *s_abort = 0;
    fence_barrier_init();
  }
  if (warp == 1) {
    tmem_alloc(s_tmem, 512);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tbase = *s_tmem;
  const uint32_t tO = tbase + 256;

  auto block_at = [&](int j) {
    int J = list[j];
    if (J < 0 || J >= dm.nb) {
      report(err, PBS_ERR_DEVICE_ASSERT);
      J = 0;
    }
    return J;
  };

  if (warp == 0 && lane == 0) {
    // ---------------------------------------------------- Q and K' loads
    int issued = 0;
    if (count > 0) {
      prefetch_map(&tmQ);
      prefetch_map(&tmK);
      mbar_expect_tx(&bar->q_full, C::TILE);
      for (int h = 0; h < C::H; ++h)
        tma_load_2d(sQ + h * C::HALF, &tmQ, &bar->q_full, h * 64, bg * dm.n + I * kBM);
    }
    for (int j = 0; j < count; ++j) {
      const int s = j % KS, u = j / KS;
      if (u > 0 && !mbar_wait(&bar->k_empty[s], (u - 1) & 1, s_abort, err, 11)) break;
      const int J = block_at(j);
      mbar_expect_tx(&bar->k_full[s], C::TILE);
      if (!(fault == 1 && j == 0))
        for (int h = 0; h < C::H; ++h)
          tma_load_2d(sK + s * C::TILE + h * C::HALF, &tmK, &bar->k_full[s], h * 64,
                      bh * dm.n + J * kBN);
      issued = j + 1;
    }
    // drain: every copy this thread started lands before the CTA exits
    int never = 0;
    if (count > 0) mbar_wait(&bar->q_full, 0, &never, nullptr);
    for (int t = issued > KS ? issued - KS : 0; t < issued; ++t)
      if (!(fault == 1 && t == 0)) mbar_wait(&bar->k_full[t % KS], (t / KS) & 1, &never, nullptr);
  } else if (warp == 2 && lane == 0) {
    // ------------------------------------------- V' and key position loads
    int issued = 0;
    if (count > 0) prefetch_map(&tmV);
    for (int j = 0; j < count; ++j) {
      const int s = j % VS, u = j / VS;
      if (u > 0 && !mbar_wait(&bar->v_empty[s], (u - 1) & 1, s_abort, err, 21)) break;
      const int J = block_at(j);
      mbar_expect_tx(&bar->v_full[s], C::TILE);
      for (int h = 0; h < C::H; ++h)
        tma_load_2d(sV + s * C::TILE + h * C::HALF, &tmV, &bar->v_full[s], h * 64,
                    bh * dm.n + J * kBN);
      issued = j + 1;
    }
    int never = 0;
    for (int t = issued > VS ? issued - VS : 0; t < issued; ++t)
      mbar_wait(&bar->v_full[t % VS], (t / VS) & 1, &never, nullptr);
  } else if (warp == 1 && lane == 0) {
    // -------------------------------------------------------- MMA issue
    constexpr uint32_t kIdQK = idesc_bf16(kBM, kBN, false);
    constexpr uint32_t kIdPV = idesc_bf16(kBM, D, true);
    const uint32_t aQ = smem_u32(sQ), aK = smem_u32(sK), aV = smem_u32(sV);
    if (count > 0 && mbar_wait(&bar->q_full, 0, s_abort, err, 31)) {
      tc_fence_after();
      for (int j = 0; j <= count; ++j) {
        if (j < count) {
          const int s = j % KS;
          if (!mbar_wait(&bar->k_full[s], (j / KS) & 1, s_abort, err, 32)) break;
          tc_fence_after();
          const uint32_t tS = tbase + (uint32_t)(j & 1) * 128;
#pragma unroll
          for (int ks = 0; ks < D / 16; ++ks) {
            const uint32_t off = (uint32_t)(ks >> 2) * C::HALF + (uint32_t)(ks & 3) * 32;
            mma_ss(tS, sw128_desc(aQ + off, 16, 1024),
                   sw128_desc(aK + s * C::TILE + off, 16, 1024), kIdQK, ks > 0);
          }
          mma_commit(&bar->k_empty[s]);
          mma_commit(&bar->s_full[j & 1]);
        }
        if (j >= 1) {
          const int i = j - 1, sv = i % VS;
          if (!mbar_wait(&bar->p_full[i & 1], (i >> 1) & 1, s_abort, err, 33)) break;
          if (!mbar_wait(&bar->v_full[sv], (i / VS) & 1, s_abort, err, 34)) break;
          tc_fence_after();
          const uint32_t tP = tbase + (uint32_t)(i & 1) * 128;
#pragma unroll
          for (int kk = 0; kk < kBN / 16; ++kk)
            mma_ts(tO, tP + kk * 8, sw128_desc(aV + sv * C::TILE + kk * 2048, C::HALF, 1024),
                   kIdPV, (i > 0 || kk > 0) ? 1u : 0u);
          mma_commit(&bar->v_empty[sv]);
          mma_commit(&bar->o_ready);
        }
      }
    }
    // drain: every MMA issued here completes before TMEM is released
    mma_commit(&bar->mma_done);
    int never = 0;
    mbar_wait(&bar->mma_done, 0, &never, nullptr);
  } else if (warp >= 4) {
    // ---------------------------------------------------------- softmax
    const int quarter = warp - 4;
    const int row = quarter * 32 + lane;
    const uint32_t lane_off = (uint32_t)(quarter * 32) << 16;
    const int qrow = I * kBM + row;
    const int qp = qpos ? qpos[(size_t)bh * dm.n + qrow] : qrow;
    const int segI = I / dm.spb;
    float m_used = -INFINITY, l = 0.f;
    bool ok = count > 0;
    for (int j = 0; j < count && ok; ++j) {
      const int J = list[j];
      const bool diag = J / dm.spb == segI;
      const uint32_t tS = tbase + (uint32_t)(j & 1) * 128 + lane_off;
      if (!mbar_wait_warp(&bar->s_full[j & 1], (j >> 1) & 1, s_abort, err, 41)) {
        ok = false;
        break;
      }
      tc_fence_after();
      float s[kBN];
      {
        uint32_t r0[32], r1[32], r2[32], r3[32];
        tmem_ld32(tS, r0);
        tmem_ld32(tS + 32, r1);
        tmem_ld32(tS + 64, r2);
        tmem_ld32(tS + 96, r3);
        tmem_wait_ld();
#pragma unroll
        for (int e = 0; e < 32; ++e) {
          s[e] = __uint_as_float(r0[e]);
          s[32 + e] = __uint_as_float(r1[e]);
          s[64 + e] = __uint_as_float(r2[e]);
          s[96 + e] = __uint_as_float(r3[e]);
        }
      }
      if (diag) {
        if (kpos) {
          // the block's carried original positions: the same 512 bytes for
          // every thread, read as 16-byte broadcast loads
          const int4 *kp4 = reinterpret_cast<const int4 *>(kpos + (size_t)bh * dm.n +
                                                           (size_t)(J < 0 || J >= dm.nb ? 0 : J) * kBN);
#pragma unroll
          for (int c4 = 0; c4 < kBN / 4; ++c4) {
            const int4 p = __ldg(kp4 + c4);
            if (p.x > qp) s[4 * c4] = -INFINITY;
            if (p.y > qp) s[4 * c4 + 1] = -INFINITY;
            if (p.z > qp) s[4 * c4 + 2] = -INFINITY;
            if (p.w > qp) s[4 * c4 + 3] = -INFINITY;
          }
        } else {
#pragma unroll
          for (int c = 0; c < kBN; ++c)
            if (J * kBN + c > qp) s[c] = -INFINITY;
        }
      }
      // row max as 8 independent chains (one warp per scheduler: no other
      // warp hides a 128-long dependent chain)
      float m8[8];
#pragma unroll
      for (int t = 0; t < 8; ++t) m8[t] = s[t];
#pragma unroll
      for (int c = 8; c < kBN; c += 8)
#pragma unroll
        for (int t = 0; t < 8; ++t) m8[t] = fmaxf(m8[t], s[c + t]);
      const float mx = fmaxf(fmaxf(fmaxf(m8[0], m8[1]), fmaxf(m8[2], m8[3])),
                             fmaxf(fmaxf(m8[4], m8[5]), fmaxf(m8[6], m8[7])));
      const float mxs = mx * sl2;
      float alpha = 1.f;
      if (mxs > m_used + kRescaleLog2) {
        alpha = exp2f(m_used - mxs);
        m_used = mxs;
      }
      const float mu = m_used == -INFINITY ? 0.f : m_used;
      __syncwarp();  // reconverge after the per-row mask before the aligned stores
      // p = 2^(s * sigma * log2(e) - m): packed fp32x2 FMA, the hardware
      // exp2, four packed partial sums; P goes to TMEM as bf16 pairs over
      // the first 64 columns of this S buffer.
      const float2 scale2 = make_float2(sl2, sl2), neg_m2 = make_float2(-mu, -mu);
      float2 acc[4] = {make_float2(0.f, 0.f), make_float2(0.f, 0.f), make_float2(0.f, 0.f),
                       make_float2(0.f, 0.f)};
#pragma unroll
      for (int c = 0; c < kBN / 32; ++c) {
        uint32_t pk[16];
#pragma unroll
        for (int e = 0; e < 16; ++e) {
          const float2 x =
              __ffma2_rn(make_float2(s[c * 32 + 2 * e], s[c * 32 + 2 * e + 1]), scale2, neg_m2);
          // 5 of every 16 pairs on the FMA pipe, the rest on MUFU
          const float2 p = (e % 3 == 2) ? exp2_poly2(x)
                                        : make_float2(ex2_approx(x.x), ex2_approx(x.y));
          acc[e & 3] = __fadd2_rn(acc[e & 3], p);
          pk[e] = pack_bf16(p.x, p.y);
        }
        tmem_st16(tS + c * 16, pk);
      }
      const float2 a01 = __fadd2_rn(acc[0], acc[1]), a23 = __fadd2_rn(acc[2], acc[3]);
      const float2 a = __fadd2_rn(a01, a23);
      tmem_wait_st();
      l = l * alpha + (a.x + a.y);
      if (j >= 1) {
        if (!mbar_wait_warp(&bar->o_ready, (j - 1) & 1, s_abort, err, 43)) {
          ok = false;
          break;
        }
        tc_fence_after();
        // The rescale decision is per row, but tcgen05.ld/st are warp-wide
        // (.sync.aligned): the whole warp takes the branch when any row needs
        // it, and rows with alpha == 1 multiply by one.
        if (__any_sync(0xffffffffu, alpha != 1.f)) {
          uint32_t r[32];
#pragma unroll
          for (int c = 0; c < D / 32; ++c) {
            tmem_ld32(tO + lane_off + c * 32, r);
            tmem_wait_ld();
#pragma unroll
            for (int e = 0; e < 32; ++e) r[e] = __float_as_uint(__uint_as_float(r[e]) * alpha);
            tmem_st32(tO + lane_off + c * 32, r);
          }
          tmem_wait_st();
        }
      }
      tc_fence_before();
      mbar_arrive(&bar->p_full[j & 1]);
    }
    if (ok && !mbar_wait_warp(&bar->o_ready, (count - 1) & 1, s_abort, err, 44)) ok = false;
    bf16 *orow = out + ((size_t)bg * dm.n + qrow) * D;
    if (ok) {
      tc_fence_after();
      const float inv = l > 0.f ? 1.f / l : 0.f;
      uint32_t r[32];
#pragma unroll
      for (int c = 0; c < D / 32; ++c) {
        tmem_ld32(tO + lane_off + c * 32, r);
        tmem_wait_ld();
        uint32_t pk[16];
#pragma unroll
        for (int e = 0; e < 16; ++e)
          pk[e] = pack_bf16(__uint_as_float(r[2 * e]) * inv, __uint_as_float(r[2 * e + 1]) * inv);
        uint4 *dst = reinterpret_cast<uint4 *>(orow + c * 32);
#pragma unroll
        for (int v = 0; v < 4; ++v)
          dst[v] = make_uint4(pk[4 * v], pk[4 * v + 1], pk[4 * v + 2], pk[4 * v + 3]);
      }
      if (lse)
        lse[(size_t)bg * dm.n + qrow] = l > 0.f ? (m_used + log2f(l)) * kLn2 : -INFINITY;
    } else if (count == 0) {
      for (int c = 0; c < D / 8; ++c)
        reinterpret_cast<uint4 *>(orow)[c] = make_uint4(0, 0, 0, 0);
      if (lse) lse[(size_t)bg * dm.n + qrow] = -INFINITY;
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    __syncwarp();
    tc_fence_after();
    tmem_dealloc(tbase, 512);
  }
}

// ------------------------------------------------------------- host side
typedef CUresult (*EncodeTiled)(CUtensorMap *, CUtensorMapDataType, cuuint32_t, void *,
                                const cuuint64_t *, const cuuint64_t *, const cuuint32_t *,
                                const cuuint32_t *, CUtensorMapInterleave, CUtensorMapSwizzle,
                                CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiled encode_fn() {
  static EncodeTiled fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void *p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) ==
            cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<EncodeTiled>(p);
  });
  return fn;
}

// [rows, d] bf16 rows, 128 x 64 boxes with the 128-byte swizzle.
bool make_map(CUtensorMap *map, const void *ptr, uint64_t rows, int d) {
  EncodeTiled enc = encode_fn();
  if (!enc) return false;
  cuuint64_t dims[2] = {(cuuint64_t)d, (cuuint64_t)rows};
  cuuint64_t strides[1] = {(cuuint64_t)d * 2};
  cuuint32_t box[2] = {64, 128};
  cuuint32_t estr[2] = {1, 1};
  return enc(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void *>(ptr), dims, strides,
             box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
             CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
             CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

template <int D>
cudaError_t run(const Dims &dm, const void *q, const void *kp, const void *vp,
                const int32_t *kpos, const int32_t *qpos, const int32_t *idx, const int32_t *cnt,
                void *out, float *lse, float sigma, int *err, int fault, cudaStream_t st) {
  CUtensorMap mq, mk, mv;
  if (!make_map(&mq, q, (uint64_t)dm.b * dm.hq * dm.n, D) ||
      !make_map(&mk, kp, (uint64_t)dm.b * dm.hkv * dm.n, D) ||
      !make_map(&mv, vp, (uint64_t)dm.b * dm.hkv * dm.n, D))
    return cudaErrorInvalidValue;
  const size_t smem = Cfg<D>::smem;
  cudaError_t e = cudaFuncSetAttribute(attn_tc_kernel<D>,
                                       cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return e;
  const unsigned grid = (unsigned)dm.b * dm.hq * dm.nb;
  attn_tc_kernel<D><<<grid, kThreads, smem, st>>>(mq, mk, mv, kpos, qpos, idx, cnt,
                                                  (bf16 *)out, lse, dm, sigma * kLog2e, err,
                                                  fault);
  return cudaGetLastError();
}

}  // namespace

bool attn_tc_supported(const Dims &dm) { return dm.B == 128 && (dm.d == 128 || dm.d == 64); }

cudaError_t launch_attn_tc(const Dims &dm, const void *q, const void *kp, const void *vp,
                           const int32_t *kpos, const int32_t *qpos, const int32_t *idx,
                           const int32_t *cnt, void *out, float *lse, float sigma, int *err,
                           int fault, cudaStream_t st) {
  if (dm.d == 64) return run<64>(dm, q, kp, vp, kpos, qpos, idx, cnt, out, lse, sigma, err, fault, st);
  return run<128>(dm, q, kp, vp, kpos, qpos, idx, cnt, out, lse, sigma, err, fault, st);
}

}  // namespace pbs

// Block-sparse causal attention over the permuted keys on the sm_100a
// tensor cores (tcgen05 MMA, TMEM accumulators, TMA tile loads).
//
// "Sparser Block-Sparse Attention via Token Permutation", sciencestack.ai
// Figure 1 caption (inter-segment causality is kept; the blocks of the
// on-diagonal segment are computed with a per-element mask, inter-segment
// blocks are fully visible or skipped) and gist.science summary, "Methodik"
// 4 (a permuted FlashAttention kernel walks the kept blocks).
//
// One CTA per (batch, query head, 128-row query block), 384 threads:
//   warp 0, one thread   TMA: the Q tile once, then K' tiles of the kept
//                        blocks into a KS-deep ring;
//   warp 2, one thread   TMA: V' tiles into a VS-deep ring;
//   warp 1, one thread   tcgen05.mma issue: S_j = Q K_j^T into one of two
//                        TMEM S buffers, then O += P_{j-1} V_{j-1} with P
//                        read from TMEM (it overwrites S_{j-1} as bf16);
//   warps 4-11           softmax, two threads per query row (TMEM lane),
//                        each on half of the key and output columns:
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
constexpr int VS = 3;     // V' ring depth
constexpr int kSoftmaxThreads = 256;  // two threads per query row
constexpr int kSoftmaxWarps = kSoftmaxThreads / 32;
constexpr int kThreads = 128 + kSoftmaxThreads;
constexpr float kRescaleLog2 = 8.0f;  // move the running max only past 2^8

struct Bars {
  uint64_t q_full, k_full[KS], k_empty[KS], v_full[VS], v_empty[VS], s_full[2], p_full[2],
      o_ready, mma_done, xchg[2], lsum;
};

// Row statistics the two threads of a row hand each other.
struct Xchg {
  float mx[2][2][kBM];  // [block parity][half][row] partial row max
  float l[2][kBM];      // [half][row] partial row sum
  int32_t kp[3][kBN];   // carried key positions of blocks j, j+1, j+2 (by j % 3)
};

template <int D>
struct Cfg {
  static constexpr int H = D / 64;                          // 128-byte atoms per row
  static constexpr uint32_t TILE = (uint32_t)kBM * D * 2;  // bytes per 128-row tile
  static constexpr uint32_t HALF = (uint32_t)kBM * 128;    // bytes per 64-column half
  static constexpr size_t smem =
      1024 + (size_t)TILE * (KS + VS) + sizeof(Bars) + sizeof(Xchg) + 64;
};

template <int D>
__global__ void __launch_bounds__(kThreads, 1)
    attn_tc_kernel(const bf16 *__restrict__ q, const __grid_constant__ CUtensorMap tmK,
                   const __grid_constant__ CUtensorMap tmV, const int32_t *__restrict__ kpos,
                   const int32_t *__restrict__ qpos, const int32_t *__restrict__ blk_idx,
                   const int32_t *__restrict__ blk_cnt, bf16 *__restrict__ out,
                   float *__restrict__ lse, Dims dm, float sl2, int *err, int fault,
                   int scatter) {
  using C = Cfg<D>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t *base = reinterpret_cast<uint8_t *>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~(uintptr_t)1023);
  uint8_t *sK = base;
  uint8_t *sV = sK + KS * C::TILE;
  Bars *bar = reinterpret_cast<Bars *>(sV + VS * C::TILE);
  Xchg *xc = reinterpret_cast<Xchg *>(bar + 1);
  uint32_t *s_tmem = reinterpret_cast<uint32_t *>(xc + 1);
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
    mbar_init(&bar->q_full, kSoftmaxWarps);
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
      mbar_init(&bar->p_full[s], kSoftmaxWarps);
      mbar_init(&bar->xchg[s], kSoftmaxWarps);
    }
    mbar_init(&bar->o_ready, 1);
    mbar_init(&bar->mma_done, 1);
    mbar_init(&bar->lsum, kSoftmaxWarps);
    *s_abort = 0;
    fence_barrier_init();
  }
  if (warp == 1) {
    tmem_alloc(s_tmem, 512);
    tmem_relinquish();
  }
  // The first softmax warp stages the carried key positions of the
  // on-diagonal-segment blocks two blocks ahead (blocks 0 and 1 here); the
  // row-max exchange barrier of the block in between publishes them.
  auto stage_positions = [&](int j) {
    if (!kpos || j >= count) return;
    const int J = list[j];
    if (J < 0 || J >= dm.nb || J / dm.spb != I / dm.spb) return;
    cp_async16(&xc->kp[j % 3][lane * 4], kpos + (size_t)bh * dm.n + (size_t)J * kBN + lane * 4);
    cp_async_commit();
  };
  if (warp == 4) {
    stage_positions(0);
    stage_positions(1);
    cp_async_wait<0>();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tbase = *s_tmem;
  const uint32_t tO = tbase + 256;  // O: columns 256 .. 256 + D
  const uint32_t tQ = tbase + 384;  // Q: columns 384 .. 384 + D/2, bf16 pairs

  auto block_at = [&](int j) {
    int J = list[j];
    if (J < 0 || J >= dm.nb) {
      report(err, PBS_ERR_DEVICE_ASSERT);
      J = 0;
    }
    return J;
  };

  if (warp == 0 && lane == 0) {
    // ------------------------------------------------------- K' loads
    int issued = 0;
    if (count > 0) prefetch_map(&tmK);
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
    // Shared-memory descriptors as two 32-bit words: {lo + byte offset / 16,
    // hi}. The address field never overflows (shared memory < 256 KB), so a
    // tile's descriptor is one add away from the ring's base descriptor.
    const uint32_t hi = sw128_desc_hi(1024);
    const uint32_t lo_k = sw128_desc_lo(smem_u32(sK), 16);
    const uint32_t lo_v = sw128_desc_lo(smem_u32(sV), C::HALF);
    int ks = 0, kph = 0;  // K' ring slot and phase of block j
    int vs = 0, vph = 0;  // V' ring slot and phase of block j - 1
    if (count > 0 && mbar_wait(&bar->q_full, 0, s_abort, err, 31)) {
      tc_fence_after();
      for (int j = 0; j <= count; ++j) {
        if (j < count) {
          if (!mbar_wait(&bar->k_full[ks], kph, s_abort, err, 32)) break;
          tc_fence_after();
          const uint32_t tS = tbase + (uint32_t)(j & 1) * 128;
          const uint32_t lo = lo_k + ks * (C::TILE >> 4);
#pragma unroll
          for (int kk = 0; kk < D / 16; ++kk)  // A = Q from TMEM, B = K' (K-major)
            mma_ts(tS, tQ + kk * 8,
                   desc_words(lo + ((kk >> 2) * C::HALF + (kk & 3) * 32) / 16, hi), kIdQK,
                   kk > 0);
          mma_commit(&bar->k_empty[ks]);
          mma_commit(&bar->s_full[j & 1]);
          if (++ks == KS) ks = 0, kph ^= 1;
        }
        if (j >= 1) {
          const int i = j - 1;
          if (!mbar_wait(&bar->p_full[i & 1], (i >> 1) & 1, s_abort, err, 33)) break;
          if (!mbar_wait(&bar->v_full[vs], vph, s_abort, err, 34)) break;
          tc_fence_after();
          const uint32_t tP = tbase + (uint32_t)(i & 1) * 128;
          const uint32_t lo = lo_v + vs * (C::TILE >> 4);
#pragma unroll
          for (int kk = 0; kk < kBN / 16; ++kk)  // A = P from TMEM, B = V' (MN-major)
            mma_ts(tO, tP + kk * 8, desc_words(lo + kk * (2048 / 16), hi), kIdPV,
                   (i > 0 || kk > 0) ? 1u : 0u);
          mma_commit(&bar->v_empty[vs]);
          mma_commit(&bar->o_ready);
          if (++vs == VS) vs = 0, vph ^= 1;
        }
      }
    }
    // drain: every MMA issued here completes before TMEM is released
    mma_commit(&bar->mma_done);
    int never = 0;
    mbar_wait(&bar->mma_done, 0, &never, nullptr);
  } else if (warp >= 4) {
    // ---------------------------------------------------------- softmax
    // Two threads per query row: warps 4-7 take key (and output) columns in
    // the first half, warps 8-11 the second half, of the same TMEM lanes.
    // The pair agrees on the row max through shared memory once per block
    // (a bounded mbarrier, so an abort cannot leave a thread stranded) and
    // adds its two row sums at the end.
    constexpr int OC = D / 2;  // output columns per thread
    const int sw = warp - 4;
    const int quarter = sw & 3, half = sw >> 2;
    const int row = quarter * 32 + lane;
    const uint32_t lane_off = (uint32_t)(quarter * 32) << 16;
    const int col0 = half * (kBN / 2);
    const int qrow = I * kBM + row;
    const int qp = qpos ? qpos[(size_t)bh * dm.n + qrow] : qrow;
    const int segI = I / dm.spb;
    if (count > 0) {
      // this thread's half of its Q row into TMEM as bf16 pairs: the A
      // operand of S = Q K'^T
      const uint4 *src =
          reinterpret_cast<const uint4 *>(q + ((size_t)bg * dm.n + qrow) * D + half * (D / 2));
      if constexpr (D == 128) {
        uint32_t r[32];
#pragma unroll
        for (int v = 0; v < 8; ++v) {
          const uint4 x = __ldg(src + v);
          r[4 * v] = x.x, r[4 * v + 1] = x.y, r[4 * v + 2] = x.z, r[4 * v + 3] = x.w;
        }
        __syncwarp();
        tmem_st32(tQ + lane_off + half * 32, r);
      } else {
        uint32_t r[16];
#pragma unroll
        for (int v = 0; v < 4; ++v) {
          const uint4 x = __ldg(src + v);
          r[4 * v] = x.x, r[4 * v + 1] = x.y, r[4 * v + 2] = x.z, r[4 * v + 3] = x.w;
        }
        __syncwarp();
        tmem_st16(tQ + lane_off + half * 16, r);
      }
      tmem_wait_st();
      tc_fence_before();
      warp_arrive(&bar->q_full, lane);
    }
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
      float s[kBN / 2];
      {
        uint32_t r0[32], r1[32];
        tmem_ld32(tS + col0, r0);
        tmem_ld32(tS + col0 + 32, r1);
        tmem_wait_ld();
#pragma unroll
        for (int e = 0; e < 32; ++e) {
          s[e] = __uint_as_float(r0[e]);
          s[32 + e] = __uint_as_float(r1[e]);
        }
      }
      if (diag) {
        if (kpos) {
          // the block's carried original positions, read as 16-byte loads
          // that every thread of the warp shares
          const int4 *kp4 = reinterpret_cast<const int4 *>(&xc->kp[j % 3][col0]);
#pragma unroll
          for (int c4 = 0; c4 < kBN / 8; ++c4) {
            const int4 p = kp4[c4];
            if (p.x > qp) s[4 * c4] = -INFINITY;
            if (p.y > qp) s[4 * c4 + 1] = -INFINITY;
            if (p.z > qp) s[4 * c4 + 2] = -INFINITY;
            if (p.w > qp) s[4 * c4 + 3] = -INFINITY;
          }
        } else {
#pragma unroll
          for (int c = 0; c < kBN / 2; ++c)
            if (J * kBN + col0 + c > qp) s[c] = -INFINITY;
        }
      }
      float m8[8];
#pragma unroll
      for (int t = 0; t < 8; ++t) m8[t] = s[t];
#pragma unroll
      for (int c = 8; c < kBN / 2; c += 8)
#pragma unroll
        for (int t = 0; t < 8; ++t) m8[t] = fmaxf(m8[t], s[c + t]);
      const float mpart = fmaxf(fmaxf(fmaxf(m8[0], m8[1]), fmaxf(m8[2], m8[3])),
                                fmaxf(fmaxf(m8[4], m8[5]), fmaxf(m8[6], m8[7])));
      // exchange the partial max with the other thread of this row
      float *xm = xc->mx[j & 1][0];
      xm[half * kBM + row] = mpart;
      if (sw == 0) cp_async_wait<0>();  // positions staged for block j + 1 have landed
      warp_arrive(&bar->xchg[j & 1], lane);
      if (!mbar_wait_warp(&bar->xchg[j & 1], (j >> 1) & 1, s_abort, err, 45)) {
        ok = false;
        break;
      }
      // every thread has finished masking block j - 1: its buffer can take
      // the positions of block j + 2
      if (sw == 0) stage_positions(j + 2);
      const float mx = fmaxf(mpart, xm[(half ^ 1) * kBM + row]);
      const float mxs = mx * sl2;
      float alpha = 1.f;
      if (mxs > m_used + kRescaleLog2) {
        alpha = exp2f(m_used - mxs);
        m_used = mxs;
      }
      const float mu = m_used == -INFINITY ? 0.f : m_used;
      __syncwarp();  // reconverge after the per-row mask before the aligned stores
      // p = 2^(s * sigma * log2(e) - m): packed fp32x2 FMA, the hardware
      // exp2 and an FMA-pipe exp2 for 5 of 16 pairs, packed partial sums;
      // P goes to TMEM as bf16 pairs over the first 64 columns of this S
      // buffer (this thread's 32 of them).
      const float2 scale2 = make_float2(sl2, sl2), neg_m2 = make_float2(-mu, -mu);
      float2 acc[4] = {make_float2(0.f, 0.f), make_float2(0.f, 0.f), make_float2(0.f, 0.f),
                       make_float2(0.f, 0.f)};
#pragma unroll
      for (int c = 0; c < 2; ++c) {
        uint32_t pk[16];
#pragma unroll
        for (int e = 0; e < 16; ++e) {
          const float2 x =
              __ffma2_rn(make_float2(s[c * 32 + 2 * e], s[c * 32 + 2 * e + 1]), scale2, neg_m2);
          const float2 p = (e % 3 == 2) ? exp2_poly2(x)
                                        : make_float2(ex2_approx(x.x), ex2_approx(x.y));
          acc[e & 3] = __fadd2_rn(acc[e & 3], p);
          pk[e] = pack_bf16(p.x, p.y);
        }
        tmem_st16(tS + half * 32 + c * 16, pk);
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
          for (int c = 0; c < OC / 32; ++c) {
            const uint32_t ta = tO + lane_off + half * OC + c * 32;
            tmem_ld32(ta, r);
            tmem_wait_ld();
#pragma unroll
            for (int e = 0; e < 32; ++e) r[e] = __float_as_uint(__uint_as_float(r[e]) * alpha);
            tmem_st32(ta, r);
          }
          tmem_wait_st();
        }
      }
      tc_fence_before();
      warp_arrive(&bar->p_full[j & 1], lane);
    }
    if (sw == 0) cp_async_wait<0>();  // no staging copy outlives the CTA
    if (ok && !mbar_wait_warp(&bar->o_ready, (count - 1) & 1, s_abort, err, 44)) ok = false;
    if (ok) {
      xc->l[half][row] = l;
      warp_arrive(&bar->lsum, lane);
      if (!mbar_wait_warp(&bar->lsum, 0, s_abort, err, 46)) ok = false;
    }
    // the row goes to its place in the given order, or with `scatter` to its
    // query's original position (the inverse permutation, fused)
    int orow_i = qrow;
    if (scatter) {
      orow_i = qp;
      if (qp < 0 || qp >= dm.n) {
        report(err, PBS_ERR_DEVICE_ASSERT);
        ok = false, orow_i = -1;
      }
    }
    bf16 *orow = out + ((size_t)bg * dm.n + (orow_i < 0 ? 0 : orow_i)) * D + half * OC;
    if (ok) {
      const float lt = l + xc->l[half ^ 1][row];
      tc_fence_after();
      const float inv = lt > 0.f ? 1.f / lt : 0.f;
      uint32_t r[32];
#pragma unroll
      for (int c = 0; c < OC / 32; ++c) {
        tmem_ld32(tO + lane_off + half * OC + c * 32, r);
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
      if (lse && half == 0)
        lse[(size_t)bg * dm.n + orow_i] = lt > 0.f ? (m_used + log2f(lt)) * kLn2 : -INFINITY;
    } else if (count == 0 && orow_i >= 0) {
      for (int c = 0; c < OC / 8; ++c)
        reinterpret_cast<uint4 *>(orow)[c] = make_uint4(0, 0, 0, 0);
      if (lse && half == 0) lse[(size_t)bg * dm.n + orow_i] = -INFINITY;
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

template <int D>
cudaError_t run(const Dims &dm, const void *q, const void *kp, const void *vp,
                const int32_t *kpos, const int32_t *qpos, const int32_t *idx, const int32_t *cnt,
                void *out, float *lse, float sigma, int *err, int fault, bool scatter,
                cudaStream_t st) {
  CUtensorMap mk, mv;
  if (!make_tile_map(&mk, kp, (uint64_t)dm.b * dm.hkv * dm.n, D, 128) ||
      !make_tile_map(&mv, vp, (uint64_t)dm.b * dm.hkv * dm.n, D, 128))
    return cudaErrorInvalidValue;
  const size_t smem = Cfg<D>::smem;
  cudaError_t e = cudaFuncSetAttribute(attn_tc_kernel<D>,
                                       cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return e;
  const unsigned grid = (unsigned)dm.b * dm.hq * dm.nb;
  attn_tc_kernel<D><<<grid, kThreads, smem, st>>>((const bf16 *)q, mk, mv, kpos, qpos, idx, cnt,
                                                  (bf16 *)out, lse, dm, sigma * kLog2e, err,
                                                  fault, scatter ? 1 : 0);
  return cudaGetLastError();
}

}  // namespace

bool attn_tc_supported(const Dims &dm) { return dm.B == 128 && (dm.d == 128 || dm.d == 64); }

cudaError_t launch_attn_tc(const Dims &dm, const void *q, const void *kp, const void *vp,
                           const int32_t *kpos, const int32_t *qpos, const int32_t *idx,
                           const int32_t *cnt, void *out, float *lse, float sigma, int *err,
                           int fault, bool scatter, cudaStream_t st) {
  if (dm.d == 64)
    return run<64>(dm, q, kp, vp, kpos, qpos, idx, cnt, out, lse, sigma, err, fault, scatter, st);
  return run<128>(dm, q, kp, vp, kpos, qpos, idx, cnt, out, lse, sigma, err, fault, scatter, st);
}

}  // namespace pbs

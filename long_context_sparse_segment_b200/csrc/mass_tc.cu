// Diagnostics: the exact attention mass of every (query block, key block)
// pair, on the sm_100a tensor cores.
//
// "Sparser Block-Sparse Attention via Token Permutation", sciencestack.ai
// Figure 2 caption (the attention coverage of a selection is the total
// attention score its blocks hold) and Figure 4 (block-level density with
// and without permutation).
//
// For query row i (natural order) the keys are the permuted slots p with
// original position kpos[p] <= i, over all n keys (dense causal softmax).
// mass[b, g, I, J] = (1/B) * sum over rows i of block I and slots p of key
// block J of P_ip; entries J past the admissible blocks are written as 0.
//
// One CTA per (batch, KV head, query block I), heaviest I first; its rows
// are block I of the G query heads that share the KV head (R = G*128 rows,
// one 128-column TMEM slice per head, thread = row, as in the first pass of
// the tcgen05 scoring kernel). The CTA walks the admissible key tiles twice:
// pass 1 keeps each row's running max and sum of exp2 (complete inside the
// CTA: it sees every key of its rows), pass 2 sums p = 2^(s - M - log2 L)
// over the tile's 128 keys per row and adds the 128 rows of each head in a
// fixed order (warp shuffles, then the four warps). Deterministic, no
// atomics. B = 128 only (a key tile is one block).
#include <math.h>

#include "common.cuh"
#include "internal.h"
#include "tc.cuh"

namespace pbs {
namespace {

using bf16 = __nv_bfloat16;
using namespace tc;

constexpr int kKT = 128;   // keys per tile = one block
constexpr int kMaxW = 4;   // G <= 4
constexpr int kMaxKS = 4;
constexpr int kMaxThreads = kMaxW * 128 + 64;

template <int D>
struct MCfg {
  static constexpr int H = D / 64;
  static constexpr uint32_t TILE = 128u * D * 2;
  static constexpr uint32_t HALF = 128u * 128;
  static constexpr int KS = D == 128 ? 2 : 4;
  static size_t smem(int W) {
    return 1024 + (size_t)W * TILE + (size_t)KS * TILE + (size_t)KS * kKT * 4 +
           sizeof(uint64_t) * 32 + 2 * kMaxW * 4 * 4 + 16;
  }
};

struct MBars {
  uint64_t q_full, k_full[kMaxKS], k_empty[kMaxKS], s_full[kMaxW], s_free[kMaxW], mma_done;
};
static_assert(sizeof(MBars) <= sizeof(uint64_t) * 32, "barrier block");

__device__ __forceinline__ void head_bar(int id, int nthreads) {
  asm volatile("bar.sync %0, %1;" ::"r"(id), "r"(nthreads) : "memory");
}

template <int D>
__global__ void __launch_bounds__(kMaxThreads, 1)
    mass_tc_kernel(const __grid_constant__ CUtensorMap tmQ,
                   const __grid_constant__ CUtensorMap tmK, const int32_t *__restrict__ kpos,
                   float *__restrict__ mass, Dims dm, float sl2, int *err) {
  using C = MCfg<D>;
  extern __shared__ uint8_t smem_raw[];
  const int W = dm.G;
  uint8_t *base = reinterpret_cast<uint8_t *>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~(uintptr_t)1023);
  uint8_t *sQ = base;
  uint8_t *sK = sQ + (size_t)W * C::TILE;
  int32_t *sKP = reinterpret_cast<int32_t *>(sK + (size_t)C::KS * C::TILE);  // [KS][kKT]
  MBars *bar = reinterpret_cast<MBars *>(sKP + C::KS * kKT);
  float *red = reinterpret_cast<float *>(reinterpret_cast<uint8_t *>(bar) +
                                         sizeof(uint64_t) * 32);  // [2][kMaxW][4]
  uint32_t *s_tmem = reinterpret_cast<uint32_t *>(red + 2 * kMaxW * 4);
  volatile int *s_abort = reinterpret_cast<volatile int *>(s_tmem + 1);

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int pw = 4 * W;  // producer warp; the MMA warp is pw + 1
  const int I = dm.nb - 1 - (int)blockIdx.x;  // heaviest query blocks first
  const int bh = blockIdx.y, b = bh / dm.hkv, h = bh % dm.hkv;
  const int seg0 = (I / dm.spb) * dm.spb;   // first block of I's segment
  const int adm = min(dm.nb, seg0 + dm.spb);  // admissible key blocks 0 .. adm-1
  const int nt = 2 * adm;                     // two passes over them
  const uint32_t tcols = W == 1 ? 128 : W == 2 ? 256 : 512;

  if (tid == 0) {
    mbar_init(&bar->q_full, 1);
    // a K slot (with the tile's carried positions) is free once the MMA has
    // read it and every row warp has masked with its positions
    for (int s = 0; s < C::KS; ++s) {
      mbar_init(&bar->k_full[s], 1);
      mbar_init(&bar->k_empty[s], 1 + 4 * W);
    }
    for (int w = 0; w < W; ++w) {
      mbar_init(&bar->s_full[w], 1);
      mbar_init(&bar->s_free[w], 4);
    }
    mbar_init(&bar->mma_done, 1);
    *s_abort = 0;
    fence_barrier_init();
  }
  if (warp == pw + 1) {
    tmem_alloc(s_tmem, tcols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tbase = *s_tmem;

  if (warp == pw) {
    // ------------------------------------------------------- TMA loads
    const bool leader = elect_one();
    int issued = 0;
    if (leader) {
      prefetch_map(&tmQ);
      prefetch_map(&tmK);
      mbar_expect_tx(&bar->q_full, (uint32_t)W * C::TILE);
      for (int w = 0; w < W; ++w)
        for (int hh = 0; hh < C::H; ++hh)
          tma_load_2d(sQ + (size_t)w * C::TILE + hh * C::HALF, &tmQ, &bar->q_full, hh * 64,
                      (b * dm.hq + h * dm.G + w) * dm.n + I * kKT);
    }
    __syncwarp();
    for (int it = 0; it < nt; ++it) {
      const int s = it % C::KS, u = it / C::KS, t = it % adm;
      if (u > 0 && !mbar_wait_warp(&bar->k_empty[s], (u - 1) & 1, s_abort, err, 51)) break;
      const bool with_pos = kpos && t >= seg0;
      if (leader) {
        mbar_expect_tx(&bar->k_full[s], C::TILE + (with_pos ? kKT * 4 : 0));
        for (int hh = 0; hh < C::H; ++hh)
          tma_load_2d(sK + (size_t)s * C::TILE + hh * C::HALF, &tmK, &bar->k_full[s], hh * 64,
                      bh * dm.n + t * kKT);
        if (with_pos)
          bulk_load(sKP + s * kKT, kpos + (size_t)bh * dm.n + (size_t)t * kKT, kKT * 4,
                    &bar->k_full[s]);
      }
      __syncwarp();
      issued = it + 1;
    }
    // drain: every copy started here lands before the CTA exits
    int never = 0;
    mbar_wait(&bar->q_full, 0, &never, nullptr);
    for (int t = issued > C::KS ? issued - C::KS : 0; t < issued; ++t)
      mbar_wait(&bar->k_full[t % C::KS], (t / C::KS) & 1, &never, nullptr);
  } else if (warp == pw + 1) {
    // -------------------------------------------------------- MMA issue
    const bool leader = elect_one();
    constexpr uint32_t kId = idesc_bf16(128, kKT, false);
    const uint32_t hi = sw128_desc_hi(1024);
    const uint32_t lo_q = sw128_desc_lo(smem_u32(sQ), 16);
    const uint32_t lo_k = sw128_desc_lo(smem_u32(sK), 16);
    if (mbar_wait_warp(&bar->q_full, 0, s_abort, err, 52)) {
      tc_fence_after();
      int ks = 0, kph = 0;
      bool ok = true;
      for (int it = 0; it < nt && ok; ++it) {
        if (!mbar_wait_warp(&bar->k_full[ks], kph, s_abort, err, 53)) break;
        tc_fence_after();
        for (int w = 0; w < W; ++w) {
          if (it > 0 && !mbar_wait_warp(&bar->s_free[w], (it - 1) & 1, s_abort, err, 54)) {
            ok = false;
            break;
          }
          tc_fence_after();
          const uint32_t lq = lo_q + w * (C::TILE >> 4), lk = lo_k + ks * (C::TILE >> 4);
          if (leader) {
#pragma unroll
            for (int kk = 0; kk < D / 16; ++kk) {
              const uint32_t step = ((kk >> 2) * C::HALF + (kk & 3) * 32) >> 4;
              mma_ss(tbase + w * 128, desc_words(lq + step, hi), desc_words(lk + step, hi), kId,
                     kk > 0);  // rows x keys
            }
            mma_commit(&bar->s_full[w]);
          }
          __syncwarp();
        }
        if (!ok) break;
        if (leader) mma_commit(&bar->k_empty[ks]);
        __syncwarp();
        if (++ks == C::KS) ks = 0, kph ^= 1;
      }
    }
    if (leader) mma_commit(&bar->mma_done);
    __syncwarp();
    int never = 0;
    mbar_wait(&bar->mma_done, 0, &never, nullptr);
  } else if (warp < pw) {
    // ----------------------------------------------------------- rows
    const int w = warp >> 2, quarter = warp & 3;
    const int lrow = quarter * 32 + lane;
    const int pos = I * kKT + lrow;  // this row's sequence position
    const uint32_t tS = tbase + w * 128 + ((uint32_t)(quarter * 32) << 16);
    const float2 sl2x2 = make_float2(sl2, sl2);
    float *out = mass + ((size_t)(b * dm.hq + h * dm.G + w) * dm.nb + I) * dm.nb;
    float m = -INFINITY, l = 0.f, off = 0.f;
    bool ok = true;
    for (int it = 0; it < nt; ++it) {
      const int t = it % adm, s = it % C::KS;
      const bool pass2 = it >= adm;
      if (it == adm) off = m + log2f(l);  // l > 0: every row sees its own position
      float rsum = 0.f;
      if (ok && !mbar_wait_warp(&bar->s_full[w], it & 1, s_abort, err, 55)) ok = false;
      if (!ok) warp_arrive(&bar->k_empty[s], lane);  // keep the slot's count whole
      if (ok) {
        tc_fence_after();
        uint32_t v[64];
#pragma unroll 1
        for (int hf = 0; hf < 2; ++hf) {
          tmem_ld32(tS + hf * 64, *reinterpret_cast<uint32_t(*)[32]>(&v[0]));
          tmem_ld32(tS + hf * 64 + 32, *reinterpret_cast<uint32_t(*)[32]>(&v[32]));
          tmem_wait_ld();
          if (hf == 1) {  // the slice is in registers: the next tile may overwrite it
            tc_fence_before();
            warp_arrive(&bar->s_free[w], lane);
          }
          if (t >= seg0) {  // the query's own segment: mask by original position
#pragma unroll
            for (int c = 0; c < 64; ++c) {
              const int key = t * kKT + hf * 64 + c;
              const int orig = kpos ? sKP[s * kKT + hf * 64 + c] : key;
              if (orig > pos) v[c] = 0xff800000u;  // -inf
            }
          }
          if (hf == 1) warp_arrive(&bar->k_empty[s], lane);  // done with the slot
          if (!pass2) {
            float c4[4] = {__uint_as_float(v[0]), __uint_as_float(v[1]), __uint_as_float(v[2]),
                           __uint_as_float(v[3])};
#pragma unroll
            for (int c = 4; c < 64; c += 4)
#pragma unroll
              for (int e = 0; e < 4; ++e) c4[e] = fmaxf(c4[e], __uint_as_float(v[c + e]));
            const float mn = fmaxf(m, fmaxf(fmaxf(c4[0], c4[1]), fmaxf(c4[2], c4[3])) * sl2);
            if (mn > m) {
              l *= ex2_approx(m - mn);
              m = mn;
            }
            const float mu = m == -INFINITY ? 0.f : m;
            const float2 nm = make_float2(-mu, -mu);
            float2 a[4];
#pragma unroll
            for (int x = 0; x < 4; ++x) a[x] = make_float2(0.f, 0.f);
#pragma unroll
            for (int c = 0; c < 64; c += 2) {
              const float2 tt = __ffma2_rn(
                  make_float2(__uint_as_float(v[c]), __uint_as_float(v[c + 1])), sl2x2, nm);
              a[(c >> 1) & 3] =
                  __fadd2_rn(a[(c >> 1) & 3], make_float2(ex2_approx(tt.x), ex2_approx(tt.y)));
            }
            const float2 sm = __fadd2_rn(__fadd2_rn(a[0], a[1]), __fadd2_rn(a[2], a[3]));
            l += sm.x + sm.y;
          } else {
            const float2 no = make_float2(-off, -off);
            float2 a[4];
#pragma unroll
            for (int x = 0; x < 4; ++x) a[x] = make_float2(0.f, 0.f);
#pragma unroll
            for (int c = 0; c < 64; c += 2) {
              const float2 tt = __ffma2_rn(
                  make_float2(__uint_as_float(v[c]), __uint_as_float(v[c + 1])), sl2x2, no);
              a[(c >> 1) & 3] =
                  __fadd2_rn(a[(c >> 1) & 3], make_float2(ex2_approx(tt.x), ex2_approx(tt.y)));
            }
            const float2 sm = __fadd2_rn(__fadd2_rn(a[0], a[1]), __fadd2_rn(a[2], a[3]));
            rsum += sm.x + sm.y;
          }
        }
      }
      if (pass2) {
        // the head's 128 rows, added in a fixed order; every thread of the
        // warpgroup takes this barrier once per tile, also after a failed wait
#pragma unroll
        for (int o = 16; o; o >>= 1) rsum += __shfl_xor_sync(0xffffffffu, rsum, o);
        float *rb = red + ((it & 1) * kMaxW + w) * 4;
        if (lane == 0) rb[quarter] = rsum;
        head_bar(1 + w, 128);
        if (quarter == 0 && lane == 0 && ok)
          out[t] = ((rb[0] + rb[1]) + (rb[2] + rb[3])) * (1.0f / kKT);
      }
    }
    // blocks past the admissible ones hold no mass
    for (int J = adm + lrow; J < dm.nb; J += 128) out[J] = 0.f;
  }
  tc_fence_before();
  __syncthreads();
  if (warp == pw + 1) {
    __syncwarp();
    tc_fence_after();
    tmem_dealloc(tbase, tcols);
  }
}

template <int D>
cudaError_t run_mass(const Dims &dm, const void *q, const void *kp, const int32_t *kpos,
                     float *mass, float sigma, int *err, cudaStream_t st) {
  CUtensorMap mq, mk;
  if (!make_tile_map(&mq, q, (uint64_t)dm.b * dm.hq * dm.n, D, kKT) ||
      !make_tile_map(&mk, kp, (uint64_t)dm.b * dm.hkv * dm.n, D, kKT))
    return cudaErrorInvalidValue;
  const size_t smem = MCfg<D>::smem(dm.G);
  cudaError_t e = cudaFuncSetAttribute(mass_tc_kernel<D>,
                                       cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return e;
  const dim3 grid(dm.nb, dm.b * dm.hkv);
  mass_tc_kernel<D><<<grid, dm.G * 128 + 64, smem, st>>>(mq, mk, kpos, mass, dm, sigma * kLog2e,
                                                          err);
  return cudaGetLastError();
}

// --------------------------------------------- coverage and block counts
// One warp per (batch, head, query block) row of mass: the mass the row's
// list holds (fixed-order fp64 sums), and the fewest blocks that hold at
// least `target` of it: the largest mass value v such that the blocks of
// mass >= v reach the target (bisection over the 32-bit patterns, which
// order non-negative floats), then the blocks above v plus as many blocks
// equal to v as the remainder needs.
__global__ void coverage_kernel(const float *__restrict__ mass, const int32_t *__restrict__ idx,
                                const int32_t *__restrict__ cnt, double target, int rows, int nb,
                                float *__restrict__ cov, int32_t *__restrict__ kmin) {
  const int warps = blockDim.x >> 5;
  const int r = blockIdx.x * warps + (threadIdx.x >> 5), lane = threadIdx.x & 31;
  if (r >= rows) return;
  const float *row = mass + (size_t)r * nb;
  auto wsum = [](double x) {
#pragma unroll
    for (int o = 16; o; o >>= 1) x += __shfl_xor_sync(0xffffffffu, x, o);
    return x;
  };
  auto wcount = [](int x) {
#pragma unroll
    for (int o = 16; o; o >>= 1) x += __shfl_xor_sync(0xffffffffu, x, o);
    return x;
  };
  if (idx && cov) {
    const int c = cnt[r];
    const int32_t *list = idx + (size_t)r * nb;
    double s = 0.0;
    for (int k = lane; k < c; k += 32) {
      const int J = list[k];
      if (J >= 0 && J < nb) s += row[J];
    }
    s = wsum(s);
    if (lane == 0) cov[r] = (float)s;
  }
  if (kmin) {
    auto mass_ge = [&](uint32_t u) {
      double s = 0.0;
      for (int J = lane; J < nb; J += 32)
        if (__float_as_uint(row[J]) >= u) s += row[J];
      return wsum(s);
    };
    int count;
    if (mass_ge(0u) < target) {
      count = nb;
    } else {
      uint32_t u = 0;  // largest pattern whose blocks still reach the target
      for (int bit = 31; bit >= 0; --bit) {
        const uint32_t cand = u | (1u << bit);
        if (mass_ge(cand) >= target) u = cand;
      }
      const float vu = __uint_as_float(u);
      double gt = 0.0;
      int ngt = 0;
      for (int J = lane; J < nb; J += 32)
        if (row[J] > vu) gt += row[J], ++ngt;
      gt = wsum(gt);
      count = wcount(ngt);
      // blocks equal to v in ascending J until the target is reached
      for (int base = 0; base < nb && gt < target; base += 32) {
        const int J = base + lane;
        unsigned bal = __ballot_sync(0xffffffffu, J < nb && row[J] == vu);
        while (bal && gt < target) {
          gt += (double)vu;
          ++count;
          bal &= bal - 1;
        }
      }
    }
    if (lane == 0) kmin[r] = count;
  }
}

}  // namespace

bool mass_supported(const Dims &dm) {
  return dm.B == 128 && dm.G >= 1 && dm.G <= kMaxW && (dm.d == 64 || dm.d == 128) &&
         (dm.d == 64 ? MCfg<64>::smem(dm.G) : MCfg<128>::smem(dm.G)) <= 227 * 1024;
}

cudaError_t launch_block_mass(const Dims &dm, const void *q, const void *kp, const int32_t *kpos,
                              float *mass, float sigma, int *err, cudaStream_t st) {
  if (dm.d == 64) return run_mass<64>(dm, q, kp, kpos, mass, sigma, err, st);
  return run_mass<128>(dm, q, kp, kpos, mass, sigma, err, st);
}

cudaError_t launch_coverage(const float *mass, const int32_t *idx, const int32_t *cnt,
                            double target, int rows, int nb, float *cov, int32_t *kmin,
                            cudaStream_t st) {
  const int warps = 8;
  coverage_kernel<<<(rows + warps - 1) / warps, warps * 32, 0, st>>>(mass, idx, cnt, target, rows,
                                                                     nb, cov, kmin);
  return cudaGetLastError();
}

}  // namespace pbs

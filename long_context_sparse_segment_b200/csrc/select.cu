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
// rows). Two kernels:
//   scores: a_IJ = sigma * qbar_I . kbar_J for every admissible (I, J) on the
//     fp64 tensor cores (mma.sync m8n8k4, 64 x 64 tiles of query blocks by
//     key blocks, d staged 64 columns at a time in shared memory so three tiles
//     run per SM), written to the workspace
//     as 64-bit order keys: every pooled key block is read once per tile
//     instead of once per query block;
//   selection: one warp per query block decides, without sorting, reading
//     its row of keys from the workspace (L1/L2):
//   TOPK_FRAC: k = max(1, floor(f * (I + 1))); the t = max(0, k - own)
//     earlier-segment blocks of largest score (ties: lower J) are found by
//     a radix select over the order keys (8-bit digit histograms from the
//     first byte in which the row's keys differ: the t-th largest key and
//     how many of the keys equal to it are taken);
//   THRESHOLD: softmax over the admissible blocks (weights to the
//     workspace); bisection finds the largest score s such that the
//     own-segment mass plus the mass of the earlier blocks scoring >= s
//     reaches tau; blocks scoring above s are kept and blocks tied at s are
//     added in ascending J until it does. This is the set the descending
//     walk of the definition stops at.
// then the warp compacts the kept flags into the ascending list. Masses are
// summed in a fixed order, so results are deterministic.
#include <math.h>

#include "common.cuh"
#include "internal.h"

namespace pbs {
namespace {

constexpr int kThreads = 256;  // selection: 8 warps, one query block each
constexpr int kTile = 64;      // score tiles: 64 query blocks x 64 key blocks
constexpr int kPad = 4;        // doubles of padding per staged row (bank spread)

constexpr int kWarps = kThreads / 32;

// selection shared memory: per warp, the kept flags of its row and a digit
// histogram
size_t sel_smem(int nb) { return (size_t)kWarps * ((size_t)nb + 256 * 8) + 64; }

__device__ __forceinline__ double f64_from_order_key(unsigned long long u) {
  return __longlong_as_double(
      (long long)((u & 0x8000000000000000ull) ? (u ^ 0x8000000000000000ull) : ~u));
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

// The bits every key[0 .. cnt) shares: on return *pre holds them (the other
// bits 0) and the result is the index of the highest bit at which two keys
// differ, or -1 when all are equal (then *pre is the common key).
__device__ __forceinline__ int common_prefix(const unsigned long long *key, int cnt, int lane,
                                             unsigned long long *pre) {
  unsigned long long mn = ~0ull, mx = 0ull;
  for (int J = lane; J < cnt; J += 32) {
    const unsigned long long k = key[J];
    mn = k < mn ? k : mn;
    mx = k > mx ? k : mx;
  }
#pragma unroll
  for (int o = 16; o; o >>= 1) {
    const unsigned long long a = __shfl_xor_sync(0xffffffffu, mn, o);
    const unsigned long long b = __shfl_xor_sync(0xffffffffu, mx, o);
    mn = a < mn ? a : mn;
    mx = b > mx ? b : mx;
  }
  const unsigned long long diff = mn ^ mx;
  if (diff == 0) {
    *pre = mx;
    return -1;
  }
  const int top = 63 - __clzll((long long)diff);
  *pre = top == 63 ? 0ull : mx & ~((2ull << top) - 1);
  return top;
}

// D[8x8] += A[8x4] * B[4x8] in fp64: lane t holds A[t/4][t%4], B[t%4][t/4],
// D[t/4][2(t%4)] and D[t/4][2(t%4)+1].
__device__ __forceinline__ void dmma_8x8x4(double (&d)[2], double a, double b) {
  asm volatile("mma.sync.aligned.m8n8k4.row.col.f64.f64.f64.f64 {%0,%1}, {%2}, {%3}, {%0,%1};\n"
               : "+d"(d[0]), "+d"(d[1])
               : "d"(a), "d"(b));
}

// Scores of one 64 x 64 tile of (query block I, key block J) pairs of one
// (batch, query head): a_IJ = sigma * qbar_I . kbar_J with the block means
// qbar = qsum / B, kbar = ksum / B, as 64-bit order keys into
// keys[bg][I][J] for the admissible J (segment of J <= segment of I).
// 8 warps as 2 x 4: a warp owns 32 query blocks x 16 key blocks, i.e. 4 x 2
// m8n8k4 products per 4-wide step of d.
template <int D>
__global__ void __launch_bounds__(kThreads)
    scores_kernel(const double *__restrict__ qsum, const double *__restrict__ ksum, Dims dm,
                  double sigma, unsigned long long *__restrict__ keys) {
  extern __shared__ __align__(16) unsigned char smem[];
  constexpr int KC = 64;           // columns of d staged at a time (three CTAs per SM)
  constexpr int LD = KC + kPad;
  double *As = reinterpret_cast<double *>(smem);  // [kTile][LD] query block means
  double *Bs = As + kTile * LD;                   // [kTile][LD] key block means
  const int nb = dm.nb;
  const int bg = blockIdx.z, b = bg / dm.hq, g = bg % dm.hq;
  const int kv = b * dm.hkv + g / dm.G;
  const int R0 = blockIdx.y * kTile, C0 = blockIdx.x * kTile;
  const int last = min(nb, R0 + kTile) - 1;
  if (C0 >= min(nb, (last / dm.spb + 1) * dm.spb)) return;  // nothing admissible here
  const int tid = threadIdx.x, w = tid >> 5, lane = tid & 31;
  const double inv_b = 1.0 / (double)dm.B;  // a power of two: exact
  const int wr = (w >> 2) * 32, wc = (w & 3) * 16;
  double acc[4][2][2];
#pragma unroll
  for (int mt = 0; mt < 4; ++mt)
#pragma unroll
    for (int nt = 0; nt < 2; ++nt) acc[mt][nt][0] = acc[mt][nt][1] = 0.0;
  const double *ap = As + (wr + (lane >> 2)) * LD + (lane & 3);
  const double *bp = Bs + (wc + (lane >> 2)) * LD + (lane & 3);
#pragma unroll 1
  for (int k0 = 0; k0 < D; k0 += KC) {
    if (k0) __syncthreads();  // the previous columns are consumed
    for (int e = tid; e < kTile * KC; e += kThreads) {
      const int r = e / KC, c = e % KC;
      As[r * LD + c] = R0 + r < nb ? qsum[((size_t)bg * nb + R0 + r) * D + k0 + c] * inv_b : 0.0;
      Bs[r * LD + c] = C0 + r < nb ? ksum[((size_t)kv * nb + C0 + r) * D + k0 + c] * inv_b : 0.0;
    }
    __syncthreads();
#pragma unroll 4
    for (int k = 0; k < KC; k += 4) {
      double af[4], bf[2];
#pragma unroll
      for (int mt = 0; mt < 4; ++mt) af[mt] = ap[mt * 8 * LD + k];
#pragma unroll
      for (int nt = 0; nt < 2; ++nt) bf[nt] = bp[nt * 8 * LD + k];
#pragma unroll
      for (int mt = 0; mt < 4; ++mt)
#pragma unroll
        for (int nt = 0; nt < 2; ++nt) dmma_8x8x4(acc[mt][nt], af[mt], bf[nt]);
    }
  }
#pragma unroll
  for (int mt = 0; mt < 4; ++mt) {
    const int I = R0 + wr + mt * 8 + (lane >> 2);
    if (I >= nb) continue;
    const int adm = min(nb, (I / dm.spb + 1) * dm.spb);
    unsigned long long *row = keys + ((size_t)bg * nb + I) * nb;
#pragma unroll
    for (int nt = 0; nt < 2; ++nt)
#pragma unroll
      for (int u = 0; u < 2; ++u) {
        const int J = C0 + wc + nt * 8 + 2 * (lane & 3) + u;
        if (J < adm) row[J] = f64_order_key(sigma * acc[mt][nt][u]);
      }
  }
}

// One warp per (batch, query head, query block): the kept list from the
// row's score keys (and, for THRESHOLD, softmax weights written next to
// them in `pis`).
__global__ void __launch_bounds__(kThreads)
    select_kernel(const unsigned long long *__restrict__ keys, double *__restrict__ pis_all,
                  Dims dm, int mode, float param, int32_t *__restrict__ idx_out,
                  int32_t *__restrict__ cnt_out, uint8_t *__restrict__ mask_out) {
  extern __shared__ __align__(16) unsigned char smem[];
  const int nb = dm.nb;
  const int tid = threadIdx.x, w = tid >> 5, lane = tid & 31;
  const long long rowid = (long long)blockIdx.x * kWarps + w;
  if (rowid >= (long long)dm.b * dm.hq * nb) return;  // whole warp; no block barrier follows
  // per warp: a 256-bin digit histogram (32-bit counts for TOP-K, 64-bit
  // fixed-point masses for THRESHOLD), then the row's kept flags
  unsigned long long *hist64 = reinterpret_cast<unsigned long long *>(smem) + w * 256;
  unsigned char *flag =
      reinterpret_cast<unsigned char *>(smem) + (size_t)kWarps * 256 * 8 + (size_t)w * nb;
  const int bg = (int)(rowid / nb);
  const bool scored = mode == PBS_SEL_THRESHOLD || mode == PBS_SEL_TOPK_FRAC;

  const int I = (int)(rowid % nb);
  const int seg = I / dm.spb;
  const int f0 = seg * dm.spb;  // own segment: [f0, adm); earlier blocks: [0, f0)
  const int adm = min(nb, f0 + dm.spb);
  const unsigned long long *key = keys + (size_t)rowid * nb;
  double *pi = pis_all + (size_t)rowid * nb;

  // Selected earlier blocks: key > kcut, plus `tie_take` of those with
  // key == kcut in ascending J.
  unsigned long long kcut = ~0ull;
  int tie_take = 0;
  bool all_earlier = false;
  if (scored && f0 > 0) {
    if (mode == PBS_SEL_TOPK_FRAC) {
      const int k_i = max(1, (int)floor((double)param * (double)(I + 1)));
      const int t = min(f0, max(0, k_i - (adm - f0)));
      if (t == f0) {
        all_earlier = true;
      } else if (t > 0) {
        // The t-th largest key, one 8-bit digit at a time from the top: among
        // the keys that share the digits found so far, count each value of
        // the next digit, and take the digit at which the count from the top
        // reaches the number still needed.
        // The bits all keys share are skipped: they would send every key to
        // one histogram bin.
        unsigned *hist = reinterpret_cast<unsigned *>(hist64);
        unsigned long long pre = 0;
        const int top = common_prefix(key, f0, lane, &pre);
        int need = t;
        const int first = top < 0 ? -8 : (top / 8) * 8;  // the byte holding the top bit
        unsigned long long pmask = first + 8 >= 64 ? 0ull : ~((1ull << (first + 8)) - 1);
        pre &= pmask;  // the shared bits inside the first byte come with its digit
        for (int shift = first; shift >= 0; shift -= 8) {
          for (int d = lane; d < 256; d += 32) hist[d] = 0;
          __syncwarp();
          for (int J = lane; J < f0; J += 32) {
            const unsigned long long kj = key[J];
            if ((kj & pmask) == pre) atomicAdd(&hist[(unsigned)(kj >> shift) & 255u], 1u);
          }
          __syncwarp();
          // lane l holds digits 255 - 8l .. 248 - 8l (descending)
          unsigned c[8], tot = 0;
#pragma unroll
          for (int e = 0; e < 8; ++e) tot += (c[e] = hist[255 - 8 * lane - e]);
          unsigned incl = tot;  // inclusive prefix over lanes, from digit 255 down
#pragma unroll
          for (int o = 1; o < 32; o <<= 1) {
            const unsigned u = __shfl_up_sync(0xffffffffu, incl, o);
            if (lane >= o) incl += u;
          }
          const unsigned excl = incl - tot;
          const unsigned hit = __ballot_sync(0xffffffffu, excl < (unsigned)need && incl >= (unsigned)need);
          const int src = __ffs(hit) - 1;
          int digit = 0, above = 0;
          if (lane == src) {
            unsigned run = excl;
#pragma unroll
            for (int e = 0; e < 8; ++e) {
              if (run + c[e] >= (unsigned)need) {
                digit = 255 - 8 * lane - e;
                break;
              }
              run += c[e];
            }
            above = (int)run;
          }
          digit = __shfl_sync(0xffffffffu, digit, src);
          above = __shfl_sync(0xffffffffu, above, src);
          need -= above;
          pre |= (unsigned long long)digit << shift;
          pmask |= 255ull << shift;
          __syncwarp();
        }
        kcut = pre;  // all keys equal (top < 0): the common key
        tie_take = need;  // keys equal to the cut that are still taken
      }
    } else {
      const double tau = (double)param;
      double amax = -INFINITY;
      for (int J = lane; J < adm; J += 32) amax = fmax(amax, f64_from_order_key(key[J]));
      amax = warp_max_d(amax);
      double z = 0.0, own = 0.0;
      for (int J = lane; J < adm; J += 32) {
        const double e = exp(f64_from_order_key(key[J]) - amax);
        pi[J] = e;
        z += e;
        if (J >= f0) own += e;
      }
      z = warp_sum_d(z);
      own = warp_sum_d(own) / z;
      for (int J = lane; J < f0; J += 32) pi[J] = pi[J] / z;
      __syncwarp();
      auto mass_ge = [&](unsigned long long v) {  // own + mass of earlier keys >= v
        double m = 0.0;
        for (int J = lane; J < f0; J += 32)
          if (key[J] >= v) m += pi[J];
        return own + warp_sum_d(m);
      };
      if (own < tau) {
        if (mass_ge(0ull) < tau) {
          all_earlier = true;  // the mass never reaches tau: every block
        } else {
          // The cut: the largest key whose mass from the top (with the own
          // segment's) reaches tau. Found one 8-bit digit at a time from the
          // top, as TOP-K finds its count: among the keys that share the
          // digits found so far, the masses per value of the next digit
          // (fixed point in units of 2^-62, whose integer sums do not depend
          // on their order), and the digit at which the mass from the top
          // reaches what is still needed. The fixed point resolves the mass
          // to ~1e-17; should it not reach what the fp64 sums above say is
          // there, the cut is found bit by bit on the fp64 sums instead.
          unsigned long long k = 0;
          const int top = common_prefix(key, f0, lane, &k);
          bool found = top < 0;  // all keys equal: the common key
          if (!found) {
            constexpr double kFx = 4611686018427387904.0;  // 2^62
            const unsigned long long tau_fx = __double2ull_rn(tau * kFx);
            const unsigned long long own_fx = __double2ull_rn(own * kFx);
            unsigned long long need = tau_fx > own_fx ? tau_fx - own_fx : 1ull;
            const int first = (top / 8) * 8;  // the byte holding the top bit
            unsigned long long pmask = first + 8 >= 64 ? 0ull : ~((1ull << (first + 8)) - 1);
            unsigned long long pre = k & pmask;
            found = true;
            for (int shift = first; shift >= 0 && found; shift -= 8) {
              for (int d = lane; d < 256; d += 32) hist64[d] = 0ull;
              __syncwarp();
              for (int J = lane; J < f0; J += 32) {
                const unsigned long long kj = key[J];
                if ((kj & pmask) == pre)
                  atomicAdd(&hist64[(unsigned)(kj >> shift) & 255u], __double2ull_rn(pi[J] * kFx));
              }
              __syncwarp();
              // lane l holds digits 255 - 8l .. 248 - 8l (descending)
              unsigned long long c[8], tot = 0;
#pragma unroll
              for (int e = 0; e < 8; ++e) tot += (c[e] = hist64[255 - 8 * lane - e]);
              unsigned long long incl = tot;  // inclusive prefix over lanes
#pragma unroll
              for (int o = 1; o < 32; o <<= 1) {
                const unsigned long long u = __shfl_up_sync(0xffffffffu, incl, o);
                if (lane >= o) incl += u;
              }
              const unsigned long long excl = incl - tot;
              const unsigned hit = __ballot_sync(0xffffffffu, excl < need && incl >= need);
              if (hit == 0u) {
                found = false;
                break;
              }
              const int src = __ffs(hit) - 1;
              int digit = 0;
              unsigned long long above = 0;
              if (lane == src) {
                unsigned long long run = excl;
#pragma unroll
                for (int e = 0; e < 8; ++e) {
                  if (run + c[e] >= need) {
                    digit = 255 - 8 * lane - e;
                    break;
                  }
                  run += c[e];
                }
                above = run;
              }
              digit = __shfl_sync(0xffffffffu, digit, src);
              above = __shfl_sync(0xffffffffu, above, src);
              need -= above;
              pre |= (unsigned long long)digit << shift;
              pmask |= 255ull << shift;
              __syncwarp();
            }
            if (found) k = pre;
          }
          if (!found) {
            // largest value whose mass still reaches tau; it lies between
            // the smallest and largest key, so the bits they share are fixed
            k = 0;
            for (int bit = common_prefix(key, f0, lane, &k); bit >= 0; --bit) {
              const unsigned long long cand = k | (1ull << bit);
              if (mass_ge(cand) >= tau) k = cand;
            }
          }
          kcut = k;
          // blocks above the cut fall short of tau; add the tied ones in J order
          double run = 0.0;
          for (int J = lane; J < f0; J += 32)
            if (key[J] > k) run += pi[J];
          run = own + warp_sum_d(run);
          for (int base = 0; base < f0 && run < tau; base += 32) {
            const int J = base + lane;
            unsigned bal = __ballot_sync(0xffffffffu, J < f0 && key[J] == k);
            while (bal && run < tau) {
              const int l = __ffs(bal) - 1;
              run += __shfl_sync(0xffffffffu, J < f0 ? pi[J] : 0.0, l);
              ++tie_take;
              bal &= bal - 1;
            }
          }
        }
      }
    }
  }

  // kept flags, then the ascending list
  for (int J = lane; J < nb; J += 32) flag[J] = 0;
  __syncwarp();
  if (scored) {
    for (int J = f0 + lane; J < adm; J += 32) flag[J] = 1;
    if (all_earlier) {
      for (int J = lane; J < f0; J += 32) flag[J] = 1;
    } else if (kcut != ~0ull) {
      int ties_before = 0;
      for (int base = 0; base < f0; base += 32) {
        const int J = base + lane;
        const bool in = J < f0;
        const unsigned long long kj = in ? key[J] : 0ull;
        const bool tie = in && kj == kcut;
        const unsigned bal = __ballot_sync(0xffffffffu, tie);
        const int rank = ties_before + __popc(bal & ((1u << lane) - 1u));
        if (in && (kj > kcut || (tie && rank < tie_take))) flag[J] = 1;
        ties_before += __popc(bal);
      }
    }
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

// Workspace: the pooled query sums, [the pooled key sums,] then the score
// keys and the softmax weights of every (batch, query head, query block,
// key block).
size_t select_qsum_bytes(const Dims &dm) { return (size_t)dm.b * dm.hq * dm.nb * dm.d * 8; }

size_t select_scratch_bytes(const Dims &dm) { return 2 * (size_t)dm.b * dm.hq * dm.nb * dm.nb * 8; }

size_t select_ws_bytes(const Dims &dm, bool need_kbar) {
  const size_t k = need_kbar ? (size_t)dm.b * dm.hkv * dm.nb * dm.d * 8 : 0;
  return select_qsum_bytes(dm) + k + select_scratch_bytes(dm);
}

cudaError_t launch_select(const Dims &dm, const double *qsum, const double *ksum, int mode,
                          float param, double sigma, int32_t *idx, int32_t *cnt, uint8_t *mask,
                          void *scratch, int *err, cudaStream_t st) {
  (void)err;
  const bool scored = mode == PBS_SEL_THRESHOLD || mode == PBS_SEL_TOPK_FRAC;
  unsigned long long *keys = reinterpret_cast<unsigned long long *>(scratch);
  double *pis = reinterpret_cast<double *>(keys + (size_t)dm.b * dm.hq * dm.nb * dm.nb);
  cudaError_t e;
  if (scored) {
    auto sk = dm.d == 64 ? scores_kernel<64> : scores_kernel<128>;
    const size_t ssm = (size_t)2 * kTile * (64 + kPad) * 8;
    e = cudaFuncSetAttribute(sk, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)ssm);
    if (e != cudaSuccess) return e;
    const int tiles = (dm.nb + kTile - 1) / kTile;
    sk<<<dim3(tiles, tiles, dm.b * dm.hq), kThreads, ssm, st>>>(qsum, ksum, dm, sigma, keys);
    if ((e = cudaGetLastError()) != cudaSuccess) return e;
  }
  const size_t smem = sel_smem(dm.nb);
  if (smem > 227 * 1024) return cudaErrorInvalidValue;
  e = cudaFuncSetAttribute(select_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return e;
  const long long rows = (long long)dm.b * dm.hq * dm.nb;
  select_kernel<<<(unsigned)((rows + kWarps - 1) / kWarps), kThreads, smem, st>>>(
      keys, pis, dm, mode, param, idx, cnt, mask);
  return cudaGetLastError();
}

}  // namespace pbs

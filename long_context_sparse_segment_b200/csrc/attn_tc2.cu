// Block-sparse causal attention over the permuted keys on the sm_100a
// tensor cores, two query tiles per CTA.
//
// "Sparser Block-Sparse Attention via Token Permutation", sciencestack.ai
// Figure 1 caption (inter-segment causality is kept; the blocks of the
// on-diagonal segment are computed with a per-element mask, inter-segment
// blocks are fully visible or skipped) and gist.science summary, "Methodik"
// 4 (a permuted FlashAttention kernel walks the kept blocks).
//
// A CTA takes two work items (batch, query head, 128-row query block),
// tiles A and B, each with its own list of kept key blocks and its own
// stream of K'/V' tiles. The tensor core alternates between them:
//   S_A(0), S_B(0), then per block j:  O_A += P_A(j) V'_A(j), S_A(j+1),
//                                      O_B += P_B(j) V'_B(j), S_B(j+1),
// so that the products of one tile run while the softmax of the other
// works. TMEM (512 columns): S_A, S_B (P is written over the first 64
// columns of its S as bf16 pairs), O_A, O_B. Q_A and Q_B stay in shared
// memory. 384 threads, three warpgroups:
//   warp 0               TMA: Q_A, Q_B, then K' and V' tiles in exactly the
//                        order the tensor core consumes them, into a K'
//                        ring and a V' ring; a V' tile of an on-diagonal-
//                        segment block brings the block's carried key
//                        positions (512 bytes);
//   warp 1               tcgen05.mma issue in the order above;
//   (both warps run their loops warp-wide and issue from one elected lane)
//   warps 2, 3           idle, or with GATHER (pbs_attn_fwd_gather), and
//                        warp 0 once Q is issued, the K and V tiles: each
//                        row read from the natural K, V at its carried
//                        position with cp.async, into the layout the TMA
//                        would write.
//   warps 4-7, 8-11      softmax of tile A, of tile B: one thread per query
//                        row (TMEM lane), all 128 key columns of a block:
//                        mask, row max, exp2 (MUFU), P to TMEM in two
//                        halves, row sum; final normalisation and store.
// A softmax thread holds a whole row of S, so the first warpgroup (warps
// 0-3) gives registers to the other two (setmaxnreg): 128 x 56 + 256 x 224
// = 64,512, exactly the 384 x 168 the CTA is launched with.
// S_X(j+1) is only signalled once every earlier product has completed, so
// O_X holds P_X(j) V'_X(j) by then and the softmax rescales it in place
// when needed without waiting. The running max is only moved when it grows
// by more than 2^8, so O is rescaled rarely. Every mbarrier wait is
// bounded; on expiry the CTA records PBS_ERR_TIMEOUT, drains what it issued,
// frees TMEM and exits.
#include <math.h>

#include "common.cuh"
#include "internal.h"
#include "tc.cuh"

namespace pbs {
namespace {

using bf16 = __nv_bfloat16;
using namespace tc;

constexpr int kBM = 128;  // query rows per tile (MMA M)
constexpr int kBN = 128;  // keys per block
constexpr int kThreads = 384;
constexpr int kLaunchRegs = 168;   // per thread at launch (checked on the host)
constexpr int kCtrlRegs = 56;      // warps 0-3 after setmaxnreg.dec
constexpr int kSoftmaxRegs = 224;  // warps 4-11 after setmaxnreg.inc
static_assert(128 * kCtrlRegs + 256 * kSoftmaxRegs <= kThreads * kLaunchRegs,
              "register split exceeds the launch allocation");
constexpr float kRescaleLog2 = 8.0f;  // move the running max only past 2^8

template <int D>
struct Cfg2 {
  static constexpr int H = D / 64;                          // 128-byte atoms per row
  static constexpr uint32_t TILE = (uint32_t)kBM * D * 2;  // bytes per 128-row tile
  static constexpr uint32_t HALF = (uint32_t)kBM * 128;    // bytes per 64-column box
  static constexpr int KS = D == 128 ? 2 : 4;              // K' ring depth
  static constexpr int VS = D == 128 ? 3 : 4;              // V' ring depth
};

template <int D>
struct Bars2 {
  uint64_t q_full, k_full[Cfg2<D>::KS], k_empty[Cfg2<D>::KS], v_full[Cfg2<D>::VS],
      v_empty[Cfg2<D>::VS], s_full[2], p_full[2][2], o_final[2], mma_done;
};

template <int D>
constexpr size_t smem2() {
  return 1024 + 2 * (size_t)Cfg2<D>::TILE + (size_t)(Cfg2<D>::KS + Cfg2<D>::VS) * Cfg2<D>::TILE +
         (size_t)Cfg2<D>::VS * kBN * 4 + sizeof(Bars2<D>) + 16;
}
static_assert(smem2<128>() <= 232448, "shared memory (d = 128)");
static_assert(smem2<64>() <= 232448, "shared memory (d = 64)");

// One work item: a 128-row query tile and its list of kept key blocks.
struct Tile {
  int bg, I, bh, count, segI;
  const int32_t *list;
};

__device__ __forceinline__ Tile make_tile(int item, int total, const Dims &dm,
                                          const int32_t *blk_idx, const int32_t *blk_cnt,
                                          int *err) {
  Tile t;
  if (item >= total) {
    t.bg = 0, t.I = 0, t.bh = 0, t.count = 0, t.segI = 0, t.list = blk_idx;
    return t;
  }
  // KV groups one after the other, so that the K'/V' tiles in use at a time
  // are one KV head's (L2-resident reuse across the group's query heads
  // and neighbouring query blocks); inside a group heavy query blocks first,
  // the G query heads of a block adjacent (a CTA's two tiles share a block
  // index whenever G is even)
  const int per_group = dm.G * dm.nb;
  const int r = item % per_group;
  t.bh = item / per_group;
  t.I = dm.nb - 1 - r / dm.G;
  t.bg = (t.bh / dm.hkv) * dm.hq + (t.bh % dm.hkv) * dm.G + r % dm.G;
  t.segI = t.I / dm.spb;
  t.list = blk_idx + ((size_t)t.bg * dm.nb + t.I) * dm.nb;
  t.count = blk_cnt[(size_t)t.bg * dm.nb + t.I];
  if (t.count < 0 || t.count > dm.nb) {
    report(err, PBS_ERR_DEVICE_ASSERT);
    t.count = 0;
  }
  return t;
}

__device__ __forceinline__ int checked_block(const Tile &t, int j, const Dims &dm, int *err) {
  int J = t.list[j];
  if (J < 0 || J >= dm.nb) {
    report(err, PBS_ERR_DEVICE_ASSERT);
    J = 0;
  }
  return J;
}

// How many of the 16 exponent pairs of a 32-column chunk go to the FMA-pipe
// cubic instead of the MUFU unit. Measured on B200 (llama32k, llama128k):
// 0 is fastest; 4-8 of 16 cost 8-10%. The MUFU unit is not this kernel's
// limit, and under the power cap the extra FMA-pipe instructions lower the
// clock more than they save.
constexpr int kPolyPairs = 0;
__device__ __forceinline__ constexpr bool poly_pair(int e) {
  return (e * kPolyPairs) % 16 >= 16 - kPolyPairs;  // spread evenly over the chunk
}

// Position of block j of tile x (0 = A, 1 = B) in the interleaved stream
// A0 B0 A1 B1 ... (a list that has ended drops out).
__device__ __forceinline__ int stream_pos(int x, int j, int cA, int cB) {
  return x == 0 ? j + min(j, cB) : j + min(j + 1, cA);
}

// Rows of a K'/V' tile that gathering warp g (of kGatherWarps) fills:
// [gather_lo(g), gather_lo(g + 1)), at most 64, in multiples of 4.
constexpr int kGatherWarps = 3;
__device__ __forceinline__ constexpr int gather_lo(int g) { return g == 3 ? kBN : 44 * g; }

// Carried positions of keys lo + lane and lo + 32 + lane of block J of KV
// head bh (rows past `rows` are not read). A position outside block J's
// segment is reported and replaced by the key's own index.
__device__ __forceinline__ int2 carried_rows(const int32_t *__restrict__ kpos, int bh, int J,
                                             int lo, int rows, int lane, const Dims &dm,
                                             int *err) {
  const int p0 = J * kBN + lo + lane;
  const int32_t *p = kpos + (size_t)bh * dm.n + p0;
  const int unused = J * kBN;  // any key of block J: inside its segment, never read
  int2 r = make_int2(lane < rows ? __ldg(p) : unused, lane + 32 < rows ? __ldg(p + 32) : unused);
  const int seg0 = (J / dm.spb) * dm.S;
  const unsigned span = (unsigned)min(dm.S, dm.n - seg0);  // the last segment may be short
  if ((unsigned)(r.x - seg0) >= span || (unsigned)(r.y - seg0) >= span) {
    report(err, PBS_ERR_DEVICE_ASSERT);
    r = make_int2(lane < rows ? p0 : unused, lane + 32 < rows ? p0 + 32 : unused);
  }
  return r;
}

// GATHER: the permutation is applied on the fly. kg and vg are the natural
// K and V; warps 0 (after Q), 2 and 3 fetch each block's rows by their
// carried positions with cp.async into the same swizzled tiles the TMA
// would write (no K', V' copies); tmK and tmV are unused.
template <int D, bool GATHER>
__global__ void __launch_bounds__(kThreads, 1)
    attn_tc2_kernel(const __grid_constant__ CUtensorMap tmQ,
                    const __grid_constant__ CUtensorMap tmK,
                    const __grid_constant__ CUtensorMap tmV, const int32_t *__restrict__ kpos,
                    const int32_t *__restrict__ qpos, const int32_t *__restrict__ blk_idx,
                    const int32_t *__restrict__ blk_cnt, const __grid_constant__ OutSet outs,
                    float *__restrict__ lse, Dims dm, float sl2, int *err, int fault,
                    int scatter, const bf16 *__restrict__ kg, const bf16 *__restrict__ vg) {
  using C = Cfg2<D>;
  constexpr int KS = C::KS, VS = C::VS;
  extern __shared__ uint8_t smem_raw[];
  uint8_t *base = reinterpret_cast<uint8_t *>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~(uintptr_t)1023);
  uint8_t *sQ = base;                          // [2] tiles
  uint8_t *sK = sQ + 2 * C::TILE;              // [KS] tiles
  uint8_t *sV = sK + KS * C::TILE;             // [VS] tiles
  int32_t *sKP = reinterpret_cast<int32_t *>(sV + VS * C::TILE);  // [VS][kBN]
  Bars2<D> *bar = reinterpret_cast<Bars2<D> *>(sKP + VS * kBN);
  uint32_t *s_tmem = reinterpret_cast<uint32_t *>(bar + 1);
  volatile int *s_abort = reinterpret_cast<volatile int *>(s_tmem + 1);

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int total = dm.b * dm.hq * dm.nb;
  const Tile tA = make_tile(2 * blockIdx.x, total, dm, blk_idx, blk_cnt, tid == 0 ? err : nullptr);
  const Tile tB = make_tile(2 * blockIdx.x + 1, total, dm, blk_idx, blk_cnt, tid == 0 ? err : nullptr);
  const int cA = tA.count, cB = tB.count;
  const int cmax = cA > cB ? cA : cB;

  if (tid == 0) {
    mbar_init(&bar->q_full, 1);
    // full: the TMA's expect-tx arrival, or one cp.async arrival per
    // gathering thread
    const int fill_count = GATHER ? 32 * kGatherWarps : 1;
    for (int s = 0; s < KS; ++s) {
      mbar_init(&bar->k_full[s], fill_count);
      mbar_init(&bar->k_empty[s], 1);
    }
    for (int s = 0; s < VS; ++s) {
      mbar_init(&bar->v_full[s], fill_count);
      mbar_init(&bar->v_empty[s], 1);
    }
    for (int x = 0; x < 2; ++x) {
      mbar_init(&bar->s_full[x], 1);
      mbar_init(&bar->p_full[x][0], 4);  // the four warps of the tile's softmax,
      mbar_init(&bar->p_full[x][1], 4);  // for keys 0-63 and 64-127 of P
      mbar_init(&bar->o_final[x], 1);
    }
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
  if (warp < 4) {
  // =============================================== warpgroup 0: TMA and MMA
  asm volatile("setmaxnreg.dec.sync.aligned.u32 %0;" ::"n"(kCtrlRegs));
  if (warp == 0) {
    // ------------------------------------------------------- TMA loads
    // Order: K'_A(0), K'_B(0), then per block j and tile x: V'_x(j),
    // K'_x(j+1) -- the tensor core's order, so that a load only ever waits
    // for a slot that an earlier product frees. The whole warp runs the loop;
    // one elected lane issues the copies.
    const bool leader = elect_one();
    bool q_issued = false;
    int kseq = 0, vseq = 0;
    if (cmax > 0) {
      prefetch_map(&tmQ);
      if (!GATHER) {
        prefetch_map(&tmK);
        prefetch_map(&tmV);
      }
      if (leader) {
        mbar_expect_tx(&bar->q_full, ((cA > 0) + (cB > 0)) * C::TILE);
        for (int x = 0; x < 2; ++x) {
          const Tile &t = x ? tB : tA;
          if (t.count == 0) continue;
          for (int h = 0; h < C::H; ++h)
            tma_load_2d(sQ + x * C::TILE + h * C::HALF, &tmQ, &bar->q_full, h * 64,
                        t.bg * dm.n + t.I * kBM);
        }
      }
      __syncwarp();
      q_issued = true;
      auto load_k = [&](const Tile &t, int j) -> bool {
        const int s = kseq % KS, u = kseq / KS;
        if (u > 0 && !mbar_wait_warp(&bar->k_empty[s], (u - 1) & 1, s_abort, err, 11))
          return false;
        const int J = checked_block(t, j, dm, leader ? err : nullptr);
        if (leader) {
          mbar_expect_tx(&bar->k_full[s], C::TILE);
          if (!(fault == 1 && kseq == 0))
            for (int h = 0; h < C::H; ++h)
              tma_load_2d(sK + s * C::TILE + h * C::HALF, &tmK, &bar->k_full[s], h * 64,
                          t.bh * dm.n + J * kBN);
        }
        __syncwarp();
        ++kseq;
        return true;
      };
      auto load_v = [&](const Tile &t, int j) -> bool {
        const int s = vseq % VS, u = vseq / VS;
        if (u > 0 && !mbar_wait_warp(&bar->v_empty[s], (u - 1) & 1, s_abort, err, 21))
          return false;
        const int J = checked_block(t, j, dm, leader ? err : nullptr);
        const bool with_pos = kpos && J / dm.spb == t.segI;
        if (leader) {
          mbar_expect_tx(&bar->v_full[s], C::TILE + (with_pos ? kBN * 4 : 0));
          for (int h = 0; h < C::H; ++h)
            tma_load_2d(sV + s * C::TILE + h * C::HALF, &tmV, &bar->v_full[s], h * 64,
                        t.bh * dm.n + J * kBN);
          if (with_pos)
            bulk_load(sKP + s * kBN, kpos + (size_t)t.bh * dm.n + (size_t)J * kBN, kBN * 4,
                      &bar->v_full[s]);
        }
        __syncwarp();
        ++vseq;
        return true;
      };
      bool ok = !GATHER;  // with GATHER, warps 2 and 3 load K and V
      if (ok && cA > 0) ok = load_k(tA, 0);
      if (ok && cB > 0) ok = load_k(tB, 0);
      for (int j = 0; j < cmax && ok; ++j)
        for (int x = 0; x < 2 && ok; ++x) {
          const Tile &t = x ? tB : tA;
          if (j >= t.count) continue;
          ok = load_v(t, j);
          if (ok && j + 1 < t.count) ok = load_k(t, j + 1);
        }
    }
    // drain: every copy this thread started lands before the CTA exits
    int never = 0;
    if (q_issued) mbar_wait(&bar->q_full, 0, &never, nullptr);
    for (int t = kseq > KS ? kseq - KS : 0; t < kseq; ++t)
      if (!(fault == 1 && t == 0)) mbar_wait(&bar->k_full[t % KS], (t / KS) & 1, &never, nullptr);
    for (int t = vseq > VS ? vseq - VS : 0; t < vseq; ++t)
      mbar_wait(&bar->v_full[t % VS], (t / VS) & 1, &never, nullptr);
  } else if (warp == 1) {
    // -------------------------------------------------------- MMA issue
    // The whole warp runs the loop (waits and descriptor arithmetic stay
    // warp-uniform); one elected lane issues every MMA and every commit.
    const bool leader = elect_one();
    constexpr uint32_t kIdQK = idesc_bf16(kBM, kBN, false);
    constexpr uint32_t kIdPV = idesc_bf16(kBM, D, true);
    const uint32_t hi = sw128_desc_hi(1024);
    const uint32_t lo_q = sw128_desc_lo(smem_u32(sQ), 16);
    const uint32_t lo_k = sw128_desc_lo(smem_u32(sK), 16);
    const uint32_t lo_v = sw128_desc_lo(smem_u32(sV), C::HALF);
    int ks = 0, kph = 0, vs = 0, vph = 0;
    bool ok = cmax > 0 && mbar_wait_warp(&bar->q_full, 0, s_abort, err, 31);
    if (ok) tc_fence_after();
    // S_x = Q_x K'^T: A = Q_x, B = the K' tile, both K-major in shared memory
    auto qk = [&](int x) -> bool {
      if (!mbar_wait_warp(&bar->k_full[ks], kph, s_abort, err, 32)) return false;
      tc_fence_after();
      if constexpr (GATHER) fence_proxy_async_smem();  // rows written by cp.async
      const uint32_t lq = lo_q + x * (C::TILE >> 4), lk = lo_k + ks * (C::TILE >> 4);
      if (leader) {
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk) {
          const uint32_t step = ((kk >> 2) * C::HALF + (kk & 3) * 32) >> 4;
          mma_ss(tbase + x * 128, desc_words(lq + step, hi), desc_words(lk + step, hi), kIdQK,
                 kk > 0);
        }
        mma_commit(&bar->k_empty[ks]);
        mma_commit(&bar->s_full[x]);
      }
      __syncwarp();
      if (++ks == KS) ks = 0, kph ^= 1;
      return true;
    };
    // O_x += P_x V': A = P_x from TMEM (bf16 pairs over S_x), B = the V' tile
    // (MN-major); the first block of a tile overwrites O_x
    // The first half of P (keys 0-63) is consumed while the softmax still
    // writes the second.
    auto pv = [&](int x, int j) -> bool {
      if (!mbar_wait_warp(&bar->p_full[x][0], j & 1, s_abort, err, 33)) return false;
      if (!mbar_wait_warp(&bar->v_full[vs], vph, s_abort, err, 34)) return false;
      tc_fence_after();
      if constexpr (GATHER) fence_proxy_async_smem();
      const uint32_t lv = lo_v + vs * (C::TILE >> 4);
      for (int h = 0; h < 2; ++h) {
        if (h == 1) {
          if (!mbar_wait_warp(&bar->p_full[x][1], j & 1, s_abort, err, 35)) return false;
          tc_fence_after();
        }
        if (leader) {
#pragma unroll
          for (int k2 = 0; k2 < kBN / 32; ++k2) {
            const int kk = h * (kBN / 32) + k2;
            mma_ts(tbase + 256 + x * 128, tbase + x * 128 + kk * 8,
                   desc_words(lv + kk * (2048 >> 4), hi), kIdPV, (j > 0 || kk > 0) ? 1u : 0u);
          }
        }
        __syncwarp();
      }
      if (leader) mma_commit(&bar->v_empty[vs]);
      __syncwarp();
      if (++vs == VS) vs = 0, vph ^= 1;
      return true;
    };
    if (ok && cA > 0) ok = qk(0);
    if (ok && cB > 0) ok = qk(1);
    for (int j = 0; j < cmax && ok; ++j)
      for (int x = 0; x < 2 && ok; ++x) {
        const int c = x ? cB : cA;
        if (j >= c) continue;
        ok = pv(x, j);
        if (!ok) break;
        if (j + 1 < c) {
          ok = qk(x);
        } else {
          if (leader) mma_commit(&bar->o_final[x]);  // O_x is complete once this lands
          __syncwarp();
        }
      }
    // drain: every MMA issued here completes before TMEM is released
    if (leader) mma_commit(&bar->mma_done);
    __syncwarp();
    int never = 0;
    mbar_wait(&bar->mma_done, 0, &never, nullptr);
  }
  if (GATHER && warp != 1) {
    // ---------------------------------------- K, V gathers (warps 0, 2, 3)
    // The K and V tiles in the TMA producer's order, each row read from its
    // carried position: warp 0 (once Q is issued) fills rows 0-43 of every
    // tile, warp 2 rows 44-87, warp 3 rows 88-127. A warp instruction moves
    // 32 16-byte chunks (whole rows, 2 of them at d = 128) into the
    // 128-byte-swizzled layout; each thread's cp.async arrival on the tile's
    // full barrier (96 expected) lands when its copies have. The positions
    // of a K block are kept for the V block of the same tile that follows it.
    const int gw = warp == 0 ? 0 : warp - 1;
    const int lo = gather_lo(gw), nrows = gather_lo(gw + 1) - lo;
    constexpr int CPR = D / 8;    // 16-byte chunks per row
    constexpr int RPI = 32 / CPR; // rows per warp instruction
    const int sub = lane / CPR, ch = lane % CPR;
    const uint32_t col = (uint32_t)(ch >> 3) * C::HALF;  // 128-byte column block
    const int cc = ch & 7;
    int2 rows_a = make_int2(0, 0), rows_b = rows_a;
    int kseq = 0, vseq = 0;
    auto fill = [&](uint8_t *tile, const bf16 *src, int bh, int2 r) {
      const bf16 *head = src + (size_t)bh * dm.n * D + ch * 8;
#pragma unroll 4
      for (int it = 0; it < nrows / RPI; ++it) {
        const int rl = it * RPI + sub;  // row within the warp's range; warp-uniform half of r
        const int pos = __shfl_sync(0xffffffffu, it * RPI < 32 ? r.x : r.y, rl & 31);
        const int row = lo + rl;
        cp_async16(tile + col + row * 128 + ((cc ^ (row & 7)) << 4), head + (size_t)pos * D);
      }
    };
    auto load_k = [&](const Tile &t, int x, int j) -> bool {
      const int s = kseq % KS, u = kseq / KS;
      const int J = checked_block(t, j, dm, gw == 0 && lane == 0 ? err : nullptr);
      // the positions are read before the wait for the slot: their latency
      // hides behind it
      const int2 r = carried_rows(kpos, t.bh, J, lo, nrows, lane, dm, err);
      if (x) rows_b = r;
      else rows_a = r;
      if (u > 0 && !mbar_wait_warp(&bar->k_empty[s], (u - 1) & 1, s_abort, err, 12))
        return false;
      if (!(fault == 1 && kseq == 0)) {
        fill(sK + s * C::TILE, kg, t.bh, r);
        cp_async_mbar_arrive(&bar->k_full[s]);
      }
      ++kseq;
      return true;
    };
    auto load_v = [&](const Tile &t, int x, int j) -> bool {
      const int s = vseq % VS, u = vseq / VS;
      if (u > 0 && !mbar_wait_warp(&bar->v_empty[s], (u - 1) & 1, s_abort, err, 22))
        return false;
      const int J = checked_block(t, j, dm, nullptr);
      fill(sV + s * C::TILE, vg, t.bh, x ? rows_b : rows_a);
      if (J / dm.spb == t.segI && gw == 0)  // the mask's positions, 4 per lane
        cp_async16(sKP + s * kBN + 4 * lane,
                   kpos + (size_t)t.bh * dm.n + (size_t)J * kBN + 4 * lane);
      cp_async_mbar_arrive(&bar->v_full[s]);
      ++vseq;
      return true;
    };
    bool ok = true;
    if (cA > 0) ok = load_k(tA, 0, 0);
    if (ok && cB > 0) ok = load_k(tB, 1, 0);
    for (int j = 0; j < cmax && ok; ++j)
      for (int x = 0; x < 2 && ok; ++x) {
        const Tile &t = x ? tB : tA;
        if (j >= t.count) continue;
        ok = load_v(t, x, j);
        if (ok && j + 1 < t.count) ok = load_k(t, x, j + 1);
      }
    cp_async_wait_all();  // every copy lands before the CTA exits
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    __syncwarp();
    tc_fence_after();
    tmem_dealloc(tbase, 512);
  }
  } else {
    // ========================================== warpgroups 1, 2: softmax
    asm volatile("setmaxnreg.inc.sync.aligned.u32 %0;" ::"n"(kSoftmaxRegs));
    const int x = (warp - 4) >> 2;  // 0 = tile A, 1 = tile B
    const Tile &t = x ? tB : tA;
    const bool valid = 2 * (int)blockIdx.x + x < total;
    const int quarter = warp & 3;
    const int row = quarter * 32 + lane;
    const uint32_t lane_off = (uint32_t)(quarter * 32) << 16;
    const uint32_t tS = tbase + x * 128 + lane_off;
    const uint32_t tO = tbase + 256 + x * 128 + lane_off;
    const int qrow = t.I * kBM + row;
    const int qp = (valid && qpos) ? qpos[(size_t)t.bh * dm.n + qrow] : qrow;
    const float2 sl2x2 = make_float2(sl2, sl2);
    float m_used = -INFINITY, l = 0.f;
    bool ok = t.count > 0;
    for (int j = 0; j < t.count && ok; ++j) {
      const int J = t.list[j];
      const bool diag = J / dm.spb == t.segI;
      if (!mbar_wait_warp(&bar->s_full[x], j & 1, s_abort, err, 41)) {
        ok = false;
        break;
      }
      tc_fence_after();
      uint32_t v[kBN];
      // the first half of S, then the second half in flight while the first
      // half's row max runs; the empty asm ties each half's registers to its
      // wait so that no use is scheduled before the data has landed
#pragma unroll
      for (int c = 0; c < 2; ++c)
        tmem_ld32(tS + c * 32, *reinterpret_cast<uint32_t(*)[32]>(&v[c * 32]));
      tmem_wait_ld();
#pragma unroll
      for (int c = 0; c < 64; ++c) asm volatile("" : "+r"(v[c]));
#pragma unroll
      for (int c = 2; c < 4; ++c)
        tmem_ld32(tS + c * 32, *reinterpret_cast<uint32_t(*)[32]>(&v[c * 32]));
      float m8[8];
      if (!diag) {
#pragma unroll
        for (int e = 0; e < 8; ++e) m8[e] = __uint_as_float(v[e]);
#pragma unroll
        for (int c = 8; c < 64; c += 8)
#pragma unroll
          for (int e = 0; e < 8; ++e) m8[e] = fmaxf(m8[e], __uint_as_float(v[c + e]));
      }
      tmem_wait_ld();
#pragma unroll
      for (int c = 64; c < kBN; ++c) asm volatile("" : "+r"(v[c]));
      if (diag) {
        if (kpos) {
          // the block's carried original key positions arrived with its V' tile
          const int seq = stream_pos(x, j, cA, cB);
          const int vsl = seq % VS;
          if (!mbar_wait_warp(&bar->v_full[vsl], (seq / VS) & 1, s_abort, err, 42)) {
            ok = false;
            break;
          }
          const int4 *kp4 = reinterpret_cast<const int4 *>(sKP + vsl * kBN);
#pragma unroll
          for (int c4 = 0; c4 < kBN / 4; ++c4) {
            const int4 p = kp4[c4];
            if (p.x > qp) v[4 * c4] = 0xff800000u;  // -inf
            if (p.y > qp) v[4 * c4 + 1] = 0xff800000u;
            if (p.z > qp) v[4 * c4 + 2] = 0xff800000u;
            if (p.w > qp) v[4 * c4 + 3] = 0xff800000u;
          }
        } else {
          const int lim = qp - J * kBN;  // last visible column
#pragma unroll
          for (int c = 0; c < kBN; ++c)
            if (c > lim) v[c] = 0xff800000u;
        }
      }
      // row max: eight independent chains over the 128 columns (the
      // three-input max.f32 measured no faster); off the
      // diagonal segment the first half was taken while the second loaded
      if (diag) {
#pragma unroll
        for (int e = 0; e < 8; ++e) m8[e] = __uint_as_float(v[e]);
#pragma unroll
        for (int c = 8; c < 64; c += 8)
#pragma unroll
          for (int e = 0; e < 8; ++e) m8[e] = fmaxf(m8[e], __uint_as_float(v[c + e]));
      }
#pragma unroll
      for (int c = 64; c < kBN; c += 8)
#pragma unroll
        for (int e = 0; e < 8; ++e) m8[e] = fmaxf(m8[e], __uint_as_float(v[c + e]));
      const float mx = fmaxf(fmaxf(fmaxf(m8[0], m8[1]), fmaxf(m8[2], m8[3])),
                             fmaxf(fmaxf(m8[4], m8[5]), fmaxf(m8[6], m8[7])));
      const float mxs = mx * sl2;
      float alpha = 1.f;
      if (mxs > m_used + kRescaleLog2) {
        alpha = exp2f(m_used - mxs);
        m_used = mxs;
      }
      const float mu = m_used == -INFINITY ? 0.f : m_used;
      __syncwarp();  // reconverge after the per-row branches before aligned TMEM work
      // O_x already holds every block before j (S_x(j) was signalled after
      // those products completed). The rescale decision is per row but
      // tcgen05.ld/st are warp-wide: the warp takes the branch when any row
      // needs it, and rows with alpha == 1 multiply by one.
      if (j > 0 && __any_sync(0xffffffffu, alpha != 1.f)) {
#pragma unroll 1
        for (int c = 0; c < D / 32; ++c) {
          uint32_t r[32];
          tmem_ld32(tO + c * 32, r);
          tmem_wait_ld();
#pragma unroll
          for (int e = 0; e < 32; ++e) r[e] = __float_as_uint(__uint_as_float(r[e]) * alpha);
          tmem_st32(tO + c * 32, r);
        }
        tmem_wait_st();
      }
      // p = 2^(s sigma log2(e) - m): packed fp32x2 FMA and the hardware exp2
      // (the FMA-pipe cubic for kPolyPairs of every 16 pairs); P to TMEM as
      // bf16 pairs over the first 64 columns of S_x, each half signalled as
      // soon as it is written
      const float2 neg_m2 = make_float2(-mu, -mu);
      float2 acc[4] = {make_float2(0.f, 0.f), make_float2(0.f, 0.f), make_float2(0.f, 0.f),
                       make_float2(0.f, 0.f)};
#pragma unroll
      for (int c = 0; c < kBN / 32; ++c) {
        uint32_t pk[16];
#pragma unroll
        for (int e = 0; e < 16; ++e) {
          const float2 xx = __ffma2_rn(make_float2(__uint_as_float(v[c * 32 + 2 * e]),
                                                   __uint_as_float(v[c * 32 + 2 * e + 1])),
                                       sl2x2, neg_m2);
          const float2 p = poly_pair(e) ? exp2_poly2(xx)
                                        : make_float2(ex2_approx(xx.x), ex2_approx(xx.y));
          acc[e & 3] = __fadd2_rn(acc[e & 3], p);
          pk[e] = pack_bf16(p.x, p.y);
        }
        tmem_st16(tS + c * 16, pk);
        if (c == 1 || c == 3) {
          tmem_wait_st();
          tc_fence_before();
          warp_arrive(&bar->p_full[x][c >> 1], lane);
        }
      }
      const float2 a = __fadd2_rn(__fadd2_rn(acc[0], acc[1]), __fadd2_rn(acc[2], acc[3]));
      l = l * alpha + (a.x + a.y);
    }
    if (ok && !mbar_wait_warp(&bar->o_final[x], 0, s_abort, err, 44)) ok = false;
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
    // in every output buffer, at head head_offset + g of hq_total
    const size_t orow_off =
        ((size_t)((t.bg / dm.hq) * outs.hq_total + outs.head_offset + t.bg % dm.hq) * dm.n +
         (orow_i < 0 ? 0 : orow_i)) * D;
    if (ok) {
      tc_fence_after();
      const float inv = l > 0.f ? 1.f / l : 0.f;
#pragma unroll
      for (int c = 0; c < D / 32; ++c) {
        uint32_t r[32];
        tmem_ld32(tO + c * 32, r);
        tmem_wait_ld();
        uint32_t pk[16];
#pragma unroll
        for (int e = 0; e < 16; ++e)
          pk[e] = pack_bf16(__uint_as_float(r[2 * e]) * inv, __uint_as_float(r[2 * e + 1]) * inv);
        for (int o = 0; o < outs.n; ++o) {
          uint4 *dst = reinterpret_cast<uint4 *>(static_cast<bf16 *>(outs.p[o]) + orow_off + c * 32);
#pragma unroll
          for (int q4 = 0; q4 < 4; ++q4)
            dst[q4] = make_uint4(pk[4 * q4], pk[4 * q4 + 1], pk[4 * q4 + 2], pk[4 * q4 + 3]);
        }
      }
      if (lse)
        lse[(size_t)t.bg * dm.n + orow_i] = l > 0.f ? (m_used + log2f(l)) * kLn2 : -INFINITY;
    } else if (valid && t.count == 0 && orow_i >= 0) {
      for (int o = 0; o < outs.n; ++o)
        for (int c = 0; c < D / 8; ++c)
          reinterpret_cast<uint4 *>(static_cast<bf16 *>(outs.p[o]) + orow_off)[c] =
              make_uint4(0, 0, 0, 0);
      if (lse) lse[(size_t)t.bg * dm.n + orow_i] = -INFINITY;
    }
    tc_fence_before();
    __syncthreads();
  }
}

template <int D, bool GATHER>
cudaError_t run2(const Dims &dm, const void *q, const void *kp, const void *vp,
                 const int32_t *kpos, const int32_t *qpos, const int32_t *idx, const int32_t *cnt,
                 const OutSet &outs, float *lse, float sigma, int *err, int fault, bool scatter,
                 cudaStream_t st) {
  if (GATHER && !kpos) return cudaErrorInvalidValue;
  CUtensorMap mq, mk, mv;
  if (!make_tile_map(&mq, q, (uint64_t)dm.b * dm.hq * dm.n, D, kBM)) return cudaErrorInvalidValue;
  if (GATHER) {
    mk = mq, mv = mq;  // unused: K and V rows are gathered with cp.async
  } else if (!make_tile_map(&mk, kp, (uint64_t)dm.b * dm.hkv * dm.n, D, kBN) ||
             !make_tile_map(&mv, vp, (uint64_t)dm.b * dm.hkv * dm.n, D, kBN)) {
    return cudaErrorInvalidValue;
  }
  constexpr size_t smem = smem2<D>();
  auto kern = attn_tc2_kernel<D, GATHER>;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       (int)smem);
  if (e != cudaSuccess) return e;
  // The setmaxnreg split above is only safe at the launch allocation it was
  // sized for; with any other count the softmax warps could wait forever.
  cudaFuncAttributes fa;
  e = cudaFuncGetAttributes(&fa, kern);
  if (e != cudaSuccess) return e;
  if (fa.numRegs != kLaunchRegs) return cudaErrorInvalidConfiguration;
  const long long total = (long long)dm.b * dm.hq * dm.nb;
  const unsigned grid = (unsigned)((total + 1) / 2);
  kern<<<grid, kThreads, smem, st>>>(mq, mk, mv, kpos, qpos, idx, cnt, outs, lse, dm,
                                    sigma * kLog2e, err, fault, scatter ? 1 : 0,
                                    (const bf16 *)kp, (const bf16 *)vp);
  return cudaGetLastError();
}

}  // namespace

cudaError_t launch_attn_tc2(const Dims &dm, const void *q, const void *kp, const void *vp,
                            const int32_t *kpos, const int32_t *qpos, const int32_t *idx,
                            const int32_t *cnt, const OutSet &outs, float *lse, float sigma,
                            int *err, int fault, bool scatter, bool gather, cudaStream_t st) {
  if (gather) {
    if (dm.d == 64)
      return run2<64, true>(dm, q, kp, vp, kpos, qpos, idx, cnt, outs, lse, sigma, err, fault,
                            scatter, st);
    return run2<128, true>(dm, q, kp, vp, kpos, qpos, idx, cnt, outs, lse, sigma, err, fault,
                           scatter, st);
  }
  if (dm.d == 64)
    return run2<64, false>(dm, q, kp, vp, kpos, qpos, idx, cnt, outs, lse, sigma, err, fault,
                           scatter, st);
  return run2<128, false>(dm, q, kp, vp, kpos, qpos, idx, cnt, outs, lse, sigma, err, fault,
                          scatter, st);
}

cudaError_t launch_attn_bcast(const Dims &dm, const void *q, const void *kp, const void *vp,
                              const int32_t *kpos, const int32_t *idx, const int32_t *cnt,
                              const OutSet &outs, float sigma, int *err, cudaStream_t st) {
  cudaError_t e = cudaErrorNotSupported;
  if (attn_tc_supported(dm))
    e = launch_attn_tc2(dm, q, kp, vp, kpos, nullptr, idx, cnt, outs, nullptr, sigma, err, 0,
                        false, false, st);
  else if (attn_tc64_supported(dm))
    e = launch_attn_tc64(dm, q, kp, vp, kpos, nullptr, idx, cnt, outs, nullptr, sigma, err, 0,
                         false, false, st);
  return e == cudaErrorInvalidConfiguration ? cudaErrorNotSupported : e;
}

}  // namespace pbs

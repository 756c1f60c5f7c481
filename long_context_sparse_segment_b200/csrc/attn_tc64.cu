// Block-sparse causal attention over the permuted keys on the sm_100a
// tensor cores for key blocks of B = 64, two query tiles per CTA.
//
// "Sparser Block-Sparse Attention via Token Permutation", sciencestack.ai
// Figure 1 caption (inter-segment causality is kept; the blocks of the
// on-diagonal segment are computed with a per-element mask, inter-segment
// blocks are fully visible or skipped) and gist.science summary, "Methodik"
// 4 (a permuted FlashAttention kernel walks the kept blocks); the block size
// B is the method's free parameter.
//
// The MMA's M is 128 rows, so a query tile is two consecutive 64-row query
// blocks 2P and 2P + 1 of one head, each with its own list of kept key
// blocks. The tile walks the union of the two lists (merged, ascending),
// two key blocks at a time: a step j takes union entries 2j and 2j + 1
// (J0, J1), loads them as the two 64-row halves of one 128-row K' tile and
// V' tile (two TMA boxes each), and runs one 128 x 128 product
// S = Q [K'_J0; K'_J1]^T and one O += P [V'_J0; V'_J1] with K = 128. The
// rows of a query block whose list does not hold J0 (J1) see that half of
// the step masked, so each row attends to exactly its own list; an odd last
// entry is loaded twice and its second copy masked everywhere. A CTA takes
// two such tiles, A and B, and the tensor core alternates between them as in
// the B = 128 kernel (attn_tc2.cu):
//   S_A(0), S_B(0), then per step j:  O_A += P_A(j) V'_A(j), S_A(j+1),
//                                     O_B += P_B(j) V'_B(j), S_B(j+1).
// TMEM: S_A, S_B (P over the first 64 columns of its S as bf16 pairs), O_A,
// O_B. 384 threads:
//   warp 0        TMA: Q_A, Q_B, then K' and V' tiles in the order the
//                 tensor core consumes them; a key block in the own segment
//                 of either query block brings its carried key positions
//                 with its V' half;
//   warp 1        tcgen05.mma issue;
//   warps 2, 3    idle, or with GATHER (pbs_attn_fwd_gather), and warp 0
//                 once Q is issued, the K' and V' tiles: each row read from
//                 the natural K, V at its carried position with cp.async,
//                 into the layout the TMA would write;
//   warps 4-11    softmax of tile A, of tile B: one thread per query row,
//                 the 128 key columns of a step in registers.
// Each role walks the same merged list. Every mbarrier wait is bounded; on
// expiry the CTA records PBS_ERR_TIMEOUT, drains what it issued, frees TMEM
// and exits.
#include <math.h>

#include "common.cuh"
#include "internal.h"
#include "tc.cuh"

namespace pbs {
namespace {

using bf16 = __nv_bfloat16;
using namespace tc;

constexpr int kBM = 128;  // query rows per tile (MMA M): two query blocks
constexpr int kQB = 64;   // rows per query block
constexpr int kSB = 64;   // keys per block
constexpr int kBN = 128;  // keys per step: two blocks
constexpr int kThreads = 384;
constexpr int kLaunchRegs = 168;   // per thread at launch (checked on the host)
constexpr int kCtrlRegs = 56;      // warps 0-3 after setmaxnreg.dec
constexpr int kSoftmaxRegs = 224;  // warps 4-11 after setmaxnreg.inc
static_assert(128 * kCtrlRegs + 256 * kSoftmaxRegs <= kThreads * kLaunchRegs,
              "register split exceeds the launch allocation");
constexpr float kRescaleLog2 = 8.0f;  // move the running max only past 2^8

template <int D>
struct Cfg64 {
  static constexpr int H = D / 64;                           // 128-byte atoms per row
  static constexpr uint32_t TILE = (uint32_t)kBM * D * 2;    // bytes of a 128-row tile
  static constexpr uint32_t HALF = (uint32_t)kBM * 128;      // one 64-column box of it
  static constexpr uint32_t SUB = (uint32_t)kSB * 128;       // its 64-row part (one TMA box)
  static constexpr int KS = D == 128 ? 2 : 4;                // K' ring depth
  static constexpr int VS = D == 128 ? 3 : 4;                // V' ring depth
};

template <int D>
struct Bars64 {
  uint64_t q_full, k_full[Cfg64<D>::KS], k_empty[Cfg64<D>::KS], v_full[Cfg64<D>::VS],
      v_empty[Cfg64<D>::VS], s_full[2], p_full[2][2], o_final[2], mma_done;
};

template <int D>
constexpr size_t smem64() {
  return 1024 + 2 * (size_t)Cfg64<D>::TILE + (size_t)(Cfg64<D>::KS + Cfg64<D>::VS) * Cfg64<D>::TILE +
         (size_t)Cfg64<D>::VS * kBN * 4 + sizeof(Bars64<D>) + 16;
}
static_assert(smem64<128>() <= 232448, "shared memory (d = 128)");
static_assert(smem64<64>() <= 232448, "shared memory (d = 64)");

// One query tile: query blocks 2P and 2P + 1 of head bg (the second may lie
// past the end of the sequence), each with its list of kept key blocks.
struct Tile64 {
  int bg, P, bh, seg[2], c[2];
  bool has[2];
  const int32_t *list[2];
};

__device__ __forceinline__ Tile64 make_tile(int item, int total, const Dims &dm,
                                            const int32_t *blk_idx, const int32_t *blk_cnt,
                                            int *err) {
  Tile64 t;
  t.bg = 0, t.P = 0, t.bh = 0;
  for (int h = 0; h < 2; ++h) t.seg[h] = 0, t.c[h] = 0, t.has[h] = false, t.list[h] = blk_idx;
  if (item >= total) return t;
  // KV groups one after the other (the K'/V' tiles in use at a time are one
  // KV head's), inside a group heavy query tiles first, the G query heads
  // of a tile adjacent
  const int np = (dm.nb + 1) / 2;
  const int per_group = dm.G * np;
  const int r = item % per_group;
  t.bh = item / per_group;
  t.P = np - 1 - r / dm.G;
  t.bg = (t.bh / dm.hkv) * dm.hq + (t.bh % dm.hkv) * dm.G + r % dm.G;
  for (int h = 0; h < 2; ++h) {
    const int qb = 2 * t.P + h;
    t.has[h] = qb < dm.nb;
    if (!t.has[h]) continue;
    t.seg[h] = qb / dm.spb;
    t.list[h] = blk_idx + ((size_t)t.bg * dm.nb + qb) * dm.nb;
    int c = blk_cnt[(size_t)t.bg * dm.nb + qb];
    if (c < 0 || c > dm.nb) {
      report(err, PBS_ERR_DEVICE_ASSERT);
      c = 0;
    }
    t.c[h] = c;
  }
  return t;
}

// The ascending union of a tile's two lists, walked one block at a time. An
// entry outside [0, nb) is reported and read as block 0; the walk ends after
// at most c[0] + c[1] steps whatever the lists hold.
struct Union {
  const int32_t *l[2];
  int c[2], i[2];
  __device__ __forceinline__ void init(const Tile64 &t) {
    for (int h = 0; h < 2; ++h) l[h] = t.list[h], c[h] = t.c[h], i[h] = 0;
  }
  __device__ __forceinline__ bool more() const { return i[0] < c[0] || i[1] < c[1]; }
  // the next step's two blocks (the second a masked copy of the first when
  // the union has one entry left) and which lists hold each
  __device__ __forceinline__ void next2(int nb, int *err, int (&J)[2], int (&in)[2]) {
    J[0] = next(nb, err, &in[0]);
    if (more()) {
      J[1] = next(nb, err, &in[1]);
    } else {
      J[1] = J[0];
      in[1] = 0;
    }
  }
  // the next block and which of the two lists hold it (bit h)
  __device__ __forceinline__ int next(int nb, int *err, int *in) {
    int v[2];
    for (int h = 0; h < 2; ++h) {
      v[h] = 0x7fffffff;
      if (i[h] < c[h]) {
        v[h] = l[h][i[h]];
        if (v[h] < 0 || v[h] >= nb) {
          report(err, PBS_ERR_DEVICE_ASSERT);
          v[h] = 0;
        }
      }
    }
    const int J = min(v[0], v[1]);
    *in = 0;
    for (int h = 0; h < 2; ++h)
      if (i[h] < c[h] && v[h] == J) *in |= 1 << h, ++i[h];
    return J;
  }
};

// Rows of a step's K'/V' tile that gathering warp g (of three) fills:
// [gather_lo(g), gather_lo(g + 1)), at most 64, in multiples of 4.
__device__ __forceinline__ constexpr int gather_lo(int g) { return g == 3 ? kBN : 44 * g; }

// Carried positions of rows lo + lane and lo + 32 + lane of a step's tile
// (row r is key r mod 64 of block J[r / 64]) of KV head bh; rows past `rows`
// are not read. A position outside its block's segment is reported and
// replaced by the key's own index.
__device__ __forceinline__ int2 carried_rows(const int32_t *__restrict__ kpos, int bh,
                                             const int (&J)[2], int lo, int rows, int lane,
                                             const Dims &dm, int *err) {
  int r2[2];
  for (int k = 0; k < 2; ++k) {
    const int r = lo + lane + 32 * k;
    const int Jr = J[r >> 6];
    const int own = Jr * kSB + (r & (kSB - 1));
    if (lane + 32 * k >= rows) {
      r2[k] = Jr * kSB;  // any key of the block: inside its segment, never read
      continue;
    }
    int pos = __ldg(kpos + (size_t)bh * dm.n + own);
    const int seg0 = (Jr / dm.spb) * dm.S;
    const unsigned span = (unsigned)min(dm.S, dm.n - seg0);  // the last segment may be short
    if ((unsigned)(pos - seg0) >= span) {
      report(err, PBS_ERR_DEVICE_ASSERT);
      pos = own;
    }
    r2[k] = pos;
  }
  return make_int2(r2[0], r2[1]);
}

// Position of step j of tile x (0 = A, 1 = B) in the interleaved stream
// A0 B0 A1 B1 ... (a list that has ended drops out).
__device__ __forceinline__ int stream_pos(int x, int j, int cA, int cB) {
  return x == 0 ? j + min(j, cB) : j + min(j + 1, cA);
}

// GATHER: the permutation is applied on the fly. kg and vg are the natural
// K and V; warps 0 (after Q), 2 and 3 fetch each step's rows by their
// carried positions with cp.async (no K', V' copies); tmK and tmV are unused.
template <int D, bool GATHER>
__global__ void __launch_bounds__(kThreads, 1)
    attn_tc64_kernel(const __grid_constant__ CUtensorMap tmQ,
                     const __grid_constant__ CUtensorMap tmK,
                     const __grid_constant__ CUtensorMap tmV, const int32_t *__restrict__ kpos,
                     const int32_t *__restrict__ qpos, const int32_t *__restrict__ blk_idx,
                     const int32_t *__restrict__ blk_cnt, const __grid_constant__ OutSet outs,
                     float *__restrict__ lse, Dims dm, float sl2, int *err, int fault,
                     int scatter, const bf16 *__restrict__ kg, const bf16 *__restrict__ vg) {
  using C = Cfg64<D>;
  constexpr int KS = C::KS, VS = C::VS;
  extern __shared__ uint8_t smem_raw[];
  uint8_t *base = reinterpret_cast<uint8_t *>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~(uintptr_t)1023);
  uint8_t *sQ = base;                    // [2] query tiles
  uint8_t *sK = sQ + 2 * C::TILE;        // [KS] K' tiles of two blocks
  uint8_t *sV = sK + KS * C::TILE;       // [VS] V' tiles of two blocks
  int32_t *sKP = reinterpret_cast<int32_t *>(sV + VS * C::TILE);  // [VS][kBN]
  Bars64<D> *bar = reinterpret_cast<Bars64<D> *>(sKP + VS * kBN);
  uint32_t *s_tmem = reinterpret_cast<uint32_t *>(bar + 1);
  volatile int *s_abort = reinterpret_cast<volatile int *>(s_tmem + 1);
  int *s_cnt = const_cast<int *>(s_abort) + 1;  // [2] steps of each tile

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int total = dm.b * dm.hq * ((dm.nb + 1) / 2);
  const Tile64 tA = make_tile(2 * blockIdx.x, total, dm, blk_idx, blk_cnt, tid == 0 ? err : nullptr);
  const Tile64 tB = make_tile(2 * blockIdx.x + 1, total, dm, blk_idx, blk_cnt, nullptr);

  if (tid == 0) {
    mbar_init(&bar->q_full, 1);
    // full: the TMA's expect-tx arrival, or one cp.async arrival per
    // gathering thread
    const int fill_count = GATHER ? 96 : 1;
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
      mbar_init(&bar->p_full[x][1], 4);  // for the step's first and second block
      mbar_init(&bar->o_final[x], 1);
    }
    mbar_init(&bar->mma_done, 1);
    *s_abort = 0;
    // every role walks the same unions; their step counts are found once here
    for (int x = 0; x < 2; ++x) {
      Union u;
      u.init(x ? tB : tA);
      int n = 0, in;
      while (u.more()) u.next(dm.nb, err, &in), ++n;
      s_cnt[x] = (n + 1) / 2;
    }
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
  const int cA = s_cnt[0], cB = s_cnt[1];
  const int cmax = cA > cB ? cA : cB;
  if (warp < 4) {
  // =============================================== warpgroup 0: TMA and MMA
  asm volatile("setmaxnreg.dec.sync.aligned.u32 %0;" ::"n"(kCtrlRegs));
  if (warp == 0) {
    // ------------------------------------------------------- TMA loads
    // Order: K'_A(0), K'_B(0), then per step j and tile x: V'_x(j),
    // K'_x(j+1) -- the tensor core's order. A tile is two 64-row boxes per
    // 64 columns, one from each of the step's blocks. The whole warp runs
    // the loop; one elected lane issues the copies.
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
          const Tile64 &t = x ? tB : tA;
          if ((x ? cB : cA) == 0) continue;
          for (int h = 0; h < C::H; ++h)
            tma_load_2d(sQ + x * C::TILE + h * C::HALF, &tmQ, &bar->q_full, h * 64,
                        t.bg * dm.n + t.P * kBM);
        }
      }
      __syncwarp();
      q_issued = true;
      // a step's K' tile is loaded before its V' tile, so the pair of
      // blocks found for the K' tile is kept for the V' tile that follows
      Union uA, uB;
      uA.init(tA), uB.init(tB);
      int JA[2] = {0, 0}, JB[2] = {0, 0};
      auto load_k = [&](int x) -> bool {
        const int s = kseq % KS, u = kseq / KS;
        if (u > 0 && !mbar_wait_warp(&bar->k_empty[s], (u - 1) & 1, s_abort, err, 11))
          return false;
        int in[2];
        int(&J)[2] = x ? JB : JA;
        (x ? uB : uA).next2(dm.nb, nullptr, J, in);
        const int row0 = (x ? tB : tA).bh * dm.n;
        if (leader) {
          mbar_expect_tx(&bar->k_full[s], C::TILE);
          if (!(fault == 1 && kseq == 0))
            for (int h = 0; h < C::H; ++h)
              for (int b = 0; b < 2; ++b)
                tma_load_2d(sK + s * C::TILE + h * C::HALF + b * C::SUB, &tmK, &bar->k_full[s],
                            h * 64, row0 + J[b] * kSB);
        }
        __syncwarp();
        ++kseq;
        return true;
      };
      auto load_v = [&](int x) -> bool {
        const int s = vseq % VS, u = vseq / VS;
        if (u > 0 && !mbar_wait_warp(&bar->v_empty[s], (u - 1) & 1, s_abort, err, 21))
          return false;
        const Tile64 &t = x ? tB : tA;
        const int(&J)[2] = x ? JB : JA;
        bool with_pos[2];
        for (int b = 0; b < 2; ++b) {
          const int sj = J[b] / dm.spb;
          with_pos[b] = kpos && ((t.has[0] && sj == t.seg[0]) || (t.has[1] && sj == t.seg[1]));
        }
        if (leader) {
          mbar_expect_tx(&bar->v_full[s], C::TILE + (with_pos[0] + with_pos[1]) * kSB * 4);
          for (int h = 0; h < C::H; ++h)
            for (int b = 0; b < 2; ++b)
              tma_load_2d(sV + s * C::TILE + h * C::HALF + b * C::SUB, &tmV, &bar->v_full[s],
                          h * 64, t.bh * dm.n + J[b] * kSB);
          for (int b = 0; b < 2; ++b)
            if (with_pos[b])
              bulk_load(sKP + s * kBN + b * kSB, kpos + (size_t)t.bh * dm.n + (size_t)J[b] * kSB,
                        kSB * 4, &bar->v_full[s]);
        }
        __syncwarp();
        ++vseq;
        return true;
      };
      bool ok = !GATHER;  // with GATHER, warps 0, 2 and 3 load K' and V' below
      if (ok && cA > 0) ok = load_k(0);
      if (ok && cB > 0) ok = load_k(1);
      for (int j = 0; j < cmax && ok; ++j)
        for (int x = 0; x < 2 && ok; ++x) {
          const int c = x ? cB : cA;
          if (j >= c) continue;
          ok = load_v(x);
          if (ok && j + 1 < c) ok = load_k(x);
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
    // warp-wide loop, one elected lane issues every MMA and every commit
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
    // S_x = Q_x K'^T: A = Q_x, B = the step's K' tile, both K-major
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
    // O_x += P_x V': A = P_x from TMEM (bf16 pairs over S_x), B = the V'
    // tile (MN-major); the first block's 64 keys while the softmax still
    // writes the second's; the first step of a tile overwrites O_x
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
    // The K' and V' tiles in the TMA loader's order, each row read from its
    // carried position: warp 0 (once Q is issued) fills rows 0-43 of every
    // tile, warp 2 rows 44-87, warp 3 rows 88-127. A warp instruction moves
    // 32 16-byte chunks into the 128-byte-swizzled layout; each thread's
    // cp.async arrival on the tile's full barrier (96 expected) lands when
    // its copies have. The positions of a step's K' tile are kept for its V'
    // tile, which also brings the positions of the step's two blocks.
    const int gw = warp == 0 ? 0 : warp - 1;
    const int lo = gather_lo(gw), nrows = gather_lo(gw + 1) - lo;
    constexpr int CPR = D / 8;    // 16-byte chunks per row
    constexpr int RPI = 32 / CPR; // rows per warp instruction
    const int sub = lane / CPR, ch = lane % CPR;
    const uint32_t col = (uint32_t)(ch >> 3) * C::HALF;  // 128-byte column block
    const int cc = ch & 7;
    int2 rows_a = make_int2(0, 0), rows_b = rows_a;
    int JA[2] = {0, 0}, JB[2] = {0, 0};
    Union uA, uB;
    uA.init(tA), uB.init(tB);
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
    auto load_k = [&](int x) -> bool {
      const int s = kseq % KS, u = kseq / KS;
      const Tile64 &t = x ? tB : tA;
      int in[2];
      int(&J)[2] = x ? JB : JA;
      (x ? uB : uA).next2(dm.nb, nullptr, J, in);
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
    auto load_v = [&](int x) -> bool {
      const int s = vseq % VS, u = vseq / VS;
      if (u > 0 && !mbar_wait_warp(&bar->v_empty[s], (u - 1) & 1, s_abort, err, 22))
        return false;
      const Tile64 &t = x ? tB : tA;
      const int(&J)[2] = x ? JB : JA;
      fill(sV + s * C::TILE, vg, t.bh, x ? rows_b : rows_a);
      if (gw == 0)  // the mask's positions of both blocks, 4 per lane
        cp_async16(sKP + s * kBN + 4 * lane,
                   kpos + (size_t)t.bh * dm.n + (size_t)J[lane >> 4] * kSB + 4 * (lane & 15));
      cp_async_mbar_arrive(&bar->v_full[s]);
      ++vseq;
      return true;
    };
    bool ok = true;
    if (cA > 0) ok = load_k(0);
    if (ok && cB > 0) ok = load_k(1);
    for (int j = 0; j < cmax && ok; ++j)
      for (int x = 0; x < 2 && ok; ++x) {
        const int c = x ? cB : cA;
        if (j >= c) continue;
        ok = load_v(x);
        if (ok && j + 1 < c) ok = load_k(x);
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
    const Tile64 &t = x ? tB : tA;
    const int cnt = x ? cB : cA;
    const int quarter = warp & 3;
    const int row = quarter * 32 + lane;
    const int hr = row / kQB;  // which query block of the tile (warp-uniform)
    const bool real = t.has[hr] && 2 * (int)blockIdx.x + x < total;
    const uint32_t lane_off = (uint32_t)(quarter * 32) << 16;
    const uint32_t tS = tbase + x * 128 + lane_off;
    const uint32_t tO = tbase + 256 + x * 128 + lane_off;
    const int qrow = t.P * kBM + row;
    const int qp = (real && qpos) ? qpos[(size_t)t.bh * dm.n + qrow] : qrow;
    const float2 sl2x2 = make_float2(sl2, sl2);
    float m_used = -INFINITY, l = 0.f;
    bool ok = cnt > 0;
    Union un;
    un.init(t);
    for (int j = 0; j < cnt && ok; ++j) {
      int J[2], in[2];
      un.next2(dm.nb, nullptr, J, in);
      if (!mbar_wait_warp(&bar->s_full[x], j & 1, s_abort, err, 41)) {
        ok = false;
        break;
      }
      tc_fence_after();
      uint32_t v[kBN];
#pragma unroll
      for (int c = 0; c < kBN / 32; ++c)
        tmem_ld32(tS + c * 32, *reinterpret_cast<uint32_t(*)[32]>(&v[c * 32]));
      tmem_wait_ld();
#pragma unroll
      for (int c = 0; c < kBN; ++c) asm volatile("" : "+r"(v[c]));
      // per block of the step: masked whole where this row's list does not
      // keep it (or the row has no query), per element in the own segment
      const bool mine0 = real && (in[0] >> hr & 1), mine1 = real && (in[1] >> hr & 1);
      const bool diag0 = mine0 && J[0] / dm.spb == t.seg[hr];
      const bool diag1 = mine1 && J[1] / dm.spb == t.seg[hr];
      const int4 *kp4 = nullptr;
      if (kpos && __any_sync(0xffffffffu, diag0 || diag1)) {
        // the blocks' carried original key positions arrived with the V' tile
        const int seq = stream_pos(x, j, cA, cB);
        const int vsl = seq % VS;
        if (!mbar_wait_warp(&bar->v_full[vsl], (seq / VS) & 1, s_abort, err, 42)) {
          ok = false;
          break;
        }
        kp4 = reinterpret_cast<const int4 *>(sKP + vsl * kBN);
      }
      // Columns past lim_b of block b are hidden: none when the row's list
      // keeps the block off its own segment (the common step), all when it
      // does not keep it, the causal limit on the own segment; with carried
      // positions the own segment's blocks are masked per column instead.
      // One branch skips the selects when no column is hidden (run on every
      // step they took ~10 % of the kernel at llama32k).
      const int lim0 = !mine0 ? -1 : (diag0 && !kp4) ? qp - J[0] * kSB : kSB;
      const int lim1 = !mine1 ? -1 : (diag1 && !kp4) ? qp - J[1] * kSB : kSB;
      if (lim0 < kSB - 1 || lim1 < kSB - 1) {
#pragma unroll
        for (int c = 0; c < kSB; ++c) {
          if (c > lim0) v[c] = 0xff800000u;  // -inf
          if (c > lim1) v[kSB + c] = 0xff800000u;
        }
      }
      if (kp4) {
#pragma unroll
        for (int b = 0; b < 2; ++b) {
          if (!(b ? diag1 : diag0)) continue;
#pragma unroll
          for (int c4 = 0; c4 < kSB / 4; ++c4) {
            const int4 p = kp4[b * (kSB / 4) + c4];
            const int c = b * kSB + 4 * c4;
            if (p.x > qp) v[c] = 0xff800000u;
            if (p.y > qp) v[c + 1] = 0xff800000u;
            if (p.z > qp) v[c + 2] = 0xff800000u;
            if (p.w > qp) v[c + 3] = 0xff800000u;
          }
        }
      }
      // row max: eight independent chains over the 128 columns
      float m8[8];
#pragma unroll
      for (int e = 0; e < 8; ++e) m8[e] = __uint_as_float(v[e]);
#pragma unroll
      for (int c = 8; c < kBN; c += 8)
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
      // O_x already holds every step before j; rows with alpha == 1
      // multiply by one when any row of the warp rescales
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
      // p = 2^(s sigma log2(e) - m) on the hardware exp2; P to TMEM as bf16
      // pairs over the first 64 columns of S_x, each block's half signalled
      // as soon as it is written
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
          const float2 p = make_float2(ex2_approx(xx.x), ex2_approx(xx.y));
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
    if (scatter && real) {
      orow_i = qp;
      if (qp < 0 || qp >= dm.n) {
        report(err, PBS_ERR_DEVICE_ASSERT);
        ok = false, orow_i = -1;
      }
    }
    const size_t orow_off =
        ((size_t)((t.bg / dm.hq) * outs.hq_total + outs.head_offset + t.bg % dm.hq) * dm.n +
         (orow_i < 0 ? 0 : orow_i)) * D;
    if (ok && real) {
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
    } else if (real && cnt == 0 && orow_i >= 0) {
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
cudaError_t run64(const Dims &dm, const void *q, const void *kp, const void *vp,
                  const int32_t *kpos, const int32_t *qpos, const int32_t *idx, const int32_t *cnt,
                  const OutSet &outs, float *lse, float sigma, int *err, int fault, bool scatter,
                  cudaStream_t st) {
  if (GATHER && !kpos) return cudaErrorInvalidValue;
  CUtensorMap mq, mk, mv;
  if (!make_tile_map(&mq, q, (uint64_t)dm.b * dm.hq * dm.n, D, kBM)) return cudaErrorInvalidValue;
  if (GATHER) {
    mk = mq, mv = mq;  // unused: K and V rows are gathered with cp.async
  } else if (!make_tile_map(&mk, kp, (uint64_t)dm.b * dm.hkv * dm.n, D, kSB) ||
             !make_tile_map(&mv, vp, (uint64_t)dm.b * dm.hkv * dm.n, D, kSB)) {
    return cudaErrorInvalidValue;
  }
  constexpr size_t smem = smem64<D>();
  auto kern = attn_tc64_kernel<D, GATHER>;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       (int)smem);
  if (e != cudaSuccess) return e;
  // The setmaxnreg split is only safe at the launch allocation it was sized
  // for; with any other count the softmax warps could wait forever.
  cudaFuncAttributes fa;
  e = cudaFuncGetAttributes(&fa, kern);
  if (e != cudaSuccess) return e;
  if (fa.numRegs != kLaunchRegs) return cudaErrorInvalidConfiguration;
  const long long total = (long long)dm.b * dm.hq * ((dm.nb + 1) / 2);
  const unsigned grid = (unsigned)((total + 1) / 2);
  kern<<<grid, kThreads, smem, st>>>(mq, mk, mv, kpos, qpos, idx, cnt, outs, lse, dm,
                                    sigma * kLog2e, err, fault, scatter ? 1 : 0,
                                    (const bf16 *)kp, (const bf16 *)vp);
  return cudaGetLastError();
}

}  // namespace

bool attn_tc64_supported(const Dims &dm) { return dm.B == 64 && (dm.d == 128 || dm.d == 64); }

cudaError_t launch_attn_tc64(const Dims &dm, const void *q, const void *kp, const void *vp,
                             const int32_t *kpos, const int32_t *qpos, const int32_t *idx,
                             const int32_t *cnt, const OutSet &outs, float *lse, float sigma,
                             int *err, int fault, bool scatter, bool gather, cudaStream_t st) {
  if (gather) {
    if (dm.d == 64)
      return run64<64, true>(dm, q, kp, vp, kpos, qpos, idx, cnt, outs, lse, sigma, err, fault,
                             scatter, st);
    return run64<128, true>(dm, q, kp, vp, kpos, qpos, idx, cnt, outs, lse, sigma, err, fault,
                            scatter, st);
  }
  if (dm.d == 64)
    return run64<64, false>(dm, q, kp, vp, kpos, qpos, idx, cnt, outs, lse, sigma, err, fault,
                            scatter, st);
  return run64<128, false>(dm, q, kp, vp, kpos, qpos, idx, cnt, outs, lse, sigma, err, fault,
                           scatter, st);
}

}  // namespace pbs

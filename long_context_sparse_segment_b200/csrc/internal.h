// Internal launcher interface of libpbs (not part of the public ABI).
#pragma once

#include <cuda_runtime.h>
#include <stddef.h>
#include <stdint.h>

#include "../../include/pbs.h"

namespace pbs {

struct Dims {
  int b, hq, hkv, n, d, B, S;
  int G;    // hq / hkv
  int nb;   // n / B
  int spb;  // S / B
  int nseg; // ceil(n / S)
};

// Argument checks shared by the entry points: the shape (PBS_OK and *dm
// filled, or the status to return), an empty problem, 16-byte alignment.
pbs_status check_shape(const pbs_shape &s, Dims *dm);
bool empty(const Dims &dm);
bool aligned16(const void *p);

// pass-1/2 importance scoring
size_t score_ws_bytes(const Dims &dm);
bool score_supported(const Dims &dm);
cudaError_t launch_score(const Dims &dm, const void *q, const void *k, float *imp,
                         float sigma, void *ws, int *err, cudaStream_t st);

// the same two passes on the tcgen05 tensor cores (G*B a multiple of 128, <= 512)
bool score_tc_supported(const Dims &dm);
size_t score_tc_ws_bytes(const Dims &dm);
cudaError_t launch_score_tc(const Dims &dm, const void *q, const void *k, float *imp,
                            float sigma, void *ws, int *err, cudaStream_t st);

// segment sort (imp -> kpos) and the gather of K, V (and Q) by kpos
cudaError_t launch_segsort(const Dims &dm, const float *imp, int32_t *kpos, int *err,
                           cudaStream_t st);
cudaError_t launch_gather(const Dims &dm, const int32_t *kpos, const void *k, const void *v,
                          const void *q, void *kp, void *vp, void *qp, double *kbar, int *err,
                          cudaStream_t st);

// fp64 sums of every run of B rows: x [heads, n, d] bf16 -> out [heads, nb, d]
cudaError_t launch_blocksum(const Dims &dm, int heads, const void *x, double *out,
                            cudaStream_t st);

// SMs of the current device (148 when the query fails)
int sm_count();

// block lists from pooled sums
// workspace: pooled query sums [+ pooled key sums] + scratch (score keys and
// softmax weights per (batch, query head, query block, key block))
size_t select_ws_bytes(const Dims &dm, bool need_kbar);
size_t select_qsum_bytes(const Dims &dm);
size_t select_scratch_bytes(const Dims &dm);
cudaError_t launch_select(const Dims &dm, const double *qsum, const double *ksum, int mode,
                          float param, double sigma, int32_t *idx, int32_t *cnt,
                          uint8_t *mask, void *scratch, int *err, cudaStream_t st);

// block-sparse forward; with `scatter` each output row is written at its
// query's original position (qpos) instead of its place in the given order;
// with `gather` kp and vp are the natural K and V and key p of the permuted
// order is read from row kpos[p] (no K', V' copies)
cudaError_t launch_attn(const Dims &dm, const void *q, const void *kp, const void *vp,
                        const int32_t *kpos, const int32_t *qpos, const int32_t *idx,
                        const int32_t *cnt, void *out, float *lse, float sigma, int *err,
                        bool scatter, bool gather, cudaStream_t st);

// the forward on the tcgen05 tensor cores (B = 128, d in {64, 128})
bool attn_tc_supported(const Dims &dm);
cudaError_t launch_attn_tc(const Dims &dm, const void *q, const void *kp, const void *vp,
                           const int32_t *kpos, const int32_t *qpos, const int32_t *idx,
                           const int32_t *cnt, void *out, float *lse, float sigma, int *err,
                           int fault, bool scatter, cudaStream_t st);

// Where the forward writes its rows: n buffers of [b, hq_total, n, d] bf16;
// query head g of the call lands at head head_offset + g of each. One
// buffer with hq_total = hq and offset 0 is the plain case.
constexpr int kMaxOuts = 8;
struct OutSet {
  void *p[kMaxOuts];
  int n, hq_total, head_offset;
};

// the same forward with two query tiles per CTA (tcgen05; B = 128, d in {64, 128})
cudaError_t launch_attn_tc2(const Dims &dm, const void *q, const void *kp, const void *vp,
                            const int32_t *kpos, const int32_t *qpos, const int32_t *idx,
                            const int32_t *cnt, const OutSet &outs, float *lse, float sigma,
                            int *err, int fault, bool scatter, bool gather, cudaStream_t st);

// the same forward for key blocks of B = 64 (tcgen05, d in {64, 128}): a
// 128-row query tile is two 64-row query blocks walking the union of their
// lists, two key blocks per step; with `gather` K and V rows are read
// through kpos as in launch_attn_tc2
bool attn_tc64_supported(const Dims &dm);
cudaError_t launch_attn_tc64(const Dims &dm, const void *q, const void *kp, const void *vp,
                             const int32_t *kpos, const int32_t *qpos, const int32_t *idx,
                             const int32_t *cnt, const OutSet &outs, float *lse, float sigma,
                             int *err, int fault, bool scatter, bool gather, cudaStream_t st);

// the forward writing every row into several buffers (the two-tile tcgen05
// kernels only; cudaErrorNotSupported where they do not run)
cudaError_t launch_attn_bcast(const Dims &dm, const void *q, const void *kp, const void *vp,
                              const int32_t *kpos, const int32_t *idx, const int32_t *cnt,
                              const OutSet &outs, float sigma, int *err, cudaStream_t st);

// the same forward on the legacy warp-MMA path
cudaError_t launch_attn_mma(const Dims &dm, const void *q, const void *kp, const void *vp,
                            const int32_t *kpos, const int32_t *qpos, const int32_t *idx,
                            const int32_t *cnt, void *out, float *lse, float sigma, int *err,
                            bool scatter, bool gather, cudaStream_t st);

// diagnostics: block attention mass (tcgen05, B = 128, G <= 4), and per row
// the coverage of a list and the fewest blocks for a target coverage
bool mass_supported(const Dims &dm);
cudaError_t launch_block_mass(const Dims &dm, const void *q, const void *kp, const int32_t *kpos,
                              float *mass, float sigma, int *err, cudaStream_t st);
cudaError_t launch_coverage(const float *mass, const int32_t *idx, const int32_t *cnt,
                            double target, int rows, int nb, float *cov, int32_t *kmin,
                            cudaStream_t st);

// out[qpos[p]] = out_perm[p]
cudaError_t launch_unpermute(const Dims &dm, const void *op, const int32_t *qpos, void *out,
                             int *err, cudaStream_t st);

}  // namespace pbs

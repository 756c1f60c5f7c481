// The C ABI of libpbs: argument checks, workspace layout, the device error
// word, and the launches of the five steps. Declared in include/pbs.h.
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

#include <mutex>
#include <vector>

#include "../../include/pbs.h"
#include "common.cuh"
#include "internal.h"

namespace pbs {

// One error word per device: kernels record the first problem they meet in
// [0] and, for a wait that ran out, the place of that wait in [1].
__device__ int g_error_word[2];

namespace {

constexpr int kMaxDevices = 64;
int *g_err_ptr[kMaxDevices];
std::once_flag g_err_once[kMaxDevices];

int *error_word() {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return nullptr;
  std::call_once(g_err_once[dev], [dev] {
    void *p = nullptr;
    if (cudaGetSymbolAddress(&p, g_error_word) == cudaSuccess) g_err_ptr[dev] = (int *)p;
  });
  return g_err_ptr[dev];
}

}  // namespace

bool aligned16(const void *p) { return ((uintptr_t)p & 15u) == 0; }

pbs_status check_shape(const pbs_shape &s, Dims *dm) {
  if (s.batch < 0 || s.hq < 1 || s.hkv < 1 || s.n < 0 || s.block < 1 || s.segment < 1)
    return PBS_ERR_INVALID_ARG;
  if (s.hq % s.hkv != 0) return PBS_ERR_INVALID_ARG;
  if (s.d != 64 && s.d != 128) return PBS_ERR_UNSUPPORTED;
  if (s.block != 64 && s.block != 128) return PBS_ERR_UNSUPPORTED;
  if (s.segment % s.block != 0 || s.n % s.block != 0) return PBS_ERR_INVALID_ARG;
  if (s.segment > 8192) return PBS_ERR_UNSUPPORTED;
  dm->b = s.batch;
  dm->hq = s.hq;
  dm->hkv = s.hkv;
  dm->n = s.n;
  dm->d = s.d;
  dm->B = s.block;
  dm->S = s.segment;
  dm->G = s.hq / s.hkv;
  dm->nb = s.n / s.block;
  dm->spb = s.segment / s.block;
  dm->nseg = (s.n + s.segment - 1) / s.segment;
  return PBS_OK;
}

bool empty(const Dims &dm) { return dm.b == 0 || dm.n == 0; }

namespace {

pbs_status cuda_status(cudaError_t e) { return e == cudaSuccess ? PBS_OK : PBS_ERR_CUDA; }

double resolve_sigma(float scale, int d) {
  return scale > 0.f ? (double)scale : 1.0 / sqrt((double)d);
}

// ------------------------------------------- the host-buffer path's slots
// pbs_attention_host works one KV group (batch b, KV head h: its G query
// heads) at a time, in device slots used in turn by consecutive groups:
// with three, group i + 1 can be copied in while group i computes and group
// i - 1 is still being copied out.
constexpr size_t kSlotAlign = 256;
constexpr int kSlots = 3;
size_t aup(size_t x) { return (x + kSlotAlign - 1) & ~(kSlotAlign - 1); }

Dims group_dims(const Dims &dm) {
  Dims g = dm;
  g.b = 1;
  g.hq = dm.G;
  g.hkv = 1;
  return g;
}

// The host path's unit of selection, forward and copies: `hs` query heads
// of one KV group, the fewest (a divisor of G) whose forward still fills
// three waves of two-tile CTAs, so that splitting a group costs no
// occupancy.
// PBS_HOST_STEP_HEADS=<k> (a divisor of G) sets the step instead (a
// diagnostic switch: the tests check that every step size gives the same
// result).
int heads_per_step(const Dims &g) {
  if (const char *env = getenv("PBS_HOST_STEP_HEADS")) {
    const int k = atoi(env);
    if (k >= 1 && k <= g.G && g.G % k == 0) return k;
  }
  const long long want = 3LL * sm_count();
  for (int hs = 1; hs < g.G; ++hs)
    if (g.G % hs == 0 && (long long)hs * ((g.nb + 1) / 2) >= want) return hs;
  return g.G;
}

Dims step_dims(const Dims &g, int hs) {
  Dims h = g;
  h.hq = hs;
  h.G = hs;
  return h;
}

struct Slot {
  void *q, *k, *v, *kp, *vp, *o, *score_ws;
  float *imp;
  int32_t *kpos, *idx, *cnt;
  double *kbar, *qsum;
};

// Lays a slot out from `base` (256-byte aligned); returns its size.
size_t carve_slot(uint8_t *base, const Dims &g, Slot *sl) {
  const size_t qb = (size_t)g.hq * g.n * g.d * 2, kb = (size_t)g.n * g.d * 2;
  size_t off = 0;
  auto take = [&](size_t bytes) {
    uint8_t *p = base ? base + off : nullptr;
    off += aup(bytes);
    return p;
  };
  Slot t;
  t.q = take(qb);
  t.o = take(qb);
  t.k = take(kb);
  t.v = take(kb);
  t.kp = take(kb);
  t.vp = take(kb);
  t.imp = (float *)take((size_t)g.n * 4);
  t.kpos = (int32_t *)take((size_t)g.n * 4);
  t.kbar = (double *)take((size_t)g.nb * g.d * 8);
  t.idx = (int32_t *)take((size_t)g.hq * g.nb * g.nb * 4);
  t.cnt = (int32_t *)take((size_t)g.hq * g.nb * 4);
  t.score_ws = take(score_ws_bytes(g));
  // the steps of a group are selected one after the other on one stream,
  // so one step's selection workspace serves them all
  t.qsum = (double *)take(select_ws_bytes(step_dims(g, heads_per_step(g)), false));
  if (sl) *sl = t;
  return off;
}

size_t host_path_ws_bytes(const Dims &dm) {
  return kSlots * carve_slot(nullptr, group_dims(dm), nullptr) + kSlotAlign;
}

}  // namespace
}  // namespace pbs

using namespace pbs;

extern "C" {

size_t pbs_workspace_bytes(pbs_shape s, int op) {
  Dims dm;
  if (check_shape(s, &dm) != PBS_OK || empty(dm)) return 0;
  switch (op) {
    case PBS_OP_SCORE:
      return score_ws_bytes(dm);
    case PBS_OP_SELECT:
      return select_ws_bytes(dm, true);
    case PBS_OP_HOST_PATH:
      return host_path_ws_bytes(dm);
    default:
      return 0;
  }
}

pbs_status pbs_score(const void *q, const void *k, float *imp, pbs_shape s, float scale,
                     void *ws, size_t ws_bytes, pbs_stream_t st) {
  Dims dm;
  pbs_status r = check_shape(s, &dm);
  if (r != PBS_OK) return r;
  if (empty(dm)) return PBS_OK;
  if (!q || !k || !imp || !ws || !aligned16(q) || !aligned16(k) || !aligned16(ws) ||
      ((uintptr_t)imp & 3u))
    return PBS_ERR_INVALID_ARG;
  if (!score_supported(dm)) return PBS_ERR_UNSUPPORTED;
  if (ws_bytes < score_ws_bytes(dm)) return PBS_ERR_WORKSPACE;
  int *err = error_word();
  const float sigma = (float)resolve_sigma(scale, dm.d);
  return cuda_status(launch_score(dm, q, k, imp, sigma, ws, err, (cudaStream_t)st));
}

pbs_status pbs_permute(const float *imp, const void *k, const void *v, const void *q,
                       void *k_perm, void *v_perm, void *q_perm, int32_t *kpos,
                       double *kbar_sum, pbs_shape s, pbs_stream_t st) {
  Dims dm;
  pbs_status r = check_shape(s, &dm);
  if (r != PBS_OK) return r;
  if (empty(dm)) return PBS_OK;
  if (!imp || !k || !v || !kpos) return PBS_ERR_INVALID_ARG;
  // K' and V' are both written or (order only: the forward gathers) neither
  if ((k_perm == nullptr) != (v_perm == nullptr)) return PBS_ERR_INVALID_ARG;
  if ((q == nullptr) != (q_perm == nullptr)) return PBS_ERR_INVALID_ARG;
  if (!aligned16(k) || !aligned16(v) || (k_perm && !aligned16(k_perm)) ||
      (v_perm && !aligned16(v_perm)) || !aligned16(kpos) ||
      (q && (!aligned16(q) || !aligned16(q_perm))) || (kbar_sum && !aligned16(kbar_sum)) ||
      ((uintptr_t)imp & 3u))
    return PBS_ERR_INVALID_ARG;
  if (k == k_perm || v == v_perm || (q && q == q_perm)) return PBS_ERR_INVALID_ARG;
  int *err = error_word();
  cudaStream_t cs = (cudaStream_t)st;
  cudaError_t e = launch_segsort(dm, imp, kpos, err, cs);
  if (e != cudaSuccess) return PBS_ERR_CUDA;
  return cuda_status(launch_gather(dm, kpos, k, v, q, k_perm, v_perm, q_perm, kbar_sum, err, cs));
}

pbs_status pbs_select_blocks(const void *q_or_qperm, const void *k_perm, const double *kbar_sum,
                             pbs_shape s, int mode, float param, float scale, int32_t *blk_idx,
                             int32_t *blk_cnt, uint8_t *blk_mask, void *ws, size_t ws_bytes,
                             pbs_stream_t st) {
  Dims dm;
  pbs_status r = check_shape(s, &dm);
  if (r != PBS_OK) return r;
  if (mode < PBS_SEL_THRESHOLD || mode > PBS_SEL_DENSE_CAUSAL) return PBS_ERR_INVALID_ARG;
  if ((mode == PBS_SEL_THRESHOLD || mode == PBS_SEL_TOPK_FRAC) &&
      !(param > 0.f && param <= 1.f))
    return PBS_ERR_INVALID_ARG;
  if (empty(dm)) return PBS_OK;
  if (!blk_idx || !blk_cnt || ((uintptr_t)blk_idx & 3u) || ((uintptr_t)blk_cnt & 3u))
    return PBS_ERR_INVALID_ARG;
  const bool scored = mode == PBS_SEL_THRESHOLD || mode == PBS_SEL_TOPK_FRAC;
  if (scored) {
    if (!q_or_qperm || !aligned16(q_or_qperm)) return PBS_ERR_INVALID_ARG;
    if (!kbar_sum && (!k_perm || !aligned16(k_perm))) return PBS_ERR_INVALID_ARG;
    if (kbar_sum && !aligned16(kbar_sum)) return PBS_ERR_INVALID_ARG;
    if (!ws || !aligned16(ws)) return PBS_ERR_INVALID_ARG;
    if (ws_bytes < select_ws_bytes(dm, kbar_sum == nullptr)) return PBS_ERR_WORKSPACE;
  }
  int *err = error_word();
  cudaStream_t cs = (cudaStream_t)st;
  // workspace (scored modes only): qsum | [ksum when not given] | scratch
  double *qsum = (double *)ws;
  const double *ksum = kbar_sum;
  uint8_t *scratch = scored ? (uint8_t *)ws + select_qsum_bytes(dm) : nullptr;
  if (scored) {
    cudaError_t e = launch_blocksum(dm, dm.b * dm.hq, q_or_qperm, qsum, cs);
    if (e != cudaSuccess) return PBS_ERR_CUDA;
    if (!kbar_sum) {
      double *kbuf = (double *)scratch;
      e = launch_blocksum(dm, dm.b * dm.hkv, k_perm, kbuf, cs);
      if (e != cudaSuccess) return PBS_ERR_CUDA;
      ksum = kbuf;
      scratch += (size_t)dm.b * dm.hkv * dm.nb * dm.d * 8;
    }
  }
  return cuda_status(launch_select(dm, qsum, ksum, mode, param, resolve_sigma(scale, dm.d),
                                   blk_idx, blk_cnt, blk_mask, scratch, err, cs));
}

namespace {

pbs_status attn_fwd(const void *q_or_qperm, const void *k_perm, const void *v_perm,
                    const int32_t *kpos, const int32_t *qpos, const int32_t *blk_idx,
                    const int32_t *blk_cnt, void *out, float *lse, pbs_shape s, float scale,
                    bool scatter, bool gather, pbs_stream_t st) {
  Dims dm;
  pbs_status r = check_shape(s, &dm);
  if (r != PBS_OK) return r;
  if (empty(dm)) return PBS_OK;
  if (!q_or_qperm || !k_perm || !v_perm || !blk_idx || !blk_cnt || !out || (gather && !kpos))
    return PBS_ERR_INVALID_ARG;
  if (!aligned16(q_or_qperm) || !aligned16(k_perm) || !aligned16(v_perm) || !aligned16(out) ||
      (kpos && !aligned16(kpos)) || (qpos && ((uintptr_t)qpos & 3u)) ||
      ((uintptr_t)blk_idx & 3u) || ((uintptr_t)blk_cnt & 3u) || (lse && ((uintptr_t)lse & 3u)))
    return PBS_ERR_INVALID_ARG;
  // rows land out of order: the output must not be an input still being read
  if (scatter && (out == q_or_qperm || out == k_perm || out == v_perm)) return PBS_ERR_INVALID_ARG;
  int *err = error_word();
  const float sigma = (float)resolve_sigma(scale, dm.d);
  return cuda_status(launch_attn(dm, q_or_qperm, k_perm, v_perm, kpos, qpos, blk_idx, blk_cnt,
                                 out, lse, sigma, err, scatter && qpos, gather, (cudaStream_t)st));
}

}  // namespace

pbs_status pbs_attn_fwd(const void *q_or_qperm, const void *k_perm, const void *v_perm,
                        const int32_t *kpos, const int32_t *qpos, const int32_t *blk_idx,
                        const int32_t *blk_cnt, void *out, float *lse, pbs_shape s, float scale,
                        pbs_stream_t st) {
  return attn_fwd(q_or_qperm, k_perm, v_perm, kpos, qpos, blk_idx, blk_cnt, out, lse, s, scale,
                  false, false, st);
}

pbs_status pbs_attn_fwd_unpermute(const void *q_perm, const void *k_perm, const void *v_perm,
                                  const int32_t *kpos, const int32_t *qpos,
                                  const int32_t *blk_idx, const int32_t *blk_cnt, void *out,
                                  float *lse, pbs_shape s, float scale, pbs_stream_t st) {
  return attn_fwd(q_perm, k_perm, v_perm, kpos, qpos, blk_idx, blk_cnt, out, lse, s, scale, true,
                  false, st);
}

pbs_status pbs_attn_fwd_gather(const void *q_or_qperm, const void *k, const void *v,
                               const int32_t *kpos, const int32_t *qpos, const int32_t *blk_idx,
                               const int32_t *blk_cnt, void *out, float *lse, pbs_shape s,
                               float scale, int unpermute, pbs_stream_t st) {
  return attn_fwd(q_or_qperm, k, v, kpos, qpos, blk_idx, blk_cnt, out, lse, s, scale,
                  unpermute != 0, true, st);
}

pbs_status pbs_attn_fwd_bcast(const void *q, const void *k_perm, const void *v_perm,
                              const int32_t *kpos, const int32_t *blk_idx,
                              const int32_t *blk_cnt, void *const *outs, int n_out,
                              int hq_total, int head_offset, pbs_shape s, float scale,
                              pbs_stream_t st) {
  Dims dm;
  pbs_status r = check_shape(s, &dm);
  if (r != PBS_OK) return r;
  if (!outs || n_out < 1 || n_out > kMaxOuts || head_offset < 0 ||
      (long long)head_offset + dm.hq > hq_total)
    return PBS_ERR_INVALID_ARG;
  if (empty(dm)) return PBS_OK;
  if (!q || !k_perm || !v_perm || !blk_idx || !blk_cnt || !aligned16(q) || !aligned16(k_perm) ||
      !aligned16(v_perm) || (kpos && !aligned16(kpos)) || ((uintptr_t)blk_idx & 3u) ||
      ((uintptr_t)blk_cnt & 3u))
    return PBS_ERR_INVALID_ARG;
  OutSet set{};
  for (int i = 0; i < n_out; ++i) {
    if (!outs[i] || !aligned16(outs[i]) || outs[i] == q || outs[i] == k_perm ||
        outs[i] == v_perm)
      return PBS_ERR_INVALID_ARG;
    set.p[i] = outs[i];
  }
  set.n = n_out, set.hq_total = hq_total, set.head_offset = head_offset;
  if (!attn_tc_supported(dm) && !attn_tc64_supported(dm)) return PBS_ERR_UNSUPPORTED;
  const float sigma = (float)resolve_sigma(scale, dm.d);
  const cudaError_t e = launch_attn_bcast(dm, q, k_perm, v_perm, kpos, blk_idx, blk_cnt, set,
                                          sigma, error_word(), (cudaStream_t)st);
  return e == cudaErrorNotSupported ? PBS_ERR_UNSUPPORTED : cuda_status(e);
}

pbs_status pbs_unpermute(const void *out_perm, const int32_t *qpos, void *out, pbs_shape s,
                         pbs_stream_t st) {
  Dims dm;
  pbs_status r = check_shape(s, &dm);
  if (r != PBS_OK) return r;
  if (empty(dm)) return PBS_OK;
  if (!out_perm || !out || !aligned16(out_perm) || !aligned16(out) ||
      (qpos && ((uintptr_t)qpos & 3u)))
    return PBS_ERR_INVALID_ARG;
  cudaStream_t cs = (cudaStream_t)st;
  if (!qpos) {
    if (out == out_perm) return PBS_OK;
    const size_t bytes = (size_t)dm.b * dm.hq * dm.n * dm.d * 2;
    return cuda_status(cudaMemcpyAsync(out, out_perm, bytes, cudaMemcpyDeviceToDevice, cs));
  }
  if (out == out_perm) return PBS_ERR_INVALID_ARG;
  return cuda_status(launch_unpermute(dm, out_perm, qpos, out, error_word(), cs));
}

pbs_status pbs_attention_host(const void *q, const void *k, const void *v, void *out,
                              pbs_shape s, int mode, float param, float scale, void *ws,
                              size_t ws_bytes, pbs_stream_t compute, pbs_stream_t h2d,
                              pbs_stream_t d2h) {
  Dims dm;
  pbs_status r = check_shape(s, &dm);
  if (r != PBS_OK) return r;
  if (mode < PBS_SEL_THRESHOLD || mode > PBS_SEL_DENSE_CAUSAL) return PBS_ERR_INVALID_ARG;
  const bool scored = mode == PBS_SEL_THRESHOLD || mode == PBS_SEL_TOPK_FRAC;
  if (scored && !(param > 0.f && param <= 1.f)) return PBS_ERR_INVALID_ARG;
  if (empty(dm)) return PBS_OK;
  if (!q || !k || !v || !out || !ws) return PBS_ERR_INVALID_ARG;
  const Dims g = group_dims(dm);
  if (!score_supported(g)) return PBS_ERR_UNSUPPORTED;
  if (ws_bytes < host_path_ws_bytes(dm)) return PBS_ERR_WORKSPACE;
  uint8_t *base = (uint8_t *)(((uintptr_t)ws + kSlotAlign - 1) & ~(uintptr_t)(kSlotAlign - 1));
  Slot slot[kSlots];
  const size_t slot_bytes = carve_slot(base, g, &slot[0]);
  for (int i = 1; i < kSlots; ++i) carve_slot(base + i * slot_bytes, g, &slot[i]);

  cudaStream_t cs = (cudaStream_t)compute, hst = (cudaStream_t)h2d, ds = (cudaStream_t)d2h;
  // per slot: [0] K, V and the last query block of every head copied in,
  // [1 + st] the query heads of step st copied in, [1 + steps + st] step st
  // computed, [1 + 2 steps] the slot's last output copied out
  const int G = dm.G, hs = heads_per_step(g), steps = G / hs, per_slot = 2 + 2 * steps;
  std::vector<cudaEvent_t> evs(kSlots * (size_t)per_slot, nullptr);
  cudaError_t e = cudaSuccess;
  for (auto &x : evs)
    if (e == cudaSuccess) e = cudaEventCreateWithFlags(&x, cudaEventDisableTiming);
  if (e != cudaSuccess) {
    for (auto &x : evs)
      if (x) cudaEventDestroy(x);
    return PBS_ERR_CUDA;
  }
  auto ev = [&](int sid, int k) { return evs[(size_t)sid * per_slot + k]; };
  const Dims h1 = step_dims(g, hs);
  int *err = error_word();
  const float sigma_f = (float)resolve_sigma(scale, dm.d);
  const double sigma_d = resolve_sigma(scale, dm.d);
  const size_t hb = (size_t)g.n * g.d * 2;  // one head's rows (Q, O, K or V)
  const size_t lastb = (size_t)g.B * g.d * 2, restb = hb - lastb;
  const size_t nb = (size_t)g.nb;
  const int groups = dm.b * dm.hkv;
  auto at = [](const void *p, size_t off) { return (const uint8_t *)p + off; };
  for (int i = 0; i < groups && e == cudaSuccess; ++i) {
    const int sid = i % kSlots, bi = i / dm.hkv, h = i % dm.hkv;
    const Slot &sl = slot[sid];
    const size_t qoff = ((size_t)bi * dm.hq + (size_t)h * G) * hb;  // head h*G of batch bi
    const size_t koff = ((size_t)bi * dm.hkv + h) * hb;
    uint8_t *sq = (uint8_t *)sl.q, *so = (uint8_t *)sl.o;
    // in: the slot is free once group i - 2 has been copied out. First what
    // the scoring and the permutation need (K, V, the last query block of
    // each head), then the query heads one by one
    if (i >= kSlots) e = cudaStreamWaitEvent(hst, ev(sid, 1 + 2 * steps), 0);
    for (int gl = 0; gl < G && e == cudaSuccess; ++gl)
      e = cudaMemcpyAsync(sq + gl * hb + restb, at(q, qoff + gl * hb + restb), lastb,
                          cudaMemcpyHostToDevice, hst);
    if (e == cudaSuccess) e = cudaMemcpyAsync(sl.k, at(k, koff), hb, cudaMemcpyHostToDevice, hst);
    if (e == cudaSuccess) e = cudaMemcpyAsync(sl.v, at(v, koff), hb, cudaMemcpyHostToDevice, hst);
    if (e == cudaSuccess) e = cudaEventRecord(ev(sid, 0), hst);
    for (int st = 0; st < steps && e == cudaSuccess; ++st) {
      for (int gl = st * hs; gl < (st + 1) * hs && e == cudaSuccess && restb; ++gl)
        e = cudaMemcpyAsync(sq + gl * hb, at(q, qoff + gl * hb), restb, cudaMemcpyHostToDevice,
                            hst);
      if (e == cudaSuccess) e = cudaEventRecord(ev(sid, 1 + st), hst);
    }
    // the group's scoring and permutation
    if (e == cudaSuccess) e = cudaStreamWaitEvent(cs, ev(sid, 0), 0);
    if (e == cudaSuccess) e = launch_score(g, sl.q, sl.k, sl.imp, sigma_f, sl.score_ws, err, cs);
    if (e == cudaSuccess) e = launch_segsort(g, sl.imp, sl.kpos, err, cs);
    if (e == cudaSuccess)
      e = launch_gather(g, sl.kpos, sl.k, sl.v, nullptr, sl.kp, sl.vp, nullptr, sl.kbar, err, cs);
    // then per step of hs query heads, as they arrive: selection, forward,
    // copy out
    for (int st = 0; st < steps && e == cudaSuccess; ++st) {
      const int gl = st * hs;
      const uint8_t *qh = sq + gl * hb;
      int32_t *idx = sl.idx + (size_t)gl * nb * nb, *cnt = sl.cnt + (size_t)gl * nb;
      e = cudaStreamWaitEvent(cs, ev(sid, 1 + st), 0);
      if (e == cudaSuccess && scored) e = launch_blocksum(h1, hs, qh, sl.qsum, cs);
      if (e == cudaSuccess)
        e = launch_select(h1, sl.qsum, sl.kbar, mode, param, sigma_d, idx, cnt, nullptr,
                          (uint8_t *)sl.qsum + select_qsum_bytes(h1), err, cs);
      if (e == cudaSuccess)
        e = launch_attn(h1, qh, sl.kp, sl.vp, sl.kpos, nullptr, idx, cnt, so + gl * hb, nullptr,
                        sigma_f, err, false, false, cs);
      if (e == cudaSuccess) e = cudaEventRecord(ev(sid, 1 + steps + st), cs);
      if (e == cudaSuccess) e = cudaStreamWaitEvent(ds, ev(sid, 1 + steps + st), 0);
      if (e == cudaSuccess)
        e = cudaMemcpyAsync((uint8_t *)out + qoff + gl * hb, so + gl * hb, hs * hb,
                            cudaMemcpyDeviceToHost, ds);
    }
    if (e == cudaSuccess) e = cudaEventRecord(ev(sid, 1 + 2 * steps), ds);
  }
  // work queued on the copy streams is ordered before later work on `compute`
  for (int sid = 0; sid < kSlots && sid < groups && e == cudaSuccess; ++sid)
    e = cudaStreamWaitEvent(cs, ev(sid, 1 + 2 * steps), 0);
  for (auto &x : evs) cudaEventDestroy(x);  // released once their work completes
  return cuda_status(e);
}

pbs_status pbs_block_mass(const void *q, const void *k_perm, const int32_t *kpos, float *mass,
                          pbs_shape s, float scale, pbs_stream_t st) {
  Dims dm;
  pbs_status r = check_shape(s, &dm);
  if (r != PBS_OK) return r;
  if (empty(dm)) return PBS_OK;
  if (!q || !k_perm || !mass || !aligned16(q) || !aligned16(k_perm) || (kpos && !aligned16(kpos)) ||
      ((uintptr_t)mass & 3u))
    return PBS_ERR_INVALID_ARG;
  if (!mass_supported(dm)) return PBS_ERR_UNSUPPORTED;
  const float sigma = (float)resolve_sigma(scale, dm.d);
  return cuda_status(
      launch_block_mass(dm, q, k_perm, kpos, mass, sigma, error_word(), (cudaStream_t)st));
}

pbs_status pbs_coverage(const float *mass, const int32_t *blk_idx, const int32_t *blk_cnt,
                        double target, float *coverage, int32_t *blocks_needed, pbs_shape s,
                        pbs_stream_t st) {
  Dims dm;
  pbs_status r = check_shape(s, &dm);
  if (r != PBS_OK) return r;
  if (empty(dm)) return PBS_OK;
  if (!mass || ((uintptr_t)mass & 3u)) return PBS_ERR_INVALID_ARG;
  if (coverage && (!blk_idx || !blk_cnt)) return PBS_ERR_INVALID_ARG;
  if (blocks_needed && !(target > 0.0 && target <= 1.0)) return PBS_ERR_INVALID_ARG;
  const int rows = dm.b * dm.hq * dm.nb;
  return cuda_status(launch_coverage(mass, coverage ? blk_idx : nullptr, blk_cnt, target, rows,
                                     dm.nb, coverage, blocks_needed, (cudaStream_t)st));
}

pbs_status pbs_get_device_status(pbs_stream_t st, int *code, int *detail) {
  if (!code) return PBS_ERR_INVALID_ARG;
  if (cudaStreamSynchronize((cudaStream_t)st) != cudaSuccess) return PBS_ERR_CUDA;
  int *err = error_word();
  if (!err) return PBS_ERR_CUDA;
  int v[2] = {0, 0};
  if (cudaMemcpy(v, err, sizeof(v), cudaMemcpyDeviceToHost) != cudaSuccess) return PBS_ERR_CUDA;
  const int zero[2] = {0, 0};
  if (cudaMemcpy(err, zero, sizeof(zero), cudaMemcpyHostToDevice) != cudaSuccess)
    return PBS_ERR_CUDA;
  *code = v[0];
  if (detail) *detail = v[1];
  return PBS_OK;
}

const char *pbs_status_string(int status) {
  switch (status) {
    case PBS_OK: return "PBS_OK";
    case PBS_ERR_INVALID_ARG: return "PBS_ERR_INVALID_ARG";
    case PBS_ERR_UNSUPPORTED: return "PBS_ERR_UNSUPPORTED";
    case PBS_ERR_CUDA: return "PBS_ERR_CUDA";
    case PBS_ERR_TIMEOUT: return "PBS_ERR_TIMEOUT";
    case PBS_ERR_DEVICE_ASSERT: return "PBS_ERR_DEVICE_ASSERT";
    case PBS_ERR_WORKSPACE: return "PBS_ERR_WORKSPACE";
    default: return "PBS_ERR_UNKNOWN";
  }
}

const char *pbs_version(void) { return "pbs-b200 0.1 (sm_100a)"; }

}  // extern "C"

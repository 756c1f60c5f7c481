// pbs_score_static: pbs_score without a caller-supplied workspace.
//
// Some callers cannot allocate device memory when they call the library: a
// plugin inside an inference engine that owns every device allocation and
// forbids its plugins to call cudaMalloc, or a latency-critical loop that
// cannot afford cudaMalloc's implicit device synchronisation. For them the
// scoring scratch (per-row partial softmax statistics) lives in a fixed
// array in this library's device memory instead of in a workspace buffer.
//
// The array has PBS_SCORE_STATIC_SCRATCH_BYTES bytes and exists on every GPU
// that loads the library until the process exits. The arguments are checked
// first, as pbs_score checks them (an empty shape returns PBS_OK, a bad one
// its error, without touching CUDA); shapes whose scoring scratch is larger
// than the array are rejected with PBS_ERR_WORKSPACE. The device address of
// the array is looked up on the first call made with a device current, and
// looked up again on the next call if that lookup failed (for example inside
// a stream capture); make the first call before any stream capture. Every
// call shares the one array: two calls that overlap on the GPU (other
// streams, other threads) race on it. Nothing needs clearing between calls,
// because every byte the scoring kernels read is written earlier in the same
// call.
#include <mutex>

#include "../../include/pbs.h"
#include "internal.h"

namespace pbs {
namespace {

__device__ __align__(256) unsigned char g_score_scratch[PBS_SCORE_STATIC_SCRATCH_BYTES];

constexpr int kMaxDevices = 64;
void *g_scratch[kMaxDevices];
std::mutex g_scratch_mu;

// Device address of the scratch array on the current device. The symbol's
// name is only a host-side handle; kernels must be given this address. Only
// a successful lookup is kept.
pbs_status scratch_address(void **out) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return PBS_ERR_CUDA;
  std::lock_guard<std::mutex> lock(g_scratch_mu);
  if (g_scratch[dev] == nullptr) {
    void *p = nullptr;
    if (cudaGetSymbolAddress(&p, g_score_scratch) != cudaSuccess || p == nullptr) {
      cudaGetLastError();  // leave no error behind for the caller's next call
      return PBS_ERR_CUDA;
    }
    g_scratch[dev] = p;
  }
  *out = g_scratch[dev];
  return PBS_OK;
}

}  // namespace
}  // namespace pbs

extern "C" pbs_status pbs_score_static(const void *q, const void *k, float *imp, pbs_shape s,
                                       float scale, pbs_stream_t st) {
  pbs::Dims dm;
  const pbs_status shape_ok = pbs::check_shape(s, &dm);
  if (shape_ok != PBS_OK) return shape_ok;
  if (pbs::empty(dm)) return PBS_OK;
  if (!q || !k || !imp || !pbs::aligned16(q) || !pbs::aligned16(k) || ((uintptr_t)imp & 3u))
    return PBS_ERR_INVALID_ARG;
  if (pbs_workspace_bytes(s, PBS_OP_SCORE) > (size_t)PBS_SCORE_STATIC_SCRATCH_BYTES)
    return PBS_ERR_WORKSPACE;
  void *scratch = nullptr;
  pbs_status r = pbs::scratch_address(&scratch);
  if (r != PBS_OK) return r;
  return pbs_score(q, k, imp, s, scale, scratch, (size_t)PBS_SCORE_STATIC_SCRATCH_BYTES, st);
}

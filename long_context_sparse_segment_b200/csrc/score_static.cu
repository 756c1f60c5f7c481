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
// that loads the library until the process exits. Shapes whose scoring
// scratch is larger are rejected with PBS_ERR_WORKSPACE. The device address
// of the array is looked up once per device, on the first call made with
// that device current; make that first call before any stream capture.
// Every call shares the one array: two calls that overlap on the GPU (other
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
cudaError_t g_scratch_err[kMaxDevices];
std::once_flag g_scratch_once[kMaxDevices];

// Device address of the scratch array on the current device. The symbol's
// name is only a host-side handle; kernels must be given this address.
pbs_status scratch_address(void **out) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return PBS_ERR_CUDA;
  std::call_once(g_scratch_once[dev], [dev] {
    void *p = nullptr;
    g_scratch_err[dev] = cudaGetSymbolAddress(&p, g_score_scratch);
    g_scratch[dev] = p;
  });
  if (g_scratch_err[dev] != cudaSuccess || g_scratch[dev] == nullptr) return PBS_ERR_CUDA;
  *out = g_scratch[dev];
  return PBS_OK;
}

}  // namespace
}  // namespace pbs

extern "C" pbs_status pbs_score_static(const void *q, const void *k, float *imp, pbs_shape s,
                                       float scale, pbs_stream_t st) {
  if (pbs_workspace_bytes(s, PBS_OP_SCORE) > (size_t)PBS_SCORE_STATIC_SCRATCH_BYTES)
    return PBS_ERR_WORKSPACE;
  void *scratch = nullptr;
  pbs_status r = pbs::scratch_address(&scratch);
  if (r != PBS_OK) return r;
  return pbs_score(q, k, imp, s, scale, scratch, (size_t)PBS_SCORE_STATIC_SCRATCH_BYTES, st);
}

// rqlut_static_scratch.cu -- rq_lut_logits_static: the logits call for
// callers that cannot allocate device memory themselves.
//
// rq_lut_logits needs a device workspace (per-chunk partial sums, argmax
// keys).  Some callers have no way to provide one: hosts whose device memory
// is owned by another runtime's pool, which this library cannot draw from,
// or embedded and real-time serving loops that must never allocate once
// they have started.  This entry point takes the workspace from a fixed
// array in the library's own device memory instead.
#include <mutex>

#include "rq_common.cuh"

// The scratch: RQ_STATIC_SCRATCH_BYTES on every GPU that loads the library,
// held until the process exits.  Every call on a device shares it.
static __device__ __align__(256) unsigned char g_rq_static_scratch[RQ_STATIC_SCRATCH_BYTES];

namespace {

std::mutex g_scratch_mu;
void *g_scratch_ptr[128] = {};

// Device address of the scratch on the current device, looked up once per
// device (cudaGetSymbolAddress, with that device current) and cached.
int static_scratch(void **out) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return RQ_ERR_CUDA;
  if (dev < 0 || dev >= 128) return RQ_ERR_UNSUPPORTED;
  std::lock_guard<std::mutex> lock(g_scratch_mu);
  if (g_scratch_ptr[dev] == nullptr) {
    void *p = nullptr;
    if (cudaGetSymbolAddress(&p, g_rq_static_scratch) != cudaSuccess || p == nullptr)
      return RQ_ERR_CUDA;
    g_scratch_ptr[dev] = p;
  }
  *out = g_scratch_ptr[dev];
  return RQ_OK;
}

}  // namespace

extern "C" int rq_lut_logits_static(const void *codes, int fmt, rq_dims d, const float *lut,
                                    int B, float softcap, float *logits, int32_t *argmax,
                                    void *stream) {
  // Refuse early, launching nothing, what cannot fit on a B200; the call
  // below checks the scratch size again against the plan of the device it
  // runs on, which may differ.
  const size_t need = rq_logits_workspace_bytes(d, B, fmt, argmax != nullptr ? 1 : 0);
  if (need > (size_t)RQ_STATIC_SCRATCH_BYTES) return RQ_ERR_WORKSPACE_TOO_SMALL;
  void *ws = nullptr;
  const int st = static_scratch(&ws);
  if (st != RQ_OK) return st;
  // Nothing in the scratch has to start at zero: the partial sums are
  // written before they are read, and the code pass zeroes the argmax keys
  // at the start of every call, before the reduce folds values into them.
  return rq_lut_logits(codes, fmt, d, lut, B, softcap, logits, argmax, ws,
                       (size_t)RQ_STATIC_SCRATCH_BYTES, stream);
}

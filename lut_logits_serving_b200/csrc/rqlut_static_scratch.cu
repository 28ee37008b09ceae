// rqlut_static_scratch.cu -- rq_lut_logits_static: the logits call for
// callers that cannot allocate device memory themselves.
//
// rq_lut_logits needs a device workspace (per-chunk partial sums, argmax
// partials, a reduction counter).  Some callers have no way to provide one:
// code recorded into a CUDA graph while capture is active (no allocation
// allowed then), hosts whose device memory is owned by another runtime's
// pool, or embedded/real-time loops that must never allocate after start-up.
// This entry point takes the workspace from a fixed array in the library's
// own device memory instead.
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
  // The same workspace rq_lut_logits would ask for; refuse what does not fit.
  const size_t need = rq_logits_workspace_bytes(d, B, fmt, argmax != nullptr ? 1 : 0);
  if (need > (size_t)RQ_STATIC_SCRATCH_BYTES) return RQ_ERR_WORKSPACE_TOO_SMALL;
  void *ws = nullptr;
  if (need > 0) {
    const int st = static_scratch(&ws);
    if (st != RQ_OK) return st;
  }
  // Nothing in the scratch has to start at zero: the partial sums and argmax
  // partials are written before they are read, and the reduction counter is
  // reset by the code-pass kernel at the start of every call.
  return rq_lut_logits(codes, fmt, d, lut, B, softcap, logits, argmax, ws,
                       need > 0 ? (size_t)RQ_STATIC_SCRATCH_BYTES : 0, stream);
}

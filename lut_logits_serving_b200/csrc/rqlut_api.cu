// rqlut_api.cu -- the C ABI of librqlut (see include/rqlut.h): argument
// validation, workspace layout, path selection and launches.
#include <map>
#include <mutex>
#include <tuple>
#include <utility>

#include "rq_common.cuh"

// The device error word (RQ_DEVERR_* bits), one per device that loads the
// library.  Kernels receive its device address; rq_device_error reads it.
__device__ unsigned int g_rq_device_error = 0u;

namespace rq {

cudaError_t dev_info(DevInfo *out) {
  static std::mutex mu;
  static DevInfo cache[128];
  static bool valid[128] = {};
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  if (dev >= 0 && dev < 128) {
    std::lock_guard<std::mutex> g(mu);
    if (valid[dev]) {
      *out = cache[dev];
      return cudaSuccess;
    }
  }
  DevInfo d{};
  d.device = dev;
  if ((e = cudaDeviceGetAttribute(&d.sms, cudaDevAttrMultiProcessorCount, dev)) != cudaSuccess)
    return e;
  if ((e = cudaDeviceGetAttribute(&d.max_smem_optin, cudaDevAttrMaxSharedMemoryPerBlockOptin,
                                  dev)) != cudaSuccess)
    return e;
  void *p = nullptr;
  if ((e = cudaGetSymbolAddress(&p, g_rq_device_error)) != cudaSuccess) return e;
  d.err = static_cast<unsigned *>(p);
  if (dev >= 0 && dev < 128) {
    std::lock_guard<std::mutex> g(mu);
    cache[dev] = d;
    valid[dev] = true;
  }
  *out = d;
  return cudaSuccess;
}

namespace {
std::mutex g_attr_mu;
std::map<std::pair<const void *, int>, size_t> g_smem_limit;
std::map<std::tuple<const void *, int, int, size_t>, int> g_occupancy;
}  // namespace

cudaError_t ensure_smem_limit(const void *fn, int device, size_t smem) {
  std::lock_guard<std::mutex> g(g_attr_mu);
  size_t &have = g_smem_limit[std::make_pair(fn, device)];
  if (smem <= have) return cudaSuccess;
  cudaError_t e = cudaFuncSetAttribute(fn, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e == cudaSuccess) have = smem;
  return e;
}

int occupancy_cached(const void *fn, int device, int threads, size_t smem) {
  std::lock_guard<std::mutex> g(g_attr_mu);
  int &occ = g_occupancy[std::make_tuple(fn, device, threads, smem)];
  if (occ == 0) {
    int n = 0;
    if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&n, fn, threads, smem) != cudaSuccess ||
        n < 1)
      n = 1;
    occ = n;
  }
  return occ;
}

// Device-independent sizing: the B200 limits (148 SMs, 227 KB opt-in shared
// memory per block) decide which kernel variant a workspace must cover.
static DevInfo nominal_devinfo() {
  DevInfo d{};
  d.device = 0;
  d.sms = 148;
  d.max_smem_optin = 232448;
  d.err = nullptr;
  return d;
}

}  // namespace rq

using namespace rq;

namespace {

constexpr int64_t kAlign = 256;

// rq_set_profile_events state (per host thread).
thread_local cudaEvent_t t_prof_start = nullptr;
thread_local cudaEvent_t t_prof_stop = nullptr;

cudaError_t prof_mark(cudaEvent_t ev, cudaStream_t s) {
  return ev ? cudaEventRecord(ev, s) : cudaSuccess;
}

bool dims_ok(const rq_dims &d) {
  if (d.V < 1 || d.V > (int64_t)0x7fffffff - 1024) return false;
  if (d.D < 1 || d.M < 1 || d.L < 1 || d.K < 1) return false;
  if (d.D % d.M != 0) return false;
  if (d.K > 65536) return false;
  if ((int64_t)d.M * d.L > (1 << 20)) return false;
  return true;
}

bool fmt_known(int fmt) {
  return fmt == RQ_CODES_U16 || fmt == RQ_CODES_PACKED10 || fmt == RQ_CODES_SCHED ||
         fmt == RQ_CODES_U8 || fmt == RQ_CODES_PACKED10_ROT;
}

bool fmt_ok(const rq_dims &d, int fmt) {
  if (fmt == RQ_CODES_U16) return true;
  if (fmt == RQ_CODES_PACKED10) return d.K <= 1024;
  if (fmt == RQ_CODES_SCHED) return d.K <= 1024 && ((int64_t)d.M * d.L) % 32 == 0;
  if (fmt == RQ_CODES_U8) return d.K <= 256;
  if (fmt == RQ_CODES_PACKED10_ROT) return d.K <= 1024 && ((int64_t)d.M * d.L) % 64 == 0;
  return false;
}

bool aligned(const void *p, uintptr_t a) { return (reinterpret_cast<uintptr_t>(p) & (a - 1)) == 0; }

// The last CUDA error a call of this host thread met (rq_last_cuda_error).
thread_local int t_last_cuda_error = 0;

int status_of(cudaError_t e) {
  if (e == cudaSuccess) return RQ_OK;
  t_last_cuda_error = (int)e;
  return RQ_ERR_CUDA;
}

// Workspace layout of rq_lut_logits:
//   tiled path (B <= 4):  [partials: nch*B*V floats][argmax keys: B x u64]
//   token-group path:     [argmax block partials: values][indices]
struct WsLayout {
  bool chunk;
  ChunkPlan cp;
  size_t partial_off, partial_bytes;
  size_t amv_off, ami_off, am_bytes;   // argmax block partials (token-group path)
  size_t keys_off;                      // argmax keys (tiled path)
  size_t total;
};

WsLayout ws_layout(const rq_dims &d, int B, int fmt, bool want_argmax, const DevInfo &di) {
  WsLayout w{};
  const int P = d.M * d.L;
  w.cp = plan_chunk(d.V, P, d.K, B, fmt, di);
  w.chunk = w.cp.ok;
  size_t off = 0;
  if (w.chunk) {
    w.partial_off = off;
    w.partial_bytes = chunk_partial_bytes(w.cp, B, d.V);
    off += (size_t)align_up((int64_t)w.partial_bytes, kAlign);
  }
  if (want_argmax && w.chunk) {
    w.keys_off = off;
    off += (size_t)align_up((int64_t)B * 8, kAlign);
  } else if (want_argmax) {
    w.am_bytes = (size_t)B * kMaxSweepBlocks * 4;
    w.amv_off = off;
    off += (size_t)align_up((int64_t)w.am_bytes, kAlign);
    w.ami_off = off;
    off += (size_t)align_up((int64_t)w.am_bytes, kAlign);
  }
  w.total = off;
  return w;
}

int sweep_blocks(const rq_dims &d, const DevInfo &di, bool chunk) {
  if (chunk) {  // reduce kernel: 4 rows per thread, 256 threads per block
    int64_t n = (d.V + 1023) / 1024;
    const int64_t cap = (int64_t)di.sms * 8;
    if (n > cap) n = cap;
    if (n > kMaxSweepBlocks) n = kMaxSweepBlocks;
    return n < 1 ? 1 : (int)n;
  }
  return l2_grid_blocks(d.V, di);
}

// Path shared by rq_lut_logits, rq_logits_from_hidden and rq_greedy_step.
// `after_build`: the kernel just before is this library's table build (which
// writes nothing the code stream reads), so the tiled pass may overlap it.
// `rows_spec`/`rows`: also rebuild the input rows of the picked tokens.
int run_logits(const void *codes, int fmt, const rq_dims &d, const float *lut, int B, int Bs,
               float cap, float *logits, int32_t *argmax, unsigned char *ws,
               const WsLayout &w, const DevInfo &di, cudaStream_t s, bool after_build,
               const DecodeSpec *rows_spec = nullptr, uint16_t *rows = nullptr) {
  const int P = d.M * d.L;
  const int nblk = sweep_blocks(d, di, w.chunk);
  cudaError_t e;
  if (w.chunk) {
    float *partial = reinterpret_cast<float *>(ws + w.partial_off);
    unsigned long long *keys =
        argmax ? reinterpret_cast<unsigned long long *>(ws + w.keys_off) : nullptr;
    if ((e = prof_mark(t_prof_start, s)) != cudaSuccess) return status_of(e);
    const bool prof = t_prof_start != nullptr;   // events between kernels break the overlap
    e = launch_logits_chunk(w.cp, codes, fmt, d.V, P, d.K, B, lut, partial, keys,
                            after_build && !prof, di, s);
    if (e != cudaSuccess) return status_of(e);
    if ((e = prof_mark(t_prof_stop, s)) != cudaSuccess) return status_of(e);
    e = launch_reduce_partials(partial, w.cp.nch, B, d.V, cap, logits, keys, nblk, s);
    if (e != cudaSuccess) return status_of(e);
    if (argmax) return status_of(launch_argmax_keys(keys, B, argmax, rows_spec, rows, s));
    return RQ_OK;
  }
  float *amv = argmax ? reinterpret_cast<float *>(ws + w.amv_off) : nullptr;
  int *ami = argmax ? reinterpret_cast<int *>(ws + w.ami_off) : nullptr;
  if ((e = prof_mark(t_prof_start, s)) != cudaSuccess) return status_of(e);
  for (int b0 = 0; b0 < B; b0 += kTokenGroup) {
    const int nb = B - b0 < kTokenGroup ? B - b0 : kTokenGroup;
    e = launch_logits_l2(codes, fmt, d.V, P, d.K, lut, Bs, b0, b0, nb, cap, logits, amv, ami,
                         nblk, s);
    if (e != cudaSuccess) return status_of(e);
  }
  if ((e = prof_mark(t_prof_stop, s)) != cudaSuccess) return status_of(e);
  if (argmax) return status_of(launch_argmax_finalize(amv, ami, nblk, B, argmax, rows_spec, rows, s));
  return RQ_OK;
}

int fused_group(int B) { return B <= 4 ? B : (B < kTokenGroup ? B : kTokenGroup); }

// First region of the fused calls' workspace: the token group's tables, or,
// for a group decoded on the tensor cores, that kernel's scratch (scales,
// split hidden operand, split codebooks) -- whichever is larger, for every
// shape the tensor-core kernel can take.
size_t table_region_bytes(const rq_dims &d, int B, int fmt) {
  size_t n = (size_t)align_up((int64_t)rq_lut_bytes(d, fused_group(B)), kAlign);
  if (B > 4 && decode_mma_shape_ok(fmt, d.V, d.D, d.M, d.L, d.K)) {
    const size_t tc = (size_t)align_up((int64_t)decode_mma_hop_bytes(d.M, 64, d.K), kAlign);
    if (tc > n) n = tc;
  }
  return n;
}

// Smallest partial token group (fewer than 32 tokens) that the fused calls
// send to the tensor cores: with RQ_PATH_DECODE_TC every group does (down to
// one token); by default from the size where the tables measured slower.
constexpr int kTcPartialMin = 17;
int tc_partial_min(int path) { return path == RQ_PATH_DECODE_TC ? 1 : kTcPartialMin; }


// rq_logits_from_hidden and rq_greedy_step: table build per token group,
// code pass, softcap, logits/argmax, optionally the picked tokens' rows.
int run_fused(const float *h, const float *C, const void *codes, int fmt, const rq_dims &d, int B,
              float softcap, float *logits, int32_t *argmax, void *ws, size_t ws_bytes,
              const DecodeSpec *rows_spec, uint16_t *rows, cudaStream_t s,
              int path = RQ_PATH_AUTO) {
  DevInfo di;
  if (dev_info(&di) != cudaSuccess) return RQ_ERR_CUDA;
  const int G = fused_group(B);
  const int Bs = rq_lut_token_stride(G);
  if ((size_t)Bs * (d.D / d.M) * 4 > 48 * 1024) return RQ_ERR_UNSUPPORTED;
  const size_t lut_bytes = table_region_bytes(d, B, fmt);
  const WsLayout w = ws_layout(d, B, fmt, argmax != nullptr, di);
  if (ws_bytes < lut_bytes + w.total) return RQ_ERR_WORKSPACE_TOO_SMALL;
  float *lut = static_cast<float *>(ws);
  unsigned char *rest = static_cast<unsigned char *>(ws) + lut_bytes;
  if (w.chunk) {
    // B <= 4: one table for all tokens, then the vocabulary-tiled pass
    cudaError_t e = launch_lut_build(h, C, B, 0, B, d.D, d.M, d.L, d.K, Bs, lut, true, s);
    if (e != cudaSuccess) return status_of(e);
    return run_logits(codes, fmt, d, lut, B, Bs, softcap, logits, argmax, rest, w, di, s, true,
                      rows_spec, rows);
  }
  const int P = d.M * d.L;
  float *amv = argmax ? reinterpret_cast<float *>(rest + w.amv_off) : nullptr;
  int *ami = argmax ? reinterpret_cast<int *>(rest + w.ami_off) : nullptr;
  // Token groups decode their rows and multiply them with the hidden states:
  // on the tensor cores by default (groups of 64, then 32, then a rest of 17
  // or more tokens; measured fastest), else the FP32 kernel (groups of 32);
  // other groups read their tables through L2.  All write argmax partials
  // into the same [B][nblk].
  const int nblk = sweep_blocks(d, di, false);
  const bool grid_ok = decode_fma_blocks(d.V, di) <= nblk;
  const bool dfma = grid_ok && decode_fma_applies(fmt, d.V, d.D, d.M, d.L, d.K, B, C, codes, di);
  const bool tc_fmt = grid_ok && decode_mma_applies(fmt, d.V, d.D, d.M, d.L, d.K, C, codes);
  // the tensor-core kernel keeps its scratch (scales, split hidden operand,
  // split codebooks) in the (here unused) table region
  auto tc_fits = [&](int n) {
    return tc_fmt && decode_mma_smem(d.K, n, fmt) <= (size_t)di.max_smem_optin &&
           decode_mma_hop_bytes(d.M, n, d.K) <= lut_bytes;
  };
  const bool tc32 = tc_fits(32), tc64 = tc_fits(64);
  if ((path == RQ_PATH_DECODE_FP32 && !dfma) || (path == RQ_PATH_DECODE_TC && !tc32))
    return RQ_ERR_UNSUPPORTED;
  const bool use_tc = (path == RQ_PATH_DECODE_TC || path == RQ_PATH_AUTO) && tc32;
  const bool use_fma = !use_tc && (path == RQ_PATH_DECODE_FP32 || path == RQ_PATH_AUTO) && dfma;
  cudaError_t e = cudaSuccess;
  bool marked = false;   // the profile start goes before the first logits kernel
  for (int b0 = 0; b0 < B && e == cudaSuccess;) {
    const int rem = B - b0;
    // a group of fewer than 32 tokens also takes the tensor cores from
    // kTcPartialMin tokens on: their time hardly depends on the group's fill,
    // the tables' grows with it
    const int nd = use_tc && tc64 && rem >= 64                 ? 64
                   : (use_tc || use_fma) && rem >= 32          ? 32
                   : use_tc && rem >= tc_partial_min(path)     ? rem
                                                               : 0;
    if (nd > 0) {
      if (!marked && (e = prof_mark(t_prof_start, s)) != cudaSuccess) break;
      marked = true;
      if (use_tc)
        e = launch_logits_decode_mma(h, C, codes, fmt, d.V, d.D, d.M, d.K, b0, nd,
                                     nd > 32 ? 64 : 32, softcap, lut, logits, amv, ami, nblk, di,
                                     s);
      else
        e = launch_logits_decode_fma(h, C, codes, d.V, d.D, d.M, d.K, b0, nd, softcap, logits,
                                     amv, ami, nblk, di, s);
      b0 += nd;
      continue;
    }
    const int nb = rem < G ? rem : G;
    e = launch_lut_build(h, C, B, b0, nb, d.D, d.M, d.L, d.K, Bs, lut, false, s);
    if (e == cudaSuccess && !marked) e = prof_mark(t_prof_start, s);
    marked = true;
    if (e == cudaSuccess)
      e = launch_logits_l2(codes, fmt, d.V, P, d.K, lut, Bs, 0, b0, nb, softcap, logits, amv, ami,
                           nblk, s);
    b0 += nb;
  }
  if (e != cudaSuccess) return status_of(e);
  if (cudaError_t e = prof_mark(t_prof_stop, s)) return status_of(e);
  if (argmax)
    return status_of(launch_argmax_finalize(amv, ami, nblk, B, argmax, rows_spec, rows, s));
  return RQ_OK;
}

}  // namespace

namespace rq {
// Greedy pick over a vocabulary split across ranks (shard_argmax.cu).
cudaError_t launch_argmax_candidates(const float *logits, const int32_t *argmax, int B, int64_t V,
                                     int64_t row0, float *val, int32_t *gidx, cudaStream_t s);
cudaError_t launch_argmax_merge(const float *val, const int32_t *gidx, int n, int B,
                                int32_t *argmax, cudaStream_t s);
}  // namespace rq

extern "C" {

const char *rq_status_string(int status) {
  switch (status) {
    case RQ_OK: return "RQ_OK";
    case RQ_ERR_INVALID_ARGUMENT: return "RQ_ERR_INVALID_ARGUMENT";
    case RQ_ERR_UNSUPPORTED: return "RQ_ERR_UNSUPPORTED";
    case RQ_ERR_WORKSPACE_TOO_SMALL: return "RQ_ERR_WORKSPACE_TOO_SMALL";
    case RQ_ERR_CUDA: return "RQ_ERR_CUDA";
    case RQ_ERR_MISALIGNED: return "RQ_ERR_MISALIGNED";
    default: return "RQ_ERR_UNKNOWN";
  }
}

int rq_version(void) { return 100; }

size_t rq_codes_bytes(rq_dims d, int fmt) {
  if (!dims_ok(d) || !fmt_ok(d, fmt)) return 0;
  const int64_t P = (int64_t)d.M * d.L;
  if (fmt == RQ_CODES_U16 || fmt == RQ_CODES_SCHED) return (size_t)(d.V * P * 2);
  if (fmt == RQ_CODES_U8) return (size_t)(d.V * P);
  if (fmt == RQ_CODES_PACKED10_ROT) return (size_t)(d.V * (10 * P / 8) + d.V * (P / 32));
  return (size_t)(d.V * ((10 * P + 7) / 8));
}

int rq_lut_token_stride(int B) {
  if (B < 1) return 0;
  if (B <= 2) return B;
  return (B + 3) / 4 * 4;
}

size_t rq_lut_bytes(rq_dims d, int B) {
  if (!dims_ok(d) || B < 1) return 0;
  return (size_t)d.M * d.L * d.K * rq_lut_token_stride(B) * sizeof(float);
}

size_t rq_logits_workspace_bytes(rq_dims d, int B, int fmt, int want_argmax) {
  if (!dims_ok(d) || !fmt_ok(d, fmt) || B < 1) return 0;
  return ws_layout(d, B, fmt, want_argmax != 0, nominal_devinfo()).total;
}

size_t rq_fused_workspace_bytes(rq_dims d, int B, int fmt, int want_argmax) {
  if (!dims_ok(d) || !fmt_ok(d, fmt) || B < 1) return 0;
  const size_t lut = table_region_bytes(d, B, fmt);
  return lut + ws_layout(d, B, fmt, want_argmax != 0, nominal_devinfo()).total;
}

int rq_lut_build(const float *h, const float *C, rq_dims d, int B, float *lut, void *stream) {
  if (!h || !C || !lut || B < 1 || !dims_ok(d)) return RQ_ERR_INVALID_ARGUMENT;
  if (!aligned(h, 4) || !aligned(C, 4) || !aligned(lut, 16)) return RQ_ERR_MISALIGNED;
  const int Bs = rq_lut_token_stride(B);
  if ((size_t)Bs * (d.D / d.M) * 4 > 48 * 1024) return RQ_ERR_UNSUPPORTED;
  return status_of(launch_lut_build(h, C, B, 0, B, d.D, d.M, d.L, d.K, Bs, lut, false,
                                    static_cast<cudaStream_t>(stream)));
}

int rq_lut_logits(const void *codes, int fmt, rq_dims d, const float *lut, int B, float softcap,
                  float *logits, int32_t *argmax, void *ws, size_t ws_bytes, void *stream) {
  if (!codes || !lut || B < 1 || !dims_ok(d)) return RQ_ERR_INVALID_ARGUMENT;
  if (!logits && !argmax) return RQ_ERR_INVALID_ARGUMENT;
  if (!fmt_known(fmt)) return RQ_ERR_INVALID_ARGUMENT;
  if (!fmt_ok(d, fmt)) return RQ_ERR_UNSUPPORTED;
  if (!aligned(codes, 16) || !aligned(lut, 16) || (ws && !aligned(ws, 16)) ||
      (logits && !aligned(logits, 4)) || (argmax && !aligned(argmax, 4)))
    return RQ_ERR_MISALIGNED;
  DevInfo di;
  if (dev_info(&di) != cudaSuccess) return RQ_ERR_CUDA;
  const WsLayout w = ws_layout(d, B, fmt, argmax != nullptr, di);
  if (w.total > 0 && (!ws || ws_bytes < w.total)) return RQ_ERR_WORKSPACE_TOO_SMALL;
  return run_logits(codes, fmt, d, lut, B, rq_lut_token_stride(B), softcap, logits, argmax,
                    static_cast<unsigned char *>(ws), w, di, static_cast<cudaStream_t>(stream),
                    false);
}

int rq_logits_from_hidden(const float *h, const float *C, const void *codes, int fmt, rq_dims d,
                          int B, float softcap, float *logits, int32_t *argmax, void *ws,
                          size_t ws_bytes, void *stream) {
  return rq_logits_from_hidden_path(h, C, codes, fmt, d, B, softcap, logits, argmax, ws, ws_bytes,
                                    RQ_PATH_AUTO, stream);
}

int rq_logits_from_hidden_path(const float *h, const float *C, const void *codes, int fmt,
                               rq_dims d, int B, float softcap, float *logits, int32_t *argmax,
                               void *ws, size_t ws_bytes, int path, void *stream) {
  if (path < RQ_PATH_AUTO || path > RQ_PATH_DECODE_TC) return RQ_ERR_INVALID_ARGUMENT;
  if (!h || !C || !codes || B < 1 || !dims_ok(d)) return RQ_ERR_INVALID_ARGUMENT;
  if (!logits && !argmax) return RQ_ERR_INVALID_ARGUMENT;
  if (!fmt_known(fmt)) return RQ_ERR_INVALID_ARGUMENT;
  if (!fmt_ok(d, fmt)) return RQ_ERR_UNSUPPORTED;
  if (!ws) return RQ_ERR_WORKSPACE_TOO_SMALL;
  if (!aligned(h, 4) || !aligned(C, 4) || !aligned(codes, 16) || !aligned(ws, 16) ||
      (logits && !aligned(logits, 4)) || (argmax && !aligned(argmax, 4)))
    return RQ_ERR_MISALIGNED;
  return run_fused(h, C, codes, fmt, d, B, softcap, logits, argmax, ws, ws_bytes, nullptr,
                   nullptr, static_cast<cudaStream_t>(stream), path);
}

int rq_greedy_step(const float *h, const float *C, const void *codes, int fmt, rq_dims d, int B,
                   float softcap, float *logits, int32_t *argmax, float scale, uint16_t *rows,
                   void *ws, size_t ws_bytes, void *stream) {
  if (!h || !C || !codes || !argmax || !rows || B < 1 || !dims_ok(d))
    return RQ_ERR_INVALID_ARGUMENT;
  if (!fmt_known(fmt)) return RQ_ERR_INVALID_ARGUMENT;
  if (!fmt_ok(d, fmt)) return RQ_ERR_UNSUPPORTED;
  if (!ws) return RQ_ERR_WORKSPACE_TOO_SMALL;
  if (!aligned(h, 4) || !aligned(C, 4) || !aligned(codes, 16) || !aligned(ws, 16) ||
      (logits && !aligned(logits, 4)) || !aligned(argmax, 4) || !aligned(rows, 2))
    return RQ_ERR_MISALIGNED;
  DecodeSpec rs;
  rs.codes = codes;
  rs.fmt = fmt;
  rs.C = C;
  rs.V = d.V;
  rs.D = d.D;
  rs.M = d.M;
  rs.L = d.L;
  rs.K = d.K;
  rs.scale = scale;
  rs.fix = make_codefix(d.K);
  return run_fused(h, C, codes, fmt, d, B, softcap, logits, argmax, ws, ws_bytes, &rs, rows,
                   static_cast<cudaStream_t>(stream));
}

int rq_decode_rows(const int32_t *ids, int64_t N, const void *codes, int fmt, const float *C,
                   rq_dims d, float scale, uint16_t *out, void *stream) {
  if (N < 0 || !dims_ok(d)) return RQ_ERR_INVALID_ARGUMENT;
  if (N == 0) return RQ_OK;
  if (!ids || !codes || !C || !out) return RQ_ERR_INVALID_ARGUMENT;
  if (!fmt_known(fmt)) return RQ_ERR_INVALID_ARGUMENT;
  if (!fmt_ok(d, fmt)) return RQ_ERR_UNSUPPORTED;
  if (!aligned(ids, 4) ||
      !aligned(codes, fmt == RQ_CODES_SCHED ? 16 : (fmt == RQ_CODES_U8 ? 1 : 2)) || !aligned(C, 4) ||
      !aligned(out, 2))
    return RQ_ERR_MISALIGNED;
  DevInfo di;
  if (dev_info(&di) != cudaSuccess) return RQ_ERR_CUDA;
  return status_of(launch_decode_rows(ids, N, codes, fmt, C, d.V, d.D, d.M, d.L, d.K, scale, out,
                                      di.err, static_cast<cudaStream_t>(stream)));
}

int rq_pack10(const uint16_t *codes_u16, rq_dims d, uint8_t *packed, void *stream) {
  if (!codes_u16 || !packed || !dims_ok(d)) return RQ_ERR_INVALID_ARGUMENT;
  if (!aligned(codes_u16, 2)) return RQ_ERR_MISALIGNED;
  return status_of(
      launch_pack10(codes_u16, d.V, d.M * d.L, packed, static_cast<cudaStream_t>(stream)));
}

int rq_pack8(const uint16_t *codes_u16, rq_dims d, uint8_t *packed, void *stream) {
  if (!codes_u16 || !packed || !dims_ok(d)) return RQ_ERR_INVALID_ARGUMENT;
  if (!fmt_ok(d, RQ_CODES_U8)) return RQ_ERR_UNSUPPORTED;
  if (!aligned(codes_u16, 2)) return RQ_ERR_MISALIGNED;
  return status_of(launch_pack8(codes_u16, d.V * d.M * d.L, packed,
                                static_cast<cudaStream_t>(stream)));
}

int rq_prepare_sched(const uint16_t *codes_u16, rq_dims d, uint16_t *out, uint64_t *stats,
                     void *stream) {
  if (!codes_u16 || !out || !dims_ok(d)) return RQ_ERR_INVALID_ARGUMENT;
  if (!fmt_ok(d, RQ_CODES_SCHED)) return RQ_ERR_UNSUPPORTED;
  if (!aligned(codes_u16, 2) || !aligned(out, 2) || (stats && !aligned(stats, 8)))
    return RQ_ERR_MISALIGNED;
  const size_t bytes = rq_codes_bytes(d, RQ_CODES_U16);
  const uintptr_t a0 = reinterpret_cast<uintptr_t>(codes_u16), b0 = reinterpret_cast<uintptr_t>(out);
  if (a0 < b0 + bytes && b0 < a0 + bytes) return RQ_ERR_INVALID_ARGUMENT;   // overlap
  return status_of(launch_prepare_sched(codes_u16, d.V, d.M * d.L, d.K, out,
                                        reinterpret_cast<unsigned long long *>(stats),
                                        static_cast<cudaStream_t>(stream)));
}

int rq_prepare_rot10(const uint16_t *codes_u16, rq_dims d, uint8_t *out, uint64_t *stats,
                     void *stream) {
  if (!codes_u16 || !out || !dims_ok(d)) return RQ_ERR_INVALID_ARGUMENT;
  if (!fmt_ok(d, RQ_CODES_PACKED10_ROT)) return RQ_ERR_UNSUPPORTED;
  if (!aligned(codes_u16, 2) || !aligned(out, 16) || (stats && !aligned(stats, 8)))
    return RQ_ERR_MISALIGNED;
  const size_t in_bytes = rq_codes_bytes(d, RQ_CODES_U16);
  const size_t out_bytes = rq_codes_bytes(d, RQ_CODES_PACKED10_ROT);
  const uintptr_t a0 = reinterpret_cast<uintptr_t>(codes_u16), b0 = reinterpret_cast<uintptr_t>(out);
  if (a0 < b0 + out_bytes && b0 < a0 + in_bytes) return RQ_ERR_INVALID_ARGUMENT;   // overlap
  return status_of(launch_prepare_rot10(codes_u16, d.V, d.M * d.L, d.K, out,
                                        reinterpret_cast<unsigned long long *>(stats),
                                        static_cast<cudaStream_t>(stream)));
}

int rq_encode(const float *X, rq_dims d, const float *C, uint16_t *codes, void *stream) {
  rq_dims d1 = d;
  if (d1.V == 0) d1.V = 1;
  if (!dims_ok(d1)) return RQ_ERR_INVALID_ARGUMENT;
  if (d.V == 0) return RQ_OK;
  if (!X || !C || !codes) return RQ_ERR_INVALID_ARGUMENT;
  if (d.D / d.M > 32) return RQ_ERR_UNSUPPORTED;
  if (!aligned(X, 4) || !aligned(C, 4) || !aligned(codes, 2)) return RQ_ERR_MISALIGNED;
  const uintptr_t c0 = reinterpret_cast<uintptr_t>(codes);
  const size_t cb = rq_codes_bytes(d, RQ_CODES_U16);
  const uintptr_t x0 = reinterpret_cast<uintptr_t>(X), k0 = reinterpret_cast<uintptr_t>(C);
  const size_t xb = (size_t)d.V * d.D * sizeof(float);
  const size_t kb = (size_t)d.M * d.L * d.K * (d.D / d.M) * sizeof(float);
  if ((c0 < x0 + xb && x0 < c0 + cb) || (c0 < k0 + kb && k0 < c0 + cb))
    return RQ_ERR_INVALID_ARGUMENT;   // overlap
  return status_of(launch_encode(X, d.V, C, d.D, d.M, d.L, d.K, codes,
                                 static_cast<cudaStream_t>(stream)));
}

size_t rq_topk_workspace_bytes(int64_t V, int B, int k) {
  if (V < 1 || V > (int64_t)0x7fffffff - 1024 || B < 1 || B > 65535 || k < 1 || k > 1024 ||
      k > V)
    return 0;
  return topk_workspace_bytes(V, B, k);
}

int rq_topk_sample(const float *logits, int64_t V, int B, int k, float temperature,
                   uint64_t seed, uint64_t step, float *topk_val, int32_t *topk_idx,
                   int32_t *token, void *ws, size_t ws_bytes, void *stream) {
  if (!logits || !ws || V < 1 || V > (int64_t)0x7fffffff - 1024 || B < 1 || B > 65535 ||
      k < 1 || k > V)
    return RQ_ERR_INVALID_ARGUMENT;
  if (k > 1024) return RQ_ERR_UNSUPPORTED;
  if (!aligned(logits, 4) || !aligned(ws, 256) || (topk_val && !aligned(topk_val, 4)) ||
      (topk_idx && !aligned(topk_idx, 4)) || (token && !aligned(token, 4)))
    return RQ_ERR_MISALIGNED;
  if (ws_bytes < rq_topk_workspace_bytes(V, B, k)) return RQ_ERR_WORKSPACE_TOO_SMALL;
  return status_of(launch_topk_sample(logits, V, B, k, (double)temperature, seed, step,
                                      topk_val, topk_idx, token, ws,
                                      static_cast<cudaStream_t>(stream)));
}

int rq_last_cuda_error(int clear) {
  const int e = t_last_cuda_error;
  if (clear) t_last_cuda_error = 0;
  return e;
}

const char *rq_cuda_error_name(int err) { return cudaGetErrorName(static_cast<cudaError_t>(err)); }

int rq_set_profile_events(void *start, void *stop) {
  if ((start == nullptr) != (stop == nullptr)) return RQ_ERR_INVALID_ARGUMENT;
  t_prof_start = static_cast<cudaEvent_t>(start);
  t_prof_stop = static_cast<cudaEvent_t>(stop);
  return RQ_OK;
}

int rq_argmax_candidates(const float *logits, const int32_t *argmax, int B, int64_t V,
                         int64_t row0, float *val, int32_t *gidx, void *stream) {
  if (!logits || !argmax || !val || !gidx || B < 1 || V < 1 || row0 < 0 ||
      row0 + V > (int64_t)INT_MAX)
    return RQ_ERR_INVALID_ARGUMENT;
  if (!aligned(logits, 4) || !aligned(argmax, 4) || !aligned(val, 4) || !aligned(gidx, 4))
    return RQ_ERR_MISALIGNED;
  return status_of(launch_argmax_candidates(logits, argmax, B, V, row0, val, gidx,
                                            static_cast<cudaStream_t>(stream)));
}

int rq_argmax_merge(const float *val, const int32_t *gidx, int n, int B, int32_t *argmax,
                    void *stream) {
  if (!val || !gidx || !argmax || n < 1 || B < 1) return RQ_ERR_INVALID_ARGUMENT;
  if (!aligned(val, 4) || !aligned(gidx, 4) || !aligned(argmax, 4)) return RQ_ERR_MISALIGNED;
  return status_of(launch_argmax_merge(val, gidx, n, B, argmax, static_cast<cudaStream_t>(stream)));
}

int rq_device_error(uint32_t *out, int clear) {
  if (!out) return RQ_ERR_INVALID_ARGUMENT;
  DevInfo di;
  if (dev_info(&di) != cudaSuccess) return RQ_ERR_CUDA;
  unsigned v = 0;
  cudaError_t e = cudaMemcpy(&v, di.err, sizeof v, cudaMemcpyDeviceToHost);
  if (e != cudaSuccess) return RQ_ERR_CUDA;
  *out = v;
  if (clear) {
    e = cudaMemset(di.err, 0, sizeof(unsigned));
    if (e != cudaSuccess) return RQ_ERR_CUDA;
  }
  return RQ_OK;
}

}  // extern "C"

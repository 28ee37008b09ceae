// logits_chunk.cu -- LUT lookup+sum logits for small token counts (B <= 4),
// the code matrix streamed once from HBM.
//
// "Gemma-2 runtime compression: NF4 + LUT serving", LUT section: output
// logits by lookup + sum over each vocabulary row's codes instead of the
// full matmul, followed by Gemma-2's softcap:
//   z[b][v] = sum_p T[p][code[v][p]][b],   y = cap * tanh(z / cap).
//
// Design for sm_100a.  One token's tables are P*K*4 bytes (3.1 MB at the
// Gemma-2 shape): far more than one SM's shared memory, but a chunk of PC
// (m, l) pairs (PC*K*TB*4 bytes) fits.  Work units are (chunk, tile of R
// vocabulary rows), ordered chunk-major and split evenly over a persistent
// grid of one CTA per SM, so a CTA loads one or two table chunks into shared
// memory (from L2, where the build kernel left them) and then streams its
// code tiles:
//   * each tile is a TMA 2-D box {PC codes, 256 rows} of the uint16 code
//     matrix (a 2*PC-byte slice of every 2*P-byte row), landing in an
//     NST-deep ring of shared-memory stages guarded by mbarriers; the code
//     stream carries an L2 evict-first policy;
//   * thread r owns row r of the tile: it reads its 2*PC code bytes with
//     16-byte shared loads (row pitch = an odd multiple of 16 bytes, so the
//     8 lanes of each load phase hit distinct bank groups) and performs PC
//     table lookups, summing TB tokens in fp32 registers;
//   * the per-chunk sums go to partial[c][b][v]; a second kernel adds the
//     chunks in order, applies the softcap, writes logits and argmax
//     partials.  Partials are 4*nch bytes per row and token (L2-resident).
#include <cfloat>
#include <climits>

#include "rq_common.cuh"

namespace rq {

struct ChunkArgs {
  const float *lut;   // [P][K][TB]
  float *partial;     // [nch][B][V]
  int64_t V;
  int64_t ntiles;     // tiles of THREADS rows
  int64_t nunits;     // nch * ntiles
  int P, K, B, nch;
  CodeFix fix;
  unsigned *err;
};

template <int KT>
__device__ __forceinline__ uint32_t fix_code(uint32_t c, const CodeFix &f) {
  if (KT > 0 && (KT & (KT - 1)) == 0) return c & (uint32_t)(KT - 1);
  return f(c);
}

template <int TB>
__device__ __forceinline__ void add_entry(const float *e, float (&acc)[TB]) {
  if (TB == 1) {
    acc[0] += e[0];
  } else if (TB == 2) {
    const float2 t = *reinterpret_cast<const float2 *>(e);
    acc[0] += t.x;
    acc[1] += t.y;
  } else {
    const float4 t = *reinterpret_cast<const float4 *>(e);
    acc[0] += t.x;
    acc[1] += t.y;
    acc[2] += t.z;
    acc[3] += t.w;
  }
}

// 8 consecutive pairs (one 16-byte code vector) of one row.
template <int TB, int KT>
__device__ __forceinline__ void lookup8(const float *Tg, int K, uint4 w, const CodeFix &f,
                                        float (&acc)[TB]) {
  const uint32_t ws[4] = {w.x, w.y, w.z, w.w};
#pragma unroll
  for (int q = 0; q < 4; ++q) {
    const uint32_t c0 = fix_code<KT>(ws[q] & 0xFFFFu, f);
    const uint32_t c1 = fix_code<KT>(ws[q] >> 16, f);
    add_entry<TB>(Tg + ((size_t)(2 * q) * K + c0) * TB, acc);
    add_entry<TB>(Tg + ((size_t)(2 * q + 1) * K + c1) * TB, acc);
  }
}

template <int TB, int KT, int PC, int NST, int THREADS>
__global__ void __launch_bounds__(THREADS, 1)
    logits_chunk_u16_kernel(const __grid_constant__ CUtensorMap tmap, const ChunkArgs a) {
  static_assert(PC % 8 == 0 && (PC / 8) % 2 == 1, "row pitch must be an odd multiple of 16 B");
  static_assert(THREADS % 256 == 0, "tiles are whole TMA boxes of 256 rows");
  constexpr int STAGE_BYTES = THREADS * PC * 2;
  constexpr int BOX_BYTES = 256 * PC * 2;

  extern __shared__ unsigned char smem_raw[];
  unsigned char *smem = reinterpret_cast<unsigned char *>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const int K = KT > 0 ? KT : a.K;
  float *Ts = reinterpret_cast<float *>(smem);
  const size_t t_bytes = (size_t)align_up((int64_t)PC * K * TB * 4, 1024);
  unsigned char *stages = smem + t_bytes;
  uint64_t *bars = reinterpret_cast<uint64_t *>(stages + (size_t)NST * STAGE_BYTES);

  const int64_t per = a.nunits / gridDim.x, rem = a.nunits % gridDim.x;
  const int64_t bx = blockIdx.x;
  const int64_t u0 = bx * per + (bx < rem ? bx : rem);
  const int64_t u1 = u0 + per + (bx < rem ? 1 : 0);

  if (threadIdx.x == 0) {
    prefetch_tmap(&tmap);
    for (int s = 0; s < NST; ++s) mbar_init(smem_addr(&bars[s]), 1);
    fence_mbar_init();
  }
  __syncthreads();

  const uint64_t pol = l2_policy_evict_first();
  auto issue = [&](int64_t u, int s) {
    const int c = (int)(u / a.ntiles);
    const int64_t t = u % a.ntiles;
    const uint32_t bar = smem_addr(&bars[s]);
    mbar_arrive_expect_tx(bar, STAGE_BYTES);
#pragma unroll
    for (int q = 0; q < THREADS / 256; ++q)
      tma_load_2d(smem_addr(stages + (size_t)s * STAGE_BYTES + q * BOX_BYTES), &tmap, c * PC,
                  (int)(t * THREADS + q * 256), bar, pol);
  };

  if (threadIdx.x == 0) {
    for (int s = 0; s < NST; ++s)
      if (u0 + s < u1) issue(u0 + s, s);
  }

  int cur = -1;
  bool failed = false;
  int64_t u = u0;
  for (; u < u1; ++u) {
    const int64_t i = u - u0;
    const int c = (int)(u / a.ntiles);
    const int64_t t = u % a.ntiles;
    const int np = min(PC, a.P - c * PC);
    if (c != cur) {
      // Table chunk c -> shared memory (all threads finished the previous
      // tile at the barrier that ended the last iteration).
      const float4 *src = reinterpret_cast<const float4 *>(a.lut + (size_t)c * PC * K * TB);
      float4 *dst = reinterpret_cast<float4 *>(Ts);
      const int n4 = np * K * TB / 4;
      for (int q = threadIdx.x; q < n4; q += THREADS) dst[q] = __ldg(src + q);
      __syncthreads();
      cur = c;
    }
    const int s = (int)(i % NST);
    const uint32_t par = (uint32_t)((i / NST) & 1);
    const bool ok = mbar_wait_bounded(smem_addr(&bars[s]), par);
    if (ok) {
      const int64_t v = t * THREADS + threadIdx.x;
      const int ng = np / 8;
      const uint4 *row =
          reinterpret_cast<const uint4 *>(stages + (size_t)s * STAGE_BYTES + threadIdx.x * PC * 2);
      float acc[TB];
#pragma unroll
      for (int b = 0; b < TB; ++b) acc[b] = 0.f;
#pragma unroll
      for (int g = 0; g < PC / 8; ++g) {
        if (g < ng) lookup8<TB, KT>(Ts + (size_t)g * 8 * K * TB, K, row[g], a.fix, acc);
      }
      if (v < a.V) {
#pragma unroll
        for (int b = 0; b < TB; ++b)
          if (b < a.B) a.partial[((size_t)c * a.B + b) * a.V + v] = acc[b];
      }
    }
    if (__syncthreads_or(!ok)) {
      failed = true;
      break;
    }
    if (threadIdx.x == 0 && u + NST < u1) issue(u + NST, s);
  }
  if (failed && threadIdx.x == 0) {
    atomicOr(a.err, RQ_DEVERR_TIMEOUT);
    // Let copies already in flight land before the CTA's shared memory goes.
    for (int64_t w = u; w < u1 && w < u + NST; ++w) {
      const int64_t i = w - u0;
      mbar_wait_bounded(smem_addr(&bars[i % NST]), (uint32_t)((i / NST) & 1));
    }
  }
}

// ------------------------------------------------------------ reduction

__global__ void __launch_bounds__(256) reduce_partials_kernel(const float *__restrict__ partial,
                                                              int nch, int B, int64_t V,
                                                              float cap, float *logits,
                                                              float *am_val, int *am_idx) {
  const int b = blockIdx.y;
  ArgBest best{-FLT_MAX, INT_MAX};
  bool any = false;
  for (int64_t v = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; v < V;
       v += (int64_t)gridDim.x * blockDim.x) {
    float z = 0.f;
    for (int c = 0; c < nch; ++c) z += __ldcs(partial + ((size_t)c * B + b) * V + v);
    const float y = softcap_f(z, cap);
    if (logits) logits[(size_t)b * V + v] = y;
    const ArgBest cand{y, (int)v};
    best = any ? arg_better(best, cand) : cand;
    any = true;
  }
  if (am_val == nullptr) return;
  if (!any) best = ArgBest{-FLT_MAX, INT_MAX};
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) best = arg_better(best, arg_shfl_xor(best, o));
  __shared__ ArgBest wbest[8];
  const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
  if (lane == 0) wbest[warp] = best;
  __syncthreads();
  if (threadIdx.x == 0) {
    ArgBest r = wbest[0];
    for (int w = 1; w < (int)blockDim.x / 32; ++w) r = arg_better(r, wbest[w]);
    am_val[(size_t)b * gridDim.x + blockIdx.x] = r.v;
    am_idx[(size_t)b * gridDim.x + blockIdx.x] = r.i;
  }
}

__global__ void __launch_bounds__(256) argmax_finalize_kernel(const float *__restrict__ am_val,
                                                              const int *__restrict__ am_idx,
                                                              int nblk, int32_t *argmax) {
  const int b = blockIdx.x;
  ArgBest best{-FLT_MAX, INT_MAX};
  for (int k = threadIdx.x; k < nblk; k += blockDim.x)
    best = arg_better(best, ArgBest{am_val[(size_t)b * nblk + k], am_idx[(size_t)b * nblk + k]});
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) best = arg_better(best, arg_shfl_xor(best, o));
  __shared__ ArgBest wbest[8];
  const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
  if (lane == 0) wbest[warp] = best;
  __syncthreads();
  if (threadIdx.x == 0) {
    ArgBest r = wbest[0];
    for (int w = 1; w < (int)blockDim.x / 32; ++w) r = arg_better(r, wbest[w]);
    argmax[b] = r.i;
  }
}

// ------------------------------------------------------------ host side

namespace {

typedef CUresult (*EncodeTiledFn)(CUtensorMap *, CUtensorMapDataType, cuuint32_t, void *,
                                  const cuuint64_t *, const cuuint64_t *, const cuuint32_t *,
                                  const cuuint32_t *, CUtensorMapInterleave, CUtensorMapSwizzle,
                                  CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn encode_fn() {
  static EncodeTiledFn fn = nullptr;
  static bool tried = false;
  if (!tried) {
    tried = true;
    void *p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) ==
            cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<EncodeTiledFn>(p);
  }
  return fn;
}

struct Variant {
  int TB, KT, PC, NST, THREADS;
  const void *fn;
};

#define RQ_CHUNK_VARIANT(TB, KT, PC, NST, TH)                                   \
  Variant {                                                                     \
    TB, KT, PC, NST, TH,                                                        \
        reinterpret_cast<const void *>(&logits_chunk_u16_kernel<TB, KT, PC, NST, TH>) \
  }

// Chosen so table chunk + NST stages fit in 227 KB with one CTA per SM.
const Variant kVariants[] = {
    RQ_CHUNK_VARIANT(1, 1024, 40, 3, 256),   // 160 KB table + 3 x 20 KB
    RQ_CHUNK_VARIANT(2, 1024, 24, 2, 256),   // 192 KB table + 2 x 12 KB
    RQ_CHUNK_VARIANT(4, 1024, 8, 6, 256),    // 128 KB table + 6 x 4 KB
    RQ_CHUNK_VARIANT(1, 0, 40, 3, 256),      // any K (runtime)
    RQ_CHUNK_VARIANT(2, 0, 24, 3, 256),
    RQ_CHUNK_VARIANT(4, 0, 8, 4, 256),
};

size_t variant_smem(const Variant &v, int K) {
  return 1024 + (size_t)align_up((int64_t)v.PC * K * v.TB * 4, 1024) +
         (size_t)v.NST * v.THREADS * v.PC * 2 + 1024;
}

}  // namespace

ChunkPlan plan_chunk(int64_t V, int P, int K, int B, int fmt, const DevInfo &di) {
  ChunkPlan cp{};
  cp.ok = false;
  if (fmt != RQ_CODES_U16 || B < 1 || B > 4 || P % 8 != 0) return cp;
  if (V > (int64_t)INT_MAX - 512) return cp;
  const int TB = rq_lut_token_stride(B);
  for (int i = 0; i < (int)(sizeof(kVariants) / sizeof(kVariants[0])); ++i) {
    const Variant &v = kVariants[i];
    if (v.TB != TB) continue;
    if (v.KT != 0 && v.KT != K) continue;
    const size_t smem = variant_smem(v, K);
    if (smem > (size_t)di.max_smem_optin) continue;
    cp.ok = true;
    cp.TB = TB;
    cp.PC = v.PC;
    cp.nch = (P + v.PC - 1) / v.PC;
    cp.R = v.THREADS;
    cp.variant = i;
    cp.smem = smem;
    return cp;
  }
  return cp;
}

size_t chunk_partial_bytes(const ChunkPlan &cp, int B, int64_t V) {
  return (size_t)cp.nch * B * V * sizeof(float);
}

cudaError_t launch_logits_chunk(const ChunkPlan &cp, const void *codes, int fmt, int64_t V,
                                int P, int K, int B, const float *lut, float *partial,
                                const DevInfo &di, cudaStream_t s) {
  (void)fmt;
  const Variant &var = kVariants[cp.variant];
  if (encode_fn() == nullptr) return cudaErrorNotSupported;
  CUtensorMap tmap;
  const cuuint64_t gdim[2] = {(cuuint64_t)P, (cuuint64_t)V};
  const cuuint64_t gstride[1] = {(cuuint64_t)P * 2};
  const cuuint32_t box[2] = {(cuuint32_t)var.PC, 256u};
  const cuuint32_t estride[2] = {1u, 1u};
  CUresult r = encode_fn()(&tmap, CU_TENSOR_MAP_DATA_TYPE_UINT16, 2, const_cast<void *>(codes),
                           gdim, gstride, box, estride, CU_TENSOR_MAP_INTERLEAVE_NONE,
                           CU_TENSOR_MAP_SWIZZLE_NONE, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                           CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  if (r != CUDA_SUCCESS) return cudaErrorInvalidValue;

  static bool attr_set[64][sizeof(kVariants) / sizeof(kVariants[0])] = {};
  if (di.device < 64 && !attr_set[di.device][cp.variant]) {
    cudaError_t e = cudaFuncSetAttribute(var.fn, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         (int)cp.smem);
    if (e != cudaSuccess) return e;
    attr_set[di.device][cp.variant] = true;
  }

  ChunkArgs a;
  a.lut = lut;
  a.partial = partial;
  a.V = V;
  a.ntiles = (V + var.THREADS - 1) / var.THREADS;
  a.nunits = a.ntiles * cp.nch;
  a.P = P;
  a.K = K;
  a.B = B;
  a.nch = cp.nch;
  a.fix = make_codefix(K);
  a.err = di.err;
  int64_t grid = di.sms;
  if (grid > a.nunits) grid = a.nunits;
  if (grid < 1) grid = 1;
  void *args[] = {&tmap, &a};
  return cudaLaunchKernel(var.fn, dim3((unsigned)grid), dim3(var.THREADS), args, cp.smem, s);
}

cudaError_t launch_reduce_partials(const float *partial, int nch, int B, int64_t V, float cap,
                                   float *logits, float *am_val, int *am_idx, int nblk,
                                   cudaStream_t s) {
  reduce_partials_kernel<<<dim3((unsigned)nblk, (unsigned)B), 256, 0, s>>>(
      partial, nch, B, V, cap, logits, am_val, am_idx);
  return cudaGetLastError();
}

cudaError_t launch_argmax_finalize(const float *am_val, const int *am_idx, int nblk, int B,
                                   int32_t *argmax, cudaStream_t s) {
  argmax_finalize_kernel<<<(unsigned)B, 256, 0, s>>>(am_val, am_idx, nblk, argmax);
  return cudaGetLastError();
}

}  // namespace rq

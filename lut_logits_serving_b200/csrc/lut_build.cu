// lut_build.cu -- per-token lookup tables for LUT serving.
//
// "Gemma-2 runtime compression: NF4 + LUT serving", LUT section: output
// logits come from lookup + sum instead of the V x D matmul.  The tables are
//   T[p = m*L + l][k][t] = sum_{j<ds} h[b0 + t][m*ds + j] * C[m][l][k][j]
// stored token-innermost with stride Bs so one table row (p, k) of a token
// group is a contiguous run of Bs floats.
//
// Work: P*K*nb*ds FMAs (4.7 M per token at the Gemma-2 shape) and one read
// of the 18.9 MB codebook; HBM/L2-bound and small next to the code stream.
#include "rq_common.cuh"

namespace rq {

template <int DSMAX>
__global__ void __launch_bounds__(256) lut_build_kernel(const float *__restrict__ h,
                                                        const float *__restrict__ C, int b0,
                                                        int nb, int D, int M, int L, int K,
                                                        int Bs, float *__restrict__ lut) {
  extern __shared__ float hs[];  // [Bs][ds] hidden slice of subspace m
  griddep_wait();
  const int p = blockIdx.y;
  const int m = p / L;
  const int ds = D / M;
  for (int i = threadIdx.x; i < Bs * ds; i += blockDim.x) {
    int t = i / ds, j = i % ds;
    hs[i] = t < nb ? h[(size_t)(b0 + t) * D + (size_t)m * ds + j] : 0.f;
  }
  __syncthreads();
  const int k = blockIdx.x * blockDim.x + threadIdx.x;
  if (k >= K) return;
  const float *cw = C + ((size_t)p * K + k) * ds;
  float *out = lut + ((size_t)p * K + k) * Bs;
  if (DSMAX > 0) {
    float c[DSMAX > 0 ? DSMAX : 1];
#pragma unroll
    for (int j = 0; j < DSMAX; ++j) c[j] = j < ds ? __ldg(cw + j) : 0.f;
    for (int t = 0; t < Bs; ++t) {
      float acc = 0.f;
#pragma unroll
      for (int j = 0; j < DSMAX; ++j)
        if (j < ds) acc = fmaf(hs[t * ds + j], c[j], acc);
      out[t] = acc;
    }
  } else {
    for (int t = 0; t < Bs; ++t) {
      float acc = 0.f;
      for (int j = 0; j < ds; ++j) acc = fmaf(hs[t * ds + j], __ldg(cw + j), acc);
      out[t] = acc;
    }
  }
}

// Small tables, B <= 2 (e.g. the RQ-coded MLP matrices: ds = 2, K = 128 or
// 256): one thread per table row (p, k) over the flattened P*K rows, so every
// block is full whatever K is.
template <int DS>
__global__ void __launch_bounds__(256) lut_build_flat_kernel(const float *__restrict__ h,
                                                            const float *__restrict__ C, int b0,
                                                            int nb, int D, int L, int K, int Bs,
                                                            int rows, float *__restrict__ lut) {
  griddep_wait();
  const int e = blockIdx.x * blockDim.x + threadIdx.x;   // p*K + k (< 2^31, checked)
  if (e >= rows) return;
  const int p = e / K, m = p / L;
  float c[DS];
#pragma unroll
  for (int j = 0; j < DS; ++j) c[j] = __ldg(C + (size_t)e * DS + j);
  for (int t = 0; t < Bs; ++t) {
    float acc = 0.f;
    if (t < nb) {
      const float *hm = h + (size_t)(b0 + t) * D + (size_t)m * DS;
#pragma unroll
      for (int j = 0; j < DS; ++j) acc = fmaf(__ldg(hm + j), c[j], acc);
    }
    lut[(size_t)e * Bs + t] = acc;
  }
}

// ds = 6 (the Gemma-2 shape: D = 2304, M = 384): one thread per 4
// consecutive codewords of a table = 96 contiguous bytes of C read as six
// 16-byte loads with an L2 evict-last hint (the 18.9 MB codebook is reused
// by every call and then stays in L2 beside the evict-first code stream).
__device__ __forceinline__ float4 ldg_v4_keep(const float *p, uint64_t pol) {
  float4 v;
  asm volatile("ld.global.nc.L2::cache_hint.v4.f32 {%0, %1, %2, %3}, [%4], %5;"
               : "=f"(v.x), "=f"(v.y), "=f"(v.z), "=f"(v.w)
               : "l"(p), "l"(pol));
  return v;
}

__global__ void __launch_bounds__(256) lut_build_ds6_kernel(const float *__restrict__ h,
                                                           const float *__restrict__ C, int b0,
                                                           int nb, int D, int L, int K, int Bs,
                                                           int quads, int early,
                                                           float *__restrict__ lut) {
  // One wave.  `early`: let the next kernel start now; the shared-memory
  // chunk pass loads its first codes before it waits on this one.  A pass
  // that reads its tables through L2 is not started early: measured on a
  // B200 at V = 256000, P = 768, K = 1024, one token, it then ran 3x longer.
  if (early) griddep_launch_dependents();
  griddep_wait();                          // h and the table buffer: earlier kernels
  // P*K < 2^31 (checked by the launcher): 32-bit index math, no 64-bit divides
  const int g = blockIdx.x * blockDim.x + threadIdx.x;
  if (g >= quads) return;
  const int e0 = 4 * g;                     // first codeword (p*K + k) of this thread
  const int p = e0 / K;
  const int m = p / L;
  const uint64_t pol = l2_policy_evict_last();
  float c[24];
#pragma unroll
  for (int q = 0; q < 6; ++q) {
    const float4 v = ldg_v4_keep(C + (size_t)e0 * 6 + 4 * q, pol);
    c[4 * q + 0] = v.x;
    c[4 * q + 1] = v.y;
    c[4 * q + 2] = v.z;
    c[4 * q + 3] = v.w;
  }
  float *out = lut + (size_t)e0 * Bs;
  for (int t = 0; t < Bs; ++t) {
    float hv[6];
#pragma unroll
    for (int j = 0; j < 6; ++j) hv[j] = t < nb ? __ldg(h + (size_t)(b0 + t) * D + m * 6 + j) : 0.f;
    float r[4];
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      float acc = 0.f;
#pragma unroll
      for (int j = 0; j < 6; ++j) acc = fmaf(hv[j], c[6 * i + j], acc);
      r[i] = acc;
    }
    if (Bs == 1) {
      *reinterpret_cast<float4 *>(out) = make_float4(r[0], r[1], r[2], r[3]);
    } else {
#pragma unroll
      for (int i = 0; i < 4; ++i) out[(size_t)i * Bs + t] = r[i];
    }
  }
}

// ds = 6, token groups (Bs % 4 == 0): grid (K*Bs/4/256, P), one pair per
// block so the block's hidden slice h[b0..b0+Bs][m*6..m*6+6] is staged once in
// shared memory; one thread per (codeword, 4 tokens) writes a float4, a warp
// 8 codewords x 32 tokens... as contiguous runs.
__global__ void __launch_bounds__(256) lut_build_ds6_tok_kernel(
    const float *__restrict__ h, const float *__restrict__ C, int b0, int nb, int D, int L, int K,
    int Bs, float *__restrict__ lut) {
  __shared__ float hs[64][6];
  griddep_wait();
  const int p = blockIdx.y;
  const int m = p / L;
  for (int i = threadIdx.x; i < Bs * 6; i += blockDim.x) {
    const int t = i / 6, j = i % 6;
    hs[t][j] = t < nb ? __ldg(h + (size_t)(b0 + t) * D + m * 6 + j) : 0.f;
  }
  __syncthreads();
  const int q = Bs / 4;
  const int g = blockIdx.x * blockDim.x + threadIdx.x;   // (k, token quad) within the pair
  if (g < K * q) {
    const int k = g / q;
    const int t0 = (g - k * q) * 4;
    const size_t e = (size_t)p * K + k;
    const float *cw = C + e * 6;
    const float2 c01 = __ldg(reinterpret_cast<const float2 *>(cw));
    const float2 c23 = __ldg(reinterpret_cast<const float2 *>(cw + 2));
    const float2 c45 = __ldg(reinterpret_cast<const float2 *>(cw + 4));
    const float c[6] = {c01.x, c01.y, c23.x, c23.y, c45.x, c45.y};
    float r[4];
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      float acc = 0.f;
#pragma unroll
      for (int j = 0; j < 6; ++j) acc = fmaf(hs[t0 + i][j], c[j], acc);
      r[i] = acc;
    }
    *reinterpret_cast<float4 *>(lut + e * Bs + t0) = make_float4(r[0], r[1], r[2], r[3]);
  }
  griddep_launch_dependents();
}

cudaError_t launch_lut_build(const float *h, const float *C, int B, int b0, int nb, int D,
                             int M, int L, int K, int Bs, float *lut, bool early_dependents,
                             cudaStream_t s) {
  (void)B;
  const int ds = D / M;
  const int P = M * L;
  if (ds == 6 && Bs % 4 == 0 && Bs <= 64 && (reinterpret_cast<uintptr_t>(C) & 7) == 0 &&
      (reinterpret_cast<uintptr_t>(lut) & 15) == 0) {
    const int64_t items = (int64_t)K * (Bs / 4);     // per pair
    const int64_t bx = (items + 255) / 256;
    if (items < 0x7fffffffLL - 256 && P <= 65535)
      return pdl_launch(lut_build_ds6_tok_kernel, dim3((unsigned)bx, (unsigned)P), dim3(256), 0, s,
                        h, C, b0, nb, D, L, K, Bs, lut);
  }
  if (ds == 6 && Bs <= 2 && K % 4 == 0 && (reinterpret_cast<uintptr_t>(C) & 15) == 0 &&
      (reinterpret_cast<uintptr_t>(lut) & 15) == 0) {
    const int64_t quads = (int64_t)P * K / 4;
    const int64_t blocks = (quads + 255) / 256;
    if (4 * quads < 0x7fffffffLL - 1024)
      return pdl_launch(lut_build_ds6_kernel, dim3((unsigned)blocks), dim3(256), 0, s, h, C, b0,
                        nb, D, L, K, Bs, (int)quads, early_dependents ? 1 : 0, lut);
  }
  const int64_t rows = (int64_t)P * K;
  if (Bs <= 2 && rows < 0x7fffffffLL - 256) {
    const dim3 g((unsigned)((rows + 255) / 256));
    switch (ds) {
      case 1: return pdl_launch(lut_build_flat_kernel<1>, g, dim3(256), 0, s, h, C, b0, nb, D, L, K, Bs, (int)rows, lut);
      case 2: return pdl_launch(lut_build_flat_kernel<2>, g, dim3(256), 0, s, h, C, b0, nb, D, L, K, Bs, (int)rows, lut);
      case 3: return pdl_launch(lut_build_flat_kernel<3>, g, dim3(256), 0, s, h, C, b0, nb, D, L, K, Bs, (int)rows, lut);
      case 4: return pdl_launch(lut_build_flat_kernel<4>, g, dim3(256), 0, s, h, C, b0, nb, D, L, K, Bs, (int)rows, lut);
      case 8: return pdl_launch(lut_build_flat_kernel<8>, g, dim3(256), 0, s, h, C, b0, nb, D, L, K, Bs, (int)rows, lut);
      default: break;
    }
  }
  dim3 grid((unsigned)((K + 255) / 256), (unsigned)P);
  size_t smem = (size_t)Bs * ds * sizeof(float);
  if (smem > 48 * 1024) return cudaErrorInvalidValue;
  if (ds <= 8)
    return pdl_launch(lut_build_kernel<8>, grid, dim3(256), smem, s, h, C, b0, nb, D, M, L, K, Bs,
                      lut);
  return pdl_launch(lut_build_kernel<0>, grid, dim3(256), smem, s, h, C, b0, nb, D, M, L, K, Bs,
                    lut);
}

}  // namespace rq

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

cudaError_t launch_lut_build(const float *h, const float *C, int B, int b0, int nb, int D,
                             int M, int L, int K, int Bs, float *lut, cudaStream_t s) {
  (void)B;
  const int ds = D / M;
  const int P = M * L;
  dim3 grid((unsigned)((K + 255) / 256), (unsigned)P);
  size_t smem = (size_t)Bs * ds * sizeof(float);
  if (smem > 48 * 1024) return cudaErrorInvalidValue;
  if (ds <= 8)
    lut_build_kernel<8><<<grid, 256, smem, s>>>(h, C, b0, nb, D, M, L, K, Bs, lut);
  else
    lut_build_kernel<0><<<grid, 256, smem, s>>>(h, C, b0, nb, D, M, L, K, Bs, lut);
  return cudaGetLastError();
}

}  // namespace rq

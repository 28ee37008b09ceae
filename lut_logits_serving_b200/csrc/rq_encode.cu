// rq_encode.cu -- greedy residual nearest-codeword encoder (the producer of
// the code matrix).
//
// "Gemma-2-2B combined RQ+NF4" names the embedding compression residual
// product quantization (M = 384 subspaces, K = 1024, L = 2) without giving
// the assignment rule.  Encoded here, per row x and subspace m, with the
// residual r = x[m*ds, (m+1)*ds):
//   for l = 0..L-1:  code_l = argmin_k  sum_j (r_j - C[m][l][k][j])^2
//                    r_j   -= C[m][l][code_l][j]
// "argmin" is a decision taken in fp32: t = r_j - c_j rounded, the sum
// accumulated over j = 0..ds-1 in order as acc = fma(t, t, acc), the first
// (lowest) k wins ties, and the residual update is an fp32 subtraction.
// Every one of those steps is an IEEE round-to-nearest operation, so the
// codes are reproducible bit for bit on any conforming machine.
//
// Design for sm_100a.  The work is ds-dim distance arithmetic (6 dims at the
// Gemma-2 shape): far too short a contraction for the tensor cores, and the
// fp32 order above is part of the result, so it runs on the FP32 pipes.
// A CTA owns one subspace and a tile of rows; the subspace's level-l
// codebook (K * ds * 4 bytes, 24 KB at the Gemma-2 shape) is staged in shared
// memory, chunk by chunk when it is larger, and read as warp broadcasts.
// Each thread keeps R rows' residuals, best codes and best distances in
// registers, so one codeword read feeds R distance computations.
#include "rq_common.cuh"

namespace rq {

constexpr int kEncThreads = 256;
constexpr int kEncSmemFloats = 12 * 1024;   // 48 KB of codewords per chunk

// DS > 0: ds is a compile-time constant; DS = 0: runtime ds <= 32 (a slow
// path for shapes outside the templates: residuals in local memory).
template <int DS, int R>
__global__ void __launch_bounds__(kEncThreads) encode_kernel(const float *__restrict__ X,
                                                             int64_t N, const float *__restrict__ C,
                                                             int D, int M, int L, int K, int ds_rt,
                                                             uint16_t *__restrict__ codes) {
  constexpr int DSR = DS > 0 ? DS : 32;
  extern __shared__ float cb[];
  const int ds = DS > 0 ? DS : ds_rt;
  const int m = (int)(blockIdx.x % (unsigned)M);
  const int64_t tile = blockIdx.x / (unsigned)M;
  const int64_t row0 = tile * (int64_t)(kEncThreads * R) + threadIdx.x;

  float r[R][DSR];
  int best[R];
#pragma unroll
  for (int q = 0; q < R; ++q) {
    int64_t n = row0 + (int64_t)q * kEncThreads;
    n = n < N ? n : N - 1;                     // rows past the end compute row N-1, unstored
    const float *xr = X + n * D + (int64_t)m * ds;
#pragma unroll
    for (int j = 0; j < DSR; ++j)
      if (DS > 0 || j < ds) r[q][j] = __ldg(xr + j);
  }

  const int kc = kEncSmemFloats / ds < K ? kEncSmemFloats / ds : K;   // codewords per chunk
  for (int l = 0; l < L; ++l) {
    const float *book = C + ((int64_t)m * L + l) * K * ds;
    float bestd[R];
#pragma unroll
    for (int q = 0; q < R; ++q) {
      bestd[q] = __int_as_float(0x7f800000);   // +inf: a NaN distance never wins
      best[q] = 0;
    }
    for (int k0 = 0; k0 < K; k0 += kc) {
      const int nk = K - k0 < kc ? K - k0 : kc;
      __syncthreads();                         // the previous chunk is no longer read
      for (int i = threadIdx.x; i < nk * ds; i += kEncThreads) cb[i] = __ldg(book + (int64_t)k0 * ds + i);
      __syncthreads();
      if constexpr (DS > 0) {
#pragma unroll 4
        for (int k = 0; k < nk; ++k) {
          float c[DSR];
#pragma unroll
          for (int j = 0; j < DSR; ++j) c[j] = cb[k * DSR + j];
#pragma unroll
          for (int q = 0; q < R; ++q) {
            float acc = 0.f;
#pragma unroll
            for (int j = 0; j < DSR; ++j) {
              const float t = __fsub_rn(r[q][j], c[j]);
              acc = __fmaf_rn(t, t, acc);
            }
            if (acc < bestd[q]) {
              bestd[q] = acc;
              best[q] = k0 + k;
            }
          }
        }
      } else {
        for (int k = 0; k < nk; ++k)
#pragma unroll
          for (int q = 0; q < R; ++q) {
            float acc = 0.f;
            for (int j = 0; j < ds; ++j) {
              const float t = __fsub_rn(r[q][j], cb[k * ds + j]);
              acc = __fmaf_rn(t, t, acc);
            }
            if (acc < bestd[q]) {
              bestd[q] = acc;
              best[q] = k0 + k;
            }
          }
      }
    }
#pragma unroll
    for (int q = 0; q < R; ++q) {
      const float *cw = book + (int64_t)best[q] * ds;
#pragma unroll
      for (int j = 0; j < DSR; ++j)
        if (DS > 0 || j < ds) r[q][j] = __fsub_rn(r[q][j], __ldg(cw + j));
      const int64_t n = row0 + (int64_t)q * kEncThreads;
      if (n < N) codes[(n * M + m) * L + l] = (uint16_t)best[q];
    }
  }
}

template <int DS, int R>
cudaError_t encode_launch(const float *X, int64_t N, const float *C, int D, int M, int L, int K,
                          uint16_t *codes, cudaStream_t s) {
  const int ds = D / M;
  const int64_t tiles = (N + kEncThreads * R - 1) / (kEncThreads * R);   // R rows per thread
  const int64_t blocks = tiles * M;
  if (blocks > 0x7fffffffLL) return cudaErrorInvalidValue;
  const int kc = kEncSmemFloats / ds < K ? kEncSmemFloats / ds : K;
  const size_t smem = (size_t)kc * ds * sizeof(float);
  // a plain stream-ordered launch: the rows may come from the kernel before
  encode_kernel<DS, R><<<dim3((unsigned)blocks), dim3(kEncThreads), smem, s>>>(X, N, C, D, M, L,
                                                                               K, ds, codes);
  return cudaGetLastError();
}

cudaError_t launch_encode(const float *X, int64_t N, const float *C, int D, int M, int L, int K,
                          uint16_t *codes, cudaStream_t s) {
  if (N <= 0) return cudaSuccess;
  const int ds = D / M;
  if (ds < 1 || ds > 32) return cudaErrorInvalidValue;
  switch (ds) {
    case 2: return encode_launch<2, 2>(X, N, C, D, M, L, K, codes, s);
    case 4: return encode_launch<4, 2>(X, N, C, D, M, L, K, codes, s);
    case 6: return encode_launch<6, 2>(X, N, C, D, M, L, K, codes, s);
    case 8: return encode_launch<8, 2>(X, N, C, D, M, L, K, codes, s);
    default: return encode_launch<0, 1>(X, N, C, D, M, L, K, codes, s);
  }
}

}  // namespace rq

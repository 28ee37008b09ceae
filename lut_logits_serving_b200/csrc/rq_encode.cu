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
// registers, so one codeword read feeds R distance computations.  The
// specialised kernels (ds 2, 4, 6, 8) work on two codewords at once with the
// packed fp32x2 subtract and fma of sm_100 (each lane an ordinary rn fp32
// operation, so the results are those of the scalar definition): the chunk
// is stored in shared memory as interleaved codeword pairs, [k/2][j][2], and
// a 16-byte load gives two dims of both codewords; the two distances are
// compared in index order, so ties still go to the lower index.
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

__device__ __forceinline__ unsigned long long f2_pack(float lo, float hi) {
  unsigned long long r;
  asm("mov.b64 %0, {%1, %2};" : "=l"(r) : "f"(lo), "f"(hi));
  return r;
}

__device__ __forceinline__ void f2_unpack(unsigned long long v, float &lo, float &hi) {
  asm("mov.b64 {%0, %1}, %2;" : "=f"(lo), "=f"(hi) : "l"(v));
}

// lane-wise rn fp32 a - b and a * b + c (no flush to zero)
__device__ __forceinline__ unsigned long long f2_sub(unsigned long long a, unsigned long long b) {
  unsigned long long d;
  asm("sub.rn.f32x2 %0, %1, %2;" : "=l"(d) : "l"(a), "l"(b));
  return d;
}

__device__ __forceinline__ unsigned long long f2_fma(unsigned long long a, unsigned long long b,
                                                     unsigned long long c) {
  unsigned long long d;
  asm("fma.rn.f32x2 %0, %1, %2, %3;" : "=l"(d) : "l"(a), "l"(b), "l"(c));
  return d;
}

template <int DS, int R>
__global__ void __launch_bounds__(kEncThreads) encode_pair_kernel(
    const float *__restrict__ X, int64_t N, const float *__restrict__ C, int D, int M, int L,
    int K, uint16_t *__restrict__ codes) {
  static_assert(DS % 2 == 0, "16-byte pair loads need an even ds");
  extern __shared__ __align__(16) float cbp[];  // [kc/2][DS][2]
  float *cb = cbp;
  const int m = (int)(blockIdx.x % (unsigned)M);
  const int64_t tile = blockIdx.x / (unsigned)M;
  const int64_t row0 = tile * (int64_t)(kEncThreads * R) + threadIdx.x;

  float r[R][DS];
#pragma unroll
  for (int q = 0; q < R; ++q) {
    int64_t n = row0 + (int64_t)q * kEncThreads;
    n = n < N ? n : N - 1;                     // rows past the end compute row N-1, unstored
    const float *xr = X + n * D + (int64_t)m * DS;
#pragma unroll
    for (int j = 0; j < DS; ++j) r[q][j] = __ldg(xr + j);
  }

  constexpr int kc = (kEncSmemFloats / DS) & ~1;   // codewords per chunk, even
  const float qnan = __int_as_float(0x7fffffff);
  for (int l = 0; l < L; ++l) {
    const float *book = C + ((int64_t)m * L + l) * K * DS;
    unsigned long long rr[R][DS];              // {r_j, r_j}
    // Best distance as its bit pattern: a distance is +0, positive, +inf or
    // NaN, and for those the signed-integer order of the bits is the float
    // order with NaN above +inf, so starting from +inf a NaN never wins.
    // The compares and selects then run on the integer pipe, beside the
    // FP32 pipe that computes the distances.
    int bestd[R];
    int best[R];
#pragma unroll
    for (int q = 0; q < R; ++q) {
#pragma unroll
      for (int j = 0; j < DS; ++j) rr[q][j] = f2_pack(r[q][j], r[q][j]);
      bestd[q] = 0x7f800000;                   // +inf
      best[q] = 0;
    }
    for (int k0 = 0; k0 < K; k0 += kc) {
      const int nk = K - k0 < kc ? K - k0 : kc;
      const int npair = (nk + 1) / 2;
      __syncthreads();                         // the previous chunk is no longer read
      // codeword k, dim j -> [k/2][j][k&1]; an odd chunk's missing partner
      // is NaN, whose distance never wins
      for (int i = threadIdx.x; i < 2 * npair * DS; i += kEncThreads) {
        const int k = i / DS, j = i - k * DS;
        cb[((k >> 1) * DS + j) * 2 + (k & 1)] =
            k < nk ? __ldg(book + (int64_t)(k0 + k) * DS + j) : qnan;
      }
      __syncthreads();
      const ulonglong2 *cp = reinterpret_cast<const ulonglong2 *>(cb);
#pragma unroll 2
      for (int p = 0; p < npair; ++p) {
        unsigned long long c2[DS];
#pragma unroll
        for (int j2 = 0; j2 < DS / 2; ++j2) {
          const ulonglong2 v = cp[p * (DS / 2) + j2];
          c2[2 * j2] = v.x;
          c2[2 * j2 + 1] = v.y;
        }
        const int k = k0 + 2 * p;
#pragma unroll
        for (int q = 0; q < R; ++q) {
          unsigned long long acc = 0ull;
#pragma unroll
          for (int j = 0; j < DS; ++j) {
            const unsigned long long t = f2_sub(rr[q][j], c2[j]);
            acc = f2_fma(t, t, acc);
          }
          // codeword k first, then k + 1: ties keep the lower index
          const int d0 = (int)(acc & 0xffffffffull), d1 = (int)(acc >> 32);
          if (d0 < bestd[q]) {
            bestd[q] = d0;
            best[q] = k;
          }
          if (d1 < bestd[q]) {
            bestd[q] = d1;
            best[q] = k + 1;
          }
        }
      }
    }
#pragma unroll
    for (int q = 0; q < R; ++q) {
      const float *cw = book + (int64_t)best[q] * DS;
#pragma unroll
      for (int j = 0; j < DS; ++j) r[q][j] = __fsub_rn(r[q][j], __ldg(cw + j));
      const int64_t n = row0 + (int64_t)q * kEncThreads;
      if (n < N) codes[(n * M + m) * L + l] = (uint16_t)best[q];
    }
  }
}

template <int DS, int R>
cudaError_t encode_pair_launch(const float *X, int64_t N, const float *C, int D, int M, int L,
                               int K, uint16_t *codes, cudaStream_t s) {
  const int64_t tiles = (N + kEncThreads * R - 1) / (kEncThreads * R);   // R rows per thread
  const int64_t blocks = tiles * M;
  if (blocks > 0x7fffffffLL) return cudaErrorInvalidValue;
  constexpr int kc = (kEncSmemFloats / DS) & ~1;
  const int npair = ((K < kc ? K : kc) + 1) / 2;   // an odd chunk's last pair has a NaN partner
  const size_t smem = (size_t)npair * 2 * DS * sizeof(float);   // <= kEncSmemFloats floats
  encode_pair_kernel<DS, R><<<dim3((unsigned)blocks), dim3(kEncThreads), smem, s>>>(
      X, N, C, D, M, L, K, codes);
  return cudaGetLastError();
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
    case 2: return encode_pair_launch<2, 4>(X, N, C, D, M, L, K, codes, s);
    case 4: return encode_pair_launch<4, 4>(X, N, C, D, M, L, K, codes, s);
    case 6: return encode_pair_launch<6, 4>(X, N, C, D, M, L, K, codes, s);
    case 8: return encode_pair_launch<8, 4>(X, N, C, D, M, L, K, codes, s);
    default: return encode_launch<0, 1>(X, N, C, D, M, L, K, codes, s);
  }
}

}  // namespace rq

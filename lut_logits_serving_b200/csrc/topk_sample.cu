// topk_sample.cu -- top-k of the softcapped logits and a temperature draw
// among them (generation beyond greedy argmax).
//
// The pages decode greedily and state no sampler ("Gemma-2-2B combined
// RQ+NF4", closing note on generation).  The plain reading implemented here:
//   * top-k: the k largest logits of each token row, descending, the lower
//     vocabulary index first among equal values;
//   * draw: weights w_i = exp((y_i - y_0) / T) over the sorted top-k, the
//     token is the first i whose running sum exceeds u * (sum of all w),
//     in fp64; T <= 0 or k = 1 is greedy;
//   * u in [0, 1): the top 53 bits of word 0 of Philox4x64-10 (Salmon et al.,
//     "Parallel random numbers: as easy as 1, 2, 3", SC'11) for counter
//     (step, row, 0, 0) and key (seed, 0), times 2^-53.
//
// Design for sm_100a.  The logits of a token (1 MB at V = 256000) are read
// once.  Each value becomes a 64-bit key: the order-preserving transform of
// its fp32 bits (high word) and the complement of its index (low word), so
// that one unsigned compare orders by value, then by lower index.
//   stage 1 -- one CTA per 2048-logit slice and token sorts its keys with a
//              bitonic network in shared memory and keeps the first KP
//              (k rounded up to a power of two);
//   stage 2 -- a CTA loads G such lists and merges them pairwise in shared
//              memory: the elementwise max of list A and reversed list B is
//              a bitonic sequence holding the top KP of both, and log2(KP)
//              half-cleaner passes sort it.  Launches repeat until one list
//              per token is left; that last launch also writes the outputs
//              and makes the draw (one warp: lane-chunked sums, a warp scan).
#include <cfloat>
#include <climits>

#include "rq_common.cuh"

namespace rq {

constexpr int kTopkSlice = 2048;         // logits per stage-1 CTA
constexpr int kTopkThreads = 1024;
constexpr int kTopkMergeSmem = 96 * 1024;

__device__ __forceinline__ unsigned long long topk_key(float v, int64_t idx) {
  unsigned b = __float_as_uint(v);
  if (b == 0x80000000u) b = 0u;          // -0 orders as +0
  b = (b & 0x80000000u) ? ~b : (b | 0x80000000u);
  return ((unsigned long long)b << 32) | (unsigned long long)(0xFFFFFFFFu - (unsigned)idx);
}

__device__ __forceinline__ float topk_value(unsigned long long key) {
  const unsigned b = (unsigned)(key >> 32);
  return __uint_as_float((b & 0x80000000u) ? (b ^ 0x80000000u) : ~b);
}

__device__ __forceinline__ int topk_index(unsigned long long key) {
  return (int)(0xFFFFFFFFu - (unsigned)(key & 0xFFFFFFFFull));
}

// Philox4x64-10: two 64 x 64 -> 128-bit products per round with the
// published multipliers, key bumped by the published Weyl constants.
__device__ double philox_uniform(unsigned long long seed, unsigned long long step,
                                 unsigned long long row) {
  unsigned long long c0 = step, c1 = row, c2 = 0ull, c3 = 0ull, k0 = seed, k1 = 0ull;
#pragma unroll
  for (int r = 0; r < 10; ++r) {
    const unsigned long long a = 0xD2E7470EE14C6C93ull, b = 0xCA5A826395121157ull;
    const unsigned long long hi0 = __umul64hi(c0, a), lo0 = c0 * a;
    const unsigned long long hi1 = __umul64hi(c2, b), lo1 = c2 * b;
    const unsigned long long n0 = hi1 ^ c1 ^ k0, n2 = hi0 ^ c3 ^ k1;
    c0 = n0;
    c1 = lo1;
    c2 = n2;
    c3 = lo0;
    k0 += 0x9E3779B97F4A7C15ull;
    k1 += 0xBB67AE8584CAA73Bull;
  }
  return (double)(c0 >> 11) * (1.0 / 9007199254740992.0);
}

// Stage 1: grid (nblk, B).  Keys of slice blockIdx.x sorted descending;
// the first KP go to lists[b][blk][0..KP).  Keys past V are 0 (below every
// real key: the smallest real key has a nonzero high word).
__global__ void __launch_bounds__(kTopkThreads) topk_slice_kernel(const float *__restrict__ y,
                                                                 int64_t V, int KP,
                                                                 unsigned long long *lists) {
  __shared__ unsigned long long sk[kTopkSlice];
  griddep_wait();
  const int b = blockIdx.y;
  const int64_t v0 = (int64_t)blockIdx.x * kTopkSlice;
  const float *row = y + (int64_t)b * V;
  for (int i = threadIdx.x; i < kTopkSlice; i += kTopkThreads) {
    const int64_t v = v0 + i;
    sk[i] = v < V ? topk_key(__ldg(row + v), v) : 0ull;
  }
  for (int size = 2; size <= kTopkSlice; size <<= 1)
    for (int stride = size >> 1; stride > 0; stride >>= 1) {
      __syncthreads();
      for (int t = threadIdx.x; t < kTopkSlice / 2; t += kTopkThreads) {
        const int i = 2 * t - (t & (stride - 1)), j = i + stride;
        const bool desc = (i & size) == 0;  // the last merge (size = slice) is descending
        const unsigned long long a = sk[i], c = sk[j];
        if (desc ? a < c : a > c) {
          sk[i] = c;
          sk[j] = a;
        }
      }
    }
  __syncthreads();
  griddep_launch_dependents();
  unsigned long long *out = lists + ((int64_t)b * gridDim.x + blockIdx.x) * KP;
  for (int i = threadIdx.x; i < KP; i += kTopkThreads) out[i] = sk[i];
}

struct TopkOut {
  int k;
  double temperature;
  unsigned long long seed, step;
  float *val;      // [B][k] or null
  int32_t *idx;    // [B][k] or null
  int32_t *token;  // [B] or null
};

// Stage 2: grid (ceil(nl / G), B).  G lists of KP keys (sorted descending)
// merged into one; with `fin` (one CTA per token left) the outputs and the
// draw are made here.
__global__ void __launch_bounds__(kTopkThreads) topk_merge_kernel(
    const unsigned long long *__restrict__ in, int nl, int KP, int G,
    unsigned long long *out, int fin, TopkOut o) {
  extern __shared__ unsigned long long sm[];   // [G][KP]
  griddep_wait();
  const int b = blockIdx.y;
  const int l0 = blockIdx.x * G;
  for (int i = threadIdx.x; i < G * KP; i += kTopkThreads) {
    const int l = i / KP;
    sm[i] = l0 + l < nl ? in[((int64_t)b * nl + l0 + l) * KP + (i - l * KP)] : 0ull;
  }
  for (int w = 1; w < G; w <<= 1) {
    const int npairs = G / (2 * w);
    __syncthreads();
    // A[i] = max(A[i], B[KP-1-i]): the top KP of A and B, as a bitonic sequence
    for (int t = threadIdx.x; t < npairs * KP; t += kTopkThreads) {
      const int p = t / KP, i = t - p * KP;
      unsigned long long *A = sm + (int64_t)(2 * w * p) * KP;
      const unsigned long long *Bl = A + (int64_t)w * KP;
      const unsigned long long x = A[i], z = Bl[KP - 1 - i];
      A[i] = x > z ? x : z;
    }
    for (int stride = KP >> 1; stride > 0; stride >>= 1) {
      __syncthreads();
      for (int t = threadIdx.x; t < npairs * (KP / 2); t += kTopkThreads) {
        const int p = t / (KP / 2), r = t - p * (KP / 2);
        unsigned long long *A = sm + (int64_t)(2 * w * p) * KP;
        const int i = 2 * r - (r & (stride - 1)), j = i + stride;
        const unsigned long long x = A[i], z = A[j];
        if (x < z) {
          A[i] = z;
          A[j] = x;
        }
      }
    }
  }
  __syncthreads();
  griddep_launch_dependents();
  if (!fin) {
    unsigned long long *dst = out + ((int64_t)b * gridDim.x + blockIdx.x) * KP;
    for (int i = threadIdx.x; i < KP; i += kTopkThreads) dst[i] = sm[i];
    return;
  }
  const int k = o.k;
  for (int i = threadIdx.x; i < k; i += kTopkThreads) {
    if (o.val) o.val[(int64_t)b * k + i] = topk_value(sm[i]);
    if (o.idx) o.idx[(int64_t)b * k + i] = topk_index(sm[i]);
  }
  if (o.token == nullptr || threadIdx.x >= 32) return;
  const int lane = threadIdx.x;
  if (k == 1 || !(o.temperature > 0.0)) {
    if (lane == 0) o.token[b] = topk_index(sm[0]);
    return;
  }
  const double y0 = (double)topk_value(sm[0]);
  const int per = (k + 31) / 32;
  const int lo = lane * per, hi = min(k, lo + per);
  double s = 0.0;
  for (int i = lo; i < hi; ++i) s += exp(((double)topk_value(sm[i]) - y0) / o.temperature);
  double incl = s;                        // inclusive scan of the lane sums
#pragma unroll
  for (int d = 1; d < 32; d <<= 1) {
    const double t = __shfl_up_sync(0xffffffffu, incl, d);
    if (lane >= d) incl += t;
  }
  const double total = __shfl_sync(0xffffffffu, incl, 31);
  double cum = __shfl_up_sync(0xffffffffu, incl, 1);
  if (lane == 0) cum = 0.0;
  const double target = philox_uniform(o.seed, o.step, (unsigned long long)b) * total;
  int pick = INT_MAX;
  for (int i = lo; i < hi; ++i) {
    cum += exp(((double)topk_value(sm[i]) - y0) / o.temperature);
    if (cum > target) {
      pick = i;
      break;
    }
  }
#pragma unroll
  for (int d = 16; d > 0; d >>= 1) pick = min(pick, __shfl_xor_sync(0xffffffffu, pick, d));
  if (lane == 0) o.token[b] = topk_index(sm[pick == INT_MAX ? k - 1 : pick]);
}

int topk_pow2(int k) {
  int p = 1;
  while (p < k) p <<= 1;
  return p;
}

static int topk_max_group(int KP) {
  int g = 1;
  while (2 * g * KP * (int)sizeof(unsigned long long) <= kTopkMergeSmem) g <<= 1;
  return g;
}

size_t topk_workspace_bytes(int64_t V, int B, int k) {
  const int KP = topk_pow2(k);
  const int64_t nblk = (V + kTopkSlice - 1) / kTopkSlice;
  const int G = topk_max_group(KP);
  const int64_t n2 = (nblk + G - 1) / G;
  const size_t a = (size_t)B * nblk * KP * sizeof(unsigned long long);
  const size_t b = (size_t)B * (n2 > 1 ? n2 : 1) * KP * sizeof(unsigned long long);
  return align_up((int64_t)a, 256) + align_up((int64_t)b, 256);
}

cudaError_t launch_topk_sample(const float *logits, int64_t V, int B, int k, double temperature,
                               unsigned long long seed, unsigned long long step, float *val,
                               int32_t *idx, int32_t *token, void *ws, cudaStream_t s) {
  const int KP = topk_pow2(k);
  const int64_t nblk = (V + kTopkSlice - 1) / kTopkSlice;
  if (nblk > 0x7fffffffLL || B > 65535) return cudaErrorInvalidValue;
  const int G = topk_max_group(KP);
  unsigned long long *bufA = static_cast<unsigned long long *>(ws);
  unsigned long long *bufB = reinterpret_cast<unsigned long long *>(
      static_cast<unsigned char *>(ws) +
      align_up((int64_t)B * nblk * KP * (int64_t)sizeof(unsigned long long), 256));
  static bool attr[128] = {};
  int dev = 0;
  cudaGetDevice(&dev);
  if (dev < 128 && !attr[dev]) {
    cudaError_t e = cudaFuncSetAttribute(topk_merge_kernel,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         kTopkMergeSmem);
    if (e != cudaSuccess) return e;
    attr[dev] = true;
  }
  cudaError_t e = pdl_launch(topk_slice_kernel, dim3((unsigned)nblk, (unsigned)B),
                             dim3(kTopkThreads), 0, s, logits, V, KP, bufA);
  if (e != cudaSuccess) return e;
  TopkOut o{k, temperature, seed, step, val, idx, token};
  int nl = (int)nblk;
  const unsigned long long *in = bufA;
  unsigned long long *out = bufB;
  while (true) {
    int g = 1;
    while (g < nl && g < G) g <<= 1;
    const int nout = (nl + g - 1) / g;
    const int fin = nout == 1;
    e = pdl_launch(topk_merge_kernel, dim3((unsigned)nout, (unsigned)B), dim3(kTopkThreads),
                   (size_t)g * KP * sizeof(unsigned long long), s, in, nl, KP, g, out, fin, o);
    if (e != cudaSuccess || fin) return e;
    nl = nout;
    unsigned long long *t = const_cast<unsigned long long *>(in);
    in = out;
    out = t;
  }
}

}  // namespace rq

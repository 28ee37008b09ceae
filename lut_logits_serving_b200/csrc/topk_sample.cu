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
// Design for sm_100a: a radix select, then a sort of the few survivors.
// Each logit's fp32 bits map to an order-preserving 32-bit word (ord), and
// the 64-bit key (ord, complement of the index) orders by value, then lower
// index, under one unsigned compare.
//   pass 1 -- a grid of CTAs histograms the top 12 bits of ord of every
//             logit (shared-memory counts, then one global add per occupied
//             bin);
//   pass 2 -- the same CTAs find the threshold bin t (the highest bin whose
//             suffix count reaches k) and append the keys of bin >= t to a
//             candidate list (about k to 3k keys for logit-like values).  The
//             last CTA of each token (a completion counter) sorts the
//             candidates with a bitonic network in shared memory, writes the
//             top k and makes the draw (one warp: lane-chunked fp64 sums and a
//             warp scan).  When bin t holds more keys than the list (heavy
//             ties), the last CTA instead refines the threshold exactly over
//             the row (two more 10-bit histograms) and takes the keys above it
//             plus the tied ones in index order.
#include <cfloat>
#include <climits>

#include "rq_common.cuh"

namespace rq {

constexpr int kTopkThreads = 512;
constexpr int kTopkBins = 4096;            // top 12 bits of ord
constexpr int kTopkCap = 8192;             // candidate keys per token
constexpr int kTopkMaxK = 1024;

struct TopkWs {
  unsigned *hist;              // [B][kTopkBins]       zeroed per call
  unsigned *cnt;               // [B] candidates        zeroed per call
  unsigned *done;              // [B] finished CTAs     zeroed per call
  unsigned long long *cand;    // [B][kTopkCap]
};

struct TopkOut {
  int k;
  double temperature;
  unsigned long long seed, step;
  float *val;      // [B][k] or null
  int32_t *idx;    // [B][k] or null
  int32_t *token;  // [B] or null
};

__device__ __forceinline__ unsigned topk_ord(float v) {
  unsigned b = __float_as_uint(v);
  if (b == 0x80000000u) b = 0u;          // -0 orders as +0
  return (b & 0x80000000u) ? ~b : (b | 0x80000000u);
}

__device__ __forceinline__ unsigned long long topk_key(unsigned ord, int64_t idx) {
  return ((unsigned long long)ord << 32) | (unsigned long long)(0xFFFFFFFFu - (unsigned)idx);
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

// This CTA's range of row elements: nb CTAs split V evenly.
__device__ __forceinline__ void topk_range(int64_t V, int64_t &v0, int64_t &v1) {
  v0 = V * blockIdx.x / gridDim.x;
  v1 = V * (blockIdx.x + 1) / gridDim.x;
}

// Pass 1: grid (nb, B).
__global__ void __launch_bounds__(kTopkThreads) topk_hist_kernel(const float *__restrict__ y,
                                                                int64_t V, TopkWs w) {
  __shared__ unsigned h[kTopkBins];
  for (int i = threadIdx.x; i < kTopkBins; i += kTopkThreads) h[i] = 0u;
  griddep_wait();
  __syncthreads();
  const int b = blockIdx.y;
  int64_t v0, v1;
  topk_range(V, v0, v1);
  const float *row = y + (int64_t)b * V;
  for (int64_t v = v0 + threadIdx.x; v < v1; v += kTopkThreads)
    atomicAdd(&h[topk_ord(__ldg(row + v)) >> 20], 1u);
  __syncthreads();
  griddep_launch_dependents();
  unsigned *H = w.hist + (int64_t)b * kTopkBins;
  for (int i = threadIdx.x; i < kTopkBins; i += kTopkThreads)
    if (h[i]) atomicAdd(&H[i], h[i]);
}

// Block-wide: of the counts c[0..n) (n = 8 * kTopkThreads at most, given as
// 8 per thread in `mine`), the highest index t whose suffix sum reaches
// `need`, that suffix sum (ge) and the sum above t (gt).  Every thread gets
// the result.  need >= 1 and the total reaches it.
struct SuffixPick {
  int t;
  unsigned ge, gt;
};

template <int PER>
__device__ SuffixPick suffix_pick(const unsigned (&mine)[PER], unsigned need, unsigned *scr) {
  // thread i owns entries [i*PER, (i+1)*PER); suffix order is thread order reversed
  unsigned s = 0;
#pragma unroll
  for (int j = 0; j < PER; ++j) s += mine[j];
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  // exclusive suffix sum over threads: sum of threads with a higher index
  unsigned incl = s;   // inclusive suffix within the warp (lanes >= this one)
#pragma unroll
  for (int d = 1; d < 32; d <<= 1) {
    const unsigned t = __shfl_down_sync(0xffffffffu, incl, d);
    if (lane + d < 32) incl += t;
  }
  if (lane == 0) scr[warp] = incl;       // warp total
  __syncthreads();
  unsigned above_warp = 0;
  for (int w2 = warp + 1; w2 < kTopkThreads / 32; ++w2) above_warp += scr[w2];
  const unsigned above = above_warp + incl - s;   // entries after this thread's
  __syncthreads();
  // the thread whose range holds t: above < need <= above + s
  if (above < need && need <= above + s) {
    unsigned acc = above;
    for (int j = PER - 1; j >= 0; --j) {
      if (acc + mine[j] >= need) {
        scr[0] = (unsigned)(threadIdx.x * PER + j);
        scr[1] = acc + mine[j];
        scr[2] = acc;
        break;
      }
      acc += mine[j];
    }
  }
  __syncthreads();
  SuffixPick r{(int)scr[0], scr[1], scr[2]};
  __syncthreads();
  return r;
}

// Bitonic sort of n (a power of two) keys in shared memory, descending.
__device__ void sort_desc(unsigned long long *sk, int n) {
  for (int size = 2; size <= n; size <<= 1)
    for (int stride = size >> 1; stride > 0; stride >>= 1) {
      __syncthreads();
      for (int t = threadIdx.x; t < n / 2; t += kTopkThreads) {
        const int i = 2 * t - (t & (stride - 1)), j = i + stride;
        const bool desc = (i & size) == 0;
        const unsigned long long a = sk[i], c = sk[j];
        if (desc ? a < c : a > c) {
          sk[i] = c;
          sk[j] = a;
        }
      }
    }
  __syncthreads();
}

// Outputs of token b from its top keys sk[0..k), sorted descending.
__device__ void topk_finish(const unsigned long long *sk, int b, const TopkOut &o) {
  const int k = o.k;
  for (int i = threadIdx.x; i < k; i += kTopkThreads) {
    if (o.val) o.val[(int64_t)b * k + i] = topk_value(sk[i]);
    if (o.idx) o.idx[(int64_t)b * k + i] = topk_index(sk[i]);
  }
  if (o.token == nullptr || threadIdx.x >= 32) return;
  const int lane = threadIdx.x;
  if (k == 1 || !(o.temperature > 0.0)) {
    if (lane == 0) o.token[b] = topk_index(sk[0]);
    return;
  }
  const double y0 = (double)topk_value(sk[0]);
  const int per = (k + 31) / 32;
  const int lo = lane * per, hi = min(k, lo + per);
  double s = 0.0;
  for (int i = lo; i < hi; ++i) s += exp(((double)topk_value(sk[i]) - y0) / o.temperature);
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
    cum += exp(((double)topk_value(sk[i]) - y0) / o.temperature);
    if (cum > target) {
      pick = i;
      break;
    }
  }
#pragma unroll
  for (int d = 16; d > 0; d >>= 1) pick = min(pick, __shfl_xor_sync(0xffffffffu, pick, d));
  if (lane == 0) o.token[b] = topk_index(sk[pick == INT_MAX ? k - 1 : pick]);
}

// Heavy ties: the exact k-th key over the whole row by one CTA.  `bin` is
// the threshold bin of the top 12 bits and `gt` the count above it.
__device__ void topk_exact_row(const float *__restrict__ row, int64_t V, unsigned bin,
                               unsigned gt, unsigned long long *sk, unsigned *scr,
                               unsigned *h, int b, const TopkOut &o) {
  const unsigned k = (unsigned)o.k;
  // refine ord below the top 12 bits: bits 19..10, then 9..0
  unsigned prefix = bin, shift = 20, above = gt;
  for (int level = 0; level < 2; ++level) {
    const unsigned sub = 10, nsub = 1u << sub;
    for (unsigned i = threadIdx.x; i < nsub; i += kTopkThreads) h[i] = 0u;
    __syncthreads();
    for (int64_t v = threadIdx.x; v < V; v += kTopkThreads) {
      const unsigned ord = topk_ord(__ldg(row + v));
      if ((ord >> shift) == prefix) atomicAdd(&h[(ord >> (shift - sub)) & (nsub - 1)], 1u);
    }
    __syncthreads();
    unsigned mine[2] = {h[2 * threadIdx.x], h[2 * threadIdx.x + 1]};
    const SuffixPick p = suffix_pick<2>(mine, k - above, scr);
    prefix = (prefix << sub) | (unsigned)p.t;
    above += p.gt;
    shift -= sub;
  }
  // prefix is now the full ord of the k-th largest value; `above` values
  // exceed it and k - above of its copies are taken in index order
  const unsigned tau = prefix;
  const unsigned need_eq = k - above;
  if (threadIdx.x == 0) {
    scr[0] = 0u;    // keys placed
    scr[1] = 0u;    // ties taken so far
  }
  __syncthreads();
  for (int64_t base = 0; base < V; base += kTopkThreads) {
    const int64_t v = base + threadIdx.x;
    const unsigned ord = v < V ? topk_ord(__ldg(row + v)) : 0u;
    const bool gtv = v < V && ord > tau, eqv = v < V && ord == tau;
    if (gtv) sk[atomicAdd(&scr[0], 1u)] = topk_key(ord, v);
    // ties in index order: rank among this tile's ties, offset by earlier tiles
    const unsigned ball = __ballot_sync(0xffffffffu, eqv);
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    if (lane == 0) h[warp] = __popc(ball);
    __syncthreads();
    unsigned before = scr[1];
    for (int w2 = 0; w2 < warp; ++w2) before += h[w2];
    before += __popc(ball & ((1u << lane) - 1u));
    if (eqv && before < need_eq) sk[atomicAdd(&scr[0], 1u)] = topk_key(ord, v);
    __syncthreads();
    if (threadIdx.x == 0)
      for (int w2 = 0; w2 < kTopkThreads / 32; ++w2) scr[1] += h[w2];
    __syncthreads();
  }
  int n = 1;
  while (n < (int)k) n <<= 1;
  for (int i = (int)k + threadIdx.x; i < n; i += kTopkThreads) sk[i] = 0ull;
  sort_desc(sk, n);
  topk_finish(sk, b, o);
}

// Pass 2: grid (nb, B); dynamic shared memory kTopkCap keys.
__global__ void __launch_bounds__(kTopkThreads) topk_gather_kernel(const float *__restrict__ y,
                                                                  int64_t V, TopkWs w,
                                                                  TopkOut o) {
  extern __shared__ unsigned long long sk[];   // [kTopkCap]
  __shared__ unsigned scr[kTopkThreads / 32 + 4];
  __shared__ unsigned h[1024];
  __shared__ int last;
  griddep_wait();
  const int b = blockIdx.y;
  const unsigned *H = w.hist + (int64_t)b * kTopkBins;
  constexpr int PER = kTopkBins / kTopkThreads;
  unsigned mine[PER];
#pragma unroll
  for (int j = 0; j < PER; ++j) mine[j] = H[threadIdx.x * PER + j];
  const SuffixPick p = suffix_pick<PER>(mine, (unsigned)o.k, scr);
  const bool fits = p.ge <= (unsigned)kTopkCap;
  const float *row = y + (int64_t)b * V;
  if (fits) {
    int64_t v0, v1;
    topk_range(V, v0, v1);
    unsigned long long *cand = w.cand + (int64_t)b * kTopkCap;
    for (int64_t v = v0 + threadIdx.x; v < v1; v += kTopkThreads) {
      const unsigned ord = topk_ord(__ldg(row + v));
      if ((int)(ord >> 20) >= p.t) cand[atomicAdd(&w.cnt[b], 1u)] = topk_key(ord, v);
    }
  }
  __threadfence();
  __syncthreads();
  if (threadIdx.x == 0) last = atomicAdd(&w.done[b], 1u) == gridDim.x - 1;
  __syncthreads();
  griddep_launch_dependents();
  if (!last) return;
  __threadfence();
  if (fits) {
    const unsigned long long *cand = w.cand + (int64_t)b * kTopkCap;
    int n = 1;
    while (n < (int)p.ge) n <<= 1;
    for (int i = threadIdx.x; i < n; i += kTopkThreads)
      sk[i] = i < (int)p.ge ? __ldcg(cand + i) : 0ull;
    sort_desc(sk, n);
    topk_finish(sk, b, o);
  } else {
    topk_exact_row(row, V, (unsigned)p.t, p.gt, sk, scr, h, b, o);
  }
}

size_t topk_workspace_bytes(int64_t V, int B, int k) {
  (void)V;
  (void)k;
  const size_t counters = (size_t)B * (kTopkBins + 2) * sizeof(unsigned);
  return align_up((int64_t)counters, 256) + (size_t)B * kTopkCap * sizeof(unsigned long long);
}

static int topk_blocks(int64_t V, int B, int sms) {
  int64_t nb = (2 * (int64_t)sms + B - 1) / B;           // about two CTAs per SM in all
  const int64_t most = (V + 1023) / 1024;               // at least ~1024 logits per CTA
  if (nb > most) nb = most;
  return (int)(nb < 1 ? 1 : nb);
}

cudaError_t launch_topk_sample(const float *logits, int64_t V, int B, int k, double temperature,
                               unsigned long long seed, unsigned long long step, float *val,
                               int32_t *idx, int32_t *token, void *ws, cudaStream_t s) {
  if (B > 65535 || k < 1 || k > kTopkMaxK) return cudaErrorInvalidValue;
  TopkWs w;
  w.hist = static_cast<unsigned *>(ws);
  w.cnt = w.hist + (size_t)B * kTopkBins;
  w.done = w.cnt + B;
  w.cand = reinterpret_cast<unsigned long long *>(
      static_cast<unsigned char *>(ws) +
      align_up((int64_t)B * (kTopkBins + 2) * (int64_t)sizeof(unsigned), 256));
  int dev = 0, sms = 148;
  cudaGetDevice(&dev);
  cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  const size_t smem = (size_t)kTopkCap * sizeof(unsigned long long);
  {
    cudaError_t e =
        ensure_smem_limit(reinterpret_cast<const void *>(&topk_gather_kernel), dev, smem);
    if (e != cudaSuccess) return e;
  }
  cudaError_t e = cudaMemsetAsync(w.hist, 0, (size_t)B * (kTopkBins + 2) * sizeof(unsigned), s);
  if (e != cudaSuccess) return e;
  const dim3 grid((unsigned)topk_blocks(V, B, sms), (unsigned)B);
  e = pdl_launch(topk_hist_kernel, grid, dim3(kTopkThreads), 0, s, logits, V, w);
  if (e != cudaSuccess) return e;
  TopkOut o{k, temperature, seed, step, val, idx, token};
  return pdl_launch(topk_gather_kernel, grid, dim3(kTopkThreads), smem, s, logits, V, w, o);
}

}  // namespace rq

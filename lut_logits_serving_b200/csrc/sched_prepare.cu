// sched_prepare.cu -- the bank-scheduled code layout (RQ_CODES_SCHED).
//
// Not from the pages: a layout of this library for the lookup+sum logits
// pass ("Gemma-2 runtime compression: NF4 + LUT serving", LUT section).  In
// the batch-1 pass a warp handles 32 rows x one 32-pair chunk (one lane per
// row), one table lookup per lane per step, from a shared-
// memory table whose bank for code c is c mod 32.  A step costs as many
// shared-memory passes as its most repeated bank; with the codes in their
// natural order that is ~3.5 for random codes.  Here each lane's 32 codes
// are reordered so that every step is, as far as possible, a matching of
// lanes to distinct banks: step by step, a maximum bipartite matching
// (augmenting paths, Kuhn's method) between the lanes and the banks of
// their remaining codes, grown from the banks with the most codes left (the
// sets of banks a matching can cover form a transversal matroid, so that
// greedy order covers the heaviest banks); a lane left unmatched takes the
// remaining code whose bank is least used in that step, heaviest first.
// Any order gives the same logits up to fp32 summation order; only the
// speed depends on it.
//
// Entry format: (i << s) | c, i = pair position in the 32-pair chunk,
// c = code, 2^s = the table stride (the smallest power of two >= K, at least
// 32): for tables of that stride laid out back to back it is the word offset
// of the table entry, and its bank (entry mod 32) is the code's.  Layout:
// chunk-major [P/32][V][32], so the 32-pair slice that one CTA of the
// batch-1 pass streams is contiguous.
#include "rq_common.cuh"

namespace rq {

constexpr int kSchedThreads = 16;   // one problem per thread, state in smem

__global__ void __launch_bounds__(kSchedThreads) prepare_sched_kernel(
    const uint16_t *__restrict__ codes, int64_t V, int P, int sh, uint16_t *__restrict__ out,
    unsigned long long *stats) {
  __shared__ uint16_t s_code[kSchedThreads][32][32];   // codes of each lane (row)
  __shared__ uint32_t s_lmask[kSchedThreads][32];      // per bank: lanes with unused codes in it
  __shared__ int8_t s_lbank[kSchedThreads][32];        // lane -> matched bank
  const int T = threadIdx.x;
  uint16_t(*cd)[32] = s_code[T];
  uint32_t *bm = s_lmask[T];
  int8_t *lbank = s_lbank[T];

  const int nch = P / 32;
  const int64_t nrb = (V + 31) / 32;
  const int64_t prob = (int64_t)blockIdx.x * kSchedThreads + T;
  if (prob >= nrb * nch) return;
  const int64_t rb = prob / nch;
  const int c = (int)(prob % nch);

  uint32_t present = 0;
  uint32_t used[32];
  for (int ln = 0; ln < 32; ++ln) {
    const int64_t row = rb * 32 + ln;
    used[ln] = 0;
    if (row < V) {
      present |= 1u << ln;
      const uint16_t *src = codes + row * P + c * 32;
      for (int k = 0; k < 32; ++k) cd[ln][k] = src[k] & ((1u << sh) - 1u);
    }
  }

  unsigned long long passes = 0;
  for (int step = 0; step < 32; ++step) {
    // per bank: lanes holding an unused code in it, and how many such codes
    int deg[32];
    for (int b = 0; b < 32; ++b) {
      bm[b] = 0u;
      deg[b] = 0;
    }
    for (int ln = 0; ln < 32; ++ln) {
      lbank[ln] = -1;
      if (!((present >> ln) & 1)) continue;
      for (int k = 0; k < 32; ++k)
        if (!((used[ln] >> k) & 1)) {
          const int b = cd[ln][k] & 31;
          bm[b] |= 1u << ln;
          deg[b] += 1;
        }
    }
    // Maximum matching lanes <-> banks by augmenting paths started from the
    // banks in decreasing order of remaining codes: the matched bank sets
    // form a matroid, so this greedy order covers the most loaded banks.
    uint32_t done_banks = 0u;
    for (int it = 0; it < 32; ++it) {
      int start = -1, best = 0;
      for (int b = 0; b < 32; ++b)
        if (!((done_banks >> b) & 1) && deg[b] > best) {
          best = deg[b];
          start = b;
        }
      if (start < 0) break;
      done_banks |= 1u << start;
      int stack_bank[33];
      uint32_t stack_cand[33];
      int8_t stack_lane[33];
      uint32_t seen = 0;   // lanes visited
      int depth = 0;
      stack_bank[0] = start;
      stack_cand[0] = bm[start];
      bool found = false;
      while (depth >= 0 && !found) {
        const uint32_t cand = stack_cand[depth] & ~seen;
        if (cand == 0) {
          --depth;
          continue;
        }
        const int ln = __ffs(cand) - 1;
        stack_cand[depth] = cand & ~(1u << ln);
        seen |= 1u << ln;
        stack_lane[depth] = (int8_t)ln;
        if (lbank[ln] < 0) {
          for (int d = depth; d >= 0; --d) lbank[stack_lane[d]] = (int8_t)stack_bank[d];
          found = true;
        } else if (depth < 32) {
          ++depth;
          stack_bank[depth] = lbank[ln];
          stack_cand[depth] = bm[lbank[ln]];
        }
      }
    }
    // choose the codes; an unmatched lane takes its least used bank in this
    // step, the most loaded one among equals
    int cnt[32];
    for (int b = 0; b < 32; ++b) cnt[b] = 0;
    for (int ln = 0; ln < 32; ++ln)
      if (lbank[ln] >= 0) cnt[lbank[ln]] += 1;
    int maxc = 0;
    for (int ln = 0; ln < 32; ++ln) {
      if (!((present >> ln) & 1)) continue;
      int pick = -1;
      if (lbank[ln] >= 0) {
        for (int k = 0; k < 32 && pick < 0; ++k)
          if (!((used[ln] >> k) & 1) && (cd[ln][k] & 31) == lbank[ln]) pick = k;
      } else {
        int bc = 1 << 30, bd = -1;
        for (int k = 0; k < 32; ++k)
          if (!((used[ln] >> k) & 1)) {
            const int b = cd[ln][k] & 31;
            if (cnt[b] < bc || (cnt[b] == bc && deg[b] > bd)) {
              bc = cnt[b];
              bd = deg[b];
              pick = k;
            }
          }
        cnt[cd[ln][pick] & 31] += 1;
      }
      used[ln] |= 1u << pick;
      const int64_t row = rb * 32 + ln;
      // chunk-major: chunk c of every row is one contiguous [V][32] block
      out[((int64_t)c * V + row) * 32 + step] = (uint16_t)((pick << sh) | cd[ln][pick]);
    }
    for (int b = 0; b < 32; ++b) maxc = cnt[b] > maxc ? cnt[b] : maxc;
    passes += (unsigned long long)maxc;
  }
  if (stats) {
    atomicAdd(stats + 0, 32ull);
    atomicAdd(stats + 1, passes);
  }
}

cudaError_t launch_prepare_sched(const uint16_t *codes, int64_t V, int P, int K, uint16_t *out,
                                 unsigned long long *stats, cudaStream_t s) {
  const int64_t probs = (V + 31) / 32 * (P / 32);
  const int64_t blocks = (probs + kSchedThreads - 1) / kSchedThreads;
  if (blocks > 0x7fffffffLL) return cudaErrorInvalidValue;
  if (stats) {
    cudaError_t e = cudaMemsetAsync(stats, 0, 2 * sizeof(unsigned long long), s);
    if (e != cudaSuccess) return e;
  }
  prepare_sched_kernel<<<(unsigned)blocks, kSchedThreads, 0, s>>>(codes, V, P, sched_shift(K),
                                                                 out, stats);
  return cudaGetLastError();
}

}  // namespace rq

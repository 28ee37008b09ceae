// sched_prepare.cu -- the bank-scheduled code layout (RQ_CODES_SCHED).
//
// Not from the pages: a layout of this library for the lookup+sum logits
// pass ("Gemma-2 runtime compression: NF4 + LUT serving", LUT section).  In
// the batch-1 pass a warp handles 16 rows x 2 groups of 16 pairs (one lane
// per row and group), one table lookup per lane per step, from a shared-
// memory table whose bank for code c is c mod 32.  A step costs as many
// shared-memory passes as its most repeated bank; with the codes in their
// natural order that is ~3.5 for random codes.  Here each lane's 16 codes
// are reordered so that every step is, as far as possible, a matching of
// lanes to distinct banks: step by step, a maximum bipartite matching
// (augmenting paths, Kuhn's method) between the lanes and the banks of
// their remaining codes; a lane left unmatched takes the remaining code
// whose bank is least used in that step.  Any order gives the same logits
// up to fp32 summation order; only the speed depends on it.
//
// Entry format: (i << 12) | (c << 2), i = pair position in the group,
// c = code (< 1024).  For a 4-byte table entry per code and a 4 KB table
// per pair laid out back to back, the entry is the byte offset itself.
// Layout: chunk-major [P/32][V][32], so the 32-pair slice that one CTA of
// the batch-1 pass streams is contiguous in memory.
#include "rq_common.cuh"

namespace rq {

constexpr int kSchedThreads = 32;   // one problem per thread, state in smem

__global__ void __launch_bounds__(kSchedThreads) prepare_sched_kernel(
    const uint16_t *__restrict__ codes, int64_t V, int P, uint16_t *__restrict__ out,
    unsigned long long *stats) {
  __shared__ uint16_t s_code[kSchedThreads][32][16];   // codes of each lane
  __shared__ uint32_t s_bmask[kSchedThreads][32];      // banks of unused codes
  __shared__ int8_t s_match[kSchedThreads][32];        // bank -> lane
  __shared__ int8_t s_lbank[kSchedThreads][32];        // lane -> bank
  const int T = threadIdx.x;
  uint16_t(*cd)[16] = s_code[T];
  uint32_t *bm = s_bmask[T];
  int8_t *match = s_match[T];
  int8_t *lbank = s_lbank[T];

  const int nch = (P + 31) / 32;
  const int64_t nrb = (V + 15) / 16;
  const int64_t prob = (int64_t)blockIdx.x * kSchedThreads + T;
  if (prob >= nrb * nch) return;
  const int64_t rb = prob / nch;
  const int c = (int)(prob % nch);

  uint32_t present = 0;
  uint32_t used[32];
  for (int ln = 0; ln < 32; ++ln) {
    const int64_t row = rb * 16 + (ln >> 1);
    const int grp = 2 * c + (ln & 1);
    used[ln] = 0;
    if (row < V && grp * 16 < P) {
      present |= 1u << ln;
      const uint16_t *src = codes + row * P + grp * 16;
      for (int k = 0; k < 16; ++k) cd[ln][k] = src[k] & 0x3FFu;
    }
  }

  unsigned long long passes = 0;
  for (int step = 0; step < 16; ++step) {
    for (int ln = 0; ln < 32; ++ln) {
      uint32_t m = 0;
      if ((present >> ln) & 1)
        for (int k = 0; k < 16; ++k)
          if (!((used[ln] >> k) & 1)) m |= 1u << (cd[ln][k] & 31);
      bm[ln] = m;
      lbank[ln] = -1;
      match[ln] = -1;
    }
    // maximum matching lanes -> banks by augmenting paths
    for (int start = 0; start < 32; ++start) {
      if (!((present >> start) & 1)) continue;
      int stack_lane[33];
      uint32_t stack_cand[33];
      int8_t stack_bank[33];
      uint32_t seen = 0;
      int depth = 0;
      stack_lane[0] = start;
      stack_cand[0] = bm[start];
      bool done = false;
      while (depth >= 0 && !done) {
        const uint32_t cand = stack_cand[depth] & ~seen;
        if (cand == 0) {
          --depth;
          continue;
        }
        const int b = __ffs(cand) - 1;
        stack_cand[depth] = cand & ~(1u << b);
        seen |= 1u << b;
        stack_bank[depth] = (int8_t)b;
        if (match[b] < 0) {
          for (int d = depth; d >= 0; --d) {   // flip the augmenting path
            match[stack_bank[d]] = (int8_t)stack_lane[d];
            lbank[stack_lane[d]] = stack_bank[d];
          }
          done = true;
        } else if (depth < 32) {
          ++depth;
          stack_lane[depth] = match[b];
          stack_cand[depth] = bm[match[b]];
        }
      }
    }
    // choose the items; unmatched lanes take their least crowded bank
    int cnt[32];
    for (int b = 0; b < 32; ++b) cnt[b] = match[b] >= 0 ? 1 : 0;
    int maxc = 0;
    for (int ln = 0; ln < 32; ++ln) {
      if (!((present >> ln) & 1)) continue;
      int pick = -1;
      if (lbank[ln] >= 0) {
        for (int k = 0; k < 16 && pick < 0; ++k)
          if (!((used[ln] >> k) & 1) && (cd[ln][k] & 31) == lbank[ln]) pick = k;
      } else {
        int best = 1 << 30;
        for (int k = 0; k < 16; ++k)
          if (!((used[ln] >> k) & 1) && cnt[cd[ln][k] & 31] < best) {
            best = cnt[cd[ln][k] & 31];
            pick = k;
          }
        cnt[cd[ln][pick] & 31] += 1;
      }
      used[ln] |= 1u << pick;
      const int64_t row = rb * 16 + (ln >> 1);
      // chunk-major: chunk c of every row is one contiguous [V][32] block
      out[((int64_t)c * V + row) * 32 + (ln & 1) * 16 + step] =
          (uint16_t)((pick << 12) | ((uint32_t)cd[ln][pick] << 2));
    }
    for (int b = 0; b < 32; ++b) maxc = cnt[b] > maxc ? cnt[b] : maxc;
    passes += (unsigned long long)maxc;
  }
  if (stats) {
    atomicAdd(stats + 0, 16ull);
    atomicAdd(stats + 1, passes);
  }
}

cudaError_t launch_prepare_sched(const uint16_t *codes, int64_t V, int P, uint16_t *out,
                                 unsigned long long *stats, cudaStream_t s) {
  const int64_t probs = (V + 15) / 16 * ((P + 31) / 32);
  const int64_t blocks = (probs + kSchedThreads - 1) / kSchedThreads;
  if (blocks > 0x7fffffffLL) return cudaErrorInvalidValue;
  if (stats) {
    cudaError_t e = cudaMemsetAsync(stats, 0, 2 * sizeof(unsigned long long), s);
    if (e != cudaSuccess) return e;
  }
  prepare_sched_kernel<<<(unsigned)blocks, kSchedThreads, 0, s>>>(codes, V, P, out, stats);
  return cudaGetLastError();
}

}  // namespace rq

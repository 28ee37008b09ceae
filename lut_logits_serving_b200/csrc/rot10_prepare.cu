// rot10_prepare.cu -- the rotated 10-bit layout (RQ_CODES_PACKED10_ROT).
//
// Not from the pages: a layout of this library for the batch-1 lookup+sum
// pass on 10-bit codes ("Gemma-2 runtime compression: NF4 + LUT serving",
// LUT section; the 10-bit storage of the "Gemma-2-2B combined RQ+NF4" page).
// In that pass a warp takes 32 rows x one 32-pair chunk, one lane per row,
// one table lookup per lane per step, and a step costs as many shared-memory
// passes as its most repeated bank (bank = (pair * K + code) mod 32); with
// the codes in their natural order that is ~3.5 for random codes.  Packed
// rows have no spare bits for a full per-code schedule (RQ_CODES_SCHED), but
// a rotation of each row's 32-code slice costs 5 bits per 32 codes: slot j
// of the slice then holds the code of pair (j + r) mod 32, and r is chosen
// per (row, slice) so that the warp's 32 steps spread over the banks --
// greedily row after row (each row takes the rotation that least raises the
// sum over steps of the largest bank count), then once more with every row
// re-choosing against the others.  Any rotation gives the same logits up to
// fp32 summation order; only the speed depends on it.
//
// Layout: bytes [V][rb] (rb = 10 P / 8, P = M L a multiple of 64) holding
// the rotated slices bit-packed as in RQ_CODES_PACKED10, followed by the
// rotations, uint8 [P/32][V] (chunk-major, as a pass over one chunk reads
// them).
#include "rq_common.cuh"

namespace rq {

constexpr int kRotWarps = 8;   // problems (32 rows x one slice) per block, one per warp

// Cost of giving row i rotation r: the sum over steps j of the largest bank
// count once the row's code of step j is added.
__device__ __forceinline__ int rot_cost(const uint8_t (*cnt)[32], const uint8_t *cmax,
                                        const uint8_t *bk, int r) {
  int cost = 0;
#pragma unroll 8
  for (int j = 0; j < 32; ++j) {
    const int c = cnt[j][bk[(j + r) & 31]] + 1;
    cost += c > cmax[j] ? c : cmax[j];
  }
  return cost;
}

__global__ void __launch_bounds__(32 * kRotWarps) prepare_rot10_kernel(
    const uint16_t *__restrict__ codes, int64_t V, int P, int K, uint8_t *__restrict__ out,
    unsigned long long *stats) {
  __shared__ uint8_t s_bank[kRotWarps][32][32];   // [row][pair] bank of the row's code
  __shared__ uint8_t s_cnt[kRotWarps][32][32];    // [step][bank] codes so far
  __shared__ uint8_t s_max[kRotWarps][32];        // [step] largest count
  __shared__ uint8_t s_rot[kRotWarps][32];        // [row] chosen rotation
  __shared__ uint16_t s_code[kRotWarps][32][33];  // [row][pair] code (padded row)
  const int w = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int nslice = P / 32;
  const int64_t prob = (int64_t)blockIdx.x * kRotWarps + w;   // (row group, slice)
  const int64_t ngroups = (V + 31) / 32;
  if (prob >= ngroups * nslice) return;                      // warp-uniform
  const int64_t g = prob / nslice;
  const int sl = (int)(prob % nslice);
  uint8_t(*bank)[32] = s_bank[w];
  uint8_t(*cnt)[32] = s_cnt[w];
  uint8_t *cmax = s_max[w];
  uint8_t *rot = s_rot[w];
  const uint32_t kmax = (uint32_t)(K - 1);
  const uint32_t kmask = ((K & (K - 1)) == 0) ? kmax : 0xFFFFFFFFu;
  // lane = row; rows past V: no codes (bank 0, never counted)
  const int64_t v = g * 32 + lane;
  const bool live = v < V;
  uint16_t *code = s_code[w][lane];
#pragma unroll
  for (int pl = 0; pl < 32; ++pl) {
    const uint32_t c = live ? (uint32_t)codes[v * P + sl * 32 + pl] & 0x3FFu : 0u;
    code[pl] = (uint16_t)c;
    uint32_t cf = c & kmask;                  // the pass's clamp of codes >= K
    cf = cf > kmax ? kmax : cf;
    bank[lane][pl] = (uint8_t)(((uint32_t)pl * (uint32_t)K + cf) & 31u);
  }
#pragma unroll
  for (int b = 0; b < 32; ++b) cnt[lane][b] = 0;
  cmax[lane] = 0;
  rot[lane] = 0;
  __syncwarp();
  const int nrows = (int)((V - g * 32) < 32 ? (V - g * 32) : 32);
  for (int pass = 0; pass < 2; ++pass) {
    for (int i = 0; i < nrows; ++i) {
      if (pass == 1) {
        // take row i out: lane j is step j
        const uint32_t b = bank[i][(lane + rot[i]) & 31];
        cnt[lane][b] -= 1;
        __syncwarp();
        int m = 0;
#pragma unroll 8
        for (int bb = 0; bb < 32; ++bb) m = cnt[lane][bb] > m ? cnt[lane][bb] : m;
        cmax[lane] = (uint8_t)m;
        __syncwarp();
      }
      // lane r prices rotation r for row i; the cheapest (lowest r on ties) wins
      int cost = rot_cost(cnt, cmax, bank[i], lane);
      int best = lane;
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) {
        const int c2 = __shfl_xor_sync(0xffffffffu, cost, o);
        const int b2 = __shfl_xor_sync(0xffffffffu, best, o);
        if (c2 < cost || (c2 == cost && b2 < best)) {
          cost = c2;
          best = b2;
        }
      }
      __syncwarp();
      const uint32_t b = bank[i][(lane + best) & 31];
      const int c = cnt[lane][b] + 1;
      cnt[lane][b] = (uint8_t)c;
      if (c > cmax[lane]) cmax[lane] = (uint8_t)c;
      if (lane == 0) rot[i] = (uint8_t)best;
      __syncwarp();
    }
  }
  if (stats) {
    int passes = cmax[lane];
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) passes += __shfl_xor_sync(0xffffffffu, passes, o);
    if (lane == 0) {
      atomicAdd(stats + 0, 32ull);
      atomicAdd(stats + 1, (unsigned long long)passes);
    }
  }
  if (!live) return;
  // the row's rotated slice, bit-packed: slot j = code of pair (j + r) mod 32
  const int r = rot[lane];
  uint32_t wd[10];
#pragma unroll
  for (int k = 0; k < 10; ++k) wd[k] = 0u;
#pragma unroll
  for (int j = 0; j < 32; ++j) {
    const uint32_t c = code[(j + r) & 31];
    const int bit = 10 * j;
    wd[bit >> 5] |= c << (bit & 31);
    if ((bit & 31) > 22) wd[(bit >> 5) + 1] |= c >> (32 - (bit & 31));
  }
  const int64_t rb = (int64_t)P / 8 * 10;
  uint32_t *dst = reinterpret_cast<uint32_t *>(out + v * rb + (int64_t)sl * 40);
#pragma unroll
  for (int k = 0; k < 10; ++k) dst[k] = wd[k];
  out[V * rb + (int64_t)sl * V + v] = (uint8_t)r;
}

cudaError_t launch_prepare_rot10(const uint16_t *codes, int64_t V, int P, int K, uint8_t *out,
                                 unsigned long long *stats, cudaStream_t s) {
  const int64_t probs = (V + 31) / 32 * (P / 32);
  const int64_t blocks = (probs + kRotWarps - 1) / kRotWarps;
  if (blocks > 0x7fffffffLL) return cudaErrorInvalidValue;
  if (stats) {
    cudaError_t e = cudaMemsetAsync(stats, 0, 2 * sizeof(unsigned long long), s);
    if (e != cudaSuccess) return e;
  }
  prepare_rot10_kernel<<<(unsigned)blocks, 32 * kRotWarps, 0, s>>>(codes, V, P, K, out, stats);
  return cudaGetLastError();
}

}  // namespace rq

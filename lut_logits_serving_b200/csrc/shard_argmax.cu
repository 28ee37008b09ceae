// shard_argmax.cu -- the greedy pick over a vocabulary split across ranks.
//
// "Gemma-2 runtime compression: NF4 + LUT serving", LUT section: the output
// head takes the argmax of the softcapped logits of every vocabulary row.
// Vocabulary rows are independent, so rank g can hold the code rows
// [row0_g, row0_g + V_g) and compute its rows' logits alone; the global pick
// then needs one exchange of each rank's winner per token.  These kernels are
// the two ends of that exchange:
//   * candidates: per token, the shard's winning value and its global row
//     index (row0 + the shard's own argmax);
//   * merge: per token, the best of the n ranks' candidates under the same
//     order as the single-GPU argmax -- larger value first, lower index on
//     equal values, NaN never above a number -- so the sharded pick equals
//     the unsharded one whenever the shards' logits equal the full run's.
#include <cfloat>
#include <climits>

#include "rq_common.cuh"

namespace rq {

namespace {

__global__ void __launch_bounds__(256) argmax_candidates_kernel(
    const float *__restrict__ logits, const int32_t *__restrict__ argmax, int B, int64_t V,
    int64_t row0, float *__restrict__ val, int32_t *__restrict__ gidx) {
  griddep_wait();
  const int b = blockIdx.x * blockDim.x + threadIdx.x;
  if (b < B) {
    const int32_t i = argmax[b];
    val[b] = logits[(int64_t)b * V + i];
    gidx[b] = (int32_t)(row0 + i);
  }
  griddep_launch_dependents();
}

// one warp per token over the n candidates (rank-major [n][B])
__global__ void __launch_bounds__(256) argmax_merge_kernel(const float *__restrict__ val,
                                                           const int32_t *__restrict__ gidx,
                                                           int n, int B,
                                                           int32_t *__restrict__ argmax) {
  griddep_wait();
  const int b = blockIdx.x * (blockDim.x / 32) + threadIdx.x / 32, lane = threadIdx.x & 31;
  if (b < B) {
    ArgBest best{-FLT_MAX, INT_MAX};
    for (int k = lane; k < n; k += 32)
      best = arg_better(best, ArgBest{val[(int64_t)k * B + b], gidx[(int64_t)k * B + b]});
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) best = arg_better(best, arg_shfl_xor(best, o));
    if (lane == 0) argmax[b] = best.i == INT_MAX ? 0 : best.i;
  }
  griddep_launch_dependents();
}

}  // namespace

cudaError_t launch_argmax_candidates(const float *logits, const int32_t *argmax, int B, int64_t V,
                                     int64_t row0, float *val, int32_t *gidx, cudaStream_t s) {
  return pdl_launch(argmax_candidates_kernel, dim3((unsigned)((B + 255) / 256)), dim3(256), 0, s,
                    logits, argmax, B, V, row0, val, gidx);
}

cudaError_t launch_argmax_merge(const float *val, const int32_t *gidx, int n, int B,
                                int32_t *argmax, cudaStream_t s) {
  return pdl_launch(argmax_merge_kernel, dim3((unsigned)((B + 7) / 8)), dim3(256), 0, s, val, gidx,
                    n, B, argmax);
}

}  // namespace rq

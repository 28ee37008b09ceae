// rq_launch.h -- host-side declarations shared by the librqlut translation
// units: launch helpers, device information and the kernel launchers.  Not
// part of the public ABI.
#pragma once

#include <cuda.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "../../include/rqlut.h"

namespace rq {
struct DecodeSpec;
}

// Launchers implemented by the kernel translation units (host side).
namespace rq {

// Launch with programmatic stream serialization: the kernel may be scheduled
// while the previous kernel of the stream drains.  Every kernel launched so
// calls griddep_wait() before it touches memory an earlier kernel may write
// or read, so completion still orders all kernels transitively.
template <typename... KArgs, typename... Args>
inline cudaError_t pdl_launch(void (*kern)(KArgs...), dim3 grid, dim3 block, size_t smem,
                              cudaStream_t s, Args... args) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = smem;
  cfg.stream = s;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, kern, args...);
}

// cudaLaunchKernel, or with programmatic stream serialization when `pdl`:
// the kernel may start while the previous one in the stream drains and
// must call griddep_wait() before reading that kernel's outputs.
inline cudaError_t launch_maybe_pdl(const void *fn, dim3 grid, dim3 block, size_t smem,
                                    cudaStream_t s, void **args, bool pdl) {
  if (!pdl) return cudaLaunchKernel(fn, grid, block, args, smem, s);
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = smem;
  cfg.stream = s;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelExC(&cfg, fn, args);
}

struct DevInfo {
  int device;
  int sms;
  int max_smem_optin;
  unsigned *err;   // device address of the error word
};

cudaError_t dev_info(DevInfo *out);

// Raises the dynamic shared-memory limit of kernel `fn` on `device` (the
// current device) to at least `smem` bytes.  The limit set so far is kept per
// (kernel, device) under a lock, so concurrent host threads may launch.
cudaError_t ensure_smem_limit(const void *fn, int device, size_t smem);

// CTAs of `fn` resident per SM with `threads` threads and `smem` bytes of
// dynamic shared memory (at least 1), computed once per (kernel, device,
// smem) under a lock.
int occupancy_cached(const void *fn, int device, int threads, size_t smem);

// early_dependents: the kernel launched next on `s` (with the programmatic
// dependency attribute) may start while the build runs; pass true only when
// that kernel is the shared-memory chunk pass.
cudaError_t launch_lut_build(const float *h, const float *C, int B, int b0, int nb, int D,
                             int M, int L, int K, int Bs, float *lut, bool early_dependents,
                             cudaStream_t s);

cudaError_t launch_decode_rows(const int32_t *ids, int64_t N, const void *codes, int fmt,
                               const float *C, int64_t V, int D, int M, int L, int K,
                               float scale, uint16_t *out, unsigned *err, cudaStream_t s);

cudaError_t launch_pack10(const uint16_t *codes, int64_t V, int P, uint8_t *packed,
                          cudaStream_t s);
cudaError_t launch_pack8(const uint16_t *codes, int64_t n, uint8_t *packed, cudaStream_t s);

size_t topk_workspace_bytes(int64_t V, int B, int k);
cudaError_t launch_topk_sample(const float *logits, int64_t V, int B, int k, double temperature,
                               unsigned long long seed, unsigned long long step, float *val,
                               int32_t *idx, int32_t *token, void *ws, cudaStream_t s);
cudaError_t launch_encode(const float *X, int64_t N, const float *C, int D, int M, int L, int K,
                          uint16_t *codes, cudaStream_t s);
cudaError_t launch_prepare_sched(const uint16_t *codes, int64_t V, int P, int K, uint16_t *out,
                                 unsigned long long *stats, cudaStream_t s);
cudaError_t launch_prepare_rot10(const uint16_t *codes, int64_t V, int P, int K, uint8_t *out,
                                 unsigned long long *stats, cudaStream_t s);

// Vocabulary-tiled pass with the LUT chunk resident in shared memory.
struct ChunkPlan {
  bool ok;      // this path applies
  int TB;       // token stride of the LUT (1, 2 or 4)
  int PC;       // pairs per chunk
  int nch;      // chunks
  int R;        // rows per tile
  int variant;  // kernel instance
  size_t smem;  // dynamic shared memory per CTA
};
ChunkPlan plan_chunk(int64_t V, int P, int K, int B, int fmt, const DevInfo &di);
size_t chunk_partial_bytes(const ChunkPlan &cp, int B, int64_t V);
// `early_codes`: the previous kernel writes nothing the code stream reads,
// so the code tiles may be fetched before waiting for it.
cudaError_t launch_logits_chunk(const ChunkPlan &cp, const void *codes, int fmt, int64_t V,
                                int P, int K, int B, const float *lut, float *partial,
                                unsigned long long *keys, bool early_codes,
                                const DevInfo &di, cudaStream_t s);
// Sums the chunk partials, softcap, logits; with `keys` set also folds each
// block's best (value, index) into keys[b] (finished by launch_argmax_keys).
cudaError_t launch_reduce_partials(const float *partial, int nch, int B, int64_t V, float cap,
                                   float *logits, unsigned long long *keys, int nblk,
                                   cudaStream_t s);
// keys -> argmax[b] (keys cleared); with `rows` set, also rebuilds the bf16
// input row of each picked token (the next step's embeddings).
cudaError_t launch_argmax_keys(unsigned long long *keys, int B, int32_t *argmax,
                               const DecodeSpec *rows_spec, uint16_t *rows, cudaStream_t s);

// 2-D uint16 tensor map (driver entry point looked up once); false on failure.
bool encode_tmap_2d_u16(CUtensorMap *map, const void *base, uint64_t inner, uint64_t outer,
                        uint64_t stride_bytes, uint32_t box_inner, uint32_t box_outer,
                        CUtensorMapSwizzle swz);

// Token groups (<= 32) by decoding rows into shared memory and fp32 FMAs
// with the hidden states (ds = 6, L = 2, uint16 codes, K <= 1024).  Argmax
// partials go to columns [0, grid) of [B][nblk]; the rest are set to -inf.
bool decode_fma_applies(int fmt, int64_t V, int D, int M, int L, int K, int B, const float *C,
                        const void *codes, const DevInfo &di);
int decode_fma_blocks(int64_t V, const DevInfo &di);
cudaError_t launch_logits_decode_fma(const float *h, const float *C, const void *codes,
                                     int64_t V, int D, int M, int K, int t0, int nb, float cap,
                                     float *logits, float *am_val, int *am_idx, int nblk,
                                     const DevInfo &di, cudaStream_t s);

// The same on the tcgen05 tensor cores (tf32 MMAs with a hi/lo split for
// fp32 accuracy): token groups of N = 32 or 64, uint16 or 10-bit packed
// codes (decode_mma_applies).  hop: device scratch of decode_mma_hop_bytes(M,
// N, K) for the group's scales, split hidden operand and split codebooks.
bool decode_mma_shape_ok(int fmt, int64_t V, int D, int M, int L, int K);
bool decode_mma_applies(int fmt, int64_t V, int D, int M, int L, int K, const float *C,
                        const void *codes);
cudaError_t launch_logits_decode_mma(const float *h, const float *C, const void *codes, int fmt,
                                     int64_t V, int D, int M, int K, int t0, int nb, int N,
                                     float cap, float *hop, float *logits, float *am_val,
                                     int *am_idx, int nblk, const DevInfo &di, cudaStream_t s);
size_t decode_mma_smem(int K, int N, int fmt);
size_t decode_mma_hop_bytes(int M, int N, int K);

// Batched pass with the LUT read through L2 (token groups of <= 32).
cudaError_t launch_logits_l2(const void *codes, int fmt, int64_t V, int P, int K,
                             const float *lut, int Bs, int lut_t0, int out_t0, int nb,
                             float cap, float *logits, float *am_val, int *am_idx, int nblk,
                             cudaStream_t s);
int l2_grid_blocks(int64_t V, const DevInfo &di);

cudaError_t launch_argmax_finalize(const float *am_val, const int *am_idx, int nblk, int B,
                                   int32_t *argmax, const DecodeSpec *rows_spec, uint16_t *rows,
                                   cudaStream_t s);

}  // namespace rq

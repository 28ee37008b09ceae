// rq_common.cuh -- internal helpers shared by the librqlut kernels (sm_100a).
// Not part of the public ABI.
#pragma once

#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "../../include/rqlut.h"

namespace rq {

// Roughly one second at B200 clocks: every spin on an mbarrier gives up
// after this many SM cycles, sets RQ_DEVERR_TIMEOUT and returns.
constexpr long long kWaitLimitCycles = 2000000000LL;

// Upper bound on the CTAs of any vocabulary-sweep grid.  Argmax partials are
// sized from it so workspace sizes do not depend on the device.
constexpr int kMaxSweepBlocks = 2048;

// Tokens handled by one pass of the L2-served batched kernel.
constexpr int kTokenGroup = 32;

__host__ __device__ constexpr int64_t align_up(int64_t x, int64_t a) {
  return (x + a - 1) / a * a;
}

// ----------------------------------------------------------------- codes

// Keeps every table index in bounds whatever the code value: modulo K for a
// power-of-two K (free: it is the extraction mask), else clamp to K-1.
struct CodeFix {
  uint32_t mask;   // K-1 when K is a power of two, else 0xFFFFFFFF
  uint32_t kmax;   // K-1
  __device__ __forceinline__ uint32_t operator()(uint32_t c) const {
    c &= mask;
    return c > kmax ? kmax : c;
  }
};

inline CodeFix make_codefix(int K) {
  CodeFix f;
  f.kmax = (uint32_t)(K - 1);
  f.mask = ((K & (K - 1)) == 0) ? (uint32_t)(K - 1) : 0xFFFFFFFFu;
  return f;
}

// Code p of a 10-bit packed row: bits [10p, 10p+10), little-endian.
__device__ __forceinline__ uint32_t packed10_code(const uint8_t *row, int p) {
  const int bit = 10 * p;
  const int byte = bit >> 3;
  const uint32_t w = (uint32_t)row[byte] | ((uint32_t)row[byte + 1] << 8);
  return (w >> (bit & 7)) & 0x3FFu;
}

// Code p of row v of RQ_CODES_PACKED10_ROT (all: the layout's first byte, P
// a multiple of 64): slot ((p mod 32) - r) mod 32 of the row's slice p / 32,
// r the slice's rotation byte [p / 32][v] after the V packed rows.
__device__ __forceinline__ uint32_t rot10_code(const uint8_t *all, int64_t V, int P, int64_t v,
                                               int p) {
  const int64_t rb = (int64_t)P / 8 * 10;
  const int r = all[V * rb + (int64_t)(p >> 5) * V + v] & 31;
  return packed10_code(all + v * rb, (p & ~31) | (((p & 31) - r) & 31));
}

// RQ_CODES_SCHED entry = (i << s) | c: i the pair's position in its 32-pair
// slice, c the code, and 2^s the table stride -- the smallest power of two
// >= K, at least 32, so that the shared-memory bank of the entry's table
// word (entry mod 32) is the code's own bank (c mod 32).
__host__ __device__ __forceinline__ int sched_shift(int K) {
  int s = 5;
  while ((1 << s) < K) ++s;
  return s;
}

// Code of pair p of row `id` in RQ_CODES_SCHED (chunk-major [P/32][V][32]):
// find position p % 32 in the row's chunk slice.
__device__ __forceinline__ uint32_t sched_code(const uint16_t *codes, int64_t V, int64_t id,
                                               int p, int sh) {
  // the slice is 64 bytes at a 64-byte aligned offset: four 16-byte loads
  const uint4 *g = reinterpret_cast<const uint4 *>(codes + ((int64_t)(p >> 5) * V + id) * 32);
  const uint32_t want = (uint32_t)(p & 31);
  const uint32_t cmask = (1u << sh) - 1u;
  uint32_t c = 0;
#pragma unroll
  for (int q = 0; q < 4; ++q) {
    const uint4 v = __ldg(g + q);
    const uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
    for (int k = 0; k < 4; ++k) {
      const uint32_t lo = w[k] & 0xFFFFu, hi = w[k] >> 16;
      if (((lo >> sh) & 31u) == want) c = lo & cmask;
      if (((hi >> sh) & 31u) == want) c = hi & cmask;
    }
  }
  return c;
}

// Everything the input-row rebuild needs ("Gemma-2 runtime compression: NF4
// + LUT serving", LUT section: input rows are reconstructed on demand).
struct DecodeSpec {
  const void *codes;
  int fmt;
  const float *C;
  int64_t V;
  int D, M, L, K;
  float scale;
  CodeFix fix;
};

// Subspace m of input row `id`:
//   out[j] = bf16_rne( fp32( fp32(sum_l C[m][l][c_l][j]) * scale ) ),  j < ds,
// level sum in l order with explicit round-to-nearest fp32 operations.
template <int DS>
__device__ __forceinline__ void decode_subspace(const DecodeSpec &a, int64_t id, int m,
                                                uint16_t *out_row) {
  const int ds = DS > 0 ? DS : a.D / a.M;
  const int P = a.M * a.L;
  const int64_t rb = (10LL * P + 7) / 8;
  const uint16_t *all16 = static_cast<const uint16_t *>(a.codes);
  const uint16_t *crow16 = all16 + id * P;
  const uint8_t *crow10 = static_cast<const uint8_t *>(a.codes) + id * rb;
  uint16_t *o = out_row + (int64_t)m * ds;
  auto code = [&](int p) -> uint32_t {
    uint32_t c;
    if (a.fmt == RQ_CODES_U16) c = crow16[p];
    else if (a.fmt == RQ_CODES_SCHED) c = sched_code(all16, a.V, id, p, sched_shift(a.K));
    else if (a.fmt == RQ_CODES_U8) c = static_cast<const uint8_t *>(a.codes)[id * P + p];
    else if (a.fmt == RQ_CODES_PACKED10_ROT)
      c = rot10_code(static_cast<const uint8_t *>(a.codes), a.V, P, id, p);
    else c = packed10_code(crow10, p);
    return a.fix(c);
  };
  if (DS > 0) {
    float e[DS > 0 ? DS : 1];
#pragma unroll
    for (int j = 0; j < DS; ++j) e[j] = 0.f;
    for (int l = 0; l < a.L; ++l) {
      const int p = m * a.L + l;
      const float *cw = a.C + ((size_t)p * a.K + code(p)) * DS;
#pragma unroll
      for (int j = 0; j < DS; ++j) e[j] = __fadd_rn(e[j], __ldg(cw + j));
    }
#pragma unroll
    for (int j = 0; j < DS; ++j)
      o[j] = __bfloat16_as_ushort(__float2bfloat16_rn(__fmul_rn(e[j], a.scale)));
  } else {
    for (int j = 0; j < ds; ++j) {
      float e = 0.f;
      for (int l = 0; l < a.L; ++l) {
        const int p = m * a.L + l;
        e = __fadd_rn(e, __ldg(a.C + ((size_t)p * a.K + code(p)) * ds + j));
      }
      o[j] = __bfloat16_as_ushort(__float2bfloat16_rn(__fmul_rn(e, a.scale)));
    }
  }
}

// ---------------------------------------------------------- shared memory

__device__ __forceinline__ uint32_t smem_addr(const void *p) {
  return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

__device__ __forceinline__ void mbar_init(uint32_t bar, uint32_t count) {
  asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(bar), "r"(count) : "memory");
}

__device__ __forceinline__ void fence_mbar_init() {
  asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
}

__device__ __forceinline__ void mbar_arrive_expect_tx(uint32_t bar, uint32_t bytes) {
  asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(bar), "r"(bytes)
               : "memory");
}

__device__ __forceinline__ bool mbar_try_wait(uint32_t bar, uint32_t parity) {
  uint32_t done;
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
      "selp.u32 %0, 1, 0, p;\n\t}"
      : "=r"(done)
      : "r"(bar), "r"(parity)
      : "memory");
  return done != 0;
}

// Spin until the phase with `parity` completes; false after the limit.
__device__ __forceinline__ bool mbar_wait_bounded(uint32_t bar, uint32_t parity) {
  if (mbar_try_wait(bar, parity)) return true;
  long long t0 = clock64();
  while (!mbar_try_wait(bar, parity)) {
    if (clock64() - t0 > kWaitLimitCycles) return false;
  }
  return true;
}

// ------------------------------------------------------------------- TMA

__device__ __forceinline__ uint64_t l2_policy_evict_first() {
  uint64_t pol;
  asm volatile("createpolicy.fractional.L2::evict_first.b64 %0, 1.0;" : "=l"(pol));
  return pol;
}

__device__ __forceinline__ uint64_t l2_policy_evict_last() {
  uint64_t pol;
  asm volatile("createpolicy.fractional.L2::evict_last.b64 %0, 1.0;" : "=l"(pol));
  return pol;
}

// 2-D tiled TMA load (no multicast) into this CTA's shared memory.
__device__ __forceinline__ void tma_load_2d(uint32_t dst, const CUtensorMap *map, int x, int y,
                                            uint32_t bar, uint64_t policy) {
  asm volatile(
      "cp.async.bulk.tensor.2d.shared::cluster.global.tile.mbarrier::complete_tx::bytes"
      ".L2::cache_hint [%0], [%1, {%2, %3}], [%4], %5;" ::"r"(dst),
      "l"(reinterpret_cast<uint64_t>(map)), "r"(x), "r"(y), "r"(bar), "l"(policy)
      : "memory");
}

// 2-D tiled TMA prefetch of a box into L2 only (no shared memory written),
// normal L2 priority.
__device__ __forceinline__ void tma_prefetch_2d(const CUtensorMap *map, int x, int y) {
  asm volatile("cp.async.bulk.prefetch.tensor.2d.L2.global.tile [%0, {%1, %2}];" ::"l"(
                   reinterpret_cast<uint64_t>(map)),
               "r"(x), "r"(y)
               : "memory");
}

// 1-D bulk copy global -> this CTA's shared memory (16-byte aligned, size a
// multiple of 16), completing on an mbarrier.  No multicast.
__device__ __forceinline__ void bulk_g2s(uint32_t dst, const void *src, uint32_t bytes,
                                         uint32_t bar) {
  asm volatile(
      "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::
          "r"(dst),
      "l"(src), "r"(bytes), "r"(bar)
      : "memory");
}

// Programmatic dependent launch: wait for the previous kernel of the stream
// (a no-op when this kernel was launched without the attribute) / allow the
// next one to start its prologue.
__device__ __forceinline__ void griddep_wait() {
  asm volatile("griddepcontrol.wait;" ::: "memory");
}
__device__ __forceinline__ void griddep_launch_dependents() {
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
}

__device__ __forceinline__ void prefetch_tmap(const CUtensorMap *map) {
  asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(map)) : "memory");
}

// ------------------------------------------------------------- softcap

__device__ __forceinline__ float softcap_f(float z, float cap) {
  return cap > 0.f ? cap * tanhf(z / cap) : z;
}

// ---------------------------------------------------------------- argmax

struct ArgBest {
  float v;
  int i;
};

// Larger value wins; equal values: lower index wins.  NaN never wins over a
// number.  Order-independent, so any reduction tree gives the same answer.
__device__ __forceinline__ ArgBest arg_better(ArgBest a, ArgBest b) {
  bool a_nan = a.v != a.v, b_nan = b.v != b.v;
  if (a_nan != b_nan) return a_nan ? b : a;
  if (a.v > b.v) return a;
  if (b.v > a.v) return b;
  return a.i <= b.i ? a : b;
}

// 64-bit key whose unsigned order is the argmax order: value (NaN lowest,
// -0 == +0) in the high word, then the lower index in the low word.  One
// atomicMax per warp then finds the argmax in any arrival order.
__device__ __forceinline__ unsigned long long arg_key(ArgBest a) {
  if (a.v != a.v) return 0ull;
  uint32_t u = a.v == 0.f ? 0u : __float_as_uint(a.v);
  u = (u & 0x80000000u) ? ~u : (u | 0x80000000u);
  return ((unsigned long long)u << 32) | (uint32_t)(0xFFFFFFFFu - (uint32_t)a.i);
}
__device__ __forceinline__ int arg_key_index(unsigned long long k) {
  return k == 0ull ? 0 : (int)(0xFFFFFFFFu - (uint32_t)(k & 0xFFFFFFFFull));
}

__device__ __forceinline__ ArgBest arg_shfl_xor(ArgBest a, int lane_mask,
                                                unsigned members = 0xffffffffu) {
  ArgBest o;
  o.v = __shfl_xor_sync(members, a.v, lane_mask);
  o.i = __shfl_xor_sync(members, a.i, lane_mask);
  return o;
}

}  // namespace rq

#include "rq_launch.h"

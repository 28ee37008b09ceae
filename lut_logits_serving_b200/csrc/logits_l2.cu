// logits_l2.cu -- LUT lookup+sum logits for token groups of up to 32, with
// the tables read through L2, softcap and argmax partials fused.
//
// "Gemma-2 runtime compression: NF4 + LUT serving", LUT section (lookup +
// sum replaces the output matmul; Gemma-2's softcap follows).  For a batch
// the tables of 32 tokens are 100.7 MB at the Gemma-2 shape: they fit in
// L2 but not in shared memory, and one vocabulary row touches all P of
// them, so each (row, pair) lookup fetches the 32 tokens' entries as one
// contiguous 128-byte line (token-innermost layout):
//   * G lanes share a row, lane q holding tokens 4q..4q+3 as a float4;
//   * codes are read once per row (16-byte vectors broadcast to the G
//     lanes); 10-bit packed rows are unpacked with funnel shifts;
//   * the softcap, the logits store and a running (value, index) argmax
//     per lane form the epilogue; per-CTA argmax partials go to workspace.
// One pass over the code matrix serves the whole token group.
#include <cfloat>
#include <climits>

#include "rq_common.cuh"

namespace rq {

struct L2Args {
  const void *codes;
  const float *lut;   // [P][K][Bs]
  int64_t V;
  int P, K, Bs;
  int lut_t0;         // first token of this group inside the table
  int out_t0;         // index of that token in the caller's batch
  int nb;             // tokens in this group (<= 32)
  float cap;
  float *logits;      // [Btot][V] or null
  float *am_val;      // [Btot][nblk] or null
  int *am_idx;
  CodeFix fix;
  int ssh;            // RQ_CODES_SCHED entry shift (table stride 2^ssh)
};

// 16-byte loads with an L2 eviction hint: the code stream is read once
// (evict first), the group's tables are read throughout the pass (evict
// last), so the stream does not push table lines out to DRAM.
__device__ __forceinline__ uint4 ldg_u4_hint(const uint4 *p, uint64_t pol) {
  uint4 v;
  asm volatile("ld.global.nc.L2::cache_hint.v4.u32 {%0, %1, %2, %3}, [%4], %5;"
               : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w)
               : "l"(p), "l"(pol));
  return v;
}

__device__ __forceinline__ float4 ldg_f4_hint(const float *p, uint64_t pol) {
  float4 v;
  asm volatile("ld.global.nc.L2::cache_hint.v4.f32 {%0, %1, %2, %3}, [%4], %5;"
               : "=f"(v.x), "=f"(v.y), "=f"(v.z), "=f"(v.w)
               : "l"(p), "l"(pol));
  return v;
}

template <int VW>
__device__ __forceinline__ void add_vec(const float *e, float (&acc)[VW]) {
  if (VW == 1) {
    acc[0] += __ldg(e);
  } else if (VW == 2) {
    const float2 t = __ldg(reinterpret_cast<const float2 *>(e));
    acc[0] += t.x;
    acc[1] += t.y;
  } else {
    // (the policy made at each load: measured faster than one kept in a
    // register across the loop, 1394 vs 1490 us for a 32-token group)
    const float4 t = ldg_f4_hint(e, l2_policy_evict_last());
    acc[0] += t.x;
    acc[1] += t.y;
    acc[2] += t.z;
    acc[3] += t.w;
  }
}

template <int VW, int G, int FMT>
__global__ void __launch_bounds__(256) logits_l2_kernel(const L2Args a) {
  griddep_wait();
  const uint64_t pcode = l2_policy_evict_first();
  constexpr int RPW = 32 / G;     // rows per warp
  constexpr int RPB = 8 * RPW;    // rows per CTA step
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int q = lane % G;
  const int rw = lane / G;
  const int tok = q * VW;         // first token of this lane, within the group
  // G is a power of two, so lanes can lie past the group's last token (and
  // past the table's token stride Bs): they read token 0's entries instead,
  // and their sums are never stored
  const float *tl = a.lut + a.lut_t0 + (tok < a.nb ? tok : 0);
  const int K = a.K, Bs = a.Bs;

  ArgBest best[VW];
#pragma unroll
  for (int i = 0; i < VW; ++i) best[i] = ArgBest{-FLT_MAX, INT_MAX};

  for (int64_t base = (int64_t)blockIdx.x * RPB; base < a.V; base += (int64_t)gridDim.x * RPB) {
    const int64_t v = base + warp * RPW + rw;
    if (v >= a.V) continue;
    float acc[VW];
#pragma unroll
    for (int i = 0; i < VW; ++i) acc[i] = 0.f;
    if (FMT == RQ_CODES_U16) {
      const uint4 *crow = reinterpret_cast<const uint4 *>(
          static_cast<const uint16_t *>(a.codes) + v * a.P);
      // 64 codes per step, all lookups of a step independent (L2 latency)
      const int n64 = a.P / 64;
      for (int g = 0; g < n64; ++g) {
        uint32_t wd[32];
#pragma unroll
        for (int k = 0; k < 8; ++k) {
          const uint4 w = ldg_u4_hint(crow + 8 * g + k, pcode);
          wd[4 * k + 0] = w.x;
          wd[4 * k + 1] = w.y;
          wd[4 * k + 2] = w.z;
          wd[4 * k + 3] = w.w;
        }
        const float *tg = tl + (size_t)(64 * g) * K * Bs;
#pragma unroll
        for (int j = 0; j < 64; ++j) {
          const uint32_t c = a.fix((j & 1) ? (wd[j >> 1] >> 16) : (wd[j >> 1] & 0xFFFFu));
          add_vec<VW>(tg + ((size_t)j * K + c) * Bs, acc);
        }
      }
      for (int g = n64 * 8; g < a.P / 8; ++g) {
        const uint4 w = ldg_u4_hint(crow + g, pcode);
        const uint32_t ws[4] = {w.x, w.y, w.z, w.w};
        const float *tg = tl + (size_t)(8 * g) * K * Bs;
#pragma unroll
        for (int k = 0; k < 4; ++k) {
          const uint32_t c0 = a.fix(ws[k] & 0xFFFFu), c1 = a.fix(ws[k] >> 16);
          add_vec<VW>(tg + ((size_t)(2 * k) * K + c0) * Bs, acc);
          add_vec<VW>(tg + ((size_t)(2 * k + 1) * K + c1) * Bs, acc);
        }
      }
    } else if (FMT == RQ_CODES_U8) {
      // 16 byte codes per 16-byte vector; rows are 16-byte aligned (P % 16 == 0)
      const uint4 *crow = reinterpret_cast<const uint4 *>(
          static_cast<const uint8_t *>(a.codes) + v * a.P);
      const int n16 = a.P / 16;
      for (int g = 0; g < n16; g += 4) {
        uint32_t wd[16];
#pragma unroll
        for (int k = 0; k < 4; ++k) {
          const uint4 w = g + k < n16 ? ldg_u4_hint(crow + g + k, pcode) : make_uint4(0, 0, 0, 0);
          wd[4 * k + 0] = w.x;
          wd[4 * k + 1] = w.y;
          wd[4 * k + 2] = w.z;
          wd[4 * k + 3] = w.w;
        }
        const float *tg = tl + (size_t)(16 * g) * K * Bs;
        const int nj = (n16 - g < 4 ? n16 - g : 4) * 16;   // codes of this step
#pragma unroll
        for (int j = 0; j < 64; ++j) {
          if (j < nj) {
            const uint32_t c = a.fix((wd[j >> 2] >> (8 * (j & 3))) & 0xFFu);
            add_vec<VW>(tg + ((size_t)j * K + c) * Bs, acc);
          }
        }
      }
    } else if (FMT == RQ_CODES_SCHED) {
      // chunk-major [P/32][V][32]; 32 entries (i << ssh | c) per chunk
      // slice, in any order
      const uint16_t *cbase = static_cast<const uint16_t *>(a.codes) + v * 32;
      const int nc = a.P / 32;
      const uint32_t cmask = (1u << a.ssh) - 1u;
      const bool kfull = K > (int)cmask;  // every masked code indexes a real entry
      for (int cc = 0; cc < nc; ++cc) {
        const uint4 *crow = reinterpret_cast<const uint4 *>(cbase + (size_t)cc * a.V * 32);
        uint32_t wd[16];
#pragma unroll
        for (int k = 0; k < 4; ++k) {
          const uint4 w = ldg_u4_hint(crow + k, pcode);
          wd[4 * k + 0] = w.x;
          wd[4 * k + 1] = w.y;
          wd[4 * k + 2] = w.z;
          wd[4 * k + 3] = w.w;
        }
        const float *tc = tl + (size_t)(32 * cc) * K * Bs;
#pragma unroll
        for (int j = 0; j < 32; ++j) {
          const uint32_t e = (j & 1) ? (wd[j >> 1] >> 16) : (wd[j >> 1] & 0xFFFFu);
          const uint32_t c = e & cmask;
          const uint32_t pp = (e >> a.ssh) & 31u;              // pair within the chunk
          if (kfull || c < (uint32_t)K) add_vec<VW>(tc + ((size_t)pp * K + c) * Bs, acc);
        }
      }
    } else {
      // 64 codes = 640 bits = 5 x 16 bytes per group; rows are 16-byte aligned
      const int64_t rb = (int64_t)a.P / 64 * 80;
      const uint4 *crow = reinterpret_cast<const uint4 *>(
          static_cast<const uint8_t *>(a.codes) + v * rb);
      const int ng = a.P / 64;
      // rotated slices: the rotation bytes [P/32][V] after the V packed rows
      const uint8_t *rotp = static_cast<const uint8_t *>(a.codes) + a.V * rb + v;
      for (int g = 0; g < ng; ++g) {
        int r0 = 0, r1 = 0;
        if (FMT == RQ_CODES_PACKED10_ROT) {
          r0 = __ldg(rotp + (int64_t)(2 * g) * a.V) & 31;
          r1 = __ldg(rotp + (int64_t)(2 * g + 1) * a.V) & 31;
        }
        uint32_t w[21];
#pragma unroll
        for (int k = 0; k < 5; ++k) {
          const uint4 x = ldg_u4_hint(crow + 5 * g + k, pcode);
          w[4 * k + 0] = x.x;
          w[4 * k + 1] = x.y;
          w[4 * k + 2] = x.z;
          w[4 * k + 3] = x.w;
        }
        w[20] = 0u;
        const float *tg = tl + (size_t)(64 * g) * K * Bs;
#pragma unroll
        for (int j = 0; j < 64; ++j) {
          const int bit = 10 * j;
          const uint32_t c = a.fix(__funnelshift_r(w[bit >> 5], w[(bit >> 5) + 1], bit & 31) & 0x3FFu);
          // slot j of a rotated slice holds pair (j + r) mod 32 of that slice
          const int pj = FMT == RQ_CODES_PACKED10_ROT
                             ? ((j & 32) | (((j & 31) + ((j & 32) ? r1 : r0)) & 31))
                             : j;
          add_vec<VW>(tg + ((size_t)pj * K + c) * Bs, acc);
        }
      }
    }
#pragma unroll
    for (int i = 0; i < VW; ++i) {
      if (tok + i < a.nb) {
        const float y = softcap_f(acc[i], a.cap);
        if (a.logits) a.logits[(size_t)(a.out_t0 + tok + i) * a.V + v] = y;
        best[i] = arg_better(best[i], ArgBest{y, (int)v});
      }
    }
  }

  griddep_launch_dependents();
  if (a.am_val == nullptr) return;
  // lanes with equal q hold the same tokens: reduce across row slots
#pragma unroll
  for (int i = 0; i < VW; ++i)
#pragma unroll
    for (int o = G; o < 32; o <<= 1) best[i] = arg_better(best[i], arg_shfl_xor(best[i], o));
  __shared__ ArgBest wb[8][32];
  if (rw == 0) {
#pragma unroll
    for (int i = 0; i < VW; ++i) wb[warp][tok + i] = best[i];
  }
  __syncthreads();
  const int t = threadIdx.x;
  if (t < G * VW && t < a.nb) {
    ArgBest r = wb[0][t];
    for (int w2 = 1; w2 < 8; ++w2) r = arg_better(r, wb[w2][t]);
    a.am_val[(size_t)(a.out_t0 + t) * gridDim.x + blockIdx.x] = r.v;
    a.am_idx[(size_t)(a.out_t0 + t) * gridDim.x + blockIdx.x] = r.i;
  }
}

// Any shape, any format: one thread per (row, token), scalar loads.  Used
// when the fast kernels' alignment or size preconditions do not hold.
__global__ void __launch_bounds__(256) logits_generic_kernel(const L2Args a, int fmt) {
  griddep_wait();
  const int t = blockIdx.y;  // token within the group
  const int64_t rb = (10LL * a.P + 7) / 8;
  const float *tl = a.lut + a.lut_t0 + t;
  ArgBest best{-FLT_MAX, INT_MAX};
  for (int64_t v = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; v < a.V;
       v += (int64_t)gridDim.x * blockDim.x) {
    const uint16_t *c16 = static_cast<const uint16_t *>(a.codes) + v * a.P;
    const uint8_t *c8 = static_cast<const uint8_t *>(a.codes) + v * rb;
    float z = 0.f;
    for (int p = 0; p < a.P; ++p) {
      if (fmt == RQ_CODES_SCHED) {
        const uint32_t e =
            static_cast<const uint16_t *>(a.codes)[((size_t)(p >> 5) * a.V + v) * 32 + (p & 31)];
        const uint32_t c = e & ((1u << a.ssh) - 1u);
        const int pp = (p & ~31) + (int)((e >> a.ssh) & 31u);
        if (c < (uint32_t)a.K) z += __ldg(tl + ((size_t)pp * a.K + c) * a.Bs);
        continue;
      }
      const uint32_t c = a.fix(
          fmt == RQ_CODES_U16 ? (uint32_t)c16[p]
          : fmt == RQ_CODES_U8 ? (uint32_t)static_cast<const uint8_t *>(a.codes)[v * a.P + p]
          : fmt == RQ_CODES_PACKED10_ROT
              ? rot10_code(static_cast<const uint8_t *>(a.codes), a.V, a.P, v, p)
              : packed10_code(c8, p));
      z += __ldg(tl + ((size_t)p * a.K + c) * a.Bs);
    }
    const float y = softcap_f(z, a.cap);
    if (a.logits) a.logits[(size_t)(a.out_t0 + t) * a.V + v] = y;
    best = arg_better(best, ArgBest{y, (int)v});
  }
  if (a.am_val == nullptr) return;
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) best = arg_better(best, arg_shfl_xor(best, o));
  __shared__ ArgBest wb[8];
  if ((threadIdx.x & 31) == 0) wb[threadIdx.x >> 5] = best;
  __syncthreads();
  if (threadIdx.x == 0) {
    ArgBest r = wb[0];
    for (int w = 1; w < (int)blockDim.x / 32; ++w) r = arg_better(r, wb[w]);
    a.am_val[(size_t)(a.out_t0 + t) * gridDim.x + blockIdx.x] = r.v;
    a.am_idx[(size_t)(a.out_t0 + t) * gridDim.x + blockIdx.x] = r.i;
  }
}

// ------------------------------------------------------------ host side

template <int VW, int G, int FMT>
static cudaError_t launch_fast(const L2Args &a, int nblk, cudaStream_t s) {
  return pdl_launch(logits_l2_kernel<VW, G, FMT>, dim3(nblk), dim3(256), 0, s, a);
}

template <int VW, int FMT>
static cudaError_t launch_vw(const L2Args &a, int G, int nblk, cudaStream_t s) {
  switch (G) {
    case 1: return launch_fast<VW, 1, FMT>(a, nblk, s);
    case 2: return launch_fast<VW, 2, FMT>(a, nblk, s);
    case 4: return launch_fast<VW, 4, FMT>(a, nblk, s);
    default: return launch_fast<VW, 8, FMT>(a, nblk, s);
  }
}

cudaError_t launch_logits_l2(const void *codes, int fmt, int64_t V, int P, int K,
                             const float *lut, int Bs, int lut_t0, int out_t0, int nb,
                             float cap, float *logits, float *am_val, int *am_idx, int nblk,
                             cudaStream_t s) {
  L2Args a;
  a.codes = codes;
  a.lut = lut;
  a.V = V;
  a.P = P;
  a.K = K;
  a.Bs = Bs;
  a.lut_t0 = lut_t0;
  a.out_t0 = out_t0;
  a.nb = nb;
  a.cap = cap;
  a.logits = logits;
  a.am_val = am_val;
  a.am_idx = am_idx;
  a.fix = make_codefix(K);
  a.ssh = sched_shift(K);
  const bool codes16 = (reinterpret_cast<uintptr_t>(codes) & 15) == 0;
  const bool fast_fmt = fmt == RQ_CODES_U16     ? (P % 8 == 0)
                        : fmt == RQ_CODES_SCHED ? (P % 32 == 0)
                        : fmt == RQ_CODES_U8    ? (P % 16 == 0)
                                                : (P % 64 == 0);
  int VW;
  if (Bs == 1) VW = 1;
  else if (Bs == 2) VW = 2;
  else VW = 4;
  const bool lut_ok = VW < 4 || ((reinterpret_cast<uintptr_t>(lut + lut_t0) & 15) == 0 &&
                                 Bs % 4 == 0);
  if (!(codes16 && fast_fmt && lut_ok) || nb > 32 || (VW < 4 && nb > VW)) {
    return pdl_launch(logits_generic_kernel, dim3((unsigned)nblk, (unsigned)nb), dim3(256), 0, s,
                      a, fmt);
  }
  int G = 1;
  if (VW == 4) {
    const int need = (nb + 3) / 4;
    while (G < need) G <<= 1;
  }
  if (fmt == RQ_CODES_U16) {
    if (VW == 1) return launch_fast<1, 1, RQ_CODES_U16>(a, nblk, s);
    if (VW == 2) return launch_fast<2, 1, RQ_CODES_U16>(a, nblk, s);
    return launch_vw<4, RQ_CODES_U16>(a, G, nblk, s);
  }
  if (fmt == RQ_CODES_SCHED) {
    if (VW == 1) return launch_fast<1, 1, RQ_CODES_SCHED>(a, nblk, s);
    if (VW == 2) return launch_fast<2, 1, RQ_CODES_SCHED>(a, nblk, s);
    return launch_vw<4, RQ_CODES_SCHED>(a, G, nblk, s);
  }
  if (fmt == RQ_CODES_U8) {
    if (VW == 1) return launch_fast<1, 1, RQ_CODES_U8>(a, nblk, s);
    if (VW == 2) return launch_fast<2, 1, RQ_CODES_U8>(a, nblk, s);
    return launch_vw<4, RQ_CODES_U8>(a, G, nblk, s);
  }
  if (fmt == RQ_CODES_PACKED10_ROT) {
    if (VW == 1) return launch_fast<1, 1, RQ_CODES_PACKED10_ROT>(a, nblk, s);
    if (VW == 2) return launch_fast<2, 1, RQ_CODES_PACKED10_ROT>(a, nblk, s);
    return launch_vw<4, RQ_CODES_PACKED10_ROT>(a, G, nblk, s);
  }
  if (VW == 1) return launch_fast<1, 1, RQ_CODES_PACKED10>(a, nblk, s);
  if (VW == 2) return launch_fast<2, 1, RQ_CODES_PACKED10>(a, nblk, s);
  return launch_vw<4, RQ_CODES_PACKED10>(a, G, nblk, s);
}

int l2_grid_blocks(int64_t V, const DevInfo &di) {
  int64_t n = (int64_t)di.sms * 4;
  const int64_t need = (V + 255) / 256;
  if (n > need) n = need;
  if (n > kMaxSweepBlocks) n = kMaxSweepBlocks;
  if (n < 1) n = 1;
  return (int)n;
}

}  // namespace rq

// logits_decode_fma.cu -- logits of a token group (up to 32) by decoding
// vocabulary rows into shared memory and multiplying them with the hidden
// states, for batches where the per-token tables no longer fit on chip.
//
// "Gemma-2 runtime compression: NF4 + LUT serving", LUT section: the lookup
// + sum is algebraically the decode-then-matmul the pages check it against,
//   z[b][v] = sum_m sum_j h[b][m*ds + j] * (C[m][0][c0][j] + C[m][1][c1][j]),
// with c_l = code[v][m*L + l]; Gemma-2's softcap follows.  For B tokens the
// table form reads a B-wide table line per (row, pair) -- 25 GB of L2 traffic
// at B = 32 -- while this form reads each subspace's codebook (48 KB at
// K = 1024) once per 1024-row tile and does 6 fp32 FMAs per (row, subspace,
// token) on the FP32 pipe.
//
// Design for sm_100a (ds = 6, L = 2, uint16 codes, K <= 1024).  Persistent
// CTAs, one per SM, each over an even share of the rows, in tiles of up to
// 1024 rows; per subspace m of a tile:
//   * the codebooks of subspace m (both levels, [2][K][6] floats) arrive by
//     one bulk copy into a double buffer, issued two subspaces ahead;
//   * the tile's codes arrive by 2-D TMA boxes {16 codes, 256 rows} (8
//     subspaces per stage, 32-byte swizzle), double-buffered;
//   * decode: one thread per row rebuilds e[j] = fp32(c0[j] + c1[j]) from the
//     shared codebooks into a j-major tile E[row group][j][8 rows];
//   * FMA: thread (row group of 8, token group of 8) accumulates 8 x 8 sums
//     in registers from two 16-byte loads of E and of the hidden slice per j,
//     two tokens per packed fp32x2 FMA (each lane an ordinary rn fp32 FMA).
// Decoding subspace m+1 overlaps the FMAs of m (two E buffers, one barrier
// per subspace).  The epilogue applies the softcap, stores the logits and
// folds a per-token (value, index) argmax partial per CTA.
#include <cfloat>
#include <climits>

#include "rq_common.cuh"

namespace rq {

namespace {

constexpr int kDfThreads = 512;
constexpr int kDfRows = 1024;                         // rows per tile: 128 groups of 8
constexpr int kDfStageCodes = 16;                     // 8 subspaces x 2 levels
constexpr int kDfStageBytes = kDfRows * kDfStageCodes * 2;   // 32 KB
constexpr int kDfGS = 52;                             // floats per 8-wide group (48 + 4 pad)
constexpr int kDfEBytes = 128 * kDfGS * 4;            // one E tile
constexpr int kDfHBytes = 4 * kDfGS * 4;              // one hidden slice (32 tokens)

struct DfArgs {
  const float *h;      // [Btot][D]
  const float *C;      // [M][2][K][6]
  int64_t V;
  int M, K, D;
  int t0, nb;          // tokens t0 .. t0 + nb - 1 of h (and of the outputs)
  float cap;
  float *logits;       // [Btot][V] or null
  float *am_val;       // [Btot][nblk] or null (columns past the grid get -inf)
  int *am_idx;
  int nblk;            // argmax-partial columns (>= the grid)
  CodeFix fix;
  unsigned *err;
};

__device__ __forceinline__ uint4 lds_u4(uint32_t addr) {
  uint4 v;
  asm volatile("ld.shared.v4.u32 {%0, %1, %2, %3}, [%4];"
               : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w)
               : "r"(addr));
  return v;
}

__device__ __forceinline__ float4 lds_f4(uint32_t addr) {
  float4 v;
  asm volatile("ld.shared.v4.f32 {%0, %1, %2, %3}, [%4];"
               : "=f"(v.x), "=f"(v.y), "=f"(v.z), "=f"(v.w)
               : "r"(addr));
  return v;
}

__device__ __forceinline__ float2 lds_f2(uint32_t addr) {
  float2 v;
  asm volatile("ld.shared.v2.f32 {%0, %1}, [%2];" : "=f"(v.x), "=f"(v.y) : "r"(addr));
  return v;
}

__device__ __forceinline__ void sts_f32(uint32_t addr, float x) {
  asm volatile("st.shared.f32 [%0], %1;" ::"r"(addr), "f"(x));
}

__device__ __forceinline__ unsigned long long pack2(float lo, float hi) {
  unsigned long long r;
  asm("mov.b64 %0, {%1, %2};" : "=l"(r) : "f"(lo), "f"(hi));
  return r;
}

__device__ __forceinline__ void unpack2(unsigned long long v, float &lo, float &hi) {
  asm("mov.b64 {%0, %1}, %2;" : "=f"(lo), "=f"(hi) : "l"(v));
}

// lane-wise rn fp32 a * b + c: two ordinary FMAs in one instruction
__device__ __forceinline__ unsigned long long fma2(unsigned long long a, unsigned long long b,
                                                   unsigned long long c) {
  unsigned long long d;
  asm("fma.rn.f32x2 %0, %1, %2, %3;" : "=l"(d) : "l"(a), "l"(b), "l"(c));
  return d;
}

}  // namespace

__global__ void __launch_bounds__(kDfThreads, 1)
    logits_decode_fma_kernel(const __grid_constant__ CUtensorMap tmap, const DfArgs a) {
  extern __shared__ __align__(1024) unsigned char smem_raw[];
  unsigned char *smem = smem_raw + ((1024u - (smem_addr(smem_raw) & 1023u)) & 1023u);
  const int cbf = 2 * a.K * 6;                      // floats of one subspace's codebooks
  const uint32_t cbb = (uint32_t)cbf * 4u;
  unsigned char *st = smem;                                        // 2 code stages
  float *cb = reinterpret_cast<float *>(st + 2 * kDfStageBytes);  // 2 codebook buffers
  float *Es = cb + 2 * (size_t)align_up(cbf, 256);                 // 2 E tiles
  float *Hs = Es + 2 * 128 * kDfGS;                                // 2 hidden slices
  uint64_t *bar = reinterpret_cast<uint64_t *>(Hs + 2 * 4 * kDfGS);   // [0,1] codes, [2,3] books
  ArgBest *wbest = reinterpret_cast<ArgBest *>(bar + 4);            // [16 warps][32 tokens]
  ArgBest *cbest = wbest + 16 * 32;                                 // [32 tokens], CTA-wide

  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  if (tid == 0) {
    prefetch_tmap(&tmap);
    for (int i = 0; i < 4; ++i) mbar_init(smem_addr(&bar[i]), 1);
    fence_mbar_init();
  }
  if (tid < 32) cbest[tid] = ArgBest{-FLT_MAX, INT_MAX};
  __syncthreads();
  griddep_wait();

  const uint64_t pol_codes = l2_policy_evict_first();
  const int M = a.M, ng = a.M / 8;
  // this CTA's rows, split into tiles of at most 1024
  const int64_t r0 = a.V * blockIdx.x / gridDim.x, r1 = a.V * (blockIdx.x + 1) / gridDim.x;
  const int ntile = (int)((r1 - r0 + kDfRows - 1) / kDfRows);
  // mbarrier parities follow from the fill order: code stage g & 1 takes
  // groups g, g+2, ... and codebook buffer m & 1 takes subspaces m, m+2, ...
  // of every tile, so the n-th fill of a buffer is awaited with parity n & 1;
  // `cbase` / `bbase` count the fills of earlier tiles.  A wait that gives up
  // marks `to`; the block leaves together at the next barrier.
  uint32_t cbase0 = 0u, cbase1 = 0u, bbase0 = 0u, bbase1 = 0u;
  bool to = false, stop = false;

  auto issue_codes = [&](int64_t tr0, int g) {   // group g of the tile at tr0 -> stage g & 1
    const int sidx = g & 1;
    const uint32_t b = smem_addr(&bar[sidx]);
    mbar_arrive_expect_tx(b, kDfStageBytes);
    const uint32_t dst = smem_addr(st + sidx * kDfStageBytes);
#pragma unroll
    for (int q = 0; q < 4; ++q)
      tma_load_2d(dst + q * (kDfStageBytes / 4), &tmap, g * kDfStageCodes, (int)(tr0 + q * 256), b,
                  pol_codes);
  };
  auto issue_book = [&](int m) {                 // subspace m's codebooks -> buffer m & 1
    const int bidx = m & 1;
    const uint32_t b = smem_addr(&bar[2 + bidx]);
    mbar_arrive_expect_tx(b, cbb);
    bulk_g2s(smem_addr(cb + (size_t)bidx * align_up(cbf, 256)), a.C + (size_t)m * cbf, cbb, b);
  };
  auto wait_bar = [&](int i, uint32_t parity) {
    const uint32_t b = smem_addr(&bar[i]);
    if (!mbar_try_wait(b, parity) && !mbar_wait_bounded(b, parity)) to = true;
  };

  // rows this thread decodes (r and r + 512 of the tile) and their codes
  uint4 cw[2] = {make_uint4(0, 0, 0, 0), make_uint4(0, 0, 0, 0)};
  // FMA role: rows rg*8 .. rg*8+7, tokens tg*8 .. tg*8+7
  const int rg = warp * 8 + (lane >> 2), tg = lane & 3;

  for (int ti = 0; ti < ntile && !stop; ++ti) {
    const int64_t tr0 = r0 + (r1 - r0) * ti / ntile;
    const int tn = (int)(r0 + (r1 - r0) * (ti + 1) / ntile - tr0);   // rows of this tile (<= 1024)
    if (tid == 0) {
      issue_codes(tr0, 0);
      if (ng > 1) issue_codes(tr0, 1);
      issue_book(0);
      if (M > 1) issue_book(1);
    }
    unsigned long long acc[8][4];               // rows x token pairs
#pragma unroll
    for (int r = 0; r < 8; ++r)
#pragma unroll
      for (int t = 0; t < 4; ++t) acc[r][t] = 0ull;

    // Decoding subspace m into E buffer m & 1 (and its hidden slice into H
    // buffer m & 1) comes in three pieces, one per pair of dims, so that the
    // shared-memory gathers of one subspace interleave with the FMAs of the
    // previous one inside each warp.
    uint32_t dp0[2], dp1[2];          // the two rows' codewords (levels 0, 1), shared addresses
    uint32_t dout[2];                 // the two rows' slots in the E tile
    bool dok[2];
    auto decode_begin = [&](int m) -> bool {   // waits, codes, addresses
      const int g = m / 8, sidx = g & 1, i = m % 8;
      if (i == 0) wait_bar(sidx, ((sidx ? cbase1 : cbase0) + (uint32_t)(g >> 1)) & 1u);
      wait_bar(2 + (m & 1), (((m & 1) ? bbase1 : bbase0) + (uint32_t)(m >> 1)) & 1u);
      if (to) return false;
      const uint32_t stage = smem_addr(st + sidx * kDfStageBytes);
      const uint32_t book = smem_addr(cb + (size_t)(m & 1) * align_up(cbf, 256));
      const uint32_t E = smem_addr(Es + (size_t)(m & 1) * 128 * kDfGS);
#pragma unroll
      for (int h2 = 0; h2 < 2; ++h2) {
        const int r = tid + h2 * 512;
        if ((i & 3) == 0) {
          // 16-byte chunk q of row r after the 32-byte swizzle
          const int q = (i >> 2) ^ ((r >> 2) & 1);
          cw[h2] = lds_u4(stage + (uint32_t)r * 32u + 16u * q);
        }
        const uint32_t w = (i & 3) == 0 ? cw[h2].x : (i & 3) == 1 ? cw[h2].y
                                                   : (i & 3) == 2 ? cw[h2].z : cw[h2].w;
        const uint32_t c0 = a.fix(w & 0xFFFFu), c1 = a.fix(w >> 16);
        dp0[h2] = book + c0 * 24u;
        dp1[h2] = book + ((uint32_t)a.K + c1) * 24u;
        dout[h2] = E + (uint32_t)((r >> 3) * kDfGS + (r & 7)) * 4u;
        dok[h2] = r < tn;
      }
      // hidden slice: Hs[token group][j][8 tokens], zero past the group
      if (tid < 192) {
        const int t = tid / 6, j = tid % 6;
        float *H = Hs + (size_t)(m & 1) * 4 * kDfGS;
        H[(t >> 3) * kDfGS + j * 8 + (t & 7)] =
            t < a.nb ? __ldg(a.h + (int64_t)(a.t0 + t) * a.D + m * 6 + j) : 0.f;
      }
      return true;
    };
    auto decode_piece = [&](int jp) {          // dims 2jp, 2jp+1 of both rows
#pragma unroll
      for (int h2 = 0; h2 < 2; ++h2)
        if (dok[h2]) {
          const float2 x = lds_f2(dp0[h2] + 8u * jp), y = lds_f2(dp1[h2] + 8u * jp);
          sts_f32(dout[h2] + (2 * jp) * 32u, __fadd_rn(x.x, y.x));
          sts_f32(dout[h2] + (2 * jp + 1) * 32u, __fadd_rn(x.y, y.y));
        }
    };

    if (decode_begin(0)) {
      decode_piece(0);
      decode_piece(1);
      decode_piece(2);
    }
    stop = __syncthreads_or(to);
    if (stop) break;
    if (tid == 0 && M > 2) issue_book(2);                  // buffer 0 is free again
    const bool fa = warp * 64 < tn;                        // warps past the tile skip the FMAs
    for (int m = 0; m < M; ++m) {
      const bool dec = m + 1 < M && decode_begin(m + 1);
      const uint32_t E = smem_addr(Es + (size_t)(m & 1) * 128 * kDfGS + rg * kDfGS);
      const uint32_t H = smem_addr(Hs + (size_t)(m & 1) * 4 * kDfGS + tg * kDfGS);
#pragma unroll
      for (int jp = 0; jp < 3; ++jp) {
        if (fa) {
#pragma unroll
          for (int j = 2 * jp; j < 2 * jp + 2; ++j) {
            const float4 e0 = lds_f4(E + j * 32u), e1 = lds_f4(E + j * 32u + 16u);
            const float4 h0 = lds_f4(H + j * 32u), h1 = lds_f4(H + j * 32u + 16u);
            const float ev[8] = {e0.x, e0.y, e0.z, e0.w, e1.x, e1.y, e1.z, e1.w};
            const unsigned long long hp[4] = {pack2(h0.x, h0.y), pack2(h0.z, h0.w),
                                              pack2(h1.x, h1.y), pack2(h1.z, h1.w)};
#pragma unroll
            for (int r = 0; r < 8; ++r) {
              const unsigned long long ep = pack2(ev[r], ev[r]);
#pragma unroll
              for (int t = 0; t < 4; ++t) acc[r][t] = fma2(ep, hp[t], acc[r][t]);
            }
          }
        }
        if (dec) decode_piece(jp);
      }
      stop = __syncthreads_or(to);
      if (stop) break;
      if (tid == 0) {
        // decode(m+1) is done: its codebook buffer takes subspace m+3, and the
        // code stage of a finished group takes the group two ahead
        if (m + 3 < M) issue_book(m + 3);
        if ((m + 2) % 8 == 0 && (m + 2) / 8 + 1 < ng) issue_codes(tr0, (m + 2) / 8 + 1);
      }
    }
    if (stop) break;
    cbase0 += (uint32_t)(ng + 1) / 2;
    cbase1 += (uint32_t)ng / 2;
    bbase0 += (uint32_t)(M + 1) / 2;
    bbase1 += (uint32_t)M / 2;
    // epilogue: softcap, logits, per-token best of this thread's rows
    if (warp * 64 < tn) {
#pragma unroll
      for (int t = 0; t < 8; ++t) {
        const int tok = tg * 8 + t;
        ArgBest best{-FLT_MAX, INT_MAX};
#pragma unroll
        for (int r = 0; r < 8; ++r) {
          const int row = rg * 8 + r;
          if (row < tn && tok < a.nb) {
            const int64_t v = tr0 + row;
            float z0, z1;
            unpack2(acc[r][t >> 1], z0, z1);
            const float y = softcap_f((t & 1) ? z1 : z0, a.cap);
            if (a.logits) a.logits[(int64_t)(a.t0 + tok) * a.V + v] = y;
            best = arg_better(best, ArgBest{y, (int)v});
          }
        }
        // combine the 8 row groups of this warp that share the token group
#pragma unroll
        for (int o = 4; o < 32; o <<= 1) best = arg_better(best, arg_shfl_xor(best, o));
        if (lane < 4) wbest[warp * 32 + tok] = best;   // lane == tg here
      }
    } else if (lane < 4) {
      for (int t = 0; t < 8; ++t) wbest[warp * 32 + lane * 8 + t] = ArgBest{-FLT_MAX, INT_MAX};
    }
    __syncthreads();
    if (tid < 32) {
      ArgBest b = cbest[tid];
      for (int w = 0; w < 16; ++w) b = arg_better(b, wbest[w * 32 + tid]);
      cbest[tid] = b;
    }
    __syncthreads();
  }
  griddep_launch_dependents();
  if (a.am_val && tid < a.nb) {
    const int64_t row = (int64_t)(a.t0 + tid) * a.nblk;
    a.am_val[row + blockIdx.x] = cbest[tid].v;
    a.am_idx[row + blockIdx.x] = cbest[tid].i;
    // columns past this grid (a wider grid of another pass shares the layout)
    for (int c = gridDim.x + blockIdx.x; c < a.nblk; c += gridDim.x) {
      a.am_val[row + c] = -FLT_MAX;
      a.am_idx[row + c] = INT_MAX;
    }
  }
  if (tid == 0 && stop) {
    atomicOr(a.err, RQ_DEVERR_TIMEOUT);
    // let copies still in flight land before the CTA's shared memory goes:
    // each buffer's fills complete in order, so waiting for both parities
    // (bounded) covers the last one issued
    for (int i = 0; i < 4; ++i) {
      mbar_wait_bounded(smem_addr(&bar[i]), 0u);
      mbar_wait_bounded(smem_addr(&bar[i]), 1u);
    }
  }
}

size_t decode_fma_smem(int K) {
  const size_t cbf = (size_t)align_up(2 * K * 6, 256);
  return 1024 + 2 * (size_t)kDfStageBytes + 2 * cbf * 4 + 2 * (size_t)kDfEBytes +
         2 * (size_t)kDfHBytes + 4 * 8 + (16 * 32 + 32) * sizeof(ArgBest) + 16;
}

bool decode_fma_applies(int fmt, int64_t V, int D, int M, int L, int K, int B, const float *C,
                        const void *codes, const DevInfo &di) {
  if (fmt != RQ_CODES_U16 || L != 2 || D != 6 * M || M % 8 != 0 || K > 1024 || B < 1) return false;
  if (V < 1 || V > (int64_t)INT_MAX - 2048) return false;
  if ((reinterpret_cast<uintptr_t>(C) & 15) != 0 || (reinterpret_cast<uintptr_t>(codes) & 15) != 0)
    return false;
  return decode_fma_smem(K) <= (size_t)di.max_smem_optin;
}

int decode_fma_blocks(int64_t V, const DevInfo &di) {
  int64_t n = di.sms;
  const int64_t most = (V + 255) / 256;
  if (n > most) n = most;
  return n < 1 ? 1 : (int)n;
}

cudaError_t launch_logits_decode_fma(const float *h, const float *C, const void *codes,
                                     int64_t V, int D, int M, int K, int t0, int nb, float cap,
                                     float *logits, float *am_val, int *am_idx, int nblk,
                                     const DevInfo &di, cudaStream_t s) {
  CUtensorMap tmap;
  const int P = 2 * M;
  if (!encode_tmap_2d_u16(&tmap, codes, (uint64_t)P, (uint64_t)V, (uint64_t)P * 2,
                          kDfStageCodes, 256, CU_TENSOR_MAP_SWIZZLE_32B))
    return cudaErrorInvalidValue;
  const size_t smem = decode_fma_smem(K);
  {
    cudaError_t e = ensure_smem_limit(reinterpret_cast<const void *>(&logits_decode_fma_kernel),
                                      di.device, smem);
    if (e != cudaSuccess) return e;
  }
  DfArgs a;
  a.h = h;
  a.C = C;
  a.V = V;
  a.M = M;
  a.K = K;
  a.D = D;
  a.t0 = t0;
  a.nb = nb;
  a.cap = cap;
  a.logits = logits;
  a.am_val = am_val;
  a.am_idx = am_idx;
  a.nblk = nblk;
  a.fix = make_codefix(K);
  a.err = di.err;
  void *args[] = {&tmap, &a};
  return launch_maybe_pdl(reinterpret_cast<const void *>(&logits_decode_fma_kernel),
                          dim3((unsigned)decode_fma_blocks(V, di)), dim3(kDfThreads), smem, s,
                          args, true);
}

}  // namespace rq

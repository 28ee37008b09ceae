// logits_decode_mma.cu -- logits of a token group by decoding vocabulary rows
// into tensor memory and multiplying them with the hidden states on the
// tcgen05 tensor cores.
//
// "Gemma-2 runtime compression: NF4 + LUT serving", LUT section: the lookup
// + sum equals the decode-then-matmul the pages check it against,
//   z[b][v] = sum_m sum_j h[b][m*ds + j] * (C[m][0][c0][j] + C[m][1][c1][j]);
// Gemma-2's softcap follows.  For a batch this is a dense contraction of the
// decoded rows with the hidden states, which is what the tensor cores do.
//
// fp32 accuracy from tf32 operands: every operand x is split into x_hi = x
// rounded to nearest (even) at the tf32 boundary (low 13 mantissa bits zero,
// so a tf32 MMA reads it exactly) and x_lo = x - x_hi (exact in fp32, at most
// half a tf32 ulp of x), and
//   E . h = E_hi h_hi + E_hi h_lo + E_lo h_hi + (E_lo h_lo, dropped),
// with error about 2^-22 of |E||h| per product.  Two MMAs per tile and
// subspace: E_hi against the 64 columns [h_hi | h_lo] (an N = 64 MMA costs
// what an N = 32 one does), and E_lo against h_hi into the first 32.  The
// tensor core's fp32 accumulation does not round to nearest and its error
// grows with the length of an accumulation chain, so a chain covers 16
// subspaces; the threads that own a finished chain's rows add it into fp32
// registers (round to nearest) before the next chain starts over it.
// Measured against fp64 this keeps the logits near 1e-6 of their scale; one
// chain over all 384 subspaces was ~3e-5.
//
// Design for sm_100a (ds = 6, L = 2, K <= 1024), described below for groups
// of 32 tokens and uint16 codes; DmShape gives the 64-token and 10-bit packed
// instances.  One CTA per SM walks an even share of the vocabulary in passes
// of up to 512 rows = 4 M = 128 tiles, running every subspace once per pass.
// Warp-specialised and mbarrier-driven, nothing waits on a CTA barrier:
//   * 16 decoder warps (4 warpgroups).  Thread (warpgroup g, warp q, lane)
//     owns row 32 q + lane of tile g.  Per subspace it gathers the row's two
//     codewords from the shared-memory codebook, adds them, splits the sum
//     into hi and lo and stores both (6 dims + 2 zero pads each) into its own
//     TMEM lane of a double-buffered A slot with one tcgen05.st: the MMA reads
//     its A operand from tensor memory;
//   * one copy warp: TMA code tiles ({8 codes, 128 rows}, 3 stages of 4
//     subspaces), and per subspace one bulk copy of the codebook pair (48 KB
//     at K = 1024, double-buffered) plus the pre-split hidden operand (2 KB,
//     4-slot ring) on the same barrier, which the decoders wait for;
//   * one MMA warp: per subspace it waits for the A slot alone and issues the
//     2 x 4 MMAs (M = 128, K = 8; A in TMEM, B in shared memory).  Issuing
//     small MMAs costs ~100 cycles each, so nothing else sits on this warp.
//   * TMEM: 4 tiles x 64 accumulator columns, then 2 A slots x 4 tiles x 16.
// Every wait is bounded; a timed-out wait raises a CTA-wide abort flag, the
// copy and MMA warps wait (bounded) for their copies and MMAs in flight, and
// the CTA frees its TMEM and ends.
#include <cfloat>
#include <climits>

#include "rq_common.cuh"

namespace rq {

namespace {

// Shape of one instance: NT tokens per group, FMT the code format.
//   NT = 32: 16 decoder warps, 4 tiles (512 rows) per pass, 32 register sums;
//   NT = 64: 12 decoder warps, 3 tiles (384 rows), 64 register sums (14 warps
//            leave 128 registers a thread, where 18 leave 96).
//   uint16 codes: stages of 4 subspaces, 16 bytes per row (TMA {8 codes,
//   128 rows}); 10-bit packed codes: stages of 32 subspaces, 80 bytes per
//   row (TMA boxes of {40 16-bit units, 128 rows} over the 960-byte rows).
template <int NT, int FMT>
struct DmShape {
  static constexpr int DEC_WARPS = NT == 32 ? 16 : 12;
  static constexpr int THREADS = (DEC_WARPS + 2) * 32;   // + the MMA warp and the copy warp
  static constexpr int TILES = DEC_WARPS / 4;              // M = 128 tiles per pass
  static constexpr int ROWS = TILES * 128;                 // rows per pass
  static constexpr bool PACKED = FMT == RQ_CODES_PACKED10;
  static constexpr int GROUP = PACKED ? 32 : 4;            // subspaces per code stage
  static constexpr int ROW_BYTES = PACKED ? 80 : 16;       // code bytes per row and stage
  static constexpr int STAGE_BYTES = ROWS * ROW_BYTES;
  static constexpr int STAGES = PACKED ? 2 : 3;
  static constexpr int BOX_INNER = ROW_BYTES / 2;          // TMA box inner extent (16-bit units)
  static constexpr int HFLOATS = 2 * NT * 8;               // hidden operand: [h_hi | h_lo] x K = 8
  static constexpr uint32_t ACC = 2 * NT;                  // accumulator columns per tile
  static constexpr uint32_t ACOL = TILES * ACC;            // first A-slot column
  static constexpr uint32_t ASLOT = TILES * 16;            // per slot: tiles x (hi 8, lo 8)
  static_assert(ACOL + 2 * ASLOT <= 512, "tensor memory");
};

constexpr int kDmASlots = 2;                         // A slots: decoding runs 2 subspaces ahead
constexpr int kDmChain = 16;                         // subspaces per accumulation chain
constexpr int kDmHSlots = 4;
constexpr uint32_t kDmTmemCols = 512;

struct DmArgs {
  const float *C;      // [M][2][K][6]
  const float *hop;    // [M][2 NT][8]: per subspace rows 0..NT-1 h_hi, NT..2NT-1 h_lo
  int64_t V;
  int M, K;
  int t0, nb;          // tokens t0 .. t0 + nb - 1
  float cap;
  float *logits;       // [Btot][V] or null
  float *am_val;       // [Btot][nblk] or null (columns past the grid get -inf)
  int *am_idx;
  int nblk;
  CodeFix fix;
  unsigned *err;
};

// Canonical K-major, no-swizzle operand of 32-bit elements: 8-row groups of
// two 128-byte core matrices (K halves 0..3, 4..7); float offset of (row, k).
__host__ __device__ __forceinline__ int opnd_idx(int row, int k) {
  return (row >> 3) * 64 + (k >> 2) * 32 + (row & 7) * 4 + (k & 3);
}

// Shared-memory matrix descriptor (sm_100): start, leading-dimension byte
// offset (between the K halves: 128 B), stride byte offset (between 8-row
// groups: 256 B), all in 16-byte units; version 1; no swizzle.
__device__ __forceinline__ unsigned long long opnd_desc(uint32_t saddr) {
  return (unsigned long long)((saddr >> 4) & 0x3FFFu) | ((unsigned long long)(128 >> 4) << 16) |
         ((unsigned long long)(256 >> 4) << 32) | (1ull << 46);
}

// Instruction descriptor: D fp32, A and B tf32, both K-major, M = 128, N.
__device__ __forceinline__ uint32_t mma_idesc(int n) {
  return (1u << 4) | (2u << 7) | (2u << 10) | ((uint32_t)(n >> 3) << 17) |
         ((uint32_t)(128 >> 4) << 24);
}

// D[tmem] (+)= A[tmem] . B[smem]^T
__device__ __forceinline__ void mma_tf32_ts(uint32_t d, uint32_t a, unsigned long long b,
                                            uint32_t idesc, uint32_t accum) {
  asm volatile(
      "{\n\t.reg .pred p;\n\tsetp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::tf32 [%0], [%1], %2, %3, p;\n\t}\n" ::"r"(d),
      "r"(a), "l"(b), "r"(idesc), "r"(accum));
}

__device__ __forceinline__ void mma_commit(uint32_t bar) {
  asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(
                   bar)
               : "memory");
}

__device__ __forceinline__ void mbar_arrive(uint32_t bar) {
  asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(bar) : "memory");
}

__device__ __forceinline__ void tc_fence_after() {
  asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
}

__device__ __forceinline__ void tc_fence_before() {
  asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
}

__device__ __forceinline__ void tmem_ld16(uint32_t taddr, uint32_t (&r)[16]) {
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x16.b32 {%0, %1, %2, %3, %4, %5, %6, %7, %8, %9, %10, "
      "%11, %12, %13, %14, %15}, [%16];"
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]),
        "=r"(r[7]), "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]),
        "=r"(r[13]), "=r"(r[14]), "=r"(r[15])
      : "r"(taddr));
}

__device__ __forceinline__ void tmem_wait_ld() {
  asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
}

// one row of an A slot in tensor memory: hi[0..5], 0, 0, lo[0..5], 0, 0
__device__ __forceinline__ void tmem_st_hilo(uint32_t taddr, const float (&hi)[6],
                                             const float (&lo)[6]) {
  asm volatile(
      "tcgen05.st.sync.aligned.32x32b.x16.b32 [%0], {%1, %2, %3, %4, %5, %6, %7, %7, %8, %9, %10, "
      "%11, %12, %13, %7, %7};" ::"r"(taddr),
      "r"(__float_as_uint(hi[0])), "r"(__float_as_uint(hi[1])), "r"(__float_as_uint(hi[2])),
      "r"(__float_as_uint(hi[3])), "r"(__float_as_uint(hi[4])), "r"(__float_as_uint(hi[5])),
      "r"(0u), "r"(__float_as_uint(lo[0])), "r"(__float_as_uint(lo[1])),
      "r"(__float_as_uint(lo[2])), "r"(__float_as_uint(lo[3])), "r"(__float_as_uint(lo[4])),
      "r"(__float_as_uint(lo[5])));
}

__device__ __forceinline__ void tmem_wait_st() {
  asm volatile("tcgen05.wait::st.sync.aligned;" ::: "memory");
}

// x rounded to nearest (ties to even) with the low 13 mantissa bits cleared
// (finite inputs of logit magnitude; no overflow handling is needed here)
__device__ __forceinline__ float tf32_hi(float x) {
  const uint32_t u = __float_as_uint(x);
  return __uint_as_float((u + 0xFFFu + ((u >> 13) & 1u)) & 0xFFFFE000u);
}

__device__ __forceinline__ uint4 lds_u4(uint32_t addr) {
  uint4 v;
  asm volatile("ld.shared.v4.u32 {%0, %1, %2, %3}, [%4];"
               : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w)
               : "r"(addr));
  return v;
}

__device__ __forceinline__ uint32_t lds_u32(uint32_t addr) {
  uint32_t v;
  asm volatile("ld.shared.u32 %0, [%1];" : "=r"(v) : "r"(addr));
  return v;
}

}  // namespace

// Hidden operand of one token group, per subspace m: 2 NT rows of K = 8 in the
// canonical K-major layout, rows 0..NT-1 the tokens' hi parts and NT..2NT-1
// their lo parts (dims 6, 7 and tokens past the group are zero).
template <int NT>
__global__ void __launch_bounds__(NT * 8) split_hidden_kernel(const float *__restrict__ h, int D,
                                                              int t0, int nb,
                                                              float *__restrict__ hop) {
  griddep_wait();
  const int m = blockIdx.x, tok = threadIdx.x >> 3, k = threadIdx.x & 7;
  const float x = (k < 6 && tok < nb) ? h[(int64_t)(t0 + tok) * D + m * 6 + k] : 0.f;
  const float xh = tf32_hi(x);
  float *o = hop + (size_t)m * (2 * NT * 8);
  o[opnd_idx(tok, k)] = xh;
  o[opnd_idx(NT + tok, k)] = __fsub_rn(x, xh);
  griddep_launch_dependents();
}

template <int NT, int FMT>
__global__ void __launch_bounds__(DmShape<NT, FMT>::THREADS, 1)
    logits_decode_mma_kernel(const __grid_constant__ CUtensorMap tmap, const DmArgs a) {
  using S_ = DmShape<NT, FMT>;
  constexpr int DW = S_::DEC_WARPS;
  // mbarriers
  constexpr int kBarCodes = 0;                         // code stage g % STAGES landed (TMA)
  constexpr int kBarBook = kBarCodes + S_::STAGES;     // 2: codebook pair + hidden operand (bulk)
  constexpr int kBarFull = kBarBook + 2;               // A slot s % 2 written (decoder warps)
  constexpr int kBarMma = kBarFull + kDmASlots;        // MMAs of subspace s done, on s % 2 (commit)
  constexpr int kBarFlush = kBarMma + kDmASlots;       // a chain read out (decoder warps)
  constexpr int kBars = kBarFlush + 1;

  extern __shared__ __align__(1024) unsigned char smem_raw[];
  unsigned char *smem = smem_raw + ((1024u - (smem_addr(smem_raw) & 1023u)) & 1023u);
  const int cbf = 2 * a.K * 6;                                     // floats per codebook pair
  const uint32_t cbb = (uint32_t)cbf * 4u;
  const size_t cbs = (size_t)align_up(cbf, 256);                   // floats per book buffer
  unsigned char *st = smem;                                        // code stages
  float *cb = reinterpret_cast<float *>(st + S_::STAGES * S_::STAGE_BYTES);
  float *hs = cb + 2 * cbs;                                        // hidden operand slots
  uint64_t *bar = reinterpret_cast<uint64_t *>(hs + kDmHSlots * S_::HFLOATS);
  ArgBest *wbest = reinterpret_cast<ArgBest *>(bar + kBars);      // [decoder warps][NT]
  uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(wbest + DW * NT);
  volatile int *abort_flag = reinterpret_cast<volatile int *>(tmem_slot + 1);

  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  if (tid == 0) {
    prefetch_tmap(&tmap);
    for (int i = 0; i < kBars; ++i)
      mbar_init(smem_addr(&bar[i]),
                ((i >= kBarFull && i < kBarFull + kDmASlots) || i == kBarFlush) ? (uint32_t)DW
                                                                                : 1u);
    fence_mbar_init();
    *abort_flag = 0;
  }
  if (warp == DW) {
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(
                     smem_addr(tmem_slot)),
                 "r"(kDmTmemCols));
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;");
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  griddep_wait();

  const int M = a.M, G = a.M / S_::GROUP, NC = (a.M + kDmChain - 1) / kDmChain;
  const int64_t r0 = a.V * blockIdx.x / gridDim.x, r1 = a.V * (blockIdx.x + 1) / gridDim.x;
  const int npass = (int)((r1 - r0 + S_::ROWS - 1) / S_::ROWS);   // full passes, then the rest
  const int S = npass * M;                   // steps: (pass, subspace)
  const int NG = npass * G;                  // code groups
  auto bar_at = [&](int i) { return smem_addr(&bar[i]); };

  if (warp == DW + 1) {
    // ------------------------------------------------------------ copies
    // code tiles, codebooks and hidden operands; a buffer is refilled once
    // the A slot of the step that read it is full (its decode is done, and
    // the decoders had waited for the MMAs of two steps before)
    if (lane == 0 && S > 0) {
      const uint64_t pol_codes = l2_policy_evict_first();
      int last_codes[S_::STAGES], last_book[2] = {-1, -1};
      for (int i = 0; i < S_::STAGES; ++i) last_codes[i] = -1;
      bool to = false;
      auto wait = [&](int i, uint32_t parity) {
        if (!to && !mbar_try_wait(bar_at(i), parity) && !mbar_wait_bounded(bar_at(i), parity)) {
          to = true;
          *abort_flag = 1;
        }
      };
      auto issue_codes = [&](int g) {
        const int sidx = g % S_::STAGES, p = g / G, gi = g % G;
        const uint32_t b = bar_at(kBarCodes + sidx);
        mbar_arrive_expect_tx(b, S_::STAGE_BYTES);
        const uint32_t dst = smem_addr(st + sidx * S_::STAGE_BYTES);
#pragma unroll
        for (int q = 0; q < S_::ROWS / 128; ++q)
          tma_load_2d(dst + q * (128 * S_::ROW_BYTES), &tmap, gi * S_::BOX_INNER,
                      (int)(r0 + (int64_t)p * S_::ROWS + q * 128), b, pol_codes);
        last_codes[sidx] = g;
      };
      // the decoders wait for both before decoding s, so a full A slot of s
      // also tells the MMA warp that the hidden operand of s has landed
      auto issue_book = [&](int s, int m) {
        const uint32_t b = bar_at(kBarBook + (s & 1));
        mbar_arrive_expect_tx(b, cbb + S_::HFLOATS * 4);
        bulk_g2s(smem_addr(cb + (size_t)(s & 1) * cbs), a.C + (size_t)m * cbf, cbb, b);
        bulk_g2s(smem_addr(hs + (s & 3) * S_::HFLOATS), a.hop + (size_t)m * S_::HFLOATS,
                 S_::HFLOATS * 4, b);
        last_book[s & 1] = s;
      };
      for (int g = 0; g < NG && g < S_::STAGES; ++g) issue_codes(g);
      for (int s = 0; s < S && s < 2; ++s) issue_book(s, s % M);
      int p = 0, m = 0;
      for (int s = 0; s < S; ++s) {
        if (*abort_flag) break;
        wait(kBarFull + s % kDmASlots, (uint32_t)(s / kDmASlots) & 1u);   // decode of s done
        if (to) break;
        if (s + 2 < S) issue_book(s + 2, m + 2 < M ? m + 2 : m + 2 - M);
        if (m % S_::GROUP == S_::GROUP - 1) {
          const int g = p * G + m / S_::GROUP;                 // its stage is read out
          if (g + S_::STAGES < NG) issue_codes(g + S_::STAGES);
        }
        if (++m == M) {
          m = 0;
          ++p;
        }
      }
      if (*abort_flag) {
        // let the copies in flight land before the CTA's shared memory goes
        for (int i = 0; i < S_::STAGES; ++i)
          if (last_codes[i] >= 0)
            mbar_wait_bounded(bar_at(kBarCodes + i), (uint32_t)(last_codes[i] / S_::STAGES) & 1u);
        for (int i = 0; i < 2; ++i)
          if (last_book[i] >= 0)
            mbar_wait_bounded(bar_at(kBarBook + i), (uint32_t)(last_book[i] >> 1) & 1u);
        atomicOr(a.err, RQ_DEVERR_TIMEOUT);
      }
    }
  } else if (warp == DW) {
    // ------------------------------------------------------------ MMA issue
    if (lane == 0 && S > 0) {
      const uint32_t idw = mma_idesc(2 * NT), idn = mma_idesc(NT);
      int issued = 0;                          // steps whose MMAs are committed
      bool to = false;
      auto wait = [&](int i, uint32_t parity) {
        if (!to && !mbar_try_wait(bar_at(i), parity) && !mbar_wait_bounded(bar_at(i), parity)) {
          to = true;
          *abort_flag = 1;
        }
      };
      // descriptor of hidden slot i: the start field counts 16-byte units
      const unsigned long long bd0 = opnd_desc(smem_addr(hs));
      int p = 0, m = 0, nt = 0;
      for (int s = 0; s < S; ++s) {
        if (m == 0) {
          const int64_t rows = (r1 - r0) - (int64_t)p * S_::ROWS;
          nt = (int)(((rows < S_::ROWS ? rows : S_::ROWS) + 127) / 128);
        }
        if (*abort_flag) break;
        // A slot of s written (and, as the decoders waited for it, the hidden
        // operand of s landed)
        wait(kBarFull + s % kDmASlots, (uint32_t)(s / kDmASlots) & 1u);
        const int c = p * NC + m / kDmChain;
        const bool first = m % kDmChain == 0;
        // one accumulator set: the previous chain is read out before this one
        // starts over it
        if (first && c >= 1) wait(kBarFlush, (uint32_t)(c - 1) & 1u);
        if (to) break;
        tc_fence_after();
        const uint32_t slot = tmem + S_::ACOL + (uint32_t)(s % kDmASlots) * S_::ASLOT;
        const unsigned long long b =
            bd0 + (unsigned long long)((s & 3) * (S_::HFLOATS * 4 / 16));
#pragma unroll
        for (int t = 0; t < S_::TILES; ++t) {
          if (t < nt) {
            const uint32_t d = tmem + (uint32_t)t * S_::ACC;
            const uint32_t ah = slot + (uint32_t)(t * 16);
            mma_tf32_ts(d, ah, b, idw, first ? 0u : 1u);   // E_hi . [h_hi | h_lo]
            mma_tf32_ts(d, ah + 8u, b, idn, 1u);           // E_lo . h_hi
          }
        }
        mma_commit(bar_at(kBarMma + s % kDmASlots));
        issued = s + 1;
        if (++m == M) {
          m = 0;
          ++p;
        }
      }
      if (*abort_flag) {
        // let the MMAs in flight finish before the CTA's tensor memory goes
        for (int s = issued - kDmASlots; s < issued; ++s)
          if (s >= 0)
            mbar_wait_bounded(bar_at(kBarMma + s % kDmASlots), (uint32_t)(s / kDmASlots) & 1u);
        atomicOr(a.err, RQ_DEVERR_TIMEOUT);
      }
    }
  } else {
    // ------------------------------------------------------------ decoders
    const int wg = warp >> 2, q = warp & 3;
    const int r = wg * 128 + q * 32 + lane;   // this thread's row of a pass
    const uint32_t lane_base = (uint32_t)(q * 32) << 16;
    ArgBest mine[NT / 32];                    // lane l: this warp's best row for token 32 i + l
#pragma unroll
    for (int i = 0; i < NT / 32; ++i) mine[i] = ArgBest{-FLT_MAX, INT_MAX};
    float acc[NT];
    bool to = false;
    auto wait = [&](int i, uint32_t parity) {
      bool ok = to || mbar_try_wait(bar_at(i), parity) || mbar_wait_bounded(bar_at(i), parity);
      ok = __all_sync(0xffffffffu, ok);
      if (!ok && !to) {
        to = true;
        *abort_flag = 1;
      }
    };
    // add chain c (its MMAs are done) into the register sums; tiles past the
    // pass's rows are skipped warp-uniformly but every warp arrives
    auto flush = [&](int nt) {
      if (wg < nt) {
        tc_fence_after();
        const uint32_t base = tmem + lane_base + (uint32_t)wg * S_::ACC;
        uint32_t x[16], y[16];
#pragma unroll
        for (int c0 = 0; c0 < NT; c0 += 16) {
          tmem_ld16(base + (uint32_t)c0, x);
          tmem_ld16(base + (uint32_t)(NT + c0), y);
          tmem_wait_ld();
#pragma unroll
          for (int j = 0; j < 16; ++j)
            acc[c0 + j] = __fadd_rn(acc[c0 + j],
                                    __fadd_rn(__uint_as_float(x[j]), __uint_as_float(y[j])));
        }
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(bar_at(kBarFlush));
    };

    for (int p = 0; p < npass && !to; ++p) {
      const int64_t pr0 = r0 + (int64_t)p * S_::ROWS;
      const int64_t rows = (r1 - pr0) < S_::ROWS ? (r1 - pr0) : S_::ROWS;
      const int nt = (int)((rows + 127) / 128);
#pragma unroll
      for (int t = 0; t < NT; ++t) acc[t] = 0.f;
      uint4 cw = make_uint4(0, 0, 0, 0);
      uint32_t stage = 0;
      for (int m = 0; m < M; ++m) {
        if (__any_sync(0xffffffffu, *abort_flag != 0)) {
          to = true;
          break;
        }
        const int s = p * M + m, ig = m % S_::GROUP;
        if (ig == 0) {
          const int g = p * G + m / S_::GROUP, sidx = g % S_::STAGES;
          wait(kBarCodes + sidx, (uint32_t)(g / S_::STAGES) & 1u);
          if (to) break;
          stage = smem_addr(st + sidx * S_::STAGE_BYTES) + (uint32_t)r * S_::ROW_BYTES;
          if (!S_::PACKED) cw = lds_u4(stage);
        }
        wait(kBarBook + (s & 1), (uint32_t)(s >> 1) & 1u);
        if (s >= kDmASlots)                                     // A slot free
          wait(kBarMma + s % kDmASlots, (uint32_t)((s - kDmASlots) / kDmASlots) & 1u);
        if (to) break;
        // the MMAs of s - 2, the last of the previous chain, are done (waited
        // for above): read it out before the next chain starts over it
        if (m % kDmChain == 1 && m > kDmChain) flush(nt);
        tc_fence_after();
        if (wg < nt) {
          uint32_t c0, c1;
          if (S_::PACKED) {
            // codes 2m and 2m + 1 of the row: bits [20 ig, 20 ig + 20) of its
            // 80-byte slice, LSB first (a field spans at most two words)
            const int bit = 20 * ig, wi = bit >> 5, sh = bit & 31;
            const uint32_t w0 = lds_u32(stage + 4u * wi);
            const uint32_t w1 = lds_u32(stage + 4u * (wi + 1 < 20 ? wi + 1 : wi));
            const uint32_t v = sh == 0 ? w0 : __funnelshift_r(w0, w1, sh);
            c0 = a.fix(v & 1023u);
            c1 = a.fix((v >> 10) & 1023u);
          } else {
            const uint32_t w = ig == 0 ? cw.x : ig == 1 ? cw.y : ig == 2 ? cw.z : cw.w;
            c0 = a.fix(w & 0xFFFFu);
            c1 = a.fix(w >> 16);
          }
          const float *book = cb + (size_t)(s & 1) * cbs;
          const float2 *p0 = reinterpret_cast<const float2 *>(book + c0 * 6);
          const float2 *p1 = reinterpret_cast<const float2 *>(book + (a.K + c1) * 6);
          float hi[6], lo[6];
#pragma unroll
          for (int j2 = 0; j2 < 3; ++j2) {
            const float2 x = p0[j2], y = p1[j2];
            const float e0 = __fadd_rn(x.x, y.x), e1 = __fadd_rn(x.y, y.y);
            hi[2 * j2] = tf32_hi(e0);
            hi[2 * j2 + 1] = tf32_hi(e1);
            lo[2 * j2] = __fsub_rn(e0, hi[2 * j2]);
            lo[2 * j2 + 1] = __fsub_rn(e1, hi[2 * j2 + 1]);
          }
          tmem_st_hilo(tmem + lane_base + S_::ACOL + (uint32_t)(s % kDmASlots) * S_::ASLOT +
                           (uint32_t)(wg * 16),
                       hi, lo);
          tmem_wait_st();
        }
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(bar_at(kBarFull + s % kDmASlots));
      }
      if (to) break;
      // the chains not read inside the loop, once the pass's last MMAs are done
      {
        const int sl = p * M + M - 1;
        wait(kBarMma + sl % kDmASlots, (uint32_t)(sl / kDmASlots) & 1u);
        if (to) break;
        if (NC >= 2 && (NC - 1) * kDmChain + 1 > M - 1) flush(nt);
        flush(nt);
      }

      // epilogue: softcap, logits, per-token best row of this warp
#pragma unroll
      for (int tok = 0; tok < NT; ++tok) {
        ArgBest best{-FLT_MAX, INT_MAX};
        if (r < rows && tok < a.nb) {
          const int64_t v = pr0 + r;
          const float y = softcap_f(acc[tok], a.cap);
          if (a.logits) a.logits[(int64_t)(a.t0 + tok) * a.V + v] = y;
          best = ArgBest{y, (int)v};
        }
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) best = arg_better(best, arg_shfl_xor(best, o));
        if (lane == (tok & 31)) mine[tok >> 5] = arg_better(mine[tok >> 5], best);
      }
    }
#pragma unroll
    for (int i = 0; i < NT / 32; ++i) wbest[warp * NT + 32 * i + lane] = mine[i];
  }

  griddep_launch_dependents();
  tc_fence_before();
  __syncthreads();
  if (a.am_val && tid < a.nb && tid < NT) {
    ArgBest bb{-FLT_MAX, INT_MAX};
    for (int w2 = 0; w2 < DW; ++w2) bb = arg_better(bb, wbest[w2 * NT + tid]);
    const int64_t rowi = (int64_t)(a.t0 + tid) * a.nblk;
    a.am_val[rowi + blockIdx.x] = bb.v;
    a.am_idx[rowi + blockIdx.x] = bb.i;
    for (int c = gridDim.x + blockIdx.x; c < a.nblk; c += gridDim.x) {
      a.am_val[rowi + c] = -FLT_MAX;
      a.am_idx[rowi + c] = INT_MAX;
    }
  }
  if (warp == DW) {
    __syncwarp();
    tc_fence_after();
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem),
                 "r"(kDmTmemCols));
  }
}

namespace {

template <int NT, int FMT>
size_t dm_smem(int K) {
  using S_ = DmShape<NT, FMT>;
  const size_t cbs = (size_t)align_up(2 * K * 6, 256) * 4;
  return 1024 + (size_t)S_::STAGES * S_::STAGE_BYTES + 2 * cbs + kDmHSlots * S_::HFLOATS * 4 +
         (S_::STAGES + 2 + 2 * kDmASlots + 1) * 8 + (size_t)S_::DEC_WARPS * NT * sizeof(ArgBest) +
         16;
}

template <int NT, int FMT>
cudaError_t launch_dm(const float *h, const float *C, const void *codes, int64_t V, int D, int M,
                      int K, int t0, int nb, float cap, float *hop, float *logits, float *am_val,
                      int *am_idx, int nblk, const DevInfo &di, cudaStream_t s) {
  using S_ = DmShape<NT, FMT>;
  if (nb < 1 || nb > NT || M % S_::GROUP != 0) return cudaErrorInvalidValue;
  CUtensorMap tmap;
  const int P = 2 * M;
  // packed rows (P * 10 / 8 bytes, a multiple of 16 as M % 32 == 0) are
  // copied as 16-bit units: the copy moves bytes whatever the element type
  const uint64_t row_bytes = S_::PACKED ? (uint64_t)P * 10 / 8 : (uint64_t)P * 2;
  if (!encode_tmap_2d_u16(&tmap, codes, row_bytes / 2, (uint64_t)V, row_bytes, S_::BOX_INNER, 128,
                          CU_TENSOR_MAP_SWIZZLE_NONE))
    return cudaErrorInvalidValue;
  {
    void *args[] = {&h, &D, &t0, &nb, &hop};
    cudaError_t e = launch_maybe_pdl(reinterpret_cast<const void *>(&split_hidden_kernel<NT>),
                                     dim3((unsigned)M), dim3(NT * 8), 0, s, args, true);
    if (e != cudaSuccess) return e;
  }
  const size_t smem = dm_smem<NT, FMT>(K);
  const void *fn = reinterpret_cast<const void *>(&logits_decode_mma_kernel<NT, FMT>);
  {
    cudaError_t e = ensure_smem_limit(fn, di.device, smem);
    if (e != cudaSuccess) return e;
  }
  DmArgs a;
  a.C = C;
  a.hop = hop;
  a.V = V;
  a.M = M;
  a.K = K;
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
  return launch_maybe_pdl(fn, dim3((unsigned)decode_fma_blocks(V, di)), dim3(S_::THREADS), smem, s,
                          args, true);
}

}  // namespace

size_t decode_mma_smem(int K, int N, int fmt) {
  const bool packed = fmt == RQ_CODES_PACKED10;
  if (N == 32) return packed ? dm_smem<32, RQ_CODES_PACKED10>(K) : dm_smem<32, RQ_CODES_U16>(K);
  return packed ? dm_smem<64, RQ_CODES_PACKED10>(K) : dm_smem<64, RQ_CODES_U16>(K);
}

size_t decode_mma_hop_bytes(int M, int N) { return (size_t)M * 2 * N * 8 * 4; }

bool decode_mma_applies(int fmt, int64_t V, int D, int M, int L, int K, const float *C,
                        const void *codes) {
  if (fmt != RQ_CODES_U16 && fmt != RQ_CODES_PACKED10) return false;
  if (L != 2 || D != 6 * M || K > 1024 || K < 1) return false;
  if (M % (fmt == RQ_CODES_PACKED10 ? 32 : 8) != 0) return false;
  if (V < 1 || V > (int64_t)INT_MAX - 2048) return false;
  return (reinterpret_cast<uintptr_t>(C) & 15) == 0 && (reinterpret_cast<uintptr_t>(codes) & 15) == 0;
}

cudaError_t launch_logits_decode_mma(const float *h, const float *C, const void *codes, int fmt,
                                     int64_t V, int D, int M, int K, int t0, int nb, int N,
                                     float cap, float *hop, float *logits, float *am_val,
                                     int *am_idx, int nblk, const DevInfo &di, cudaStream_t s) {
  const bool packed = fmt == RQ_CODES_PACKED10;
  if (N == 32)
    return packed ? launch_dm<32, RQ_CODES_PACKED10>(h, C, codes, V, D, M, K, t0, nb, cap, hop,
                                                      logits, am_val, am_idx, nblk, di, s)
                  : launch_dm<32, RQ_CODES_U16>(h, C, codes, V, D, M, K, t0, nb, cap, hop, logits,
                                                am_val, am_idx, nblk, di, s);
  if (N == 64)
    return packed ? launch_dm<64, RQ_CODES_PACKED10>(h, C, codes, V, D, M, K, t0, nb, cap, hop,
                                                      logits, am_val, am_idx, nblk, di, s)
                  : launch_dm<64, RQ_CODES_U16>(h, C, codes, V, D, M, K, t0, nb, cap, hop, logits,
                                                am_val, am_idx, nblk, di, s);
  return cudaErrorInvalidValue;
}

}  // namespace rq

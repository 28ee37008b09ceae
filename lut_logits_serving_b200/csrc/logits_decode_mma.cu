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
// fp32 accuracy from fp16 operands.  Both operands are scaled by powers of
// two (exact) so that their magnitudes stay below 2^14: the decoded rows by
// one scale sE taken from a bound on |c0| + |c1| over the codebooks, each
// token's hidden state by its own scale sh[t].  A scaled value x is split into
// x_hi = fp16_rn(x) and x_lo = fp16_rn(x - x_hi) (x - x_hi is exact in fp32),
// so x = x_hi + x_lo within 2^-22 |x| over fp16's normal range, and
//   E . h = E_hi h_hi + E_lo h_hi + E_hi h_lo + (E_lo h_lo, dropped)
// with an error of about 2^-22 of |E||h| per product.  Per tile and subspace
// the A operand is one K = 16 row [E_hi(6) 0 0 | E_lo(6) 0 0] and two MMAs
// with that A accumulate into the same columns: B1 = [h_hi 0 0 | h_hi 0 0]
// (the first two terms) and B2 = [h_lo 0 0 | 0 ...] (the third).  The tensor
// core's fp32 accumulation does not round to nearest and its error grows with
// the length of an accumulation chain, so a chain covers 16 subspaces (32
// MMAs); the threads that own a finished chain's rows add it into fp32
// registers (round to nearest) before the next chain starts over it.  The sums
// are unscaled by 1 / (sE sh[t]), a power of two, before the softcap.
//
// Design for sm_100a (ds = 6, L = 2, K <= 1024); DmShape gives the instances.
// One CTA per SM walks an even share of the vocabulary in passes of up to
// TILES x 128 rows (1024 for 32-token groups), running every
// subspace once per pass, so a subspace's codebook pair (48 KB at K = 1024)
// is copied into shared memory once per pass.  Warp-specialised and
// mbarrier-driven; no CTA barrier inside the loop:
//   * 16 decoder warps.  Warp (g, q) owns lanes 32q..32q+31 of tiles
//     g*RPT .. g*RPT+RPT-1; per subspace each thread gathers its rows' two
//     codewords from the shared codebook, adds them, scales and splits the
//     sums into fp16 hi and lo and stores each row's A operand (8 TMEM
//     columns) into its TMEM lane of a double-buffered A slot;
//   * one copy warp: TMA code tiles (uint16: {8 codes, 128 rows} boxes, stages
//     of 4 subspaces; 10-bit packed rows: stages of 16 subspaces, whose 40
//     bytes start at byte 40j of the row -- 8 bytes off a 16-byte boundary for
//     odd j -- so each box is the 48-byte, 16-byte-aligned window around them,
//     {48 bytes, 128 rows}; bank-scheduled codes: one stage of 16 subspaces,
//     the rows' whole 64-byte slices {32 entries, 128 rows}, which the decoders
//     put back in pair order in place when the stage lands),
//     and per subspace one bulk copy of the codebook pair into a ring of
//     NBOOK buffers plus the pre-split hidden operand (B1, B2) into a ring of
//     6 slots, on one transaction barrier;
//   * one MMA warp: per subspace it waits for the A slot and issues the 2 x
//     TILES MMAs (M = 128, N = tokens, K = 16; A in TMEM, B in shared memory).
// Every buffer has its own release barrier (decoders release a codebook
// buffer and a code stage once their loads are consumed; MMA completion
// releases an A slot and a hidden slot), so no barrier phase is ever awaited
// after it could have been passed again.  Every wait is bounded; a timed-out
// wait raises a CTA-wide abort flag, the copy and MMA warps wait (bounded) for
// their copies and MMAs in flight, the CTA frees its TMEM, sets
// RQ_DEVERR_TIMEOUT and ends.
#include <cfloat>
#include <climits>

#include <cuda_fp16.h>

#include "rq_common.cuh"

namespace rq {

namespace {

// Bulk copy global -> this CTA's shared memory (no multicast) with an L2
// cache policy for the source lines.
__device__ __forceinline__ void bulk_g2s_keep(uint32_t dst, const void *src, uint32_t bytes,
                                              uint32_t bar, uint64_t pol) {
  asm volatile(
      "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes.L2::cache_hint"
      " [%0], [%1], %2, [%3], %4;" ::"r"(dst),
      "l"(src), "r"(bytes), "r"(bar), "l"(pol)
      : "memory");
}

// Shape of one instance: NT tokens per group, FMT the code format.
template <int NT, int FMT>
struct DmShape {
  static constexpr bool PACKED = FMT == RQ_CODES_PACKED10;
  static constexpr bool SCHED = FMT == RQ_CODES_SCHED;
  static constexpr int TILES = NT == 32 ? 8 : 4;                // M = 128 tiles per pass
  static constexpr int RPT = TILES / 4;                         // rows per decoder thread
  static constexpr int DEC_WARPS = 16;                          // 4 lane quarters x 4
  static constexpr int THREADS = (DEC_WARPS + 2) * 32;          // + copy warp + MMA warp
  static constexpr int ROWS = TILES * 128;                      // rows per pass
  static constexpr int GROUP = PACKED || SCHED ? 16 : 4;        // subspaces per code stage
  static constexpr int ROW_BYTES = PACKED ? 48 : SCHED ? 64 : 16;   // code bytes per row and stage
  static constexpr int STAGE_BYTES = ROWS * ROW_BYTES;
  // a scheduled stage (64 KB at 1024 rows) leaves room for one only
  static constexpr int STAGES = SCHED ? 1 : 2;
  static constexpr int NBOOK = (PACKED && NT == 32) ? 2 : 3;    // codebook buffers (shared memory)
  static constexpr int BOX_INNER = ROW_BYTES / 2;               // TMA box inner extent (16-bit units)
  static constexpr int HBYTES = 2 * NT * 32;                    // B1 and B2: NT rows x 16 fp16 each
  static constexpr uint32_t ACOL = TILES * NT;                  // first A-slot column
  static constexpr uint32_t ASLOT = TILES * 8;                  // A-slot columns: 8 per tile
  // Running sums per decoder thread: RPT x NT; the first 32 in registers, the
  // rest in this thread's TMEM lane from column RCOL (each of the 4 warps of a
  // lane quarter owns XSUMS columns).  With 18 warps no SM sub-partition has
  // more than 5, so a thread has at most 96 registers.
  static constexpr int XSUMS = RPT * NT - 32;
  static constexpr uint32_t RCOL = ACOL + 2 * ASLOT;
  static_assert(RCOL + 4 * XSUMS <= 512, "tensor memory");
};

constexpr int kDmASlots = 2;                         // A slots: decoding runs 2 subspaces ahead
constexpr int kDmHSlots = 6;                         // hidden-operand slots
constexpr int kDmChain = 16;                         // subspaces per accumulation chain
constexpr uint32_t kDmTmemCols = 512;
constexpr int kDmCbBlocks = 64;                      // codebook-bound partial blocks
constexpr int kDmHopHead = 1024;                     // bytes: token scales, bound partials

struct DmArgs {
  const float *C;      // [M][2][K][6]
  const float *hop;    // scales + [M][B1 | B2] fp16 hidden operands (see dm_hop_*)
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

// Scratch ("hop") layout: floats [0, 64) the token scales sh[t]; floats
// [64, 64 + 2 kDmCbBlocks) the codebook-bound partials (level 0, level 1);
// from byte kDmHopHead the hidden operands, HBYTES per subspace.
__host__ __device__ __forceinline__ const float *dm_hop_scales(const float *hop) { return hop; }
__host__ __device__ __forceinline__ const float *dm_hop_bounds(const float *hop) { return hop + 64; }

// Largest power of two s (clamped to 2^-60 .. 2^60) with bound * s < 2^14; 1
// for a bound that is zero, infinite or NaN.  Exact scaling keeps every
// product the one the unscaled operands give.
__device__ __forceinline__ float dm_pow2_scale(float bound) {
  if (!(bound > 0.f) || !(bound <= FLT_MAX)) return 1.f;
  int e;
  frexpf(bound, &e);                    // bound = f 2^e, f in [0.5, 1)
  int k = 14 - e;
  k = k < -60 ? -60 : (k > 60 ? 60 : k);
  return ldexpf(1.f, k);
}

// Canonical K-major, no-swizzle operand of 16-bit elements, K = 16 per row:
// 8-row groups of two 128-byte core matrices (K halves 0..7, 8..15); byte
// offset of (row, k).
__host__ __device__ __forceinline__ int opnd_byte(int row, int k) {
  return (row >> 3) * 256 + (k >> 3) * 128 + (row & 7) * 16 + (k & 7) * 2;
}

// Shared-memory matrix descriptor (sm_100): start, leading-dimension byte
// offset (between the K halves: 128 B), stride byte offset (between 8-row
// groups: 256 B), all in 16-byte units; version 1; no swizzle.
__device__ __forceinline__ unsigned long long opnd_desc(uint32_t saddr) {
  return (unsigned long long)((saddr >> 4) & 0x3FFFu) | ((unsigned long long)(128 >> 4) << 16) |
         ((unsigned long long)(256 >> 4) << 32) | (1ull << 46);
}

// Instruction descriptor, kind::f16: D fp32, A and B both fp16 (format 0),
// both K-major, M = 128, N.
__device__ __forceinline__ uint32_t mma_idesc_f16(int n) {
  return (1u << 4) | ((uint32_t)(n >> 3) << 17) | ((uint32_t)(128 >> 4) << 24);
}

// D[tmem] (+)= A[tmem] . B[smem]^T, fp16 operands, fp32 accumulation
__device__ __forceinline__ void mma_f16_ts(uint32_t d, uint32_t a, unsigned long long b,
                                           uint32_t idesc, uint32_t accum) {
  asm volatile(
      "{\n\t.reg .pred p;\n\tsetp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], [%1], %2, %3, p;\n\t}\n" ::"r"(d),
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

__device__ __forceinline__ void tmem_st16(uint32_t taddr, const uint32_t (&r)[16]) {
  asm volatile(
      "tcgen05.st.sync.aligned.32x32b.x16.b32 [%0], {%1, %2, %3, %4, %5, %6, %7, %8, %9, %10, "
      "%11, %12, %13, %14, %15, %16};" ::"r"(taddr),
      "r"(r[0]), "r"(r[1]), "r"(r[2]), "r"(r[3]), "r"(r[4]), "r"(r[5]), "r"(r[6]), "r"(r[7]),
      "r"(r[8]), "r"(r[9]), "r"(r[10]), "r"(r[11]), "r"(r[12]), "r"(r[13]), "r"(r[14]),
      "r"(r[15]));
}

__device__ __forceinline__ void tmem_wait_ld() {
  asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
}

// one row of an A slot: 8 columns, {hi01, hi23, hi45, 0, lo01, lo23, lo45, 0}
// (element 2c in the low half of column c)
__device__ __forceinline__ void tmem_st8(uint32_t taddr, const uint32_t (&v)[6]) {
  asm volatile(
      "tcgen05.st.sync.aligned.32x32b.x8.b32 [%0], {%1, %2, %3, %7, %4, %5, %6, %7};" ::"r"(
          taddr),
      "r"(v[0]), "r"(v[1]), "r"(v[2]), "r"(v[3]), "r"(v[4]), "r"(v[5]), "r"(0u));
}

__device__ __forceinline__ void tmem_wait_st() {
  asm volatile("tcgen05.wait::st.sync.aligned;" ::: "memory");
}

__device__ __forceinline__ uint32_t lds_u32(uint32_t addr) {
  uint32_t v;
  asm volatile("ld.shared.u32 %0, [%1];" : "=r"(v) : "r"(addr));
  return v;
}

__device__ __forceinline__ uint4 lds_u4(uint32_t addr) {
  uint4 v;
  asm volatile("ld.shared.v4.u32 {%0, %1, %2, %3}, [%4];"
               : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w)
               : "r"(addr)
               : "memory");
  return v;
}

__device__ __forceinline__ void sts_u16(uint32_t addr, uint32_t v) {
  asm volatile("st.shared.u16 [%0], %1;" ::"r"(addr), "h"((unsigned short)v) : "memory");
}

__device__ __forceinline__ float2 lds_f2(uint32_t addr) {
  float2 v;
  asm volatile("ld.shared.v2.f32 {%0, %1}, [%2];" : "=f"(v.x), "=f"(v.y) : "r"(addr));
  return v;
}

__device__ __forceinline__ uint32_t h2_bits(__half2 h) {
  return *reinterpret_cast<uint32_t *>(&h);
}

// Scaled fp16 split of a pair: x = (a, b) * s; hi = fp16_rn(x), lo =
// fp16_rn(x - hi); the low halves hold a's parts.
__device__ __forceinline__ void split_pair(float a, float b, float s, uint32_t &hi,
                                           uint32_t &lo) {
  const float xa = __fmul_rn(a, s), xb = __fmul_rn(b, s);
  const __half2 h = __floats2half2_rn(xa, xb);
  const float2 hf = __half22float2(h);
  const __half2 l = __floats2half2_rn(__fsub_rn(xa, hf.x), __fsub_rn(xb, hf.y));
  hi = h2_bits(h);
  lo = h2_bits(l);
}

}  // namespace

// Scales of one token group: blocks [0, NT) the tokens' hidden scales sh[t]
// (tokens past the group: 1); blocks [NT, NT + kDmCbBlocks) partial maxima of
// |C| per level over slices of the subspaces.
template <int NT>
__global__ void __launch_bounds__(256) dm_scale_kernel(const float *__restrict__ h, int D,
                                                       int t0, int nb,
                                                       const float *__restrict__ C, int M,
                                                       int K, float *__restrict__ hop) {
  griddep_wait();
  __shared__ float red[2][8];
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  float m0 = 0.f, m1 = 0.f;
  if (blockIdx.x < NT) {
    const int t = blockIdx.x;
    if (t < nb)
      for (int i = tid; i < D; i += 256) m0 = fmaxf(m0, fabsf(h[(int64_t)(t0 + t) * D + i]));
  } else {
    const int j = blockIdx.x - NT;
    const int ma = (int)((int64_t)M * j / kDmCbBlocks);
    const int mb = (int)((int64_t)M * (j + 1) / kDmCbBlocks);
    const int per = K * 6;                               // floats per (subspace, level)
    for (int m = ma; m < mb; ++m) {
      const float *c0 = C + (size_t)m * 2 * per;
      for (int i = tid; i < per; i += 256) {
        m0 = fmaxf(m0, fabsf(c0[i]));
        m1 = fmaxf(m1, fabsf(c0[per + i]));
      }
    }
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) {
    m0 = fmaxf(m0, __shfl_xor_sync(0xffffffffu, m0, o));
    m1 = fmaxf(m1, __shfl_xor_sync(0xffffffffu, m1, o));
  }
  if (lane == 0) {
    red[0][warp] = m0;
    red[1][warp] = m1;
  }
  __syncthreads();
  if (tid == 0) {
    float x0 = 0.f, x1 = 0.f;
    for (int w = 0; w < 8; ++w) {
      x0 = fmaxf(x0, red[0][w]);
      x1 = fmaxf(x1, red[1][w]);
    }
    if (blockIdx.x < NT) {
      hop[blockIdx.x] = dm_pow2_scale(x0);
    } else {
      hop[64 + 2 * (blockIdx.x - NT)] = x0;
      hop[64 + 2 * (blockIdx.x - NT) + 1] = x1;
    }
  }
  griddep_launch_dependents();
}

// Hidden operands of one token group, per subspace m: B1 = [h_hi 0 0 | h_hi 0 0]
// and B2 = [h_lo 0 0 | 0 x 8], NT rows of K = 16 fp16 each in the canonical
// K-major layout (tokens past the group are zero), from h scaled by sh[t].
template <int NT>
__global__ void __launch_bounds__(NT * 16) dm_split_kernel(const float *__restrict__ h, int D,
                                                           int t0, int nb,
                                                           float *__restrict__ hop) {
  griddep_wait();
  const int m = blockIdx.x, tok = threadIdx.x >> 4, k = threadIdx.x & 15, j = k & 7;
  float x = 0.f;
  if (j < 6 && tok < nb)
    x = __fmul_rn(h[(int64_t)(t0 + tok) * D + m * 6 + j], dm_hop_scales(hop)[tok]);
  const __half xh = __float2half_rn(x);
  const __half xl = __float2half_rn(__fsub_rn(x, __half2float(xh)));
  unsigned char *o =
      reinterpret_cast<unsigned char *>(hop) + kDmHopHead + (size_t)m * (2 * NT * 32);
  *reinterpret_cast<__half *>(o + opnd_byte(tok, k)) = xh;                    // B1
  *reinterpret_cast<__half *>(o + NT * 32 + opnd_byte(tok, k)) =              // B2
      k < 8 ? xl : __float2half_rn(0.f);
  griddep_launch_dependents();
}

template <int NT, int FMT>
__global__ void __launch_bounds__(DmShape<NT, FMT>::THREADS, 1)
    logits_decode_mma_kernel(const __grid_constant__ CUtensorMap tmap, const DmArgs a) {
  using S_ = DmShape<NT, FMT>;
  constexpr int DW = S_::DEC_WARPS, RPT = S_::RPT, NB = S_::NBOOK, ST = S_::STAGES;
  // mbarriers
  constexpr int kBarCodes = 0;                       // code stage landed (TMA, tx)
  constexpr int kBarCFree = kBarCodes + ST;          // code stage read out (decoder warps)
  constexpr int kBarBook = kBarCFree + ST;           // codebook pair + hidden operand landed (tx)
  constexpr int kBarBFree = kBarBook + NB;           // codebook buffer read out (decoder warps)
  constexpr int kBarFull = kBarBFree + NB;           // A slot written (decoder warps)
  constexpr int kBarMma = kBarFull + kDmASlots;      // MMAs of a step done (commit)
  constexpr int kBarHFree = kBarMma + kDmASlots;     // hidden slot read by its MMAs (commit)
  constexpr int kBarFlush = kBarHFree + kDmHSlots;   // a chain read out (decoder warps)
  constexpr int kBars = kBarFlush + 1;

  extern __shared__ __align__(1024) unsigned char smem_raw[];
  unsigned char *smem = smem_raw + ((1024u - (smem_addr(smem_raw) & 1023u)) & 1023u);
  const int cbf = 2 * a.K * 6;                                     // floats per codebook pair
  const uint32_t cbb = (uint32_t)cbf * 4u;
  const size_t cbs = (size_t)align_up(cbf, 64);                    // floats per book buffer
  unsigned char *st = smem;                                        // code stages
  float *cb = reinterpret_cast<float *>(st + ST * S_::STAGE_BYTES);
  unsigned char *hs = reinterpret_cast<unsigned char *>(cb + NB * cbs);   // hidden slots
  uint64_t *bar = reinterpret_cast<uint64_t *>(hs + kDmHSlots * S_::HBYTES);
  ArgBest *wbest = reinterpret_cast<ArgBest *>(bar + kBars);       // [decoder warps][NT]
  float *inv = reinterpret_cast<float *>(wbest + DW * NT);         // [NT] unscale factors
  float *esc = inv + NT;                                           // [1] sE
  uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(esc + 1);
  volatile int *abort_flag = reinterpret_cast<volatile int *>(tmem_slot + 1);

  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  if (tid == 0) {
    prefetch_tmap(&tmap);
    for (int i = 0; i < kBars; ++i) {
      const bool by_dec = (i >= kBarCFree && i < kBarCFree + ST) ||
                          (i >= kBarBFree && i < kBarBFree + NB) ||
                          (i >= kBarFull && i < kBarFull + kDmASlots) || i == kBarFlush;
      mbar_init(smem_addr(&bar[i]), by_dec ? (uint32_t)DW : 1u);
    }
    fence_mbar_init();
    *abort_flag = 0;
  }
  if (warp == DW) {
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(
                     smem_addr(tmem_slot)),
                 "r"(kDmTmemCols));
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;");
  }
  griddep_wait();
  if (warp == DW + 1) {
    // the operand scales: sE from the bound on |c0| + |c1|, and per token the
    // factor that undoes sE sh[t] (both powers of two)
    float b0 = 0.f, b1 = 0.f;
    for (int i = lane; i < kDmCbBlocks; i += 32) {
      b0 = fmaxf(b0, dm_hop_bounds(a.hop)[2 * i]);
      b1 = fmaxf(b1, dm_hop_bounds(a.hop)[2 * i + 1]);
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) {
      b0 = fmaxf(b0, __shfl_xor_sync(0xffffffffu, b0, o));
      b1 = fmaxf(b1, __shfl_xor_sync(0xffffffffu, b1, o));
    }
    const float se = dm_pow2_scale(b0 + b1);
    for (int t = lane; t < NT; t += 32) inv[t] = 1.f / (se * dm_hop_scales(a.hop)[t]);
    if (lane == 0) *esc = se;
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  const float sE = *esc;

  const int M = a.M, G = a.M / S_::GROUP, NC = (a.M + kDmChain - 1) / kDmChain;
  const int ssh = sched_shift(a.K);          // bank-scheduled entries: (i << ssh) | c
  const int64_t r0 = a.V * blockIdx.x / gridDim.x, r1 = a.V * (blockIdx.x + 1) / gridDim.x;
  const int npass = (int)((r1 - r0 + S_::ROWS - 1) / S_::ROWS);
  const int S = npass * M;                   // steps: (pass, subspace)
  const int NG = npass * G;                  // code groups
  auto bar_at = [&](int i) { return smem_addr(&bar[i]); };

  if (warp == DW + 1) {
    // ------------------------------------------------------------ copies
    if (lane == 0 && S > 0) {
      // codes stream once (evict first); the codebooks (a few tens of MB) are
      // read by every CTA on every pass and should stay in L2 (evict last)
      const uint64_t pol_codes = l2_policy_evict_first(), pol_books = l2_policy_evict_last();
      int last_codes[ST], last_book[NB];
      for (int i = 0; i < ST; ++i) last_codes[i] = -1;
      for (int i = 0; i < NB; ++i) last_book[i] = -1;
      bool to = false;
      auto wait = [&](int i, uint32_t parity) {
        if (!to && !mbar_try_wait(bar_at(i), parity) && !mbar_wait_bounded(bar_at(i), parity)) {
          to = true;
          *abort_flag = 1;
        }
      };
      auto issue_codes = [&](int g) {
        const int sidx = g % ST, p = g / G, gi = g % G;
        const uint32_t b = bar_at(kBarCodes + sidx);
        mbar_arrive_expect_tx(b, S_::STAGE_BYTES);
        const uint32_t dst = smem_addr(st + sidx * S_::STAGE_BYTES);
#pragma unroll
        for (int q = 0; q < S_::TILES; ++q)
          tma_load_2d(dst + q * (128 * S_::ROW_BYTES), &tmap,
                      S_::PACKED  ? ((40 * gi) & ~15) / 2
                      : S_::SCHED ? 0
                                  : gi * S_::BOX_INNER,
                      (int)((S_::SCHED ? (int64_t)gi * a.V : 0) + r0 + (int64_t)p * S_::ROWS +
                            q * 128),
                      b, pol_codes);
        last_codes[sidx] = g;
      };
      auto issue_book = [&](int s) {
        const int m = s % M;
        const uint32_t b = bar_at(kBarBook + s % NB);
        mbar_arrive_expect_tx(b, cbb + S_::HBYTES);
        bulk_g2s_keep(smem_addr(cb + (size_t)(s % NB) * cbs), a.C + (size_t)m * cbf, cbb, b,
                      pol_books);
        bulk_g2s(smem_addr(hs + (s % kDmHSlots) * S_::HBYTES),
                 reinterpret_cast<const unsigned char *>(a.hop) + kDmHopHead +
                     (size_t)m * S_::HBYTES,
                 S_::HBYTES, b);
        last_book[s % NB] = s;
      };
      for (int g = 0; g < NG && g < ST; ++g) issue_codes(g);
      for (int s = 0; s < S && s < NB; ++s) issue_book(s);
      for (int s = 0; s < S; ++s) {
        if (*abort_flag) break;
        const int m = s % M;
        if (s + NB < S) {
          // refill this codebook buffer once every decoder warp has read it;
          // the hidden slot once the MMAs that read it are done
          wait(kBarBFree + s % NB, (uint32_t)(s / NB) & 1u);
          const int s2 = s + NB;
          if (s2 >= kDmHSlots)
            wait(kBarHFree + s2 % kDmHSlots, (uint32_t)((s2 - kDmHSlots) / kDmHSlots) & 1u);
          if (to) break;
          issue_book(s2);
        }
        if (m % S_::GROUP == S_::GROUP - 1) {
          const int g = (s / M) * G + m / S_::GROUP;
          if (g + ST < NG) {
            wait(kBarCFree + g % ST, (uint32_t)(g / ST) & 1u);
            if (to) break;
            issue_codes(g + ST);
          }
        }
      }
      if (*abort_flag) {
        // let the copies in flight land before the CTA's shared memory goes
        for (int i = 0; i < ST; ++i)
          if (last_codes[i] >= 0)
            mbar_wait_bounded(bar_at(kBarCodes + i), (uint32_t)(last_codes[i] / ST) & 1u);
        for (int i = 0; i < NB; ++i)
          if (last_book[i] >= 0)
            mbar_wait_bounded(bar_at(kBarBook + i), (uint32_t)(last_book[i] / NB) & 1u);
        atomicOr(a.err, RQ_DEVERR_TIMEOUT);
      }
    }
  } else if (warp == DW) {
    // ------------------------------------------------------------ MMA issue
    if (lane == 0 && S > 0) {
      const uint32_t idesc = mma_idesc_f16(NT);
      int issued = 0;                          // steps whose MMAs are committed
      bool to = false;
      auto wait = [&](int i, uint32_t parity) {
        if (!to && !mbar_try_wait(bar_at(i), parity) && !mbar_wait_bounded(bar_at(i), parity)) {
          to = true;
          *abort_flag = 1;
        }
      };
      // descriptor of hidden slot 0; the start field counts 16-byte units
      const unsigned long long bd0 = opnd_desc(smem_addr(hs));
      int nt = 0;
      for (int s = 0; s < S; ++s) {
        const int p = s / M, m = s % M;
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
        const unsigned long long b1 =
            bd0 + (unsigned long long)((s % kDmHSlots) * (S_::HBYTES / 16));
        const unsigned long long b2 = b1 + (unsigned long long)(NT * 32 / 16);
#pragma unroll
        for (int t = 0; t < S_::TILES; ++t) {
          if (t < nt) {
            const uint32_t d = tmem + (uint32_t)(t * NT);
            const uint32_t at = slot + (uint32_t)(t * 8);
            mma_f16_ts(d, at, b1, idesc, first ? 0u : 1u);   // E_hi h_hi + E_lo h_hi
            mma_f16_ts(d, at, b2, idesc, 1u);                 // E_hi h_lo
          }
        }
        mma_commit(bar_at(kBarMma + s % kDmASlots));
        mma_commit(bar_at(kBarHFree + s % kDmHSlots));
        issued = s + 1;
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
    const int g = warp >> 2, q = warp & 3;
    const uint32_t lane_base = (uint32_t)(q * 32) << 16;
    ArgBest mine[NT / 32];                    // lane l: this warp's best row for token 32 i + l
#pragma unroll
    for (int i = 0; i < NT / 32; ++i) mine[i] = ArgBest{-FLT_MAX, INT_MAX};
    float acc[32];                            // running sums 0..31 (see DmShape::XSUMS)
    const uint32_t xsum = tmem + lane_base + S_::RCOL + (uint32_t)(g * (S_::XSUMS > 0 ? S_::XSUMS : 0));
    bool to = false;
    auto wait = [&](int i, uint32_t parity) {
      bool ok = to || mbar_try_wait(bar_at(i), parity) || mbar_wait_bounded(bar_at(i), parity);
      ok = __all_sync(0xffffffffu, ok);
      if (!ok && !to) {
        to = true;
        *abort_flag = 1;
      }
    };
    // add the finished chain into the register sums; tiles past the pass's
    // rows are skipped warp-uniformly but every warp arrives
    auto flush = [&](int nt) {
      tc_fence_after();
#pragma unroll
      for (int i = 0; i < RPT; ++i) {
        const int ti = g * RPT + i;
        if (ti < nt) {
#pragma unroll
          for (int c0 = 0; c0 < NT; c0 += 16) {
            const int j0 = i * NT + c0;           // index of these 16 running sums
            uint32_t x[16];
            tmem_ld16(tmem + lane_base + (uint32_t)(ti * NT + c0), x);
            if (j0 < 32) {
              tmem_wait_ld();
#pragma unroll
              for (int j = 0; j < 16; ++j)
                acc[j0 + j] = __fadd_rn(acc[j0 + j], __uint_as_float(x[j]));
            } else {
              uint32_t y[16];
              tmem_ld16(xsum + (uint32_t)(j0 - 32), y);
              tmem_wait_ld();
#pragma unroll
              for (int j = 0; j < 16; ++j)
                y[j] = __float_as_uint(__fadd_rn(__uint_as_float(y[j]), __uint_as_float(x[j])));
              tmem_st16(xsum + (uint32_t)(j0 - 32), y);
            }
          }
        }
      }
      if (S_::XSUMS > 0) tmem_wait_st();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(bar_at(kBarFlush));
    };

    for (int p = 0; p < npass && !to; ++p) {
      const int64_t pr0 = r0 + (int64_t)p * S_::ROWS;
      const int64_t rows = (r1 - pr0) < S_::ROWS ? (r1 - pr0) : S_::ROWS;
      const int nt = (int)((rows + 127) / 128);
#pragma unroll
      for (int t = 0; t < 32; ++t) acc[t] = 0.f;
      if (S_::XSUMS > 0) {
        // zero this thread's TMEM running sums (its lane, its columns)
        uint32_t z[16];
#pragma unroll
        for (int j = 0; j < 16; ++j) z[j] = 0u;
#pragma unroll
        for (int c0 = 0; c0 < (S_::XSUMS > 0 ? S_::XSUMS : 0); c0 += 16) tmem_st16(xsum + (uint32_t)c0, z);
        tmem_wait_st();
      }
      uint32_t stage = 0;
      for (int m = 0; m < M; ++m) {
        if (__any_sync(0xffffffffu, *abort_flag != 0)) {
          to = true;
          break;
        }
        const int s = p * M + m, ig = m % S_::GROUP;
        const int gcode = p * G + m / S_::GROUP;
        if (ig == 0) {
          wait(kBarCodes + gcode % ST, (uint32_t)(gcode / ST) & 1u);
          if (to) break;
          stage = smem_addr(st + (gcode % ST) * S_::STAGE_BYTES);
          if (S_::SCHED) {
            // each entry (i << ssh) | c of a row's slice back to position i:
            // the row's 32 codes in pair order, in place (a thread's own rows)
            const uint32_t cmask = (1u << ssh) - 1u;
#pragma unroll
            for (int i = 0; i < RPT; ++i) {
              const int ti = g * RPT + i;
              if (ti < nt) {
                const uint32_t rowa = stage + (uint32_t)(ti * 128 + q * 32 + lane) * 64u;
                uint32_t e[16];
#pragma unroll
                for (int k = 0; k < 4; ++k) {
                  const uint4 v = lds_u4(rowa + 16u * k);
                  e[4 * k] = v.x;
                  e[4 * k + 1] = v.y;
                  e[4 * k + 2] = v.z;
                  e[4 * k + 3] = v.w;
                }
#pragma unroll
                for (int k = 0; k < 32; ++k) {
                  const uint32_t en = (k & 1) ? e[k >> 1] >> 16 : e[k >> 1] & 0xFFFFu;
                  sts_u16(rowa + 2u * ((en >> ssh) & 31u), en & cmask);
                }
              }
            }
          }
        }
        wait(kBarBook + s % NB, (uint32_t)(s / NB) & 1u);
        if (s >= kDmASlots)                                     // A slot free
          wait(kBarMma + s % kDmASlots, (uint32_t)((s - kDmASlots) / kDmASlots) & 1u);
        if (to) break;
        // the MMAs of s - 2, the last of the previous chain, are done (waited
        // for above): read it out before the next chain starts over it
        if (m % kDmChain == kDmASlots - 1 && m > kDmChain) flush(nt);
        tc_fence_after();
        // gather, add, scale and split this thread's rows, one at a time, each
        // stored into its A-slot row as soon as it is ready
        const uint32_t book = smem_addr(cb + (size_t)(s % NB) * cbs);
        const uint32_t slot =
            tmem + lane_base + S_::ACOL + (uint32_t)(s % kDmASlots) * S_::ASLOT;
#pragma unroll
        for (int i = 0; i < RPT; ++i) {
          const int ti = g * RPT + i;
          const int r = ti * 128 + q * 32 + lane;       // row within the pass
          if (ti < nt) {                                // warp-uniform
            uint32_t c0, c1;
            if (S_::PACKED) {
              // codes 2m and 2m + 1 of the row: bits [20 ig, 20 ig + 20) of its
              // group's 40 bytes, which start 8 bytes into the 48-byte window
              // for odd groups; LSB first (a field spans at most two words)
              const uint32_t rowa = stage + (uint32_t)r * S_::ROW_BYTES;
              const int bit = 20 * ig + (((40 * (m / S_::GROUP)) & 8) << 3);
              const int wi = bit >> 5, sh = bit & 31;
              const uint32_t w0 = lds_u32(rowa + 4u * wi);
              const uint32_t w1 =
                  lds_u32(rowa + 4u * (wi + 1 < S_::ROW_BYTES / 4 ? wi + 1 : wi));
              const uint32_t v = sh == 0 ? w0 : __funnelshift_r(w0, w1, sh);
              c0 = a.fix(v & 1023u);
              c1 = a.fix((v >> 10) & 1023u);
            } else if (S_::SCHED) {
              const uint32_t w = lds_u32(stage + (uint32_t)r * 64u + 4u * ig);
              c0 = a.fix(w & 0xFFFFu);
              c1 = a.fix(w >> 16);
            } else {
              const uint32_t w = lds_u32(stage + (uint32_t)r * S_::ROW_BYTES + 4u * ig);
              c0 = a.fix(w & 0xFFFFu);
              c1 = a.fix(w >> 16);
            }
            const uint32_t p0 = book + c0 * 24u, p1 = book + ((uint32_t)a.K + c1) * 24u;
            const float2 x0 = lds_f2(p0), x1 = lds_f2(p0 + 8), x2 = lds_f2(p0 + 16);
            const float2 y0 = lds_f2(p1), y1 = lds_f2(p1 + 8), y2 = lds_f2(p1 + 16);
            uint32_t av[6];
            split_pair(__fadd_rn(x0.x, y0.x), __fadd_rn(x0.y, y0.y), sE, av[0], av[3]);
            split_pair(__fadd_rn(x1.x, y1.x), __fadd_rn(x1.y, y1.y), sE, av[1], av[4]);
            split_pair(__fadd_rn(x2.x, y2.x), __fadd_rn(x2.y, y2.y), sE, av[2], av[5]);
            tmem_st8(slot + (uint32_t)(ti * 8), av);
          }
        }
        // the codebook buffer (and, at a group's end, the code stage) are read:
        // every value loaded from them has been used above
        __syncwarp();
        if (lane == 0) {
          mbar_arrive(bar_at(kBarBFree + s % NB));
          if (ig == S_::GROUP - 1) mbar_arrive(bar_at(kBarCFree + gcode % ST));
        }
        tmem_wait_st();
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
        if (NC >= 2 && (NC - 1) * kDmChain + kDmASlots - 1 > M - 1) flush(nt);
        flush(nt);
      }

      // epilogue: unscale, softcap, logits, per-token best row of this warp;
      // running sums in 16-wide chunks (registers, then TMEM)
      tc_fence_after();
#pragma unroll
      for (int j0 = 0; j0 < RPT * NT; j0 += 16) {
        const int i = j0 / NT, tok0 = j0 % NT;
        float z[16];
        if (j0 < 32) {
#pragma unroll
          for (int j = 0; j < 16; ++j) z[j] = acc[j0 + j];
        } else {
          uint32_t y[16];
          tmem_ld16(xsum + (uint32_t)(j0 - 32), y);
          tmem_wait_ld();
#pragma unroll
          for (int j = 0; j < 16; ++j) z[j] = __uint_as_float(y[j]);
        }
        const int r = (g * RPT + i) * 128 + q * 32 + lane;
        const int64_t v = pr0 + r;
#pragma unroll
        for (int j = 0; j < 16; ++j) {
          const int tok = tok0 + j;
          ArgBest best{-FLT_MAX, INT_MAX};
          if (tok < a.nb && r < rows) {
            const float y = softcap_f(__fmul_rn(z[j], inv[tok]), a.cap);
            if (a.logits) a.logits[(int64_t)(a.t0 + tok) * a.V + v] = y;
            best = ArgBest{y, (int)v};
          }
#pragma unroll
          for (int o = 16; o > 0; o >>= 1) best = arg_better(best, arg_shfl_xor(best, o));
          if (lane == (tok & 31)) mine[tok >> 5] = arg_better(mine[tok >> 5], best);
        }
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
  const size_t cbs = (size_t)align_up(2 * K * 6, 64) * 4;
  return 1024 + (size_t)S_::STAGES * S_::STAGE_BYTES + (size_t)S_::NBOOK * cbs +
         (size_t)kDmHSlots * S_::HBYTES +
         (2 * S_::STAGES + 2 * S_::NBOOK + 2 * kDmASlots + kDmHSlots + 1) * 8 +
         (size_t)S_::DEC_WARPS * NT * sizeof(ArgBest) + (NT + 1) * 4 + 16;
}

template <int NT, int FMT>
cudaError_t launch_dm(const float *h, const float *C, const void *codes, int64_t V, int D, int M,
                      int K, int t0, int nb, float cap, float *hop, float *logits, float *am_val,
                      int *am_idx, int nblk, const DevInfo &di, cudaStream_t s) {
  using S_ = DmShape<NT, FMT>;
  if (nb < 1 || nb > NT || M % S_::GROUP != 0 || M % 8 != 0) return cudaErrorInvalidValue;
  CUtensorMap tmap;
  const int P = 2 * M;
  // packed rows (P * 10 / 8 bytes, a multiple of 16 as M % 32 == 0) are
  // copied as 16-bit units: the copy moves bytes whatever the element type;
  // the last window of a row ends at the row's end (its group starts 8 bytes
  // past a 16-byte boundary)
  const uint64_t row_bytes = S_::PACKED ? (uint64_t)P * 10 / 8 : (uint64_t)P * 2;
  // the bank-scheduled layout is chunk-major [P/32][V][32]: rows of 64 bytes
  const bool ok_map =
      S_::SCHED ? encode_tmap_2d_u16(&tmap, codes, 32, (uint64_t)V * (P / 32), 64, 32, 128,
                                     CU_TENSOR_MAP_SWIZZLE_NONE)
                : encode_tmap_2d_u16(&tmap, codes, row_bytes / 2, (uint64_t)V, row_bytes,
                                     S_::BOX_INNER, 128, CU_TENSOR_MAP_SWIZZLE_NONE);
  if (!ok_map) return cudaErrorInvalidValue;
  {
    void *args[] = {&h, &D, &t0, &nb, &C, &M, &K, &hop};
    cudaError_t e = launch_maybe_pdl(reinterpret_cast<const void *>(&dm_scale_kernel<NT>),
                                     dim3((unsigned)(NT + kDmCbBlocks)), dim3(256), 0, s, args,
                                     true);
    if (e != cudaSuccess) return e;
  }
  {
    void *args[] = {&h, &D, &t0, &nb, &hop};
    cudaError_t e = launch_maybe_pdl(reinterpret_cast<const void *>(&dm_split_kernel<NT>),
                                     dim3((unsigned)M), dim3(NT * 16), 0, s, args, true);
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
  if (fmt == RQ_CODES_PACKED10)
    return N == 32 ? dm_smem<32, RQ_CODES_PACKED10>(K) : dm_smem<64, RQ_CODES_PACKED10>(K);
  if (fmt == RQ_CODES_SCHED)
    return N == 32 ? dm_smem<32, RQ_CODES_SCHED>(K) : dm_smem<64, RQ_CODES_SCHED>(K);
  return N == 32 ? dm_smem<32, RQ_CODES_U16>(K) : dm_smem<64, RQ_CODES_U16>(K);
}

size_t decode_mma_hop_bytes(int M, int N, int K) {
  (void)K;
  return (size_t)kDmHopHead + (size_t)M * 2 * N * 32;
}

bool decode_mma_shape_ok(int fmt, int64_t V, int D, int M, int L, int K) {
  if (fmt != RQ_CODES_U16 && fmt != RQ_CODES_PACKED10 && fmt != RQ_CODES_SCHED) return false;
  if (L != 2 || D != 6 * M || K > 1024 || K < 1) return false;
  if (M % (fmt == RQ_CODES_PACKED10 ? 32 : fmt == RQ_CODES_SCHED ? 16 : 8) != 0) return false;
  if (fmt == RQ_CODES_SCHED && V * (M / 16) > (int64_t)INT_MAX - 2048) return false;
  return V >= 1 && V <= (int64_t)INT_MAX - 2048;
}

bool decode_mma_applies(int fmt, int64_t V, int D, int M, int L, int K, const float *C,
                        const void *codes) {
  return decode_mma_shape_ok(fmt, V, D, M, L, K) && (reinterpret_cast<uintptr_t>(C) & 15) == 0 &&
         (reinterpret_cast<uintptr_t>(codes) & 15) == 0;
}

cudaError_t launch_logits_decode_mma(const float *h, const float *C, const void *codes, int fmt,
                                     int64_t V, int D, int M, int K, int t0, int nb, int N,
                                     float cap, float *hop, float *logits, float *am_val,
                                     int *am_idx, int nblk, const DevInfo &di, cudaStream_t s) {
#define RQ_DM_LAUNCH(NT_, FMT_)                                                                  \
  launch_dm<NT_, FMT_>(h, C, codes, V, D, M, K, t0, nb, cap, hop, logits, am_val, am_idx, nblk,  \
                       di, s)
  if (N != 32 && N != 64) return cudaErrorInvalidValue;
  if (fmt == RQ_CODES_PACKED10)
    return N == 32 ? RQ_DM_LAUNCH(32, RQ_CODES_PACKED10) : RQ_DM_LAUNCH(64, RQ_CODES_PACKED10);
  if (fmt == RQ_CODES_SCHED)
    return N == 32 ? RQ_DM_LAUNCH(32, RQ_CODES_SCHED) : RQ_DM_LAUNCH(64, RQ_CODES_SCHED);
  return N == 32 ? RQ_DM_LAUNCH(32, RQ_CODES_U16) : RQ_DM_LAUNCH(64, RQ_CODES_U16);
#undef RQ_DM_LAUNCH
}

}  // namespace rq

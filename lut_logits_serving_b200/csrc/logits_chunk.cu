// logits_chunk.cu -- LUT lookup+sum logits for small token counts (B <= 4),
// the code matrix streamed once from HBM.
//
// "Gemma-2 runtime compression: NF4 + LUT serving", LUT section: output
// logits by lookup + sum over each vocabulary row's codes instead of the
// full matmul, followed by Gemma-2's softcap:
//   z[b][v] = sum_p T[p][code[v][p]][b],   y = cap * tanh(z / cap).
//
// Design for sm_100a.  One token's tables are P*K*4 bytes (3.1 MB at the
// Gemma-2 shape): far more than one SM's shared memory, but a chunk of PC
// (m, l) pairs (PC*K*TB*4 = 128 KB) fits.  The grid is nch x cpc CTAs, one
// per SM: CTA (c, s) keeps table chunk c resident in shared memory for its
// whole life and streams slice s of the vocabulary:
//   * each tile of R rows arrives as TMA 2-D boxes {PC codes, 256 rows} of
//     the uint16 code matrix -- a 2*PC-byte slice (16, 32 or 64 bytes,
//     aligned to its own size) of every 2*P-byte row -- into an NST-deep
//     ring of stages, with the TMA swizzle matching the slice width so the
//     16-byte shared loads of consecutive rows fall in distinct bank groups;
//     the code stream carries an L2 evict-first policy;
//   * TPR threads own one row (PPT pairs each), do their table lookups from
//     shared memory and sum TB tokens in fp32 registers; the TPR partial
//     sums meet by a warp shuffle and land in partial[c][b][v];
//   * there is no block barrier per tile: the last warp to finish a stage
//     re-arms it with the TMA copy of the tile NST ahead;
//   * a second kernel adds the nch chunk sums in order, applies the softcap,
//     writes the logits and reduces the argmax (its last block finishes it).
#include <cfloat>
#include <climits>
#include <utility>

#include "rq_common.cuh"

namespace rq {

struct ChunkArgs {
  const float *lut;   // [P][K][TB]
  float *partial;     // [nch][B][V]
  unsigned long long *keys;  // reduce-kernel argmax keys [B], zeroed here
  int early_codes;    // fetch code tiles before waiting for the previous kernel
  int64_t V;
  int64_t ntiles;     // tiles of R rows
  int P, K, B, nch, cpc;
  CodeFix fix;
  unsigned *err;
  const uint8_t *rot;  // RQ_CODES_PACKED10_ROT: rotations [P/32][V]
};

// Plain uint16 codes: TPR threads per row, 1024 threads.  Bank-scheduled codes
// (one token): one thread per row owns the row's whole 32-pair slice, the
// unit the schedule was made for, 512 threads.  Byte codes: one thread per
// row and 32-pair slice (32 bytes), 512 threads.  10-bit codes (one token,
// M*L % 64 == 0): one thread per row and 32-pair slice, whose 40 bytes start
// at byte 40c of the row -- 8 bytes off a 16-byte boundary for odd c -- so
// the TMA box is the 48-byte, 16-byte-aligned window around it.
template <int TB, int FMT>
struct ChunkShape {
  static constexpr bool PK10 = FMT == RQ_CODES_PACKED10 || FMT == RQ_CODES_PACKED10_ROT;
  static constexpr bool WHOLE = FMT == RQ_CODES_SCHED || FMT == RQ_CODES_U8 || PK10;
  static constexpr int PC = WHOLE ? 32 : (TB == 1 ? 32 : (TB == 2 ? 16 : 8));  // pairs/chunk
  static constexpr int PPT = WHOLE ? 32 : (TB == 4 ? 8 : 16);                  // pairs/thread
  static constexpr int TPR = PC / PPT;                          // threads per row
  static constexpr int THREADS = WHOLE ? 512 : 1024;
  static constexpr int WARPS = THREADS / 32;
  static constexpr int R = THREADS / TPR;                       // rows per tile
  static constexpr int CB = FMT == RQ_CODES_U8 ? 1 : 2;         // bytes per code
  static constexpr int ROWB = PK10 ? 48 : PC * CB;              // code bytes per row slice
  static constexpr int BOXES = R / 256;
  static constexpr int BOX_BYTES = 256 * ROWB;
  static constexpr int STAGE_BYTES = R * ROWB;
  static constexpr int CPV = 16 / CB;                           // codes per 16-byte vector
  static constexpr int NQ = PK10 ? 3 : PPT / CPV;               // 16-byte vectors per thread
};

// 16-byte chunk j of row r (row index inside a 1024-byte-aligned TMA box) as
// placed by the TMA swizzle whose span equals the row width.
template <int ROWB>
__device__ __forceinline__ int swz(int j, int r) {
  if (ROWB == 64) return j ^ ((r >> 1) & 3);
  if (ROWB == 32) return j ^ ((r >> 2) & 1);
  return j;
}

template <int KT>
__device__ __forceinline__ uint32_t fix_code(uint32_t c, const CodeFix &f) {
  if (KT > 0 && (KT & (KT - 1)) == 0) return c & (uint32_t)(KT - 1);
  return f(c);
}

// Table entry at byte address `addr` (+ immediate OFF) of shared memory,
// TB tokens wide.  Plain (non-volatile) asm: the table is written before a
// __syncthreads and never again, so these loads may be scheduled freely.
template <int TB, int OFF>
__device__ __forceinline__ void add_entry(uint32_t addr, float (&acc)[TB]) {
  if (TB == 1) {
    float x;
    asm("ld.shared.f32 %0, [%1+%2];" : "=f"(x) : "r"(addr), "n"(OFF));
    acc[0] += x;
  } else if (TB == 2) {
    float x, y;
    asm("ld.shared.v2.f32 {%0, %1}, [%2+%3];" : "=f"(x), "=f"(y) : "r"(addr), "n"(OFF));
    acc[0] += x;
    acc[1] += y;
  } else {
    float x, y, z, w;
    asm("ld.shared.v4.f32 {%0, %1, %2, %3}, [%4+%5];"
        : "=f"(x), "=f"(y), "=f"(z), "=f"(w)
        : "r"(addr), "n"(OFF));
    acc[0] += x;
    acc[1] += y;
    acc[2] += z;
    acc[3] += w;
  }
}

// Runtime-K variant: the pair offset is a register.
template <int TB>
__device__ __forceinline__ void add_entry_rt(uint32_t addr, float (&acc)[TB]) {
  add_entry<TB, 0>(addr, acc);
}

// 8 consecutive pairs (one 16-byte code vector) of one row; `tbase` is the
// shared byte address of the first of those 8 tables.
template <int TB, int KT>
__device__ __forceinline__ void lookup8(uint32_t tbase, int K, uint4 w, const CodeFix &f,
                                        float (&acc)[TB]) {
  const uint32_t ws[4] = {w.x, w.y, w.z, w.w};
  if (KT > 0) {
    constexpr int PB = KT * TB * 4;  // bytes per table
#pragma unroll
    for (int q = 0; q < 4; ++q) {
      const uint32_t c0 = fix_code<KT>(ws[q] & 0xFFFFu, f);
      const uint32_t c1 = fix_code<KT>(ws[q] >> 16, f);
      switch (q) {  // immediates must be literal constants per unrolled step
        case 0:
          add_entry<TB, 0 * PB>(tbase + c0 * (TB * 4), acc);
          add_entry<TB, 1 * PB>(tbase + c1 * (TB * 4), acc);
          break;
        case 1:
          add_entry<TB, 2 * PB>(tbase + c0 * (TB * 4), acc);
          add_entry<TB, 3 * PB>(tbase + c1 * (TB * 4), acc);
          break;
        case 2:
          add_entry<TB, 4 * PB>(tbase + c0 * (TB * 4), acc);
          add_entry<TB, 5 * PB>(tbase + c1 * (TB * 4), acc);
          break;
        default:
          add_entry<TB, 6 * PB>(tbase + c0 * (TB * 4), acc);
          add_entry<TB, 7 * PB>(tbase + c1 * (TB * 4), acc);
          break;
      }
    }
  } else {
    const uint32_t pb = (uint32_t)K * TB * 4;
#pragma unroll
    for (int q = 0; q < 4; ++q) {
      const uint32_t c0 = fix_code<KT>(ws[q] & 0xFFFFu, f);
      const uint32_t c1 = fix_code<KT>(ws[q] >> 16, f);
      add_entry_rt<TB>(tbase + (2 * q) * pb + c0 * (TB * 4), acc);
      add_entry_rt<TB>(tbase + (2 * q + 1) * pb + c1 * (TB * 4), acc);
    }
  }
}

// RQ_CODES_U8: 16 consecutive pairs (one 16-byte vector of byte codes) of
// one row; `tbase` is the shared byte address of the first of those tables.
template <int TB, int KT>
__device__ __forceinline__ void lookup16_u8(uint32_t tbase, int K, uint4 w, const CodeFix &f,
                                            float (&acc)[TB]) {
  const uint32_t ws[4] = {w.x, w.y, w.z, w.w};
  const uint32_t pb = (uint32_t)(KT > 0 ? KT : K) * TB * 4;   // bytes per table
#pragma unroll
  for (int q = 0; q < 4; ++q)
#pragma unroll
    for (int b = 0; b < 4; ++b) {
      const uint32_t c = fix_code<KT>((ws[q] >> (8 * b)) & 0xFFu, f);
      add_entry_rt<TB>(tbase + (uint32_t)(4 * q + b) * pb + c * (TB * 4), acc);
    }
}

__device__ __forceinline__ float lds_f32(uint32_t addr) {
  float x;
  asm("ld.shared.f32 %0, [%1];" : "=f"(x) : "r"(addr));
  return x;
}

// RQ_CODES_SCHED, one token: the 32 entries (i << KSH | c) of a row's chunk
// slice (four 16-byte code vectors), each the word offset of its table entry
// in the chunk's 32 tables of stride 2^KSH at shared address `tbase`.  All
// 32 loads are issued before any add; the sum is a tree.  The (5 + KSH)-bit
// masks keep every address aligned and inside the 32 * 2^KSH * 4 bytes of
// tables.
template <int KSH, int N>
__device__ __forceinline__ float chunk32_sched_tb1(uint32_t tbase, const uint4 (&w)[N]) {
  static_assert(N == 4, "a scheduled slice is four 16-byte vectors");
  constexpr uint32_t EM = (1u << (5 + KSH)) - 1u;
  const uint32_t ws[16] = {w[0].x, w[0].y, w[0].z, w[0].w, w[1].x, w[1].y, w[1].z, w[1].w,
                           w[2].x, w[2].y, w[2].z, w[2].w, w[3].x, w[3].y, w[3].z, w[3].w};
  float x[32];
#pragma unroll
  for (int q = 0; q < 16; ++q) {
    x[2 * q] = lds_f32(tbase + ((ws[q] & EM) << 2));
    // high entry: ((w & EM << 16) * 2^18) >> 32 = ((w >> 16) & EM) * 4
    x[2 * q + 1] = lds_f32(tbase + __umulhi(ws[q] & (EM << 16), 1u << 18));
  }
#pragma unroll
  for (int st = 1; st < 32; st <<= 1)
#pragma unroll
    for (int q = 0; q < 32; q += 2 * st) x[q] += x[q + st];
  return x[0];
}

template <int OFF>
__device__ __forceinline__ float lds_f32_imm(uint32_t addr) {
  float x;
  asm("ld.shared.f32 %0, [%1+%2];" : "=f"(x) : "r"(addr), "n"(OFF));
  return x;
}

// Code j of a 32-code, 10-bit slice held LSB-first in x[0..9] (x[10] = 0).
template <int J>
__device__ __forceinline__ uint32_t pk10_code(const uint32_t (&x)[11]) {
  return __funnelshift_r(x[(10 * J) >> 5], x[((10 * J) >> 5) + 1], (10 * J) & 31) & 0x3FFu;
}

template <int KT, int... J>
__device__ __forceinline__ void pk10_loads(uint32_t tbase, int K, const uint32_t (&x)[11],
                                           const CodeFix &f, float (&y)[32],
                                           std::integer_sequence<int, J...>) {
  if (KT > 0)   // table offsets as immediates
    ((y[J] = lds_f32_imm<J * KT * 4>(tbase + 4u * fix_code<KT>(pk10_code<J>(x), f))), ...);
  else
    ((y[J] = lds_f32(tbase + (uint32_t)J * K * 4 + 4u * fix_code<KT>(pk10_code<J>(x), f))), ...);
}

// Rotated slices: slot J holds pair (J + rot) mod 32 of the chunk.
template <int KT, int... J>
__device__ __forceinline__ void pk10r_loads(uint32_t tbase, int K, const uint32_t (&x)[11],
                                            const CodeFix &f, int rot, float (&y)[32],
                                            std::integer_sequence<int, J...>) {
  const uint32_t pb = (uint32_t)(KT > 0 ? KT : K) * 4u;
  ((y[J] = lds_f32(tbase + (uint32_t)((J + rot) & 31) * pb + 4u * fix_code<KT>(pk10_code<J>(x), f))),
   ...);
}

// RQ_CODES_PACKED10, one token: the row's 32 codes of this chunk are bits
// [10j, 10j + 10) of its 40-byte slice, which begins 8 bytes into the
// 48-byte window w when `skip8`, else at its start.  All 32 table loads are
// issued before any add; the sum is a tree.
template <int KT, bool ROT>
__device__ __forceinline__ float chunk32_packed_tb1(uint32_t tbase, int K, const uint4 (&w)[3],
                                                    bool skip8, const CodeFix &f, int rot) {
  const uint32_t a[12] = {w[0].x, w[0].y, w[0].z, w[0].w, w[1].x, w[1].y,
                          w[1].z, w[1].w, w[2].x, w[2].y, w[2].z, w[2].w};
  uint32_t x[11];
#pragma unroll
  for (int i = 0; i < 10; ++i) x[i] = skip8 ? a[i + 2] : a[i];
  x[10] = 0u;
  float y[32];
  if (ROT)
    pk10r_loads<KT>(tbase, K, x, f, rot, y, std::make_integer_sequence<int, 32>{});
  else
    pk10_loads<KT>(tbase, K, x, f, y, std::make_integer_sequence<int, 32>{});
#pragma unroll
  for (int st = 1; st < 32; st <<= 1)
#pragma unroll
    for (int q = 0; q < 32; q += 2 * st) y[q] += y[q + st];
  return y[0];
}

__device__ __forceinline__ uint4 ld_shared_v4(uint32_t addr) {
  uint4 v;
  asm volatile("ld.shared.v4.u32 {%0, %1, %2, %3}, [%4];"
               : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w)
               : "r"(addr)
               : "memory");
  return v;
}

__device__ __forceinline__ void fence_proxy_async_smem() {
  asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}

// KSH: the table stride 2^KSH of RQ_CODES_SCHED entries (unused otherwise);
// MINB: CTAs per SM the register budget is made for.
template <int TB, int KT, int NST, int FMT, int KSH, int MINB>
__global__ void __launch_bounds__(ChunkShape<TB, FMT>::THREADS, MINB)
    logits_chunk_u16_kernel(const __grid_constant__ CUtensorMap tmap, const ChunkArgs a) {
  constexpr bool SCHED = FMT == RQ_CODES_SCHED;
  constexpr bool U8 = FMT == RQ_CODES_U8;
  constexpr bool PK10 = FMT == RQ_CODES_PACKED10 || FMT == RQ_CODES_PACKED10_ROT;
  constexpr bool ROT = FMT == RQ_CODES_PACKED10_ROT;
  using S = ChunkShape<TB, FMT>;
  static_assert(!PK10 || (TB == 1 && S::PPT == 32), "a thread owns a whole 10-bit slice");
  static_assert(!SCHED || (TB == 1 && S::PPT == 32), "a thread owns a whole scheduled slice");
  extern __shared__ __align__(1024) unsigned char smem_raw[];
  // 1024-byte alignment (TMA swizzle atoms) by pointer arithmetic, so the
  // compiler keeps the shared address space
  unsigned char *smem = smem_raw + ((1024u - (smem_addr(smem_raw) & 1023u)) & 1023u);
  const int K = KT > 0 ? KT : a.K;
  const int KS = SCHED ? (1 << KSH) : K;     // table stride (entries) in shared memory
  float *Ts = reinterpret_cast<float *>(smem);
  const size_t t_bytes = (size_t)align_up((int64_t)S::PC * KS * TB * 4, 1024);
  unsigned char *stages = smem + t_bytes;
  uint64_t *full = reinterpret_cast<uint64_t *>(stages + (size_t)NST * S::STAGE_BYTES);
  uint64_t *tbar = full + NST;
  unsigned *released = reinterpret_cast<unsigned *>(tbar + 1);
  int *abort_flag = reinterpret_cast<int *>(released + NST);

  const int c = blockIdx.x / a.cpc;          // table chunk of this CTA
  const int sl = blockIdx.x % a.cpc;         // vocabulary slice
  const int64_t t0 = a.ntiles * sl / a.cpc;
  const int64_t t1 = a.ntiles * (sl + 1) / a.cpc;
  const int n = (int)(t1 - t0);              // tiles of this CTA
  const int np = min(S::PC, a.P - c * S::PC);
  const int tid = threadIdx.x, lane = tid & 31;
  // bulk copies need 16-byte sizes and addresses
  const bool bulk_table = (K * TB) % 4 == 0;

  if (tid == 0) {
    prefetch_tmap(&tmap);
    for (int s = 0; s < NST; ++s) {
      mbar_init(smem_addr(&full[s]), 1);
      released[s] = 0u;
    }
    mbar_init(smem_addr(tbar), 1);
    *abort_flag = 0;
    fence_mbar_init();
  }
  __syncthreads();

  const uint64_t pol = l2_policy_evict_first();
  const uint32_t stage0 = smem_addr(stages);
  // Box origin of this CTA's code slice: column c*PC of the [V][P] matrix,
  // or, for the chunk-major scheduled layout [P/32][V][32], rows c32*V + v
  // at column (c % (32/PC)) * PC, or, for 10-bit codes, byte 40c of the row
  // rounded down to 16 bytes.
  const int box_x = SCHED ? (c % (32 / S::PC)) * S::PC : PK10 ? (40 * c) & ~15 : c * S::PC;
  const bool skip8 = PK10 && ((40 * c) & 15) != 0;
  const int64_t box_y0 = SCHED ? (int64_t)(c / (32 / S::PC)) * a.V : 0;
  auto issue = [&](int i, int s) {           // tile t0 + i into stage s
    const uint32_t bar = smem_addr(&full[s]);
    mbar_arrive_expect_tx(bar, S::STAGE_BYTES);
    const int y = (int)(box_y0 + (t0 + i) * S::R);
#pragma unroll
    for (int q = 0; q < S::BOXES; ++q)
      tma_load_2d(stage0 + s * S::STAGE_BYTES + q * S::BOX_BYTES, &tmap, box_x, y + q * 256,
                  bar, pol);
  };
  // When the previous kernel is the table build (which writes nothing the
  // code stream reads) the code tiles start before waiting for it.
  if (!a.early_codes) griddep_wait();
  if (tid == 0)
    for (int s = 0; s < NST && s < n; ++s) issue(s, s);
  if (a.early_codes) griddep_wait();
  if (tid == 0 && blockIdx.x == 0 && a.keys)
    for (int b = 0; b < a.B; ++b) a.keys[b] = 0ull;

  // table chunk c -> shared memory
  const float *src = a.lut + (size_t)c * S::PC * K * TB;
  if (bulk_table) {
    if (tid == 0) {
      const uint32_t tb = smem_addr(tbar);
      const uint32_t per = (uint32_t)K * TB * 4;
      if (!SCHED) {
        mbar_arrive_expect_tx(tb, per * np);
        bulk_g2s(smem_addr(Ts), src, per * np, tb);
      } else {
        mbar_arrive_expect_tx(tb, per * np);
        for (int p = 0; p < np; ++p)
          bulk_g2s(smem_addr(Ts) + (uint32_t)p * KS * TB * 4, src + (size_t)p * K * TB, per, tb);
      }
    }
    if constexpr (SCHED) {
      if (K < KS) {                          // codes >= K read zeros
        const int pad = (KS - K) * TB;
        for (int q = tid; q < np * pad; q += S::THREADS)
          Ts[(q / pad) * KS * TB + K * TB + q % pad] = 0.f;
      }
    }
  } else {
    const int per = KS * TB;
    for (int q = tid; q < np * per; q += S::THREADS) {
      const int pp = q / per, e = q % per;
      Ts[q] = e < K * TB ? __ldg(src + (size_t)pp * K * TB + e) : 0.f;
    }
  }
  __syncthreads();
  const bool table_ok = !bulk_table || mbar_wait_bounded(smem_addr(tbar), 0u);
  if (!table_ok) *reinterpret_cast<volatile int *>(abort_flag) = 1;

  const int r = tid / S::TPR;                // row of the tile owned by this thread
  const int hh = tid % S::TPR;               // which PPT pairs of the row
  const int box = r >> 8, rr = r & 255;
  const uint32_t tt = smem_addr(Ts) + (uint32_t)hh * S::PPT * KS * TB * 4;
  constexpr int NQ = S::NQ;                  // 16-byte code vectors per thread
  uint32_t voff[NQ];                         // this thread's code vectors in a stage
#pragma unroll
  for (int q = 0; q < NQ; ++q)
    voff[q] = (uint32_t)(box * S::BOX_BYTES + rr * S::ROWB) + 16 * swz<S::ROWB>(hh * NQ + q, rr);
  int nq = 0;                                // vectors holding real pairs
#pragma unroll
  for (int q = 0; q < NQ; ++q) nq += (PK10 || (hh * NQ + q) * S::CPV < np) ? 1 : 0;
  float *out = a.partial + (size_t)c * a.B * a.V;
  int64_t v = t0 * S::R + r;

  int s = 0;
  uint32_t phase = 0;
  int rot_next = ROT && n > 0 && v < a.V ? __ldg(a.rot + (int64_t)c * a.V + v) & 31 : 0;
  for (int i = 0; i < n && table_ok; ++i) {
    // this row's rotation of the chunk's slice (rotated 10-bit codes), loaded
    // one tile ahead so that its latency hides behind a tile's lookups
    const int rot = rot_next;
    if (ROT)
      rot_next = i + 1 < n && v + S::R < a.V ? __ldg(a.rot + (int64_t)c * a.V + v + S::R) & 31 : 0;
    const uint32_t fb = smem_addr(&full[s]);
    if (!mbar_try_wait(fb, phase) && !mbar_wait_bounded(fb, phase)) {
      *reinterpret_cast<volatile int *>(abort_flag) = 1;
      break;
    }
    const uint32_t st = stage0 + s * S::STAGE_BYTES;
    // Codes -> registers first, then give the stage back, so its refill (the
    // tile NST ahead) is in flight while this tile's lookups run.
    uint4 w[NQ];
#pragma unroll
    for (int q = 0; q < NQ; ++q)
      if (q < nq) w[q] = ld_shared_v4(st + voff[q]);
    __syncwarp();
    if (lane == 0) {
      __threadfence_block();                 // this warp's code reads are done
      if (atomicAdd(&released[s], 1u) == S::WARPS - 1) {
        released[s] = 0u;
        if (i + NST < n && !*reinterpret_cast<volatile int *>(abort_flag)) {
          fence_proxy_async_smem();
          issue(i + NST, s);
        }
      }
    }
    float acc[TB];
#pragma unroll
    for (int b = 0; b < TB; ++b) acc[b] = 0.f;
    if constexpr (SCHED) {
      acc[0] = chunk32_sched_tb1<KSH>(tt, w);   // the row's whole 32-pair slice
    } else if constexpr (PK10) {
      acc[0] = chunk32_packed_tb1<KT, ROT>(tt, K, w, skip8, a.fix, rot);
    } else if constexpr (U8) {
#pragma unroll
      for (int q = 0; q < NQ; ++q)
        if (q < nq) lookup16_u8<TB, KT>(tt + (uint32_t)q * 16 * K * TB * 4, K, w[q], a.fix, acc);
    } else {
#pragma unroll
      for (int q = 0; q < NQ; ++q)
        if (q < nq) lookup8<TB, KT>(tt + (uint32_t)q * 8 * K * TB * 4, K, w[q], a.fix, acc);
    }
    if (S::TPR == 2) {
#pragma unroll
      for (int b = 0; b < TB; ++b) acc[b] += __shfl_xor_sync(0xffffffffu, acc[b], 1);
    }
    if (hh == 0 && v < a.V) {
#pragma unroll
      for (int b = 0; b < TB; ++b)
        if (b < a.B) out[(size_t)b * a.V + v] = acc[b];
    }
    v += S::R;
    if (++s == NST) {
      s = 0;
      phase ^= 1u;
    }
  }
  griddep_launch_dependents();
  __syncthreads();
  if (tid == 0 && *reinterpret_cast<volatile int *>(abort_flag)) {
    atomicOr(a.err, RQ_DEVERR_TIMEOUT);
    // let copies still in flight land before the CTA's shared memory goes
    mbar_wait_bounded(smem_addr(tbar), 0u);
    for (int s2 = 0; s2 < NST; ++s2) {
      for (int i = s2; i < n; i += NST) {
        if (!mbar_try_wait(smem_addr(&full[s2]), (uint32_t)((i / NST) & 1))) {
          mbar_wait_bounded(smem_addr(&full[s2]), (uint32_t)((i / NST) & 1));
          break;
        }
      }
    }
  }
}

// ------------------------------------------------------------ reduction

// Block-wide argmax of one (value, index) per thread; result in thread 0.
__device__ __forceinline__ ArgBest block_argbest(ArgBest best, ArgBest *scratch) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) best = arg_better(best, arg_shfl_xor(best, o));
  const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
  __syncthreads();
  if (lane == 0) scratch[warp] = best;
  __syncthreads();
  ArgBest r = scratch[0];
  if (threadIdx.x == 0)
    for (int w = 1; w < (int)blockDim.x / 32; ++w) r = arg_better(r, scratch[w]);
  return r;
}

// z = sum of the nch chunk sums in chunk order; softcap; logits; argmax.
// Grid (nblk, B).  With `keys` set, each block folds its best (value, index)
// into keys[b] with one 64-bit atomicMax (argmax_keys_kernel finishes).
// Rows go 4 per thread (16-byte loads) when V is a multiple of 4 and the
// logits are 16-byte aligned.
__global__ void __launch_bounds__(256) reduce_partials_kernel(
    const float *__restrict__ partial, int nch, int B, int64_t V, float cap, float *logits,
    unsigned long long *keys) {
  griddep_wait();   // the partial sums come from the kernel before this one
  const int b = blockIdx.y;
  ArgBest best{-FLT_MAX, INT_MAX};
  const int64_t stride = (int64_t)gridDim.x * blockDim.x;
  if ((V & 3) == 0 && (reinterpret_cast<uintptr_t>(logits) & 15) == 0) {
    const int64_t V4 = V / 4;
    for (int64_t v4 = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; v4 < V4; v4 += stride) {
      float4 z = make_float4(0.f, 0.f, 0.f, 0.f);
      const float4 *src = reinterpret_cast<const float4 *>(partial + (size_t)b * V) + v4;
      const size_t cstride = (size_t)B * V4;
#pragma unroll 8
      for (int c = 0; c < nch; ++c) {
        const float4 t = __ldcs(src + c * cstride);
        z.x += t.x;
        z.y += t.y;
        z.z += t.z;
        z.w += t.w;
      }
      const float4 y = make_float4(softcap_f(z.x, cap), softcap_f(z.y, cap),
                                   softcap_f(z.z, cap), softcap_f(z.w, cap));
      if (logits) reinterpret_cast<float4 *>(logits + (size_t)b * V)[v4] = y;
      const int v = (int)(4 * v4);
      best = arg_better(best, ArgBest{y.x, v});
      best = arg_better(best, ArgBest{y.y, v + 1});
      best = arg_better(best, ArgBest{y.z, v + 2});
      best = arg_better(best, ArgBest{y.w, v + 3});
    }
  } else {
    for (int64_t v = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; v < V; v += stride) {
      float z = 0.f;
      for (int c = 0; c < nch; ++c) z += __ldcs(partial + ((size_t)c * B + b) * V + v);
      const float y = softcap_f(z, cap);
      if (logits) logits[(size_t)b * V + v] = y;
      best = arg_better(best, ArgBest{y, (int)v});
    }
  }
  griddep_launch_dependents();
  if (keys == nullptr) return;
  // block-wide best first: one atomic per block on the token's key
  __shared__ unsigned long long wkey[8];
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) best = arg_better(best, arg_shfl_xor(best, o));
  if ((threadIdx.x & 31) == 0) wkey[threadIdx.x >> 5] = best.i != INT_MAX ? arg_key(best) : 0ull;
  __syncthreads();
  if (threadIdx.x == 0) {
    unsigned long long k = wkey[0];
    for (int w = 1; w < (int)blockDim.x / 32; ++w) k = wkey[w] > k ? wkey[w] : k;
    if (k) atomicMax(keys + b, k);
  }
}

// The same sum for few rows and many chunks (small V, e.g. an RQ-coded MLP
// matrix with 72-288 chunks): a block covers 64 rows (16 float4 lanes), and
// its 16 lane groups sum every 16th chunk; the 16 partial sums are then added
// in lane-group order (a fixed order: deterministic).  Requires V % 4 == 0
// and 16-byte aligned logits.  Grid (ceil(V/64), B), 256 threads.
__global__ void __launch_bounds__(256) reduce_partials_split_kernel(
    const float *__restrict__ partial, int nch, int B, int64_t V, float cap, float *logits,
    unsigned long long *keys) {
  __shared__ float4 part[16][16];
  griddep_wait();
  const int b = blockIdx.y;
  const int rl = threadIdx.x & 15, cs = threadIdx.x >> 4;
  const int64_t V4 = V / 4;
  const int64_t v4 = (int64_t)blockIdx.x * 16 + rl;
  float4 z = make_float4(0.f, 0.f, 0.f, 0.f);
  if (v4 < V4) {
    const float4 *src = reinterpret_cast<const float4 *>(partial + (size_t)b * V) + v4;
    const size_t cstride = (size_t)B * V4;
    for (int c = cs; c < nch; c += 16) {
      const float4 t = __ldcs(src + c * cstride);
      z.x += t.x;
      z.y += t.y;
      z.z += t.z;
      z.w += t.w;
    }
  }
  part[cs][rl] = z;
  __syncthreads();
  griddep_launch_dependents();
  if (cs != 0) return;                       // lanes 0..15 of warp 0 finish
  float4 y = part[0][rl];
  for (int c = 1; c < 16; ++c) {
    const float4 t = part[c][rl];
    y.x += t.x;
    y.y += t.y;
    y.z += t.z;
    y.w += t.w;
  }
  ArgBest best{-FLT_MAX, INT_MAX};
  if (v4 < V4) {
    y = make_float4(softcap_f(y.x, cap), softcap_f(y.y, cap), softcap_f(y.z, cap),
                    softcap_f(y.w, cap));
    if (logits) reinterpret_cast<float4 *>(logits + (size_t)b * V)[v4] = y;
    const int v = (int)(4 * v4);
    best = arg_better(best, ArgBest{y.x, v});
    best = arg_better(best, ArgBest{y.y, v + 1});
    best = arg_better(best, ArgBest{y.z, v + 2});
    best = arg_better(best, ArgBest{y.w, v + 3});
  }
  if (keys == nullptr) return;
#pragma unroll
  for (int o = 8; o > 0; o >>= 1) best = arg_better(best, arg_shfl_xor(best, o, 0x0000ffffu));
  if (rl == 0 && best.i != INT_MAX) atomicMax(keys + b, arg_key(best));
}

// keys[b] -> argmax[b] (and clears the key).  With `rows` set, the block then
// rebuilds the picked token's bf16 input row (one thread per subspace).
template <int DS>
__global__ void __launch_bounds__(1024) argmax_keys_kernel(unsigned long long *keys,
                                                          int32_t *argmax, DecodeSpec rs,
                                                          uint16_t *rows) {
  __shared__ int pick;
  griddep_wait();
  const int b = blockIdx.x;
  if (threadIdx.x == 0) {
    const unsigned long long k = keys[b];
    keys[b] = 0ull;
    pick = arg_key_index(k);
    argmax[b] = pick;
  }
  griddep_launch_dependents();
  if (rows == nullptr) return;
  __syncthreads();
  for (int m = threadIdx.x; m < rs.M; m += blockDim.x)
    decode_subspace<DS>(rs, pick, m, rows + (int64_t)b * rs.D);
}

template <int DS>
__global__ void __launch_bounds__(1024) argmax_finalize_kernel(const float *__restrict__ am_val,
                                                              const int *__restrict__ am_idx,
                                                              int nblk, int32_t *argmax,
                                                              DecodeSpec rs, uint16_t *rows) {
  __shared__ ArgBest wbest[32];
  __shared__ int pick;
  griddep_wait();
  const int b = blockIdx.x;
  ArgBest best{-FLT_MAX, INT_MAX};
  for (int k = threadIdx.x; k < nblk; k += blockDim.x)
    best = arg_better(best, ArgBest{am_val[(size_t)b * nblk + k], am_idx[(size_t)b * nblk + k]});
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) best = arg_better(best, arg_shfl_xor(best, o));
  const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
  if (lane == 0) wbest[warp] = best;
  __syncthreads();
  if (threadIdx.x == 0) {
    ArgBest r = wbest[0];
    for (int w = 1; w < (int)blockDim.x / 32; ++w) r = arg_better(r, wbest[w]);
    pick = r.i == INT_MAX ? 0 : r.i;
    argmax[b] = pick;
  }
  griddep_launch_dependents();
  if (rows == nullptr) return;
  __syncthreads();
  for (int m = threadIdx.x; m < rs.M; m += blockDim.x)
    decode_subspace<DS>(rs, pick, m, rows + (int64_t)b * rs.D);
}

// ------------------------------------------------------------ host side

namespace {

typedef CUresult (*EncodeTiledFn)(CUtensorMap *, CUtensorMapDataType, cuuint32_t, void *,
                                  const cuuint64_t *, const cuuint64_t *, const cuuint32_t *,
                                  const cuuint32_t *, CUtensorMapInterleave, CUtensorMapSwizzle,
                                  CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

// looked up once (a function-local static: initialised by one thread)
EncodeTiledFn encode_fn() {
  static const EncodeTiledFn fn = []() -> EncodeTiledFn {
    void *p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) ==
            cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      return reinterpret_cast<EncodeTiledFn>(p);
    return nullptr;
  }();
  return fn;
}

}  // namespace

bool encode_tmap_2d_u16(CUtensorMap *map, const void *base, uint64_t inner, uint64_t outer,
                        uint64_t stride_bytes, uint32_t box_inner, uint32_t box_outer,
                        CUtensorMapSwizzle swz) {
  if (encode_fn() == nullptr) return false;
  const cuuint64_t gdim[2] = {(cuuint64_t)inner, (cuuint64_t)outer};
  const cuuint64_t gstride[1] = {(cuuint64_t)stride_bytes};
  const cuuint32_t box[2] = {box_inner, box_outer};
  const cuuint32_t estride[2] = {1u, 1u};
  return encode_fn()(map, CU_TENSOR_MAP_DATA_TYPE_UINT16, 2, const_cast<void *>(base), gdim,
                     gstride, box, estride, CU_TENSOR_MAP_INTERLEAVE_NONE, swz,
                     CU_TENSOR_MAP_L2_PROMOTION_NONE,
                     CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

namespace {

struct Variant {
  int TB, KT, NST, FMT, KSH;
  int PC, R, THREADS, STAGE_BYTES;
  const void *fn;
};

#define RQ_CHUNK_VARIANT(TB, KT, NST, FMT, KSH, MINB)                                      \
  Variant {                                                                                \
    TB, KT, NST, FMT, KSH, ChunkShape<TB, FMT>::PC, ChunkShape<TB, FMT>::R,                \
        ChunkShape<TB, FMT>::THREADS, ChunkShape<TB, FMT>::STAGE_BYTES,                    \
        reinterpret_cast<const void *>(&logits_chunk_u16_kernel<TB, KT, NST, FMT, KSH, MINB>) \
  }

// Plain uint16 codes: 128 KB table chunk + NST stages (3 x 32 KB or 5 x 16
// KB) per CTA, one CTA per SM; K = 1024 has its own instances (table offsets
// as immediates).  Scheduled codes: one instance per table stride 2^KSH; up to
// 256 entries a chunk's tables (<= 32 KB) and two 32 KB stages leave room
// for two CTAs per SM.
const Variant kVariants[] = {
    RQ_CHUNK_VARIANT(1, 1024, 3, RQ_CODES_U16, 0, 1),
    RQ_CHUNK_VARIANT(2, 1024, 3, RQ_CODES_U16, 0, 1),
    RQ_CHUNK_VARIANT(4, 1024, 5, RQ_CODES_U16, 0, 1),
    RQ_CHUNK_VARIANT(1, 0, 3, RQ_CODES_U16, 0, 1),
    RQ_CHUNK_VARIANT(2, 0, 3, RQ_CODES_U16, 0, 1),
    RQ_CHUNK_VARIANT(4, 0, 5, RQ_CODES_U16, 0, 1),
    RQ_CHUNK_VARIANT(1, 0, 3, RQ_CODES_SCHED, 10, 1),
    RQ_CHUNK_VARIANT(1, 0, 3, RQ_CODES_SCHED, 9, 1),
    RQ_CHUNK_VARIANT(1, 0, 2, RQ_CODES_SCHED, 8, 2),
    RQ_CHUNK_VARIANT(1, 0, 2, RQ_CODES_SCHED, 7, 2),
    RQ_CHUNK_VARIANT(1, 0, 2, RQ_CODES_SCHED, 6, 2),
    RQ_CHUNK_VARIANT(1, 0, 2, RQ_CODES_SCHED, 5, 2),
    // byte codes (K <= 256): tables of at most 32 KB per token, 16 KB stages
    RQ_CHUNK_VARIANT(1, 256, 3, RQ_CODES_U8, 0, 2),
    RQ_CHUNK_VARIANT(1, 0, 3, RQ_CODES_U8, 0, 2),
    RQ_CHUNK_VARIANT(2, 0, 3, RQ_CODES_U8, 0, 1),
    RQ_CHUNK_VARIANT(4, 0, 3, RQ_CODES_U8, 0, 1),
    // 10-bit codes, one token: 128 KB of tables (K = 1024), three 24 KB stages
    RQ_CHUNK_VARIANT(1, 1024, 3, RQ_CODES_PACKED10, 0, 1),
    RQ_CHUNK_VARIANT(1, 0, 3, RQ_CODES_PACKED10, 0, 1),
    RQ_CHUNK_VARIANT(1, 1024, 3, RQ_CODES_PACKED10_ROT, 0, 1),
    RQ_CHUNK_VARIANT(1, 0, 3, RQ_CODES_PACKED10_ROT, 0, 1),
};

size_t variant_smem(const Variant &v, int K) {
  const int KS = v.FMT == RQ_CODES_SCHED ? (1 << v.KSH) : K;
  return 1024 + (size_t)align_up((int64_t)v.PC * KS * v.TB * 4, 1024) +
         (size_t)v.NST * v.STAGE_BYTES + 1024;
}

}  // namespace

ChunkPlan plan_chunk(int64_t V, int P, int K, int B, int fmt, const DevInfo &di) {
  ChunkPlan cp{};
  cp.ok = false;
  const bool pk10 = fmt == RQ_CODES_PACKED10 || fmt == RQ_CODES_PACKED10_ROT;
  if ((fmt != RQ_CODES_U16 && fmt != RQ_CODES_SCHED && fmt != RQ_CODES_U8 && !pk10) || B < 1 ||
      B > 4 || P % 8 != 0 || K > 1024)
    return cp;
  // 10-bit codes: one token, whole 64-code groups (80-byte, 16-byte-aligned rows)
  if (pk10 && (B != 1 || P % 64 != 0)) return cp;
  if (fmt == RQ_CODES_U8 && (K > 256 || P % 16 != 0)) return cp;   // 16-byte row pitch
  if (fmt == RQ_CODES_SCHED && P % 32 != 0) return cp;
  if (V > (int64_t)INT_MAX - 2048) return cp;
  const int TB = rq_lut_token_stride(B);
  for (int i = 0; i < (int)(sizeof(kVariants) / sizeof(kVariants[0])); ++i) {
    const Variant &v = kVariants[i];
    if (v.TB != TB || v.FMT != fmt) continue;
    if (v.KT != 0 && v.KT != K) continue;
    if (fmt == RQ_CODES_SCHED && v.KSH != sched_shift(K)) continue;
    const size_t smem = variant_smem(v, K);
    if (smem > (size_t)di.max_smem_optin) continue;
    cp.ok = true;
    cp.TB = TB;
    cp.PC = v.PC;
    cp.nch = (P + cp.PC - 1) / cp.PC;
    cp.R = v.R;
    cp.variant = i;
    cp.smem = smem;
    return cp;
  }
  return cp;
}

size_t chunk_partial_bytes(const ChunkPlan &cp, int B, int64_t V) {
  return (size_t)cp.nch * B * V * sizeof(float);
}

cudaError_t launch_logits_chunk(const ChunkPlan &cp, const void *codes, int fmt, int64_t V,
                                int P, int K, int B, const float *lut, float *partial,
                                unsigned long long *keys, bool early_codes,
                                const DevInfo &di, cudaStream_t s) {
  const Variant &var = kVariants[cp.variant];
  if (encode_fn() == nullptr) return cudaErrorNotSupported;
  CUtensorMap tmap;
  const bool pk = fmt == RQ_CODES_PACKED10 || fmt == RQ_CODES_PACKED10_ROT;
  const int cb = fmt == RQ_CODES_U8 || pk ? 1 : 2;   // bytes per element of the map
  const int rowb = pk ? 48 : cp.PC * cb;
  // [V][P] for plain codes; the scheduled layout is chunk-major [P/32][V][32];
  // 10-bit codes are bytes [V][P/64*80], read in 48-byte windows
  const bool cm = fmt == RQ_CODES_SCHED;
  const int64_t pk_row = (int64_t)P / 64 * 80;
  const cuuint64_t gdim[2] = {(cuuint64_t)(cm ? 32 : pk ? pk_row : P),
                              (cuuint64_t)(cm ? (int64_t)V * (P / 32) : V)};
  const cuuint64_t gstride[1] = {(cuuint64_t)(cm ? 64 : pk ? pk_row : P * cb)};
  const cuuint32_t box[2] = {(cuuint32_t)(pk ? 48 : cp.PC), 256u};
  const cuuint32_t estride[2] = {1u, 1u};
  const CUtensorMapSwizzle swz = rowb == 64   ? CU_TENSOR_MAP_SWIZZLE_64B
                                 : rowb == 32 ? CU_TENSOR_MAP_SWIZZLE_32B
                                              : CU_TENSOR_MAP_SWIZZLE_NONE;
  CUresult r = encode_fn()(&tmap,
                           cb == 1 ? CU_TENSOR_MAP_DATA_TYPE_UINT8 : CU_TENSOR_MAP_DATA_TYPE_UINT16,
                           2, const_cast<void *>(codes),
                           gdim, gstride, box, estride, CU_TENSOR_MAP_INTERLEAVE_NONE, swz,
                           CU_TENSOR_MAP_L2_PROMOTION_NONE, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  if (r != CUDA_SUCCESS) return cudaErrorInvalidValue;

  // the shared-memory limit is raised when a larger K needs more (plain-code
  // tables scale with K)
  {
    cudaError_t e = ensure_smem_limit(reinterpret_cast<const void *>(var.fn), di.device, cp.smem);
    if (e != cudaSuccess) return e;
  }

  ChunkArgs a;
  a.lut = lut;
  a.partial = partial;
  a.keys = keys;
  a.early_codes = early_codes ? 1 : 0;
  a.V = V;
  a.ntiles = (V + cp.R - 1) / cp.R;
  a.P = P;
  a.K = K;
  a.B = B;
  a.nch = cp.nch;
  // CTAs per SM this instance reaches (shared memory and registers)
  const int occ =
      occupancy_cached(reinterpret_cast<const void *>(var.fn), di.device, var.THREADS, cp.smem);
  int64_t cpc = (int64_t)di.sms * occ / cp.nch;
  if (cpc < 1) cpc = 1;
  if (cpc > a.ntiles) cpc = a.ntiles;
  a.cpc = (int)cpc;
  a.fix = make_codefix(K);
  a.err = di.err;
  a.rot = fmt == RQ_CODES_PACKED10_ROT
              ? static_cast<const uint8_t *>(codes) + V * ((int64_t)P / 64 * 80)
              : nullptr;
  const int64_t grid = (int64_t)cp.nch * cpc;
  void *args[] = {&tmap, &a};
  return launch_maybe_pdl(var.fn, dim3((unsigned)grid), dim3(var.THREADS), cp.smem, s, args,
                          true);
}

cudaError_t launch_reduce_partials(const float *partial, int nch, int B, int64_t V, float cap,
                                   float *logits, unsigned long long *keys, int nblk,
                                   cudaStream_t s) {
  // few rows per chunk: split the chunks over the block (fewer than ~one
  // 1024-row block per SM otherwise)
  int dev = 0, sms = 148;
  if (cudaGetDevice(&dev) == cudaSuccess)
    cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  if (V < 1024LL * sms && nch >= 32 && (V & 3) == 0 &&
      (reinterpret_cast<uintptr_t>(logits) & 15) == 0)
    return pdl_launch(reduce_partials_split_kernel, dim3((unsigned)((V + 63) / 64), (unsigned)B),
                      dim3(256), 0, s, partial, nch, B, V, cap, logits, keys);
  return pdl_launch(reduce_partials_kernel, dim3((unsigned)nblk, (unsigned)B), dim3(256), 0, s,
                    partial, nch, B, V, cap, logits, keys);
}

static DecodeSpec no_rows() {
  DecodeSpec r{};
  r.M = 0;
  r.D = 1;
  return r;
}

// One thread per subspace of the row (up to 1024), so the rebuild costs two
// dependent memory round trips.
static unsigned rows_block(const DecodeSpec &rs, bool rows) {
  if (!rows) return 32;
  const int t = (rs.M + 31) / 32 * 32;
  return (unsigned)(t > 1024 ? 1024 : t);
}

cudaError_t launch_argmax_keys(unsigned long long *keys, int B, int32_t *argmax,
                               const DecodeSpec *rows_spec, uint16_t *rows, cudaStream_t s) {
  const DecodeSpec rs = rows_spec ? *rows_spec : no_rows();
  const dim3 blk(rows_block(rs, rows != nullptr));
  if (rows && rs.D / rs.M == 6)
    return pdl_launch(argmax_keys_kernel<6>, dim3((unsigned)B), blk, 0, s, keys, argmax, rs, rows);
  return pdl_launch(argmax_keys_kernel<0>, dim3((unsigned)B), blk, 0, s, keys, argmax, rs, rows);
}

cudaError_t launch_argmax_finalize(const float *am_val, const int *am_idx, int nblk, int B,
                                   int32_t *argmax, const DecodeSpec *rows_spec, uint16_t *rows,
                                   cudaStream_t s) {
  const DecodeSpec rs = rows_spec ? *rows_spec : no_rows();
  unsigned t = rows_block(rs, rows != nullptr);
  if (t < 256) t = 256;
  if (rows && rs.D / rs.M == 6)
    return pdl_launch(argmax_finalize_kernel<6>, dim3((unsigned)B), dim3(t), 0, s, am_val, am_idx,
                      nblk, argmax, rs, rows);
  return pdl_launch(argmax_finalize_kernel<0>, dim3((unsigned)B), dim3(t), 0, s, am_val, am_idx,
                    nblk, argmax, rs, rows);
}

}  // namespace rq

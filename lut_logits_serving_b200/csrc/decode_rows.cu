// decode_rows.cu -- on-demand rebuild of input-embedding rows, and the
// 10-bit code packer.
//
// "Gemma-2 runtime compression: NF4 + LUT serving", LUT section: input token
// rows are reconstructed on demand (the ids of a prompt, not the whole
// vocabulary).  Row element i = m*ds + j of id v:
//   out = bf16_rne( fp32( fp32(sum_l C[m][l][code[v][m*L+l]][j]) * scale ) )
// with the level sum in l order and explicit round-to-nearest fp32 ops, so
// the bf16 result is reproducible bit for bit.
//
// Packing: the "Gemma-2-2B combined RQ+NF4" page stores the M=384, K=1024,
// L=2 artifact at 3.59 bits/param, i.e. 10-bit codes; code p of a row sits
// at bits [10p, 10p+10) of the row's little-endian bit string.
#include "rq_common.cuh"

namespace rq {

// Grid (N, ceil(M / 128)): one thread per (row, subspace); the L code loads,
// then all L*ds codeword loads of a subspace are independent, so a single
// row costs two dependent memory round trips.
template <int DS>
__global__ void __launch_bounds__(128) decode_rows_kernel(const int32_t *__restrict__ ids,
                                                          const DecodeSpec a,
                                                          uint16_t *__restrict__ out,
                                                          unsigned *err) {
  griddep_launch_dependents();
  griddep_wait();   // the ids may be the argmax the previous kernel wrote
  const int64_t n = blockIdx.x;
  const int m = blockIdx.y * blockDim.x + threadIdx.x;
  if (m >= a.M) return;
  const int32_t id = ids[n];
  uint16_t *orow = out + n * (int64_t)a.D;
  if (id < 0 || (int64_t)id >= a.V) {
    const int ds = a.D / a.M;
    for (int j = 0; j < ds; ++j) orow[(int64_t)m * ds + j] = 0;
    if (m == 0) atomicOr(err, RQ_DEVERR_BAD_ID);
    return;
  }
  decode_subspace<DS>(a, id, m, orow);
}

// ds = 6 rows, three threads per (row, subspace): thread q of subspace m
// rebuilds elements 2q and 2q+1.  A warp then spans about eleven subspaces, so
// each float2 codeword load touches about eleven lines instead of one per
// lane, and the bf16 pairs leave as coalesced 4-byte stores.  Each thread
// takes R consecutive rows and issues their loads together: the launch picks
// R = 1 or 2 when that grid is resident in one wave, else 4, so the
// id -> code -> codeword round trips are paid once per wave of R rows.  The
// element arithmetic is that of decode_subspace: level sum from 0 in l order,
// then the scale, then bf16 round to nearest even.
constexpr int kPairSub = 128;   // subspaces per block

template <int R>
__global__ void __launch_bounds__(3 * kPairSub) decode_rows_pair_kernel(
    const int32_t *__restrict__ ids, int64_t N, const DecodeSpec a, uint32_t *__restrict__ out,
    unsigned *err) {
  griddep_launch_dependents();
  griddep_wait();   // the ids may be the argmax the previous kernel wrote
  const int64_t n0 = (int64_t)blockIdx.x * R;
  const int t = blockIdx.y * (3 * kPairSub) + threadIdx.x;
  const int m = t / 3, q = t - 3 * m;
  if (m >= a.M) return;
  const int P = a.M * a.L;
  const int64_t rb10 = (10LL * P + 7) / 8;
  const uint16_t *all16 = static_cast<const uint16_t *>(a.codes);
  const uint8_t *all8 = static_cast<const uint8_t *>(a.codes);
  int32_t id[R];
  uint32_t ok = 0u;   // bit r: row n0 + r exists and its id is in [0, V)
#pragma unroll
  for (int r = 0; r < R; ++r) {
    const bool in = n0 + r < N;
    const int32_t v = in ? ids[n0 + r] : 0;
    const bool good = in && v >= 0 && (int64_t)v < a.V;
    ok |= (uint32_t)good << r;
    id[r] = good ? v : 0;
    if (in && !good && t == 0) atomicOr(err, RQ_DEVERR_BAD_ID);
  }
  float e0[R], e1[R];
#pragma unroll
  for (int r = 0; r < R; ++r) e0[r] = e1[r] = 0.f;
  for (int l = 0; l < a.L; ++l) {
    const int p = m * a.L + l;
    uint32_t c[R];
#pragma unroll
    for (int r = 0; r < R; ++r) {
      c[r] = 0u;
      if (ok >> r & 1u) {
        const int64_t v = id[r];
        if (a.fmt == RQ_CODES_U16) c[r] = all16[v * P + p];
        else if (a.fmt == RQ_CODES_SCHED) c[r] = sched_code(all16, a.V, v, p, sched_shift(a.K));
        else if (a.fmt == RQ_CODES_U8) c[r] = all8[v * P + p];
        else if (a.fmt == RQ_CODES_PACKED10_ROT) c[r] = rot10_code(all8, a.V, P, v, p);
        else c[r] = packed10_code(all8 + v * rb10, p);
      }
    }
#pragma unroll
    for (int r = 0; r < R; ++r) {
      if (ok >> r & 1u) {
        const float2 w =
            __ldg(reinterpret_cast<const float2 *>(a.C + ((size_t)p * a.K + a.fix(c[r])) * 6) + q);
        e0[r] = __fadd_rn(e0[r], w.x);
        e1[r] = __fadd_rn(e1[r], w.y);
      }
    }
  }
#pragma unroll
  for (int r = 0; r < R; ++r) {
    if (n0 + r >= N) break;
    uint32_t v = 0u;
    if (ok >> r & 1u) {
      const uint32_t lo = __bfloat16_as_ushort(__float2bfloat16_rn(__fmul_rn(e0[r], a.scale)));
      const uint32_t hi = __bfloat16_as_ushort(__float2bfloat16_rn(__fmul_rn(e1[r], a.scale)));
      v = lo | (hi << 16);
    }
    out[(n0 + r) * (int64_t)(3 * a.M) + t] = v;
  }
}

template <int R>
cudaError_t launch_pair(const int32_t *ids, int64_t N, const DecodeSpec &a, uint16_t *out,
                        unsigned *err, cudaStream_t s) {
  const int64_t gx = (N + R - 1) / R;
  if (gx > 0x7fffffffLL) return cudaErrorInvalidValue;
  return pdl_launch(decode_rows_pair_kernel<R>,
                    dim3((unsigned)gx, (unsigned)((a.M + kPairSub - 1) / kPairSub)),
                    dim3(3 * kPairSub), 0, s, ids, N, a, reinterpret_cast<uint32_t *>(out), err);
}

// Whether the grid of R rows per thread is resident in one wave.
template <int R>
bool pair_fits(int64_t N, int M, int sms) {
  int per_sm = 0;
  if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, decode_rows_pair_kernel<R>,
                                                    3 * kPairSub, 0) != cudaSuccess)
    return false;
  return (N + R - 1) / R * ((M + kPairSub - 1) / kPairSub) <= (int64_t)per_sm * sms;
}

cudaError_t launch_decode_rows(const int32_t *ids, int64_t N, const void *codes, int fmt,
                               const float *C, int64_t V, int D, int M, int L, int K,
                               float scale, uint16_t *out, unsigned *err, cudaStream_t s) {
  if (N <= 0) return cudaSuccess;
  if (N > 0x7fffffffLL) return cudaErrorInvalidValue;
  const dim3 grid((unsigned)N, (unsigned)((M + 127) / 128));
  DecodeSpec a;
  a.codes = codes;
  a.fmt = fmt;
  a.C = C;
  a.V = V;
  a.D = D;
  a.M = M;
  a.L = L;
  a.K = K;
  a.scale = scale;
  a.fix = make_codefix(K);
  if (D == 6 * M && ((uintptr_t)out & 3) == 0 && ((uintptr_t)C & 7) == 0) {
    DevInfo di;
    const int sms = dev_info(&di) == cudaSuccess ? di.sms : 148;
    (void)cudaGetLastError();
    if (pair_fits<1>(N, M, sms)) return launch_pair<1>(ids, N, a, out, err, s);
    if (pair_fits<2>(N, M, sms)) return launch_pair<2>(ids, N, a, out, err, s);
    (void)cudaGetLastError();
    return launch_pair<4>(ids, N, a, out, err, s);
  }
  if (D / M == 6) return pdl_launch(decode_rows_kernel<6>, grid, dim3(128), 0, s, ids, a, out, err);
  return pdl_launch(decode_rows_kernel<0>, grid, dim3(128), 0, s, ids, a, out, err);
}

// One thread per group of 4 codes = 5 output bytes.
__global__ void pack10_kernel(const uint16_t *__restrict__ codes, int64_t V, int P,
                              uint8_t *__restrict__ packed) {
  const int groups = (P + 3) / 4;
  const int64_t rb = (10LL * P + 7) / 8;
  const int64_t gid = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
  if (gid >= V * groups) return;
  const int64_t v = gid / groups;
  const int g = (int)(gid % groups);
  uint64_t bits = 0;
  for (int q = 0; q < 4; ++q) {
    const int p = 4 * g + q;
    if (p < P) bits |= (uint64_t)(codes[v * P + p] & 0x3FFu) << (10 * q);
  }
  uint8_t *row = packed + v * rb;
  for (int q = 0; q < 5; ++q) {
    const int64_t byte = 5LL * g + q;
    if (byte < rb) row[byte] = (uint8_t)(bits >> (8 * q));
  }
}

cudaError_t launch_pack10(const uint16_t *codes, int64_t V, int P, uint8_t *packed,
                          cudaStream_t s) {
  const int64_t total = V * ((P + 3) / 4);
  if (total == 0) return cudaSuccess;
  const int64_t blocks = (total + 255) / 256;
  if (blocks > 0x7fffffffLL) return cudaErrorInvalidValue;
  pack10_kernel<<<(unsigned)blocks, 256, 0, s>>>(codes, V, P, packed);
  return cudaGetLastError();
}

}  // namespace rq

namespace rq {

// uint16 codes -> one byte each (grid-stride, 16 codes per thread step).
__global__ void pack8_kernel(const uint16_t *__restrict__ codes, int64_t n,
                             uint8_t *__restrict__ out) {
  for (int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; i < n;
       i += (int64_t)gridDim.x * blockDim.x)
    out[i] = (uint8_t)codes[i];
}

cudaError_t launch_pack8(const uint16_t *codes, int64_t n, uint8_t *packed, cudaStream_t s) {
  if (n == 0) return cudaSuccess;
  int64_t blocks = (n + 255) / 256;
  if (blocks > 65536) blocks = 65536;
  pack8_kernel<<<(unsigned)blocks, 256, 0, s>>>(codes, n, packed);
  return cudaGetLastError();
}

}  // namespace rq

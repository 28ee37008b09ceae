/*
 * rq_oracle.c -- plain, slow CPU oracle for LUT-based serving of a
 * residual-product-quantized (RQ) tied embedding.
 *
 * TEST INFRASTRUCTURE ONLY.  Only the test suite, the smoke check and the
 * benchmark's CPU-baseline leg may load this file's library.  The product
 * path (the CUDA library) never links, loads or calls it, and it shares no
 * code, header, table or constant with that path.
 *
 * What is computed, and where the pages define it
 * ("Gemma-2 runtime compression: NF4 + LUT serving", section on LUT-based
 * serving and its correctness-check table; "Gemma-2-2B combined RQ+NF4",
 * paragraph giving M=384, K=1024, L=2):
 *
 *   The embedding E is V rows by D columns.  Each row is cut into M
 *   contiguous subspaces of ds = D/M dims (subspace m = dims [m*ds,
 *   (m+1)*ds)).  Subspace m of row v is the sum over L residual levels of
 *   codewords taken from per-(subspace, level) codebooks:
 *       E[v, m*ds + j] = sum_{l<L} C[m][l][code[v][m][l]][j].
 *   Output logits of hidden state h are z[v] = <h, E[v]>.  LUT serving never
 *   forms E: per token it builds
 *       T[m][l][k] = sum_{j<ds} h[m*ds + j] * C[m][l][k][j]
 *   and then z[v] = sum_{m<M} sum_{l<L} T[m][l][code[v][m][l]].
 *   The pages check the LUT result against direct decode-then-matmul, both
 *   in fp32.  Gemma-2's final softcap y = cap * tanh(z / cap) follows
 *   (cap = 30).  Input rows are rebuilt on demand: the decode function
 *   below returns bf16(fp32(fp32(sum of levels) * scale)).
 *
 * Precision.  Every function exists in an fp64 form (the parity
 * reference) and, where the pages' own check is fp32, an fp32 form.  All
 * sums run in the order written (j, then m-major / l-minor, then i), and the
 * file is compiled with -ffp-contract=off so no multiply-add is fused.
 *
 * Threads.  Built with OpenMP, the loops over vocabulary rows (and over
 * the rows to decode or encode, and the table entries) are split across
 * host threads.  Each output element is still computed by one thread in the
 * order written above, so the results do not depend on the thread count;
 * rqo_set_threads(1) gives the single-threaded timing.
 *
 * Layouts (plain row-major C arrays):
 *   h      float  [B][D]
 *   C      float  [M][L][K][ds]
 *   codes  uint16 [V][M][L]           (code index of pair (m,l) is m*L + l)
 *   T      [B][M][L][K]               (double or float)
 *   z, y   [B][nrows]                 (rows listed explicitly)
 *   packed uint8  [V][ceil(10*M*L/8)] (10-bit codes, little-endian bit
 *                                      stream per row, code j in bits
 *                                      [10j, 10j+10))
 *   X      float  [N][D]              (rows to encode)
 *
 * Top-k and sampling.  The pages cap generation length and state no sampler
 * ("Gemma-2-2B combined RQ+NF4", closing note on generation).  Plain reading for
 * generation beyond greedy: the k largest softcapped logits (descending,
 * the lower index first among equal values), then a draw from the
 * temperature softmax restricted to them by inverse CDF: weights
 * w_i = exp((y_i - y_max) / T) in sorted order, S_i their running sums, and
 * the token is the first i with S_i > u * S_k.  The uniform u in [0, 1) is
 * the top 53 bits of word 0 of Philox4x64-10 (Salmon et al., SC'11) with
 * counter (step, token row, 0, 0) and key (seed, 0), times 2^-53.  The
 * sampling arithmetic here is fp64.
 *
 * Encoder.  The pages call the embedding compression residual product
 * quantization and give no assignment rule ("Gemma-2-2B combined RQ+NF4",
 * RQ paragraph).  The plain reading, used here: per subspace, level 0 takes
 * the nearest codeword of the subspace's level-0 codebook, and each later
 * level the nearest codeword to what the earlier levels left over (the
 * residual).  "Nearest" is a decision taken in fp32: the squared distance
 * is accumulated over j = 0..ds-1 in order as acc = fma(t, t, acc) with
 * t = r[j] - c[j] rounded to fp32 (fmaf is exactly rounded, so the result
 * is fixed by IEEE 754), ties go to the lowest codeword index, and the
 * residual is updated as r[j] = r[j] - c[j] in fp32.
 */
#include <math.h>
#include <stdint.h>
#include <stddef.h>
#include <string.h>
#ifdef _OPENMP
#include <omp.h>
#endif

/* ------------------------------------------------------------------ threads */

/* Host threads the parallel loops use (n < 1: all the runtime offers). */
void rqo_set_threads(int n)
{
#ifdef _OPENMP
    omp_set_num_threads(n > 0 ? n : omp_get_num_procs());
#else
    (void)n;
#endif
}

int rqo_max_threads(void)
{
#ifdef _OPENMP
    return omp_get_max_threads();
#else
    return 1;
#endif
}

/* ---------------------------------------------------------------- LUT build */

void rqo_lut_build_f64(const float *h, int B, const float *C, int D, int M,
                       int L, int K, double *T)
{
    int ds = D / M;
    #pragma omp parallel for collapse(2) schedule(static)
    for (int b = 0; b < B; ++b)
        for (int m = 0; m < M; ++m)
            for (int l = 0; l < L; ++l)
                for (int k = 0; k < K; ++k) {
                    const float *cw = C + (((size_t)m * L + l) * K + k) * ds;
                    const float *hm = h + (size_t)b * D + (size_t)m * ds;
                    double acc = 0.0;
                    for (int j = 0; j < ds; ++j)
                        acc += (double)hm[j] * (double)cw[j];
                    T[(((size_t)b * M + m) * L + l) * K + k] = acc;
                }
}

void rqo_lut_build_f32(const float *h, int B, const float *C, int D, int M,
                       int L, int K, float *T)
{
    int ds = D / M;
    #pragma omp parallel for collapse(2) schedule(static)
    for (int b = 0; b < B; ++b)
        for (int m = 0; m < M; ++m)
            for (int l = 0; l < L; ++l)
                for (int k = 0; k < K; ++k) {
                    const float *cw = C + (((size_t)m * L + l) * K + k) * ds;
                    const float *hm = h + (size_t)b * D + (size_t)m * ds;
                    float acc = 0.0f;
                    for (int j = 0; j < ds; ++j) {
                        float p = hm[j] * cw[j];
                        acc = acc + p;
                    }
                    T[(((size_t)b * M + m) * L + l) * K + k] = acc;
                }
}

/* ------------------------------------------------------ LUT lookup and sum */

void rqo_logits_lut_f64(const uint16_t *codes, int64_t V, int M, int L, int K,
                        const double *T, int B, const int64_t *rows,
                        int64_t nrows, double *z)
{
    (void)V;
    #pragma omp parallel for collapse(2) schedule(static)
    for (int b = 0; b < B; ++b)
        for (int64_t r = 0; r < nrows; ++r) {
            const uint16_t *cr = codes + (size_t)rows[r] * M * L;
            double acc = 0.0;
            for (int m = 0; m < M; ++m)
                for (int l = 0; l < L; ++l) {
                    int k = cr[m * L + l];
                    acc += T[(((size_t)b * M + m) * L + l) * K + k];
                }
            z[(size_t)b * nrows + r] = acc;
        }
}

void rqo_logits_lut_f32(const uint16_t *codes, int64_t V, int M, int L, int K,
                        const float *T, int B, const int64_t *rows,
                        int64_t nrows, float *z)
{
    (void)V;
    #pragma omp parallel for collapse(2) schedule(static)
    for (int b = 0; b < B; ++b)
        for (int64_t r = 0; r < nrows; ++r) {
            const uint16_t *cr = codes + (size_t)rows[r] * M * L;
            float acc = 0.0f;
            for (int m = 0; m < M; ++m)
                for (int l = 0; l < L; ++l) {
                    int k = cr[m * L + l];
                    acc = acc + T[(((size_t)b * M + m) * L + l) * K + k];
                }
            z[(size_t)b * nrows + r] = acc;
        }
}

/* ------------------------------------------- direct decode, then the matmul */

void rqo_logits_direct_f64(const uint16_t *codes, int64_t V, const float *C,
                           int D, int M, int L, int K, const float *h, int B,
                           const int64_t *rows, int64_t nrows, double *z)
{
    (void)V;
    int ds = D / M;
    #pragma omp parallel for collapse(2) schedule(static)
    for (int b = 0; b < B; ++b)
        for (int64_t r = 0; r < nrows; ++r) {
            const uint16_t *cr = codes + (size_t)rows[r] * M * L;
            double acc = 0.0;
            for (int i = 0; i < D; ++i) {
                int m = i / ds, j = i % ds;
                double e = 0.0;               /* E[v][i], decoded */
                for (int l = 0; l < L; ++l) {
                    int k = cr[m * L + l];
                    e += (double)C[(((size_t)m * L + l) * K + k) * ds + j];
                }
                acc += (double)h[(size_t)b * D + i] * e;
            }
            z[(size_t)b * nrows + r] = acc;
        }
}

void rqo_logits_direct_f32(const uint16_t *codes, int64_t V, const float *C,
                           int D, int M, int L, int K, const float *h, int B,
                           const int64_t *rows, int64_t nrows, float *z)
{
    (void)V;
    int ds = D / M;
    #pragma omp parallel for collapse(2) schedule(static)
    for (int b = 0; b < B; ++b)
        for (int64_t r = 0; r < nrows; ++r) {
            const uint16_t *cr = codes + (size_t)rows[r] * M * L;
            float acc = 0.0f;
            for (int i = 0; i < D; ++i) {
                int m = i / ds, j = i % ds;
                float e = 0.0f;
                for (int l = 0; l < L; ++l) {
                    int k = cr[m * L + l];
                    e = e + C[(((size_t)m * L + l) * K + k) * ds + j];
                }
                float p = h[(size_t)b * D + i] * e;
                acc = acc + p;
            }
            z[(size_t)b * nrows + r] = acc;
        }
}

/* ----------------------------------------------------- softcap and argmax */

/* y = cap * tanh(z / cap); cap <= 0 leaves z unchanged. */
void rqo_softcap_f64(double *y, int64_t n, double cap)
{
    if (cap <= 0.0)
        return;
    for (int64_t i = 0; i < n; ++i)
        y[i] = cap * tanh(y[i] / cap);
}

/* First index of the largest value (ties go to the lowest index).  NaN
 * entries never win. */
int64_t rqo_argmax_f32(const float *y, int64_t n)
{
    int64_t best = 0;
    for (int64_t i = 1; i < n; ++i)
        if (y[i] > y[best])
            best = i;
    return best;
}

int64_t rqo_argmax_f64(const double *y, int64_t n)
{
    int64_t best = 0;
    for (int64_t i = 1; i < n; ++i)
        if (y[i] > y[best])
            best = i;
    return best;
}

/* ---------------------------------------------------------- row decoding */

/* IEEE-754 binary32 -> bfloat16, round to nearest, ties to even.  NaN maps
 * to a quiet NaN with the same sign. */
uint16_t rqo_f32_to_bf16_rne(float x)
{
    uint32_t u;
    memcpy(&u, &x, sizeof u);
    if ((u & 0x7F800000u) == 0x7F800000u && (u & 0x007FFFFFu) != 0)
        return (uint16_t)((u >> 16) | 0x0040u);
    uint32_t upper = u >> 16;
    uint32_t lower = u & 0xFFFFu;
    if (lower > 0x8000u || (lower == 0x8000u && (upper & 1u)))
        upper += 1u;                /* a carry into the exponent is correct */
    return (uint16_t)upper;
}

/* out[n][m*ds + j] = bf16( fp32( fp32(sum_l C[m][l][c_l][j]) * scale ) ),
 * c_l = codes[ids[n]][m][l]; the level sum runs l = 0..L-1 in fp32. */
void rqo_decode_rows_bf16(const int32_t *ids, int64_t N, const uint16_t *codes,
                          int64_t V, const float *C, int D, int M, int L, int K,
                          float scale, uint16_t *out)
{
    (void)V;
    int ds = D / M;
    #pragma omp parallel for schedule(static)
    for (int64_t n = 0; n < N; ++n) {
        const uint16_t *cr = codes + (size_t)ids[n] * M * L;
        for (int m = 0; m < M; ++m)
            for (int j = 0; j < ds; ++j) {
                float e = 0.0f;
                for (int l = 0; l < L; ++l) {
                    int k = cr[m * L + l];
                    e = e + C[(((size_t)m * L + l) * K + k) * ds + j];
                }
                float s = e * scale;
                out[(size_t)n * D + (size_t)m * ds + j] = rqo_f32_to_bf16_rne(s);
            }
    }
}

/* ------------------------------------------------------ 10-bit code packing */

int64_t rqo_packed10_row_bytes(int P) { return ((int64_t)P * 10 + 7) / 8; }

/* Code j of a row occupies bits [10j, 10j+10) of that row's byte string,
 * bit b of the string being bit (b % 8) of byte b / 8.  Unused trailing
 * bits are zero.  Codes must be < 1024. */
void rqo_pack10(const uint16_t *codes, int64_t V, int P, uint8_t *packed)
{
    int64_t rb = rqo_packed10_row_bytes(P);
    memset(packed, 0, (size_t)(V * rb));
    for (int64_t v = 0; v < V; ++v)
        for (int j = 0; j < P; ++j) {
            unsigned c = codes[(size_t)v * P + j];
            for (int t = 0; t < 10; ++t) {
                int64_t bit = (int64_t)j * 10 + t;
                if ((c >> t) & 1u)
                    packed[(size_t)(v * rb + bit / 8)] |= (uint8_t)(1u << (bit % 8));
            }
        }
}

void rqo_unpack10(const uint8_t *packed, int64_t V, int P, uint16_t *codes)
{
    int64_t rb = rqo_packed10_row_bytes(P);
    for (int64_t v = 0; v < V; ++v)
        for (int j = 0; j < P; ++j) {
            unsigned c = 0;
            for (int t = 0; t < 10; ++t) {
                int64_t bit = (int64_t)j * 10 + t;
                unsigned byte = packed[(size_t)(v * rb + bit / 8)];
                c |= ((byte >> (bit % 8)) & 1u) << t;
            }
            codes[(size_t)v * P + j] = (uint16_t)c;
        }
}

/* ----------------------------------------------------------------- encoder */

/* codes[n][m][l] = greedy residual nearest-codeword assignment of row n
 * (definition in the file header). */
void rqo_encode_f32(const float *X, int64_t N, const float *C, int D, int M,
                    int L, int K, uint16_t *codes)
{
    int ds = D / M;
    #pragma omp parallel for schedule(static)
    for (int64_t n = 0; n < N; ++n)
        for (int m = 0; m < M; ++m) {
            float r[64];
            for (int j = 0; j < ds; ++j)
                r[j] = X[n * D + (int64_t)m * ds + j];
            for (int l = 0; l < L; ++l) {
                const float *book = C + ((size_t)m * L + l) * K * ds;
                int best = 0;
                float bestd = INFINITY;
                for (int k = 0; k < K; ++k) {
                    const float *cw = book + (size_t)k * ds;
                    float acc = 0.0f;
                    for (int j = 0; j < ds; ++j) {
                        float t = r[j] - cw[j];
                        acc = fmaf(t, t, acc);
                    }
                    if (acc < bestd) {
                        bestd = acc;
                        best = k;
                    }
                }
                codes[(n * M + m) * L + l] = (uint16_t)best;
                for (int j = 0; j < ds; ++j)
                    r[j] = r[j] - book[(size_t)best * ds + j];
            }
        }
}

/* ------------------------------------------------------ top-k and sampling */

/* Philox4x64 with 10 rounds: the multipliers and Weyl key increments of the
 * published generator. */
void rqo_philox4x64_10(const uint64_t *ctr, const uint64_t *key, uint64_t *out)
{
    uint64_t c0 = ctr[0], c1 = ctr[1], c2 = ctr[2], c3 = ctr[3];
    uint64_t k0 = key[0], k1 = key[1];
    for (int r = 0; r < 10; ++r) {
        unsigned __int128 p0 = (unsigned __int128)c0 * 0xD2E7470EE14C6C93ull;
        unsigned __int128 p1 = (unsigned __int128)c2 * 0xCA5A826395121157ull;
        uint64_t hi0 = (uint64_t)(p0 >> 64), lo0 = (uint64_t)p0;
        uint64_t hi1 = (uint64_t)(p1 >> 64), lo1 = (uint64_t)p1;
        uint64_t n0 = hi1 ^ c1 ^ k0, n2 = hi0 ^ c3 ^ k1;
        c0 = n0;
        c1 = lo1;
        c2 = n2;
        c3 = lo0;
        k0 += 0x9E3779B97F4A7C15ull;
        k1 += 0xBB67AE8584CAA73Bull;
    }
    out[0] = c0;
    out[1] = c1;
    out[2] = c2;
    out[3] = c3;
}

double rqo_uniform(uint64_t seed, uint64_t step, int64_t row)
{
    uint64_t ctr[4] = {step, (uint64_t)row, 0, 0}, key[2] = {seed, 0}, out[4];
    rqo_philox4x64_10(ctr, key, out);
    return (double)(out[0] >> 11) * (1.0 / 9007199254740992.0);
}

/* The k largest of y[0..n): repeated scans for the largest value not yet
 * taken, the lower index winning among equal values. */
void rqo_topk_f32(const float *y, int64_t n, int k, float *val, int32_t *idx,
                  unsigned char *taken)
{
    memset(taken, 0, (size_t)n);
    for (int i = 0; i < k; ++i) {
        int64_t best = -1;
        for (int64_t v = 0; v < n; ++v)
            if (!taken[v] && (best < 0 || y[v] > y[best]))
                best = v;
        taken[best] = 1;
        val[i] = y[best];
        idx[i] = (int32_t)best;
    }
}

/* Position (0..k-1) in the sorted top-k of the token drawn with uniform u;
 * temperature <= 0 or k == 1 is greedy (position 0). */
int rqo_sample_position(const float *val, int k, double temperature, double u)
{
    if (k <= 1 || temperature <= 0.0)
        return 0;
    double S = 0.0;
    for (int i = 0; i < k; ++i)
        S += exp(((double)val[i] - (double)val[0]) / temperature);
    double t = u * S, cum = 0.0;
    for (int i = 0; i < k; ++i) {
        cum += exp(((double)val[i] - (double)val[0]) / temperature);
        if (cum > t)
            return i;
    }
    return k - 1;
}

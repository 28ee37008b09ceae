/*
 * rqlut.h -- C ABI of librqlut: LUT-based serving of a residual-product-
 * quantized (RQ) tied embedding on one NVIDIA B200 (sm_100a).
 *
 * The method ("Gemma-2 runtime compression: NF4 + LUT serving" page, section
 * on LUT-based serving; "Gemma-2-2B combined RQ+NF4" page, paragraph on the
 * RQ reconstruction with M=384, K=1024, L=2):
 *
 *   A V x D embedding is stored as codes [V][M][L] into per-(subspace,
 *   level) codebooks C[M][L][K][ds], ds = D/M, subspace m = dims
 *   [m*ds, (m+1)*ds):  E[v, m*ds+j] = sum_l C[m][l][code[v][m][l]][j].
 *   Output logits are computed without forming E: per token b a lookup
 *   table T[b][m][l][k] = <h_b[m*ds : m*ds+ds], C[m][l][k]> is built, then
 *   z[b][v] = sum_m sum_l T[b][m][l][code[v][m][l]]  (lookup + sum), and
 *   Gemma-2's final softcap y = cap * tanh(z / cap) follows.  Input rows are
 *   rebuilt on demand for the few ids of a step.
 *
 * Conventions shared by every call
 *   - Pointers named device_* / "(device)" are CUDA device pointers; the
 *     caller owns every buffer.  The library never allocates device memory.
 *   - `stream` is a cudaStream_t passed as void*; NULL is the legacy default
 *     stream.  Every call only enqueues work and never synchronizes.
 *   - Kernels are launched with programmatic dependent launch: each waits
 *     for the kernels before it in the stream before it reads their outputs
 *     (h, tables, partial sums).  The code matrix and the codebooks are
 *     treated as a resident artifact: a code pass may start fetching code
 *     tiles as soon as the kernel ahead of it in the stream has signalled
 *     that its dependents may launch, so codes must not be written by a
 *     kernel that lets its dependents start early.  The library's own layout
 *     calls (rq_pack10, rq_pack8, rq_prepare_sched) launch without that
 *     signal: what follows them starts after they end.
 *   - Return value: rq_status (0 = RQ_OK).  Argument errors are detected on
 *     the host before anything is launched.  RQ_ERR_CUDA reports a launch
 *     error (cudaGetLastError); kernel faults surface at the caller's next
 *     synchronization, as usual for CUDA.
 *   - Codes >= K are never read out of bounds: with K a power of two a code
 *     is taken modulo K, otherwise it is clamped to K-1.  Ids outside
 *     [0, V) in rq_decode_rows give zero rows and set RQ_DEVERR_BAD_ID in
 *     the device error word (rq_device_error).
 *   - Any wait inside a kernel is bounded (about one second); on expiry
 *     the kernel sets RQ_DEVERR_TIMEOUT and returns.
 *
 * Layouts (row-major, little-endian)
 *   h        float [B][D]
 *   C        float [M][L][K][ds]
 *   codes    RQ_CODES_U16:      uint16 [V][M*L], code of pair (m,l) at
 *                               column p = m*L + l
 *            RQ_CODES_PACKED10: uint8 [V][rb], rb = ceil(10*M*L/8); code
 *                               p occupies bits [10p, 10p+10) of the row,
 *                               bit i being bit (i%8) of byte i/8
 *            RQ_CODES_U8:       uint8 [V][M*L], K <= 256: the byte form
 *                               of small codebooks (the per-matrix K of
 *                               the MLP-RQ page, 8 bits per code), half the
 *                               bytes of RQ_CODES_U16; written by rq_pack8
 *            RQ_CODES_SCHED:    uint16 [M*L/32][V][32] (K <= 1024, M*L % 32
 *                               == 0), written by rq_prepare_sched: chunk-
 *                               major (columns 32c..32c+31 of every row form
 *                               one contiguous [V][32] block, the row's
 *                               "slice"); each slice holds its 32 codes in a
 *                               permuted order, entry = (i << s) | c with i
 *                               in [0,32) the pair's position in the slice,
 *                               c its code and 2^s the smallest power of two
 *                               >= K, at least 32 (s = 10 at K = 1024).  The order only changes the
 *                               summation order; entries with c >= K add 0
 *                               to the logits (rq_decode_rows clamps them to
 *                               K-1).  Batch 1 streams it fastest; full
 *                               token groups of larger batches decode it on
 *                               the tensor cores (M % 16 == 0; 1.15-1.3x the
 *                               time of RQ_CODES_U16 there, one stage of
 *                               codes in flight instead of two), other groups
 *                               read it in the generic lookup order.
 *            RQ_CODES_PACKED10_ROT: uint8, the 10-bit rows (M*L % 64 == 0,
 *                               K <= 1024) with each 32-code slice rotated,
 *                               then one rotation byte per (slice, row),
 *                               written by rq_prepare_rot10 (see there).
 *                               Batch 1 and token groups read through L2
 *                               take it; the decode paths do not.
 *   lut      float [M*L][K][Bs], Bs = rq_lut_token_stride(B): token b of
 *            table (p, k) at lut[(p*K + k)*Bs + b]
 *   logits   float [B][V]
 *   argmax   int32 [B]: lowest index of the largest softcapped logit
 *   rows     uint16 bf16 bit patterns [N][D]
 */
#ifndef RQLUT_H
#define RQLUT_H

#include <stddef.h>
#include <stdint.h>

#if defined(__GNUC__)
#define RQ_API __attribute__((visibility("default")))
#else
#define RQ_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

typedef struct {
    int64_t V;   /* vocabulary rows                                  */
    int32_t D;   /* model dim; must be a multiple of M               */
    int32_t M;   /* subspaces                                        */
    int32_t L;   /* residual levels                                  */
    int32_t K;   /* codewords per (subspace, level) codebook         */
} rq_dims;

enum rq_code_fmt {
    RQ_CODES_U16 = 0,       /* one uint16 per code (K <= 65536)           */
    RQ_CODES_PACKED10 = 1,  /* 10-bit codes, bit stream per row (K<=1024) */
    RQ_CODES_SCHED = 2,     /* bank-scheduled uint16 (rq_prepare_sched)   */
    RQ_CODES_U8 = 3,        /* one byte per code (K <= 256, rq_pack8)     */
    RQ_CODES_PACKED10_ROT = 4 /* 10-bit codes, rotated slices (rq_prepare_rot10) */
};

enum rq_status {
    RQ_OK = 0,
    RQ_ERR_INVALID_ARGUMENT = 1,   /* null pointer, bad shape or value      */
    RQ_ERR_UNSUPPORTED = 2,        /* valid but not handled by this build   */
    RQ_ERR_WORKSPACE_TOO_SMALL = 3,
    RQ_ERR_CUDA = 4,               /* a CUDA runtime call failed            */
    RQ_ERR_MISALIGNED = 5          /* a pointer breaks the stated alignment */
};

/* Bits of the device error word. */
#define RQ_DEVERR_TIMEOUT 0x1u  /* a bounded wait inside a kernel expired */
#define RQ_DEVERR_BAD_ID  0x2u  /* rq_decode_rows saw an id outside [0,V) */

/* Human-readable name of a status code (static string, never NULL). */
RQ_API const char *rq_status_string(int status);

/* Library version, major*10000 + minor*100 + patch. */
RQ_API int rq_version(void);

/* Bytes of the code matrix in format `fmt` (0 on invalid arguments). */
RQ_API size_t rq_codes_bytes(rq_dims d, int fmt);

/* Token stride Bs of the LUT layout: B for B <= 2, else B rounded up to a
 * multiple of 4 (so a token group is a whole number of 16-byte vectors). */
RQ_API int rq_lut_token_stride(int B);

/* Bytes of the lookup table for B tokens: M*L*K*Bs*4 (0 on bad args). */
RQ_API size_t rq_lut_bytes(rq_dims d, int B);

/* Device workspace that rq_lut_logits needs for these arguments: partial
 * sums of the vocabulary-tiled pass plus argmax partials.  0 is possible.
 * `want_argmax` is 0 or 1. */
RQ_API size_t rq_logits_workspace_bytes(rq_dims d, int B, int fmt, int want_argmax);

/* Device workspace of rq_logits_from_hidden (includes the lookup table of
 * one token group or, where the shape can take the tensor-core decode, that
 * kernel's scratch -- split hidden states and codebooks -- if larger). */
RQ_API size_t rq_fused_workspace_bytes(rq_dims d, int B, int fmt, int want_argmax);

/*
 * rq_lut_build -- per-token lookup tables (LUT serving section: the tables
 * that replace the output matmul).
 *   lut[(p*K + k)*Bs + b] = sum_{j<ds} h[b][m*ds + j] * C[m][l][k][j],
 *   p = m*L + l, in fp32 (fused multiply-adds, j ascending).
 *   h   (device) float [B][D], 4-byte aligned
 *   C   (device) float [M][L][K][ds], 4-byte aligned
 *   lut (device) float, rq_lut_bytes(d, B) bytes, 16-byte aligned; padding
 *       tokens b in [B, Bs) are written as 0.
 * Errors: RQ_ERR_INVALID_ARGUMENT (null, B < 1, bad dims),
 *         RQ_ERR_MISALIGNED, RQ_ERR_UNSUPPORTED (one subspace's slice of
 *         all Bs padded tokens, Bs * ds floats, above 48 KB of shared
 *         memory; token groups go through rq_logits_from_hidden),
 *         RQ_ERR_CUDA.
 */
RQ_API int rq_lut_build(const float *h, const float *C, rq_dims d, int B, float *lut,
                 void *stream);

/*
 * rq_lut_logits -- logits by lookup and sum over each vocabulary row's codes,
 * never forming the V x D matrix (LUT serving section and its correctness
 * table: LUT vs direct decode+matmul), then Gemma-2's final softcap and an
 * optional greedy argmax.
 *   z[b][v] = sum_p lut[(p*K + code[v][p])*Bs + b]    (fp32 sums)
 *   y = softcap > 0 ? softcap * tanhf(z / softcap) : z
 *   codes  (device) code matrix in format `fmt`, 16-byte aligned
 *   lut    (device) as written by rq_lut_build for the same B, 16-byte
 *          aligned
 *   logits (device) float [B][V] or NULL (then only argmax is produced)
 *   argmax (device) int32 [B] or NULL; at least one of logits/argmax set
 *   ws     (device) workspace of >= rq_logits_workspace_bytes(d, B, fmt,
 *          argmax != NULL) bytes, 16-byte aligned (may be NULL if that is 0)
 * Errors: RQ_ERR_INVALID_ARGUMENT, RQ_ERR_MISALIGNED,
 *         RQ_ERR_WORKSPACE_TOO_SMALL, RQ_ERR_UNSUPPORTED (PACKED10 with
 *         K > 1024), RQ_ERR_CUDA.
 */
RQ_API int rq_lut_logits(const void *codes, int fmt, rq_dims d, const float *lut,
                  int B, float softcap, float *logits, int32_t *argmax,
                  void *ws, size_t ws_bytes, void *stream);

/*
 * rq_logits_from_hidden -- rq_lut_build + rq_lut_logits in one call; large
 * batches are processed in token groups so each group's table stays in L2.
 * Same arguments and errors as the two calls; the table lives in `ws`
 * (>= rq_fused_workspace_bytes(d, B, fmt, argmax != NULL) bytes).
 */
RQ_API int rq_logits_from_hidden(const float *h, const float *C, const void *codes,
                          int fmt, rq_dims d, int B, float softcap,
                          float *logits, int32_t *argmax, void *ws,
                          size_t ws_bytes, void *stream);

/*
 * Kernel choice for the token groups of rq_logits_from_hidden_path (batches
 * of up to 4 tokens always take the shared-memory table pass).  The decode
 * paths rebuild each vocabulary row once per group (the decode-then-matmul
 * the LUT section checks the lookup against) and contract it with the
 * group's hidden states; they need L = 2, D = 6 M, K <= 1024 and 16-byte
 * aligned C and codes.
 *   RQ_PATH_AUTO        -- RQ_PATH_DECODE_TC where it applies (for a group
 *                          of fewer than 32 tokens from 17 tokens on), else
 *                          RQ_PATH_DECODE_FP32 where that applies, else tables
 *   RQ_PATH_TABLES      -- per-group tables read through L2 (lookup + sum)
 *   RQ_PATH_DECODE_FP32 -- groups of 32; rows decoded into shared memory,
 *                          fp32 FMAs; RQ_CODES_U16 with M % 8 == 0
 *   RQ_PATH_DECODE_TC   -- groups of 64, then 32, then the rest; rows
 *                          decoded into tensor memory, tcgen05 fp16 MMAs on
 *                          hi/lo splits of the rows and hidden states (with
 *                          power-of-two scales), fp32 sums of short MMA
 *                          chains; RQ_CODES_U16 with M % 8 == 0,
 *                          RQ_CODES_SCHED with M % 16 == 0 (codes >= K
 *                          clamped to K-1, as rq_decode_rows does) or
 *                          RQ_CODES_PACKED10 with M % 32 == 0 (its scratch
 *                          lives in the workspace's table region)
 */
enum { RQ_PATH_AUTO = 0, RQ_PATH_TABLES = 1, RQ_PATH_DECODE_FP32 = 2, RQ_PATH_DECODE_TC = 3 };

/*
 * rq_logits_from_hidden_path -- rq_logits_from_hidden with an explicit
 * kernel choice for full token groups.  Same arguments, workspace and
 * errors; an unknown `path` is RQ_ERR_INVALID_ARGUMENT, a decode path the
 * shape, format or alignment cannot take is RQ_ERR_UNSUPPORTED.
 */
RQ_API int rq_logits_from_hidden_path(const float *h, const float *C, const void *codes,
                                      int fmt, rq_dims d, int B, float softcap,
                                      float *logits, int32_t *argmax, void *ws,
                                      size_t ws_bytes, int path, void *stream);

/*
 * rq_greedy_step -- one greedy decoding step of the output head in one call:
 * rq_logits_from_hidden with argmax, then the bf16 input rows of the picked
 * tokens (the embeddings the next step consumes), rebuilt on demand as in
 * rq_decode_rows (LUT serving section: output logits by lookup + sum, input
 * rows reconstructed for the ids of the step).  The row rebuild runs inside
 * the kernel that finishes the argmax.
 *   logits (device) float [B][V] or NULL; argmax (device) int32 [B] and
 *   rows (device) uint16 bf16 [B][D] are required; scale as rq_decode_rows;
 *   ws as rq_logits_from_hidden (rq_fused_workspace_bytes(d, B, fmt, 1)).
 * Errors: as rq_logits_from_hidden.
 */
RQ_API int rq_greedy_step(const float *h, const float *C, const void *codes, int fmt,
                          rq_dims d, int B, float softcap, float *logits, int32_t *argmax,
                          float scale, uint16_t *rows, void *ws, size_t ws_bytes,
                          void *stream);

/*
 * rq_decode_rows -- rebuild input-embedding rows on demand (LUT serving
 * section: input token rows are reconstructed for the ids of a prompt, not
 * for the whole vocabulary).
 *   out[n][m*ds + j] = bf16_rne( fp32( fp32(sum_l C[m][l][c_l][j]) * scale ) ),
 *   c_l = code[ids[n]][m*L + l]; the level sum runs l = 0..L-1 in fp32.
 *   Gemma-2 uses scale = sqrt(D).
 *   ids    (device) int32 [N]; ids outside [0, V) give zero rows and set
 *          RQ_DEVERR_BAD_ID
 *   codes  (device) as for rq_lut_logits (2-byte aligned; 16-byte for
 *          RQ_CODES_SCHED); C (device) float [M][L][K][ds], 4-byte aligned
 *   out    (device) uint16 [N][D] bf16 bit patterns, 2-byte aligned
 *   N = 0 is a no-op.  With ds = 6, out 4-byte aligned and C 8-byte
 *   aligned, three threads share a (row, subspace) and each thread takes up
 *   to four rows; otherwise one thread per (row, subspace).  The results are
 *   the same bits either way.
 * Errors: RQ_ERR_INVALID_ARGUMENT (null pointer, N < 0, bad dims or format),
 * RQ_ERR_UNSUPPORTED (the format cannot hold the shape), RQ_ERR_MISALIGNED,
 * RQ_ERR_CUDA.
 */
RQ_API int rq_decode_rows(const int32_t *ids, int64_t N, const void *codes, int fmt,
                   const float *C, rq_dims d, float scale, uint16_t *out,
                   void *stream);

/*
 * rq_pack10 -- convert uint16 codes [V][M*L] (values < 1024) into the
 * PACKED10 layout above (the 10-bit storage implied by the 3.59 bits/param
 * figure of the combined RQ+NF4 page).  Codes >= 1024 keep their low 10
 * bits.  codes_u16 (device) 2-byte aligned; packed (device) uint8 [V][rb],
 * rb = ceil(10*M*L/8).
 * Errors: RQ_ERR_INVALID_ARGUMENT, RQ_ERR_MISALIGNED, RQ_ERR_CUDA.
 */
RQ_API int rq_pack10(const uint16_t *codes_u16, rq_dims d, uint8_t *packed,
              void *stream);

/*
 * rq_last_cuda_error -- the CUDA runtime error code behind the last
 * RQ_ERR_CUDA returned to the calling host thread (0 if none); clear != 0
 * resets it.  rq_cuda_error_name gives the runtime's name for a code (a
 * static string).  Diagnostics of this library, no counterpart in the pages.
 */
RQ_API int rq_last_cuda_error(int clear);
RQ_API const char *rq_cuda_error_name(int err);

/*
 * rq_topk_sample -- top-k of softcapped logits and a temperature draw among
 * them (generation beyond greedy argmax; the pages state no sampler, see the
 * "Gemma-2-2B combined RQ+NF4" note on generation, so this is the plain
 * reading).  Per token row b of logits [B][V]:
 *   topk_val[b][i], topk_idx[b][i], i < k: the k largest logits, descending,
 *     the lower vocabulary index first among equal values (-0 equals +0;
 *     NaN logits are not supported);
 *   token[b]: with T > 0 and k > 1, w_i = exp((y_i - y_0) / T) in fp64 over
 *     the sorted top-k, and token = topk_idx[b][i] for the first i whose
 *     running sum of w exceeds u * sum(w), where u = (word0 >> 11) * 2^-53,
 *     word0 the first output word of Philox4x64-10 (Salmon et al., SC'11) for
 *     counter (step, b, 0, 0) and key (seed, 0); T <= 0 or k = 1: the top
 *     index (greedy).
 *   logits   (device) float [B][V], 4-byte aligned (e.g. rq_lut_logits')
 *   topk_val (device) float [B][k] or NULL; topk_idx (device) int32 [B][k]
 *            or NULL; token (device) int32 [B] or NULL
 *   ws       (device) workspace of rq_topk_workspace_bytes(V, B, k) bytes,
 *            256-byte aligned; contents need no initialisation
 * Supported: 1 <= k <= min(V, 1024), 1 <= B <= 65535.
 * Errors: RQ_ERR_INVALID_ARGUMENT, RQ_ERR_UNSUPPORTED (k > 1024),
 *         RQ_ERR_WORKSPACE_TOO_SMALL, RQ_ERR_MISALIGNED, RQ_ERR_CUDA.
 */
RQ_API size_t rq_topk_workspace_bytes(int64_t V, int B, int k);
RQ_API int rq_topk_sample(const float *logits, int64_t V, int B, int k, float temperature,
                          uint64_t seed, uint64_t step, float *topk_val, int32_t *topk_idx,
                          int32_t *token, void *ws, size_t ws_bytes, void *stream);

/*
 * rq_encode -- produce the codes: greedy residual nearest-codeword
 * assignment of V rows ("Gemma-2-2B combined RQ+NF4" names the compression
 * residual product quantization, M subspaces x L levels of K codewords,
 * without stating the assignment; this is its plain reading).  Per row x
 * and subspace m, with r = x[m*ds, (m+1)*ds):
 *   for l = 0..L-1: code[v][m*L + l] = argmin_k sum_j (r_j - C[m][l][k][j])^2
 *                   r_j -= C[m][l][code][j]
 * The argmin is an fp32 decision: t_j = fp32(r_j - c_j), the sum
 * accumulated j = 0..ds-1 as fma(t_j, t_j, acc), the lowest k wins ties
 * (a NaN distance never wins: an all-NaN subspace gets code 0), and the
 * residual update is an fp32 subtraction.  The codes are therefore
 * reproducible bit for bit.  Training the codebooks is not part of it.
 *   X     (device) float [V][D], 4-byte aligned (the rows; d.V of them)
 *   C     (device) float [M][L][K][ds]
 *   codes (device) uint16 [V][M*L] (RQ_CODES_U16), 2-byte aligned; must
 *         not overlap X or C
 *   V = 0 is a no-op.  Supported: ds = D/M <= 32 (ds 2, 4, 6, 8 have
 *   specialised kernels), K <= 65536.
 * Errors: RQ_ERR_INVALID_ARGUMENT, RQ_ERR_UNSUPPORTED (ds > 32),
 *         RQ_ERR_MISALIGNED, RQ_ERR_CUDA.
 */
RQ_API int rq_encode(const float *X, rq_dims d, const float *C, uint16_t *codes,
                     void *stream);

/*
 * rq_pack8 -- convert uint16 codes [V][M*L] into RQ_CODES_U8 (one byte per
 * code; K <= 256).  Codes >= 256 keep their low 8 bits.  packed (device)
 * uint8 [V][M*L].
 * Errors: RQ_ERR_INVALID_ARGUMENT, RQ_ERR_UNSUPPORTED (K > 256),
 *         RQ_ERR_MISALIGNED, RQ_ERR_CUDA.
 */
RQ_API int rq_pack8(const uint16_t *codes_u16, rq_dims d, uint8_t *packed, void *stream);

/*
 * rq_prepare_sched -- convert uint16 codes [V][M*L] into RQ_CODES_SCHED
 * (same size; chunk-major so that each 32-pair slice streams contiguously).
 * Not on the pages: a layout of this library.  The lookups of the batch-1
 * logits pass run 32 rows x one 32-pair slice per warp, one lookup per lane
 * per step, and shared memory serves a step in as many passes as the most
 * repeated bank (bank = code mod 32).  Random codes give ~3.5 passes; this
 * call orders each slice so that every step's 32 lookups hit as few
 * repeated banks as a maximum bipartite matching per step allows (~1.5).
 * Same bytes, same sums (in another order).  Run once per artifact.
 *   codes_u16 (device) uint16 [V][M*L], values < K (larger values keep
 *             their low s bits); out (device) uint16 [V][M*L], must not
 *             overlap codes_u16; stats (device) uint64 [2] or NULL:
 *             receives (steps scheduled, bank passes needed) summed over
 *             all warps, for reporting the schedule's quality.
 * Errors: RQ_ERR_INVALID_ARGUMENT (null, bad dims), RQ_ERR_UNSUPPORTED
 *         (K > 1024 or M*L % 32 != 0), RQ_ERR_MISALIGNED, RQ_ERR_CUDA.
 */
RQ_API int rq_prepare_sched(const uint16_t *codes_u16, rq_dims d, uint16_t *out,
                            uint64_t *stats, void *stream);

/*
 * rq_prepare_rot10 -- convert uint16 codes [V][M*L] into
 * RQ_CODES_PACKED10_ROT: the 10-bit packed rows with each 32-code slice
 * rotated, plus one rotation byte per (row, slice).  Not on the pages: a
 * layout of this library for the batch-1 pass on 10-bit codes, which has no
 * room for RQ_CODES_SCHED's per-code positions; a rotation of each slice
 * (5 bits per 32 codes) lets the 32 rows of a warp's step spread over the
 * shared-memory banks (bank = (pair * K + code) mod 32): ~2.6 passes per step
 * for random codes instead of ~3.5.  Same sums in another order.  Run once
 * per artifact.
 *   Layout: bytes [V][rb], rb = 10*M*L/8, then uint8 [M*L/32][V];
 *   rq_codes_bytes(d, RQ_CODES_PACKED10_ROT) = V*rb + V*M*L/32.  Bits
 *   [10j, 10j+10) of slice s (bits [320s, 320s+320) of the row, LSB first as
 *   in RQ_CODES_PACKED10) hold the code of pair 32s + ((j + r) mod 32), with
 *   r = the low 5 bits of rotation byte [s][v].
 *   codes_u16 (device) uint16 [V][M*L], values < K (values >= 1024 keep
 *             their low 10 bits); out (device) uint8, rq_codes_bytes(d,
 *             RQ_CODES_PACKED10_ROT) bytes, 16-byte aligned, not
 *             overlapping codes_u16; stats (device) uint64 [2] or NULL:
 *             (steps, bank passes needed) summed over all warps.
 * Errors: RQ_ERR_INVALID_ARGUMENT (null, bad dims), RQ_ERR_UNSUPPORTED
 *         (K > 1024 or M*L % 64 != 0), RQ_ERR_MISALIGNED, RQ_ERR_CUDA.
 */
RQ_API int rq_prepare_rot10(const uint16_t *codes_u16, rq_dims d, uint8_t *out,
                            uint64_t *stats, void *stream);

/*
 * Greedy pick over a vocabulary split across ranks ("Gemma-2 runtime
 * compression: NF4 + LUT serving", LUT section: argmax of the softcapped
 * logits of every vocabulary row; rows are independent, so rank g may hold
 * only the code rows [row0_g, row0_g + V_g) and run the calls above on them).
 *
 * rq_argmax_candidates -- per token b of the shard's results: val[b] =
 *   logits[b][argmax[b]] and gidx[b] = row0 + argmax[b] (the global row).
 *   logits [B][V] fp32 and argmax [B] int32 as written for the shard; val
 *   [B] fp32, gidx [B] int32 out.  row0 + V must fit in int32.  Device
 *   pointers, 4-byte aligned; stream-ordered.
 * rq_argmax_merge -- argmax[b] = the best of the n candidates val[k][b],
 *   gidx[k][b] (rank-major [n][B], as an all-gather of the ranks' candidate
 *   arrays lays them out): larger value first, lower index on equal values,
 *   NaN never above a number -- the order of the single-GPU argmax, so the
 *   merged pick equals the unsharded one.  argmax [B] int32 out.
 * Errors: RQ_ERR_INVALID_ARGUMENT (null pointer, B < 1, n < 1, V < 1,
 * row0 < 0 or an int32 overflow), RQ_ERR_MISALIGNED, RQ_ERR_CUDA.
 */
RQ_API int rq_argmax_candidates(const float *logits, const int32_t *argmax, int B, int64_t V,
                                int64_t row0, float *val, int32_t *gidx, void *stream);
RQ_API int rq_argmax_merge(const float *val, const int32_t *gidx, int n, int B, int32_t *argmax,
                           void *stream);

/*
 * rq_device_error -- read (and, if `clear`, reset) the device error word
 * of the current device.  Synchronous: call after synchronizing the streams
 * that ran the kernels of interest.  *out receives RQ_DEVERR_* bits.
 * Errors: RQ_ERR_INVALID_ARGUMENT (out NULL), RQ_ERR_CUDA.
 */
RQ_API int rq_device_error(uint32_t *out, int clear);

/*
 * rq_lut_logits_static -- rq_lut_logits without a caller-provided workspace,
 * for callers that cannot allocate device memory: processes whose device
 * memory belongs to another runtime's allocator, which this library cannot
 * draw from, and serving loops that must not allocate once they have
 * started.  The paper has no counterpart; this is a convenience of this
 * library.
 *   Arguments, results and errors are those of rq_lut_logits, without ws and
 *   ws_bytes.  The workspace comes from a fixed device array inside the
 *   library, RQ_STATIC_SCRATCH_BYTES on every GPU that loads it, held until
 *   the process exits; a call whose workspace (rq_logits_workspace_bytes)
 *   would exceed it returns RQ_ERR_WORKSPACE_TOO_SMALL and launches nothing.
 *   At the Gemma-2 shape this covers batch 1 (24.6 MB), not batch 2 (98 MB)
 *   of the B <= 4 pass; batches > 4 need only kilobytes.
 *   The first call on a device looks the array's address up (once per
 *   device, with that device current); make that first call before any
 *   stream capture.  All calls on a device share the one array: calls that
 *   may run at the same time on the GPU (different streams without an
 *   ordering between them) race on it and must be serialized by the caller.
 *   Nothing in it needs to start at zero; the kernels reset what they use.
 *   The looked-up address is cached per device index for the life of the
 *   process: do not use the library across a cudaDeviceReset (the same holds
 *   for the device error word behind rq_device_error).
 */
#define RQ_STATIC_SCRATCH_BYTES (32u * 1024u * 1024u)
RQ_API int rq_lut_logits_static(const void *codes, int fmt, rq_dims d, const float *lut,
                                 int B, float softcap, float *logits, int32_t *argmax,
                                 void *stream);

/*
 * rq_set_profile_events -- optional timing hook for benchmarks.  With both
 * arguments non-NULL (cudaEvent_t handles passed as void*), each later
 * rq_lut_logits / rq_logits_from_hidden call made from this host thread
 * records `start` on its stream just before its first code-streaming kernel
 * and `stop` just after its last one, so cudaEventElapsedTime(start, stop)
 * is the device time of that pass alone (for token-grouped batches it spans
 * the groups and the table builds between them).  NULL, NULL turns it off.
 * The setting is thread-local; the events stay owned by the caller.
 * Errors: RQ_ERR_INVALID_ARGUMENT if exactly one argument is NULL.
 */
RQ_API int rq_set_profile_events(void *start, void *stop);

#ifdef __cplusplus
}
#endif
#endif /* RQLUT_H */

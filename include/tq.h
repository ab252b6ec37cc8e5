/*
 * tq.h -- C ABI of libtq, a B200 (sm_100a) library for TurboQuant-style
 * online vector quantization: batched encode of fp32/bf16 vectors into packed
 * low-bit codes plus a 1-bit QJL sketch of the residual, and asymmetric
 * inner-product scoring of fp32 queries against those codes (all logits, or
 * top-k).
 *
 * Sources of the method ("TurboQuant article" = the intelliparadigm.com page
 * "TurboQuant 技术概览与核心价值"; "TurboQuant blog" = the blog.hotdry.top page
 * "TurboQuant 深度解读"):
 *   - online, training-free quantization ........ TurboQuant article 1.1, 3.3; blog 一
 *   - random rotation (Haar, or 3 rounds of
 *     +-1 diagonal then Walsh-Hadamard) .......... TurboQuant article 1.2.1, 2.1.1-2.1.2
 *   - (b-1)-bit Lloyd-Max codebook on the
 *     Beta((d-1)/2,(d-1)/2) coordinate law ....... TurboQuant article 1.2.2, 2.2.1-2.2.2
 *   - residual + 1-bit QJL sketch, unbiased
 *     inner products ............................. TurboQuant article 1.2.3, 2.3.1-2.3.2; blog 三
 *   - stored L2 norm, same rotation on queries,
 *     top-K retrieval ............................ TurboQuant article 4.2.1-4.2.2
 *   - outlier channels at more bits (3.5-bit) ... TurboQuant article 3.2, 4.1.1; blog 四
 *
 * Conventions for every call:
 *   - Return a tq_status; calls never abort and never throw across the ABI.
 *     Arguments are validated before anything is launched; on error nothing
 *     is written.  A CUDA launch error maps to TQ_ERR_CUDA; an asynchronous
 *     fault surfaces at the next synchronization of the stream.
 *   - Device calls are asynchronous on `stream` (a cudaStream_t passed as
 *     void*, NULL = legacy default stream) and run on the device that was
 *     current when the quantizer was created.
 *   - The caller allocates and frees every data buffer (device memory unless
 *     stated).  The library owns only the quantizer's read-only device tables.
 *   - A quantizer is immutable after creation and may be shared by threads.
 *   - n == 0 (or nq == 0) is a successful no-op.
 *
 * Packed layouts (per vector, d a multiple of 32, m = d):
 *   codes: w*d/8 bytes, w = b-1 bits per coordinate, in groups of 32
 *          coordinates; group g occupies w 32-bit little-endian words
 *          starting at word w*g.  Within a group (coordinate j = 32g + i):
 *            w = 1: word 0 bit i                      = code
 *            w = 2: word i/16, bits 4*(i%8) + 2*((i/8)%2) .. +1 = code
 *            w = 3: i < 24: word i/8, bits 4*(i%8) .. +2 = code;
 *                   i >= 24 (k = i-24): bit 4k+3 of words 0, 1, 2 hold
 *                   code bits 2, 1, 0 respectively
 *            w = 4: word i/8, bits 4*(i%8) .. +3 = code
 *          (layouts chosen so that one logical AND / shift exposes 4-bit
 *          byte selectors for the scorer's table lookups).
 *   signs: m/8 bytes; bit i of 32-bit word i/32 is 1 iff (S r)_i >= 0.
 *   norms: 2 floats: ||x|| and gamma = ||r||.
 */
#ifndef TQ_H
#define TQ_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef struct tq_quantizer tq_quantizer;

typedef enum {
  TQ_OK = 0,
  TQ_ERR_INVALID_ARG = 1,  /* null pointer, negative size, bad enum, ...        */
  TQ_ERR_UNSUPPORTED = 2,  /* (d, b, m, rotation, dtype) outside what is built   */
  TQ_ERR_ALIGNMENT = 3,    /* a pointer or leading dimension breaks the stated alignment */
  TQ_ERR_NOMEM = 4,        /* host or device allocation of the quantizer tables failed */
  TQ_ERR_CUDA = 5,         /* a CUDA runtime call or kernel launch failed        */
  TQ_ERR_WORKSPACE = 6,    /* workspace pointer null or smaller than required    */
  TQ_ERR_TOO_LARGE = 7,    /* request needs more than a fixed internal buffer    */
  TQ_ERR_TIMEOUT = 8       /* a kernel gave up a bounded wait (see tq_sync_check) */
} tq_status;

typedef enum { TQ_F32 = 0, TQ_BF16 = 1 } tq_dtype;

typedef enum {
  TQ_ROT_AUTO = 0,      /* Hadamard for power-of-two d, Haar otherwise          */
  TQ_ROT_HADAMARD = 1,  /* R = H D3 H D2 H D1 (orthonormal Walsh-Hadamard H)   */
  TQ_ROT_HAAR = 2       /* seeded Haar orthogonal matrix, stored fp32          */
} tq_rotation;

typedef struct {
  int d, b, w, m;          /* dimension, total bits, MSE bits (b-1), QJL rows */
  int rotation;            /* TQ_ROT_HADAMARD or TQ_ROT_HAAR actually used     */
  int device;              /* CUDA device the tables live on, -1 if host-only   */
  uint64_t seed;
  size_t code_bytes;       /* w*d/8  per vector */
  size_t sign_bytes;       /* m/8    per vector */
  double coord_mse;        /* Lloyd-Max distortion per coordinate, D_w          */
} tq_info_t;

/* Human-readable name of a status code (static string, never NULL). */
const char *tq_status_string(tq_status s);

/* Packed bytes of one encoded vector: codes (w*d/8) + sign bits (m/8) + the
 * two fp32 norms (8), i.e. what one row occupies across the three output
 * arrays of tq_encode.  0 for a NULL quantizer.  (tq_info gives the split.) */
size_t tq_code_bytes(const tq_quantizer *q);

/* ---------------------------------------------------------------- set-up
 * tq_codebook: build a quantizer on the current CUDA device.
 *   d: dimension, a multiple of 32 in [32, 4096]; b: total bits per
 *   coordinate in [2, 5] (w = b-1 MSE bits, then 1 QJL bit); m: QJL rows,
 *   must equal d (0 = d); seed: selects every random draw; rot: rotation kind
 *   (Hadamard needs power-of-two d).
 * Host work: the w-bit Lloyd-Max quantizer of the coordinate density
 * proportional to (1-x^2)^((d-3)/2) on [-1,1] (TurboQuant article 1.2.2,
 * 2.2.1; fitted on the exact density, equal-probability start, symmetric,
 * stops when no centroid moves by more than 1e-14 of the largest);
 * D1..D3 in {+-1}^d or a Haar matrix (QR of a Gaussian matrix with the sign
 * fix, TurboQuant article 1.2.1); S in R^{m x d} Gaussian stored at fp16
 * precision (TurboQuant article 2.3.2).  Random draws use SplitMix64
 * (Steele, Lea, Flood 2014) streams keyed by seed: stream 0-2 the diagonals,
 * 3 the entries of S, 4 the Gaussian matrix of the Haar rotation;
 * Box-Muller (cosine branch) turns word pairs into N(0,1).
 * Deterministic in (d, b, m, seed, rot).  *out receives an owned handle;
 * release it with tq_destroy. */
tq_status tq_codebook(int d, int b, int m, uint64_t seed, tq_rotation rot,
                      tq_quantizer **out);
/* tq_codebook_host: the same tables, host memory only (no CUDA device is
 * touched).  For inspection and cross-checks on machines without a GPU;
 * device entry points return TQ_ERR_UNSUPPORTED for such a quantizer. */
tq_status tq_codebook_host(int d, int b, int m, uint64_t seed, tq_rotation rot,
                           tq_quantizer **out);
/* tq_codebook_mse: a TurboQuant-MSE quantizer (TurboQuant article 4.1.1,
 * which recommends 3-bit TurboQuant-MSE for most heads, and 4.2.1, which
 * quantizes a vector index with it): all b bits of a coordinate go to the
 * Lloyd-Max codebook (w = b, b in [1, 4]) and there is no QJL stage (m = 0,
 * no sign bits: tq_encode's `signs` and tq_prepare_queries' `p` may be NULL
 * and are not touched).  The same rotation and codebook fit as tq_codebook.
 * The score is ||x|| <y~, c[codes]>: biased, every inner product is shrunk
 * on average by 1 - d D_b (D_b = coord_mse of tq_info), which the
 * inner-product mode's QJL stage removes.  Supported: encode of bf16 or fp32
 * keys with the Hadamard rotation at d in {32, 64, 128}; scoring and top-k
 * at d <= 128.  Other configurations return TQ_ERR_UNSUPPORTED. */
tq_status tq_codebook_mse(int d, int b, uint64_t seed, tq_rotation rot, tq_quantizer **out);
tq_status tq_codebook_mse_host(int d, int b, uint64_t seed, tq_rotation rot,
                               tq_quantizer **out);
void tq_destroy(tq_quantizer *q);
tq_status tq_info(const tq_quantizer *q, tq_info_t *info);

/* Host copies of the quantizer's tables, for inspection and cross-checks.
 * centroids: 2^w doubles, thresholds: 2^w - 1 doubles (either may be NULL).
 * rotation: d*d floats, row-major R (u = R x); Hadamard quantizers write the
 * dense product H D3 H D2 H D1 rounded to fp32.  diag_signs: 3*d int8 (+-1,
 * D1 then D2 then D3; Hadamard only, else untouched).  qjl: m*d fp16 bit
 * patterns of S, row-major.  Any pointer may be NULL. */
tq_status tq_codebook_get(const tq_quantizer *q, double *centroids,
                          double *thresholds, double *coord_mse);
tq_status tq_tables_get(const tq_quantizer *q, float *rotation,
                        int8_t *diag_signs, uint16_t *qjl);

/* ---------------------------------------------------------------- attention
 * tq_attend: attention of queries over a quantized KV cache (TurboQuant
 * article 4.1.1: the cache's keys and values are both quantized, with
 * TurboQuant-MSE recommended for most heads; 4.1.2: the values are
 * dequantized for the attention product, fp16 on the critical path).
 *   qv: the values' quantizer: TurboQuant-MSE (tq_codebook_mse), Hadamard,
 *       d = 64 or 128, b in [2, 4].
 *   logits: device fp32; row g*G + q at logits + (g*G + q)*ldl holds the
 *       logits of query q of group g against keys key_base .. key_base +
 *       nkeys - 1 of the group (tq_score's output layout; ldl >= nkeys).
 *   scale: multiplies the logits before the softmax (1/sqrt(d) for scaled
 *       dot-product attention); finite.
 *   vcodes, vnorms: device, tq_encode(qv) of the values; group g's keys are
 *       rows [g*keys_per_group, (g+1)*keys_per_group), of which keys
 *       [key_base, key_base + nkeys) are attended (nkeys >= 1).
 *   out: device fp32, row g*G + q at out + (g*G + q)*ldo (ldo >= d):
 *       sum_k softmax_k(scale * logits) v^_k with v^_k = ||v_k|| R^T c[codes_k]
 *       (the TurboQuant-MSE reconstruction of value k), d floats.
 *   G in [1, 16]; workspace: device, 16-byte aligned, at least
 *       tq_attend_workspace_bytes(qv, groups, G, nkeys) bytes (it depends on
 *       the device's SM count: query it on the device that runs the call).
 * The weights softmax_k ||v_k|| / max ||v|| and the centroids are fp16, the
 * products are accumulated in fp32 on the tensor cores: each output
 * coordinate is within about 2^-10 sum_k softmax_k ||v_k|| of the exact
 * value.  groups == 0 or G == 0: no-op.  Other d, b, rotation or a
 * non-MSE quantizer: TQ_ERR_UNSUPPORTED. */
size_t tq_attend_workspace_bytes(const tq_quantizer *qv, int64_t groups, int64_t G, int64_t nkeys);
tq_status tq_attend(const tq_quantizer *qv, const float *logits, int64_t ldl, int64_t groups,
                    int64_t G, float scale, const void *vcodes, const float *vnorms,
                    int64_t keys_per_group, int64_t key_base, int64_t nkeys, float *out,
                    int64_t ldo, void *workspace, size_t workspace_bytes, void *stream);

/* On-the-fly QJL matrix (TurboQuant article 2.3.2: the random projection is
 * generated from a pseudo-random sequence instead of being stored).
 * tq_set_qjl_onthefly(q, enable): with enable != 0 the kernels that can
 * generate S do so from the quantizer seed instead of reading the stored
 * table: the bf16 Hadamard encode at d = 64 and 128 (each CTA generates S in
 * shared memory) and the fused Hadamard query preparation of tq_score at
 * d <= 128 (each thread generates its row of S).  The generator is the one
 * described under tq_codebook (SplitMix64 stream 3, Box-Muller in double,
 * one rounding to fp16), so every output is bit-identical to the stored-S
 * result; other paths keep reading the table, which stays allocated.
 * The generation costs time (Box-Muller in double precision per entry);
 * the stored table is 2*m*d bytes and stays in L2, so the default is off.
 * Not thread-safe with launches that use q.  TQ_ERR_INVALID_ARG for NULL. */
tq_status tq_set_qjl_onthefly(tq_quantizer *q, int enable);
/* tq_qjl_matrix: S (m x d fp16 bit patterns, row-major) generated on the
 * device by that generator into the caller's device buffer s16 (2*m*d
 * bytes), on `stream`.  TQ_ERR_UNSUPPORTED for host-only or m = 0
 * quantizers. */
tq_status tq_qjl_matrix(const tq_quantizer *q, uint16_t *s16, void *stream);

/* ---------------------------------------------------------------- encode
 * tq_encode: quantize n vectors (TurboQuant article 1.2.3, 2.3, 4.2.1).
 *   x: device, row r at x + r*ldx elements of `dtype`; 16-byte aligned, and
 *      ldx*sizeof(dtype) a multiple of 16.
 *   chan: NULL, or device int32 [groups][d] channel map: coordinate j of row r
 *      is x[r*ldx + chan[(r / chan_rows)*d + j]] (used to encode a subset of
 *      channels, e.g. a head's outlier channels).  chan_rows > 0 when chan is
 *      given.  Without chan, coordinate j is x[r*ldx + j] and ldx >= d.
 *   codes, signs, norms: device outputs; row r is written at
 *      codes + r*out_stride*code_bytes, signs + r*out_stride*sign_bytes,
 *      norms + 2*r*out_stride (out_stride >= 1; a caller appends into a
 *      cache by offsetting the pointers).  codes/signs 4-byte aligned, norms
 *      8-byte aligned.
 * Per row: ||x|| (fp32), x_hat = x/||x|| (0 for a zero row), u = R x_hat,
 * code_j = #{thresholds < u_j}, r = u - c[code], gamma = ||r||,
 * sign bit i = [(S r)_i >= 0].
 * tq_encode takes no workspace and allocates nothing: it serves the
 * quantizers whose encode needs no scratch (tq_encode_workspace_bytes == 0,
 * the Hadamard rotation at d <= 128) and returns TQ_ERR_WORKSPACE for the
 * others, which are encoded with tq_encode_ws and a caller-owned workspace. */
tq_status tq_encode(const tq_quantizer *q, const void *x, tq_dtype dtype,
                    int64_t n, int64_t ldx, const int32_t *chan,
                    int64_t chan_rows, void *codes, void *signs, float *norms,
                    int64_t out_stride, void *stream);

/* Scratch (bytes of device memory) tq_encode needs for n rows; 0 for
 * Hadamard quantizers of d <= 128.  The others (Haar, and Hadamard above
 * d = 128) process rows in batches through this workspace; pass it to
 * tq_encode_ws (16-byte aligned; a smaller workspace means smaller batches,
 * TQ_ERR_WORKSPACE when it cannot hold one).  From d = 256 the batches run
 * as integer tensor-core GEMMs on 31-bit fixed-point operands (exact
 * products), up to 32768 rows and about 8*d bytes per row. */
size_t tq_encode_workspace_bytes(const tq_quantizer *q, int64_t n);
tq_status tq_encode_ws(const tq_quantizer *q, const void *x, tq_dtype dtype,
                       int64_t n, int64_t ldx, const int32_t *chan,
                       int64_t chan_rows, void *codes, void *signs,
                       float *norms, int64_t out_stride, void *workspace,
                       size_t workspace_bytes, void *stream);

/* ---------------------------------------------------------------- queries
 * tq_prepare_queries: y~ = R y and p = S y~ in fp32 (the same rotation as the
 * keys, TurboQuant article 4.2.2).  y: device fp32, row i at y + i*ldy (or
 * gathered through ychan [groups][d] with group = i / ychan_rows, as in
 * tq_encode).  ytil: nq x d, p: nq x m, device fp32, caller-allocated. */
tq_status tq_prepare_queries(const tq_quantizer *q, const float *y, int64_t nq,
                             int64_t ldy, const int32_t *ychan,
                             int64_t ychan_rows, float *ytil, float *p,
                             void *stream);

/* ---------------------------------------------------------------- score
 * tq_score: asymmetric estimate of <y, x> for grouped keys and queries
 * (KV-cache attention logits; blog 四).
 *   Keys: groups*keys_per_group encoded rows (codes/signs/norms as written by
 *   tq_encode with out_stride 1); key k of group g is row g*keys_per_group+k.
 *   Queries: groups*G fp32 rows of y (ldy, optional ychan gather with
 *   ychan_rows = G); query i of group g is row g*G + i.
 *   out: device fp32 [groups*G][keys_per_group]; query row g*G+i, column k
 *   receives s = ||x|| * (<y~, c[codes]> + gamma*sqrt(pi/2)/m * <p, 2*bits-1>)
 *   (added to the existing value when accumulate != 0).
 *   workspace: device, at least tq_score_workspace_bytes(q, groups*G) bytes,
 *   16-byte aligned (holds the prepared queries; for d > 128 also the
 *   queries' fp16 pieces and one 32768-key chunk of decoded keys, 2*(2d+m)
 *   bytes per key, for the tensor-core GEMM that scores them).
 * Arithmetic: d <= 128 scores with exact integer products of 16-bit
 * fixed-point limbs; d > 128 with fp16 pieces and fp32 accumulation (error
 * well inside 1e-3 of max(|s|, ||x|| ||y|| / sqrt(d))). */
size_t tq_score_workspace_bytes(const tq_quantizer *q, int64_t nq);
tq_status tq_score(const tq_quantizer *q, const float *y, int64_t groups,
                   int64_t G, int64_t ldy, const int32_t *ychan,
                   const void *codes, const void *signs, const float *norms,
                   int64_t keys_per_group, float *out, int accumulate,
                   void *workspace, size_t workspace_bytes, void *stream);

/* ---------------------------------------------------------------- score in two halves
 * tq_score split at the point where the queries and the keys meet (blog 四:
 * the query is rotated and projected once, then scored against every packed
 * key).  Together the two calls compute exactly what tq_score computes, with
 * the same kernels and the same logits bit for bit, when the keys are 16-byte
 * aligned (tq_encode's outputs are).  The query half depends on the queries
 * only, so it may run on another stream while the keys are still being
 * encoded, or once for several key sets.
 *
 * tq_score_prepare: the query half.  Arguments as tq_score's (y, groups, G,
 *   ldy, ychan); writes the prepared queries into `workspace` (at least
 *   tq_score_workspace_bytes(q, groups*G) bytes, 16-byte aligned).  For
 *   d <= 128 that is the scorer's full query operand (the rotated query y~ and
 *   its projection p = S y~, as 16-bit fixed-point limbs with their scales);
 *   for d > 128, y~ and p in fp32 (the scoring GEMM builds its fp16 pieces).
 * tq_score_prepared: the key half.  Arguments as tq_score's (codes, signs,
 *   norms, keys_per_group, out, accumulate), with groups and G equal to the
 *   prepare call's and the workspace it wrote, unchanged since.  codes and
 *   signs must be 16-byte aligned (4-byte for quantizers that score on the CUDA
 *   cores: d > 128 without the tensor-core route, or G > 48), else
 *   TQ_ERR_ALIGNMENT.  For d > 128 the call also uses the workspace's scratch
 *   region (the decoded-key chunk): two such calls must not share a workspace
 *   at the same time.
 * Ownership and errors as tq_score; both calls are asynchronous on `stream`,
 * and the caller orders the prepare before the prepared call when they are on
 * different streams. */
tq_status tq_score_prepare(const tq_quantizer *q, const float *y, int64_t groups,
                           int64_t G, int64_t ldy, const int32_t *ychan,
                           void *workspace, size_t workspace_bytes, void *stream);
tq_status tq_score_prepared(const tq_quantizer *q, int64_t groups, int64_t G,
                            const void *codes, const void *signs,
                            const float *norms, int64_t keys_per_group,
                            float *out, int accumulate, void *workspace,
                            size_t workspace_bytes, void *stream);

/* ---------------------------------------------------------------- score, no allocation
 * tq_score_noalloc: the same scores as tq_score, for callers that cannot hand
 * the library a workspace.  (No counterpart in the TurboQuant pages; this is
 * an interface for embedding.)  Typical such callers: code running while a
 * framework's caching allocator holds the device memory (a direct allocation
 * would fail or fragment that pool), latency-critical paths where the device
 * synchronization an allocation can cause is not acceptable, and plugin hosts
 * that forbid device allocation once started.
 *
 * Scratch comes from one buffer of TQ_NOALLOC_SCRATCH_BYTES compiled into the
 * library as a device variable: every GPU that loads the library holds it
 * until the process exits.  Arguments and layouts are those of tq_score.
 * Results: for d <= 128 the same kernels run as in tq_score (the integer
 * tensor-core scorer), so the logits are bit-identical to tq_score's; for
 * d > 128 the scores come from the CUDA-core scorer (tq_score uses a
 * tensor-core GEMM there, whose decoded-key chunk does not fit the buffer),
 * equal to tq_score's within the score tolerance stated at tq_score.  The
 * call allocates and frees nothing.
 *   - Needed scratch: per query 4*(d + m) + 16 bytes, plus 384 bytes for each
 *     of roundup(5*G, 16) operand rows per group when G <= 48 (each piece
 *     rounded up to 256 bytes).  Larger requests return TQ_ERR_TOO_LARGE
 *     before anything is launched.
 *   - The first call on each device looks up the buffer's device address
 *     (cudaGetSymbolAddress) with that device current; make that first call
 *     outside any stream capture.
 *   - All calls share the one buffer and it keeps the last call's contents:
 *     calls whose work overlaps on the GPU (other streams, other host
 *     threads) race on it and return wrong scores.  Order them on one stream. */
#define TQ_NOALLOC_SCRATCH_BYTES (8u << 20)
tq_status tq_score_noalloc(const tq_quantizer *q, const float *y, int64_t groups,
                           int64_t G, int64_t ldy, const int32_t *ychan,
                           const void *codes, const void *signs,
                           const float *norms, int64_t keys_per_group,
                           float *out, int accumulate, void *stream);

/* ---------------------------------------------------------------- top-k
 * tq_topk: the k highest estimates per query over n keys (TurboQuant article
 * 4.2.2, first stage of two-stage retrieval).  y: nq fp32 rows (ldy).
 * out_scores: nq x k fp32, out_idx: nq x k int64 (device), sorted by
 * descending score, equal scores by ascending key index.  1 <= k <= 64 and
 * k <= n (the bound of this library's selection kernels; retrieval keeps a
 * short candidate list).  workspace: at least tq_topk_workspace_bytes(q, nq,
 * n, k) bytes.  For d > 128 and k <= 16 the selection is fused into the
 * scoring GEMM: each CTA keeps the 16 best (score, key) pairs per query in
 * registers and only those candidates reach memory, never the logits; codes
 * and signs must then be 16-byte aligned (TQ_ERR_ALIGNMENT otherwise).  The
 * other cases score 65536-key chunks into the workspace and select from
 * there.  Either way the returned scores are bit-identical to tq_score's
 * logits of the returned keys. */
size_t tq_topk_workspace_bytes(const tq_quantizer *q, int64_t nq, int64_t n,
                               int k);
tq_status tq_topk(const tq_quantizer *q, const float *y, int64_t nq,
                  int64_t ldy, const void *codes, const void *signs,
                  const float *norms, int64_t n, int k, float *out_scores,
                  int64_t *out_idx, void *workspace, size_t workspace_bytes,
                  void *stream);

/* ---------------------------------------------------------------- rerank
 * tq_rerank: the second stage of two-stage retrieval (TurboQuant article
 * 4.2.2: screen a top-K on the quantized vectors, then refine that candidate
 * set).  For query i, every candidate key cand[i][c] is re-scored with the
 * exact inner product <y_i, x_key> against the raw database vectors (fp32
 * arithmetic), and the k best are written, by descending score, equal
 * scores by ascending key index.  Typical use: cand = tq_topk's out_idx for
 * K' > k, x = the vectors that were encoded.
 *   y: device fp32 [nq][ldy] (ldy >= d); x: device [n][ldx] of `dtype`
 *   (16-byte aligned, ldx*sizeof(dtype) a multiple of 16, ldx >= d); d a
 *   multiple of 8.  cand: device int64 [nq][kc], 1 <= kc <= 4096; entries
 *   outside [0, n) are empty slots and duplicates count once.  out_scores
 *   fp32 / out_idx int64 [nq][k], 1 <= k <= min(64, kc); a row with fewer
 *   than k valid candidates is padded with (-inf, -1).  No workspace; the
 *   call needs no quantizer. */
tq_status tq_rerank(const float *y, int64_t nq, int64_t ldy, const void *x,
                    tq_dtype dtype, int64_t n, int64_t ldx, int d,
                    const int64_t *cand, int kc, int k, float *out_scores,
                    int64_t *out_idx, void *stream);

/* ---------------------------------------------------------------- outliers
 * tq_outlier_channels: per group of rows, the `count` channels of highest
 * mean square (the outlier channels kept at more bits; TurboQuant article
 * 4.1.1 suggests about 25%).  x: device, groups*rows_per_group rows of `dim`
 * channels (ldx, dtype).  Sums of squares are accumulated in fp64 on the
 * device; ties go to the lower channel index.  out_sel: device int32
 * [groups][count] selected channels ascending; out_rest: device int32
 * [groups][dim-count] the other channels ascending (either may be NULL).
 * workspace: tq_outlier_workspace_bytes(groups, dim) bytes.  Synchronizes
 * `stream` (the selection runs on the host). */
size_t tq_outlier_workspace_bytes(int64_t groups, int dim);
tq_status tq_outlier_channels(const void *x, tq_dtype dtype, int64_t groups,
                              int64_t rows_per_group, int dim, int64_t ldx,
                              int count, int32_t *out_sel, int32_t *out_rest,
                              void *workspace, size_t workspace_bytes,
                              void *stream);

/* ---------------------------------------------------------------- failures
 * Every wait inside the tensor-core kernels is bounded (about 2 s).  A kernel
 * whose wait ran out records a nonzero code in the quantizer's device error
 * word, stops, frees what it holds and returns; the outputs of that call are
 * not valid, and the CUDA context stays usable.  (No counterpart in the
 * TurboQuant pages: this is how the library reports a stalled pipeline.)
 *
 * tq_sync_check: synchronizes `stream`, then reads the error word of q.
 * Returns TQ_OK if no wait ran out since the last check, TQ_ERR_TIMEOUT if
 * one did (the word is cleared), TQ_ERR_CUDA if the stream itself failed.
 *
 * tq_selftest_timeout: launches on `stream` one kernel whose wait can never
 * be satisfied, so that it runs out (after about 2 s) and records its code:
 * a test of the failure path that faults and hangs nothing.  Follow it with
 * tq_sync_check, which then returns TQ_ERR_TIMEOUT. */
tq_status tq_sync_check(const tq_quantizer *q, void *stream);
tq_status tq_selftest_timeout(const tq_quantizer *q, void *stream);

#ifdef __cplusplus
}
#endif

#endif /* TQ_H */

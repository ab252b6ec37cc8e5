// Internal kernel entry points of libtq (called by the C ABI in tq_api.cu).
#pragma once

#include <cuda_runtime.h>
#include <cudaTypedefs.h>

#include "tq_common.cuh"

namespace tq {

tq_status v1_encode_fwht(const tq_quantizer *q, const RowSource &src, int64_t n, void *codes,
                         void *signs, float *norms, int64_t out_stride, cudaStream_t st);
size_t v1_dense_ws_bytes(const tq_quantizer *q, int64_t n);
size_t v1_dense_batch_rows(const tq_quantizer *q, size_t ws_bytes);
tq_status v1_encode_dense(const tq_quantizer *q, const RowSource &src, int64_t n, void *codes,
                          void *signs, float *norms, int64_t out_stride, void *ws, size_t ws_bytes,
                          cudaStream_t st);
tq_status v1_prepare_queries(const tq_quantizer *q, const RowSource &src, int64_t nq, float *ytil,
                             float *p, cudaStream_t st);
tq_status v1_score(const tq_quantizer *q, const float *ytil, const float *p, int64_t nq_rows, int64_t G,
                   int64_t keys_per_group, int64_t key_base, int64_t nkeys, const void *codes,
                   const void *signs, const float *norms, float *out, int64_t ldo, int accumulate,
                   cudaStream_t st);
tq_status v1_topk_select(float *score, const int64_t *idx, int64_t rows, int64_t row_stride, int64_t cnt,
                         int64_t slice, int64_t base, int k, float *out_s, int64_t *out_i,
                         int64_t out_row_stride, cudaStream_t st);
tq_status v1_sumsq(const RowSource &src, int64_t groups, int64_t rows_per_group, double *part, int nchunks,
                   double *out, cudaStream_t st);

// One CTA whose mbarrier wait can never complete: the bounded wait runs out
// and records its code in *err (the failure path, tested without a fault).
tq_status launch_wait_selftest(int *err, cudaStream_t st);

// cuTensorMapEncodeTiled from the driver (null if unavailable)
PFN_cuTensorMapEncodeTiled_v12000 tensor_map_encoder();

// Dense rotation (any d that is a multiple of 64, from 256 up) on the tensor
// cores: both projections as fp16-piece GEMMs with fused epilogues.
bool dense_tc_supported(const tq_quantizer *q);
size_t dense_tc_ws_bytes(const tq_quantizer *q, int64_t n);
tq_status dense_tc_encode(const tq_quantizer *q, const RowSource &src, int64_t n, void *codes, void *signs,
                          float *norms, int64_t out_stride, void *ws, size_t ws_bytes, cudaStream_t st);

// Scoring for d > 128 as an fp16 tensor-core GEMM over decoded keys (same
// arguments and output as v1_score, plus its workspace).
bool dense_score_supported(const tq_quantizer *q);
size_t dense_score_ws_bytes(const tq_quantizer *q, int64_t nq);
tq_status dense_score(const tq_quantizer *q, const float *ytil, const float *p, int64_t nq_rows, int64_t G,
                      int64_t kpg, int64_t key_base, int64_t nkeys, const void *codes, const void *signs,
                      const float *norms, float *out, int64_t ldo, int accumulate, void *ws, size_t ws_bytes,
                      cudaStream_t st);

// Top-k for d > 128 with the selection fused into the scoring GEMM (no
// logits in memory); k <= 16.
size_t dense_topk_ws_bytes(const tq_quantizer *q, int64_t nq, int64_t n);
tq_status dense_topk(const tq_quantizer *q, const float *ytil, const float *p, int64_t nq, int64_t n, int k,
                     const void *codes, const void *signs, const float *norms, float *out_s, int64_t *out_i,
                     void *ws, size_t ws_bytes, cudaStream_t st);

// Exact re-scoring of candidate keys against raw vectors, then top-k.
// attention over a quantized KV cache (values in TurboQuant-MSE)
bool attend_supported(const tq_quantizer *qv);
size_t attend_ws_bytes(int64_t groups, int64_t G, int d, int64_t nkeys);
tq_status attend_launch(const tq_quantizer *qv, const float *logits, int64_t ldl, int64_t groups, int64_t G,
                        float scale, const void *vcodes, const float *vnorms, int64_t kpg, int64_t key_base,
                        int64_t nkeys, float *out, int64_t ldo, void *ws, size_t ws_bytes, cudaStream_t st);
// S generated on the device from its stream key: count fp16 entries, row-major
tq_status qjl_matrix_launch(uint64_t key, int64_t count, uint16_t *s16, cudaStream_t st);
tq_status rerank_launch(const float *y, int64_t nq, int64_t ldy, const void *x, bool bf16, int64_t n, int64_t ldx,
                        int d, const int64_t *cand, int kc, int k, float *out_s, int64_t *out_i, cudaStream_t st);

// fp32 (or gathered) rows, Hadamard d in {32, 64, 128}: rotation on the CUDA
// cores, QJL projection on the tensor cores.
bool fwht_tc_encode_supported(const tq_quantizer *q);
tq_status fwht_tc_encode(const tq_quantizer *q, const RowSource &src, int64_t n, void *codes, void *signs,
                         float *norms, int64_t out_stride, cudaStream_t st);

bool tc_encode_supported(const tq_quantizer *q, int dtype, int64_t ldx, bool gather);
tq_status tc_encode(const tq_quantizer *q, const void *x, int64_t n, int64_t ldx, const int32_t *chan,
                    int64_t chan_rows, void *codes, void *signs, float *norms, int64_t out_stride,
                    cudaStream_t st);

// Gathered bf16 rows (per-group channel map), d in {32, 64, 96}, Hadamard or
// Haar: the tc2 structure with a gather step.
bool tcg_encode_supported(const tq_quantizer *q, int dtype, int64_t ldx, bool gather);
tq_status tcg_encode(const tq_quantizer *q, const void *x, int64_t n, int64_t ldx, const int32_t *chan,
                     int64_t chan_rows, void *codes, void *signs, float *norms, int64_t out_stride,
                     cudaStream_t st);

bool tc2_encode_supported(const tq_quantizer *q, int dtype, bool gather);
tq_status tc2_encode(const tq_quantizer *q, const void *x, int64_t n, int64_t ldx, void *codes, void *signs,
                     float *norms, int64_t out_stride, cudaStream_t st);

// Integer tensor-core scorer (d <= 128), in two halves: the query operand
// and scales (qop, qsc) from the queries alone, then the scores of packed
// keys against them.  tc_score and tc_score_y run both halves.
bool tc_score_supported(const tq_quantizer *q, int64_t G);
// the query half from raw queries for Hadamard d = 32, 64, 128: query
// preparation and the operand fused in one kernel (bit-identical to
// tc_score_queries after v1_prepare_queries)
bool tc_score_y_supported(const tq_quantizer *q, int64_t G);
tq_status tc_score_y_queries(const tq_quantizer *q, const RowSource &src, int64_t groups, int64_t G, int8_t *qop,
                             float4 *qsc, cudaStream_t st);
tq_status tc_score_y(const tq_quantizer *q, const RowSource &src, int64_t groups, int64_t G, int64_t kpg,
                     const void *codes, const void *signs, const float *norms, float *out, int64_t ldo,
                     int accumulate, int8_t *qop, float4 *qsc, cudaStream_t st);
size_t tc_score_qop_bytes(const tq_quantizer *q, int64_t groups, int64_t G);
// the query half from prepared queries (y~, p)
tq_status tc_score_queries(const tq_quantizer *q, const float *ytil, const float *pq, int64_t groups, int64_t G,
                           int8_t *qop, float4 *qsc, cudaStream_t st);
// the key half: keys [key_base, key_base + nkeys) of every group.  keys_ready:
// the previous kernel of the stream is the query half (the scorer may read
// keys and allocate TMEM before its dependency wait); otherwise it waits first
tq_status tc_score_keys(const tq_quantizer *q, int64_t groups, int64_t G, int64_t kpg, int64_t key_base,
                        int64_t nkeys, const void *codes, const void *signs, const float *norms, float *out,
                        int64_t ldo, int accumulate, const int8_t *qop, const float4 *qsc, bool keys_ready,
                        cudaStream_t st);
tq_status tc_score(const tq_quantizer *q, const float *ytil, const float *pq, int64_t groups, int64_t G,
                   int64_t kpg, int64_t key_base, int64_t nkeys, const void *codes, const void *signs,
                   const float *norms, float *out, int64_t ldo, int accumulate, int8_t *qop, float4 *qsc,
                   cudaStream_t st);

}  // namespace tq

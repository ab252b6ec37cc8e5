// C ABI entry points of libtq that launch device work (encode, query
// preparation, scoring, top-k, outlier-channel choice).  Argument checks
// happen here, before anything is launched; see include/tq.h for the
// contract of each call.
#include <cmath>
#include <algorithm>
#include <cstring>
#include <mutex>
#include <vector>

#include "tq_kernels.h"

namespace {

using namespace tq;

struct DeviceGuard {
  int prev = -1;
  bool ok = true;
  explicit DeviceGuard(int dev) {
    if (cudaGetDevice(&prev) != cudaSuccess) {
      ok = false;
      return;
    }
    if (prev != dev && cudaSetDevice(dev) != cudaSuccess) ok = false;
  }
  ~DeviceGuard() {
    int cur = -1;
    if (prev >= 0 && cudaGetDevice(&cur) == cudaSuccess && cur != prev) cudaSetDevice(prev);
  }
};

inline bool aligned(const void *p, size_t a) { return (reinterpret_cast<uintptr_t>(p) % a) == 0; }
inline size_t round_up(size_t v, size_t a) { return (v + a - 1) / a * a; }
inline bool fwht_fast(const tq_quantizer *q) {
  return q->rotation == TQ_ROT_HADAMARD && (q->d == 32 || q->d == 64 || q->d == 128);
}

// Validates a row source; *empty is set when n == 0 (a no-op that needs no
// pointers), in which case TQ_OK is returned before any pointer check.
tq_status check_rows(const tq_quantizer *q, const void *x, int dtype, int64_t n, int64_t ldx,
                     const int32_t *chan, int64_t chan_rows, bool *empty = nullptr) {
  if (!q || n < 0 || (dtype != TQ_F32 && dtype != TQ_BF16)) return TQ_ERR_INVALID_ARG;
  if (q->device < 0) return TQ_ERR_UNSUPPORTED;  // host-only quantizer
  if (empty) *empty = (n == 0);
  if (n == 0 && empty) return TQ_OK;
  if (!x) return TQ_ERR_INVALID_ARG;
  if (chan ? chan_rows <= 0 : ldx < q->d) return TQ_ERR_INVALID_ARG;
  if (ldx < 1) return TQ_ERR_INVALID_ARG;
  const size_t es = dtype == TQ_BF16 ? 2 : 4;
  if (!aligned(x, 16) || ((size_t)ldx * es) % 16 != 0) return TQ_ERR_ALIGNMENT;
  if (chan && !aligned(chan, 4)) return TQ_ERR_ALIGNMENT;
  return TQ_OK;
}

}  // namespace

extern "C" {

size_t tq_encode_workspace_bytes(const tq_quantizer *q, int64_t n) {
  if (!q || n <= 0 || fwht_fast(q)) return 0;
  if (q->device >= 0 && dense_tc_supported(q)) return round_up(dense_tc_ws_bytes(q, n), 256);
  return round_up(v1_dense_ws_bytes(q, n), 256);
}

tq_status tq_encode_ws(const tq_quantizer *q, const void *x, tq_dtype dtype, int64_t n, int64_t ldx,
                       const int32_t *chan, int64_t chan_rows, void *codes, void *signs, float *norms,
                       int64_t out_stride, void *workspace, size_t workspace_bytes, void *stream) {
  bool empty = false;
  tq_status st = check_rows(q, x, dtype, n, ldx, chan, chan_rows, &empty);
  if (st != TQ_OK || empty) return st;
  if (!codes || (!signs && q->m > 0) || !norms || out_stride < 1) return TQ_ERR_INVALID_ARG;
  if (!aligned(codes, 4) || !aligned(signs, 4) || !aligned(norms, 8)) return TQ_ERR_ALIGNMENT;
  DeviceGuard g(q->device);
  if (!g.ok) return TQ_ERR_CUDA;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  RowSource src{x, ldx, chan, chan_rows, q->d, dtype == TQ_BF16};
  if (q->m == 0) {  // TurboQuant-MSE: the Hadamard kernels have a variant without the QJL stage
    if (tc2_encode_supported(q, dtype, chan != nullptr))
      return tc2_encode(q, x, n, ldx, codes, signs, norms, out_stride, s);
    if (fwht_fast(q)) return v1_encode_fwht(q, src, n, codes, signs, norms, out_stride, s);
    return TQ_ERR_UNSUPPORTED;
  }
  if (tc2_encode_supported(q, dtype, chan != nullptr))
    return tc2_encode(q, x, n, ldx, codes, signs, norms, out_stride, s);
  if (tcg_encode_supported(q, dtype, ldx, chan != nullptr))
    return tcg_encode(q, x, n, ldx, chan, chan_rows, codes, signs, norms, out_stride, s);
  if (tc_encode_supported(q, dtype, ldx, chan != nullptr))
    return tc_encode(q, x, n, ldx, chan, chan_rows, codes, signs, norms, out_stride, s);
  if (fwht_tc_encode_supported(q)) return fwht_tc_encode(q, src, n, codes, signs, norms, out_stride, s);
  if (fwht_fast(q)) return v1_encode_fwht(q, src, n, codes, signs, norms, out_stride, s);
  if (!workspace || !aligned(workspace, 16)) return TQ_ERR_WORKSPACE;
  if (dense_tc_supported(q))
    return dense_tc_encode(q, src, n, codes, signs, norms, out_stride, workspace, workspace_bytes, s);
  if (v1_dense_batch_rows(q, workspace_bytes) < 1) return TQ_ERR_WORKSPACE;
  return v1_encode_dense(q, src, n, codes, signs, norms, out_stride, workspace, workspace_bytes, s);
}

tq_status tq_encode(const tq_quantizer *q, const void *x, tq_dtype dtype, int64_t n, int64_t ldx,
                    const int32_t *chan, int64_t chan_rows, void *codes, void *signs, float *norms,
                    int64_t out_stride, void *stream) {
  if (!q) return TQ_ERR_INVALID_ARG;
  // the workspace-free form: quantizers that need scratch are encoded by
  // tq_encode_ws with caller-owned memory (the library allocates nothing)
  if (n > 0 && tq_encode_workspace_bytes(q, n) != 0) {
    bool empty = false;
    tq_status st = check_rows(q, x, dtype, n, ldx, chan, chan_rows, &empty);
    return st != TQ_OK ? st : TQ_ERR_WORKSPACE;
  }
  return tq_encode_ws(q, x, dtype, n, ldx, chan, chan_rows, codes, signs, norms, out_stride, nullptr, 0,
                      stream);
}

size_t tq_attend_workspace_bytes(const tq_quantizer *qv, int64_t groups, int64_t G, int64_t nkeys) {
  if (!qv || groups < 0 || G < 0 || nkeys < 0) return 0;
  if (groups == 0 || G == 0 || nkeys == 0 || qv->device < 0) return 0;
  DeviceGuard g(qv->device);
  if (!g.ok) return 0;
  return tq::attend_ws_bytes(groups, G, qv->d, nkeys);
}

tq_status tq_attend(const tq_quantizer *qv, const float *logits, int64_t ldl, int64_t groups, int64_t G,
                    float scale, const void *vcodes, const float *vnorms, int64_t keys_per_group, int64_t key_base,
                    int64_t nkeys, float *out, int64_t ldo, void *workspace, size_t workspace_bytes, void *stream) {
  if (!qv || groups < 0 || G < 0 || keys_per_group < 0 || key_base < 0 || nkeys < 0) return TQ_ERR_INVALID_ARG;
  if (qv->device < 0 || !tq::attend_supported(qv)) return TQ_ERR_UNSUPPORTED;
  if (groups == 0 || G == 0) return TQ_OK;
  if (G > 16) return TQ_ERR_UNSUPPORTED;
  if (nkeys == 0 || key_base + nkeys > keys_per_group || ldl < nkeys || ldo < qv->d) return TQ_ERR_INVALID_ARG;
  if (!logits || !vcodes || !vnorms || !out || !std::isfinite(scale)) return TQ_ERR_INVALID_ARG;
  if (!aligned(logits, 4) || !aligned(vcodes, 4) || !aligned(vnorms, 8) || !aligned(out, 4)) return TQ_ERR_ALIGNMENT;
  if (!workspace || !aligned(workspace, 16)) return TQ_ERR_WORKSPACE;
  DeviceGuard g(qv->device);
  if (!g.ok) return TQ_ERR_CUDA;
  if (workspace_bytes < tq::attend_ws_bytes(groups, G, qv->d, nkeys)) return TQ_ERR_WORKSPACE;
  return tq::attend_launch(qv, logits, ldl, groups, G, scale, vcodes, vnorms, keys_per_group, key_base, nkeys, out,
                           ldo, workspace, workspace_bytes, static_cast<cudaStream_t>(stream));
}

tq_status tq_set_qjl_onthefly(tq_quantizer *q, int enable) {
  if (!q) return TQ_ERR_INVALID_ARG;
  q->kt.qjl_otf = enable ? 1 : 0;
  return TQ_OK;
}

tq_status tq_qjl_matrix(const tq_quantizer *q, uint16_t *s16, void *stream) {
  if (!q || !s16) return TQ_ERR_INVALID_ARG;
  if (q->device < 0 || q->m == 0) return TQ_ERR_UNSUPPORTED;
  return tq::qjl_matrix_launch(q->kt.qjl_key, (int64_t)q->m * q->d, s16, static_cast<cudaStream_t>(stream));
}

size_t tq_code_bytes(const tq_quantizer *q) {
  if (!q) return 0;
  return (size_t)q->w * q->d / 8 + (size_t)q->m / 8 + 8;
}

tq_status tq_prepare_queries(const tq_quantizer *q, const float *y, int64_t nq, int64_t ldy,
                             const int32_t *ychan, int64_t ychan_rows, float *ytil, float *p, void *stream) {
  bool empty = false;
  tq_status st = check_rows(q, y, TQ_F32, nq, ldy, ychan, ychan_rows, &empty);
  if (st != TQ_OK || empty) return st;
  if (!ytil || (!p && q->m > 0)) return TQ_ERR_INVALID_ARG;
  if (!aligned(ytil, 16) || !aligned(p, 16)) return TQ_ERR_ALIGNMENT;
  DeviceGuard g(q->device);
  if (!g.ok) return TQ_ERR_CUDA;
  RowSource src{y, ldy, ychan, ychan_rows, q->d, 0};
  return v1_prepare_queries(q, src, nq, ytil, p, static_cast<cudaStream_t>(stream));
}

// Workspace of tq_score: prepared queries (y~, p), then the integer scorer's
// query operand (at most 16 rows of 384 bytes per query) and per-query scales.
struct ScoreLayout {
  size_t ytil, p, qop, qsc, dense, total;
};
ScoreLayout score_layout(const tq_quantizer *q, int64_t nq) {
  ScoreLayout L{};
  size_t off = 0;
  L.ytil = off;
  off += round_up((size_t)nq * q->d * 4, 256);
  L.p = off;
  off += round_up((size_t)nq * q->m * 4, 256);
  L.qop = off;
  off += round_up((size_t)nq * 16 * 384, 256);
  L.qsc = off;
  off += round_up((size_t)nq * 16, 256);
  L.dense = off;
  if (dense_score_supported(q)) off += round_up(dense_score_ws_bytes(q, nq), 256);
  L.total = off;
  return L;
}

size_t tq_score_workspace_bytes(const tq_quantizer *q, int64_t nq) {
  if (!q || nq <= 0) return 0;
  return score_layout(q, nq).total;
}

tq_status tq_score(const tq_quantizer *q, const float *y, int64_t groups, int64_t G, int64_t ldy,
                   const int32_t *ychan, const void *codes, const void *signs, const float *norms,
                   int64_t keys_per_group, float *out, int accumulate, void *workspace,
                   size_t workspace_bytes, void *stream) {
  if (!q || groups < 0 || G < 0 || keys_per_group < 0) return TQ_ERR_INVALID_ARG;
  const int64_t nq = groups * G;
  bool empty = false;
  tq_status st = check_rows(q, y, TQ_F32, nq, ldy, ychan, G > 0 ? G : 1, &empty);
  if (st != TQ_OK || empty) return st;
  if (!codes || (!signs && q->m > 0) || !norms || !out) return TQ_ERR_INVALID_ARG;
  if (!aligned(codes, 4) || !aligned(signs, 4) || !aligned(norms, 8) || !aligned(out, 4)) return TQ_ERR_ALIGNMENT;
  if (nq == 0 || keys_per_group == 0) return TQ_OK;
  if (!workspace || !aligned(workspace, 16) || workspace_bytes < tq_score_workspace_bytes(q, nq))
    return TQ_ERR_WORKSPACE;
  DeviceGuard g(q->device);
  if (!g.ok) return TQ_ERR_CUDA;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  const ScoreLayout L = score_layout(q, nq);
  char *ws = static_cast<char *>(workspace);
  float *ytil = reinterpret_cast<float *>(ws + L.ytil);
  float *p = reinterpret_cast<float *>(ws + L.p);
  RowSource src{y, ldy, ychan, G, q->d, 0};
  if (tc_score_y_supported(q, G) && aligned(codes, 16) && aligned(signs, 16))
    return tc_score_y(q, src, groups, G, keys_per_group, codes, signs, norms, out, keys_per_group, accumulate,
                      reinterpret_cast<int8_t *>(ws + L.qop), reinterpret_cast<float4 *>(ws + L.qsc), s);
  st = v1_prepare_queries(q, src, nq, ytil, p, s);
  if (st != TQ_OK) return st;
  if (tc_score_supported(q, G) && aligned(codes, 16) && aligned(signs, 16))
    return tc_score(q, ytil, p, groups, G, keys_per_group, 0, keys_per_group, codes, signs, norms, out,
                    keys_per_group, accumulate, reinterpret_cast<int8_t *>(ws + L.qop),
                    reinterpret_cast<float4 *>(ws + L.qsc), s);
  if (dense_score_supported(q) && aligned(codes, 16) && aligned(signs, 16))
    return dense_score(q, ytil, p, nq, G, keys_per_group, 0, keys_per_group, codes, signs, norms, out,
                       keys_per_group, accumulate, ws + L.dense, L.total - L.dense, s);
  return v1_score(q, ytil, p, nq, G, keys_per_group, 0, keys_per_group, codes, signs, norms, out,
                  keys_per_group, accumulate, s);
}

// The scoring route for (q, G) when the keys are 16-byte aligned; the query
// half (tq_score_prepare) and the key half (tq_score_prepared) take the same one.
enum ScorePath { kPathTcY, kPathTc, kPathDense, kPathV1 };
static ScorePath score_path(const tq_quantizer *q, int64_t G) {
  if (tc_score_y_supported(q, G)) return kPathTcY;
  if (tc_score_supported(q, G)) return kPathTc;
  if (dense_score_supported(q)) return kPathDense;
  return kPathV1;
}

tq_status tq_score_prepare(const tq_quantizer *q, const float *y, int64_t groups, int64_t G, int64_t ldy,
                           const int32_t *ychan, void *workspace, size_t workspace_bytes, void *stream) {
  if (!q || groups < 0 || G < 0) return TQ_ERR_INVALID_ARG;
  const int64_t nq = groups * G;
  bool empty = false;
  tq_status st = check_rows(q, y, TQ_F32, nq, ldy, ychan, G > 0 ? G : 1, &empty);
  if (st != TQ_OK || empty || nq == 0) return st;
  if (!workspace || !aligned(workspace, 16) || workspace_bytes < tq_score_workspace_bytes(q, nq))
    return TQ_ERR_WORKSPACE;
  DeviceGuard g(q->device);
  if (!g.ok) return TQ_ERR_CUDA;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  const ScoreLayout L = score_layout(q, nq);
  char *ws = static_cast<char *>(workspace);
  float *ytil = reinterpret_cast<float *>(ws + L.ytil);
  float *p = reinterpret_cast<float *>(ws + L.p);
  RowSource src{y, ldy, ychan, G, q->d, 0};
  const ScorePath path = score_path(q, G);
  if (path == kPathTcY)
    return tc_score_y_queries(q, src, groups, G, reinterpret_cast<int8_t *>(ws + L.qop),
                              reinterpret_cast<float4 *>(ws + L.qsc), s);
  st = v1_prepare_queries(q, src, nq, ytil, p, s);
  if (st != TQ_OK || path != kPathTc) return st;
  return tc_score_queries(q, ytil, p, groups, G, reinterpret_cast<int8_t *>(ws + L.qop),
                          reinterpret_cast<float4 *>(ws + L.qsc), s);
}

tq_status tq_score_prepared(const tq_quantizer *q, int64_t groups, int64_t G, const void *codes,
                            const void *signs, const float *norms, int64_t keys_per_group, float *out,
                            int accumulate, void *workspace, size_t workspace_bytes, void *stream) {
  if (!q || groups < 0 || G < 0 || keys_per_group < 0) return TQ_ERR_INVALID_ARG;
  if (q->device < 0) return TQ_ERR_UNSUPPORTED;  // host-only quantizer
  const int64_t nq = groups * G;
  if (!codes || (!signs && q->m > 0) || !norms || !out) return TQ_ERR_INVALID_ARG;
  const ScorePath path = score_path(q, G);
  const int key_align = path == kPathV1 ? 4 : 16;
  if (!aligned(codes, key_align) || !aligned(signs, key_align) || !aligned(norms, 8) || !aligned(out, 4))
    return TQ_ERR_ALIGNMENT;
  if (nq == 0 || keys_per_group == 0) return TQ_OK;
  if (!workspace || !aligned(workspace, 16) || workspace_bytes < tq_score_workspace_bytes(q, nq))
    return TQ_ERR_WORKSPACE;
  DeviceGuard g(q->device);
  if (!g.ok) return TQ_ERR_CUDA;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  const ScoreLayout L = score_layout(q, nq);
  char *ws = static_cast<char *>(workspace);
  const float *ytil = reinterpret_cast<const float *>(ws + L.ytil);
  const float *p = reinterpret_cast<const float *>(ws + L.p);
  const int64_t kpg = keys_per_group;
  switch (path) {
    case kPathTcY:
    case kPathTc:
      // the kernel before this call may be anything (an encode of these keys):
      // the scorer waits for it before reading keys or allocating TMEM
      return tc_score_keys(q, groups, G, kpg, 0, kpg, codes, signs, norms, out, kpg, accumulate,
                           reinterpret_cast<const int8_t *>(ws + L.qop), reinterpret_cast<const float4 *>(ws + L.qsc),
                           false, s);
    case kPathDense:
      // the dense path's own scratch follows the prepared queries in the workspace
      return dense_score(q, ytil, p, nq, G, kpg, 0, kpg, codes, signs, norms, out, kpg, accumulate, ws + L.dense,
                         L.total - L.dense, s);
    default:
      return v1_score(q, ytil, p, nq, G, kpg, 0, kpg, codes, signs, norms, out, kpg, accumulate, s);
  }
}

}  // extern "C"

namespace {
constexpr int64_t kTopkChunk = 65536;
constexpr int64_t kTopkSlice = 2048;

struct TopkLayout {
  size_t ytil, p, qop, qsc, scores, part_s, part_i, dense, total;
  int64_t chunk, nparts;
};

// d > 128 with k <= 16: the selection runs inside the scoring GEMM
inline bool topk_fused_dense(const tq_quantizer *q, int k) { return dense_score_supported(q) && k <= 16; }

TopkLayout topk_layout(const tq_quantizer *q, int64_t nq, int64_t n, int k) {
  TopkLayout L{};
  L.chunk = std::min<int64_t>(n, kTopkChunk);
  L.nparts = (n + kTopkSlice - 1) / kTopkSlice;
  size_t off = 0;
  L.ytil = off;
  off += round_up((size_t)nq * q->d * 4, 256);
  L.p = off;
  off += round_up((size_t)nq * q->m * 4, 256);
  if (topk_fused_dense(q, k)) {
    L.dense = off;
    off += round_up(dense_topk_ws_bytes(q, nq, n), 256);
    L.total = off;
    return L;
  }
  L.qop = off;
  off += round_up((size_t)std::min<int64_t>(nq, 48) * 16 * 384, 256);
  L.qsc = off;
  off += round_up((size_t)nq * 16, 256);
  L.scores = off;
  off += round_up((size_t)nq * L.chunk * 4, 256);
  L.part_s = off;
  off += round_up((size_t)nq * L.nparts * k * 4, 256);
  L.part_i = off;
  off += round_up((size_t)nq * L.nparts * k * 8, 256);
  L.dense = off;
  if (dense_score_supported(q)) off += round_up(dense_score_ws_bytes(q, nq), 256);
  L.total = off;
  return L;
}
}  // namespace

extern "C" {

size_t tq_topk_workspace_bytes(const tq_quantizer *q, int64_t nq, int64_t n, int k) {
  if (!q || nq <= 0 || n <= 0 || k <= 0) return 0;
  return topk_layout(q, nq, n, k).total;
}

tq_status tq_topk(const tq_quantizer *q, const float *y, int64_t nq, int64_t ldy, const void *codes,
                  const void *signs, const float *norms, int64_t n, int k, float *out_scores, int64_t *out_idx,
                  void *workspace, size_t workspace_bytes, void *stream) {
  bool empty = false;
  tq_status st = check_rows(q, y, TQ_F32, nq, ldy, nullptr, 0, &empty);
  if (st != TQ_OK || empty) return st;
  if (n < 0 || !codes || (!signs && q->m > 0) || !norms || !out_scores || !out_idx) return TQ_ERR_INVALID_ARG;
  if (k < 1 || k > 64 || k > n) return TQ_ERR_INVALID_ARG;
  if (!aligned(codes, 4) || !aligned(signs, 4) || !aligned(norms, 8) || !aligned(out_idx, 8) ||
      !aligned(out_scores, 4))
    return TQ_ERR_ALIGNMENT;
  const TopkLayout L = topk_layout(q, nq, n, k);
  if (!workspace || !aligned(workspace, 16) || workspace_bytes < L.total) return TQ_ERR_WORKSPACE;
  DeviceGuard g(q->device);
  if (!g.ok) return TQ_ERR_CUDA;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  char *ws = static_cast<char *>(workspace);
  float *ytil = reinterpret_cast<float *>(ws + L.ytil);
  float *p = reinterpret_cast<float *>(ws + L.p);
  float *scores = reinterpret_cast<float *>(ws + L.scores);
  float *part_s = reinterpret_cast<float *>(ws + L.part_s);
  int64_t *part_i = reinterpret_cast<int64_t *>(ws + L.part_i);
  RowSource src{y, ldy, nullptr, 0, q->d, 0};
  st = v1_prepare_queries(q, src, nq, ytil, p, s);
  if (st != TQ_OK) return st;
  if (topk_fused_dense(q, k)) {
    if (!aligned(codes, 16) || !aligned(signs, 16)) return TQ_ERR_ALIGNMENT;
    return dense_topk(q, ytil, p, nq, n, k, codes, signs, norms, out_scores, out_idx, ws + L.dense, L.total - L.dense,
                      s);
  }
  const bool tc = tc_score_supported(q, std::min<int64_t>(nq, 48)) && aligned(codes, 16) && aligned(signs, 16);
  const bool dense = !tc && dense_score_supported(q) && aligned(codes, 16) && aligned(signs, 16);
  for (int64_t c0 = 0; c0 < n; c0 += L.chunk) {
    const int64_t cnt = std::min(L.chunk, n - c0);
    if (tc) {
      for (int64_t qb = 0; qb < nq; qb += 48) {  // query batches share one operand buffer
        const int64_t nb = std::min<int64_t>(48, nq - qb);
        st = tc_score(q, ytil + qb * q->d, p + qb * q->m, 1, nb, n, c0, cnt, codes, signs, norms,
                      scores + qb * L.chunk, L.chunk, 0, reinterpret_cast<int8_t *>(ws + L.qop),
                      reinterpret_cast<float4 *>(ws + L.qsc) + qb, s);
        if (st != TQ_OK) return st;
      }
    } else if (dense) {
      st = dense_score(q, ytil, p, nq, nq, n, c0, cnt, codes, signs, norms, scores, L.chunk, 0, ws + L.dense,
                       L.total - L.dense, s);
    } else {
      st = v1_score(q, ytil, p, nq, nq, n, c0, cnt, codes, signs, norms, scores, L.chunk, 0, s);
    }
    if (st != TQ_OK) return st;
    st = v1_topk_select(scores, nullptr, nq, L.chunk, cnt, kTopkSlice, c0, k, part_s + (c0 / kTopkSlice) * k,
                        part_i + (c0 / kTopkSlice) * k, L.nparts * k, s);
    if (st != TQ_OK) return st;
  }
  return v1_topk_select(part_s, part_i, nq, L.nparts * k, L.nparts * k, L.nparts * k, 0, k, out_scores, out_idx,
                        k, s);
}

tq_status tq_rerank(const float *y, int64_t nq, int64_t ldy, const void *x, tq_dtype dtype, int64_t n, int64_t ldx,
                    int d, const int64_t *cand, int kc, int k, float *out_scores, int64_t *out_idx, void *stream) {
  if (nq < 0 || n < 0 || d <= 0 || kc < 1 || k < 1 || (dtype != TQ_F32 && dtype != TQ_BF16))
    return TQ_ERR_INVALID_ARG;
  if (nq == 0) return TQ_OK;
  if (!y || !x || !cand || !out_scores || !out_idx || ldy < d || ldx < d) return TQ_ERR_INVALID_ARG;
  if (k > 64 || k > kc || kc > 4096 || d % 8 != 0 || d > 16384) return TQ_ERR_UNSUPPORTED;
  const size_t es = dtype == TQ_BF16 ? 2 : 4;
  if (!aligned(x, 16) || ((size_t)ldx * es) % 16 != 0 || !aligned(cand, 8) || !aligned(out_idx, 8) ||
      !aligned(out_scores, 4) || !aligned(y, 4))
    return TQ_ERR_ALIGNMENT;
  return rerank_launch(y, nq, ldy, x, dtype == TQ_BF16, n, ldx, d, cand, kc, k, out_scores, out_idx,
                       static_cast<cudaStream_t>(stream));
}

size_t tq_outlier_workspace_bytes(int64_t groups, int dim) {
  if (groups <= 0 || dim <= 0) return 0;
  return round_up((size_t)groups * 64 * dim * 8, 256) + round_up((size_t)groups * dim * 8, 256);
}

tq_status tq_outlier_channels(const void *x, tq_dtype dtype, int64_t groups, int64_t rows_per_group, int dim,
                              int64_t ldx, int count, int32_t *out_sel, int32_t *out_rest, void *workspace,
                              size_t workspace_bytes, void *stream) {
  if (!x || groups < 0 || rows_per_group < 0 || dim <= 0 || ldx < dim || count < 0 || count > dim ||
      (dtype != TQ_F32 && dtype != TQ_BF16))
    return TQ_ERR_INVALID_ARG;
  const size_t es = dtype == TQ_BF16 ? 2 : 4;
  if (!aligned(x, 16) || ((size_t)ldx * es) % 16 != 0) return TQ_ERR_ALIGNMENT;
  if (groups == 0) return TQ_OK;
  if (!workspace || !aligned(workspace, 16) || workspace_bytes < tq_outlier_workspace_bytes(groups, dim))
    return TQ_ERR_WORKSPACE;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  double *part = static_cast<double *>(workspace);
  double *fin = reinterpret_cast<double *>(static_cast<char *>(workspace) + round_up((size_t)groups * 64 * dim * 8, 256));
  const int nchunks = (int)std::max<int64_t>(1, std::min<int64_t>(64, rows_per_group));
  RowSource src{x, ldx, nullptr, 0, dim, dtype == TQ_BF16};
  tq_status st = v1_sumsq(src, groups, rows_per_group, part, nchunks, fin, s);
  if (st != TQ_OK) return st;
  std::vector<double> ms((size_t)groups * dim);
  if (cudaMemcpyAsync(ms.data(), fin, ms.size() * 8, cudaMemcpyDeviceToHost, s) != cudaSuccess ||
      cudaStreamSynchronize(s) != cudaSuccess)
    return TQ_ERR_CUDA;
  std::vector<int32_t> sel((size_t)groups * count), rest((size_t)groups * (dim - count));
  std::vector<int> order(dim);
  for (int64_t gi = 0; gi < groups; ++gi) {
    const double *v = &ms[(size_t)gi * dim];
    for (int c = 0; c < dim; ++c) order[c] = c;
    std::stable_sort(order.begin(), order.end(), [&](int a, int b) { return v[a] > v[b]; });
    std::vector<int> a(order.begin(), order.begin() + count), b(order.begin() + count, order.end());
    std::sort(a.begin(), a.end());
    std::sort(b.begin(), b.end());
    std::copy(a.begin(), a.end(), sel.begin() + gi * count);
    std::copy(b.begin(), b.end(), rest.begin() + gi * (dim - count));
  }
  if (out_sel && count > 0 &&
      cudaMemcpyAsync(out_sel, sel.data(), sel.size() * 4, cudaMemcpyHostToDevice, s) != cudaSuccess)
    return TQ_ERR_CUDA;
  if (out_rest && dim - count > 0 &&
      cudaMemcpyAsync(out_rest, rest.data(), rest.size() * 4, cudaMemcpyHostToDevice, s) != cudaSuccess)
    return TQ_ERR_CUDA;
  if (cudaStreamSynchronize(s) != cudaSuccess) return TQ_ERR_CUDA;
  return TQ_OK;
}


tq_status tq_sync_check(const tq_quantizer *q, void *stream) {
  if (!q) return TQ_ERR_INVALID_ARG;
  if (q->device < 0 || !q->d_err) return TQ_ERR_UNSUPPORTED;
  DeviceGuard g(q->device);
  if (!g.ok) return TQ_ERR_CUDA;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  if (cudaStreamSynchronize(s) != cudaSuccess) return TQ_ERR_CUDA;
  int code = 0;
  if (cudaMemcpy(&code, q->d_err, sizeof(int), cudaMemcpyDeviceToHost) != cudaSuccess) return TQ_ERR_CUDA;
  if (code == 0) return TQ_OK;
  if (cudaMemset(q->d_err, 0, sizeof(int)) != cudaSuccess) return TQ_ERR_CUDA;
  return TQ_ERR_TIMEOUT;
}

tq_status tq_selftest_timeout(const tq_quantizer *q, void *stream) {
  if (!q) return TQ_ERR_INVALID_ARG;
  if (q->device < 0 || !q->d_err) return TQ_ERR_UNSUPPORTED;
  DeviceGuard g(q->device);
  if (!g.ok) return TQ_ERR_CUDA;
  return launch_wait_selftest(q->d_err, static_cast<cudaStream_t>(stream));
}

}  // extern "C"

// ---------------------------------------------------------------- no-allocation scoring
// Scratch of tq_score_noalloc: a fixed device buffer, so the call needs no
// workspace from the caller and allocates nothing.  Host code cannot use the
// symbol itself as a device pointer; its address is looked up once per
// device (with that device current) and passed to the kernels.
static __device__ __align__(256) unsigned char g_tq_noalloc_scratch[TQ_NOALLOC_SCRATCH_BYTES];

namespace {
std::mutex g_noalloc_mu;
constexpr int kMaxDevices = 64;
void *g_noalloc_addr[kMaxDevices] = {};

tq_status noalloc_scratch(int dev, void **out) {
  std::lock_guard<std::mutex> lock(g_noalloc_mu);
  if (dev < 0 || dev >= kMaxDevices) return TQ_ERR_UNSUPPORTED;
  if (!g_noalloc_addr[dev]) {
    void *p = nullptr;
    if (cudaGetSymbolAddress(&p, g_tq_noalloc_scratch) != cudaSuccess || !p) {
      cudaGetLastError();
      return TQ_ERR_CUDA;
    }
    g_noalloc_addr[dev] = p;
  }
  *out = g_noalloc_addr[dev];
  return TQ_OK;
}
}  // namespace

extern "C" tq_status tq_score_noalloc(const tq_quantizer *q, const float *y, int64_t groups, int64_t G,
                                      int64_t ldy, const int32_t *ychan, const void *codes, const void *signs,
                                      const float *norms, int64_t keys_per_group, float *out, int accumulate,
                                      void *stream) {
  if (!q || groups < 0 || G < 0 || keys_per_group < 0) return TQ_ERR_INVALID_ARG;
  const int64_t nq = groups * G;
  bool empty = false;
  tq_status st = check_rows(q, y, TQ_F32, nq, ldy, ychan, G > 0 ? G : 1, &empty);
  if (st != TQ_OK || empty) return st;
  if (!codes || (!signs && q->m > 0) || !norms || !out) return TQ_ERR_INVALID_ARG;
  if (!aligned(codes, 4) || !aligned(signs, 4) || !aligned(norms, 8) || !aligned(out, 4)) return TQ_ERR_ALIGNMENT;
  if (keys_per_group == 0) return TQ_OK;
  const bool tc = tc_score_supported(q, G) && aligned(codes, 16) && aligned(signs, 16);
  // scratch pieces for this call: y~, p, then (integer scorer only) its
  // query operand and per-query scales
  const size_t b_ytil = round_up((size_t)nq * q->d * 4, 256);
  const size_t b_p = round_up((size_t)nq * q->m * 4, 256);
  const size_t b_qop = tc ? round_up(tc_score_qop_bytes(q, groups, G), 256) : 0;
  const size_t b_qsc = tc ? round_up((size_t)nq * 16, 256) : 0;
  if (b_ytil + b_p + b_qop + b_qsc > TQ_NOALLOC_SCRATCH_BYTES) return TQ_ERR_TOO_LARGE;
  DeviceGuard g(q->device);
  if (!g.ok) return TQ_ERR_CUDA;
  void *base = nullptr;
  st = noalloc_scratch(q->device, &base);
  if (st != TQ_OK) return st;
  char *ws = static_cast<char *>(base);
  float *ytil = reinterpret_cast<float *>(ws);
  float *p = reinterpret_cast<float *>(ws + b_ytil);
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  RowSource src{y, ldy, ychan, G, q->d, 0};
  st = v1_prepare_queries(q, src, nq, ytil, p, s);
  if (st != TQ_OK) return st;
  if (tc)  // the operand region is cleared inside tc_score before it is filled
    return tc_score(q, ytil, p, groups, G, keys_per_group, 0, keys_per_group, codes, signs, norms, out,
                    keys_per_group, accumulate, reinterpret_cast<int8_t *>(ws + b_ytil + b_p),
                    reinterpret_cast<float4 *>(ws + b_ytil + b_p + b_qop), s);
  return v1_score(q, ytil, p, nq, G, keys_per_group, 0, keys_per_group, codes, signs, norms, out,
                  keys_per_group, accumulate, s);
}

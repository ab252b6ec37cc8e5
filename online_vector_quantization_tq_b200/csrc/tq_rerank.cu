// Second stage of two-stage retrieval (TurboQuant article 4.2.2: a top-K is
// screened on the quantized vectors, then the candidate set is refined):
// each query's candidates are re-scored with the exact inner product against
// the stored raw vectors and the k best are kept.
//
// One CTA per query.  Warps take candidates in turn; a warp reads its
// candidate's row with one 16-byte (fp32) or 8-byte (bf16) load per lane
// per step and reduces the fp32 dot product with shuffles.  The candidates'
// scores stay in shared memory for the selection (k passes of a block-wide
// arg-max, ties to the lower key index, duplicates taken once).
#include "tq_kernels.h"

namespace tq {

namespace {

constexpr int kRerankThreads = 256;

__device__ __forceinline__ bool rerank_better(float a, int64_t ia, float b, int64_t ib) {
  return a > b || (a == b && ia < ib);
}

template <bool BF16>
__global__ void __launch_bounds__(kRerankThreads)
k_rerank(const float *y, int64_t ldy, const void *x, int64_t n, int64_t ldx, int d, const int64_t *cand, int kc,
         int k, float *out_s, int64_t *out_i) {
  extern __shared__ float4 smem4[];
  float *sy = reinterpret_cast<float *>(smem4);           // [d]
  int64_t *si = reinterpret_cast<int64_t *>(sy + d);     // [kc] candidate keys (-1: empty or taken)
  float *ss = reinterpret_cast<float *>(si + kc);         // [kc] exact scores
  __shared__ float rs[kRerankThreads / 32];
  __shared__ int64_t ri[kRerankThreads / 32];
  __shared__ int rp[kRerankThreads / 32];
  const int64_t q = blockIdx.x;
  const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
  constexpr int kWarps = kRerankThreads / 32;
  for (int j = threadIdx.x; j < d; j += kRerankThreads) sy[j] = y[q * ldy + j];
  __syncthreads();
  for (int c = warp; c < kc; c += kWarps) {
    const int64_t id = cand[q * kc + c];
    const bool valid = id >= 0 && id < n;  // out-of-range entries are treated as empty
    float acc = 0.f;
    if (valid) {
      for (int j = 4 * lane; j < d; j += 128) {
        float4 v;
        if constexpr (BF16) {
          const uint2 h = *reinterpret_cast<const uint2 *>(static_cast<const uint16_t *>(x) + id * ldx + j);
          v = make_float4(__uint_as_float(h.x << 16), __uint_as_float(h.x & 0xFFFF0000u),
                          __uint_as_float(h.y << 16), __uint_as_float(h.y & 0xFFFF0000u));
        } else {
          v = *reinterpret_cast<const float4 *>(static_cast<const float *>(x) + id * ldx + j);
        }
        acc = fmaf(v.x, sy[j], acc);
        acc = fmaf(v.y, sy[j + 1], acc);
        acc = fmaf(v.z, sy[j + 2], acc);
        acc = fmaf(v.w, sy[j + 3], acc);
      }
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, o);
    if (lane == 0) {
      ss[c] = acc;
      si[c] = valid ? id : -1;
    }
  }
  __syncthreads();
  for (int r = 0; r < k; ++r) {
    float bs = -INFINITY;
    int64_t bi = -1;
    int bp = -1;
    for (int c = threadIdx.x; c < kc; c += kRerankThreads) {
      if (si[c] < 0) continue;
      if (bp < 0 || rerank_better(ss[c], si[c], bs, bi)) {
        bs = ss[c];
        bi = si[c];
        bp = c;
      }
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) {
      const float os = __shfl_xor_sync(0xffffffffu, bs, o);
      const int64_t oi = __shfl_xor_sync(0xffffffffu, bi, o);
      const int op = __shfl_xor_sync(0xffffffffu, bp, o);
      if (op >= 0 && (bp < 0 || rerank_better(os, oi, bs, bi))) {
        bs = os;
        bi = oi;
        bp = op;
      }
    }
    if (lane == 0) {
      rs[warp] = bs;
      ri[warp] = bi;
      rp[warp] = bp;
    }
    __syncthreads();
    float fs = rs[0];
    int64_t fi = ri[0];
    int fp = rp[0];
#pragma unroll
    for (int w = 1; w < kWarps; ++w)
      if (rp[w] >= 0 && (fp < 0 || rerank_better(rs[w], ri[w], fs, fi))) {
        fs = rs[w];
        fi = ri[w];
        fp = rp[w];
      }
    if (threadIdx.x == 0) {
      out_s[q * k + r] = fp >= 0 ? fs : -INFINITY;
      out_i[q * k + r] = fp >= 0 ? fi : -1;
    }
    __syncthreads();  // every thread has read this round's winner
    if (fp >= 0)      // take it, and every duplicate of it
      for (int c = threadIdx.x; c < kc; c += kRerankThreads)
        if (si[c] == fi) si[c] = -1;
    __syncthreads();
  }
}

}  // namespace

tq_status rerank_launch(const float *y, int64_t nq, int64_t ldy, const void *x, bool bf16, int64_t n, int64_t ldx,
                        int d, const int64_t *cand, int kc, int k, float *out_s, int64_t *out_i, cudaStream_t st) {
  const size_t smem = (size_t)d * 4 + (size_t)kc * 12 + 16;
  if (bf16) {
    if (cudaFuncSetAttribute(k_rerank<true>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem) !=
        cudaSuccess)
      return TQ_ERR_CUDA;
    k_rerank<true><<<(unsigned)nq, kRerankThreads, smem, st>>>(y, ldy, x, n, ldx, d, cand, kc, k, out_s, out_i);
  } else {
    if (cudaFuncSetAttribute(k_rerank<false>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem) !=
        cudaSuccess)
      return TQ_ERR_CUDA;
    k_rerank<false><<<(unsigned)nq, kRerankThreads, smem, st>>>(y, ldy, x, n, ldx, d, cand, kc, k, out_s, out_i);
  }
  return cudaGetLastError() == cudaSuccess ? TQ_OK : TQ_ERR_CUDA;
}

}  // namespace tq

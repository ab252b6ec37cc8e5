// CUDA-core kernels of libtq: the portable path used for every configuration
// the tensor-core kernels do not cover (and as their in-library cross-check).
//
//   k_encode_fwht   one thread per vector, d in {32, 64, 128}: norm, three
//                   rounds of (+-1 diagonal, Walsh-Hadamard), scalar codebook,
//                   residual, fp32 QJL projection, bit packing
//   k_gemm_nt       fp32 tiled C = A B^T with an element-wise epilogue; dense
//                   (Haar) rotation, its QJL projection, dense query prep
//   k_pack_rows     packs the dense path's per-coordinate codes and signs
//   k_prep_fwht_block  queries: y~ = R y, p = S y~ for d in {32, 64, 128}
//   k_score_rows    asymmetric estimator, one thread per key, one query row
//                   per grid row
//   k_topk_*        per-block top-k of score rows, then a merge
//   k_sumsq_*       per-channel sums of squares (outlier channel choice)
#include "tq_common.cuh"
#include "tq_kernels.h"

namespace tq {

// ============================================================ encode (FWHT)
template <int D, int W>
__global__ void __launch_bounds__(128)
k_encode_fwht(KernelTables kt, RowSource src, int64_t n, uint32_t *codes, uint32_t *signs,
              float2 *norms, int64_t out_stride) {
  constexpr int L = 1 << W;
  const int M = kt.m;  // QJL rows: d, or 0 for TurboQuant-MSE (no sign bits)
  extern __shared__ float4 smem4[];
  float *sS = reinterpret_cast<float *>(smem4);  // M x D fp32
  __shared__ float sC[kMaxLevels];
  __shared__ float sT[kMaxLevels];
  __shared__ uint32_t sDiag[3 * D / 32];
  for (int i = threadIdx.x; i < M * D; i += blockDim.x) sS[i] = kt.qjl32[i];
  if (threadIdx.x < kMaxLevels) {
    sC[threadIdx.x] = kt.centroids[threadIdx.x];
    sT[threadIdx.x] = kt.thresholds[threadIdx.x];
  }
  if (threadIdx.x < 3 * D / 32) sDiag[threadIdx.x] = kt.diag_bits[threadIdx.x];
  __syncthreads();
  const int64_t row = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
  if (row >= n) return;

  float v[D];
#pragma unroll
  for (int j = 0; j < D; ++j) v[j] = src.at(row, j);
  float ss = 0.f;
#pragma unroll
  for (int j = 0; j < D; ++j) ss = fmaf(v[j], v[j], ss);
  const float nrm = sqrtf(ss);

#pragma unroll
  for (int r = 0; r < 3; ++r) {
    uint32_t words[D / 32];
#pragma unroll
    for (int k = 0; k < D / 32; ++k) words[k] = sDiag[r * (D / 32) + k];
    apply_signs<D>(v, words);
    fwht_regs<D>(v);
  }
  // three orthonormal rounds scale by D^-3/2; normalization by 1/||x||
  const float inv = nrm > 0.f ? 1.0f / (nrm * (float(D) * sqrtf(float(D)))) : 0.0f;

  uint32_t cw[W * D / 32];
#pragma unroll
  for (int k = 0; k < W * D / 32; ++k) cw[k] = 0u;
  float g2 = 0.f;
#pragma unroll
  for (int j = 0; j < D; ++j) {
    const float u = v[j] * inv;
    const int c = quantize<L>(u, sT);
    pack_code<W>(&cw[(j / 32) * W], j % 32, (uint32_t)c);
    const float r = u - sC[c];
    v[j] = r;
    g2 = fmaf(r, r, g2);
  }
  const int64_t orow = row * out_stride;
#pragma unroll
  for (int k = 0; k < W * D / 32; ++k) codes[orow * (W * D / 32) + k] = cw[k];

  for (int wi = 0; wi < M / 32; ++wi) {
    uint32_t word = 0u;
    for (int ii = 0; ii < 32; ++ii) {
      const float4 *srow = reinterpret_cast<const float4 *>(sS + (size_t)(wi * 32 + ii) * D);
      float z0 = 0.f, z1 = 0.f, z2 = 0.f, z3 = 0.f;
#pragma unroll
      for (int j = 0; j < D / 4; ++j) {
        const float4 s4 = srow[j];
        z0 = fmaf(s4.x, v[4 * j + 0], z0);
        z1 = fmaf(s4.y, v[4 * j + 1], z1);
        z2 = fmaf(s4.z, v[4 * j + 2], z2);
        z3 = fmaf(s4.w, v[4 * j + 3], z3);
      }
      const float z = (z0 + z1) + (z2 + z3);
      word |= (z >= 0.f ? 1u : 0u) << ii;
    }
    signs[orow * (M / 32) + wi] = word;
  }
  norms[orow] = make_float2(nrm, sqrtf(g2));
}

// ============================================================ dense GEMM
// C[i][j] = sum_k A(i,k) B(j,k); 64x64 tiles, BK = 16, 256 threads, 4x4 each.
struct LoadRows {  // A(i,k) = row i of a RowSource (dtype, channel gather)
  RowSource src;
  int64_t row0;
  __device__ __forceinline__ float operator()(int64_t i, int k) const { return src.at(row0 + i, k); }
};
struct LoadMat {  // A(i,k) = p[i*ld + k], fp32
  const float *p;
  int64_t ld;
  __device__ __forceinline__ float operator()(int64_t i, int k) const { return p[i * ld + k]; }
};

template <class LA, class LB, class Epi>
__global__ void __launch_bounds__(256)
k_gemm_nt(int64_t M, int N, int K, LA la, LB lb, Epi epi) {
  __shared__ float As[16][64 + 4];
  __shared__ float Bs[16][64 + 4];
  const int tx = threadIdx.x % 16, ty = threadIdx.x / 16;
  const int64_t i0 = (int64_t)blockIdx.x * 64;
  const int j0 = blockIdx.y * 64;
  float acc[4][4] = {};
  for (int k0 = 0; k0 < K; k0 += 16) {
    for (int e = threadIdx.x; e < 64 * 16; e += 256) {
      const int r = e / 16, k = e % 16;
      const int64_t gi = i0 + r;
      const int gj = j0 + r, gk = k0 + k;
      As[k][r] = (gi < M && gk < K) ? la(gi, gk) : 0.f;
      Bs[k][r] = (gj < N && gk < K) ? lb(gj, gk) : 0.f;
    }
    __syncthreads();
#pragma unroll
    for (int k = 0; k < 16; ++k) {
      float a[4], b[4];
#pragma unroll
      for (int q = 0; q < 4; ++q) {
        a[q] = As[k][ty + 16 * q];
        b[q] = Bs[k][tx + 16 * q];
      }
#pragma unroll
      for (int p = 0; p < 4; ++p)
#pragma unroll
        for (int q = 0; q < 4; ++q) acc[p][q] = fmaf(a[p], b[q], acc[p][q]);
    }
    __syncthreads();
  }
#pragma unroll
  for (int p = 0; p < 4; ++p)
#pragma unroll
    for (int q = 0; q < 4; ++q) {
      const int64_t gi = i0 + ty + 16 * p;
      const int gj = j0 + tx + 16 * q;
      if (gi < M && gj < N) epi(gi, gj, acc[p][q]);
    }
}

// u = acc / ||x||, then code and residual (dense rotation epilogue)
struct EpiRotQuant {
  KernelTables kt;
  const float2 *norms;  // this batch's rows
  int64_t norm_stride;  // in float2
  float *r;             // batch x d
  uint8_t *code;        // batch x d
  __device__ __forceinline__ void operator()(int64_t i, int j, float acc) const {
    const float nrm = norms[i * norm_stride].x;
    const float u = nrm > 0.f ? acc / nrm : 0.f;
    int c = 0;
    for (int t = 0; t < kt.levels - 1; ++t) c += (u > kt.thresholds[t]) ? 1 : 0;
    r[i * kt.d + j] = u - kt.centroids[c];
    code[i * kt.d + j] = (uint8_t)c;
  }
};
struct EpiSignByte {
  uint8_t *sign;
  int m;
  __device__ __forceinline__ void operator()(int64_t i, int j, float acc) const {
    sign[i * m + j] = acc >= 0.f ? 1 : 0;
  }
};
struct EpiStore {
  float *out;
  int64_t ld;
  __device__ __forceinline__ void operator()(int64_t i, int j, float acc) const { out[i * ld + j] = acc; }
};

__global__ void k_row_norms(RowSource src, int64_t n, float2 *norms, int64_t out_stride) {
  const int64_t row = (int64_t)blockIdx.x * (blockDim.x / 32) + threadIdx.x / 32;
  const int lane = threadIdx.x % 32;
  if (row >= n) return;
  float ss = 0.f;
  for (int j = lane; j < src.d; j += 32) {
    const float v = src.at(row, j);
    ss = fmaf(v, v, ss);
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) ss += __shfl_xor_sync(0xffffffffu, ss, o);
  if (lane == 0) norms[row * out_stride] = make_float2(sqrtf(ss), 0.f);
}

template <int W>
__global__ void k_pack_rows(int d, int m, int64_t rows, const uint8_t *code, const uint8_t *sign,
                            const float *r, uint32_t *codes, uint32_t *signs, float2 *norms,
                            int64_t out_stride) {
  const int64_t row = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
  if (row >= rows) return;
  const int64_t orow = row * out_stride;
  for (int g = 0; g < d / 32; ++g) {
    uint32_t w[W];
#pragma unroll
    for (int k = 0; k < W; ++k) w[k] = 0u;
#pragma unroll
    for (int i = 0; i < 32; ++i) pack_code<W>(w, i, code[row * d + g * 32 + i]);
#pragma unroll
    for (int k = 0; k < W; ++k) codes[orow * (W * d / 32) + g * W + k] = w[k];
  }
  for (int g = 0; g < m / 32; ++g) {
    uint32_t w = 0u;
    for (int i = 0; i < 32; ++i) w |= (uint32_t)sign[row * m + g * 32 + i] << i;
    signs[orow * (m / 32) + g] = w;
  }
  float g2 = 0.f;
  for (int j = 0; j < d; ++j) {
    const float v = r[row * d + j];
    g2 = fmaf(v, v, g2);
  }
  norms[orow].y = sqrtf(g2);
}

// ============================================================ queries
// One block of D threads per query: sign flips and Walsh-Hadamard butterflies
// in shared memory, then p = S y~ with each warp reducing whole rows of S.
template <int D>
__global__ void __launch_bounds__(D)
k_prep_fwht_block(KernelTables kt, RowSource src, int64_t nq, float *ytil, float *p) {
  __shared__ float v[D];
  const int64_t row = blockIdx.x;
  const int j = threadIdx.x;
  float x = src.at(row, j);
#pragma unroll
  for (int r = 0; r < 3; ++r) {
    const uint32_t word = kt.diag_bits[r * (D / 32) + j / 32];
    x = ((word >> (j % 32)) & 1u) ? -x : x;
    // butterflies: partners within a warp by shuffle, across warps through
    // shared memory (the same a + b and b - a either way)
#pragma unroll
    for (int h = 1; h < D; h <<= 1) {
      float b;
      if (h < 32) {
        b = __shfl_xor_sync(0xffffffffu, x, h);
      } else {
        __syncthreads();  // the previous reads of v are done
        v[j] = x;
        __syncthreads();
        b = v[j ^ h];
      }
      x = (j & h) ? b - x : x + b;
    }
  }
  __syncthreads();  // the last butterfly's reads of v are done
  x *= 1.0f / (float(D) * sqrtf(float(D)));
  v[j] = x;
  ytil[row * D + j] = x;
  if (kt.m == 0) return;  // TurboQuant-MSE: no QJL projection (uniform over the block)
  __syncthreads();
  // p_j = sum_k S[j][k] y~_k: thread j reads row j of S with independent
  // 16-byte loads (one L2 round trip), four partial sums over k mod 4 (the
  // same order as the integer scorer's fused query preparation)
  float acc0 = 0.f, acc1 = 0.f, acc2 = 0.f, acc3 = 0.f;
  const float4 *srow = reinterpret_cast<const float4 *>(kt.qjl32 + (size_t)j * D);
#pragma unroll
  for (int k4 = 0; k4 < D / 4; ++k4) {
    const float4 s4 = __ldg(srow + k4);
    acc0 = fmaf(s4.x, v[4 * k4], acc0);
    acc1 = fmaf(s4.y, v[4 * k4 + 1], acc1);
    acc2 = fmaf(s4.z, v[4 * k4 + 2], acc2);
    acc3 = fmaf(s4.w, v[4 * k4 + 3], acc3);
  }
  p[row * D + j] = (acc0 + acc1) + (acc2 + acc3);
}

// Dense rotation, d <= 128: one block per query; y~ = R y walks the
// transposed R and p = S y~ the transposed S, so every warp load is one
// contiguous segment.
__global__ void k_prep_dense_block(KernelTables kt, RowSource src, int64_t nq, float *ytil, float *p) {
  __shared__ float sv[128];
  const int d = kt.d, m = kt.m;
  const int64_t row = blockIdx.x;
  const int j = threadIdx.x;
  if (j < d) sv[j] = src.at(row, j);
  __syncthreads();
  // four partial sums, eight loads in flight per thread
  auto dot = [&](const float *mt, int stride, int col) {
    float a[4] = {0.f, 0.f, 0.f, 0.f};
    int k = 0;
    for (; k + 8 <= d; k += 8) {
      float v[8];
#pragma unroll
      for (int u = 0; u < 8; ++u) v[u] = __ldg(mt + (size_t)(k + u) * stride + col);
#pragma unroll
      for (int u = 0; u < 8; ++u) a[u % 4] = fmaf(v[u], sv[k + u], a[u % 4]);
    }
    for (; k < d; ++k) a[0] = fmaf(__ldg(mt + (size_t)k * stride + col), sv[k], a[0]);
    return (a[0] + a[1]) + (a[2] + a[3]);
  };
  float yt = 0.f;
  if (j < d) yt = dot(kt.rott, d, j);
  __syncthreads();
  if (j < d) {
    sv[j] = yt;
    ytil[row * d + j] = yt;
  }
  __syncthreads();
  for (int i = j; i < m; i += blockDim.x) p[row * m + i] = dot(kt.qjl32t, m, i);
}

// ============================================================ score
// One query row per grid row (blockIdx.y), one key per thread.
template <int W>
__global__ void __launch_bounds__(128)
k_score_rows(KernelTables kt, const float *ytil, const float *p, int64_t G, int64_t keys_per_group,
             int64_t key_base, int64_t nkeys, const uint32_t *codes, const uint32_t *signs,
             const float2 *norms, float *out, int64_t ldo, int accumulate) {
  extern __shared__ float4 smem4[];
  float *sy = reinterpret_cast<float *>(smem4);
  float *sp = sy + kt.d;
  __shared__ float sC[kMaxLevels];
  const int64_t qrow = blockIdx.y;
  for (int j = threadIdx.x; j < kt.d; j += blockDim.x) sy[j] = ytil[qrow * kt.d + j];
  for (int j = threadIdx.x; j < kt.m; j += blockDim.x) sp[j] = p[qrow * kt.m + j];
  if (threadIdx.x < kMaxLevels) sC[threadIdx.x] = kt.centroids[threadIdx.x];
  __syncthreads();
  const int64_t k = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;  // within this call's keys
  if (k >= nkeys) return;
  const int64_t group = qrow / G;
  const int64_t key = group * keys_per_group + key_base + k;
  const uint32_t *cw = codes + key * (W * kt.d / 32);
  const uint32_t *sw = signs + key * (kt.m / 32);
  float a1 = 0.f, a2 = 0.f;
  for (int g = 0; g < kt.d / 32; ++g) {
    uint32_t w[W];
#pragma unroll
    for (int t = 0; t < W; ++t) w[t] = cw[g * W + t];
#pragma unroll
    for (int i = 0; i < 32; ++i) a1 = fmaf(sy[g * 32 + i], sC[unpack_code<W>(w, i)], a1);
  }
  for (int g = 0; g < kt.m / 32; ++g) {
    const uint32_t s = sw[g];
#pragma unroll
    for (int i = 0; i < 32; ++i) {
      const float pv = sp[g * 32 + i];
      a2 += ((s >> i) & 1u) ? pv : -pv;
    }
  }
  const float2 nr = norms[key];
  const float sc = nr.x * fmaf(nr.y * kt.qjl_scale, a2, a1);
  float *o = out + qrow * ldo + k;
  *o = accumulate ? *o + sc : sc;
}

// ============================================================ top-k
__device__ __forceinline__ bool better(float a, int64_t ia, float b, int64_t ib) {
  return a > b || (a == b && ia < ib);
}

// Top-k of `cnt` candidates per row; candidates are (score, index) pairs, or
// raw scores with index base + position when idx == nullptr.  Destructive on
// the scores (a taken candidate is overwritten with NaN; NaN scores and
// negative indices are skipped).  Rows with fewer than k candidates are
// padded with (-inf, -1).  One block per
// (slice, row); writes k results to out[(row * nslices + slice) * k].
__global__ void __launch_bounds__(256)
k_topk_select(float *score, const int64_t *idx, int64_t row_stride, int64_t cnt, int64_t slice,
              int64_t base, int k, float *out_s, int64_t *out_i, int64_t out_row_stride) {
  const int64_t row = blockIdx.y;
  const int64_t lo = (int64_t)blockIdx.x * slice;
  const int64_t hi = min(cnt, lo + slice);
  float *s = score + row * row_stride;
  const int64_t *ix = idx ? idx + row * row_stride : nullptr;
  __shared__ float ws[32];
  __shared__ int64_t wi[32], wp[32];
  for (int r = 0; r < k; ++r) {
    float bs = -INFINITY;
    int64_t bi = INT64_MAX, bp = -1;
    for (int64_t e = lo + threadIdx.x; e < hi; e += blockDim.x) {
      const float v = s[e];
      const int64_t id = ix ? ix[e] : base + e;
      if (v != v || id < 0) continue;  // taken (NaN) or empty slot
      if (bp < 0 || better(v, id, bs, bi)) {
        bs = v;
        bi = id;
        bp = e;
      }
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) {
      const float os = __shfl_xor_sync(0xffffffffu, bs, o);
      const int64_t oi = __shfl_xor_sync(0xffffffffu, bi, o);
      const int64_t op = __shfl_xor_sync(0xffffffffu, bp, o);
      if (op >= 0 && (bp < 0 || better(os, oi, bs, bi))) {
        bs = os;
        bi = oi;
        bp = op;
      }
    }
    if (threadIdx.x % 32 == 0) {
      ws[threadIdx.x / 32] = bs;
      wi[threadIdx.x / 32] = bi;
      wp[threadIdx.x / 32] = bp;
    }
    __syncthreads();
    if (threadIdx.x == 0) {
      for (int w = 1; w < (int)(blockDim.x / 32); ++w)
        if (wp[w] >= 0 && (wp[0] < 0 || better(ws[w], wi[w], ws[0], wi[0]))) {
          ws[0] = ws[w];
          wi[0] = wi[w];
          wp[0] = wp[w];
        }
      const int64_t o = (row * out_row_stride) + (int64_t)blockIdx.x * k + r;
      out_s[o] = wp[0] >= 0 ? ws[0] : -INFINITY;
      out_i[o] = wp[0] >= 0 ? wi[0] : -1;
      if (wp[0] >= 0) s[wp[0]] = __int_as_float(0x7fffffff);
    }
    __syncthreads();
  }
}

// ============================================================ outliers
__global__ void k_sumsq_partial(RowSource src, int64_t rows_per_group, int64_t chunk, double *part,
                                int nchunks) {
  const int64_t g = blockIdx.y;
  const int64_t r0 = (int64_t)blockIdx.x * chunk;
  const int64_t r1 = min(rows_per_group, r0 + chunk);
  for (int c = threadIdx.x; c < src.d; c += blockDim.x) {
    double acc = 0.0;
    for (int64_t r = r0; r < r1; ++r) {
      const double v = src.at(g * rows_per_group + r, c);
      acc += v * v;
    }
    part[(g * nchunks + blockIdx.x) * src.d + c] = acc;
  }
}

__global__ void k_sumsq_final(const double *part, int64_t groups, int nchunks, int dim, double *out) {
  const int64_t t = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
  if (t >= groups * dim) return;
  const int64_t g = t / dim;
  const int c = (int)(t % dim);
  double acc = 0.0;
  for (int k = 0; k < nchunks; ++k) acc += part[(g * nchunks + k) * dim + c];
  out[t] = acc;
}

// ============================================================ launchers
#define TQ_CHECK_LAUNCH()                                   \
  do {                                                      \
    if (cudaGetLastError() != cudaSuccess) return TQ_ERR_CUDA; \
  } while (0)

template <int D, int W>
static tq_status launch_encode_fwht_dw(const tq_quantizer *q, const RowSource &src, int64_t n,
                                       uint32_t *codes, uint32_t *signs, float2 *norms,
                                       int64_t out_stride, cudaStream_t st) {
  const size_t smem = (size_t)D * D * sizeof(float);
  auto kern = k_encode_fwht<D, W>;
  if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem) != cudaSuccess)
    return TQ_ERR_CUDA;
  kern<<<ceil_div_i(n, 128), 128, smem, st>>>(q->kt, src, n, codes, signs, norms, out_stride);
  TQ_CHECK_LAUNCH();
  return TQ_OK;
}

template <int D>
static tq_status launch_encode_fwht_d(const tq_quantizer *q, const RowSource &src, int64_t n,
                                      uint32_t *codes, uint32_t *signs, float2 *norms,
                                      int64_t out_stride, cudaStream_t st) {
  switch (q->w) {
    case 1: return launch_encode_fwht_dw<D, 1>(q, src, n, codes, signs, norms, out_stride, st);
    case 2: return launch_encode_fwht_dw<D, 2>(q, src, n, codes, signs, norms, out_stride, st);
    case 3: return launch_encode_fwht_dw<D, 3>(q, src, n, codes, signs, norms, out_stride, st);
    case 4: return launch_encode_fwht_dw<D, 4>(q, src, n, codes, signs, norms, out_stride, st);
  }
  return TQ_ERR_UNSUPPORTED;
}

tq_status v1_encode_fwht(const tq_quantizer *q, const RowSource &src, int64_t n, void *codes,
                         void *signs, float *norms, int64_t out_stride, cudaStream_t st) {
  auto c = static_cast<uint32_t *>(codes);
  auto s = static_cast<uint32_t *>(signs);
  auto nr = reinterpret_cast<float2 *>(norms);
  switch (q->d) {
    case 32: return launch_encode_fwht_d<32>(q, src, n, c, s, nr, out_stride, st);
    case 64: return launch_encode_fwht_d<64>(q, src, n, c, s, nr, out_stride, st);
    case 128: return launch_encode_fwht_d<128>(q, src, n, c, s, nr, out_stride, st);
  }
  return TQ_ERR_UNSUPPORTED;
}

size_t v1_dense_batch_rows(const tq_quantizer *q, size_t ws_bytes) {
  const size_t per_row = (size_t)q->d * 5 + (size_t)q->m + 16;
  return ws_bytes / per_row;
}

size_t v1_dense_ws_bytes(const tq_quantizer *q, int64_t n) {
  const int64_t rows = n < 65536 ? n : 65536;
  return (size_t)rows * ((size_t)q->d * 5 + (size_t)q->m + 16) + 256;
}

template <int W>
static void launch_pack(int d, int m, int64_t rows, const uint8_t *code, const uint8_t *sign,
                        const float *r, uint32_t *codes, uint32_t *signs, float2 *norms,
                        int64_t out_stride, cudaStream_t st) {
  k_pack_rows<W><<<ceil_div_i(rows, 128), 128, 0, st>>>(d, m, rows, code, sign, r, codes, signs, norms,
                                                        out_stride);
}

tq_status v1_encode_dense(const tq_quantizer *q, const RowSource &src, int64_t n, void *codes,
                          void *signs, float *norms, int64_t out_stride, void *ws, size_t ws_bytes,
                          cudaStream_t st) {
  const int d = q->d, m = q->m, w = q->w;
  const int64_t batch = (int64_t)v1_dense_batch_rows(q, ws_bytes);
  if (batch < 1) return TQ_ERR_WORKSPACE;
  auto nr2 = reinterpret_cast<float2 *>(norms);
  k_row_norms<<<ceil_div_i(n, 8), 256, 0, st>>>(src, n, nr2, out_stride);
  TQ_CHECK_LAUNCH();
  char *base = static_cast<char *>(ws);
  float *r = reinterpret_cast<float *>(base);
  uint8_t *code = reinterpret_cast<uint8_t *>(base + (size_t)batch * d * 4);
  uint8_t *sign = code + (size_t)batch * d;
  for (int64_t r0 = 0; r0 < n; r0 += batch) {
    const int64_t rows = (n - r0) < batch ? (n - r0) : batch;
    LoadRows la{src, r0};
    LoadMat lr{q->kt.rot, d};
    EpiRotQuant e1{q->kt, nr2 + r0 * out_stride, out_stride, r, code};
    dim3 g1(ceil_div_i(rows, 64), ceil_div_i(d, 64));
    k_gemm_nt<<<g1, 256, 0, st>>>(rows, d, d, la, lr, e1);
    TQ_CHECK_LAUNCH();
    LoadMat lrr{r, d};
    LoadMat ls{q->kt.qjl32, d};
    EpiSignByte e2{sign, m};
    dim3 g2(ceil_div_i(rows, 64), ceil_div_i(m, 64));
    k_gemm_nt<<<g2, 256, 0, st>>>(rows, m, d, lrr, ls, e2);
    TQ_CHECK_LAUNCH();
    uint32_t *cw = static_cast<uint32_t *>(codes) + r0 * out_stride * (w * d / 32);
    uint32_t *sw = static_cast<uint32_t *>(signs) + r0 * out_stride * (m / 32);
    switch (w) {
      case 1: launch_pack<1>(d, m, rows, code, sign, r, cw, sw, nr2 + r0 * out_stride, out_stride, st); break;
      case 2: launch_pack<2>(d, m, rows, code, sign, r, cw, sw, nr2 + r0 * out_stride, out_stride, st); break;
      case 3: launch_pack<3>(d, m, rows, code, sign, r, cw, sw, nr2 + r0 * out_stride, out_stride, st); break;
      case 4: launch_pack<4>(d, m, rows, code, sign, r, cw, sw, nr2 + r0 * out_stride, out_stride, st); break;
    }
    TQ_CHECK_LAUNCH();
  }
  return TQ_OK;
}

tq_status v1_prepare_queries(const tq_quantizer *q, const RowSource &src, int64_t nq, float *ytil,
                             float *p, cudaStream_t st) {
  const int d = q->d;
  if (q->rotation == TQ_ROT_HADAMARD && (d == 32 || d == 64 || d == 128)) {
    switch (d) {
      case 32: k_prep_fwht_block<32><<<(unsigned)nq, 32, 0, st>>>(q->kt, src, nq, ytil, p); break;
      case 64: k_prep_fwht_block<64><<<(unsigned)nq, 64, 0, st>>>(q->kt, src, nq, ytil, p); break;
      case 128: k_prep_fwht_block<128><<<(unsigned)nq, 128, 0, st>>>(q->kt, src, nq, ytil, p); break;
    }
    TQ_CHECK_LAUNCH();
    return TQ_OK;
  }
  if (d <= 128 && q->d_rott) {
    const int threads = std::max(32, (std::max(d, q->m) + 31) / 32 * 32);
    k_prep_dense_block<<<(unsigned)nq, std::min(threads, 1024), 0, st>>>(q->kt, src, nq, ytil, p);
    TQ_CHECK_LAUNCH();
    return TQ_OK;
  }
  LoadRows la{src, 0};
  LoadMat lr{q->kt.rot, d};
  EpiStore e1{ytil, d};
  k_gemm_nt<<<dim3(ceil_div_i(nq, 64), ceil_div_i(d, 64)), 256, 0, st>>>(nq, d, d, la, lr, e1);
  TQ_CHECK_LAUNCH();
  if (q->m == 0) return TQ_OK;  // TurboQuant-MSE: no QJL projection of the query
  LoadMat ly{ytil, d};
  LoadMat ls{q->kt.qjl32, d};
  EpiStore e2{p, q->m};
  k_gemm_nt<<<dim3(ceil_div_i(nq, 64), ceil_div_i(q->m, 64)), 256, 0, st>>>(nq, q->m, d, ly, ls, e2);
  TQ_CHECK_LAUNCH();
  return TQ_OK;
}

tq_status v1_score(const tq_quantizer *q, const float *ytil, const float *p, int64_t nq_rows, int64_t G,
                   int64_t keys_per_group, int64_t key_base, int64_t nkeys, const void *codes,
                   const void *signs, const float *norms, float *out, int64_t ldo, int accumulate,
                   cudaStream_t st) {
  if (nkeys <= 0 || nq_rows <= 0) return TQ_OK;
  const size_t smem = (size_t)(q->d + q->m) * sizeof(float);
  dim3 grid(ceil_div_i(nkeys, 128), (unsigned)nq_rows);
  auto c = static_cast<const uint32_t *>(codes);
  auto s = static_cast<const uint32_t *>(signs);
  auto nr = reinterpret_cast<const float2 *>(norms);
#define TQ_SCORE_CASE(WW)                                                                          \
  case WW: {                                                                                       \
    if (cudaFuncSetAttribute(k_score_rows<WW>, cudaFuncAttributeMaxDynamicSharedMemorySize,        \
                             (int)smem) != cudaSuccess)                                            \
      return TQ_ERR_CUDA;                                                                          \
    k_score_rows<WW><<<grid, 128, smem, st>>>(q->kt, ytil, p, G, keys_per_group, key_base, nkeys, \
                                              c, s, nr, out, ldo, accumulate);                    \
    break;                                                                                         \
  }
  switch (q->w) {
    TQ_SCORE_CASE(1)
    TQ_SCORE_CASE(2)
    TQ_SCORE_CASE(3)
    TQ_SCORE_CASE(4)
    default: return TQ_ERR_UNSUPPORTED;
  }
#undef TQ_SCORE_CASE
  TQ_CHECK_LAUNCH();
  return TQ_OK;
}

tq_status v1_topk_select(float *score, const int64_t *idx, int64_t rows, int64_t row_stride, int64_t cnt,
                         int64_t slice, int64_t base, int k, float *out_s, int64_t *out_i,
                         int64_t out_row_stride, cudaStream_t st) {
  dim3 grid(ceil_div_i(cnt, slice), (unsigned)rows);
  k_topk_select<<<grid, 256, 0, st>>>(score, idx, row_stride, cnt, slice, base, k, out_s, out_i,
                                      out_row_stride);
  TQ_CHECK_LAUNCH();
  return TQ_OK;
}

tq_status v1_sumsq(const RowSource &src, int64_t groups, int64_t rows_per_group, double *part, int nchunks,
                   double *out, cudaStream_t st) {
  const int64_t chunk = (rows_per_group + nchunks - 1) / nchunks;
  k_sumsq_partial<<<dim3(nchunks, (unsigned)groups), 128, 0, st>>>(src, rows_per_group, chunk, part, nchunks);
  TQ_CHECK_LAUNCH();
  const int64_t tot = groups * src.d;
  k_sumsq_final<<<ceil_div_i(tot, 256), 256, 0, st>>>(part, groups, nchunks, src.d, out);
  TQ_CHECK_LAUNCH();
  return TQ_OK;
}

}  // namespace tq

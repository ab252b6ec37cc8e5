// Tensor-core encode for a dense rotation: the Haar rotation of any d (the
// TurboQuant article, 2.1.2: a seeded random orthogonal matrix; 3.3 uses
// d = 1536) and the Hadamard rotation at d above 128, for d a multiple of 64
// from 256 up.
//
// Both projections run as integer GEMMs on 31-bit fixed point: every operand
// row (or matrix) is scaled by a power of two so that |v| 2^e < 2^30, rounded,
// and split into four signed bytes, v 2^e = 2^24 a + 2^16 b + 2^8 c + d.  Ten
// kind::i8 MMA passes accumulate the limb products of weight 2^48 down to 2^24
// exactly in int32, grouped by weight into four TMEM accumulators (a a';
// a b' + b a'; a c' + b b' + c a'; a d' + b c' + c b' + d a'), and the epilogue
// joins them in int64.  The errors are the 2^-31 rounding of the operands and
// the dropped products of weight 2^16 and below (near 1e-9 in u at d = 1536).
// Coarser splits do not do: at 23 bits, relative to the row's largest entry,
// the rounding of x moves u by ~3e-8 and z = S r, a sum of d such terms, by
// ~1e-6; and fp32 accumulation of fp16 pieces on the tensor cores, whose adds
// truncate, leaves ~1e-5 relative error in u after K = 1536.  Per batch of rows:
//
//   1. k_dense_split   ||x||, the row's exponent and x as limbs; the factor
//                      that turns the integer product into u = R x / ||x||.
//   2. k_dense_gemm<0> U = X R^T.  Epilogue: u, the code (count of thresholds
//                      below u, the TurboQuant article 1.2.2), the residual
//                      r = u - c[code] (2.3.1) in fp32, its square sum and
//                      the row's largest |r|.
//   3. k_dense_rlimbs  r as limbs under the row's own exponent.
//   4. k_dense_gemm<1> Z = r S^T.  Epilogue: the QJL sign bits [z >= 0]
//                      (2.3.2), decided on the exact integer sum.
//   5. k_dense_gamma   gamma = sqrt(sum r^2).
//
// The GEMM is persistent over 128 x 128 output tiles: warp 0 streams 64-byte
// K chunks of the four limb planes of both operands by TMA into a ring of
// stages, warp 1 issues the MMAs (one thread), warps 2-5 run the epilogue.
#include <cudaTypedefs.h>

#include "tq_common.cuh"
#include "tq_kernels.h"
#include "tq_sm100.cuh"

namespace tq {

namespace {

constexpr int kGBM = 128, kGBN = 128, kGBK = 64;  // tile rows, tile columns, K chunk (bytes = elements)
constexpr int kGThreads = 192;
constexpr int kLimbs = 4;
constexpr uint32_t kPlaneA = kGBM * kGBK, kPlaneB = kGBN * kGBK;  // bytes of one limb plane per stage
constexpr uint32_t kStageBytes = kLimbs * (kPlaneA + kPlaneB);
constexpr int kPasses = 10;
// limb pass -> (A plane, B plane, accumulator): weights 2^48, 2^40, 2^32, 2^24
__constant__ int8_t c_pass[kPasses][3] = {{0, 0, 0}, {0, 1, 1}, {1, 0, 1}, {0, 2, 2}, {1, 1, 2},
                                          {2, 0, 2}, {0, 3, 3}, {1, 2, 3}, {2, 1, 3}, {3, 0, 3}};

struct DenseGemmParams {
  int M, N, K;  // output rows, output columns, reduction length
  int nstages;
  int *err;
  // epilogue
  KernelTables kt;
  const float *row_scale;  // [M] rotation: u = (integer product) * row_scale
  float *gam2;             // [M] rotation: sum of r^2 (accumulated)
  unsigned *rmax;          // [M] rotation: largest |r| of the row (float bits)
  float *r;                // [M][N] rotation: residual
  uint32_t *codes, *signs;
  int64_t out_stride;  // output row of batch row i: i * out_stride (pointers already at the batch)
};

// Split v (|v| 2^e < 2^30) into its four limbs (a, b, c, d).
// 2^e as a product of two floats (each a power of two inside the normal
// range for |e| <= 252): v * s.x * s.y is v 2^e exactly, as ldexpf gives it,
// whenever the result is a normal number.
__device__ __forceinline__ float2 pow2_pair(int e) {
  const int e1 = e / 2, e2 = e - e1;
  return make_float2(__uint_as_float((uint32_t)(127 + e1) << 23), __uint_as_float((uint32_t)(127 + e2) << 23));
}

// Four signed bytes of round(v 2^e), |v 2^e| < 2^30: 2^24 a + 2^16 b + 2^8 c + d.
__device__ __forceinline__ uint32_t limb_bytes(float v, float2 s) {
  int t = __float2int_rn(v * s.x * s.y);
  uint32_t out = 0u;
#pragma unroll
  for (int k = 3; k >= 1; --k) {
    const int lo = ((t + 128) & 255) - 128;
    out |= (uint32_t)(uint8_t)lo << (8 * k);
    t = (t - lo) >> 8;
  }
  return out | (uint32_t)(uint8_t)t;  // byte k = limb plane k (plane 0: the top limb)
}

__device__ __forceinline__ void limbs_of(float v, int e, int8_t (&l)[4]) {
  int t = __float2int_rn(ldexpf(v, e));
#pragma unroll
  for (int k = 3; k >= 1; --k) {
    const int lo = ((t + 128) & 255) - 128;
    l[k] = (int8_t)lo;
    t = (t - lo) >> 8;  // exact: t - lo is a multiple of 256
  }
  l[0] = (int8_t)t;
}

template <int EPI, int W>
__global__ void __launch_bounds__(kGThreads, 1)
k_dense_gemm(const __grid_constant__ CUtensorMap ma, const __grid_constant__ CUtensorMap mb, int a_plane_rows,
             int b_plane_rows, const DenseGemmParams p) {
  constexpr int L = 1 << W;
  extern __shared__ uint8_t smem_raw[];
  uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const int S = p.nstages;
  uint64_t *bars = reinterpret_cast<uint64_t *>(smem + S * kStageBytes);
  uint64_t *full = bars, *empty = bars + S, *accf = bars + 2 * S, *acce = bars + 2 * S + 1, *done = bars + 2 * S + 2;
  uint32_t *sTmem = reinterpret_cast<uint32_t *>(bars + 2 * S + 3);
  volatile int *sAbort = reinterpret_cast<volatile int *>(sTmem + 1);
  const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
  const int ntm = (p.M + kGBM - 1) / kGBM, ntn = (p.N + kGBN - 1) / kGBN;
  const int nitems = ntm * ntn, nk = (p.K + kGBK - 1) / kGBK;

  if (threadIdx.x == 0) {
    for (int i = 0; i < S; ++i) {
      sm100::mbar_init(&full[i], 1);
      sm100::mbar_init(&empty[i], 1);
    }
    sm100::mbar_init(accf, 1);
    sm100::mbar_init(acce, 4);
    sm100::mbar_init(done, 1);
    *sAbort = 0;
    sm100::fence_barrier_init();
    sm100::prefetch_tmap(&ma);
    sm100::prefetch_tmap(&mb);
  }
  if (warp == 1) {
    sm100::tmem_alloc(sTmem, 512);  // four accumulators of kGBN columns
    sm100::tmem_relinquish();
  }
  sm100::tc_fence_before();
  __syncthreads();
  sm100::tc_fence_after();
  const uint32_t tmem = *sTmem;
  auto wait = [&](uint64_t *bar, uint32_t parity, int code) {
    return sm100::mbar_wait_abort(bar, parity, sAbort, p.err, code);
  };
  int64_t loads = 0;     // K chunks whose copies were issued (warp 0)
  bool any_mma = false;  // warp 1 issued at least one MMA

  if (warp == 0) {
    // ------------------------------------------------------------ copies
    if (lane == 0) {
      int64_t c = 0;
      bool ok = true;
      for (int w = blockIdx.x; w < nitems && ok; w += gridDim.x) {
        const int m0 = (w / ntn) * kGBM, n0 = (w % ntn) * kGBN;
        for (int kc = 0; kc < nk; ++kc, ++c) {
          const int slot = (int)(c % S);
          const int64_t use = c / S;
          if (use > 0 && !wait(&empty[slot], (uint32_t)((use - 1) & 1), 41)) {
            ok = false;
            break;
          }
          uint8_t *st = smem + slot * kStageBytes;
          sm100::mbar_expect_tx(&full[slot], kStageBytes);
          // plane l of an operand is rows [l * plane_rows, (l + 1) * plane_rows) of its map;
          // rows past an operand's end read the next plane and only reach
          // outputs that are not stored
#pragma unroll
          for (int l = 0; l < kLimbs; ++l) {
            sm100::tma_load_2d(st + l * kPlaneA, &ma, kc * kGBK, l * a_plane_rows + m0, &full[slot]);
            sm100::tma_load_2d(st + kLimbs * kPlaneA + l * kPlaneB, &mb, kc * kGBK, l * b_plane_rows + n0,
                               &full[slot]);
          }
          loads = c + 1;
        }
      }
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issue
    if (lane == 0) {
      const uint32_t idesc = sm100::idesc_s8_s32(kGBM, kGBN);
      int64_t c = 0;
      int item = 0;
      bool ok = true;
      for (int w = blockIdx.x; w < nitems && ok; w += gridDim.x, ++item) {
        if (item > 0 && !wait(acce, (uint32_t)((item - 1) & 1), 42)) break;
        sm100::tc_fence_after();
        for (int kc = 0; kc < nk; ++kc, ++c) {
          const int slot = (int)(c % S);
          if (!wait(&full[slot], (uint32_t)((c / S) & 1), 43)) {
            ok = false;
            break;
          }
          sm100::tc_fence_after();
          const uint32_t sa = sm100::smem_u32(smem + slot * kStageBytes);
          const uint32_t sb = sa + kLimbs * kPlaneA;
#pragma unroll
          for (int ps = 0; ps < kPasses; ++ps) {
            const int pa = c_pass[ps][0], pb = c_pass[ps][1], g = c_pass[ps][2];
            const bool first = ps == 0 || ps == 1 || ps == 3 || ps == 6;  // first pass into its accumulator
#pragma unroll
            for (int ks = 0; ks < kGBK / 32; ++ks) {
              const uint64_t da = sm100::desc_sw64(sa + pa * kPlaneA + ks * 32);
              const uint64_t db = sm100::desc_sw64(sb + pb * kPlaneB + ks * 32);
              sm100::mma_i8(tmem + (uint32_t)(g * kGBN), da, db, idesc, !(kc == 0 && first && ks == 0));
            }
          }
          any_mma = true;
          sm100::mma_commit(&empty[slot]);  // the stage is free once these MMAs are done
        }
        if (!ok) break;
        sm100::mma_commit(accf);
      }
    }
  } else {
    // ------------------------------------------------------------ epilogue
    const int quarter = warp % 4, rin = 32 * quarter + lane;
    const uint32_t tlane = (uint32_t)(32 * quarter) << 16;
    int item = 0;
    for (int w = blockIdx.x; w < nitems; w += gridDim.x, ++item) {
      const int m0 = (w / ntn) * kGBM, n0 = (w % ntn) * kGBN;
      const int gr = m0 + rin;
      const bool valid = gr < p.M;
      float rsc = 0.f;
      if (EPI == 0 && valid) rsc = p.row_scale[gr];
      if (!__all_sync(0xffffffffu, wait(accf, (uint32_t)(item & 1), 44))) break;
      sm100::tc_fence_after();
      float gsum = 0.f, rbig = 0.f;
      for (int cc = 0; cc < kGBN / 32; ++cc) {
        const int col0 = n0 + 32 * cc;
        if (col0 >= p.N) break;  // warp-uniform
        uint32_t cw[W];
#pragma unroll
        for (int k = 0; k < W; ++k) cw[k] = 0u;
        uint32_t wbits = 0u;
#pragma unroll
        for (int hf = 0; hf < 2; ++hf) {  // 16 columns at a time
          uint32_t g[4][16];
#pragma unroll
          for (int a = 0; a < 4; ++a) sm100::tmem_ld16(tmem + tlane + (uint32_t)(a * kGBN + 32 * cc + 16 * hf), g[a]);
          sm100::tmem_wait_ld();
          if (!valid) continue;
          float rr[16];
#pragma unroll
          for (int jj = 0; jj < 16; ++jj) {
            // the product in units of 2^24
            const long long P = (long long)(int)g[0][jj] * 16777216LL + (long long)(int)g[1][jj] * 65536LL +
                                (long long)(int)g[2][jj] * 256LL + (long long)(int)g[3][jj];
            if constexpr (EPI == 0) {
              const float u = __ll2float_rn(P) * rsc;
              int c = 0;
#pragma unroll
              for (int t = 0; t < L - 1; ++t) c += u > p.kt.thresholds[t] ? 1 : 0;
              const float r = u - p.kt.centroids[c];
              gsum = fmaf(r, r, gsum);
              rbig = fmaxf(rbig, fabsf(r));
              pack_code<W>(cw, 16 * hf + jj, (uint32_t)c);
              rr[jj] = r;
            } else {
              wbits |= (P >= 0 ? 1u : 0u) << (16 * hf + jj);
            }
          }
          if constexpr (EPI == 0) {
            float4 *pr = reinterpret_cast<float4 *>(p.r + (int64_t)gr * p.N + col0 + 16 * hf);
#pragma unroll
            for (int k = 0; k < 4; ++k) pr[k] = make_float4(rr[4 * k], rr[4 * k + 1], rr[4 * k + 2], rr[4 * k + 3]);
          }
        }
        if (!valid) continue;
        if constexpr (EPI == 0) {
          uint32_t *dst = p.codes + (int64_t)gr * p.out_stride * (W * p.N / 32) + (col0 / 32) * W;
#pragma unroll
          for (int k = 0; k < W; ++k) dst[k] = cw[k];
        } else {
          p.signs[(int64_t)gr * p.out_stride * (p.N / 32) + col0 / 32] = wbits;
        }
      }
      if (EPI == 0 && valid) {
        atomicAdd(p.gam2 + gr, gsum);
        atomicMax(p.rmax + gr, __float_as_uint(rbig));  // non-negative floats order as their bits
      }
      sm100::tc_fence_before();
      __syncwarp();
      if (lane == 0) sm100::mbar_arrive(acce);
    }
  }
  // ------------------------------------------------------------ teardown
  __syncthreads();
  if (warp == 1 && lane == 0 && any_mma) {  // no MMA may still write TMEM when it is freed
    sm100::mma_commit(done);
    sm100::mbar_wait(done, 0u, p.err, 45);
  }
  if (warp == 0 && lane == 0 && *sAbort) {  // copies issued but possibly not consumed
    for (int64_t c = loads > S ? loads - S : 0; c < loads; ++c)
      sm100::mbar_wait(&full[c % S], (uint32_t)((c / S) & 1), p.err, 46);
  }
  sm100::tc_fence_before();
  __syncthreads();
  sm100::tc_fence_after();
  if (warp == 1) sm100::tmem_dealloc(tmem, 512);
}

// One warp per row: ||x||, the row's limb exponent, the factor back to u, and
// x as limbs (planes of `plane_rows` rows).
__global__ void k_dense_split(RowSource src, int64_t row0, int64_t rows, int64_t plane_rows, int rot_exp,
                              int8_t *xl, float *row_scale, float *gam2, unsigned *rmax, float2 *norms,
                              int64_t out_stride) {
  const int64_t row = (int64_t)blockIdx.x * (blockDim.x / 32) + threadIdx.x / 32;
  const int lane = threadIdx.x % 32;
  if (row >= rows) return;
  const int d = src.d;
  float ss = 0.f, big = 0.f;
  for (int j = lane; j < d; j += 32) {
    const float v = src.at(row0 + row, j);
    ss = fmaf(v, v, ss);
    big = fmaxf(big, fabsf(v));
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) {
    ss += __shfl_xor_sync(0xffffffffu, ss, o);
    big = fmaxf(big, __shfl_xor_sync(0xffffffffu, big, o));
  }
  const float nrm = sqrtf(ss);
  int E = 0;
  frexpf(big, &E);  // big < 2^E
  const int e = big > 0.f ? 30 - E : 0;
  const int64_t plane = plane_rows * d;
  if (!src.chan && !src.bf16 && d % 128 == 0) {
    // four consecutive values per lane: one 16-byte load, one 4-byte store per limb plane
    const float2 sc = pow2_pair(e);
    const float *xr = static_cast<const float *>(src.x) + (row0 + row) * src.ldx;
    for (int j = 4 * lane; j < d; j += 128) {
      const float4 v = *reinterpret_cast<const float4 *>(xr + j);
      const uint32_t b0 = limb_bytes(v.x, sc), b1 = limb_bytes(v.y, sc), b2 = limb_bytes(v.z, sc),
                     b3 = limb_bytes(v.w, sc);
#pragma unroll
      for (int k = 0; k < 4; ++k)
        *reinterpret_cast<uint32_t *>(xl + k * plane + row * d + j) =
            __byte_perm(__byte_perm(b0, b1, 0x40 + 0x11 * k), __byte_perm(b2, b3, 0x40 + 0x11 * k), 0x5410);
    }
  } else {
    for (int j = lane; j < d; j += 32) {
      int8_t l[4];
      limbs_of(src.at(row0 + row, j), e, l);
#pragma unroll
      for (int k = 0; k < 4; ++k) xl[k * plane + row * d + j] = l[k];
    }
  }
  if (lane == 0) {
    // the epilogue's integer sum counts units of 2^24
    row_scale[row] = nrm > 0.f ? ldexpf(1.0f, 24 - (e + rot_exp)) / nrm : 0.f;
    gam2[row] = 0.f;
    rmax[row] = 0u;
    norms[row * out_stride] = make_float2(nrm, 0.f);
  }
}

// One warp per row: r as limbs under the row's own exponent.
__global__ void k_dense_rlimbs(const float *r, const unsigned *rmax, int d, int64_t rows, int64_t plane_rows,
                               int8_t *rl) {
  const int64_t row = (int64_t)blockIdx.x * (blockDim.x / 32) + threadIdx.x / 32;
  const int lane = threadIdx.x % 32;
  if (row >= rows) return;
  const float big = __uint_as_float(rmax[row]);
  int E = 0;
  frexpf(big, &E);
  const int e = big > 0.f ? 30 - E : 0;
  const int64_t plane = plane_rows * d;
  if (d % 128 == 0) {
    const float2 sc = pow2_pair(e);
    for (int j = 4 * lane; j < d; j += 128) {
      const float4 v = *reinterpret_cast<const float4 *>(r + row * d + j);
      const uint32_t b0 = limb_bytes(v.x, sc), b1 = limb_bytes(v.y, sc), b2 = limb_bytes(v.z, sc),
                     b3 = limb_bytes(v.w, sc);
#pragma unroll
      for (int k = 0; k < 4; ++k)
        *reinterpret_cast<uint32_t *>(rl + k * plane + row * d + j) =
            __byte_perm(__byte_perm(b0, b1, 0x40 + 0x11 * k), __byte_perm(b2, b3, 0x40 + 0x11 * k), 0x5410);
    }
    return;
  }
  for (int j = lane; j < d; j += 32) {
    int8_t l[4];
    limbs_of(r[row * d + j], e, l);
#pragma unroll
    for (int k = 0; k < 4; ++k) rl[k * plane + row * d + j] = l[k];
  }
}

__global__ void k_dense_gamma(const float *gam2, int64_t rows, float2 *norms, int64_t out_stride) {
  const int64_t row = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
  if (row < rows) norms[row * out_stride].y = sqrtf(gam2[row]);
}

struct DenseLayout {
  size_t limbs, r, scale, gam2, rmax, per_batch;
};
DenseLayout dense_layout(int d, int64_t rows) {
  auto up = [](size_t v) { return (v + 255) / 256 * 256; };
  DenseLayout L{};
  L.limbs = 0;  // x limbs, later r limbs: [4][rows][d]
  L.r = up(4 * (size_t)rows * d);
  L.scale = L.r + up((size_t)rows * d * 4);
  L.gam2 = L.scale + up((size_t)rows * 4);
  L.rmax = L.gam2 + up((size_t)rows * 4);
  L.per_batch = L.rmax + up((size_t)rows * 4);
  return L;
}

// 2-D map over `rows` rows of `cols` int8 (four limb planes stacked as rows)
bool make_map(CUtensorMap *map, const void *base, int64_t cols, int64_t rows, uint32_t box_rows) {
  auto enc = tensor_map_encoder();
  if (!enc) return false;
  cuuint64_t gdim[2] = {(cuuint64_t)cols, (cuuint64_t)rows};
  cuuint64_t gstride[1] = {(cuuint64_t)cols};
  cuuint32_t box[2] = {(cuuint32_t)kGBK, box_rows};
  cuuint32_t estr[2] = {1, 1};
  return enc(map, CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, const_cast<void *>(base), gdim, gstride, box, estr,
             CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_64B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
             CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

template <int EPI, int W>
tq_status launch_gemm(const CUtensorMap &ma, const CUtensorMap &mb, int a_plane_rows, int b_plane_rows,
                      DenseGemmParams prm, cudaStream_t st) {
  int dev = 0, sms = 0, max_smem = 0;
  cudaGetDevice(&dev);
  cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  cudaDeviceGetAttribute(&max_smem, cudaDevAttrMaxSharedMemoryPerBlockOptin, dev);
  const int extra = 1024 + 8 * 16 + 16;
  prm.nstages = std::min(4, (int)((max_smem - extra) / kStageBytes));
  if (prm.nstages < 2) return TQ_ERR_UNSUPPORTED;
  const size_t smem = (size_t)prm.nstages * kStageBytes + extra;
  const int nitems = ((prm.M + kGBM - 1) / kGBM) * ((prm.N + kGBN - 1) / kGBN);
  auto kern = k_dense_gemm<EPI, W>;
  if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem) != cudaSuccess)
    return TQ_ERR_CUDA;
  kern<<<std::min(nitems, sms), kGThreads, smem, st>>>(ma, mb, a_plane_rows, b_plane_rows, prm);
  return cudaGetLastError() == cudaSuccess ? TQ_OK : TQ_ERR_CUDA;
}

template <int W>
tq_status dense_batch(const tq_quantizer *q, const RowSource &src, int64_t r0, int64_t rows, int64_t cap,
                      char *ws, const DenseLayout &L, uint32_t *codes, uint32_t *signs, float2 *norms,
                      int64_t out_stride, cudaStream_t st) {
  const int d = q->d, m = q->m;
  int8_t *limbs = reinterpret_cast<int8_t *>(ws + L.limbs);
  float *r = reinterpret_cast<float *>(ws + L.r);
  float *scale = reinterpret_cast<float *>(ws + L.scale), *gam2 = reinterpret_cast<float *>(ws + L.gam2);
  unsigned *rmax = reinterpret_cast<unsigned *>(ws + L.rmax);
  k_dense_split<<<(unsigned)((rows + 7) / 8), 256, 0, st>>>(src, r0, rows, cap, q->rot_limb_exp, limbs, scale,
                                                            gam2, rmax, norms, out_stride);
  if (cudaGetLastError() != cudaSuccess) return TQ_ERR_CUDA;
  CUtensorMap ma, mb;
  if (!make_map(&ma, limbs, d, kLimbs * cap, kGBM) || !make_map(&mb, q->d_rot_limbs, d, kLimbs * (int64_t)d, kGBN))
    return TQ_ERR_CUDA;
  DenseGemmParams prm{};
  prm.M = (int)rows;
  prm.N = d;
  prm.K = d;
  prm.err = q->d_err;
  prm.kt = q->kt;
  prm.row_scale = scale;
  prm.gam2 = gam2;
  prm.rmax = rmax;
  prm.r = r;
  prm.codes = codes;
  prm.out_stride = out_stride;
  tq_status s = launch_gemm<0, W>(ma, mb, (int)cap, d, prm, st);
  if (s != TQ_OK) return s;
  k_dense_rlimbs<<<(unsigned)((rows + 7) / 8), 256, 0, st>>>(r, rmax, d, rows, cap, limbs);
  if (cudaGetLastError() != cudaSuccess) return TQ_ERR_CUDA;
  CUtensorMap mb2;
  if (!make_map(&mb2, q->d_qjl_limbs, d, kLimbs * (int64_t)m, kGBN)) return TQ_ERR_CUDA;
  DenseGemmParams p2{};
  p2.M = (int)rows;
  p2.N = m;
  p2.K = d;
  p2.err = q->d_err;
  p2.kt = q->kt;
  p2.signs = signs;
  p2.out_stride = out_stride;
  s = launch_gemm<1, W>(ma, mb2, (int)cap, m, p2, st);
  if (s != TQ_OK) return s;
  k_dense_gamma<<<(unsigned)((rows + 255) / 256), 256, 0, st>>>(gam2, rows, norms, out_stride);
  return cudaGetLastError() == cudaSuccess ? TQ_OK : TQ_ERR_CUDA;
}

}  // namespace

bool dense_tc_supported(const tq_quantizer *q) {
  return q->d >= 256 && q->d % 64 == 0 && q->m >= 128 && q->m % 64 == 0 && q->d_rot_limbs && q->d_qjl_limbs &&
         q->w >= 1 && q->w <= 4;
}

// Batches of up to 32768 rows: limbs (4 bytes) and r (4 bytes) per coordinate.
size_t dense_tc_ws_bytes(const tq_quantizer *q, int64_t n) {
  const int64_t rows = std::min<int64_t>((n + kGBM - 1) / kGBM * kGBM, 32768);
  return dense_layout(q->d, rows).per_batch;
}

tq_status dense_tc_encode(const tq_quantizer *q, const RowSource &src, int64_t n, void *codes, void *signs,
                          float *norms, int64_t out_stride, void *ws, size_t ws_bytes, cudaStream_t st) {
  // the largest batch (a multiple of 128 rows) whose buffers fit the workspace
  int64_t cap = (int64_t)(ws_bytes / ((size_t)q->d * 8 + 12)) / kGBM * kGBM;
  cap = std::min<int64_t>(cap, (n + kGBM - 1) / kGBM * kGBM);
  while (cap > 0 && dense_layout(q->d, cap).per_batch > ws_bytes) cap -= kGBM;
  if (cap <= 0) return TQ_ERR_WORKSPACE;
  const DenseLayout L = dense_layout(q->d, cap);
  char *base = static_cast<char *>(ws);
  auto nr2 = reinterpret_cast<float2 *>(norms);
  for (int64_t r0 = 0; r0 < n; r0 += cap) {
    const int64_t rows = std::min(cap, n - r0);
    uint32_t *cw = static_cast<uint32_t *>(codes) + r0 * out_stride * (q->w * q->d / 32);
    uint32_t *sw = static_cast<uint32_t *>(signs) + r0 * out_stride * (q->m / 32);
    float2 *nw = nr2 + r0 * out_stride;
    tq_status s = TQ_ERR_UNSUPPORTED;
    switch (q->w) {
      case 1: s = dense_batch<1>(q, src, r0, rows, cap, base, L, cw, sw, nw, out_stride, st); break;
      case 2: s = dense_batch<2>(q, src, r0, rows, cap, base, L, cw, sw, nw, out_stride, st); break;
      case 3: s = dense_batch<3>(q, src, r0, rows, cap, base, L, cw, sw, nw, out_stride, st); break;
      case 4: s = dense_batch<4>(q, src, r0, rows, cap, base, L, cw, sw, nw, out_stride, st); break;
    }
    if (s != TQ_OK) return s;
  }
  return TQ_OK;
}

}  // namespace tq

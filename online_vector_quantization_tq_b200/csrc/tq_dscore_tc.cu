// Scoring for quantizers of d > 128 (the ANN setting of the TurboQuant
// article, 3.3, with many queries per key) as a tensor-core GEMM on fp16
// operands:
//
//   s(y, x) = ||x|| ( <y~, c[codes]> + gamma sqrt(pi/2)/m <p, 2 bits - 1> )
//           = ||x|| < [y~ | y~ | kappa p], [c_hi | c_lo | gamma (2 bits - 1)] >
//   with kappa = sqrt(pi/2)/m and c[codes] = c_hi + c_lo as two fp16 pieces.
//
//   k_dscore_queries  each query row [y~ | y~ | kappa p] scaled by a power of
//                     two (largest entry below 2^14) as two fp16 pieces hi + lo;
//   k_dscore_keys     a chunk of keys decoded to one fp16 row each;
//   k_dscore_gemm     queries x keys: the high query piece against the whole
//                     row, the low piece against all but c_lo (that product is
//                     below 2^-22 of the score), fp32 accumulation in TMEM;
//                     the epilogue scales by 2^-s and ||x|| and writes the
//                     logits.
//
// The centroids need the second piece: a single fp16 rounding of the table
// is the same error for every coordinate holding that code, so it does not
// average out over the dot product and reached 1.3e-3 of the score floor
// ||x|| ||y|| / sqrt(d) in tests.  gamma in fp16 errs by at most 2^-12 of the
// QJL term.  Persistent CTAs walk
// 128-query x 256-key tiles with the queries of one key tile on consecutive
// CTAs, so a key tile is read from HBM once and from L2 after that.
#include <cudaTypedefs.h>

#include "tq_common.cuh"
#include "tq_kernels.h"
#include "tq_sm100.cuh"

namespace tq {

namespace {

constexpr int kSBM = 128, kSBN = 256, kSBK = 64;  // queries, keys, K chunk (fp16: 128 bytes)
constexpr int kSThreads = 192;
constexpr uint32_t kSABytes = kSBM * kSBK * 2, kSBBytes = kSBN * kSBK * 2;
constexpr uint32_t kSStage = 2 * kSABytes + kSBBytes;  // query hi, query lo, keys
constexpr int64_t kKeyChunk = 32768;

constexpr int kTopSlots = 16;  // candidates kept per query row and CTA in top-k mode

struct DScoreParams {
  int M, N, K;  // queries, keys, reduction (2d + m)
  int d;
  int nstages;
  int *err;
  const float *qscale;  // [M] 2^-s of each query row
  const float2 *norms;  // [N] the keys' (||x||, gamma)
  float *out;           // [M][ldo]
  int64_t ldo;
  int accumulate;
  // top-k mode (topk != 0): no logits are written.  CTA b owns query tile
  // b % ntq and key tiles b / ntq, b / ntq + P, ...; each query row keeps
  // its kTopSlots best (score, key) pairs and writes them to
  // part_s / part_i [M][part_ld] at column part_base + (b / ntq) * kTopSlots.
  int topk, P;
  int64_t key_base;     // index of this chunk's first key
  float *part_s;
  int64_t *part_i;
  int64_t part_ld, part_base;
};

__global__ void __launch_bounds__(kSThreads, 1)
k_dscore_gemm(const __grid_constant__ CUtensorMap mqh, const __grid_constant__ CUtensorMap mql,
              const __grid_constant__ CUtensorMap mk, const DScoreParams p) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const int S = p.nstages;
  uint64_t *bars = reinterpret_cast<uint64_t *>(smem + S * kSStage);
  uint64_t *full = bars, *empty = bars + S, *accf = bars + 2 * S, *acce = bars + 2 * S + 2, *done = bars + 2 * S + 4;
  uint32_t *sTmem = reinterpret_cast<uint32_t *>(bars + 2 * S + 5);
  volatile int *sAbort = reinterpret_cast<volatile int *>(sTmem + 1);
  const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
  const int ntq = (p.M + kSBM - 1) / kSBM, ntk = (p.N + kSBN - 1) / kSBN;
  const int nitems = ntq * ntk, nk = (p.K + kSBK - 1) / kSBK;
  // i-th work item of this CTA as (query tile start, key tile start); false when done
  auto item_at = [&](int i, int &q0, int &k0) {
    if (p.topk) {
      const int kt = (int)blockIdx.x / ntq + i * p.P;
      if ((int)blockIdx.x >= ntq * p.P || kt >= ntk) return false;
      q0 = ((int)blockIdx.x % ntq) * kSBM;
      k0 = kt * kSBN;
      return true;
    }
    const int w = (int)blockIdx.x + i * (int)gridDim.x;
    if (w >= nitems) return false;
    q0 = (w % ntq) * kSBM;
    k0 = (w / ntq) * kSBN;
    return true;
  };
  const int lo_skip0 = p.d / kSBK, lo_skip1 = 2 * p.d / kSBK;  // K chunks of c_lo

  if (threadIdx.x == 0) {
    for (int i = 0; i < S; ++i) {
      sm100::mbar_init(&full[i], 1);
      sm100::mbar_init(&empty[i], 1);
    }
    for (int i = 0; i < 2; ++i) {
      sm100::mbar_init(&accf[i], 1);
      sm100::mbar_init(&acce[i], 4);
    }
    sm100::mbar_init(done, 1);
    *sAbort = 0;
    sm100::fence_barrier_init();
    sm100::prefetch_tmap(&mqh);
    sm100::prefetch_tmap(&mk);
  }
  if (warp == 1) {
    sm100::tmem_alloc(sTmem, 2 * kSBN);
    sm100::tmem_relinquish();
  }
  sm100::tc_fence_before();
  __syncthreads();
  sm100::tc_fence_after();
  const uint32_t tmem = *sTmem;
  auto wait = [&](uint64_t *bar, uint32_t parity, int code) {
    return sm100::mbar_wait_abort(bar, parity, sAbort, p.err, code);
  };
  int64_t loads = 0;
  bool any_mma = false;

  if (warp == 0) {
    // ------------------------------------------------------------ copies
    if (lane == 0) {
      int64_t c = 0;
      bool ok = true;
      int q0 = 0, k0 = 0;
      for (int i = 0; ok && item_at(i, q0, k0); ++i) {
        for (int kc = 0; kc < nk; ++kc, ++c) {
          const int slot = (int)(c % S);
          const int64_t use = c / S;
          if (use > 0 && !wait(&empty[slot], (uint32_t)((use - 1) & 1), 51)) {
            ok = false;
            break;
          }
          uint8_t *st = smem + slot * kSStage;
          sm100::mbar_expect_tx(&full[slot], kSStage);
          sm100::tma_load_2d(st, &mqh, kc * kSBK, q0, &full[slot]);
          sm100::tma_load_2d(st + kSABytes, &mql, kc * kSBK, q0, &full[slot]);
          sm100::tma_load_2d(st + 2 * kSABytes, &mk, kc * kSBK, k0, &full[slot]);
          loads = c + 1;
        }
      }
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issue
    if (lane == 0) {
      const uint32_t idesc = sm100::idesc_f16_f32(kSBM, kSBN);
      int64_t c = 0;
      bool ok = true;
      int q0 = 0, k0 = 0;
      for (int item = 0; ok && item_at(item, q0, k0); ++item) {
        const int ab = item & 1, use = item >> 1;
        if (use > 0 && !wait(&acce[ab], (uint32_t)((use - 1) & 1), 52)) break;
        sm100::tc_fence_after();
        const uint32_t td = tmem + (uint32_t)(ab * kSBN);
        for (int kc = 0; kc < nk; ++kc, ++c) {
          const int slot = (int)(c % S);
          if (!wait(&full[slot], (uint32_t)((c / S) & 1), 53)) {
            ok = false;
            break;
          }
          sm100::tc_fence_after();
          const uint32_t sa = sm100::smem_u32(smem + slot * kSStage), sb = sa + 2 * kSABytes;
#pragma unroll
          for (int pc = 0; pc < 2; ++pc) {  // query hi, then query lo (not against c_lo)
            if (pc == 1 && kc >= lo_skip0 && kc < lo_skip1) continue;
#pragma unroll
            for (int ks = 0; ks < kSBK / 16; ++ks) {
              const uint64_t da = sm100::desc_sw128(sa + pc * kSABytes + ks * 32);
              const uint64_t db = sm100::desc_sw128(sb + ks * 32);
              sm100::mma_f16(td, da, db, idesc, (kc | pc | ks) != 0);
            }
          }
          any_mma = true;
          sm100::mma_commit(&empty[slot]);
        }
        if (!ok) break;
        sm100::mma_commit(&accf[ab]);
      }
    }
  } else {
    // ------------------------------------------------------------ epilogue
    const int quarter = warp % 4, rin = 32 * quarter + lane;
    const uint32_t tlane = (uint32_t)(32 * quarter) << 16;
    float *sNorm = reinterpret_cast<float *>(sTmem + 4);  // [2][kSBN] key norms of the item (top-k mode)
    float ts[kTopSlots];
    int64_t ti[kTopSlots];
#pragma unroll
    for (int j = 0; j < kTopSlots; ++j) {
      ts[j] = -INFINITY;
      ti[j] = -1;
    }
    int q0 = 0, k0 = 0, qr = -1;
    for (int item = 0; item_at(item, q0, k0); ++item) {
      const int ab = item & 1, use = item >> 1;
      qr = q0 + rin;
      const bool valid = qr < p.M;
      const float qs = valid ? p.qscale[qr] : 0.f;
      if (p.topk) {
        // the item's key norms, once per CTA, shared by the 128 rows
        for (int j = threadIdx.x - 64; j < kSBN; j += kSThreads - 64)
          sNorm[ab * kSBN + j] = k0 + j < p.N ? p.norms[k0 + j].x : 0.f;
        sm100::named_barrier(1, kSThreads - 64);
      }
      if (!__all_sync(0xffffffffu, wait(&accf[ab], (uint32_t)(use & 1), 54))) break;
      sm100::tc_fence_after();
      if (p.topk) {
        for (int cc = 0; cc < kSBN / 32; ++cc) {
          const int col0 = k0 + 32 * cc;
          if (col0 >= p.N) break;  // warp-uniform
          uint32_t v[32];
          sm100::tmem_ld32(tmem + tlane + (uint32_t)(ab * kSBN + 32 * cc), v);
          sm100::tmem_wait_ld();
          if (!valid) continue;
#pragma unroll
          for (int j = 0; j < 32; ++j) {
            const int col = col0 + j;
            // the logit exactly as the all-logits path computes it
            float sres = __uint_as_float(v[j]) * qs * sNorm[ab * kSBN + 32 * cc + j];
            if (col < p.N && sres > ts[kTopSlots - 1]) {
              // keys arrive in ascending index order: an equal score stays
              // behind the earlier key
              int64_t id = p.key_base + col;
#pragma unroll
              for (int s2 = 0; s2 < kTopSlots; ++s2) {
                if (sres > ts[s2]) {
                  const float tv = ts[s2];
                  const int64_t tix = ti[s2];
                  ts[s2] = sres;
                  ti[s2] = id;
                  sres = tv;
                  id = tix;
                }
              }
            }
          }
        }
        sm100::tc_fence_before();
        __syncwarp();
        if (lane == 0) sm100::mbar_arrive(&acce[ab]);
        continue;
      }
      float *orow = p.out + (int64_t)qr * p.ldo;
      for (int cc = 0; cc < kSBN / 32; ++cc) {
        const int col0 = k0 + 32 * cc;
        if (col0 >= p.N) break;  // warp-uniform
        uint32_t v[32];
        sm100::tmem_ld32(tmem + tlane + (uint32_t)(ab * kSBN + 32 * cc), v);
        sm100::tmem_wait_ld();
        if (!valid) continue;
#pragma unroll
        for (int j = 0; j < 32; ++j) {
          const int col = col0 + j;
          if (col < p.N) {
            float sres = __uint_as_float(v[j]) * qs * __ldg(&p.norms[col].x);
            if (p.accumulate) sres += orow[col];
            orow[col] = sres;
          }
        }
      }
      sm100::tc_fence_before();
      __syncwarp();
      if (lane == 0) sm100::mbar_arrive(&acce[ab]);
    }
    if (p.topk && (int)blockIdx.x < ntq * p.P) {
      const int row = ((int)blockIdx.x % ntq) * kSBM + rin;
      if (row < p.M && !*sAbort) {
        const int64_t o = (int64_t)row * p.part_ld + p.part_base + (int64_t)((int)blockIdx.x / ntq) * kTopSlots;
#pragma unroll
        for (int j = 0; j < kTopSlots; ++j) {
          p.part_s[o + j] = ts[j];
          p.part_i[o + j] = ti[j];
        }
      }
    }
  }
  // ------------------------------------------------------------ teardown
  __syncthreads();
  if (warp == 1 && lane == 0 && any_mma) {
    sm100::mma_commit(done);
    sm100::mbar_wait(done, 0u, p.err, 55);
  }
  if (warp == 0 && lane == 0 && *sAbort) {
    for (int64_t c = loads > S ? loads - S : 0; c < loads; ++c)
      sm100::mbar_wait(&full[c % S], (uint32_t)((c / S) & 1), p.err, 56);
  }
  sm100::tc_fence_before();
  __syncthreads();
  sm100::tc_fence_after();
  if (warp == 1) sm100::tmem_dealloc(tmem, 2 * kSBN);
}

// One warp per query row: [y~ | y~ | kappa p] 2^s as fp16 hi + lo.
__global__ void k_dscore_queries(const float *ytil, const float *p, int d, int m, int64_t nq, float kappa,
                                 __half *qh, __half *ql, float *qscale) {
  const int64_t row = (int64_t)blockIdx.x * (blockDim.x / 32) + threadIdx.x / 32;
  const int lane = threadIdx.x % 32;
  if (row >= nq) return;
  const int K = 2 * d + m;
  auto at = [&](int j) {
    return j < 2 * d ? ytil[row * d + (j < d ? j : j - d)] : kappa * p[row * m + (j - 2 * d)];
  };
  float big = 0.f;
  for (int j = lane; j < K; j += 32) big = fmaxf(big, fabsf(at(j)));
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) big = fmaxf(big, __shfl_xor_sync(0xffffffffu, big, o));
  int E = 0;
  frexpf(big, &E);  // big < 2^E
  const int s = big > 0.f ? 14 - E : 0;
  for (int j = lane; j < K; j += 32) {
    const float v = ldexpf(at(j), s);
    const __half h = __float2half_rn(v);
    qh[row * K + j] = h;
    ql[row * K + j] = __float2half_rn(v - __half2float(h));
  }
  if (lane == 0) qscale[row] = ldexpf(1.0f, -s);
}

// One thread per (key, 32-coordinate group of the row [c_hi | c_lo | gamma (2 bits - 1)]).
template <int W>
__global__ void k_dscore_keys(KernelTables kt, int64_t cnt, const uint32_t *codes, const uint32_t *signs,
                              const float2 *norms, __half *kop) {
  // the centroids' two fp16 pieces, c = hi + lo, per code value
  __shared__ uint16_t tab[2][kMaxLevels];
  if (threadIdx.x < kMaxLevels) {
    const float c = kt.centroids[threadIdx.x];
    const __half hi = __float2half_rn(c);
    const __half lo = __float2half_rn(c - __half2float(hi));
    tab[0][threadIdx.x] = *reinterpret_cast<const uint16_t *>(&hi);
    tab[1][threadIdx.x] = *reinterpret_cast<const uint16_t *>(&lo);
  }
  __syncthreads();
  const int ng = kt.d / 32, nsg = kt.m / 32, K = 2 * kt.d + kt.m, per = 2 * ng + nsg;
  const int64_t t = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
  if (t >= cnt * per) return;
  const int64_t key = t / per;
  const int grp = (int)(t % per);
  uint32_t hv[16];
  if (grp < 2 * ng) {
    const int cg = grp < ng ? grp : grp - ng;
    const uint16_t *tb = tab[grp >= ng ? 1 : 0];
    uint32_t w[W];
#pragma unroll
    for (int k = 0; k < W; ++k) w[k] = codes[key * (W * ng) + cg * W + k];
#pragma unroll
    for (int i = 0; i < 32; i += 2)
      hv[i / 2] = (uint32_t)tb[unpack_code<W>(w, i)] | ((uint32_t)tb[unpack_code<W>(w, i + 1)] << 16);
  } else {
    const uint32_t sw = signs[key * nsg + (grp - 2 * ng)];
    const float g = norms[key].y;
#pragma unroll
    for (int i = 0; i < 32; i += 2) {
      const __half2 h = __floats2half2_rn((sw >> i) & 1u ? g : -g, (sw >> (i + 1)) & 1u ? g : -g);
      hv[i / 2] = *reinterpret_cast<const uint32_t *>(&h);
    }
  }
  uint4 *dst = reinterpret_cast<uint4 *>(kop + key * K + grp * 32);
#pragma unroll
  for (int k = 0; k < 4; ++k) dst[k] = make_uint4(hv[4 * k], hv[4 * k + 1], hv[4 * k + 2], hv[4 * k + 3]);
}

bool make_map16(CUtensorMap *map, const void *base, int64_t cols, int64_t rows, uint32_t box_rows) {
  auto enc = tensor_map_encoder();
  if (!enc) return false;
  cuuint64_t gdim[2] = {(cuuint64_t)cols, (cuuint64_t)rows};
  cuuint64_t gstride[1] = {(cuuint64_t)cols * 2};
  cuuint32_t box[2] = {(cuuint32_t)kSBK, box_rows};
  cuuint32_t estr[2] = {1, 1};
  return enc(map, CU_TENSOR_MAP_DATA_TYPE_FLOAT16, 2, const_cast<void *>(base), gdim, gstride, box, estr,
             CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
             CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

struct DScoreLayout {
  size_t qh, ql, qs, kop, total;
};
DScoreLayout dscore_layout(const tq_quantizer *q, int64_t nq) {
  auto up = [](size_t v) { return (v + 255) / 256 * 256; };
  const size_t K = 2 * (size_t)q->d + q->m;
  DScoreLayout L{};
  L.qh = 0;
  L.ql = up((size_t)nq * K * 2);
  L.qs = L.ql + up((size_t)nq * K * 2);
  L.kop = L.qs + up((size_t)nq * 4);
  L.total = L.kop + up((size_t)kKeyChunk * K * 2);
  return L;
}

}  // namespace

bool dense_score_supported(const tq_quantizer *q) {
  return q->d > 128 && q->d % 64 == 0 && q->m > 0 && q->m % 64 == 0 && q->w >= 1 && q->w <= 4;
}

size_t dense_score_ws_bytes(const tq_quantizer *q, int64_t nq) { return dscore_layout(q, nq).total; }

tq_status dense_score(const tq_quantizer *q, const float *ytil, const float *p, int64_t nq_rows, int64_t G,
                      int64_t kpg, int64_t key_base, int64_t nkeys, const void *codes, const void *signs,
                      const float *norms, float *out, int64_t ldo, int accumulate, void *ws, size_t ws_bytes,
                      cudaStream_t st) {
  const DScoreLayout L = dscore_layout(q, nq_rows);
  if (!ws || ws_bytes < L.total) return TQ_ERR_WORKSPACE;
  const int d = q->d, m = q->m, K = 2 * d + m, ng = d / 32, nsg = m / 32;
  char *base = static_cast<char *>(ws);
  __half *qh = reinterpret_cast<__half *>(base + L.qh), *ql = reinterpret_cast<__half *>(base + L.ql);
  float *qs = reinterpret_cast<float *>(base + L.qs);
  __half *kop = reinterpret_cast<__half *>(base + L.kop);
  const float kappa = q->kt.qjl_scale;
  k_dscore_queries<<<(unsigned)((nq_rows + 7) / 8), 256, 0, st>>>(ytil, p, d, m, nq_rows, kappa, qh, ql, qs);
  if (cudaGetLastError() != cudaSuccess) return TQ_ERR_CUDA;
  int dev = 0, sms = 0, max_smem = 0;
  cudaGetDevice(&dev);
  cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  cudaDeviceGetAttribute(&max_smem, cudaDevAttrMaxSharedMemoryPerBlockOptin, dev);
  const int extra = 1024 + 8 * 16 + 16 + 2 * kSBN * 4;
  const int nstages = std::min(4, (int)((max_smem - extra) / kSStage));
  if (nstages < 2) return TQ_ERR_UNSUPPORTED;
  const size_t smem = (size_t)nstages * kSStage + extra;
  if (cudaFuncSetAttribute(k_dscore_gemm, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem) != cudaSuccess)
    return TQ_ERR_CUDA;
  const int64_t groups = nq_rows / G;
  auto cw = static_cast<const uint32_t *>(codes);
  auto sw = static_cast<const uint32_t *>(signs);
  auto nr = reinterpret_cast<const float2 *>(norms);
  for (int64_t g = 0; g < groups; ++g) {
    CUtensorMap mqh, mql;
    if (!make_map16(&mqh, qh + g * G * K, K, G, kSBM) || !make_map16(&mql, ql + g * G * K, K, G, kSBM))
      return TQ_ERR_CUDA;
    for (int64_t c0 = 0; c0 < nkeys; c0 += kKeyChunk) {
      const int64_t cnt = std::min(kKeyChunk, nkeys - c0);
      const int64_t key0 = g * kpg + key_base + c0;
      const int64_t threads = cnt * (2 * ng + nsg);
      switch (q->w) {
        case 1: k_dscore_keys<1><<<(unsigned)((threads + 255) / 256), 256, 0, st>>>(q->kt, cnt, cw + key0 * ng, sw + key0 * nsg, nr + key0, kop); break;
        case 2: k_dscore_keys<2><<<(unsigned)((threads + 255) / 256), 256, 0, st>>>(q->kt, cnt, cw + key0 * 2 * ng, sw + key0 * nsg, nr + key0, kop); break;
        case 3: k_dscore_keys<3><<<(unsigned)((threads + 255) / 256), 256, 0, st>>>(q->kt, cnt, cw + key0 * 3 * ng, sw + key0 * nsg, nr + key0, kop); break;
        case 4: k_dscore_keys<4><<<(unsigned)((threads + 255) / 256), 256, 0, st>>>(q->kt, cnt, cw + key0 * 4 * ng, sw + key0 * nsg, nr + key0, kop); break;
        default: return TQ_ERR_UNSUPPORTED;
      }
      if (cudaGetLastError() != cudaSuccess) return TQ_ERR_CUDA;
      CUtensorMap mk;
      if (!make_map16(&mk, kop, K, cnt, kSBN)) return TQ_ERR_CUDA;
      DScoreParams prm{};
      prm.M = (int)G;
      prm.N = (int)cnt;
      prm.K = K;
      prm.d = d;
      prm.nstages = nstages;
      prm.err = q->d_err;
      prm.qscale = qs + g * G;
      prm.norms = nr + key0;
      prm.out = out + g * G * ldo + c0;
      prm.ldo = ldo;
      prm.accumulate = accumulate;
      const int nitems = (int)(((G + kSBM - 1) / kSBM) * ((cnt + kSBN - 1) / kSBN));
      k_dscore_gemm<<<std::min(nitems, sms), kSThreads, smem, st>>>(mqh, mql, mk, prm);
      if (cudaGetLastError() != cudaSuccess) return TQ_ERR_CUDA;
    }
  }
  return TQ_OK;
}

// Keys per chunk of the top-k GEMM: a whole number of key tiles for each of
// the P CTAs that share a query tile (at most kKeyChunk), so that they finish
// together.
static int64_t topk_chunk(int64_t P) {
  const int64_t per = P * kSBN;
  return per >= kKeyChunk ? kKeyChunk : (kKeyChunk / per) * per;
}

size_t dense_topk_ws_bytes(const tq_quantizer *q, int64_t nq, int64_t n) {
  auto up = [](size_t v) { return (v + 255) / 256 * 256; };
  int dev = 0, sms = 148;
  if (cudaGetDevice(&dev) == cudaSuccess) cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  const int64_t ntq = (nq + kSBM - 1) / kSBM;
  const int64_t P = std::max<int64_t>(1, sms / ntq);
  const int64_t nchunks = (n + topk_chunk(P) - 1) / topk_chunk(P);
  const size_t slots = (size_t)nchunks * P * kTopSlots;
  return up(dense_score_ws_bytes(q, nq)) + up((size_t)nq * slots * 4) + up((size_t)nq * slots * 8);
}

// Top-k over n keys for d > 128 without writing the logits: per 32768-key
// chunk the keys are decoded and the GEMM keeps, per query row and CTA, the
// kTopSlots best (score, key) pairs; one selection over those candidates
// gives the k best (k <= kTopSlots; ties to the lower key index).
tq_status dense_topk(const tq_quantizer *q, const float *ytil, const float *p, int64_t nq, int64_t n, int k,
                     const void *codes, const void *signs, const float *norms, float *out_s, int64_t *out_i,
                     void *ws, size_t ws_bytes, cudaStream_t st) {
  if (k < 1 || k > kTopSlots) return TQ_ERR_UNSUPPORTED;
  auto up = [](size_t v) { return (v + 255) / 256 * 256; };
  const DScoreLayout L = dscore_layout(q, nq);
  if (!ws || ws_bytes < dense_topk_ws_bytes(q, nq, n)) return TQ_ERR_WORKSPACE;
  const int d = q->d, m = q->m, K = 2 * d + m, ng = d / 32, nsg = m / 32;
  char *base = static_cast<char *>(ws);
  __half *qh = reinterpret_cast<__half *>(base + L.qh), *ql = reinterpret_cast<__half *>(base + L.ql);
  float *qs = reinterpret_cast<float *>(base + L.qs);
  __half *kop = reinterpret_cast<__half *>(base + L.kop);
  int dev = 0, sms = 0, max_smem = 0;
  cudaGetDevice(&dev);
  cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  cudaDeviceGetAttribute(&max_smem, cudaDevAttrMaxSharedMemoryPerBlockOptin, dev);
  const int ntq = (int)((nq + kSBM - 1) / kSBM);
  const int P = std::max(1, sms / ntq);
  const int64_t chunk = topk_chunk(P);
  const int64_t nchunks = (n + chunk - 1) / chunk;
  const int64_t slots = nchunks * P * kTopSlots;
  float *part_s = reinterpret_cast<float *>(base + up(L.total));
  int64_t *part_i = reinterpret_cast<int64_t *>(base + up(L.total) + up((size_t)nq * slots * 4));
  k_dscore_queries<<<(unsigned)((nq + 7) / 8), 256, 0, st>>>(ytil, p, d, m, nq, q->kt.qjl_scale, qh, ql, qs);
  if (cudaGetLastError() != cudaSuccess) return TQ_ERR_CUDA;
  const int extra = 1024 + 8 * 16 + 16 + 2 * kSBN * 4;
  const int nstages = std::min(4, (int)((max_smem - extra) / kSStage));
  if (nstages < 2) return TQ_ERR_UNSUPPORTED;
  const size_t smem = (size_t)nstages * kSStage + extra;
  if (cudaFuncSetAttribute(k_dscore_gemm, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem) != cudaSuccess)
    return TQ_ERR_CUDA;
  CUtensorMap mqh, mql;
  if (!make_map16(&mqh, qh, K, nq, kSBM) || !make_map16(&mql, ql, K, nq, kSBM)) return TQ_ERR_CUDA;
  auto cw = static_cast<const uint32_t *>(codes);
  auto sw = static_cast<const uint32_t *>(signs);
  auto nr = reinterpret_cast<const float2 *>(norms);
  for (int64_t ci = 0; ci < nchunks; ++ci) {
    const int64_t key0 = ci * chunk;
    const int64_t cnt = std::min(chunk, n - key0);
    const int64_t threads = cnt * (2 * ng + nsg);
    const unsigned blocks = (unsigned)((threads + 255) / 256);
    switch (q->w) {
      case 1: k_dscore_keys<1><<<blocks, 256, 0, st>>>(q->kt, cnt, cw + key0 * ng, sw + key0 * nsg, nr + key0, kop); break;
      case 2: k_dscore_keys<2><<<blocks, 256, 0, st>>>(q->kt, cnt, cw + key0 * 2 * ng, sw + key0 * nsg, nr + key0, kop); break;
      case 3: k_dscore_keys<3><<<blocks, 256, 0, st>>>(q->kt, cnt, cw + key0 * 3 * ng, sw + key0 * nsg, nr + key0, kop); break;
      case 4: k_dscore_keys<4><<<blocks, 256, 0, st>>>(q->kt, cnt, cw + key0 * 4 * ng, sw + key0 * nsg, nr + key0, kop); break;
      default: return TQ_ERR_UNSUPPORTED;
    }
    if (cudaGetLastError() != cudaSuccess) return TQ_ERR_CUDA;
    CUtensorMap mk;
    if (!make_map16(&mk, kop, K, cnt, kSBN)) return TQ_ERR_CUDA;
    DScoreParams prm{};
    prm.M = (int)nq;
    prm.N = (int)cnt;
    prm.K = K;
    prm.d = d;
    prm.nstages = nstages;
    prm.err = q->d_err;
    prm.qscale = qs;
    prm.norms = nr + key0;
    prm.topk = 1;
    prm.P = P;
    prm.key_base = key0;
    prm.part_s = part_s;
    prm.part_i = part_i;
    prm.part_ld = slots;
    prm.part_base = ci * P * kTopSlots;
    k_dscore_gemm<<<ntq * P, kSThreads, smem, st>>>(mqh, mql, mk, prm);
    if (cudaGetLastError() != cudaSuccess) return TQ_ERR_CUDA;
  }
  return v1_topk_select(part_s, part_i, nq, slots, slots, slots, 0, k, out_s, out_i, k, st);
}

}  // namespace tq

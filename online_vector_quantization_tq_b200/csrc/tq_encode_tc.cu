// Tensor-core encode for bf16 keys (d in {32, 64, 96, 128}), one CTA per SM,
// 256 threads, tiles of 128 vectors.  Per tile:
//
//   TMA  x tile (bf16, 128 rows) -> shared memory (double-buffered)
//   ALU  ||x|| (two threads per row, partial sums exchanged), x * 2^e -> fp16
//        (exact: bf16 has 8 significant bits) into the A operand tile
//   MMA  U = X' * Rq^T on tcgen05 (Rq: the rotation as 1 or 2 fp16 pieces;
//        the Hadamard form d^1.5 R is an integer matrix, exact in fp16), fp32
//        accumulators in TMEM
//   ALU  u = U * scale, code = #{t < u}, r = u - c[code] (scaled by 2^10),
//        gamma^2, r -> fp16 hi + lo into the QJL A operand, codes -> global
//   MMA  Z = [r_hi | r_lo] * [S | S]^T (S is fp16-exact), fp32 in TMEM
//   ALU  sign bits of Z -> global (one tile later, overlapping the next
//        tile's rotation MMA), norms -> global
//
// The rotation of tile t runs while the sign bits of tile t-1 are extracted;
// the QJL projection of tile t runs while tile t+1 is loaded and converted.
// Method: TurboQuant article 1.2.1-1.2.3 (rotation, Lloyd-Max code, residual,
// QJL sign sketch), 2.1 (structured rotation), 4.2.1 (stored norm).
#include <cudaTypedefs.h>

#include "tq_common.cuh"
#include "tq_kernels.h"
#include "tq_rng.cuh"
#include "tq_sm100.cuh"

namespace tq {

struct EncTCParams {
  int64_t n;
  int ntiles;
  const uint16_t *rot16;  // [RP][D][D] fp16 bits, row-major (out, in)
  const uint16_t *s16;    // [D][D] fp16 bits (QJL rows, in)
  uint64_t s_key;         // S's stream key, for kernels that generate S
  int s_otf;              // nonzero: generate S instead of reading s16
  float rho;              // R = rho * sum of rotation pieces
  float thr_s[kMaxLevels];   // thresholds * 2^10
  float cen_s[kMaxLevels];   // centroids * 2^10
  const int32_t *chan;
  int64_t chan_rows;
  uint32_t *codes;
  uint32_t *signs;
  float2 *norms;
  int64_t out_stride;
  int *err;
};

namespace {

constexpr int kThreads = 256;
constexpr int kRows = 128;
constexpr float kRScale = 1024.0f;  // residuals are split into fp16 at 2^10 scale

template <int D, int RP, int SRCW, int NXB>
struct EncSmem {
  static constexpr int kXBytes = kRows * SRCW * 2;          // one bf16 x tile (SW128 boxes of 64 cols)
  static constexpr int kAxBytes = kRows * D * 2;            // fp16 X'
  static constexpr int kArBytes = kRows * 2 * D * 2;        // fp16 [r_hi | r_lo]
  static constexpr int kBrBytes = RP * D * D * 2;           // rotation pieces
  static constexpr int kBsBytes = D * D * 2;                // S
  static constexpr int kOffX = 0;
  static constexpr int kOffAx = kOffX + NXB * kXBytes;
  static constexpr int kOffAr = kOffAx + kAxBytes;
  static constexpr int kOffBr = kOffAr + kArBytes;
  static constexpr int kOffBs = kOffBr + kBrBytes;
  static constexpr int kOffMisc = kOffBs + kBsBytes;
  static constexpr int kMiscBytes = 4096;
  static constexpr int kTotal = kOffMisc + kMiscBytes + 1024;  // + alignment slack
};

// Split of a row's D columns between the two threads of the row: thread half
// 0 takes [0, SPL), half 1 takes [SPL, D); SPL is a multiple of 32.
template <int D>
constexpr int split_point() {
  return 32 * ((D / 32 + 1) / 2);
}


__device__ __forceinline__ uint32_t pack_half2(float a, float b) {
  const __half2 h = __floats2half2_rn(a, b);
  return *reinterpret_cast<const uint32_t *>(&h);
}

}  // namespace

template <int D, int W, int RP, int SRCW, int NXB, bool GATHER>
__global__ void __launch_bounds__(kThreads, D == 32 ? 2 : 1)  // d = 32: two CTAs per SM hide the tile's latency chain
k_encode_tc(const __grid_constant__ CUtensorMap xmap, const EncTCParams p) {
  using SM = EncSmem<D, RP, SRCW, NXB>;
  constexpr int L = 1 << W;
  constexpr int SPL = split_point<D>();
  constexpr int NB = SRCW / 64;  // TMA boxes per x tile
  extern __shared__ uint8_t smem_raw[];
  uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t *sX = smem + SM::kOffX;
  uint8_t *sAx = smem + SM::kOffAx;
  uint8_t *sAr = smem + SM::kOffAr;
  uint8_t *sBr = smem + SM::kOffBr;
  uint8_t *sBs = smem + SM::kOffBs;
  float *sRed = reinterpret_cast<float *>(smem + SM::kOffMisc);         // [2][128][2]
  float *sCen = sRed + 2 * kRows * 2;                                   // [16]
  uint64_t *bars = reinterpret_cast<uint64_t *>(sCen + kMaxLevels);      // full[2], rot, qjl
  uint32_t *sTmem = reinterpret_cast<uint32_t *>(bars + 4);

  const int tid = threadIdx.x;
  const int row = tid & (kRows - 1);
  const int half = tid >> 7;
  const int c0 = half ? SPL : 0;
  constexpr int NC0 = SPL, NC1 = D - SPL;
  const int nc = half ? NC1 : NC0;
  const uint32_t lane_base = (uint32_t)(row & ~31) << 16;

  // ---- set-up: barriers, TMEM, constant operands
  if (tid == 0) {
    for (int i = 0; i < 4; ++i) sm100::mbar_init(&bars[i], 1);
    sm100::fence_barrier_init();
    sm100::prefetch_tmap(&xmap);
  }
  if (tid < 32) {
    sm100::tmem_alloc(sTmem, 256);
    sm100::tmem_relinquish();
  }
  if (tid < kMaxLevels) sCen[tid] = p.cen_s[tid];
#pragma unroll
  for (int pc = 0; pc < RP; ++pc) sm100::stage_kmajor<D>(sBr + pc * (D * D * 2), p.rot16 + (size_t)pc * D * D, D);
  sm100::stage_kmajor<D>(sBs, p.s16, D);
  sm100::fence_proxy_async();
  sm100::tc_fence_before();
  __syncthreads();
  sm100::tc_fence_after();
  const uint32_t tmem = *sTmem;
  const uint32_t tU = tmem, tZ = tmem + 128;
  float thr[L - 1];
#pragma unroll
  for (int i = 0; i < L - 1; ++i) thr[i] = p.thr_s[i];

  const int first = blockIdx.x;
  const int stride = gridDim.x;
  // prefetch the first NXB tiles
  if (tid == 0) {
    for (int b = 0; b < NXB; ++b) {
      const int t = first + b * stride;
      if (t < p.ntiles) {
        sm100::mbar_expect_tx(&bars[b], SM::kXBytes);
        for (int bx = 0; bx < NB; ++bx)
          sm100::tma_load_2d(sX + b * SM::kXBytes + bx * (kRows * 128), &xmap, bx * 64, t * kRows, &bars[b]);
      }
    }
  }

  uint32_t ph_full[2] = {0u, 0u}, ph_rot = 0u, ph_qjl = 0u;
  float prev_norm = 0.f, prev_gamma = 0.f;
  int64_t prev_row = -1;
  bool failed = false;
  const uint32_t idesc = sm100::idesc_f16_f32(kRows, D);
  int it = 0;

  for (int t = first; t < p.ntiles; t += stride, ++it) {
    const int buf = NXB == 2 ? (it & 1) : 0;
    const int64_t grow = (int64_t)t * kRows + row;
    // ---- A: x tile -> registers
    bool ok = sm100::mbar_wait(&bars[buf], ph_full[buf], p.err, 1);
    ph_full[buf] ^= 1u;
    float xv[NC0 > NC1 ? NC0 : NC1];
    const uint8_t *xt = sX + buf * SM::kXBytes;
    if constexpr (!GATHER) {
#pragma unroll
      for (int k = 0; k < (NC0 > NC1 ? NC0 : NC1) / 8; ++k) {
        if (k < nc / 8) {
          const int col = c0 + 8 * k;
          const uint4 v = *reinterpret_cast<const uint4 *>(xt + (col / 64) * (kRows * 128) +
                                                           sm100::sw128_offset(row, (col % 64) / 8));
          const uint32_t w4[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
          for (int e = 0; e < 4; ++e) {
            xv[8 * k + 2 * e] = __uint_as_float(w4[e] << 16);
            xv[8 * k + 2 * e + 1] = __uint_as_float(w4[e] & 0xFFFF0000u);
          }
        }
      }
    } else {
      const int32_t *ch = p.chan + (grow / p.chan_rows) * D;
#pragma unroll
      for (int j = 0; j < (NC0 > NC1 ? NC0 : NC1); ++j) {
        if (j < nc) {
          // masked to the staged tile: a channel index outside the source row
          // cannot address memory beyond it
          const int src = grow < p.n ? (__ldg(ch + c0 + j) & (SRCW - 1)) : 0;
          const uint16_t hv = *reinterpret_cast<const uint16_t *>(
              xt + (src / 64) * (kRows * 128) + sm100::sw128_offset(row, (src % 64) / 8) + (src % 8) * 2);
          xv[j] = __uint_as_float((uint32_t)hv << 16);
        }
      }
    }
    float ss = 0.f;
#pragma unroll
    for (int j = 0; j < (NC0 > NC1 ? NC0 : NC1); ++j)
      if (j < nc) ss = fmaf(xv[j], xv[j], ss);
    sRed[row * 2 + half] = ss;
    failed |= __syncthreads_or(!ok) != 0;
    if (failed) break;
    // ---- B: norm, scale, fp16 X' -> A operand
    const float nrm = sqrtf(sRed[row * 2] + sRed[row * 2 + 1]);
    int e = 0;
    float s_v = 0.f;  // acc -> u * 2^10
    if (nrm > 0.f) {
      e = 14 - (int)((__float_as_uint(nrm) >> 23) & 0xFF) + 127;
      e = max(-100, min(100, e));
      s_v = p.rho * kRScale / (nrm * __uint_as_float((uint32_t)(127 + e) << 23));
    }
    const float xs = __uint_as_float((uint32_t)(127 + e) << 23);
#pragma unroll
    for (int k = 0; k < (NC0 > NC1 ? NC0 : NC1) / 8; ++k) {
      if (k < nc / 8) {
        const int col = c0 + 8 * k;
        uint4 h;
        h.x = pack_half2(xv[8 * k + 0] * xs, xv[8 * k + 1] * xs);
        h.y = pack_half2(xv[8 * k + 2] * xs, xv[8 * k + 3] * xs);
        h.z = pack_half2(xv[8 * k + 4] * xs, xv[8 * k + 5] * xs);
        h.w = pack_half2(xv[8 * k + 6] * xs, xv[8 * k + 7] * xs);
        *reinterpret_cast<uint4 *>(sAx + (col / 32) * (kRows * 64) + sm100::sw64_offset(row, (col % 32) / 8)) = h;
      }
    }
    sm100::fence_proxy_async();
    __syncthreads();
    // ---- C: rotation MMA; prefetch the tile NXB ahead into this x buffer
    if (tid == 0) {
      sm100::tc_fence_after();
      const uint32_t ax = sm100::smem_u32(sAx), br = sm100::smem_u32(sBr);
#pragma unroll
      for (int pc = 0; pc < RP; ++pc)
#pragma unroll
        for (int ks = 0; ks < D / 16; ++ks) {
          const uint64_t a = sm100::desc_sw64(ax + (ks >> 1) * (kRows * 64) + (ks & 1) * 32);
          const uint64_t b = sm100::desc_sw64(br + pc * (D * D * 2) + (ks >> 1) * (D * 64) + (ks & 1) * 32);
          sm100::mma_f16(tU, a, b, idesc, (pc | ks) != 0);
        }
      sm100::mma_commit(&bars[2]);
      const int tn = t + NXB * stride;
      if (tn < p.ntiles) {
        sm100::mbar_expect_tx(&bars[buf], SM::kXBytes);
        for (int bx = 0; bx < NB; ++bx)
          sm100::tma_load_2d(sX + buf * SM::kXBytes + bx * (kRows * 128), &xmap, bx * 64, tn * kRows, &bars[buf]);
      }
    }
    // ---- D: sign bits of the previous tile
    if (it > 0) {
      ok = sm100::mbar_wait(&bars[3], ph_qjl, p.err, 3);
      ph_qjl ^= 1u;
      sm100::tc_fence_after();
#pragma unroll
      for (int g = 0; g < (NC0 > NC1 ? NC0 : NC1) / 32; ++g) {
        if (g < nc / 32) {
          uint32_t z[32];
          sm100::tmem_ld16(tZ + lane_base + c0 + 32 * g, *reinterpret_cast<uint32_t(*)[16]>(&z[0]));
          sm100::tmem_ld16(tZ + lane_base + c0 + 32 * g + 16, *reinterpret_cast<uint32_t(*)[16]>(&z[16]));
          sm100::tmem_wait_ld();
          uint32_t wbits = 0u;
#pragma unroll
          for (int j = 31; j >= 0; --j) wbits = __funnelshift_l(z[j], wbits, 1);
          if (prev_row >= 0 && prev_row < p.n)
            p.signs[prev_row * p.out_stride * (D / 32) + (c0 / 32) + g] = ~wbits;
        }
      }
      if (half == 0 && prev_row >= 0 && prev_row < p.n)
        p.norms[prev_row * p.out_stride] = make_float2(prev_norm, prev_gamma);
    }
    // ---- E: rotated coordinates -> codes, residual split
    ok = sm100::mbar_wait(&bars[2], ph_rot, p.err, 2) && ok;
    ph_rot ^= 1u;
    sm100::tc_fence_after();
    float g2 = 0.f;
#pragma unroll
    for (int g = 0; g < (NC0 > NC1 ? NC0 : NC1) / 32; ++g) {
      if (g < nc / 32) {
        uint32_t acc[32];
        sm100::tmem_ld16(tU + lane_base + c0 + 32 * g, *reinterpret_cast<uint32_t(*)[16]>(&acc[0]));
        sm100::tmem_ld16(tU + lane_base + c0 + 32 * g + 16, *reinterpret_cast<uint32_t(*)[16]>(&acc[16]));
        sm100::tmem_wait_ld();
        uint32_t cw[W];
#pragma unroll
        for (int k = 0; k < W; ++k) cw[k] = 0u;
        float rs[32];
#pragma unroll
        for (int j = 0; j < 32; ++j) {
          const float us = __uint_as_float(acc[j]) * s_v;
          int c = 0;
#pragma unroll
          for (int i = 0; i < L - 1; ++i) c += us > thr[i] ? 1 : 0;
          pack_code<W>(cw, j, (uint32_t)c);
          rs[j] = us - sCen[c];
          g2 = fmaf(rs[j], rs[j], g2);
        }
        if (grow < p.n) {
          uint32_t *dst = p.codes + grow * p.out_stride * (W * D / 32) + ((c0 / 32) + g) * W;
#pragma unroll
          for (int k = 0; k < W; ++k) dst[k] = cw[k];
        }
        // r = hi + lo, both fp16, into [r_hi | r_lo]
#pragma unroll
        for (int k = 0; k < 4; ++k) {
          uint32_t hi[4], lo[4];
#pragma unroll
          for (int e2 = 0; e2 < 4; ++e2) {
            const float a = rs[8 * k + 2 * e2], b = rs[8 * k + 2 * e2 + 1];
            const __half2 h = __floats2half2_rn(a, b);
            const float2 hf = __half22float2(h);
            hi[e2] = *reinterpret_cast<const uint32_t *>(&h);
            lo[e2] = pack_half2(a - hf.x, b - hf.y);
          }
          const int col = c0 + 32 * g + 8 * k;
          *reinterpret_cast<uint4 *>(sAr + (col / 32) * (kRows * 64) + sm100::sw64_offset(row, (col % 32) / 8)) =
              make_uint4(hi[0], hi[1], hi[2], hi[3]);
          *reinterpret_cast<uint4 *>(sAr + ((D + col) / 32) * (kRows * 64) +
                                     sm100::sw64_offset(row, (col % 32) / 8)) = make_uint4(lo[0], lo[1], lo[2], lo[3]);
        }
      }
    }
    sRed[2 * kRows + row * 2 + half] = g2;
    sm100::fence_proxy_async();
    sm100::tc_fence_before();
    failed |= __syncthreads_or(!ok) != 0;
    if (failed) break;
    // ---- F: QJL MMA
    if (tid == 0) {
      sm100::tc_fence_after();
      const uint32_t ar = sm100::smem_u32(sAr), bs = sm100::smem_u32(sBs);
#pragma unroll
      for (int ks = 0; ks < 2 * D / 16; ++ks) {
        const int kk = ks % (D / 16);
        const uint64_t a = sm100::desc_sw64(ar + (ks >> 1) * (kRows * 64) + (ks & 1) * 32);
        const uint64_t b = sm100::desc_sw64(bs + (kk >> 1) * (D * 64) + (kk & 1) * 32);
        sm100::mma_f16(tZ, a, b, idesc, ks != 0);
      }
      sm100::mma_commit(&bars[3]);
    }
    prev_norm = nrm;
    prev_gamma = sqrtf(sRed[2 * kRows + row * 2] + sRed[2 * kRows + row * 2 + 1]) * (1.0f / kRScale);
    prev_row = grow;
  }

  // ---- drain: sign bits of the last tile
  if (!failed && it > 0) {
    const bool ok = __syncthreads_and(sm100::mbar_wait(&bars[3], ph_qjl, p.err, 4)) != 0;  // CTA-uniform
    sm100::tc_fence_after();
    if (ok) {
#pragma unroll
      for (int g = 0; g < (NC0 > NC1 ? NC0 : NC1) / 32; ++g) {
        if (g < nc / 32) {
          uint32_t z[32];
          sm100::tmem_ld16(tZ + lane_base + c0 + 32 * g, *reinterpret_cast<uint32_t(*)[16]>(&z[0]));
          sm100::tmem_ld16(tZ + lane_base + c0 + 32 * g + 16, *reinterpret_cast<uint32_t(*)[16]>(&z[16]));
          sm100::tmem_wait_ld();
          uint32_t wbits = 0u;
#pragma unroll
          for (int j = 31; j >= 0; --j) wbits = __funnelshift_l(z[j], wbits, 1);
          if (prev_row >= 0 && prev_row < p.n)
            p.signs[prev_row * p.out_stride * (D / 32) + (c0 / 32) + g] = ~wbits;
        }
      }
      if (half == 0 && prev_row >= 0 && prev_row < p.n)
        p.norms[prev_row * p.out_stride] = make_float2(prev_norm, prev_gamma);
    }
  }
  if (failed && tid == 0) {
    // bounded wait for x-tile loads still in flight before the CTA exits
    for (int b = 0; b < NXB; ++b) sm100::mbar_wait(&bars[b], ph_full[b], p.err, 5);
  }
  sm100::tc_fence_before();
  __syncthreads();
  if (tid < 32) sm100::tmem_dealloc(tmem, 256);
}

// ------------------------------------------------------------------ host side
PFN_cuTensorMapEncodeTiled_v12000 tensor_map_encoder() {
  static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
  if (!fn) {
    cudaDriverEntryPointQueryResult q;
    void *ptr = nullptr;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &ptr, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(ptr);
  }
  return fn;
}

namespace {

template <int D, int W, int RP, int SRCW, bool GATHER>
tq_status launch_tc(const tq_quantizer *q, const void *x, int64_t n, int64_t ldx, int64_t cols,
                    const EncTCParams &prm, cudaStream_t st) {
  auto enc = tensor_map_encoder();
  if (!enc) return TQ_ERR_CUDA;
  CUtensorMap map;
  cuuint64_t gdim[2] = {(cuuint64_t)cols, (cuuint64_t)n};
  cuuint64_t gstride[1] = {(cuuint64_t)ldx * 2};
  cuuint32_t box[2] = {64, 128};
  cuuint32_t estr[2] = {1, 1};
  if (enc(&map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void *>(x), gdim, gstride, box, estr,
          CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
          CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
    return TQ_ERR_CUDA;
  int dev = 0, max_smem = 0, sms = 0;
  cudaGetDevice(&dev);
  cudaDeviceGetAttribute(&max_smem, cudaDevAttrMaxSharedMemoryPerBlockOptin, dev);
  cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  const int ntiles = (int)((n + kRows - 1) / kRows);
  EncTCParams pp = prm;
  pp.ntiles = ntiles;
  if (EncSmem<D, RP, SRCW, 2>::kTotal <= max_smem) {
    auto kern = k_encode_tc<D, W, RP, SRCW, 2, GATHER>;
    const int sm = EncSmem<D, RP, SRCW, 2>::kTotal;
    if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, sm) != cudaSuccess)
      return TQ_ERR_CUDA;
    // persistent CTAs, as many per SM as fit (each holds 256 TMEM columns);
    // ask for the largest shared-memory carveout so that two can
    if (cudaFuncSetAttribute(kern, cudaFuncAttributePreferredSharedMemoryCarveout, 100) != cudaSuccess)
      return TQ_ERR_CUDA;
    // (d = 32 is built for two: 128 registers, under half of shared memory
    // and of TMEM per CTA; the CTAs share nothing, so a pair that cannot be
    // co-resident would only run one after the other)
    const int per_sm = D == 32 ? 2 : 1;
    kern<<<std::min(ntiles, sms * per_sm), kThreads, sm, st>>>(map, pp);
  } else {
    auto kern = k_encode_tc<D, W, RP, SRCW, 1, GATHER>;
    const int sm = EncSmem<D, RP, SRCW, 1>::kTotal;
    if (sm > max_smem) return TQ_ERR_UNSUPPORTED;
    if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, sm) != cudaSuccess)
      return TQ_ERR_CUDA;
    kern<<<std::min(ntiles, sms), kThreads, sm, st>>>(map, pp);
  }
  return cudaGetLastError() == cudaSuccess ? TQ_OK : TQ_ERR_CUDA;
}

template <int D, int W, int RP>
tq_status dispatch_src(const tq_quantizer *q, const void *x, int64_t n, int64_t ldx, bool gather,
                       const EncTCParams &prm, cudaStream_t st) {
  if (gather) return launch_tc<D, W, RP, 128, true>(q, x, n, ldx, ldx, prm, st);
  constexpr int SW = (D + 63) / 64 * 64;
  return launch_tc<D, W, RP, SW, false>(q, x, n, ldx, D, prm, st);
}

template <int D, int W>
tq_status dispatch_rp(const tq_quantizer *q, const void *x, int64_t n, int64_t ldx, bool gather,
                      const EncTCParams &prm, cudaStream_t st) {
  if (q->tc_rot_pieces == 1) return dispatch_src<D, W, 1>(q, x, n, ldx, gather, prm, st);
  return dispatch_src<D, W, 2>(q, x, n, ldx, gather, prm, st);
}

template <int D>
tq_status dispatch_w(const tq_quantizer *q, const void *x, int64_t n, int64_t ldx, bool gather,
                     const EncTCParams &prm, cudaStream_t st) {
  switch (q->w) {
    case 1: return dispatch_rp<D, 1>(q, x, n, ldx, gather, prm, st);
    case 2: return dispatch_rp<D, 2>(q, x, n, ldx, gather, prm, st);
    case 3: return dispatch_rp<D, 3>(q, x, n, ldx, gather, prm, st);
    case 4: return dispatch_rp<D, 4>(q, x, n, ldx, gather, prm, st);
  }
  return TQ_ERR_UNSUPPORTED;
}

}  // namespace

bool tc_encode_supported(const tq_quantizer *q, int dtype, int64_t ldx, bool gather) {
  if (dtype != TQ_BF16 || !q->d_rot16 || q->tc_rot_pieces < 1) return false;
  const int d = q->d;
  if (d != 32 && d != 64 && d != 96 && d != 128) return false;
  if (d == 128 && q->tc_rot_pieces > 1) return false;  // operands would exceed shared memory
  if (gather) return ldx <= 128 && ldx >= 64 && ldx % 64 == 0;
  return d >= 64;  // a 32-column tile would be narrower than the 64-column load box
}

tq_status tc_encode(const tq_quantizer *q, const void *x, int64_t n, int64_t ldx, const int32_t *chan,
                    int64_t chan_rows, void *codes, void *signs, float *norms, int64_t out_stride,
                    cudaStream_t st) {
  EncTCParams prm{};
  prm.n = n;
  prm.rot16 = q->d_rot16;
  prm.s16 = q->d_qjl16;
  prm.rho = q->tc_rho;
  for (int i = 0; i < kMaxLevels; ++i) {
    prm.thr_s[i] = q->kt.thresholds[i] * kRScale;
    prm.cen_s[i] = q->kt.centroids[i] * kRScale;
  }
  prm.chan = chan;
  prm.chan_rows = chan_rows;
  prm.codes = static_cast<uint32_t *>(codes);
  prm.signs = static_cast<uint32_t *>(signs);
  prm.norms = reinterpret_cast<float2 *>(norms);
  prm.out_stride = out_stride;
  prm.err = q->d_err;
  const bool gather = chan != nullptr;
  switch (q->d) {
    case 32: return dispatch_w<32>(q, x, n, ldx, gather, prm, st);
    case 64: return dispatch_w<64>(q, x, n, ldx, gather, prm, st);
    case 96: return dispatch_w<96>(q, x, n, ldx, gather, prm, st);
    case 128: return dispatch_w<128>(q, x, n, ldx, gather, prm, st);
  }
  return TQ_ERR_UNSUPPORTED;
}

}  // namespace tq

namespace tq {

// ============================================================================
// Encode for bf16 keys with the Hadamard rotation, reading the TMA tile as
// the MMA's A operand directly (no conversion on the CUDA cores).
//
//   d^1.5 R = K is an integer matrix; K = K_hi + K_lo with both pieces exact
//   in bf16, so U = X K^T takes two bf16 MMA passes and is exact up to fp32
//   accumulation.  R is orthogonal, so ||x|| = ||U|| / d^1.5 and
//   u = U / ||U||: the norm comes from the rotated row.
//
// 128 * (d/32) threads; thread (row, p) owns columns [32p, 32p+32) of one
// row.  Per-row partial sums (||U||^2, gamma^2) go through shared memory.
// The QJL operand [r_hi | r_lo] is written to TMEM and read from there by
// the MMA (only S comes from shared memory).  The rotation of tile t+1 is
// issued before the residuals of tile t are computed (U is double-buffered
// in TMEM), and the sign bits of tile t-1 are read while the QJL projection
// of tile t is being prepared.
// ============================================================================
namespace {

// Codes arrive as the bit patterns of the floats 2^23 + code.  Adding each
// pattern shifted to the code's place and subtracting, per word, what the
// 2^23 parts sum to (mod 2^32) leaves exactly the codes: one integer
// multiply-add per code.  With W = 3 the codes of coordinates 24..31 are
// spread over the fourth bit of every nibble; they are gathered as nibbles
// first and distributed at the end.
template <int W>
__host__ __device__ constexpr uint32_t raw_offset(int word) {
  uint32_t k = 0;
  for (int i = 0; i < (W == 3 ? 24 : 32); ++i) {
    const int p0 = code_bit_pos<W>(i, 0);
    if ((p0 >> 5) == word) k += 0x4B000000u << (p0 & 31);
  }
  return k;
}
__host__ __device__ constexpr uint32_t raw_tail_offset() {
  uint32_t k = 0;
  for (int i = 0; i < 8; ++i) k += 0x4B000000u << (4 * i);
  return k;
}

template <int W>
struct RawPack {
  uint32_t w[W], tail;
  __device__ __forceinline__ RawPack() : tail(0u) {
#pragma unroll
    for (int k = 0; k < W; ++k) w[k] = 0u;
  }
  __device__ __forceinline__ void add(int i, uint32_t raw) {  // i: coordinate in the group (unrolled)
    if (W == 3 && i >= 24) {
      tail += raw << (4 * (i - 24));
    } else {
      const int p0 = code_bit_pos<W>(i, 0);
      w[p0 >> 5] += raw << (p0 & 31);
    }
  }
  __device__ __forceinline__ void finish(uint32_t (&out)[W]) const {
#pragma unroll
    for (int k = 0; k < W; ++k) out[k] = w[k] - raw_offset<W>(k);
    if constexpr (W == 3) {
      const uint32_t t = tail - raw_tail_offset();
      out[0] |= (t & 0x44444444u) << 1;
      out[1] |= (t & 0x22222222u) << 2;
      out[2] |= (t & 0x11111111u) << 3;
    }
  }
};

// d = a * b + c on two lanes, rounded down
__device__ __forceinline__ float2 ffma2_rm(float2 a, float2 b, float2 c) {
  uint64_t r;
  asm("fma.rm.f32x2 %0, %1, %2, %3;"
      : "=l"(r)
      : "l"(*reinterpret_cast<const uint64_t *>(&a)), "l"(*reinterpret_cast<const uint64_t *>(&b)),
        "l"(*reinterpret_cast<const uint64_t *>(&c)));
  return *reinterpret_cast<const float2 *>(&r);
}

template <int D>
struct Enc2Smem {
  static constexpr int kXBytes = kRows * D * 2;
  static constexpr int kOffX = 0;                            // 2 x tiles (TMA, 128-byte swizzle)
  static constexpr int kOffBr = 2 * kXBytes;                 // K_hi, K_lo bf16
  static constexpr int kOffBs = kOffBr + 2 * D * D * 2;      // S fp16
  static constexpr int kOffPart = kOffBs + D * D * 2;        // per-row partial sums, fp32 [2][2][128][4]
  static constexpr int kOffMisc = kOffPart + 2 * 2 * kRows * 4 * 4;
  static constexpr int kTotal = kOffMisc + 128 + 1024;
};

}  // namespace

template <int D, int W, bool QJL>
// 17 warps (9 for d = 64): with five warps on one SM sub-partition and 16K
// registers each, at most 96 registers per thread (d = 128)
__global__ void __launch_bounds__(128 * (D / 32) + 32, 1)
k_encode_tc2(const __grid_constant__ CUtensorMap xmap, const EncTCParams p) {
  constexpr int P = D / 32;
  constexpr int L = 1 << W;
  constexpr int HALF = L / 2;
  constexpr int NB = D / 64;  // TMA boxes of 64 columns
  constexpr int kCompute = 128 * P;  // compute threads; one more warp issues the copies and MMAs
  constexpr uint32_t kColU0 = 0, kColZ = 256, kColA = 384;  // U double buffer, QJL accumulator, QJL A operand
  using SM = Enc2Smem<D>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t *sX = smem + SM::kOffX;
  uint8_t *sBr = smem + SM::kOffBr;
  uint8_t *sBs = smem + SM::kOffBs;
  float *sPart = reinterpret_cast<float *>(smem + SM::kOffPart);
  uint64_t *bars = reinterpret_cast<uint64_t *>(smem + SM::kOffMisc);  // full[2], rot, qjl, drain
  uint32_t *sTmem = reinterpret_cast<uint32_t *>(bars + 5);

  const int tid = threadIdx.x;
  const bool compute = tid < kCompute;
  // The control thread (lane 0 of the last warp) issues every TMA load and
  // tcgen05 MMA: an issuing thread waits on the tensor core's queue for
  // about the MMA's execution time, which would stall a computing warp.
  const bool ctl = tid == kCompute;
  const int row = tid & (kRows - 1);
  const int pc = tid >> 7;  // column group (compute threads)
  const uint32_t lane = (uint32_t)(row & ~31) << 16;

  if (tid == 0) {
    for (int i = 0; i < 5; ++i) sm100::mbar_init(&bars[i], 1);
    sm100::fence_barrier_init();
    sm100::prefetch_tmap(&xmap);
  }
  if (tid < 32) {
    sm100::tmem_alloc(sTmem, 512);
    sm100::tmem_relinquish();
  }
  sm100::stage_kmajor<D>(sBr, p.rot16, D);
  sm100::stage_kmajor<D>(sBr + D * D * 2, p.rot16 + (size_t)D * D, D);
  if constexpr (QJL) {
    if (p.s_otf)
      generate_kmajor_qjl<D>(sBs, p.s_key);  // S from the seed (TurboQuant article 2.3.2)
    else
      sm100::stage_kmajor<D>(sBs, p.s16, D);
  }
  sm100::fence_proxy_async();
  sm100::tc_fence_before();
  __syncthreads();
  sm100::tc_fence_after();
  const uint32_t tmem = *sTmem;

  // Symmetric codebook (scaled 2^10): magnitude thresholds T_k, k = 1..HALF-1,
  // and centroid magnitudes C_k.  Each threshold test is the exact step
  // sat(2^40 (|u| - T_k)): the product |u| 2^40 is exact and fp32 values
  // that differ do so by far more than 2^-40, so the step is exactly 0 or 1.
  constexpr float kBig = 1099511627776.0f;  // 2^40
  float nTB[HALF], ndC[HALF];  // -T_k 2^40, minus the centroid steps
#pragma unroll
  for (int k = 0; k < HALF; ++k) {
    nTB[k] = -p.thr_s[HALF - 1 + k] * kBig;
    ndC[k] = -(k == 0 ? p.cen_s[HALF] : p.cen_s[HALF + k] - p.cen_s[HALF + k - 1]);
  }

  const uint32_t idesc_rot = sm100::idesc_bf16_f32(kRows, D);
  const uint32_t idesc_qjl = sm100::idesc_f16_f32(kRows, D);
  const int first = blockIdx.x, stride = gridDim.x;
  const int nloc = first < p.ntiles ? (p.ntiles - first + stride - 1) / stride : 0;

  auto issue_rot = [&](int buf, uint32_t ucol) {
    const uint32_t xa = sm100::smem_u32(sX + buf * SM::kXBytes), br = sm100::smem_u32(sBr);
#pragma unroll
    for (int piece = 0; piece < 2; ++piece)
#pragma unroll
      for (int ks = 0; ks < D / 16; ++ks) {
        const uint64_t a = sm100::desc_sw128(xa + (ks >> 2) * (kRows * 128) + (ks & 3) * 32);
        const uint64_t b = sm100::desc_sw64(br + piece * (D * D * 2) + (ks >> 1) * (D * 64) + (ks & 1) * 32);
        sm100::mma_f16(tmem + ucol, a, b, idesc_rot, (piece | ks) != 0);
      }
    sm100::mma_commit(&bars[2]);
  };
  // The QJL A operand is in TMEM, two fp16 per column: column group pc
  // holds r_hi of coordinates [32pc, 32pc+32) in its first 16 columns and
  // r_lo of the same coordinates in the last 16.  K-step ks = 4pc + h reads
  // columns [32pc + 8h, +8): coordinates 32pc + 16(h & 1) + [0, 16) of r_hi
  // (h < 2) or r_lo (h >= 2), against the same 16 columns of S.
  auto issue_qjl = [&]() {
    const uint32_t bs = sm100::smem_u32(sBs);
#pragma unroll
    for (int ks = 0; ks < 2 * D / 16; ++ks) {
      const int kk = 2 * (ks >> 2) + (ks & 1);
      const uint64_t b = sm100::desc_sw64(bs + (kk >> 1) * (D * 64) + (kk & 1) * 32);
      sm100::mma_f16_ts(tmem + kColZ, tmem + kColA + 8 * ks, b, idesc_qjl, ks != 0);
    }
    sm100::mma_commit(&bars[3]);
  };
  auto issue_tma = [&](int buf, int tile) {
    sm100::mbar_expect_tx(&bars[buf], SM::kXBytes);
#pragma unroll
    for (int bx = 0; bx < NB; ++bx)
      sm100::tma_load_2d(sX + buf * SM::kXBytes + bx * (kRows * 128), &xmap, bx * 64, tile * kRows, &bars[buf]);
  };
  // Per-row partial sums (one per column group) in shared memory,
  // double-buffered by tile parity: ||U||^2 parts, then gamma^2 parts.
  auto norm_part = [&](int par) { return sPart + (2 * par) * (kRows * 4) + row * 4; };
  auto gam_part = [&](int par) { return sPart + (2 * par + 1) * (kRows * 4) + row * 4; };
  auto row_partial = [&](uint32_t ucol, float *dst) {
    uint32_t u[32];
    sm100::tmem_ld32(tmem + lane + ucol + 32 * pc, u);
    sm100::tmem_wait_ld();
    float2 ss = make_float2(0.f, 0.f);
#pragma unroll
    for (int j = 0; j < 32; j += 2) {
      const float2 v = make_float2(__uint_as_float(u[j]), __uint_as_float(u[j + 1]));
      ss = __ffma2_rn(v, v, ss);
    }
    dst[pc] = ss.x + ss.y;
  };
  auto sum_parts = [&](const float *src) {
    const float4 q4 = *reinterpret_cast<const float4 *>(src);
    const float parts[4] = {q4.x, q4.y, q4.z, q4.w};
    float v = 0.f;
#pragma unroll
    for (int k = 0; k < P; ++k) v += parts[k];
    return v;
  };
  // bit j set where Z[j] >= 0 (four independent chains of eight sign bits)
  auto sign_bits = [](const uint32_t (&z)[32]) {
    uint32_t w8[4] = {0u, 0u, 0u, 0u};
#pragma unroll
    for (int j = 7; j >= 0; --j)
#pragma unroll
      for (int c = 0; c < 4; ++c) w8[c] = __funnelshift_l(z[8 * c + j], w8[c], 1);
    return ~(w8[0] | (w8[1] << 8) | (w8[2] << 16) | (w8[3] << 24));
  };
  auto sign_word = [&]() {
    uint32_t z[32];
    sm100::tmem_ld32(tmem + lane + kColZ + 32 * pc, z);
    sm100::tmem_wait_ld();
    return sign_bits(z);
  };

  // the control thread's bookkeeping of loads in flight
  bool pend_full[2] = {false, false};
  uint32_t ph_full[2] = {0u, 0u};
  uint32_t ph_rot = 0u, ph_qjl = 0u;
  bool failed = false;  // CTA-uniform: only ever set from a barrier vote
  bool ifail = false;   // the control thread's own failed wait, voted at the next barrier
  bool any_mma = false;

  // ---- prologue: tiles 0 and 1 loaded, rotation of tile 0, its norm parts
  if (nloc > 0) {
    if (ctl) {
      issue_tma(0, first);
      pend_full[0] = true;
      if (nloc > 1) {
        issue_tma(1, first + stride);
        pend_full[1] = true;
      }
      ifail = !sm100::mbar_wait(&bars[0], ph_full[0], p.err, 11);
      ph_full[0] ^= 1u;
      pend_full[0] = ifail;
      sm100::tc_fence_after();
      if (!ifail) {
        issue_rot(0, kColU0);
        any_mma = true;
      }
    }
    bool ok = true;
    if (compute) {
      ok = sm100::mbar_wait(&bars[2], ph_rot, p.err, 12);
      ph_rot ^= 1u;
      sm100::tc_fence_after();
      row_partial(kColU0, norm_part(0));
    }
    sm100::tc_fence_before();
    failed = __syncthreads_or(!ok || ifail) != 0;
    sm100::tc_fence_after();
    if (ctl && !failed) {
      if (nloc > 2) {
        issue_tma(0, first + 2 * stride);  // tile 0's rotation is done with buffer 0
        pend_full[0] = true;
      }
      if (nloc > 1) {
        ifail = !sm100::mbar_wait(&bars[1], ph_full[1], p.err, 13);
        ph_full[1] ^= 1u;
        pend_full[1] = ifail;
        sm100::tc_fence_after();
        if (!ifail) issue_rot(1, 128u);
      }
    }
  }

  float prev_norm = 0.f;
  int64_t prev_row = -1;
  const float2 base2 = make_float2(8388608.0f + (float)HALF, 8388608.0f + (float)HALF);
  // The compute warps and the issuing warp run separate copies of the tile
  // loop (each keeps only its own code in the instruction stream), meeting
  // once per tile at one named barrier that also votes on failures; both
  // copies take the same number of iterations because `failed` comes from
  // that vote.
  constexpr int kThreadsAll = kCompute + 32;
  int it = 0;
  if (compute) for (; it < nloc && !failed; ++it) {  // `failed` is CTA-uniform
    const int t = first + it * stride;
    const int par = it & 1;
    const uint32_t ucol = par ? 128u : 0u;
    const int64_t grow = (int64_t)t * kRows + row;
    bool ok = true;
    {
      // ---- (a) this tile's rotated row (its MMA completed before the last
      // barrier), loaded while the row's scale is computed
      uint32_t acc[32];
      sm100::tmem_ld32(tmem + lane + ucol + 32 * pc, acc);
      const float nacc = sqrtf(sum_parts(norm_part(par)));
      const float nrm = nacc * p.rho;
      const float s_v = nacc > 0.f ? kRScale / nacc : -0.0f;  // zero rows: u = -0 -> lower middle code
      const float2 sv2 = make_float2(s_v, s_v);
      sm100::tmem_wait_ld();
      RawPack<W> pk;
      uint32_t hi[16], lo[16];
      float2 g2 = make_float2(0.f, 0.f);
#pragma unroll
      for (int j = 0; j < 32; j += 2) {
        const float2 us = __fmul2_rn(make_float2(__uint_as_float(acc[j]), __uint_as_float(acc[j + 1])), sv2);
        // m + 1/2 (m = magnitude thresholds passed by |u|) and -c[code] magnitude
        float2 ncm = make_float2(ndC[0], ndC[0]), mh = make_float2(0.5f, 0.5f);
#pragma unroll
        for (int k = 1; k < HALF; ++k) {
          const float2 st = make_float2(__saturatef(__fmaf_rn(fabsf(us.x), kBig, nTB[k])),
                                        __saturatef(__fmaf_rn(fabsf(us.y), kBig, nTB[k])));
          ncm = __ffma2_rn(st, make_float2(ndC[k], ndC[k]), ncm);
          mh = __fadd2_rn(mh, st);
        }
        // s = +-1 from the sign bit (u = -0 takes the lower middle code); the
        // code is HALF - 1/2 + s (m + 1/2): 2^23 + HALF + s (m + 1/2) is
        // exactly 2^23 + code + 1/2 (never below 2^23), rounded down to
        // 2^23 + code
        const float2 sg = make_float2(__uint_as_float((__float_as_uint(us.x) & 0x80000000u) | 0x3F800000u),
                                      __uint_as_float((__float_as_uint(us.y) & 0x80000000u) | 0x3F800000u));
        const float2 codef = ffma2_rm(sg, mh, base2);
        const float2 rr = __ffma2_rn(sg, ncm, us);  // u - c[code]
        pk.add(j, __float_as_uint(codef.x));
        pk.add(j + 1, __float_as_uint(codef.y));
        g2 = __ffma2_rn(rr, rr, g2);
        if constexpr (QJL) {
          const __half2 h = __floats2half2_rn(rr.x, rr.y);
          const float2 hf = __half22float2(h);
          hi[j / 2] = *reinterpret_cast<const uint32_t *>(&h);
          const float2 lf = __fadd2_rn(rr, make_float2(-hf.x, -hf.y));
          lo[j / 2] = pack_half2(lf.x, lf.y);
        }
      }
      uint32_t cw[W];
      pk.finish(cw);
      if (grow < p.n) {
        uint32_t *dst = p.codes + grow * p.out_stride * (W * D / 32) + pc * W;
#pragma unroll
        for (int k = 0; k < W; ++k) dst[k] = cw[k];
      }
      if constexpr (!QJL) {
        // TurboQuant-MSE: no sign bits; the norms of the previous tile
        if (it > 0) {
          const float gam = pc == 0 ? sqrtf(sum_parts(gam_part(par ^ 1))) * (1.0f / kRScale) : 0.f;
          if (pc == 0 && prev_row >= 0 && prev_row < p.n) p.norms[prev_row * p.out_stride] = make_float2(prev_norm, gam);
        }
      }
      // ---- (b) the previous tile's projection is done: its Z is final and
      // the residual operand is free
      if (QJL && it > 0) {
        ok = sm100::mbar_wait(&bars[3], ph_qjl, p.err, 14);
        ph_qjl ^= 1u;
        sm100::tc_fence_after();
      }
      // ---- (c) residual operand into TMEM
      if constexpr (QJL) {
        uint32_t a32[32];
#pragma unroll
        for (int k = 0; k < 16; ++k) {
          a32[k] = hi[k];
          a32[16 + k] = lo[k];
        }
        sm100::tmem_st32(tmem + lane + kColA + 32 * pc, a32);
      }
      // ---- (d) once the next tile's rotation is done (the tensor core no
      // longer writes TMEM, so the loads are quick): Z of the previous tile
      // for its sign bits and norms, then the next tile's U for its norm
      // parts (TMEM loads are warp-collective: every lane runs them, only
      // stores are guarded)
      if (it + 1 < nloc) {
        ok = sm100::mbar_wait(&bars[2], ph_rot, p.err, 15) && ok;
        ph_rot ^= 1u;
        sm100::tc_fence_after();
      }
      if (QJL && it > 0) {
        uint32_t z[32];
        sm100::tmem_ld32(tmem + lane + kColZ + 32 * pc, z);
        const float gam = pc == 0 ? sqrtf(sum_parts(gam_part(par ^ 1))) * (1.0f / kRScale) : 0.f;
        sm100::tmem_wait_ld();
        const uint32_t sw = sign_bits(z);
        if (prev_row >= 0 && prev_row < p.n) {
          p.signs[prev_row * p.out_stride * (D / 32) + pc] = sw;
          if (pc == 0) p.norms[prev_row * p.out_stride] = make_float2(prev_norm, gam);
        }
      }
      if (it + 1 < nloc) row_partial(ucol ^ 128u, norm_part(par ^ 1));
      gam_part(par)[pc] = g2.x + g2.y;
      if constexpr (QJL) sm100::tmem_wait_st();
      prev_norm = nrm;
      prev_row = grow;
    }
    sm100::tc_fence_before();
    failed = sm100::named_barrier_or(1, kThreadsAll, !ok);
    if (failed) break;
  }
  else for (; it < nloc && !failed; ++it) {
    const int par = it & 1;
    const uint32_t ucol = par ? 128u : 0u;
    failed = sm100::named_barrier_or(1, kThreadsAll, ifail);
    if (failed) break;
    // ---- (e) control thread: QJL projection of this tile, then the rotation two tiles ahead
    if (ctl) {
      sm100::tc_fence_after();
      if constexpr (QJL) issue_qjl();
      if (it + 3 < nloc) {  // tile it+1's rotation is done with its buffer
        issue_tma(par ^ 1, first + (it + 3) * stride);
        pend_full[par ^ 1] = true;
      }
      if (it + 2 < nloc) {
        ifail = !sm100::mbar_wait(&bars[par], ph_full[par], p.err, 17);
        ph_full[par] ^= 1u;
        pend_full[par] = ifail;
        sm100::tc_fence_after();
        if (!ifail) issue_rot(par, ucol);  // U of this tile has been read
      }
    }
  }

  // ---- drain: sign bits and norms of the last tile
  failed = __syncthreads_or(failed || ifail) != 0;
  if (!failed && it > 0) {
    const bool ok =
        __syncthreads_and(compute && QJL ? sm100::mbar_wait(&bars[3], ph_qjl, p.err, 18) : true) != 0;
    sm100::tc_fence_after();
    if (ok && compute) {
      const uint32_t sw = QJL ? sign_word() : 0u;
      const float gam = pc == 0 ? sqrtf(sum_parts(gam_part((it - 1) & 1))) * (1.0f / kRScale) : 0.f;
      if (prev_row >= 0 && prev_row < p.n) {
        if (QJL) p.signs[prev_row * p.out_stride * (D / 32) + pc] = sw;
        if (pc == 0) p.norms[prev_row * p.out_stride] = make_float2(prev_norm, gam);
      }
    }
  }
  if (failed && ctl) {
    for (int b = 0; b < 2; ++b)
      if (pend_full[b]) sm100::mbar_wait(&bars[b], ph_full[b], p.err, 16);
    if (any_mma) {
      // MMAs issued may still run: wait (bounded) before TMEM is freed
      sm100::mma_commit(&bars[4]);
      sm100::mbar_wait(&bars[4], 0u, p.err, 19);
    }
  }
  sm100::tc_fence_before();
  __syncthreads();
  if (tid < 32) sm100::tmem_dealloc(tmem, 512);
}

// ============================================================================
// Encode of bf16 keys whose coordinates are gathered through a per-group
// channel map (the 3.5- and 2.5-bit outlier splits of the KV cache,
// TurboQuant article 4.1.1), d in {32, 64, 96}, Hadamard or Haar rotation.
// The structure of k_encode_tc2 (16-coordinate-group compute warps, a
// control warp issuing every TMA load and MMA, U double-buffered in TMEM,
// the rotation two tiles ahead), with one more step: the compute threads
// gather a tile's channels from the raw TMA tile into the rotation's A
// operand (bf16, exact), two tiles ahead of its rotation.  The rotation's B
// operand is RP exact bf16 pieces: d^1.5 R (an integer matrix, two pieces)
// for Hadamard, the fp32 Haar matrix (three pieces) for Haar.
// ============================================================================
namespace {

template <int D, int RP, int SRCW>
struct EncGSmem {
  static constexpr int kXBytes = kRows * SRCW * 2;           // the raw bf16 tile (TMA, 128-byte swizzle)
  static constexpr int kAxBytes = kRows * D * 2;             // one gathered A operand (64-byte swizzle)
  static constexpr int kOffX = 0;
  static constexpr int kOffAx = kOffX + kXBytes;             // two of them
  static constexpr int kOffBr = kOffAx + 2 * kAxBytes;       // RP rotation pieces, bf16
  static constexpr int kOffBs = kOffBr + RP * D * D * 2;     // S fp16
  static constexpr int kOffPart = kOffBs + D * D * 2;        // per-row partial sums, fp32 [2][2][128][4]
  static constexpr int kOffMisc = kOffPart + 2 * 2 * kRows * 4 * 4;
  static constexpr int kTotal = kOffMisc + 128 + 1024;
};

}  // namespace

template <int D, int W, int RP, int SRCW>
// d = 32: two CTAs per SM (one warp group each, 128 TMEM columns, under half
// the shared memory), so that one CTA's waits overlap the other's work
__global__ void __launch_bounds__(128 * (D / 32) + 32, D == 32 ? 2 : 1)
k_encode_tcg(const __grid_constant__ CUtensorMap xmap, const EncTCParams p) {
  constexpr int P = D / 32;
  constexpr int L = 1 << W;
  constexpr int HALF = L / 2;
  constexpr int NB = SRCW / 64;      // TMA boxes of 64 columns
  constexpr int kCompute = 128 * P;  // compute threads; one more warp issues the copies and MMAs
  // TMEM: U double buffer, QJL accumulator, QJL A operand, kColStep columns apart
  constexpr uint32_t kColStep = D == 32 ? 32u : 128u, kTmemCols = D == 32 ? 128u : 512u;
  constexpr uint32_t kColU0 = 0, kColU1 = kColStep, kColZ = 2 * kColStep, kColA = 3 * kColStep;
  using SM = EncGSmem<D, RP, SRCW>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t *sX = smem + SM::kOffX;
  uint8_t *sAx = smem + SM::kOffAx;
  uint8_t *sBr = smem + SM::kOffBr;
  uint8_t *sBs = smem + SM::kOffBs;
  float *sPart = reinterpret_cast<float *>(smem + SM::kOffPart);
  uint64_t *bars = reinterpret_cast<uint64_t *>(smem + SM::kOffMisc);  // full, rot, qjl, drain
  uint32_t *sTmem = reinterpret_cast<uint32_t *>(bars + 4);

  const int tid = threadIdx.x;
  const bool compute = tid < kCompute;
  const bool ctl = tid == kCompute;
  const int row = tid & (kRows - 1);
  const int pc = tid >> 7;
  const uint32_t lane = (uint32_t)(row & ~31) << 16;

  if (tid == 0) {
    for (int i = 0; i < 4; ++i) sm100::mbar_init(&bars[i], 1);
    sm100::fence_barrier_init();
    sm100::prefetch_tmap(&xmap);
  }
  if (tid < 32) {
    sm100::tmem_alloc(sTmem, kTmemCols);
    sm100::tmem_relinquish();
  }
#pragma unroll
  for (int k = 0; k < RP; ++k) sm100::stage_kmajor<D>(sBr + k * (D * D * 2), p.rot16 + (size_t)k * D * D, D);
  sm100::stage_kmajor<D>(sBs, p.s16, D);
  sm100::fence_proxy_async();
  sm100::tc_fence_before();
  __syncthreads();
  sm100::tc_fence_after();
  const uint32_t tmem = *sTmem;

  constexpr float kBig = 1099511627776.0f;  // 2^40: exact steps sat(2^40 (|u| - T_k))
  float nTB[HALF], ndC[HALF];
#pragma unroll
  for (int k = 0; k < HALF; ++k) {
    nTB[k] = -p.thr_s[HALF - 1 + k] * kBig;
    ndC[k] = -(k == 0 ? p.cen_s[HALF] : p.cen_s[HALF + k] - p.cen_s[HALF + k - 1]);
  }
  const uint32_t idesc_rot = sm100::idesc_bf16_f32(kRows, D);
  const uint32_t idesc_qjl = sm100::idesc_f16_f32(kRows, D);
  const int first = blockIdx.x, stride = gridDim.x;
  const int nloc = first < p.ntiles ? (p.ntiles - first + stride - 1) / stride : 0;

  auto issue_tma = [&](int tile, int &count) {
    sm100::mbar_expect_tx(&bars[0], SM::kXBytes);
#pragma unroll
    for (int bx = 0; bx < NB; ++bx)
      sm100::tma_load_2d(sX + bx * (kRows * 128), &xmap, bx * 64, tile * kRows, &bars[0]);
    ++count;
  };
  auto issue_rot = [&](int abuf, uint32_t ucol) {
    const uint32_t xa = sm100::smem_u32(sAx + abuf * SM::kAxBytes), br = sm100::smem_u32(sBr);
#pragma unroll
    for (int piece = 0; piece < RP; ++piece)
#pragma unroll
      for (int ks = 0; ks < D / 16; ++ks) {
        const uint64_t a = sm100::desc_sw64(xa + (ks >> 1) * (kRows * 64) + (ks & 1) * 32);
        const uint64_t b = sm100::desc_sw64(br + piece * (D * D * 2) + (ks >> 1) * (D * 64) + (ks & 1) * 32);
        sm100::mma_f16(tmem + ucol, a, b, idesc_rot, (piece | ks) != 0);
      }
    sm100::mma_commit(&bars[1]);
  };
  // The QJL A operand in TMEM, laid out as in k_encode_tc2.
  auto issue_qjl = [&]() {
    const uint32_t bs = sm100::smem_u32(sBs);
#pragma unroll
    for (int ks = 0; ks < 2 * D / 16; ++ks) {
      const int kk = 2 * (ks >> 2) + (ks & 1);
      const uint64_t b = sm100::desc_sw64(bs + (kk >> 1) * (D * 64) + (kk & 1) * 32);
      sm100::mma_f16_ts(tmem + kColZ, tmem + kColA + 8 * ks, b, idesc_qjl, ks != 0);
    }
    sm100::mma_commit(&bars[2]);
  };
  // gather this thread's 32 channels of tile `tile` from the raw tile into A operand `abuf`
  auto gather = [&](int tile, int abuf) {
    const int64_t grow = (int64_t)tile * kRows + row;
    const int32_t *ch = p.chan + (grow < p.n ? grow / p.chan_rows : 0) * D + 32 * pc;
    uint32_t w[16];
#pragma unroll
    for (int j = 0; j < 32; j += 2) {
      // masked to the staged tile: a channel index cannot address beyond it
      const int s0 = __ldg(ch + j) & (SRCW - 1), s1 = __ldg(ch + j + 1) & (SRCW - 1);
      const uint32_t h0 = *reinterpret_cast<const uint16_t *>(sX + (s0 / 64) * (kRows * 128) +
                                                              sm100::sw128_offset(row, (s0 % 64) / 8) + (s0 % 8) * 2);
      const uint32_t h1 = *reinterpret_cast<const uint16_t *>(sX + (s1 / 64) * (kRows * 128) +
                                                              sm100::sw128_offset(row, (s1 % 64) / 8) + (s1 % 8) * 2);
      w[j / 2] = h0 | (h1 << 16);
    }
    uint8_t *dst = sAx + abuf * SM::kAxBytes + pc * (kRows * 64);
#pragma unroll
    for (int k = 0; k < 4; ++k)
      *reinterpret_cast<uint4 *>(dst + sm100::sw64_offset(row, k)) =
          make_uint4(w[4 * k], w[4 * k + 1], w[4 * k + 2], w[4 * k + 3]);
    sm100::fence_proxy_async();
  };
  auto norm_part = [&](int par) { return sPart + (2 * par) * (kRows * 4) + row * 4; };
  auto gam_part = [&](int par) { return sPart + (2 * par + 1) * (kRows * 4) + row * 4; };
  auto row_partial = [&](uint32_t ucol, float *dst) {
    uint32_t u[32];
    sm100::tmem_ld32(tmem + lane + ucol + 32 * pc, u);
    sm100::tmem_wait_ld();
    float2 ss = make_float2(0.f, 0.f);
#pragma unroll
    for (int j = 0; j < 32; j += 2) {
      const float2 v = make_float2(__uint_as_float(u[j]), __uint_as_float(u[j + 1]));
      ss = __ffma2_rn(v, v, ss);
    }
    dst[pc] = ss.x + ss.y;
  };
  auto sum_parts = [&](const float *src) {
    const float4 q4 = *reinterpret_cast<const float4 *>(src);
    const float parts[4] = {q4.x, q4.y, q4.z, q4.w};
    float v = 0.f;
#pragma unroll
    for (int k = 0; k < P; ++k) v += parts[k];
    return v;
  };
  // bit j set where Z[j] >= 0 (four independent chains of eight sign bits)
  auto sign_bits = [](const uint32_t (&z)[32]) {
    uint32_t w8[4] = {0u, 0u, 0u, 0u};
#pragma unroll
    for (int j = 7; j >= 0; --j)
#pragma unroll
      for (int c = 0; c < 4; ++c) w8[c] = __funnelshift_l(z[8 * c + j], w8[c], 1);
    return ~(w8[0] | (w8[1] << 8) | (w8[2] << 16) | (w8[3] << 24));
  };
  auto sign_word = [&]() {
    uint32_t z[32];
    sm100::tmem_ld32(tmem + lane + kColZ + 32 * pc, z);
    sm100::tmem_wait_ld();
    return sign_bits(z);
  };

  uint32_t ph_full = 0u, ph_rot = 0u, ph_qjl = 0u;  // compute threads' phases
  bool pend_full = false;  // control thread: a raw-tile load in flight, the ntma-th
  int ntma = 0;
  bool failed = false;     // CTA-uniform: only ever set from a barrier vote
  bool ifail = false;
  bool any_mma = false;
  // compute threads: wait for raw tile `tile` and gather it into `abuf`
  auto wait_and_gather = [&](int tile, int abuf) {
    const bool ok = sm100::mbar_wait(&bars[0], ph_full, p.err, 61);
    ph_full ^= 1u;
    gather(tile, abuf);
    return ok;
  };

  // ---- prologue: tiles 0 and 1 gathered and rotated, the norm parts of tile 0
  if (nloc > 0) {
    if (ctl) {
      issue_tma(first, ntma);
      pend_full = true;
    }
    bool ok = compute ? wait_and_gather(first, 0) : true;
    failed = __syncthreads_or(!ok) != 0;
    if (!failed) {
      if (ctl) {
        pend_full = false;
        sm100::tc_fence_after();
        issue_rot(0, kColU0);
        any_mma = true;
        if (nloc > 1) {
          issue_tma(first + stride, ntma);
          pend_full = true;
        }
      }
      ok = (compute && nloc > 1) ? wait_and_gather(first + stride, 1) : true;
      failed = __syncthreads_or(!ok) != 0;
    }
    if (!failed) {
      if (ctl) {
        pend_full = false;
        sm100::tc_fence_after();
        if (nloc > 1) issue_rot(1, kColU1);
        if (nloc > 2) {
          issue_tma(first + 2 * stride, ntma);
          pend_full = true;
        }
      }
      ok = true;
      if (compute) {
        ok = sm100::mbar_wait(&bars[1], ph_rot, p.err, 62);
        ph_rot ^= 1u;
        sm100::tc_fence_after();
        row_partial(kColU0, norm_part(0));
      }
      sm100::tc_fence_before();
      failed = __syncthreads_or(!ok) != 0;
      sm100::tc_fence_after();
    }
  }

  float prev_norm = 0.f;
  int64_t prev_row = -1;
  const float2 base2 = make_float2(8388608.0f + (float)HALF, 8388608.0f + (float)HALF);
  int it = 0;
  for (; it < nloc && !failed; ++it) {
    const int t = first + it * stride;
    const int par = it & 1;
    const uint32_t ucol = par ? kColU1 : kColU0;
    const int64_t grow = (int64_t)t * kRows + row;
    bool ok = true;
    if (compute) {
      // ---- (a) codes and residual of this tile (U loaded while the scale is computed)
      uint32_t acc[32];
      sm100::tmem_ld32(tmem + lane + ucol + 32 * pc, acc);
      const float nacc = sqrtf(sum_parts(norm_part(par)));
      const float nrm = nacc * p.rho;
      const float s_v = nacc > 0.f ? kRScale / nacc : -0.0f;
      const float2 sv2 = make_float2(s_v, s_v);
      sm100::tmem_wait_ld();
      RawPack<W> pk;
      uint32_t hi[16], lo[16];
      float2 g2 = make_float2(0.f, 0.f);
#pragma unroll
      for (int j = 0; j < 32; j += 2) {
        const float2 us = __fmul2_rn(make_float2(__uint_as_float(acc[j]), __uint_as_float(acc[j + 1])), sv2);
        float2 ncm = make_float2(ndC[0], ndC[0]), mh = make_float2(0.5f, 0.5f);
#pragma unroll
        for (int k = 1; k < HALF; ++k) {
          const float2 st = make_float2(__saturatef(__fmaf_rn(fabsf(us.x), kBig, nTB[k])),
                                        __saturatef(__fmaf_rn(fabsf(us.y), kBig, nTB[k])));
          ncm = __ffma2_rn(st, make_float2(ndC[k], ndC[k]), ncm);
          mh = __fadd2_rn(mh, st);
        }
        const float2 sg = make_float2(__uint_as_float((__float_as_uint(us.x) & 0x80000000u) | 0x3F800000u),
                                      __uint_as_float((__float_as_uint(us.y) & 0x80000000u) | 0x3F800000u));
        const float2 codef = ffma2_rm(sg, mh, base2);
        const float2 rr = __ffma2_rn(sg, ncm, us);
        pk.add(j, __float_as_uint(codef.x));
        pk.add(j + 1, __float_as_uint(codef.y));
        g2 = __ffma2_rn(rr, rr, g2);
        const __half2 h = __floats2half2_rn(rr.x, rr.y);
        const float2 hf = __half22float2(h);
        hi[j / 2] = *reinterpret_cast<const uint32_t *>(&h);
        const float2 lf = __fadd2_rn(rr, make_float2(-hf.x, -hf.y));
        lo[j / 2] = pack_half2(lf.x, lf.y);
      }
      uint32_t cw[W];
      pk.finish(cw);
      if (grow < p.n) {
        uint32_t *dst = p.codes + grow * p.out_stride * (W * D / 32) + pc * W;
#pragma unroll
        for (int k = 0; k < W; ++k) dst[k] = cw[k];
      }
      // ---- (b) the previous tile's projection is done: its Z is final and
      // the residual operand is free
      if (it > 0) {
        ok = sm100::mbar_wait(&bars[2], ph_qjl, p.err, 63);
        ph_qjl ^= 1u;
        sm100::tc_fence_after();
      }
      // ---- (c) residual operand into TMEM
      {
        uint32_t a32[32];
#pragma unroll
        for (int k = 0; k < 16; ++k) {
          a32[k] = hi[k];
          a32[16 + k] = lo[k];
        }
        sm100::tmem_st32(tmem + lane + kColA + 32 * pc, a32);
      }
      // sign bits and norms of the previous tile
      if (it > 0) {
        uint32_t z[32];
        sm100::tmem_ld32(tmem + lane + kColZ + 32 * pc, z);
        const float gam = pc == 0 ? sqrtf(sum_parts(gam_part(par ^ 1))) * (1.0f / kRScale) : 0.f;
        sm100::tmem_wait_ld();
        const uint32_t sw = sign_bits(z);
        if (prev_row >= 0 && prev_row < p.n) {
          p.signs[prev_row * p.out_stride * (D / 32) + pc] = sw;
          if (pc == 0) p.norms[prev_row * p.out_stride] = make_float2(prev_norm, gam);
        }
      }
      // ---- (g) gather tile it+2 into this tile's A operand (its rotation is done)
      if (it + 2 < nloc) ok = wait_and_gather(first + (it + 2) * stride, par) && ok;
      // ---- (d) norm parts of the next tile, gamma parts of this one
      if (it + 1 < nloc) {
        ok = sm100::mbar_wait(&bars[1], ph_rot, p.err, 64) && ok;
        ph_rot ^= 1u;
        sm100::tc_fence_after();
        row_partial(par ? kColU0 : kColU1, norm_part(par ^ 1));
      }
      gam_part(par)[pc] = g2.x + g2.y;
      sm100::tmem_wait_st();
      prev_norm = nrm;
      prev_row = grow;
    }
    sm100::tc_fence_before();
    failed = __syncthreads_or(!ok || ifail) != 0;
    if (failed) break;
    // ---- (e) control thread: QJL of this tile, the next raw tile, the rotation two tiles ahead
    if (ctl) {
      sm100::tc_fence_after();
      issue_qjl();
      if (it + 2 < nloc) pend_full = false;  // consumed by the gather above
      if (it + 3 < nloc) {
        issue_tma(first + (it + 3) * stride, ntma);
        pend_full = true;
      }
      if (it + 2 < nloc) issue_rot(par, ucol);
    }
  }

  // ---- drain: sign bits and norms of the last tile
  failed = __syncthreads_or(failed || ifail) != 0;
  if (!failed && it > 0) {
    const bool ok = __syncthreads_and(compute ? sm100::mbar_wait(&bars[2], ph_qjl, p.err, 65) : true) != 0;
    sm100::tc_fence_after();
    if (ok && compute) {
      const uint32_t sw = sign_word();
      const float gam = pc == 0 ? sqrtf(sum_parts(gam_part((it - 1) & 1))) * (1.0f / kRScale) : 0.f;
      if (prev_row >= 0 && prev_row < p.n) {
        p.signs[prev_row * p.out_stride * (D / 32) + pc] = sw;
        if (pc == 0) p.norms[prev_row * p.out_stride] = make_float2(prev_norm, gam);
      }
    }
  }
  if (failed && ctl) {
    if (pend_full) sm100::mbar_wait(&bars[0], (uint32_t)((ntma - 1) & 1), p.err, 66);
    if (any_mma) {
      sm100::mma_commit(&bars[3]);
      sm100::mbar_wait(&bars[3], 0u, p.err, 67);
    }
  }
  sm100::tc_fence_before();
  __syncthreads();
  if (tid < 32) sm100::tmem_dealloc(tmem, kTmemCols);
}

namespace {
template <int D, int W, int RP>
tq_status launch_tcg(const void *x, int64_t n, int64_t ldx, const EncTCParams &prm, cudaStream_t st) {
  constexpr int SRCW = 128;
  auto enc = tensor_map_encoder();
  if (!enc) return TQ_ERR_CUDA;
  CUtensorMap map;
  cuuint64_t gdim[2] = {(cuuint64_t)ldx, (cuuint64_t)n};
  cuuint64_t gstride[1] = {(cuuint64_t)ldx * 2};
  cuuint32_t box[2] = {64, 128};
  cuuint32_t estr[2] = {1, 1};
  if (enc(&map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void *>(x), gdim, gstride, box, estr,
          CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
          CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
    return TQ_ERR_CUDA;
  int dev = 0, max_smem = 0, sms = 0;
  cudaGetDevice(&dev);
  cudaDeviceGetAttribute(&max_smem, cudaDevAttrMaxSharedMemoryPerBlockOptin, dev);
  cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  // d > 32: at least half the SM's shared memory, so that one CTA (which
  // takes all of TMEM) runs per SM; d = 32: two CTAs per SM
  const int per_sm = D == 32 ? 2 : 1;
  const int smem = D == 32 ? EncGSmem<D, RP, SRCW>::kTotal : std::max(EncGSmem<D, RP, SRCW>::kTotal, max_smem / 2 + 1024);
  if (smem > max_smem) return TQ_ERR_UNSUPPORTED;
  EncTCParams pp = prm;
  pp.ntiles = (int)((n + kRows - 1) / kRows);
  auto kern = k_encode_tcg<D, W, RP, SRCW>;
  if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, smem) != cudaSuccess)
    return TQ_ERR_CUDA;
  if (D == 32 && cudaFuncSetAttribute(kern, cudaFuncAttributePreferredSharedMemoryCarveout, 100) != cudaSuccess)
    return TQ_ERR_CUDA;
  kern<<<std::min(pp.ntiles, sms * per_sm), 128 * (D / 32) + 32, smem, st>>>(map, pp);
  return cudaGetLastError() == cudaSuccess ? TQ_OK : TQ_ERR_CUDA;
}

template <int D, int RP>
tq_status dispatch_tcg_w(const tq_quantizer *q, const void *x, int64_t n, int64_t ldx, const EncTCParams &prm,
                         cudaStream_t st) {
  switch (q->w) {
    case 1: return launch_tcg<D, 1, RP>(x, n, ldx, prm, st);
    case 2: return launch_tcg<D, 2, RP>(x, n, ldx, prm, st);
    case 3: return launch_tcg<D, 3, RP>(x, n, ldx, prm, st);
    case 4: return launch_tcg<D, 4, RP>(x, n, ldx, prm, st);
  }
  return TQ_ERR_UNSUPPORTED;
}
}  // namespace

bool tcg_encode_supported(const tq_quantizer *q, int dtype, int64_t ldx, bool gather) {
  if (dtype != TQ_BF16 || !gather || q->m != q->d || ldx != 128) return false;
  if (q->rotation == TQ_ROT_HADAMARD) return q->d_rot_bf16 && (q->d == 32 || q->d == 64);
  return q->d_rot_bf16x3 && (q->d == 32 || q->d == 64 || q->d == 96);
}

tq_status tcg_encode(const tq_quantizer *q, const void *x, int64_t n, int64_t ldx, const int32_t *chan,
                     int64_t chan_rows, void *codes, void *signs, float *norms, int64_t out_stride,
                     cudaStream_t st) {
  EncTCParams prm{};
  prm.n = n;
  const bool had = q->rotation == TQ_ROT_HADAMARD;
  prm.rot16 = had ? q->d_rot_bf16 : q->d_rot_bf16x3;
  prm.s16 = q->d_qjl16;
  prm.rho = had ? q->tc_rho : 1.0f;  // U = d^1.5 R x (Hadamard) or R x (Haar)
  for (int i = 0; i < kMaxLevels; ++i) {
    prm.thr_s[i] = q->kt.thresholds[i] * kRScale;
    prm.cen_s[i] = q->kt.centroids[i] * kRScale;
  }
  prm.chan = chan;
  prm.chan_rows = chan_rows;
  prm.codes = static_cast<uint32_t *>(codes);
  prm.signs = static_cast<uint32_t *>(signs);
  prm.norms = reinterpret_cast<float2 *>(norms);
  prm.out_stride = out_stride;
  prm.err = q->d_err;
  if (had) {
    if (q->d == 32) return dispatch_tcg_w<32, 2>(q, x, n, ldx, prm, st);
    if (q->d == 64) return dispatch_tcg_w<64, 2>(q, x, n, ldx, prm, st);
    return TQ_ERR_UNSUPPORTED;
  }
  switch (q->d) {
    case 32: return dispatch_tcg_w<32, 3>(q, x, n, ldx, prm, st);
    case 64: return dispatch_tcg_w<64, 3>(q, x, n, ldx, prm, st);
    case 96: return dispatch_tcg_w<96, 3>(q, x, n, ldx, prm, st);
  }
  return TQ_ERR_UNSUPPORTED;
}

namespace {
template <int D, int W, bool QJL>
tq_status launch_tc2(const void *x, int64_t n, int64_t ldx, const EncTCParams &prm, cudaStream_t st) {
  auto enc = tensor_map_encoder();
  if (!enc) return TQ_ERR_CUDA;
  CUtensorMap map;
  cuuint64_t gdim[2] = {(cuuint64_t)D, (cuuint64_t)n};
  cuuint64_t gstride[1] = {(cuuint64_t)ldx * 2};
  cuuint32_t box[2] = {64, 128};
  cuuint32_t estr[2] = {1, 1};
  if (enc(&map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void *>(x), gdim, gstride, box, estr,
          CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
          CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
    return TQ_ERR_CUDA;
  int dev = 0, max_smem = 0, sms = 0;
  cudaGetDevice(&dev);
  cudaDeviceGetAttribute(&max_smem, cudaDevAttrMaxSharedMemoryPerBlockOptin, dev);
  cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  constexpr int smem = Enc2Smem<D>::kTotal;
  if (smem > max_smem) return TQ_ERR_UNSUPPORTED;
  EncTCParams pp = prm;
  pp.ntiles = (int)((n + kRows - 1) / kRows);
  auto kern = k_encode_tc2<D, W, QJL>;
  if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, smem) != cudaSuccess)
    return TQ_ERR_CUDA;
  kern<<<std::min(pp.ntiles, sms), 128 * (D / 32) + 32, smem, st>>>(map, pp);
  return cudaGetLastError() == cudaSuccess ? TQ_OK : TQ_ERR_CUDA;
}
}  // namespace

bool tc2_encode_supported(const tq_quantizer *q, int dtype, bool gather) {
  return dtype == TQ_BF16 && !gather && q->d_rot_bf16 && (q->d == 64 || q->d == 128);
}

tq_status tc2_encode(const tq_quantizer *q, const void *x, int64_t n, int64_t ldx, void *codes, void *signs,
                     float *norms, int64_t out_stride, cudaStream_t st) {
  EncTCParams prm{};
  prm.n = n;
  prm.rot16 = q->d_rot_bf16;
  prm.s16 = q->d_qjl16;
  prm.s_key = q->kt.qjl_key;
  prm.s_otf = q->kt.qjl_otf;
  prm.rho = q->tc_rho;
  for (int i = 0; i < kMaxLevels; ++i) {
    prm.thr_s[i] = q->kt.thresholds[i] * kRScale;
    prm.cen_s[i] = q->kt.centroids[i] * kRScale;
  }
  prm.codes = static_cast<uint32_t *>(codes);
  prm.signs = static_cast<uint32_t *>(signs);
  prm.norms = reinterpret_cast<float2 *>(norms);
  prm.out_stride = out_stride;
  prm.err = q->d_err;
#define TQ_TC2(DD)                                                          \
  switch (q->w) {                                                           \
    case 1: return q->m ? launch_tc2<DD, 1, true>(x, n, ldx, prm, st)       \
                        : launch_tc2<DD, 1, false>(x, n, ldx, prm, st);     \
    case 2: return q->m ? launch_tc2<DD, 2, true>(x, n, ldx, prm, st)       \
                        : launch_tc2<DD, 2, false>(x, n, ldx, prm, st);     \
    case 3: return q->m ? launch_tc2<DD, 3, true>(x, n, ldx, prm, st)       \
                        : launch_tc2<DD, 3, false>(x, n, ldx, prm, st);     \
    case 4: return q->m ? launch_tc2<DD, 4, true>(x, n, ldx, prm, st)       \
                        : launch_tc2<DD, 4, false>(x, n, ldx, prm, st);     \
  }                                                                         \
  return TQ_ERR_UNSUPPORTED;
  if (q->d == 64) {
    TQ_TC2(64)
  }
  if (q->d == 128) {
    TQ_TC2(128)
  }
#undef TQ_TC2
  return TQ_ERR_UNSUPPORTED;
}

}  // namespace tq

// Encode of fp32 (or gathered) rows with the Hadamard rotation, d in
// {32, 64, 128}: the rotation on the CUDA cores, the QJL projection on the
// tensor cores.
//
//   one thread per row of a 128-row tile (one tile per CTA):
//   ALU  ||x||, three rounds of (+-1 diagonal, Walsh-Hadamard butterflies)
//        in fp32 registers (error about log2(d) 2^-24 of ||x||), code =
//        #{thresholds < u}, r = u - c[code], gamma; r * 2^10 as fp16 hi + lo
//        into the A operand [r_hi | r_lo] in shared memory
//   MMA  Z = [r_hi | r_lo] [S | S]^T (S is fp16-exact), fp32 in TMEM, issued
//        by one thread
//   ALU  sign bits of Z (thread = TMEM lane = row), norms
//
// Method: TurboQuant article 2.1.2 (three rounds of sign diagonal and
// Walsh-Hadamard transform), 1.2.2-1.2.3 (Lloyd-Max code, residual, QJL
// sign sketch), 4.2.1 (stored norm).
#include <cudaTypedefs.h>

#include "tq_common.cuh"
#include "tq_kernels.h"
#include "tq_sm100.cuh"

namespace tq {

namespace {

constexpr int kFRows = 128;
constexpr float kFScale = 1024.0f;  // residuals go to fp16 at 2^10 scale

template <int D>
struct FwhtTcSmem {
  static constexpr int kOffBs = 0;                       // S, fp16, 64-byte swizzled K-major
  static constexpr int kOffAr = kOffBs + D * D * 2;      // [r_hi | r_lo], fp16, 64-byte swizzled K-major
  static constexpr int kOffMisc = kOffAr + kFRows * 2 * D * 2;
  static constexpr int kTotal = kOffMisc + 64 + 1024;    // + alignment slack
};

__device__ __forceinline__ uint32_t pack_h2(float a, float b) {
  const __half2 h = __floats2half2_rn(a, b);
  return *reinterpret_cast<const uint32_t *>(&h);
}

template <int D, int W>
__global__ void __launch_bounds__(kFRows, 1)
k_encode_fwht_tc(KernelTables kt, RowSource src, int64_t n, const uint16_t *s16, uint32_t *codes, uint32_t *signs,
                 float2 *norms, int64_t out_stride, int *err) {
  constexpr int L = 1 << W;
  constexpr uint32_t kCols = D < 32 ? 32 : D;
  using SM = FwhtTcSmem<D>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t *sBs = smem + SM::kOffBs;
  uint8_t *sAr = smem + SM::kOffAr;
  uint64_t *bars = reinterpret_cast<uint64_t *>(smem + SM::kOffMisc);  // qjl, drain
  uint32_t *sTmem = reinterpret_cast<uint32_t *>(bars + 2);
  __shared__ float sC[kMaxLevels], sT[kMaxLevels];
  __shared__ uint32_t sDiag[3 * D / 32];

  const int tid = threadIdx.x;
  const int64_t grow = (int64_t)blockIdx.x * kFRows + tid;
  if (tid == 0) {
    sm100::mbar_init(&bars[0], 1);
    sm100::mbar_init(&bars[1], 1);
    sm100::fence_barrier_init();
  }
  if (tid < 32) {
    sm100::tmem_alloc(sTmem, kCols);
    sm100::tmem_relinquish();
  }
  if (tid < kMaxLevels) {
    sC[tid] = kt.centroids[tid];
    sT[tid] = kt.thresholds[tid];
  }
  if (tid < 3 * D / 32) sDiag[tid] = kt.diag_bits[tid];
  sm100::stage_kmajor<D>(sBs, s16, D);
  sm100::fence_proxy_async();
  sm100::tc_fence_before();
  __syncthreads();
  sm100::tc_fence_after();
  const uint32_t tZ = *sTmem;

  // ---- the row: norm, rotation, codes, residual
  float v[D];
#pragma unroll
  for (int j = 0; j < D; ++j) v[j] = grow < n ? src.at(grow, j) : 0.f;
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
  float g2 = 0.f;
#pragma unroll
  for (int g = 0; g < D / 32; ++g) {
    uint32_t cw[W];
#pragma unroll
    for (int k = 0; k < W; ++k) cw[k] = 0u;
#pragma unroll
    for (int i = 0; i < 32; ++i) {
      const int j = 32 * g + i;
      const float u = v[j] * inv;
      const int c = quantize<L>(u, sT);
      pack_code<W>(cw, i, (uint32_t)c);
      const float r = u - sC[c];
      v[j] = r * kFScale;
      g2 = fmaf(r, r, g2);
    }
    if (grow < n) {
#pragma unroll
      for (int k = 0; k < W; ++k) codes[grow * out_stride * (W * D / 32) + g * W + k] = cw[k];
    }
    // r -> fp16 hi + lo in the A operand, 8 coordinates per 16-byte chunk
#pragma unroll
    for (int q = 0; q < 4; ++q) {
      uint32_t hi[4], lo[4];
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        const float a = v[32 * g + 8 * q + 2 * e], b = v[32 * g + 8 * q + 2 * e + 1];
        const __half2 h = __floats2half2_rn(a, b);
        const float2 hf = __half22float2(h);
        hi[e] = *reinterpret_cast<const uint32_t *>(&h);
        lo[e] = pack_h2(a - hf.x, b - hf.y);
      }
      *reinterpret_cast<uint4 *>(sAr + g * (kFRows * 64) + sm100::sw64_offset(tid, q)) =
          make_uint4(hi[0], hi[1], hi[2], hi[3]);
      *reinterpret_cast<uint4 *>(sAr + (D / 32 + g) * (kFRows * 64) + sm100::sw64_offset(tid, q)) =
          make_uint4(lo[0], lo[1], lo[2], lo[3]);
    }
  }
  sm100::fence_proxy_async();
  sm100::tc_fence_before();
  __syncthreads();
  // ---- the QJL projection on the tensor cores
  if (tid == 0) {
    sm100::tc_fence_after();
    const uint32_t ar = sm100::smem_u32(sAr), bs = sm100::smem_u32(sBs);
    const uint32_t idesc = sm100::idesc_f16_f32(kFRows, D);
#pragma unroll
    for (int ks = 0; ks < 2 * D / 16; ++ks) {
      const int kk = ks % (D / 16);
      const uint64_t a = sm100::desc_sw64(ar + (ks >> 1) * (kFRows * 64) + (ks & 1) * 32);
      const uint64_t b = sm100::desc_sw64(bs + (kk >> 1) * (D * 64) + (kk & 1) * 32);
      sm100::mma_f16(tZ, a, b, idesc, ks != 0);
    }
    sm100::mma_commit(&bars[0]);
  }
  const bool ok = __syncthreads_and(sm100::mbar_wait(&bars[0], 0u, err, 41)) != 0;  // CTA-uniform
  sm100::tc_fence_after();
  if (ok) {
    const uint32_t lane = (uint32_t)(tid & ~31) << 16;
#pragma unroll
    for (int g = 0; g < D / 32; ++g) {
      uint32_t z[32];
      sm100::tmem_ld32(tZ + lane + 32 * g, z);
      sm100::tmem_wait_ld();
      uint32_t wbits = 0u;
#pragma unroll
      for (int j = 31; j >= 0; --j) wbits = __funnelshift_l(z[j], wbits, 1);
      if (grow < n) signs[grow * out_stride * (D / 32) + g] = ~wbits;
    }
    if (grow < n) norms[grow * out_stride] = make_float2(nrm, sqrtf(g2));
  } else if (tid == 0) {
    // the MMAs may still run: wait (bounded) before TMEM is freed
    sm100::mma_commit(&bars[1]);
    sm100::mbar_wait(&bars[1], 0u, err, 42);
  }
  sm100::tc_fence_before();
  __syncthreads();
  if (tid < 32) sm100::tmem_dealloc(tZ, kCols);
}

template <int D, int W>
tq_status launch_fwht_tc(const tq_quantizer *q, const RowSource &src, int64_t n, void *codes, void *signs,
                         float *norms, int64_t out_stride, cudaStream_t st) {
  constexpr int smem = FwhtTcSmem<D>::kTotal;
  auto kern = k_encode_fwht_tc<D, W>;
  if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, smem) != cudaSuccess)
    return TQ_ERR_CUDA;
  const int64_t tiles = (n + kFRows - 1) / kFRows;
  kern<<<(unsigned)tiles, kFRows, smem, st>>>(q->kt, src, n, q->d_qjl16, static_cast<uint32_t *>(codes),
                                              static_cast<uint32_t *>(signs), reinterpret_cast<float2 *>(norms),
                                              out_stride, q->d_err);
  return cudaGetLastError() == cudaSuccess ? TQ_OK : TQ_ERR_CUDA;
}

template <int D>
tq_status dispatch_fwht_tc(const tq_quantizer *q, const RowSource &src, int64_t n, void *codes, void *signs,
                           float *norms, int64_t out_stride, cudaStream_t st) {
  switch (q->w) {
    case 1: return launch_fwht_tc<D, 1>(q, src, n, codes, signs, norms, out_stride, st);
    case 2: return launch_fwht_tc<D, 2>(q, src, n, codes, signs, norms, out_stride, st);
    case 3: return launch_fwht_tc<D, 3>(q, src, n, codes, signs, norms, out_stride, st);
    case 4: return launch_fwht_tc<D, 4>(q, src, n, codes, signs, norms, out_stride, st);
  }
  return TQ_ERR_UNSUPPORTED;
}

}  // namespace

bool fwht_tc_encode_supported(const tq_quantizer *q) {
  return q->rotation == TQ_ROT_HADAMARD && q->m == q->d && q->d_qjl16 && (q->d == 32 || q->d == 64 || q->d == 128);
}

tq_status fwht_tc_encode(const tq_quantizer *q, const RowSource &src, int64_t n, void *codes, void *signs,
                         float *norms, int64_t out_stride, cudaStream_t st) {
  switch (q->d) {
    case 32: return dispatch_fwht_tc<32>(q, src, n, codes, signs, norms, out_stride, st);
    case 64: return dispatch_fwht_tc<64>(q, src, n, codes, signs, norms, out_stride, st);
    case 128: return dispatch_fwht_tc<128>(q, src, n, codes, signs, norms, out_stride, st);
  }
  return TQ_ERR_UNSUPPORTED;
}

}  // namespace tq

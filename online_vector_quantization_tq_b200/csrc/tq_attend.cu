// Attention over a quantized KV cache (TurboQuant article 4.1.1: keys and
// values of the cache are both quantized, TurboQuant-MSE for most heads;
// 4.1.2: values are dequantized for the attention product, fp16 on the
// critical path).  Given the keys' logits (the inner-product estimates of
// tq_score) and the values encoded by a TurboQuant-MSE quantizer, each query
// gets
//
//   o = sum_k softmax_k(scale * s) * v^_k,   v^_k = ||v_k|| R^T c[codes_k].
//
// The rotation is linear, so the sum is formed in the rotated domain,
// o~ = sum_k p_k ||v_k|| c[codes_k], and rotated back once per query.
//
// k_attend_split: one work item = (group, key range); a persistent CTA per SM
// walks items.  Four warps, thread = key of a 128-key tile:
//   pass 1  per query the largest scaled logit of the range, and the
//           largest value norm (the weights are scaled by its inverse so
//           that they fit fp16);
//   pass 2  per tile: weights w_qk = exp(scale s_qk - m_q) ||v_k|| / vmax
//           as fp16 into the A operand (row q, K-major); the value codes
//           expanded by byte tables (PRMT) into fp16 centroids, the B
//           operand (row k, MN-major: a key's d centroids contiguous);
//           one thread of a fifth warp issues the tcgen05 kind::f16 MMAs
//           (M = 128 query rows, N = d, K = 16 keys each) accumulating o~
//           in TMEM over the whole range; two operand buffers, so a tile
//           is expanded while the previous one is multiplied.
// The item's o~ rows, maxima and weight sums go to a workspace;
// k_attend_combine merges the ranges of a query (rescaling by exp(m - M))
// and applies R^T (the inverse randomized Hadamard transform).
#include <cuda_fp16.h>

#include <algorithm>

#include "tq_expand.cuh"
#include "tq_kernels.h"
#include "tq_sm100.cuh"

namespace tq {

namespace {

constexpr int kAttMaxG = 16;                 // queries per group (A rows used)
constexpr int kAttTile = 128;                // keys per tile
constexpr int kAttCompute = 128;             // compute threads
constexpr int kAttThreads = kAttCompute + 32;

struct AttendParams {
  int64_t G, kpg, key_base, nkeys;  // keys [key_base, key_base + nkeys) of every group
  int64_t split_keys;               // keys per work item (multiple of the tile)
  int64_t nsplit, nitems;
  const float *logits;  // row g*G + q, column j: key key_base + j of group g
  int64_t ldl;
  float scale;
  const uint32_t *vcodes;  // [groups*kpg][W*D/32]
  const float2 *vnorms;    // [groups*kpg]: (norm, -)
  uint32_t tlo[4], thi[4];  // low and high bytes of the fp16 centroids, four entries per word
  float *part_o;            // [nitems][G][D]
  float4 *part_st;          // [nitems][G]: (max, sum of exp, vmax, 0)
  int *err;
};

// Shared memory of one CTA (three fit on an SM): two operand buffers, each
//   A: the tile's dequantized values transposed, V^T (M = 128 coordinates,
//      K = 128 keys), MN-major: a key's coordinates contiguous; coordinates
//      beyond d (d = 64) stay zero;
//   B: the weights P^T (N = 16 query rows, K = 128 keys), K-major; rows >= G
//      stay zero.
struct AttSmem {
  static constexpr int kABytes = kAttTile * 128 * 2;
  static constexpr int kBBytes = kAttMaxG * kAttTile * 2;
  static constexpr int kOffA = 0;
  static constexpr int kOffB = 2 * kABytes;
  static constexpr int kOffRed = kOffB + 2 * kBBytes;  // float [4 warps][kAttMaxG + 1]
  static constexpr int kOffM = kOffRed + 4 * (kAttMaxG + 1) * 4;  // float [kAttMaxG]: the range's maxima
  static constexpr int kOffMisc = kOffM + kAttMaxG * 4;
  static constexpr int kTotal = kOffMisc + 64 + 1024;
};

__device__ __forceinline__ float warp_max(float v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, o));
  return v;
}
__device__ __forceinline__ float warp_sum(float v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  return v;
}

// byte offset of (row n, key k) in a K-major 128-byte-swizzled fp16 tile of
// kAttMaxG rows: keys in 64-key atom columns of kAttMaxG rows x 128 bytes
__device__ __forceinline__ uint32_t b_offset(int n, int k) {
  return (uint32_t)(k >> 6) * (kAttMaxG * 128u) + sm100::sw128_offset(n, (k & 63) >> 3) + (uint32_t)(k & 7) * 2u;
}

template <int D, int W, int MAXG>
__global__ void __launch_bounds__(kAttThreads, 3) k_attend_split(const AttendParams p) {
  using SM = AttSmem;
  constexpr int NG = D / 32;        // 32-coordinate code groups
  constexpr int CW = W * NG;        // code words per key
  constexpr uint32_t kLbo = (kAttTile / 8) * 1024;  // A: 64-coordinate blocks
  extern __shared__ uint8_t smem_raw[];
  uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t *sA = smem + SM::kOffA;
  uint8_t *sB = smem + SM::kOffB;
  float *sRed = reinterpret_cast<float *>(smem + SM::kOffRed);
  float *sM = reinterpret_cast<float *>(smem + SM::kOffM);
  uint64_t *bars = reinterpret_cast<uint64_t *>(smem + SM::kOffMisc);  // mma done [2], drain
  uint32_t *sTmem = reinterpret_cast<uint32_t *>(bars + 3);

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const bool compute = tid < kAttCompute;
  const bool ctl = tid == kAttCompute;
  const int G = (int)p.G;
  if (tid == 0) {
    for (int i = 0; i < 3; ++i) sm100::mbar_init(&bars[i], 1);
    sm100::fence_barrier_init();
  }
  if (warp == 4) {
    sm100::tmem_alloc(sTmem, 32);
    sm100::tmem_relinquish();
  }
  // all operand buffers zero: B rows >= G and A coordinates >= D are never written
  for (int i = tid; i < 2 * (SM::kABytes + SM::kBBytes) / 16; i += kAttThreads)
    reinterpret_cast<uint4 *>(sA)[i] = make_uint4(0u, 0u, 0u, 0u);
  sm100::fence_proxy_async();
  sm100::tc_fence_before();
  __syncthreads();
  sm100::tc_fence_after();
  const uint32_t tmem = *sTmem;
  const uint32_t idesc = sm100::idesc_f16_f32_amn(128, kAttMaxG);
  uint32_t tlo[4], thi[4];
#pragma unroll
  for (int k = 0; k < 4; ++k) {
    tlo[k] = p.tlo[k];
    thi[k] = p.thi[k];
  }

  int64_t T = 0;  // tiles started by this CTA (operand buffer T & 1, its phase T >> 1)
  bool failed = false;
  for (int64_t item = blockIdx.x; item < p.nitems && !failed; item += gridDim.x) {
    const int64_t g = item / p.nsplit, sp = item % p.nsplit;
    const int64_t k0 = sp * p.split_keys, k1 = min(k0 + p.split_keys, p.nkeys);
    const int ntile = (int)((k1 - k0 + kAttTile - 1) / kAttTile);
    const float *lg = p.logits + g * p.G * p.ldl;
    const int64_t vrow0 = g * p.kpg + p.key_base;
    // ---- pass 1: per-query maxima of the scaled logits, largest value norm
    float vmax = 0.f;
    if (compute) {
      float mq[MAXG];
#pragma unroll
      for (int q = 0; q < MAXG; ++q) mq[q] = -INFINITY;
#pragma unroll 4
      for (int64_t k = k0 + tid; k < k1; k += kAttCompute) {
#pragma unroll
        for (int q = 0; q < MAXG; ++q)
          if (q < G) mq[q] = fmaxf(mq[q], p.scale * __ldg(lg + q * p.ldl + k));
        vmax = fmaxf(vmax, __ldg(&p.vnorms[vrow0 + k].x));
      }
#pragma unroll
      for (int q = 0; q < MAXG; ++q)
        if (q < G) {
          const float m = warp_max(mq[q]);
          if (lane == 0) sRed[warp * (kAttMaxG + 1) + q] = m;
        }
      vmax = warp_max(vmax);
      if (lane == 0) sRed[warp * (kAttMaxG + 1) + kAttMaxG] = vmax;
    }
    __syncthreads();
    if (tid < G)
      sM[tid] = fmaxf(fmaxf(sRed[tid], sRed[(kAttMaxG + 1) + tid]),
                      fmaxf(sRed[2 * (kAttMaxG + 1) + tid], sRed[3 * (kAttMaxG + 1) + tid]));
    vmax = fmaxf(fmaxf(sRed[kAttMaxG], sRed[2 * kAttMaxG + 1]), fmaxf(sRed[3 * kAttMaxG + 2], sRed[4 * kAttMaxG + 3]));
    const float vinv = vmax > 0.f ? 1.0f / vmax : 0.f;
    float lq[MAXG];
#pragma unroll
    for (int q = 0; q < MAXG; ++q) lq[q] = 0.f;
    __syncthreads();  // sRed is read, sM is written

    // ---- pass 2: tiles; the next tile's value codes, norms and logits are
    // loaded while this one is expanded
    uint32_t cw[CW];
    float vn = 0.f, sl[MAXG];
    auto load_key = [&](int t, uint32_t (&c)[CW], float &n, float (&l)[MAXG]) {
      const int64_t k = k0 + (int64_t)t * kAttTile + tid;
#pragma unroll
      for (int i = 0; i < CW; ++i) c[i] = 0u;
      n = 0.f;
#pragma unroll
      for (int q = 0; q < MAXG; ++q) l[q] = 0.f;
      if (k < k1) {
        const uint32_t *crow = p.vcodes + (vrow0 + k) * CW;
#pragma unroll
        for (int i = 0; i < CW; ++i) c[i] = __ldg(crow + i);
        n = __ldg(&p.vnorms[vrow0 + k].x);
#pragma unroll
        for (int q = 0; q < MAXG; ++q)
          if (q < G) l[q] = __ldg(lg + q * p.ldl + k);
      }
    };
    if (compute) load_key(0, cw, vn, sl);
    for (int t = 0; t < ntile; ++t, ++T) {
      const int b = (int)(T & 1);
      bool ok = true;
      if (compute) {
        const int64_t k = k0 + (int64_t)t * kAttTile + tid;
        const bool valid = k < k1;
        uint32_t cwn[CW];
        float vnn = 0.f, sln[MAXG];
        if (t + 1 < ntile) load_key(t + 1, cwn, vnn, sln);
        // operand buffer b was last read by the MMAs of tile T - 2
        if (T >= 2) ok = sm100::mbar_wait(&bars[b], (uint32_t)(((T >> 1) - 1) & 1), p.err, 81);
        uint8_t *a = sA + b * SM::kABytes;
        uint8_t *bw = sB + b * SM::kBBytes;
#pragma unroll
        for (int q = 0; q < MAXG; ++q)
          if (q < G) {
            const float e = valid ? __expf(p.scale * sl[q] - sM[q]) : 0.f;
            lq[q] += e;
            *reinterpret_cast<__half *>(bw + b_offset(q, tid)) = __float2half_rn(e * vn * vinv);
          }
        // the key's d centroids, fp16: row `tid` of the MN-major A tile (8-key
        // groups 1024 B apart, 64-coordinate blocks kLbo apart)
        const uint32_t rowoff = (uint32_t)(tid >> 3) * 1024u + (uint32_t)(tid & 7) * 128u;
#pragma unroll
        for (int gi = 0; gi < NG; ++gi) {
          uint32_t lo[8], hi[8];
          expand_codes<W>(cw + gi * W, tlo, thi, lo, hi);
#pragma unroll
          for (int c4 = 0; c4 < 4; ++c4) {  // 8 coordinates per 16-byte chunk
            uint4 v;
            v.x = sm100::prmt(lo[2 * c4], hi[2 * c4], 0x5140u);
            v.y = sm100::prmt(lo[2 * c4], hi[2 * c4], 0x7362u);
            v.z = sm100::prmt(lo[2 * c4 + 1], hi[2 * c4 + 1], 0x5140u);
            v.w = sm100::prmt(lo[2 * c4 + 1], hi[2 * c4 + 1], 0x7362u);
            if (!valid) v = make_uint4(0u, 0u, 0u, 0u);
            const int j0 = 32 * gi + 8 * c4;  // first coordinate of the chunk
            const int chunk = (j0 & 63) >> 3;
            *reinterpret_cast<uint4 *>(a + (uint32_t)(j0 >> 6) * kLbo + rowoff +
                                       (uint32_t)((chunk ^ (tid & 7)) << 4)) = v;
          }
        }
        sm100::fence_proxy_async();
#pragma unroll
        for (int i = 0; i < CW; ++i) cw[i] = cwn[i];
#pragma unroll
        for (int q = 0; q < MAXG; ++q) sl[q] = sln[q];
        vn = vnn;
      }
      // operands complete: the issuing thread takes over (one vote per tile)
      failed = __syncthreads_or(!ok) != 0;
      if (failed) break;
      if (ctl) {
        sm100::tc_fence_after();
        const uint32_t a0 = sm100::smem_u32(sA + b * SM::kABytes), b0 = sm100::smem_u32(sB + b * SM::kBBytes);
#pragma unroll
        for (int ks = 0; ks < kAttTile / 16; ++ks) {
          const uint64_t da = sm100::desc_sw128_mn(a0 + ks * 2048, kLbo, 1024);
          const uint64_t db = sm100::desc_sw128(b0 + (ks >> 2) * (kAttMaxG * 128) + (ks & 3) * 32);
          sm100::mma_f16(tmem, da, db, idesc, (t | ks) != 0);
        }
        sm100::mma_commit(&bars[b]);
      }
    }
    if (failed) break;
    // ---- item result: wait for the last tile's MMAs; lane j of the
    // accumulator is coordinate j, column q is query q
    const int64_t Tl = T - 1;
    bool ok = true;
    if (compute) ok = sm100::mbar_wait(&bars[Tl & 1], (uint32_t)((Tl >> 1) & 1), p.err, 82);
    failed = __syncthreads_or(!ok) != 0;
    if (failed) break;
    sm100::tc_fence_after();
    if (compute) {
      uint32_t v[16];
      sm100::tmem_ld16(tmem + ((uint32_t)(32 * warp) << 16), v);
      sm100::tmem_wait_ld();
      if (tid < D) {
#pragma unroll
        for (int q = 0; q < MAXG; ++q)
          if (q < G) p.part_o[(item * p.G + q) * D + tid] = __uint_as_float(v[q]);
      }
#pragma unroll
      for (int q = 0; q < MAXG; ++q)
        if (q < G) {
          const float l = warp_sum(lq[q]);
          if (lane == 0) sRed[warp * (kAttMaxG + 1) + q] = l;
        }
    }
    sm100::tc_fence_before();
    __syncthreads();  // the accumulator is read (the next item's first MMA overwrites it); sums in sRed
    if (tid < G)
      p.part_st[item * p.G + tid] =
          make_float4(sM[tid], sRed[tid] + sRed[(kAttMaxG + 1) + tid] + sRed[2 * (kAttMaxG + 1) + tid] +
                                   sRed[3 * (kAttMaxG + 1) + tid],
                      vmax, 0.f);
    __syncthreads();
  }
  if (failed && ctl && T > 0) {
    // MMAs issued may still run: wait (bounded) before TMEM is freed
    sm100::mma_commit(&bars[2]);
    sm100::mbar_wait(&bars[2], 0u, p.err, 83);
  }
  sm100::tc_fence_before();
  __syncthreads();
  if (warp == 4) sm100::tmem_dealloc(tmem, 32);
}

// Merge the key ranges of one query and rotate back: one block of D threads.
template <int D>
__global__ void __launch_bounds__(D)
k_attend_combine(KernelTables kt, int64_t G, int64_t nsplit, const float *part_o, const float4 *part_st, float *out,
                 int64_t ldo) {
  __shared__ float v[D];
  const int64_t row = blockIdx.x;  // g * G + q
  const int64_t g = row / G, q = row % G;
  const int j = threadIdx.x;
  float M = -INFINITY;
  for (int64_t s = 0; s < nsplit; ++s) {
    const float4 st = part_st[(g * nsplit + s) * G + q];
    if (st.y > 0.f) M = fmaxf(M, st.x);
  }
  float L = 0.f, acc = 0.f;
  for (int64_t s = 0; s < nsplit; ++s) {
    const float4 st = part_st[(g * nsplit + s) * G + q];
    if (!(st.y > 0.f)) continue;
    const float f = __expf(st.x - M);
    L = fmaf(f, st.y, L);
    acc = fmaf(f * st.z, part_o[((g * nsplit + s) * G + q) * D + j], acc);
  }
  float x = L > 0.f ? acc / L : 0.f;
  // x = R^T o~ with R = H D3 H D2 H D1 / d^1.5: H, then D3, H, D2, H, D1
#pragma unroll
  for (int r = 2; r >= 0; --r) {
#pragma unroll
    for (int h = 1; h < D; h <<= 1) {
      float b;
      if (h < 32) {
        b = __shfl_xor_sync(0xffffffffu, x, h);
      } else {
        __syncthreads();
        v[j] = x;
        __syncthreads();
        b = v[j ^ h];
      }
      x = (j & h) ? b - x : x + b;
    }
    const uint32_t word = kt.diag_bits[r * (D / 32) + j / 32];
    x = ((word >> (j % 32)) & 1u) ? -x : x;
  }
  out[row * ldo + j] = x * (1.0f / (float(D) * sqrtf(float(D))));
}

int attend_nsplit(int64_t groups, int64_t nkeys, int sms, int64_t *split_keys) {
  // At least about two work items per resident CTA (three per SM), ranges of
  // at least four tiles; and ranges of at most 16 tiles, so that a range's
  // logits are still in L2 when its second pass reads them again.
  const int64_t want = std::max<int64_t>(1, (6 * (int64_t)sms + groups - 1) / groups);
  const int64_t by_len = std::max<int64_t>(1, (nkeys + 4 * kAttTile - 1) / (4 * kAttTile));
  const int64_t ns = std::max(std::min(want, by_len), (nkeys + 16 * kAttTile - 1) / (16 * kAttTile));
  const int64_t per = (nkeys + ns - 1) / ns;
  *split_keys = (per + kAttTile - 1) / kAttTile * kAttTile;
  return (int)((nkeys + *split_keys - 1) / *split_keys);
}

template <int D, int W>
tq_status launch_attend(const tq_quantizer *qv, AttendParams &prm, int64_t groups, float *out, int64_t ldo,
                        cudaStream_t st, int sms) {
  // up to four queries per group (the common grouped-query case): fewer
  // registers per thread, so the next tile's logits can be prefetched too
  auto kern = prm.G <= 4 ? k_attend_split<D, W, 4> : k_attend_split<D, W, kAttMaxG>;
  constexpr int smem = AttSmem::kTotal;
  if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, smem) != cudaSuccess)
    return TQ_ERR_CUDA;
  if (cudaFuncSetAttribute(kern, cudaFuncAttributePreferredSharedMemoryCarveout, 100) != cudaSuccess)
    return TQ_ERR_CUDA;
  kern<<<(unsigned)std::min<int64_t>(prm.nitems, 3 * (int64_t)sms), kAttThreads, smem, st>>>(prm);
  if (cudaGetLastError() != cudaSuccess) return TQ_ERR_CUDA;
  k_attend_combine<D><<<(unsigned)(groups * prm.G), D, 0, st>>>(qv->kt, prm.G, prm.nsplit, prm.part_o, prm.part_st,
                                                                 out, ldo);
  return cudaGetLastError() == cudaSuccess ? TQ_OK : TQ_ERR_CUDA;
}

template <int D>
tq_status dispatch_attend(const tq_quantizer *qv, AttendParams &prm, int64_t groups, float *out, int64_t ldo,
                          cudaStream_t st, int sms) {
  switch (qv->w) {
    case 2: return launch_attend<D, 2>(qv, prm, groups, out, ldo, st, sms);
    case 3: return launch_attend<D, 3>(qv, prm, groups, out, ldo, st, sms);
    case 4: return launch_attend<D, 4>(qv, prm, groups, out, ldo, st, sms);
  }
  return TQ_ERR_UNSUPPORTED;
}

int device_sms() {
  int dev = 0, sms = 0;
  cudaGetDevice(&dev);
  cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  return sms > 0 ? sms : 1;
}

}  // namespace

bool attend_supported(const tq_quantizer *qv) {
  return qv->m == 0 && qv->rotation == TQ_ROT_HADAMARD && (qv->d == 64 || qv->d == 128) && qv->w >= 2 &&
         qv->w <= 4;
}

size_t attend_ws_bytes(int64_t groups, int64_t G, int d, int64_t nkeys) {
  int64_t split = 0;
  const int64_t ns = attend_nsplit(groups, nkeys, device_sms(), &split);
  const int64_t items = groups * ns;
  return (size_t)items * G * (d * sizeof(float) + sizeof(float4)) + 256;
}

tq_status attend_launch(const tq_quantizer *qv, const float *logits, int64_t ldl, int64_t groups, int64_t G,
                        float scale, const void *vcodes, const float *vnorms, int64_t kpg, int64_t key_base,
                        int64_t nkeys, float *out, int64_t ldo, void *ws, size_t ws_bytes, cudaStream_t st) {
  if (G < 1 || G > kAttMaxG) return TQ_ERR_UNSUPPORTED;
  const int sms = device_sms();
  AttendParams prm{};
  prm.G = G;
  prm.kpg = kpg;
  prm.key_base = key_base;
  prm.nkeys = nkeys;
  prm.nsplit = attend_nsplit(groups, nkeys, sms, &prm.split_keys);
  prm.nitems = groups * prm.nsplit;
  const size_t need = (size_t)prm.nitems * G * (qv->d * sizeof(float) + sizeof(float4)) + 256;
  if (!ws || ws_bytes < need) return TQ_ERR_WORKSPACE;
  uint8_t *w8 = static_cast<uint8_t *>(ws);
  const uintptr_t base = (reinterpret_cast<uintptr_t>(w8) + 255) & ~uintptr_t(255);
  prm.part_st = reinterpret_cast<float4 *>(base);
  prm.part_o = reinterpret_cast<float *>(base + (size_t)prm.nitems * G * sizeof(float4));
  prm.logits = logits;
  prm.ldl = ldl;
  prm.scale = scale;
  prm.vcodes = static_cast<const uint32_t *>(vcodes);
  prm.vnorms = reinterpret_cast<const float2 *>(vnorms);
  for (int i = 0; i < 16; ++i) {
    const uint16_t h = i < (1 << qv->w) ? double_to_half_bits(qv->centroids[i]) : 0;
    prm.tlo[i / 4] |= (uint32_t)(h & 0xFF) << (8 * (i % 4));
    prm.thi[i / 4] |= (uint32_t)(h >> 8) << (8 * (i % 4));
  }
  prm.err = qv->d_err;
  if (qv->d == 64) return dispatch_attend<64>(qv, prm, groups, out, ldo, st, sms);
  return dispatch_attend<128>(qv, prm, groups, out, ldo, st, sms);
}

}  // namespace tq

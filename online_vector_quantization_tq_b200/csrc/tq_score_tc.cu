// Integer tensor-core scorer (d <= 128): one tcgen05 kind::i8 MMA chain per
// tile of 128 keys computes, for every query of the keys' group, the exact
// integer dot products the asymmetric estimator needs:
//
//   <y~, c[codes]>  with y~ and the centroids as 16-bit fixed point, each
//                   split into two signed bytes:  y = 256 yh + yl,
//                   c = 256 ch + cl,
//                   y.c = 65536 (yh.ch) + 256 (yl.ch + yh.cl) + yl.cl
//   <p, bits>       with p as 16-bit fixed point (two bytes) and the sign
//                   bits as 0/1 bytes; <p, 2 bits - 1> = 2 <p, bits> - sum p
//
// The key operand row [ch | cl | bits] (384 bytes) is expanded from the
// packed codes with byte-table lookups (PRMT selects bytes of a table held in
// registers, four codes per instruction); the query operand has five rows
// per query: [yh | 0 | 0], [yl | yh | 0], [0 | yl | 0], [0 | 0 | ph],
// [0 | 0 | pl].
// Accumulation is exact in int32; the epilogue forms
//   s = ||x|| (y.c * 2^-(sy+sc) + gamma sqrt(pi/2)/m (2 p.bits - sum p) 2^-sp)
// (TurboQuant blog 三-四: asymmetric estimator on packed keys; TurboQuant
// article 4.2.2: score against the stored codes without dequantizing).
#include "tq_common.cuh"
#include "tq_kernels.h"
#include "tq_sm100.cuh"

namespace tq {

constexpr int kScoreKBytes = 384;  // [ch 128 | cl 128 | bits 128] per key row
constexpr int kColsPerQuery = 5;   // hh, (lh + hl), ll, ph, pl
constexpr int kMaxScoreG = 48;     // 5 * 48 <= 256 = largest MMA N

struct ScoreTCParams {
  int d, m;
  int64_t G, kpg, key_base, nkeys;  // keys [key_base, key_base+nkeys) of every group
  int N;                            // MMA N = roundup(5G, 16)
  int64_t tiles_per_group, ntiles;
  const uint32_t *codes, *signs;
  const float2 *norms;
  const int8_t *qop;  // [groups][N][384]
  const float4 *qsc;  // [groups*G]: 2^-(sy+sc), 2^-sp * sqrt(pi/2)/m, sum P, 0
  uint32_t tch[4], tcl[4];  // centroid byte tables (entries 0..15)
  float *out;
  int64_t ldo;
  int accumulate;
  int *err;
};

// Byte position, inside a 32-coordinate group, of coordinate i of the codes
// (the order in which the PRMT expansion emits bytes) and of sign bit i.
__host__ __device__ constexpr int code_byte_pos(int w, int i) { return w == 1 ? 8 * (i % 4) + i / 4 : i; }
__host__ __device__ constexpr int sign_byte_pos(int i) { return 4 * (i % 8) + i / 8; }

// ------------------------------------------------------------------ query operand
__global__ void __launch_bounds__(128)
k_query_operand(const float *ytil, const float *p, int d, int m, int w, int64_t G, int N, int cexp,
                float qjl_scale, int8_t *qop, float4 *qsc) {
  const int64_t qrow = blockIdx.x;
  const int64_t g = qrow / G, ql = qrow % G;
  const float *yr = ytil + qrow * d;
  const float *pr = p + qrow * m;
  __shared__ float red[2][4];
  __shared__ int ired[4];
  float ay = 0.f, ap = 0.f;
  for (int j = threadIdx.x; j < d; j += blockDim.x) ay = fmaxf(ay, fabsf(yr[j]));
  for (int j = threadIdx.x; j < m; j += blockDim.x) ap = fmaxf(ap, fabsf(pr[j]));
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) {
    ay = fmaxf(ay, __shfl_xor_sync(0xffffffffu, ay, o));
    ap = fmaxf(ap, __shfl_xor_sync(0xffffffffu, ap, o));
  }
  if (threadIdx.x % 32 == 0) {
    red[0][threadIdx.x / 32] = ay;
    red[1][threadIdx.x / 32] = ap;
  }
  __syncthreads();
  ay = fmaxf(fmaxf(red[0][0], red[0][1]), fmaxf(red[0][2], red[0][3]));
  ap = fmaxf(fmaxf(red[1][0], red[1][1]), fmaxf(red[1][2], red[1][3]));
  int ey = 0, ep = 0;
  frexpf(ay, &ey);
  frexpf(ap, &ep);
  const int sy = ay > 0.f ? 14 - ey : 0;  // |y| 2^sy < 2^14
  const int sp = ap > 0.f ? 14 - ep : 0;
  int8_t *r0 = qop + ((g * N) + kColsPerQuery * ql) * kScoreKBytes;
  int8_t *r1 = r0 + kScoreKBytes, *rl = r1 + kScoreKBytes, *r2 = rl + kScoreKBytes, *r3 = r2 + kScoreKBytes;
  for (int j = threadIdx.x; j < d; j += blockDim.x) {
    const int v = __float2int_rn(ldexpf(yr[j], sy));
    const int hi = (v + 128) >> 8, lo = v - 256 * hi;
    const int k = (j / 32) * 32 + code_byte_pos(w, j % 32);
    r0[k] = (int8_t)hi;
    r1[k] = (int8_t)lo;
    r1[128 + k] = (int8_t)hi;
    rl[128 + k] = (int8_t)lo;
  }
  int psum = 0;
  for (int i = threadIdx.x; i < m; i += blockDim.x) {
    const int v = __float2int_rn(ldexpf(pr[i], sp));
    psum += v;
    const int hi = (v + 128) >> 8, lo = v - 256 * hi;
    const int k = 256 + (i / 32) * 32 + sign_byte_pos(i % 32);
    r2[k] = (int8_t)hi;
    r3[k] = (int8_t)lo;
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) psum += __shfl_xor_sync(0xffffffffu, psum, o);
  if (threadIdx.x % 32 == 0) ired[threadIdx.x / 32] = psum;
  __syncthreads();
  if (threadIdx.x == 0)
    qsc[qrow] = make_float4(ldexpf(1.f, -(sy + cexp)), ldexpf(qjl_scale, -sp),
                            (float)(ired[0] + ired[1] + ired[2] + ired[3]), 0.f);
}

// ------------------------------------------------------------------ key expansion
namespace {

__device__ __forceinline__ uint32_t lut16(uint32_t s16, uint32_t t0, uint32_t t1, uint32_t t2, uint32_t t3) {
  // 4 nibble codes (0..15) -> 4 table bytes
  const uint32_t sel = s16 & 0x7777u;
  const uint32_t a = sm100::prmt(t0, t1, sel), b = sm100::prmt(t2, t3, sel);
  return sm100::prmt(a, b, 0x3210u | ((s16 >> 1) & 0x4444u));
}

// Expand one 32-coordinate group: W code words -> 8 words of ch bytes and 8
// of cl bytes, in code_byte_pos order.
template <int W>
__device__ __forceinline__ void expand_codes(const uint32_t *cw, const uint32_t (&tch)[4], const uint32_t (&tcl)[4],
                                             uint32_t (&ch)[8], uint32_t (&cl)[8]) {
  if constexpr (W == 1) {
#pragma unroll
    for (int h = 0; h < 4; ++h) {
      const uint32_t s = (cw[0] >> h) & 0x11111111u;
      ch[2 * h] = sm100::prmt(tch[0], tch[0], s);
      ch[2 * h + 1] = sm100::prmt(tch[0], tch[0], s >> 16);
      cl[2 * h] = sm100::prmt(tcl[0], tcl[0], s);
      cl[2 * h + 1] = sm100::prmt(tcl[0], tcl[0], s >> 16);
    }
  } else if constexpr (W == 2) {
#pragma unroll
    for (int q = 0; q < 2; ++q) {
#pragma unroll
      for (int hh = 0; hh < 2; ++hh) {
        const uint32_t s = (cw[q] >> (2 * hh)) & 0x33333333u;
        ch[4 * q + 2 * hh] = sm100::prmt(tch[0], tch[0], s);
        ch[4 * q + 2 * hh + 1] = sm100::prmt(tch[0], tch[0], s >> 16);
        cl[4 * q + 2 * hh] = sm100::prmt(tcl[0], tcl[0], s);
        cl[4 * q + 2 * hh + 1] = sm100::prmt(tcl[0], tcl[0], s >> 16);
      }
    }
  } else if constexpr (W == 3) {
    uint32_t s[4];
    s[0] = cw[0] & 0x77777777u;
    s[1] = cw[1] & 0x77777777u;
    s[2] = cw[2] & 0x77777777u;
    s[3] = ((cw[0] >> 1) & 0x44444444u) | ((cw[1] >> 2) & 0x22222222u) | ((cw[2] >> 3) & 0x11111111u);
#pragma unroll
    for (int k = 0; k < 4; ++k) {
      ch[2 * k] = sm100::prmt(tch[0], tch[1], s[k]);
      ch[2 * k + 1] = sm100::prmt(tch[0], tch[1], s[k] >> 16);
      cl[2 * k] = sm100::prmt(tcl[0], tcl[1], s[k]);
      cl[2 * k + 1] = sm100::prmt(tcl[0], tcl[1], s[k] >> 16);
    }
  } else {  // W == 4
#pragma unroll
    for (int k = 0; k < 4; ++k) {
      ch[2 * k] = lut16(cw[k] & 0xFFFFu, tch[0], tch[1], tch[2], tch[3]);
      ch[2 * k + 1] = lut16(cw[k] >> 16, tch[0], tch[1], tch[2], tch[3]);
      cl[2 * k] = lut16(cw[k] & 0xFFFFu, tcl[0], tcl[1], tcl[2], tcl[3]);
      cl[2 * k + 1] = lut16(cw[k] >> 16, tcl[0], tcl[1], tcl[2], tcl[3]);
    }
  }
}

__device__ __forceinline__ void sts128_sw(uint8_t *atom, int row, int chunk, uint32_t a, uint32_t b, uint32_t c,
                                          uint32_t d) {
  *reinterpret_cast<uint4 *>(atom + sm100::sw128_offset(row, chunk)) = make_uint4(a, b, c, d);
}


// Scores of one key (this thread's TMEM lane) for every query of its group.
__device__ __forceinline__ void score_epilogue(const ScoreTCParams &p, const float4 *sQ, uint32_t taddr,
                                               int64_t g, int64_t kin, bool valid, float2 nr) {
  for (int q0 = 0; q0 < p.G; q0 += 3) {  // 15 of the 16 loaded columns = 3 queries
    uint32_t dv[16];
    sm100::tmem_ld16(taddr + kColsPerQuery * q0, dv);
    sm100::tmem_wait_ld();
#pragma unroll
    for (int qq = 0; qq < 3; ++qq) {
      const int q = q0 + qq;
      if (q < p.G && valid) {
        const float4 sc = sQ[q];
        const int *v = reinterpret_cast<const int *>(dv) + kColsPerQuery * qq;
        const int sb = 2 * (256 * v[3] + v[4]) - (int)sc.z;
        const float a = fmaf((float)v[0], 65536.f, fmaf((float)v[1], 256.f, (float)v[2])) * sc.x;
        float s = nr.x * fmaf(nr.y * sc.y, (float)sb, a);
        float *o = p.out + (g * p.G + q) * p.ldo + kin;
        if (p.accumulate) s += *o;
        *o = s;
      }
    }
  }
}

}  // namespace

// ------------------------------------------------------------------ scorer
// 128 threads = 128 keys per tile.  Persistent CTAs walk a contiguous range of
// tiles (a group's tiles are contiguous).  Raw key rows (codes, sign words,
// norms) arrive by bulk asynchronous copies into a ring of kStages shared
// buffers, issued kStages tiles ahead; each tile is then expanded into the
// MMA operand, multiplied, and its scores are written one tile later while
// the next tile is being prepared.
constexpr int kStages = 4;

template <int W, int NG>
struct ScoreSmem {
  static constexpr int kCW = W * NG;                // code words per key
  static constexpr int kCodeBytes = 128 * kCW * 4;  // per stage
  static constexpr int kSignBytes = 128 * NG * 4;
  static constexpr int kNormBytes = 128 * 8;
  static constexpr int kStageBytes = kCodeBytes + kSignBytes + kNormBytes;
  static constexpr int kOffA = 0;                          // 3 x 16 KB operand atoms
  static constexpr int kOffStage = 3 * 16384;
  static constexpr int kOffB = kOffStage + kStages * kStageBytes;
};

template <int W, int NG, bool BULK>
__global__ void __launch_bounds__(128)
k_score_tc(const ScoreTCParams p) {
  using SM = ScoreSmem<W, NG>;
  constexpr int CW = SM::kCW;
  extern __shared__ uint8_t smem_raw[];
  uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t *sA = smem + SM::kOffA;
  uint8_t *sStage = smem + SM::kOffStage;
  uint8_t *sB = smem + (BULK ? SM::kOffB : SM::kOffStage);
  float4 *sQ = reinterpret_cast<float4 *>(sB + 3 * p.N * 128);
  uint64_t *bars = reinterpret_cast<uint64_t *>(sQ + p.G);  // [kStages] stages, then the MMA barrier
  uint32_t *sTmem = reinterpret_cast<uint32_t *>(bars + kStages + 1);

  const int tid = threadIdx.x;
  const uint32_t lane = (uint32_t)(tid & ~31) << 16;
  const int64_t t0 = (p.ntiles * blockIdx.x) / gridDim.x;
  const int64_t t1 = (p.ntiles * (blockIdx.x + 1)) / gridDim.x;
  uint32_t ncols = 32;
  while ((int)ncols < p.N + 16) ncols <<= 1;  // epilogue loads read 16 columns from 5*q0
  if (tid == 0) {
    for (int i = 0; i <= kStages; ++i) sm100::mbar_init(&bars[i], 1);
    sm100::fence_barrier_init();
  }
  if (tid < 32) {
    sm100::tmem_alloc(sTmem, ncols);
    sm100::tmem_relinquish();
  }
  sm100::tc_fence_before();
  __syncthreads();
  sm100::tc_fence_after();
  const uint32_t tmem = *sTmem;
  uint64_t *mma_bar = &bars[kStages];
  uint32_t tch[4], tcl[4];
#pragma unroll
  for (int k = 0; k < 4; ++k) {
    tch[k] = p.tch[k];
    tcl[k] = p.tcl[k];
  }
  const uint32_t idesc = sm100::idesc_s8_s32(128, p.N);
  const int64_t tpg = p.tiles_per_group;

  // Tile t covers keys [kin0, kin0 + 128) (relative to key_base) of group
  // t / tpg; with BULK, stage slot (t - t0) % kStages holds exactly its rows.
  auto issue_stage = [&](int64_t t, int slot) {
    const int64_t g = t / tpg;
    const int64_t kin0 = (t % tpg) * 128;
    const int64_t key0 = g * p.kpg + p.key_base + kin0;
    const int64_t left = p.nkeys - kin0;
    const int rows = left < 128 ? (int)left : 128;
    uint8_t *st = sStage + slot * SM::kStageBytes;
    const uint32_t cb = rows * CW * 4, sb = rows * NG * 4, nb = rows * 8;
    sm100::mbar_expect_tx(&bars[slot], cb + sb + nb);
    sm100::bulk_load(st, p.codes + key0 * CW, cb, &bars[slot]);
    sm100::bulk_load(st + SM::kCodeBytes, p.signs + key0 * NG, sb, &bars[slot]);
    sm100::bulk_load(st + SM::kCodeBytes + SM::kSignBytes, p.norms + key0, nb, &bars[slot]);
  };
  int64_t issued = t0;  // next tile whose stage is to be issued (thread 0)
  if constexpr (BULK) {
    if (tid == 0)
      for (; issued < t1 && issued < t0 + kStages; ++issued) issue_stage(issued, (int)(issued - t0));
  }

  uint32_t ph_mma = 0u;
  bool failed = false;
  int64_t cur_group = -1;
  int64_t g = t0 / tpg, tin = t0 % tpg;  // group and tile-in-group of tile t
  int64_t prev_g = -1, prev_kin = 0;
  bool prev_valid = false;
  float2 prev_nr = make_float2(0.f, 0.f);
  int64_t t = t0;
  for (; t < t1; ++t) {
    const int slot = (int)((t - t0) % kStages);
    const int64_t kin = tin * 128 + tid;
    const bool valid = kin < p.nkeys;
    bool ok = true;
    // ---- raw row of this tile's key
    uint32_t cw[CW], sw[NG];
    float2 nr = make_float2(0.f, 0.f);
#pragma unroll
    for (int k = 0; k < CW; ++k) cw[k] = 0u;
#pragma unroll
    for (int k = 0; k < NG; ++k) sw[k] = 0u;
    if constexpr (BULK) {
      ok = sm100::mbar_wait(&bars[slot], (uint32_t)(((t - t0) / kStages) & 1), p.err, 21);
      const uint8_t *st = sStage + slot * SM::kStageBytes;
      if (valid) {
        if constexpr (CW % 4 == 0) {
#pragma unroll
          for (int k = 0; k < CW / 4; ++k) {
            const uint4 v = reinterpret_cast<const uint4 *>(st + tid * CW * 4)[k];
            cw[4 * k] = v.x; cw[4 * k + 1] = v.y; cw[4 * k + 2] = v.z; cw[4 * k + 3] = v.w;
          }
        } else {
#pragma unroll
          for (int k = 0; k < CW; ++k) cw[k] = reinterpret_cast<const uint32_t *>(st + tid * CW * 4)[k];
        }
#pragma unroll
        for (int k = 0; k < NG; ++k)
          sw[k] = reinterpret_cast<const uint32_t *>(st + SM::kCodeBytes + tid * NG * 4)[k];
        nr = reinterpret_cast<const float2 *>(st + SM::kCodeBytes + SM::kSignBytes)[tid];
      }
    } else {
      if (valid) {
        const int64_t key = g * p.kpg + p.key_base + kin;
#pragma unroll
        for (int k = 0; k < CW; ++k) cw[k] = __ldg(p.codes + key * CW + k);
#pragma unroll
        for (int k = 0; k < NG; ++k) sw[k] = __ldg(p.signs + key * NG + k);
        nr = __ldg(p.norms + key);
      }
    }
    // ---- expand into registers
    uint32_t ach[NG][8], acl[NG][8], abt[NG][8];
#pragma unroll
    for (int gi = 0; gi < NG; ++gi) {
      expand_codes<W>(cw + gi * W, tch, tcl, ach[gi], acl[gi]);
#pragma unroll
      for (int k = 0; k < 8; ++k) abt[gi][k] = (sw[gi] >> k) & 0x01010101u;
    }
    // ---- scores of the previous tile
    if (t > t0) {
      ok = sm100::mbar_wait(mma_bar, ph_mma, p.err, 22) && ok;
      ph_mma ^= 1u;
      sm100::tc_fence_after();
      score_epilogue(p, sQ, tmem + lane, prev_g, prev_kin, prev_valid, prev_nr);
    }
    // ---- the query operand of this group
    if (g != cur_group) {
      sm100::tc_fence_before();
      __syncthreads();
      const int8_t *src = p.qop + g * (int64_t)p.N * kScoreKBytes;
      for (int i = tid; i < p.N * 24; i += 128) {  // 16-byte chunks
        const int n = i / 24, c = i % 24;
        const uint4 v = __ldg(reinterpret_cast<const uint4 *>(src + n * kScoreKBytes) + c);
        *reinterpret_cast<uint4 *>(sB + (c / 8) * (p.N * 128) + sm100::sw128_offset(n, c % 8)) = v;
      }
      for (int i = tid; i < p.G; i += 128) sQ[i] = p.qsc[g * p.G + i];
      cur_group = g;
    }
    // ---- key operand row
#pragma unroll
    for (int gi = 0; gi < NG; ++gi) {
      sts128_sw(sA, tid, 2 * gi, ach[gi][0], ach[gi][1], ach[gi][2], ach[gi][3]);
      sts128_sw(sA, tid, 2 * gi + 1, ach[gi][4], ach[gi][5], ach[gi][6], ach[gi][7]);
      sts128_sw(sA + 16384, tid, 2 * gi, acl[gi][0], acl[gi][1], acl[gi][2], acl[gi][3]);
      sts128_sw(sA + 16384, tid, 2 * gi + 1, acl[gi][4], acl[gi][5], acl[gi][6], acl[gi][7]);
      sts128_sw(sA + 32768, tid, 2 * gi, abt[gi][0], abt[gi][1], abt[gi][2], abt[gi][3]);
      sts128_sw(sA + 32768, tid, 2 * gi + 1, abt[gi][4], abt[gi][5], abt[gi][6], abt[gi][7]);
    }
    sm100::fence_proxy_async();
    sm100::tc_fence_before();
    failed |= __syncthreads_or(!ok || failed) != 0;
    if (failed) break;
    sm100::tc_fence_after();
    if (tid == 0) {
      const uint32_t a0 = sm100::smem_u32(sA), b0 = sm100::smem_u32(sB);
      // coordinates beyond d (NG < 4) meet zero query bytes, so the unwritten
      // part of the key row does not contribute
#pragma unroll
      for (int ks = 0; ks < kScoreKBytes / 32; ++ks) {
        const int atom = ks / 4, off = (ks % 4) * 32;
        const uint64_t a = sm100::desc_sw128(a0 + atom * 16384 + off);
        const uint64_t b = sm100::desc_sw128(b0 + atom * (p.N * 128) + off);
        sm100::mma_i8(tmem, a, b, idesc, ks != 0);
      }
      sm100::mma_commit(mma_bar);
      // every thread has read this tile's stage: refill it kStages tiles ahead
      if constexpr (BULK) {
        if (issued < t1) {
          issue_stage(issued, slot);
          ++issued;
        }
      }
    }
    prev_g = g;
    prev_kin = kin;
    prev_valid = valid;
    prev_nr = nr;
    if (++tin == tpg) {
      tin = 0;
      ++g;
    }
  }
  if (!failed && t1 > t0) {
    const bool ok = __syncthreads_and(sm100::mbar_wait(mma_bar, ph_mma, p.err, 23)) != 0;  // CTA-uniform
    sm100::tc_fence_after();
    if (ok) score_epilogue(p, sQ, tmem + lane, prev_g, prev_kin, prev_valid, prev_nr);
  }
  if constexpr (BULK) {
    if (failed && tid == 0) {
      // bounded wait for stage copies issued but not consumed
      for (int64_t u = t + 1; u < issued; ++u)
        sm100::mbar_wait(&bars[(u - t0) % kStages], (uint32_t)(((u - t0) / kStages) & 1), p.err, 24);
    }
  }
  sm100::tc_fence_before();
  __syncthreads();
  if (tid < 32) sm100::tmem_dealloc(tmem, ncols);
}

// ------------------------------------------------------------------ host side
bool tc_score_supported(const tq_quantizer *q, int64_t G) {
  return q->d <= 128 && q->d % 32 == 0 && q->m == q->d && G >= 1 && G <= kMaxScoreG;
}

size_t tc_score_qop_bytes(const tq_quantizer *q, int64_t groups, int64_t G) {
  const int64_t N = (kColsPerQuery * G + 15) / 16 * 16;
  return (size_t)groups * N * kScoreKBytes;
}

tq_status tc_score(const tq_quantizer *q, const float *ytil, const float *pq, int64_t groups, int64_t G,
                   int64_t kpg, int64_t key_base, int64_t nkeys, const void *codes, const void *signs,
                   const float *norms, float *out, int64_t ldo, int accumulate, int8_t *qop, float4 *qsc,
                   cudaStream_t st) {
  const int N = (int)((kColsPerQuery * G + 15) / 16 * 16);
  const int64_t nq = groups * G;
  if (cudaMemsetAsync(qop, 0, tc_score_qop_bytes(q, groups, G), st) != cudaSuccess) return TQ_ERR_CUDA;
  k_query_operand<<<(unsigned)nq, 128, 0, st>>>(ytil, pq, q->d, q->m, q->w, G, N, q->score_cexp, q->kt.qjl_scale,
                                                qop, qsc);
  if (cudaGetLastError() != cudaSuccess) return TQ_ERR_CUDA;
  ScoreTCParams prm{};
  prm.d = q->d;
  prm.m = q->m;
  prm.G = G;
  prm.kpg = kpg;
  prm.key_base = key_base;
  prm.nkeys = nkeys;
  prm.N = N;
  prm.tiles_per_group = (nkeys + 127) / 128;
  prm.ntiles = prm.tiles_per_group * groups;
  prm.codes = static_cast<const uint32_t *>(codes);
  prm.signs = static_cast<const uint32_t *>(signs);
  prm.norms = reinterpret_cast<const float2 *>(norms);
  prm.qop = qop;
  prm.qsc = qsc;
  for (int k = 0; k < 4; ++k) {
    uint32_t h = 0, l = 0;
    for (int b = 0; b < 4; ++b) {
      h |= (uint32_t)(uint8_t)q->score_ch[4 * k + b] << (8 * b);
      l |= (uint32_t)(uint8_t)q->score_cl[4 * k + b] << (8 * b);
    }
    prm.tch[k] = h;
    prm.tcl[k] = l;
  }
  prm.out = out;
  prm.ldo = ldo;
  prm.accumulate = accumulate;
  prm.err = q->d_err;
  const int ng = q->d / 32, cwords = q->w * ng;
  const size_t stage_bytes = (size_t)128 * (cwords + ng) * 4 + 128 * 8;
  // bulk copies need 16-byte multiples and 16-byte aligned rows for every tile
  const bool bulk = ng == 4 && kpg % 2 == 0 && key_base % 2 == 0 && nkeys % 2 == 0 &&
                    reinterpret_cast<uintptr_t>(norms) % 16 == 0 && reinterpret_cast<uintptr_t>(codes) % 16 == 0 &&
                    reinterpret_cast<uintptr_t>(signs) % 16 == 0;
  const size_t smem = 1024 + 3 * 16384 + (bulk ? kStages * stage_bytes : 0) + 3 * (size_t)N * 128 +
                      (size_t)G * 16 + 128;
  int dev = 0, sms = 0;
  cudaGetDevice(&dev);
  cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  const int per_sm = (int)std::max<size_t>(1, std::min<size_t>(4, (228 * 1024) / (smem + 1024)));
  const int64_t grid = std::min<int64_t>(prm.ntiles, (int64_t)sms * per_sm);
  if (grid <= 0) return TQ_OK;
#define TQ_SC(WW, NGG)                                                                                   \
  {                                                                                                      \
    auto kern = bulk ? k_score_tc<WW, NGG, (NGG == 4)> : k_score_tc<WW, NGG, false>;                     \
    if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem) != cudaSuccess) \
      return TQ_ERR_CUDA;                                                                                \
    kern<<<(unsigned)grid, 128, smem, st>>>(prm);                                                        \
    break;                                                                                               \
  }
#define TQ_SC_NG(WW)                     \
  switch (q->d / 32) {                   \
    case 1: TQ_SC(WW, 1)                 \
    case 2: TQ_SC(WW, 2)                 \
    case 3: TQ_SC(WW, 3)                 \
    case 4: TQ_SC(WW, 4)                 \
    default: return TQ_ERR_UNSUPPORTED;  \
  }
  switch (q->w) {
    case 1: TQ_SC_NG(1) break;
    case 2: TQ_SC_NG(2) break;
    case 3: TQ_SC_NG(3) break;
    case 4: TQ_SC_NG(4) break;
    default: return TQ_ERR_UNSUPPORTED;
  }
#undef TQ_SC_NG
#undef TQ_SC
  return cudaGetLastError() == cudaSuccess ? TQ_OK : TQ_ERR_CUDA;
}

}  // namespace tq

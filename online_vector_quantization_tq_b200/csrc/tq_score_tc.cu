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
// The key operand is written straight into tensor memory (tcgen05.st) and the
// MMA reads it from there; the query operand is stored in global memory as the
// image of its swizzled shared-memory tile and arrives by one bulk copy.
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
  // byte k of operand row n sits where the 128-byte-swizzled K-major tile
  // (three 128-byte K atoms of N rows) keeps it in shared memory
  auto at = [N](int n, int k) { return (k / 128) * (N * 128) + sm100::sw128_offset(n, (k % 128) / 16) + k % 16; };
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
  int8_t *img = qop + g * (int64_t)N * kScoreKBytes;
  const int n0 = kColsPerQuery * (int)ql;  // rows n0..n0+4: yh, yl|yh, yl, ph, pl
  for (int j = threadIdx.x; j < d; j += blockDim.x) {
    const int v = __float2int_rn(ldexpf(yr[j], sy));
    const int hi = (v + 128) >> 8, lo = v - 256 * hi;
    const int k = (j / 32) * 32 + code_byte_pos(w, j % 32);
    img[at(n0, k)] = (int8_t)hi;
    img[at(n0 + 1, k)] = (int8_t)lo;
    img[at(n0 + 1, 128 + k)] = (int8_t)hi;
    img[at(n0 + 2, 128 + k)] = (int8_t)lo;
  }
  int psum = 0;
  for (int i = threadIdx.x; i < m; i += blockDim.x) {
    const int v = __float2int_rn(ldexpf(pr[i], sp));
    psum += v;
    const int hi = (v + 128) >> 8, lo = v - 256 * hi;
    const int k = 256 + (i / 32) * 32 + sign_byte_pos(i % 32);
    img[at(n0 + 3, k)] = (int8_t)hi;
    img[at(n0 + 4, k)] = (int8_t)lo;
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



}  // namespace

// ------------------------------------------------------------------ scorer
// Warp-specialised, one persistent CTA per SM walking a contiguous range of
// 128-key tiles (a group's tiles are contiguous):
//   warps 0-7   expanders, two groups of four taking alternate tiles; thread
//               (warp % 4, lane) expands key row 32 (warp % 4) + lane into
//               its group's key operand in TMEM;
//   warps 8-15  epilogue, two per TMEM lane quarter, queries split between
//               them; scores of a tile from its TMEM accumulator;
//   warp 16     MMA issue (one thread), query operand copies, TMEM owner;
//   warp 17     raw key rows: bulk copies into a ring of kStages buffers.
// Hand-offs are mbarriers only: stage full/empty, key operand full/empty,
// accumulator full/empty.  Every wait is bounded and gives up as soon as
// another role has failed, after which all roles leave their loops, in-flight
// copies and MMAs are waited for (bounded) and TMEM is freed.
constexpr int kStages = 4;
constexpr int kExpWarps = 8, kEpiWarps = 8;
constexpr int kMmaWarp = kExpWarps + kEpiWarps, kLoadWarp = kMmaWarp + 1;
constexpr int kScoreThreads = (kLoadWarp + 1) * 32;
constexpr int kACols = kScoreKBytes / 4;  // TMEM columns of one key operand

// TMEM plan of one CTA: accumulators (N columns + 16 for the epilogue's wide
// loads, rounded to 32) then two key operands.
struct ScoreTmem {
  int npad, nacc, ncols;
  __host__ __device__ explicit ScoreTmem(int N) {
    npad = (N + 16 + 31) / 32 * 32;
    nacc = 2 * npad + 2 * kACols <= 512 ? 2 : 1;
    const int used = nacc * npad + 2 * kACols;
    ncols = 32;
    while (ncols < used) ncols <<= 1;
  }
  __host__ __device__ int acc(int b) const { return b * npad; }
  __host__ __device__ int a(int e) const { return nacc * npad + e * kACols; }
};

template <int W, int NG>
struct ScoreSmem {
  static constexpr int kCW = W * NG;                // code words per key
  static constexpr int kCodeBytes = 128 * kCW * 4;  // per stage
  static constexpr int kSignBytes = 128 * NG * 4;
  static constexpr int kStageBytes = kCodeBytes + kSignBytes;
  static constexpr int kOffB = kStages * kStageBytes;  // multiple of 1024
  enum Bar { kFull = 0, kEmpty = kStages, kAFull = 2 * kStages, kAEmpty = kAFull + 2, kAccFull = kAEmpty + 2,
             kAccEmpty = kAccFull + 2, kBFull = kAccEmpty + 2, kMmaDone = kBFull + 1, kNumBars = kMmaDone + 1 };
};

template <int W, int NG, bool BULK>
__global__ void __launch_bounds__(kScoreThreads, 1)
k_score_tc(const ScoreTCParams p) {
  using SM = ScoreSmem<W, NG>;
  constexpr int CW = SM::kCW;
  extern __shared__ uint8_t smem_raw[];
  uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t *sStage = smem;
  uint8_t *sB = smem + (BULK ? SM::kOffB : 0);
  const uint32_t b_bytes = (uint32_t)p.N * kScoreKBytes;
  uint64_t *bars = reinterpret_cast<uint64_t *>(sB + b_bytes);
  uint32_t *sTmem = reinterpret_cast<uint32_t *>(bars + SM::kNumBars);
  volatile int *sAbort = reinterpret_cast<volatile int *>(sTmem + 1);

  const int tid = threadIdx.x, warp = tid / 32, lane = tid % 32;
  const ScoreTmem tp(p.N);
  const int64_t t0 = (p.ntiles * blockIdx.x) / gridDim.x;
  const int64_t t1 = (p.ntiles * (blockIdx.x + 1)) / gridDim.x;
  const int n_it = (int)(t1 - t0);
  const int64_t tpg = p.tiles_per_group;
  if (tid == 0) {
    for (int i = 0; i < kStages; ++i) {
      sm100::mbar_init(&bars[SM::kFull + i], 1);
      sm100::mbar_init(&bars[SM::kEmpty + i], 4);
    }
    for (int i = 0; i < 2; ++i) {
      sm100::mbar_init(&bars[SM::kAFull + i], 4);
      sm100::mbar_init(&bars[SM::kAEmpty + i], 1);
      sm100::mbar_init(&bars[SM::kAccFull + i], 1);
      sm100::mbar_init(&bars[SM::kAccEmpty + i], kEpiWarps);
    }
    sm100::mbar_init(&bars[SM::kBFull], 1);
    sm100::mbar_init(&bars[SM::kMmaDone], 1);
    *sAbort = 0;
    sm100::fence_barrier_init();
  }
  if (warp == kMmaWarp) {
    sm100::tmem_alloc(sTmem, (uint32_t)tp.ncols);
    sm100::tmem_relinquish();
  }
  sm100::tc_fence_before();
  __syncthreads();
  sm100::tc_fence_after();
  const uint32_t tmem = *sTmem;
  auto wait = [&](int bar, uint32_t parity, int code) {
    return sm100::mbar_wait_abort(&bars[bar], parity, sAbort, p.err, code);
  };
  // state the teardown needs
  int64_t issued = 0;      // stages issued (load warp)
  int mma_issued = 0;      // tiles whose MMAs were issued (MMA thread)
  bool b_pending = false;  // a query-operand copy not yet seen complete
  uint32_t b_ph = 0, md_ph = 0;

  if (warp < kExpWarps) {
    // ------------------------------------------------------------ expanders
    const int e = warp / 4, quarter = warp % 4, row = 32 * quarter + lane;
    const uint32_t tlane = (uint32_t)(32 * quarter) << 16;
    uint32_t tch[4], tcl[4];
#pragma unroll
    for (int k = 0; k < 4; ++k) {
      tch[k] = p.tch[k];
      tcl[k] = p.tcl[k];
    }
    for (int it = e; it < n_it; it += 2) {
      const int64_t t = t0 + it, g = t / tpg, kin = (t % tpg) * 128 + row;
      const bool valid = kin < p.nkeys;
      uint32_t cw[CW], sw[NG];
#pragma unroll
      for (int k = 0; k < CW; ++k) cw[k] = 0u;
#pragma unroll
      for (int k = 0; k < NG; ++k) sw[k] = 0u;
      if constexpr (BULK) {
        const int slot = it % kStages;
        if (!__all_sync(0xffffffffu, wait(SM::kFull + slot, (uint32_t)((it / kStages) & 1), 21))) break;
        const uint8_t *st = sStage + slot * SM::kStageBytes;
        if (valid) {
          const uint4 *crow = reinterpret_cast<const uint4 *>(st + row * CW * 4);
#pragma unroll
          for (int k = 0; k < CW / 4; ++k) {
            const uint4 v = crow[k];
            cw[4 * k] = v.x;
            cw[4 * k + 1] = v.y;
            cw[4 * k + 2] = v.z;
            cw[4 * k + 3] = v.w;
          }
          const uint4 sv = *reinterpret_cast<const uint4 *>(st + SM::kCodeBytes + row * NG * 4);
          sw[0] = sv.x;
          sw[1] = sv.y;
          sw[2] = sv.z;
          sw[3] = sv.w;
        }
        __syncwarp();
        if (lane == 0) sm100::mbar_arrive(&bars[SM::kEmpty + slot]);
      } else {
        if (valid) {
          const int64_t key = g * p.kpg + p.key_base + kin;
#pragma unroll
          for (int k = 0; k < CW; ++k) cw[k] = __ldg(p.codes + key * CW + k);
#pragma unroll
          for (int k = 0; k < NG; ++k) sw[k] = __ldg(p.signs + key * NG + k);
        }
      }
      // the key operand buffer was last read by the MMAs of tile it - 2
      const int use = it / 2;
      if (use > 0 && !__all_sync(0xffffffffu, wait(SM::kAEmpty + e, (uint32_t)((use - 1) & 1), 22))) break;
      sm100::tc_fence_after();
      const uint32_t ta = tmem + tlane + (uint32_t)tp.a(e);
#pragma unroll
      for (int gi = 0; gi < NG; ++gi) {
        uint32_t ch[8], cl[8], bt[8];
        expand_codes<W>(cw + gi * W, tch, tcl, ch, cl);
#pragma unroll
        for (int k = 0; k < 8; ++k) bt[k] = (sw[gi] >> k) & 0x01010101u;
        sm100::tmem_st8(ta + 8 * gi, ch);
        sm100::tmem_st8(ta + 32 + 8 * gi, cl);
        sm100::tmem_st8(ta + 64 + 8 * gi, bt);
      }
      sm100::tmem_wait_st();
      sm100::tc_fence_before();
      __syncwarp();
      if (lane == 0) sm100::mbar_arrive(&bars[SM::kAFull + e]);
    }
  } else if (warp < kMmaWarp) {
    // ------------------------------------------------------------ epilogue
    const int quarter = warp % 4, eh = (warp - kExpWarps) / 4, row = 32 * quarter + lane;
    const int q_half = (int)((p.G + 1) / 2);
    const int q_lo = eh ? q_half : 0, q_hi = eh ? (int)p.G : q_half;
    const uint32_t tlane = (uint32_t)(32 * quarter) << 16;
    for (int it = 0; it < n_it; ++it) {
      const int64_t t = t0 + it, g = t / tpg, kin = (t % tpg) * 128 + row;
      const bool valid = kin < p.nkeys;
      float2 nr = make_float2(0.f, 0.f);
      if (valid) nr = __ldg(p.norms + g * p.kpg + p.key_base + kin);
      const int ab = it % tp.nacc, use = it / tp.nacc;
      if (!__all_sync(0xffffffffu, wait(SM::kAccFull + ab, (uint32_t)(use & 1), 23))) break;
      sm100::tc_fence_after();
      const uint32_t taddr = tmem + tlane + (uint32_t)tp.acc(ab);
      const float4 *qs = p.qsc + g * p.G;
      float *orow = p.out + g * p.G * p.ldo + kin;
      for (int q0 = q_lo; q0 < q_hi; q0 += 3) {  // 15 of 16 loaded columns = 3 queries
        uint32_t dv[16];
        sm100::tmem_ld16(taddr + kColsPerQuery * q0, dv);
        float4 sc[3];
#pragma unroll
        for (int qq = 0; qq < 3; ++qq) sc[qq] = q0 + qq < q_hi ? __ldg(qs + q0 + qq) : make_float4(0.f, 0.f, 0.f, 0.f);
        sm100::tmem_wait_ld();
#pragma unroll
        for (int qq = 0; qq < 3; ++qq) {
          const int q = q0 + qq;
          if (q < q_hi && valid) {
            const int *v = reinterpret_cast<const int *>(dv) + kColsPerQuery * qq;
            const int sb = 2 * (256 * v[3] + v[4]) - (int)sc[qq].z;
            const float a = fmaf((float)v[0], 65536.f, fmaf((float)v[1], 256.f, (float)v[2])) * sc[qq].x;
            float sres = nr.x * fmaf(nr.y * sc[qq].y, (float)sb, a);
            float *o = orow + q * p.ldo;
            if (p.accumulate) sres += *o;
            *o = sres;
          }
        }
      }
      sm100::tc_fence_before();
      __syncwarp();
      if (lane == 0) sm100::mbar_arrive(&bars[SM::kAccEmpty + ab]);
    }
  } else if (warp == kMmaWarp) {
    // ------------------------------------------------------------ MMA issue
    if (lane == 0) {
      const uint32_t idesc = sm100::idesc_s8_s32(128, p.N);
      const uint32_t b0 = sm100::smem_u32(sB);
      int64_t cur_group = -1;
      for (int it = 0; it < n_it; ++it) {
        const int64_t g = (t0 + it) / tpg;
        if (g != cur_group) {
          if (it > 0) {  // every MMA reading the old query operand has completed
            sm100::mma_commit(&bars[SM::kMmaDone]);
            const bool ok = wait(SM::kMmaDone, md_ph, 24);
            md_ph ^= 1u;
            if (!ok) break;
          }
          sm100::mbar_expect_tx(&bars[SM::kBFull], b_bytes);
          sm100::bulk_load(sB, p.qop + g * (int64_t)b_bytes, b_bytes, &bars[SM::kBFull]);
          b_pending = true;
          if (!wait(SM::kBFull, b_ph, 25)) break;
          b_ph ^= 1u;
          b_pending = false;
          cur_group = g;
        }
        const int e = it & 1, ab = it % tp.nacc;
        if (!wait(SM::kAFull + e, (uint32_t)((it / 2) & 1), 26)) break;
        if (it >= tp.nacc && !wait(SM::kAccEmpty + ab, (uint32_t)((it / tp.nacc - 1) & 1), 27)) break;
        sm100::tc_fence_after();
        const uint32_t ta = tmem + (uint32_t)tp.a(e), td = tmem + (uint32_t)tp.acc(ab);
        bool first = true;
#pragma unroll
        for (int ks = 0; ks < kScoreKBytes / 32; ++ks) {
          if (ks % 4 >= NG) continue;  // coordinates beyond d
          const uint64_t db = sm100::desc_sw128(b0 + (ks / 4) * (p.N * 128) + (ks % 4) * 32);
          sm100::mma_i8_ts(td, ta + 8 * ks, db, idesc, !first);
          first = false;
        }
        sm100::mma_commit(&bars[SM::kAEmpty + e]);
        sm100::mma_commit(&bars[SM::kAccFull + ab]);
        mma_issued = it + 1;
      }
    }
  } else if (BULK && lane == 0) {
    // ------------------------------------------------------------ raw key rows
    for (; issued < n_it; ++issued) {
      const int j = (int)issued, slot = j % kStages;
      if (j >= kStages && !wait(SM::kEmpty + slot, (uint32_t)((j / kStages - 1) & 1), 28)) break;
      const int64_t t = t0 + j, g = t / tpg, kin0 = (t % tpg) * 128;
      const int64_t key0 = g * p.kpg + p.key_base + kin0;
      const int64_t left = p.nkeys - kin0;
      const int rows = left < 128 ? (int)left : 128;
      uint8_t *st = sStage + slot * SM::kStageBytes;
      const uint32_t cb = rows * CW * 4, sb = rows * NG * 4;
      sm100::mbar_expect_tx(&bars[SM::kFull + slot], cb + sb);
      sm100::bulk_load(st, p.codes + key0 * CW, cb, &bars[SM::kFull + slot]);
      sm100::bulk_load(st + SM::kCodeBytes, p.signs + key0 * NG, sb, &bars[SM::kFull + slot]);
    }
  }
  // ------------------------------------------------------------ teardown
  __syncthreads();
  if (warp == kMmaWarp && lane == 0) {
    if (mma_issued > 0) {  // no MMA may still write TMEM when it is freed
      sm100::mma_commit(&bars[SM::kMmaDone]);
      sm100::mbar_wait(&bars[SM::kMmaDone], md_ph, p.err, 29);
    }
    if (b_pending) sm100::mbar_wait(&bars[SM::kBFull], b_ph, p.err, 30);
  }
  if (BULK && warp == kLoadWarp && lane == 0 && *sAbort) {
    // copies issued but possibly not consumed: the last kStages issued
    for (int64_t j = issued > kStages ? issued - kStages : 0; j < issued; ++j)
      sm100::mbar_wait(&bars[SM::kFull + j % kStages], (uint32_t)((j / kStages) & 1), p.err, 31);
  }
  sm100::tc_fence_before();
  __syncthreads();
  sm100::tc_fence_after();
  if (warp == kMmaWarp) sm100::tmem_dealloc(tmem, (uint32_t)tp.ncols);
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
  const size_t stage_bytes = (size_t)128 * (cwords + ng) * 4;
  // bulk copies need 16-byte aligned starts and sizes: with d = 128 a key's
  // code and sign rows are multiples of 16 bytes, so any tile qualifies
  const bool bulk = ng == 4 && reinterpret_cast<uintptr_t>(codes) % 16 == 0 &&
                    reinterpret_cast<uintptr_t>(signs) % 16 == 0;
  if (reinterpret_cast<uintptr_t>(qop) % 16 != 0) return TQ_ERR_ALIGNMENT;
  const size_t smem = 1024 + (bulk ? kStages * stage_bytes : 0) + (size_t)N * kScoreKBytes + 8 * 24 + 16;
  int dev = 0, sms = 0;
  cudaGetDevice(&dev);
  cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  const int64_t grid = std::min<int64_t>(prm.ntiles, (int64_t)sms);
  if (grid <= 0) return TQ_OK;
#define TQ_SC(WW, NGG)                                                                                   \
  {                                                                                                      \
    auto kern = bulk ? k_score_tc<WW, NGG, (NGG == 4)> : k_score_tc<WW, NGG, false>;                     \
    if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem) != cudaSuccess) \
      return TQ_ERR_CUDA;                                                                                \
    kern<<<(unsigned)grid, kScoreThreads, smem, st>>>(prm);                                                        \
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

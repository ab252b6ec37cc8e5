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
#include "tq_expand.cuh"
#include "tq_kernels.h"
#include "tq_rng.cuh"
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
  int nstages;  // key-row stages in the ring (bulk copies)
  // nonzero: the kernel before this one in the stream is the query-side
  // kernel (launched normally, so the keys were complete before it started,
  // and it uses no TMEM): keys may be read, and TMEM allocated, before the
  // dependency wait
  int keys_ready;
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
  sm100::pdl_launch_dependents();  // the scorer waits for this kernel only where it reads qop and qsc
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

// Query preparation and the query operand in one kernel, for Hadamard
// quantizers of d = 32, 64, 128: one block of D threads per query.  y~ = R y
// by three rounds of signs and Walsh-Hadamard butterflies, p = S y~, then the
// query's five operand rows and its scales.  Every step repeats the
// arithmetic, in the same order, of the separate preparation
// (k_prep_fwht_block) and k_query_operand, so the scores are bit-identical
// whichever way the queries were prepared.
template <int D>
__global__ void __launch_bounds__(D)
k_prep_operand(KernelTables kt, RowSource src, int64_t G, int N, int cexp, int8_t *qop, float4 *qsc) {
  constexpr int NW = D / 32;
  __shared__ float v[D];
  __shared__ float red[2][NW];
  __shared__ int ired[NW];
  __shared__ __align__(16) int8_t stg[kColsPerQuery][kScoreKBytes];
  const int64_t row = blockIdx.x;
  const int j = threadIdx.x;
  sm100::pdl_launch_dependents();  // the scorer waits for this kernel only where it reads qop and qsc
  for (int i = j; i < kColsPerQuery * kScoreKBytes / 16; i += D) reinterpret_cast<uint4 *>(&stg[0][0])[i] = make_uint4(0, 0, 0, 0);
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
  __syncthreads();
  // p_j = sum_k S[j][k] y~_k: thread j reads row j of S with independent
  // 16-byte loads (one L2 round trip), four partial sums over k mod 4
  float acc0 = 0.f, acc1 = 0.f, acc2 = 0.f, acc3 = 0.f;
  if (kt.m > 0 && kt.qjl_otf) {
    // row j of S generated from the seed (TurboQuant article 2.3.2): the
    // same fp16 values, the same summation order
    const uint64_t base = (uint64_t)j * D;
#pragma unroll 4
    for (int k4 = 0; k4 < D / 4; ++k4) {
      acc0 = fmaf(half_bits_to_float(qjl_entry_f16(kt.qjl_key, base + 4 * k4)), v[4 * k4], acc0);
      acc1 = fmaf(half_bits_to_float(qjl_entry_f16(kt.qjl_key, base + 4 * k4 + 1)), v[4 * k4 + 1], acc1);
      acc2 = fmaf(half_bits_to_float(qjl_entry_f16(kt.qjl_key, base + 4 * k4 + 2)), v[4 * k4 + 2], acc2);
      acc3 = fmaf(half_bits_to_float(qjl_entry_f16(kt.qjl_key, base + 4 * k4 + 3)), v[4 * k4 + 3], acc3);
    }
  } else if (kt.m > 0) {  // TurboQuant-MSE quantizers have no QJL projection (p = 0)
    const float4 *srow = reinterpret_cast<const float4 *>(kt.qjl32 + (size_t)j * D);
#pragma unroll
    for (int k4 = 0; k4 < D / 4; ++k4) {
      const float4 s4 = __ldg(srow + k4);
      acc0 = fmaf(s4.x, v[4 * k4], acc0);
      acc1 = fmaf(s4.y, v[4 * k4 + 1], acc1);
      acc2 = fmaf(s4.z, v[4 * k4 + 2], acc2);
      acc3 = fmaf(s4.w, v[4 * k4 + 3], acc3);
    }
  }
  const float pj = (acc0 + acc1) + (acc2 + acc3);
  // largest |y~| and |p|: power-of-two scales of the 16-bit fixed point
  float ay = fabsf(x), ap = fabsf(pj);
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) {
    ay = fmaxf(ay, __shfl_xor_sync(0xffffffffu, ay, o));
    ap = fmaxf(ap, __shfl_xor_sync(0xffffffffu, ap, o));
  }
  if (j % 32 == 0) {
    red[0][j / 32] = ay;
    red[1][j / 32] = ap;
  }
  __syncthreads();
  ay = red[0][0];
  ap = red[1][0];
#pragma unroll
  for (int k = 1; k < NW; ++k) {
    ay = fmaxf(ay, red[0][k]);
    ap = fmaxf(ap, red[1][k]);
  }
  int ey = 0, ep = 0;
  frexpf(ay, &ey);
  frexpf(ap, &ep);
  const int sy = ay > 0.f ? 14 - ey : 0;
  const int sp = ap > 0.f ? 14 - ep : 0;
  {
    const int vi = __float2int_rn(ldexpf(x, sy));
    const int hi = (vi + 128) >> 8, lo = vi - 256 * hi;
    const int k = (j / 32) * 32 + code_byte_pos(kt.w, j % 32);
    stg[0][k] = (int8_t)hi;
    stg[1][k] = (int8_t)lo;
    stg[1][128 + k] = (int8_t)hi;
    stg[2][128 + k] = (int8_t)lo;
  }
  const int pv = __float2int_rn(ldexpf(pj, sp));
  {
    const int hi = (pv + 128) >> 8, lo = pv - 256 * hi;
    const int k = 256 + (j / 32) * 32 + sign_byte_pos(j % 32);
    stg[3][k] = (int8_t)hi;
    stg[4][k] = (int8_t)lo;
  }
  int psum = pv;
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) psum += __shfl_xor_sync(0xffffffffu, psum, o);
  if (j % 32 == 0) ired[j / 32] = psum;
  __syncthreads();
  // the five rows, 16 bytes at a time, where the 128-byte-swizzled tile keeps them
  const int64_t g = row / G, ql = row % G;
  int8_t *img = qop + g * (int64_t)N * kScoreKBytes;
  const int n0 = kColsPerQuery * (int)ql;
  for (int t = j; t < kColsPerQuery * (kScoreKBytes / 16); t += D) {
    const int r = t / (kScoreKBytes / 16), c = t % (kScoreKBytes / 16);
    *reinterpret_cast<uint4 *>(img + (c / 8) * (N * 128) + sm100::sw128_offset(n0 + r, c % 8)) =
        *reinterpret_cast<const uint4 *>(&stg[r][16 * c]);
  }
  if (j == 0) {
    int tot = 0;
#pragma unroll
    for (int k = 0; k < NW; ++k) tot += ired[k];
    qsc[row] = make_float4(ldexpf(1.f, -(sy + cexp)), ldexpf(kt.qjl_scale, -sp), (float)tot, 0.f);
  }
}


// ------------------------------------------------------------------ scorer
// Warp-specialised, one persistent CTA per SM walking a contiguous range of
// 128-key tiles (a group's tiles are contiguous):
//   warps 0-3    expanders: thread (warp, lane) expands key row 32 warp + lane
//                into one of the key operands in TMEM (up to four, so the
//                expanders run ahead of the MMAs; a second group of four
//                expander warps taking alternate tiles measured no faster);
//   warps 4-11   epilogue, two per TMEM lane quarter, queries split between
//                them; scores of a tile from its TMEM accumulator;
//   warps 12-13  MMA issue, one thread each, alternate tiles (a single issuer
//                when only one accumulator fits): an issuing thread spends
//                tens of cycles per tcgen05 instruction, so two of them keep
//                the tensor core fed;
//   warp 14      bulk copies: raw key rows into a ring of p.nstages buffers, and
//                each group's query operand into a ring of two.
// Hand-offs are mbarriers only.  Every wait is bounded and gives up as soon
// as another role has failed, after which all roles leave their loops,
// in-flight copies and MMAs are waited for (bounded) and TMEM is freed.
// Up to 12 stages of 8 KB (d = 128, b = 4) keep about 100 KB of key rows in
// flight per SM: enough to cover HBM latency at full bandwidth (4 stages
// capped the scorer near 3 TB/s).  Fewer when many queries per group leave
// less shared memory (p.nstages, at least 2).
constexpr int kStages = 12;
constexpr int kExpGroups = 1;  // expander groups (four warps each) taking tiles in turn
constexpr int kExpWarps = 4 * kExpGroups, kEpiWarps = 8;
constexpr int kMmaWarp = kExpWarps + kEpiWarps;  // and kMmaWarp + 1: the two MMA issuers
constexpr int kLoadWarp = kMmaWarp + 2;
constexpr int kScoreThreads = (kLoadWarp + 1) * 32;
constexpr int kACols = kScoreKBytes / 4;  // TMEM columns of one key operand

// TMEM plan of one CTA: nacc accumulators of N columns (rounded to 32), then
// 32 columns of slack when the epilogue's 16-column loads of the last queries
// reach past an accumulator, then nab key operands.  Where columns allow,
// four accumulators (the MMAs of a tile need not wait for the scores of the
// tile two before) and two key operands per expander group (a group fills
// one while the MMAs read the other).
struct ScoreTmem {
  int stride, lgacc, nacc, nab, dcols, ncols;
  __host__ __device__ ScoreTmem(int N, int64_t G) {
    stride = (N + 31) / 32 * 32;
    const int slack = kColsPerQuery * (int)G + 11 > stride ? 32 : 0;
    auto fit = [&](int na, int nb) { return na * stride + slack + nb * kACols <= 512; };
    if (fit(4, 4)) {
      lgacc = 2;
      nab = 4;
    } else {
      lgacc = fit(2, 2) ? 1 : 0;
      nab = fit(1 << lgacc, 4) ? 4 : 2;
    }
    nacc = 1 << lgacc;
    dcols = nacc * stride + slack;
    const int used = dcols + nab * kACols;
    ncols = 32;
    while (ncols < used) ncols <<= 1;
  }
  __host__ __device__ int acc(int b) const { return b * stride; }
  __host__ __device__ int a(int e) const { return dcols + e * kACols; }
};

// (group, tile in group) of a walk over the CTA's tiles with a fixed stride,
// advanced without 64-bit division.
struct TileWalk {
  int64_t g, tin, tpg;
  __device__ TileWalk(int64_t t, int64_t tiles_per_group) : g(t / tiles_per_group), tin(t % tiles_per_group),
                                                            tpg(tiles_per_group) {}
  __device__ void advance(int stride) {
    tin += stride;
    while (tin >= tpg) {
      tin -= tpg;
      ++g;
    }
  }
};

template <int W, int NG>
struct ScoreSmem {
  static constexpr int kCW = W * NG;                // code words per key
  static constexpr int kCodeBytes = 128 * kCW * 4;  // per stage
  static constexpr int kSignBytes = 128 * NG * 4;
  static constexpr int kStageBytes = (kCodeBytes + kSignBytes + 1023) / 1024 * 1024;  // 1024-aligned stages
  // the query operands follow the p.nstages stages (stage bytes are a multiple of 1024)
  enum Bar { kFull = 0, kEmpty = kStages, kAFull = 2 * kStages, kAEmpty = kAFull + 4, kAccFull = kAEmpty + 4,
             kAccEmpty = kAccFull + 4, kBFull = kAccEmpty + 4, kBEmpty = kBFull + 2, kMmaDone = kBEmpty + 2,
             kNumBars = kMmaDone + 2 };
};

template <int W, int NG, bool BULK>
__global__ void __launch_bounds__(kScoreThreads, 1)
k_score_tc(const ScoreTCParams p) {
  using SM = ScoreSmem<W, NG>;
  constexpr int CW = SM::kCW;
  extern __shared__ uint8_t smem_raw[];
  uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t *sStage = smem;
  uint8_t *sB = smem + (BULK ? p.nstages * SM::kStageBytes : 0);
  const int NS = p.nstages;
  const uint32_t b_bytes = (uint32_t)p.N * kScoreKBytes;  // one query operand
  uint64_t *bars = reinterpret_cast<uint64_t *>(sB + 2 * b_bytes);
  uint32_t *sTmem = reinterpret_cast<uint32_t *>(bars + SM::kNumBars);
  volatile int *sAbort = reinterpret_cast<volatile int *>(sTmem + 1);

  const int tid = threadIdx.x, warp = tid / 32, lane = tid % 32;
  const ScoreTmem tp(p.N, p.G);
  const int64_t t0 = (p.ntiles * blockIdx.x) / gridDim.x;
  const int64_t t1 = (p.ntiles * (blockIdx.x + 1)) / gridDim.x;
  const int n_it = (int)(t1 - t0);
  const int64_t tpg = p.tiles_per_group;
  const int64_t g0 = t0 / tpg;  // groups are counted from the CTA's first one
  const int nis = tp.nacc >= 2 ? 2 : 1;  // MMA issuers
  if (tid == 0) {
    for (int i = 0; i < NS; ++i) {
      sm100::mbar_init(&bars[SM::kFull + i], 1);
      sm100::mbar_init(&bars[SM::kEmpty + i], 4);
    }
    for (int i = 0; i < 4; ++i) {
      sm100::mbar_init(&bars[SM::kAFull + i], 4);
      sm100::mbar_init(&bars[SM::kAEmpty + i], 1);
    }
    for (int i = 0; i < 4; ++i) {
      sm100::mbar_init(&bars[SM::kAccFull + i], 1);
      sm100::mbar_init(&bars[SM::kAccEmpty + i], kEpiWarps);
    }
    for (int i = 0; i < 2; ++i) {
      sm100::mbar_init(&bars[SM::kBFull + i], 1);
      sm100::mbar_init(&bars[SM::kBEmpty + i], nis);
      sm100::mbar_init(&bars[SM::kMmaDone + i], 1);
    }
    *sAbort = 0;
    sm100::fence_barrier_init();
  }
  // After any other kernel, wait for it first: it may have written the keys,
  // and a TMEM allocation that has to wait for another kernel's columns also
  // holds up that kernel's MMAs on this SM.
  if (!p.keys_ready) sm100::pdl_wait();
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
  int64_t issued = 0;  // tiles the load warp has passed (their key stages and query operands issued)
  int64_t pre = 0;     // key stages issued ahead of the first query operand (load warp)
  int b_loaded = 0;    // query operands issued (load warp)
  int mma_issued = 0;  // tiles whose MMAs this thread issued (MMA issuers)

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
    TileWalk tw(t0 + e, tpg);
    // ring slot of tile it and the parity of its fill, kept as counters
    // (it % NS and (it / NS) & 1 without a division per tile)
    int slot = e % NS;
    uint32_t fill_ph = (uint32_t)((e / NS) & 1);
    for (int it = e; it < n_it; it += kExpGroups, tw.advance(kExpGroups)) {
      const int64_t g = tw.g, kin = tw.tin * 128 + row;
      const bool valid = kin < p.nkeys;
      uint32_t cw[CW], sw[NG];
#pragma unroll
      for (int k = 0; k < CW; ++k) cw[k] = 0u;
#pragma unroll
      for (int k = 0; k < NG; ++k) sw[k] = 0u;
      if constexpr (BULK) {
        if (!__all_sync(0xffffffffu, wait(SM::kFull + slot, fill_ph, 21))) break;
        const uint8_t *st = sStage + slot * SM::kStageBytes;
        if (valid) {
          if constexpr (CW % 4 == 0) {
            const uint4 *crow = reinterpret_cast<const uint4 *>(st + row * CW * 4);
#pragma unroll
            for (int k = 0; k < CW / 4; ++k) {
              const uint4 v = crow[k];
              cw[4 * k] = v.x;
              cw[4 * k + 1] = v.y;
              cw[4 * k + 2] = v.z;
              cw[4 * k + 3] = v.w;
            }
          } else {
            const uint32_t *crow = reinterpret_cast<const uint32_t *>(st + row * CW * 4);
#pragma unroll
            for (int k = 0; k < CW; ++k) cw[k] = crow[k];
          }
          if (p.m > 0) {
            const uint32_t *srow = reinterpret_cast<const uint32_t *>(st + SM::kCodeBytes + row * NG * 4);
#pragma unroll
            for (int k = 0; k < NG; ++k) sw[k] = srow[k];
          }
        }
        __syncwarp();
        if (lane == 0) sm100::mbar_arrive(&bars[SM::kEmpty + slot]);
        for (slot += kExpGroups; slot >= NS; slot -= NS) fill_ph ^= 1u;
      } else {
        if (valid) {
          const int64_t key = g * p.kpg + p.key_base + kin;
#pragma unroll
          for (int k = 0; k < CW; ++k) cw[k] = __ldg(p.codes + key * CW + k);
          if (p.m > 0) {
#pragma unroll
            for (int k = 0; k < NG; ++k) sw[k] = __ldg(p.signs + key * NG + k);
          }
        }
      }
      // key operand buffer it % nab was last read by the MMAs of tile it - nab
      const int ea = tp.nab == 4 ? (it & 3) : (it & 1), use = tp.nab == 4 ? (it >> 2) : (it >> 1);
      if (use > 0 && !__all_sync(0xffffffffu, wait(SM::kAEmpty + ea, (uint32_t)((use - 1) & 1), 22))) break;
      sm100::tc_fence_after();
      const uint32_t ta = tmem + tlane + (uint32_t)tp.a(ea);
#pragma unroll
      for (int gi = 0; gi < NG; ++gi) {
        uint32_t ch[8], cl[8], bt[8];
        expand_codes<W>(cw + gi * W, tch, tcl, ch, cl);
#pragma unroll
        for (int k = 0; k < 8; ++k) bt[k] = (sw[gi] >> k) & 0x01010101u;
        sm100::tmem_st8(ta + 8 * gi, ch);
        sm100::tmem_st8(ta + 32 + 8 * gi, cl);
        if (p.m > 0) sm100::tmem_st8(ta + 64 + 8 * gi, bt);  // uniform: no sign bytes in TurboQuant-MSE
      }
      sm100::tmem_wait_st();
      sm100::tc_fence_before();
      __syncwarp();
      if (lane == 0) sm100::mbar_arrive(&bars[SM::kAFull + ea]);
    }
  } else if (warp < kMmaWarp) {
    // ------------------------------------------------------------ epilogue
    sm100::pdl_wait();  // the query scales (qsc) are final from here on
    const int quarter = warp % 4, eh = (warp - kExpWarps) / 4, row = 32 * quarter + lane;
    const int q_half = (int)((p.G + 1) / 2);
    const int q_lo = eh ? q_half : 0, q_hi = eh ? (int)p.G : q_half;
    const uint32_t tlane = (uint32_t)(32 * quarter) << 16;
    // the norms of a tile are loaded two tiles ahead: the accumulator is often
    // ready by the time the epilogue gets to it, so the load would not hide
    auto norms_of = [&](const TileWalk &w, int i) {
      const int64_t k = w.tin * 128 + row;
      return i < n_it && k < p.nkeys ? __ldg(p.norms + w.g * p.kpg + p.key_base + k) : make_float2(0.f, 0.f);
    };
    TileWalk tw(t0, tpg), tw2(t0, tpg);
    float2 nr_next = norms_of(tw2, 0);
    tw2.advance(1);
    float2 nr_next2 = norms_of(tw2, 1);
    tw2.advance(1);
    for (int it = 0; it < n_it; ++it, tw.advance(1), tw2.advance(1)) {
      const int64_t g = tw.g, kin = tw.tin * 128 + row;
      const bool valid = kin < p.nkeys;
      const float2 nr = nr_next;
      nr_next = nr_next2;
      nr_next2 = norms_of(tw2, it + 2);
      const int ab = it & (tp.nacc - 1), use = it >> tp.lgacc;
      if (!__all_sync(0xffffffffu, wait(SM::kAccFull + ab, (uint32_t)(use & 1), 23))) break;
      sm100::tc_fence_after();
      const uint32_t taddr = tmem + tlane + (uint32_t)tp.acc(ab);
      const float4 *qs = p.qsc + g * p.G;
      float *orow = p.out + g * p.G * p.ldo + kin;
      auto score = [&](const uint32_t *dv, const float4 &sc) {
        const int *v = reinterpret_cast<const int *>(dv);
        const int sb = 2 * (256 * v[3] + v[4]) - (int)sc.z;
        const float a = fmaf((float)v[0], 65536.f, fmaf((float)v[1], 256.f, (float)v[2])) * sc.x;
        return nr.x * fmaf(nr.y * sc.y, (float)sb, a);
      };
      auto put = [&](int q, float sres) {
        float *o = orow + q * p.ldo;
        if (p.accumulate) sres += *o;
        *o = sres;
      };
      if (q_hi - q_lo <= 6) {
        // at most six queries: take the columns, free the accumulator, then score
        uint32_t d0[16], d1[16];
        float4 sc[6];
        sm100::tmem_ld16(taddr + kColsPerQuery * q_lo, d0);
        if (q_hi - q_lo > 3) sm100::tmem_ld16(taddr + kColsPerQuery * (q_lo + 3), d1);
#pragma unroll
        for (int qq = 0; qq < 6; ++qq)
          sc[qq] = q_lo + qq < q_hi ? __ldg(qs + q_lo + qq) : make_float4(0.f, 0.f, 0.f, 0.f);
        sm100::tmem_wait_ld();
        sm100::tc_fence_before();
        __syncwarp();
        if (lane == 0) sm100::mbar_arrive(&bars[SM::kAccEmpty + ab]);
        if (valid) {
#pragma unroll
          for (int qq = 0; qq < 6; ++qq)
            if (q_lo + qq < q_hi) put(q_lo + qq, score(qq < 3 ? d0 + kColsPerQuery * qq : d1 + kColsPerQuery * (qq - 3), sc[qq]));
        }
        continue;
      }
      for (int q0 = q_lo; q0 < q_hi; q0 += 3) {  // 15 of 16 loaded columns = 3 queries
        uint32_t dv[16];
        sm100::tmem_ld16(taddr + kColsPerQuery * q0, dv);
        float4 sc[3];
#pragma unroll
        for (int qq = 0; qq < 3; ++qq) sc[qq] = q0 + qq < q_hi ? __ldg(qs + q0 + qq) : make_float4(0.f, 0.f, 0.f, 0.f);
        sm100::tmem_wait_ld();
        if (valid) {
#pragma unroll
          for (int qq = 0; qq < 3; ++qq)
            if (q0 + qq < q_hi) put(q0 + qq, score(dv + kColsPerQuery * qq, sc[qq]));
        }
      }
      sm100::tc_fence_before();
      __syncwarp();
      if (lane == 0) sm100::mbar_arrive(&bars[SM::kAccEmpty + ab]);
    }
  } else if (warp < kLoadWarp) {
    // ------------------------------------------------------------ MMA issue
    const int e = warp - kMmaWarp;
    if (lane == 0 && e < nis) {
      const uint32_t idesc = sm100::idesc_s8_s32(128, p.N);
      uint64_t bdesc[kScoreKBytes / 32];  // K-steps of the current query operand
      int jcur = 0;                       // group (from g0) of the operand held
      bool have_b = false, used = false;
      TileWalk tw(t0 + e, tpg);
      for (int it = e; it < n_it; it += nis, tw.advance(nis)) {
        const int j = (int)(tw.g - g0);
        if (!have_b || j != jcur) {
          // release the operands of groups passed (committed: freed when this
          // thread's MMAs reading them complete), then take the new one
          for (int jj = jcur; jj < j; ++jj) {
            if (jj == jcur && used)
              sm100::mma_commit(&bars[SM::kBEmpty + (jj & 1)]);
            else
              sm100::mbar_arrive(&bars[SM::kBEmpty + (jj & 1)]);
          }
          jcur = j;
          used = false;
          if (!wait(SM::kBFull + (j & 1), (uint32_t)((j >> 1) & 1), 24)) break;
          have_b = true;
          const uint32_t b0 = sm100::smem_u32(sB + (j & 1) * b_bytes);
#pragma unroll
          for (int ks = 0; ks < kScoreKBytes / 32; ++ks)
            bdesc[ks] = sm100::desc_sw128(b0 + (ks / 4) * (p.N * 128) + (ks % 4) * 32);
        }
        const int ea = tp.nab == 4 ? (it & 3) : (it & 1), auses = tp.nab == 4 ? (it >> 2) : (it >> 1);
        const int ab = it & (tp.nacc - 1), ause = it >> tp.lgacc;
        if (!wait(SM::kAFull + ea, (uint32_t)(auses & 1), 26)) break;
        if (ause > 0 && !wait(SM::kAccEmpty + ab, (uint32_t)((ause - 1) & 1), 27)) break;
        sm100::tc_fence_after();
        const uint32_t ta = tmem + (uint32_t)tp.a(ea), td = tmem + (uint32_t)tp.acc(ab);
#pragma unroll
        for (int ks = 0; ks < kScoreKBytes / 32; ++ks) {
          if (ks % 4 >= NG) continue;       // coordinates beyond d
          if (ks >= 8 && p.m == 0) continue;  // TurboQuant-MSE: no sign-bit K range
          sm100::mma_i8_ts(td, ta + 8 * ks, bdesc[ks], idesc, ks != 0);
        }
        sm100::mma_commit(&bars[SM::kAEmpty + ea]);
        sm100::mma_commit(&bars[SM::kAccFull + ab]);
        used = true;
        ++mma_issued;
      }
    }
  } else if (lane == 0) {
    // ------------------------------------------------------------ copies
    // key rows of tile jt into ring slot jt % NS (the slot is free)
    auto issue_keys = [&](int jt, const TileWalk &w) {
      const int slot = jt % NS;
      const int64_t kin0 = w.tin * 128;
      const int64_t key0 = w.g * p.kpg + p.key_base + kin0;
      const int64_t left = p.nkeys - kin0;
      const int rows = left < 128 ? (int)left : 128;
      uint8_t *st = sStage + slot * SM::kStageBytes;
      const uint32_t cb = rows * CW * 4, sb = p.m > 0 ? rows * NG * 4 : 0;
      sm100::mbar_expect_tx(&bars[SM::kFull + slot], cb + sb);
      sm100::bulk_load(st, p.codes + key0 * CW, cb, &bars[SM::kFull + slot]);
      if (sb) sm100::bulk_load(st + SM::kCodeBytes, p.signs + key0 * NG, sb, &bars[SM::kFull + slot]);
    };
    // The key stages that fit in the ring go first: after the query-side
    // kernel (keys_ready) the keys were complete before it started, and
    // otherwise this thread has waited already; the query operands come from
    // that kernel, which may still be running.
    if constexpr (BULK) {
      TileWalk tp(t0, tpg);
      for (; pre < n_it && pre < NS; ++pre, tp.advance(1)) issue_keys((int)pre, tp);
    }
    sm100::pdl_wait();  // the query operands (qop) are final from here on
    TileWalk tw(t0, tpg);
    for (; issued < n_it; ++issued, tw.advance(1)) {
      const int j = (int)(tw.g - g0);
      if (j == b_loaded) {  // first tile of a group: its query operand
        if (j >= 2 && !wait(SM::kBEmpty + (j & 1), (uint32_t)(((j >> 1) - 1) & 1), 30)) break;
        sm100::mbar_expect_tx(&bars[SM::kBFull + (j & 1)], b_bytes);
        sm100::bulk_load(sB + (j & 1) * b_bytes, p.qop + tw.g * (int64_t)b_bytes, b_bytes, &bars[SM::kBFull + (j & 1)]);
        ++b_loaded;
      }
      if constexpr (BULK) {
        const int jt = (int)issued;
        if (jt < pre) continue;  // issued ahead
        if (!wait(SM::kEmpty + jt % NS, (uint32_t)((jt / NS - 1) & 1), 28)) break;
        issue_keys(jt, tw);
      }
    }
  }
  // ------------------------------------------------------------ teardown
  __syncthreads();
  if (warp >= kMmaWarp && warp < kLoadWarp && lane == 0 && mma_issued > 0) {
    // no MMA may still write TMEM when it is freed
    sm100::mma_commit(&bars[SM::kMmaDone + (warp - kMmaWarp)]);
    sm100::mbar_wait(&bars[SM::kMmaDone + (warp - kMmaWarp)], 0u, p.err, 29);
  }
  if (warp == kLoadWarp && lane == 0 && *sAbort) {
    // copies issued but possibly not consumed: the last p.nstages key stages
    // and the last two query operands
    if constexpr (BULK) {
      const int64_t kst = issued > pre ? issued : pre;  // key stages issued
      for (int64_t j = kst > NS ? kst - NS : 0; j < kst; ++j)
        sm100::mbar_wait(&bars[SM::kFull + j % NS], (uint32_t)((j / NS) & 1), p.err, 31);
    }
    for (int j = b_loaded > 2 ? b_loaded - 2 : 0; j < b_loaded; ++j)
      sm100::mbar_wait(&bars[SM::kBFull + (j & 1)], (uint32_t)((j >> 1) & 1), p.err, 32);
  }
  sm100::tc_fence_before();
  __syncthreads();
  sm100::tc_fence_after();
  if (warp == kMmaWarp) sm100::tmem_dealloc(tmem, (uint32_t)tp.ncols);
}

// ------------------------------------------------------------------ failure self-test
// An mbarrier expecting one arrival that never comes: the bounded wait gives
// up after its limit (about 2 s), records code 99 and the kernel returns.
__global__ void k_wait_selftest(int *err) {
  __shared__ uint64_t bar;
  if (threadIdx.x == 0) {
    sm100::mbar_init(&bar, 1);
    sm100::fence_barrier_init();
  }
  __syncthreads();
  if (threadIdx.x == 0) sm100::mbar_wait(&bar, 0u, err, 99);
}

tq_status launch_wait_selftest(int *err, cudaStream_t st) {
  k_wait_selftest<<<1, 32, 0, st>>>(err);
  return cudaGetLastError() == cudaSuccess ? TQ_OK : TQ_ERR_CUDA;
}

// ------------------------------------------------------------------ host side
bool tc_score_supported(const tq_quantizer *q, int64_t G) {
  return q->d <= 128 && q->d % 32 == 0 && (q->m == q->d || q->m == 0) && G >= 1 && G <= kMaxScoreG;
}

size_t tc_score_qop_bytes(const tq_quantizer *q, int64_t groups, int64_t G) {
  const int64_t N = (kColsPerQuery * G + 15) / 16 * 16;
  return (size_t)groups * N * kScoreKBytes;
}

tq_status tc_score_queries(const tq_quantizer *q, const float *ytil, const float *pq, int64_t groups, int64_t G,
                           int8_t *qop, float4 *qsc, cudaStream_t st) {
  const int N = (int)((kColsPerQuery * G + 15) / 16 * 16);
  const int64_t nq = groups * G;
  if (cudaMemsetAsync(qop, 0, tc_score_qop_bytes(q, groups, G), st) != cudaSuccess) return TQ_ERR_CUDA;
  k_query_operand<<<(unsigned)nq, 128, 0, st>>>(ytil, pq, q->d, q->m, q->w, G, N, q->score_cexp, q->kt.qjl_scale,
                                                qop, qsc);
  return cudaGetLastError() == cudaSuccess ? TQ_OK : TQ_ERR_CUDA;
}

tq_status tc_score(const tq_quantizer *q, const float *ytil, const float *pq, int64_t groups, int64_t G,
                   int64_t kpg, int64_t key_base, int64_t nkeys, const void *codes, const void *signs,
                   const float *norms, float *out, int64_t ldo, int accumulate, int8_t *qop, float4 *qsc,
                   cudaStream_t st) {
  const tq_status r = tc_score_queries(q, ytil, pq, groups, G, qop, qsc, st);
  if (r != TQ_OK) return r;
  return tc_score_keys(q, groups, G, kpg, key_base, nkeys, codes, signs, norms, out, ldo, accumulate, qop, qsc,
                       true, st);
}

bool tc_score_y_supported(const tq_quantizer *q, int64_t G) {
  return tc_score_supported(q, G) && q->rotation == TQ_ROT_HADAMARD &&
         (q->d == 32 || q->d == 64 || q->d == 128) && q->kt.diag_bits;
}

tq_status tc_score_y_queries(const tq_quantizer *q, const RowSource &src, int64_t groups, int64_t G, int8_t *qop,
                             float4 *qsc, cudaStream_t st) {
  const int N = (int)((kColsPerQuery * G + 15) / 16 * 16);
  const unsigned nq = (unsigned)(groups * G);
  switch (q->d) {
    case 32: k_prep_operand<32><<<nq, 32, 0, st>>>(q->kt, src, G, N, q->score_cexp, qop, qsc); break;
    case 64: k_prep_operand<64><<<nq, 64, 0, st>>>(q->kt, src, G, N, q->score_cexp, qop, qsc); break;
    case 128: k_prep_operand<128><<<nq, 128, 0, st>>>(q->kt, src, G, N, q->score_cexp, qop, qsc); break;
    default: return TQ_ERR_UNSUPPORTED;
  }
  return cudaGetLastError() == cudaSuccess ? TQ_OK : TQ_ERR_CUDA;
}

tq_status tc_score_y(const tq_quantizer *q, const RowSource &src, int64_t groups, int64_t G, int64_t kpg,
                     const void *codes, const void *signs, const float *norms, float *out, int64_t ldo,
                     int accumulate, int8_t *qop, float4 *qsc, cudaStream_t st) {
  const tq_status r = tc_score_y_queries(q, src, groups, G, qop, qsc, st);
  if (r != TQ_OK) return r;
  return tc_score_keys(q, groups, G, kpg, 0, kpg, codes, signs, norms, out, ldo, accumulate, qop, qsc, true, st);
}

tq_status tc_score_keys(const tq_quantizer *q, int64_t groups, int64_t G, int64_t kpg, int64_t key_base,
                        int64_t nkeys, const void *codes, const void *signs, const float *norms, float *out,
                        int64_t ldo, int accumulate, const int8_t *qop, const float4 *qsc, bool keys_ready,
                        cudaStream_t st) {
  const int N = (int)((kColsPerQuery * G + 15) / 16 * 16);
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
  prm.keys_ready = keys_ready ? 1 : 0;
  prm.err = q->d_err;
  const int ng = q->d / 32, cwords = q->w * ng;
  const size_t stage_bytes = ((size_t)128 * (cwords + ng) * 4 + 1023) / 1024 * 1024;
  // bulk copies need 16-byte aligned starts and sizes: with d = 128 a key's
  // code and sign rows are multiples of 16 bytes, so any tile qualifies;
  // otherwise every tile's first key and every tile's length must be a
  // multiple of 4 keys
  const bool rows4 = key_base % 4 == 0 && kpg % 4 == 0 && nkeys % 4 == 0;
  const bool bulk = (ng == 4 || rows4) && reinterpret_cast<uintptr_t>(codes) % 16 == 0 &&
                    (q->m == 0 || reinterpret_cast<uintptr_t>(signs) % 16 == 0);
  if (reinterpret_cast<uintptr_t>(qop) % 16 != 0) return TQ_ERR_ALIGNMENT;
  int max_smem = 0;
  {
    int dv = 0;
    cudaGetDevice(&dv);
    cudaDeviceGetAttribute(&max_smem, cudaDevAttrMaxSharedMemoryPerBlockOptin, dv);
  }
  const size_t fixed = 1024 + 2 * (size_t)N * kScoreKBytes + 8 * (2 * kStages + 26) + 16;
  int nstages = kStages;
  while (bulk && nstages > 2 && fixed + nstages * stage_bytes > (size_t)max_smem) --nstages;
  prm.nstages = nstages;
  const size_t smem = fixed + (bulk ? nstages * stage_bytes : 0);
  int dev = 0, sms = 0;
  cudaGetDevice(&dev);
  cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  const int64_t grid = std::min<int64_t>(prm.ntiles, (int64_t)sms);
  if (grid <= 0) return TQ_OK;
  // Programmatic dependent launch: after the query-side kernel (which lets
  // its dependents start at once) the scorer sets up and loads keys while
  // that kernel still runs; its threads wait for it where they read qop and
  // qsc.  After any other kernel it waits for that kernel before anything
  // else (keys_ready = 0).
  cudaLaunchAttribute pdl{};
  pdl.id = cudaLaunchAttributeProgrammaticStreamSerialization;
  pdl.val.programmaticStreamSerializationAllowed = 1;
  cudaLaunchConfig_t cfg{};
  cfg.gridDim = dim3((unsigned)grid);
  cfg.blockDim = dim3(kScoreThreads);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = st;
  cfg.attrs = &pdl;
  cfg.numAttrs = 1;
#define TQ_SC(WW, NGG)                                                                                   \
  {                                                                                                      \
    auto kern = bulk ? k_score_tc<WW, NGG, true> : k_score_tc<WW, NGG, false>;                           \
    if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem) != cudaSuccess) \
      return TQ_ERR_CUDA;                                                                                \
    if (cudaLaunchKernelEx(&cfg, kern, prm) != cudaSuccess) return TQ_ERR_CUDA;                          \
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

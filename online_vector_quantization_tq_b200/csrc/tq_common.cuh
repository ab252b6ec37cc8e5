// Device helpers shared by the libtq kernels: input loads, the packed code
// layout (documented in include/tq.h), in-register Walsh-Hadamard transform.
#pragma once

#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <cuda_runtime.h>

#include <cstdint>

#include "tq_internal.h"

namespace tq {

// Element `col` of row `row` of an fp32 or bf16 input, optionally gathered
// through a per-group channel map chan[(row / chan_rows) * d + j].
struct RowSource {
  const void *x;
  int64_t ldx;
  const int32_t *chan;
  int64_t chan_rows;
  int d;
  int bf16;
  __device__ __forceinline__ float at(int64_t row, int j) const {
    const int c = chan ? chan[(row / chan_rows) * d + j] : j;
    const int64_t off = row * ldx + c;
    if (bf16) {
      const uint16_t v = static_cast<const uint16_t *>(x)[off];
      return __uint_as_float(static_cast<uint32_t>(v) << 16);
    }
    return static_cast<const float *>(x)[off];
  }
};

// --- packed code layout -----------------------------------------------------
// Bit position (within the group's W words) of bit `bit` of the code of
// coordinate i (0..31) of a 32-coordinate group.  Returns word*32 + bit.
template <int W>
__host__ __device__ constexpr int code_bit_pos(int i, int bit) {
  return W == 1 ? i
       : W == 2 ? (i / 16) * 32 + 4 * (i % 8) + 2 * ((i / 8) % 2) + bit
       : W == 3 ? (i < 24 ? (i / 8) * 32 + 4 * (i % 8) + bit
                          : (2 - bit) * 32 + 4 * (i - 24) + 3)
       : /* W == 4 */ (i / 8) * 32 + 4 * (i % 8) + bit;
}

template <int W>
__device__ __forceinline__ int unpack_code(const uint32_t *g, int i) {
  int c = 0;
#pragma unroll
  for (int bit = 0; bit < W; ++bit) {
    const int p = code_bit_pos<W>(i, bit);
    c |= ((g[p >> 5] >> (p & 31)) & 1u) << bit;
  }
  return c;
}

template <int W>
__device__ __forceinline__ void pack_code(uint32_t *g, int i, uint32_t code) {
#pragma unroll
  for (int bit = 0; bit < W; ++bit) {
    const int p = code_bit_pos<W>(i, bit);
    g[p >> 5] |= ((code >> bit) & 1u) << (p & 31);
  }
}

// --- Walsh-Hadamard ---------------------------------------------------------
// Unnormalized Sylvester-order transform of D values held in registers.
template <int D>
__device__ __forceinline__ void fwht_regs(float (&v)[D]) {
#pragma unroll
  for (int h = 1; h < D; h <<= 1) {
#pragma unroll
    for (int i = 0; i < D; i += 2 * h) {
#pragma unroll
      for (int k = i; k < i + h; ++k) {
        const float a = v[k], b = v[k + h];
        v[k] = a + b;
        v[k + h] = a - b;
      }
    }
  }
}

// Multiply v by a +-1 diagonal given as bits (set = -1), words[j/32] bit j%32.
template <int D>
__device__ __forceinline__ void apply_signs(float (&v)[D], const uint32_t (&words)[D / 32]) {
#pragma unroll
  for (int j = 0; j < D; ++j)
    v[j] = __uint_as_float(__float_as_uint(v[j]) ^ (((words[j / 32] >> (j % 32)) & 1u) << 31));
}

// code = #{thresholds < u}; thresholds sorted, padded with +inf.
template <int L>
__device__ __forceinline__ int quantize(float u, const float *thr) {
  int c = 0;
#pragma unroll
  for (int i = 0; i < L - 1; ++i) c += (u > thr[i]) ? 1 : 0;
  return c;
}

__host__ __device__ constexpr int ceil_div_i(int64_t a, int64_t b) { return (int)((a + b - 1) / b); }

}  // namespace tq

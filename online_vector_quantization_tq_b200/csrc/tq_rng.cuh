// Device side of the quantizer's random draws: the entries of the QJL matrix
// S generated on the fly from the quantizer seed (TurboQuant article 2.3.2:
// a pseudo-random sequence stands in for the stored Gaussian matrix).
//
// The generator is the published SplitMix64 (Steele, Lea and Flood,
// OOPSLA 2014), indexed by counter: output k of the generator started from
// state s is mix64(s + (k + 1) * 0x9E3779B97F4A7C15), with Stafford's
// variant-13 mixer.  Entry i of S (row-major, m x d) is the Box-Muller draw
// (cosine branch) from outputs 2i and 2i+1 of S's stream,
//   u1 = (top53(w_2i) + 1) 2^-53,  u2 = top53(w_2i+1) 2^-53,
//   g  = sqrt(-2 ln u1) cos(2 pi u2)   (double precision),
// rounded once to fp16 (nearest, ties to even): the same numbers the host
// set-up stores.
#pragma once

#include <cstdint>

#include "tq_sm100.cuh"

namespace tq {

__device__ __forceinline__ uint64_t rng_mix64(uint64_t z) {
  z = (z ^ (z >> 30)) * 0xBF58476D1CE4E5B9ull;
  z = (z ^ (z >> 27)) * 0x94D049BB133111EBull;
  return z ^ (z >> 31);
}

__device__ __forceinline__ uint64_t rng_splitmix64(uint64_t state, uint64_t k) {
  return rng_mix64(state + (k + 1) * 0x9E3779B97F4A7C15ull);
}

// fp16 bit pattern of entry i of S for the stream key `key`
__device__ __forceinline__ uint16_t qjl_entry_f16(uint64_t key, uint64_t i) {
  const double u1 = ((double)(rng_splitmix64(key, 2 * i) >> 11) + 1.0) * 0x1.0p-53;
  const double u2 = (double)(rng_splitmix64(key, 2 * i + 1) >> 11) * 0x1.0p-53;
  const double g = sqrt(-2.0 * log(u1)) * cos(2.0 * 3.14159265358979323846 * u2);
  uint16_t h;
  asm("cvt.rn.f16.f64 %0, %1;" : "=h"(h) : "d"(g));
  return h;
}

__device__ __forceinline__ float half_bits_to_float(uint16_t h) {
  float f;
  asm("cvt.f32.f16 %0, %1;" : "=f"(f) : "h"(h));
  return f;
}

// S (D x D, the QJL rows as the MMA's N dimension, the input coordinates as
// K) generated into shared memory in the layout stage_kmajor<D> gives the
// stored table: 8 consecutive K elements per 16-byte chunk, 64-byte swizzle.
template <int D>
__device__ void generate_kmajor_qjl(uint8_t *dst, uint64_t key) {
  constexpr int chunks = D * (D / 8);
  for (int i = threadIdx.x; i < chunks; i += blockDim.x) {
    const int r = i / (D / 8), c8 = i % (D / 8);
    uint32_t w[4];
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      const uint64_t base = (uint64_t)r * D + c8 * 8 + 2 * e;
      w[e] = (uint32_t)qjl_entry_f16(key, base) | ((uint32_t)qjl_entry_f16(key, base + 1) << 16);
    }
    const int blk = c8 / 4, ch = c8 % 4;
    *reinterpret_cast<uint4 *>(dst + (size_t)blk * D * 64 + sm100::sw64_offset(r, ch)) =
        make_uint4(w[0], w[1], w[2], w[3]);
  }
}

}  // namespace tq

// Internal definitions shared by the host set-up code and the CUDA kernels
// of libtq.  Not part of the public ABI (see include/tq.h).
#pragma once

#include <cstddef>
#include <cstdint>
#include <vector>

#include "tq.h"

namespace tq {

constexpr int kMaxLevels = 16;  // 2^w for w <= 4

// Small, POD view of a quantizer that kernels take by value.
struct KernelTables {
  int d, w, m, levels;
  float centroids[kMaxLevels];
  float thresholds[kMaxLevels];       // levels-1 used; rest +inf
  float qjl_scale;                    // sqrt(pi/2) / m
  const uint32_t *diag_bits;          // Hadamard: 3 x d/32 words, bit set = -1
  const float *rot;                   // Haar: d x d row-major fp32 (u = R x)
  const uint16_t *qjl16;              // m x d fp16 bit patterns of S
  const float *qjl32;                 // m x d fp32 values of S (same numbers)
  const float *qjl32t;                // d x m: S transposed (coalesced S y~ over rows)
  const float *rott;                  // d x d: R transposed (d <= 128; coalesced R y over rows)
  uint64_t qjl_key;                   // SplitMix64 key of S's stream (entries generated from it)
  int qjl_otf;                        // nonzero: kernels that can generate S do so instead of reading it
};

}  // namespace tq

struct tq_quantizer {
  int d = 0, b = 0, w = 0, m = 0, rotation = 0, device = 0;
  uint64_t seed = 0;
  std::vector<double> centroids, thresholds;
  double coord_mse = 0.0;
  std::vector<float> rot;        // d x d fp32 (Haar, or the dense Hadamard product)
  std::vector<double> rot_exact; // d x d double (Hadamard product; empty for Haar)
  std::vector<int8_t> diag;      // 3 x d (Hadamard)
  std::vector<uint16_t> qjl16;   // m x d fp16 bits
  // device copies (owned)
  uint32_t *d_diag_bits = nullptr;
  float *d_rot = nullptr;
  uint16_t *d_qjl16 = nullptr;
  float *d_qjl32 = nullptr;
  float *d_qjl32t = nullptr;
  float *d_rott = nullptr;
  // tensor-core encode: R = tc_rho * (sum of tc_rot_pieces fp16 matrices)
  uint16_t *d_rot16 = nullptr;   // [pieces][d][d] fp16 bits
  int tc_rot_pieces = 0;
  float tc_rho = 0.f;
  uint16_t *d_rot_bf16 = nullptr;  // Hadamard: d^1.5 R as two exact bf16 pieces [2][d][d]
  uint16_t *d_rot_bf16x3 = nullptr;  // Haar (d <= 128): the fp32 R as three exact bf16 pieces [3][d][d]
  // dense tensor-core encode (d >= 256): R and S as 31-bit fixed point,
  // v 2^e = 2^24 a + 2^16 b + 2^8 c + d with signed bytes, stored as four
  // planes [4][rows][d] (a, b, c, d)
  int8_t *d_rot_limbs = nullptr;
  int rot_limb_exp = 0;
  int8_t *d_qjl_limbs = nullptr;
  int qjl_limb_exp = 0;
  int *d_err = nullptr;          // device error word (bounded waits that timed out)
  // integer scorer: centroid c_k ~ (256 * ch[k] + cl[k]) * 2^-score_cexp
  int8_t score_ch[tq::kMaxLevels] = {}, score_cl[tq::kMaxLevels] = {};
  int score_cexp = 0;
  tq::KernelTables kt{};
};

namespace tq {
// Host-side helpers exported for the CUDA translation unit.
uint16_t double_to_half_bits(double v);
double half_bits_to_double(uint16_t h);
}  // namespace tq

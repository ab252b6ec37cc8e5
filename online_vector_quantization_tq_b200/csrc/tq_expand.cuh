// Expansion of packed codes into bytes of value tables, four codes per PRMT
// (byte permute) of table words held in registers.  Used by the integer
// scorer (centroid limbs) and the attention consumer (fp16 centroids).
#pragma once

#include <cstdint>

#include "tq_sm100.cuh"

namespace tq {

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


}  // namespace tq

"""Unpacking of libtq's packed outputs, written from the layout documented in
include/tq.h (test helper; shares no code with the library)."""
import numpy as np


def code_bit_position(w: int, i: int, bit: int) -> int:
    """(word * 32 + bit) position of code bit `bit` of coordinate i of a
    32-coordinate group."""
    if w == 1:
        return i
    if w == 2:
        return (i // 16) * 32 + 4 * (i % 8) + 2 * ((i // 8) % 2) + bit
    if w == 3:
        if i < 24:
            return (i // 8) * 32 + 4 * (i % 8) + bit
        return (2 - bit) * 32 + 4 * (i - 24) + 3
    if w == 4:
        return (i // 8) * 32 + 4 * (i % 8) + bit
    raise ValueError(w)


def unpack_codes(codes_u8: np.ndarray, d: int, w: int) -> np.ndarray:
    """uint8 [n, w*d/8] -> int64 [n, d]."""
    n = codes_u8.shape[0]
    words = np.ascontiguousarray(codes_u8).view("<u4").reshape(n, d // 32, w)
    out = np.zeros((n, d // 32, 32), dtype=np.int64)
    for i in range(32):
        for bit in range(w):
            p = code_bit_position(w, i, bit)
            out[:, :, i] |= ((words[:, :, p // 32] >> np.uint32(p % 32)) & 1).astype(np.int64) << bit
    return out.reshape(n, d)


def unpack_signs(signs_u8: np.ndarray, m: int) -> np.ndarray:
    """uint8 [n, m/8] -> bool [n, m]; bit i of little-endian word i/32."""
    n = signs_u8.shape[0]
    words = np.ascontiguousarray(signs_u8).view("<u4").reshape(n, m // 32)
    bits = (words[:, :, None] >> np.arange(32, dtype=np.uint32)) & 1
    return bits.reshape(n, m).astype(bool)

"""Reads the packed W4A8 / W6A8 weight format back into codes and scales.

The layout is the one include/convrot.h documents for
convrot_quantize_weights_lowbit: tiles of 128 rows x 64 codes, each with
bits/2 planes of [128 rows][16 bytes] and then [128 rows][4 bytes] of E4M3
group scales; u = q + 2^(bits-1), the low four bits of code 8i+2j in bits
4j..4j+3 (code 8i+2j+1 in bits 16+4j..) of word i, and for 6 bits the top two
bits of code 16i+2j in bits 2j..2j+1 (code 16i+2j+1 in bits 16+2j..) of word
8+i. Plain NumPy; no arithmetic of the method.
"""

import numpy as np


def unpack_lowbit(data: np.ndarray, rows: int, k: int, bits: int):
    """Returns (q int8 [rows, K], sigma uint8 E4M3 codes [rows, K/16])."""
    planes = bits // 2
    tile = planes * 2048 + 512
    rb, kb = rows // 128, k // 64
    t = np.ascontiguousarray(data[: rb * kb * tile]).reshape(rb, kb, tile)
    cp = t[:, :, : planes * 2048].reshape(rb, kb, planes, 128, 16)
    row_bytes = np.ascontiguousarray(cp.transpose(0, 3, 1, 2, 4)).reshape(rb, 128, kb, planes * 16)
    words = row_bytes.view("<u4").astype(np.int64)  # [rb, 128, kb, 4 * planes]
    u = np.zeros((rb, 128, kb, 64), np.int64)
    for c in range(64):
        i, j, up = c >> 3, (c & 7) >> 1, c & 1
        u[..., c] = (words[..., i] >> (16 * up + 4 * j)) & 15
        if bits == 6:
            i2, j2 = c >> 4, (c & 15) >> 1
            u[..., c] |= ((words[..., 8 + i2] >> (16 * up + 2 * j2)) & 3) << 4
    q = (u - 2 ** (bits - 1)).reshape(rows, k).astype(np.int8)
    sc = t[:, :, planes * 2048:].reshape(rb, kb, 128, 4).transpose(0, 2, 1, 3)
    sigma = np.ascontiguousarray(sc).reshape(rows, kb * 4).astype(np.uint8)
    return q, sigma

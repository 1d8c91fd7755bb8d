"""The packed UINT4 weight format, restated for building test inputs by hand
(the format is this library's own; tests/golden/pack_layout.txt pins it).

Rows in tiles of 128 (the last tile has R = N mod 128 rows if that is not 0),
tile t starting at byte 128 t K/2; inside a tile, blocks of 128 K at b R 64;
inside a block, chunks of 32 K at c R 16; inside a chunk, row r's 16 bytes at
r 16, word j (little-endian) holding codes 8j..8j+7 of the chunk with byte i =
code[8j+i] | code[8j+4+i] << 4.
"""
import numpy as np


def pack_tiled(codes: np.ndarray) -> np.ndarray:
    """codes [N, K] (values 0..15, K a multiple of 32) -> qw [N, K/2] uint8."""
    codes = np.asarray(codes).astype(np.uint8)
    N, K = codes.shape
    out = np.zeros(N * K // 2, np.uint8)
    for t0 in range(0, N, 128):
        R = min(128, N - t0)
        tile = codes[t0:t0 + R]
        for b in range(0, K, 128):
            for c in range(0, min(128, K - b), 32):
                ch = tile[:, b + c:b + c + 32].reshape(R, 4, 8)
                byts = ch[:, :, 0:4] | (ch[:, :, 4:8] << 4)
                off = t0 * K // 2 + (b // 128) * R * 64 + (c // 32) * R * 16
                out[off:off + R * 16] = byts.reshape(R * 16)
    return out.reshape(N, K // 2)

"""Reader of the library's physical 2:4 layout (oracle; test infrastructure).

The page "Add CUTLASS-based row-wise scaled sparse FP8 kernel" (pytorch/ao
pull request 1671) stores the compressed weight in the SM90 CUTLASS format.
This library defines its own layout for the sm_100 sparse tensor-core
instruction (layout version 1).  This module is written from that layout's
specification, independently of the CUDA code that writes it:

    N_pad = ceil(N / 128) * 128, K % 128 == 0.

    values: N_pad x K/2 bytes, row-major.  Row n holds, group by group in
            ascending g, the two kept codes of group g (lower index first).

    meta:   N_pad x K/8 bytes, in 2048-byte tiles.  Tile (nt, kt), for
            nt < N_pad/128 and kt < K/128, starts at byte
            (nt * (K/128) + kt) * 2048.  Inside it, row r (< 128) starts at
            byte 16*r; byte b (< 16) of that row holds the index nibble of
            group 32*kt + 2*b in bits 0..3 and of group 32*kt + 2*b + 1 in
            bits 4..7, both for weight row n = 128*nt + r.

    Rows n >= N (padding) hold value 0x00 and nibble 0x4 (indices 0 and 1)
    in every group.
"""

import numpy as np

LAYOUT_VERSION = 1
TILE_ROWS = 128
TILE_K = 128


def padded_rows(n):
    return ((n + TILE_ROWS - 1) // TILE_ROWS) * TILE_ROWS


def values_bytes(n, k):
    return padded_rows(n) * k // 2


def meta_bytes(n, k):
    return padded_rows(n) * k // 8


def unpack_physical(values, meta, n, k, include_padding=False):
    """Physical buffers -> logical (vals [rows, K/2], nibbles [rows, K/4]).

    ``values`` and ``meta`` are flat uint8 arrays of the sizes above.  With
    ``include_padding`` the padded rows are returned too (rows = N_pad),
    otherwise only the first N.
    """
    if k % TILE_K:
        raise ValueError("K must be a multiple of 128")
    npad = padded_rows(n)
    values = np.asarray(values, dtype=np.uint8).reshape(-1)
    meta = np.asarray(meta, dtype=np.uint8).reshape(-1)
    if values.size != values_bytes(n, k) or meta.size != meta_bytes(n, k):
        raise ValueError("buffer size does not match (n, k)")
    vals = values.reshape(npad, k // 2).copy()
    kt_count = k // TILE_K
    # tiles[nt, kt, r, b]
    tiles = meta.reshape(npad // TILE_ROWS, kt_count, TILE_ROWS, 16)
    nib = np.zeros((npad, k // 4), dtype=np.uint8)
    for nt in range(npad // TILE_ROWS):
        for kt in range(kt_count):
            t = tiles[nt, kt]                               # [128 rows, 16 bytes]
            rows = slice(nt * TILE_ROWS, (nt + 1) * TILE_ROWS)
            g0 = 32 * kt
            nib[rows, g0 + 0:g0 + 32:2] = t & 0x0F
            nib[rows, g0 + 1:g0 + 32:2] = t >> 4
    if include_padding:
        return vals, nib
    return vals[:n], nib[:n]

"""Reader of the library's physical 2:4 layout (oracle; test infrastructure).

The page "Add CUTLASS-based row-wise scaled sparse FP8 kernel" (pytorch/ao
pull request 1671) stores the compressed weight in the SM90 CUTLASS format.
This library defines its own layout for the sm_100 sparse tensor-core
instruction (layout version 3).  This module is written from that layout's
specification, independently of the CUDA code that writes it:

    N_pad = ceil(N / 128) * 128, K % 128 == 0.  "Tile (nt, kt)" is weight
    rows 128*nt .. 128*nt+127 and K columns 128*kt .. 128*kt+127 (groups
    32*kt .. 32*kt+31); tiles are numbered t = nt * (K/128) + kt and stored
    one after another, 10240 bytes each, in a single buffer of
    N_pad * K * 5/8 bytes.  Tile t starts at byte 10240*t:

    bytes 0 .. 8191 (kept values): row r (< 128) of the tile starts at byte
            64*r and holds the 64 kept codes of its 32 groups (two per group,
            lower index first), as four 16-byte chunks: chunk c (groups
            8c .. 8c+7) is stored at chunk position c XOR ((r >> 1) & 3).

    bytes 8192 .. 10239 (index metadata): row r of the tile starts at byte
            8192 + 16*r; byte b (< 16) of that row holds the index nibble of
            group 32*kt + 2*b in bits 0..3 and of group 32*kt + 2*b + 1 in
            bits 4..7.

    Rows n >= N (padding) hold value 0x00 and nibble 0x4 (indices 0 and 1)
    in every group.
"""

import numpy as np

LAYOUT_VERSION = 3
TILE_BYTES = 10240
TILE_ROWS = 128
TILE_K = 128


def padded_rows(n):
    return ((n + TILE_ROWS - 1) // TILE_ROWS) * TILE_ROWS


def packed_bytes(n, k):
    return padded_rows(n) * k * 5 // 8


def unpack_physical(packed, n, k, include_padding=False):
    """Packed buffer -> logical (vals [rows, K/2], nibbles [rows, K/4]).

    ``packed`` is a flat uint8 array of packed_bytes(n, k) bytes.  With
    ``include_padding`` the padded rows are returned too (rows = N_pad),
    otherwise only the first N.
    """
    if k % TILE_K:
        raise ValueError("K must be a multiple of 128")
    npad = padded_rows(n)
    packed = np.asarray(packed, dtype=np.uint8).reshape(-1)
    if packed.size != packed_bytes(n, k):
        raise ValueError("buffer size does not match (n, k)")
    kt_count = k // TILE_K
    nt_count = npad // TILE_ROWS
    tiles = packed.reshape(nt_count, kt_count, TILE_BYTES)
    # Byte j (< 64) of row r of the values part sits at 16 * (c ^ ((r >> 1) & 3)) + b,
    # with c, b = divmod(j, 16).
    r_idx = np.arange(TILE_ROWS)[:, None]
    j_idx = np.arange(64)[None, :]
    src = 16 * ((j_idx // 16) ^ ((r_idx >> 1) & 3)) + (j_idx % 16)     # [128, 64]
    vt = tiles[:, :, :8192].reshape(nt_count, kt_count, TILE_ROWS, 64)
    vt = np.take_along_axis(vt, np.broadcast_to(src, vt.shape), axis=3)
    vals = vt.transpose(0, 2, 1, 3).reshape(npad, k // 2)
    # Metadata: byte b of row r of tile (nt, kt) -> groups 32*kt + 2b (low
    # nibble) and 32*kt + 2b + 1 (high nibble) of row 128*nt + r.
    mt = tiles[:, :, 8192:].reshape(nt_count, kt_count, TILE_ROWS, 16).transpose(0, 2, 1, 3)
    mt = mt.reshape(npad, kt_count * 16)                   # [row, 16*kt + b]
    nib = np.zeros((npad, k // 4), dtype=np.uint8)
    nib[:, 0::2] = mt & 0x0F
    nib[:, 1::2] = mt >> 4
    if include_padding:
        return vals, nib
    return vals[:n], nib[:n]

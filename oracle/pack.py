"""Sign packing and the residual-block record (oracle).

Test infrastructure: see the package docstring.

Follows: Review, Fig. 3 caption (the +-1 sign matrix of a residual block is packed
into GPU-supported data types to save memory; a block is the packed signs plus the
singular vectors); Rebuttal A1.A (a residual block consists of a packed sign matrix
and singular vectors); Review, Fig. 5 caption (a block of an m x n weight holds the
same bytes as 2 k' (m + n) fp16 values with k' = k + m n / (16 (m + n)), i.e.
m n / 8 bytes of signs plus 2 k (m + n) fp16 values).

The pages fix neither the bit order nor the word size.  Readings taken (the same
specification is written out in include/bitstack.h and implemented independently by
the library):

* bit value 1 <=> sign -1;
* canonical order: row-major, 8 columns per byte, column c in bit c % 8 of byte c / 8;
* device tile order: the m x d sign matrix is cut into tiles of 128 rows x 256
  columns, stored row-tile-major (tile index rt * (d / 256) + g).  A tile is 1024
  little-endian 32-bit words.  Row rr of the tile owns 8 words p = 0..7 (its 256
  columns); word p of row rr sits at index (p // 4) * 512 + rr * 4 + (p % 4).  Bit
  8 q + t of word p (q = 0..3, t = 0..7) holds column 32 t + 4 p + q of the tile;
* record: [sign words, device order][U, m x k fp16 row-major][V, d x k fp16
  row-major]; m d / 8 + 2 k (m + d) bytes.
"""
from __future__ import annotations

import numpy as np

TILE_ROWS = 128
TILE_COLS = 256
TILE_WORDS = TILE_ROWS * TILE_COLS // 32


def block_bytes(m: int, d: int, k: int) -> int:
    """Bytes of one residual block record: m d / 8 + 2 k (m + d).

    Pinned (tests): equals the block size implied by the Review, Fig. 5 caption
    (2 k' (m + n) bytes-of-fp16 with k' = k + m n / (16 (m + n))), and reproduces
    the 7.56 MB maximum block size of an 8B model given in Rebuttal A1.A.
    """
    return m * d // 8 + 2 * k * (m + d)


def pack_canonical(neg: np.ndarray) -> np.ndarray:
    """Canonical packing: uint8 m x d/8, column c in bit c % 8 of byte c / 8."""
    neg = np.asarray(neg, dtype=bool)
    return np.packbits(neg, axis=1, bitorder="little")


def unpack_canonical(packed: np.ndarray, d: int) -> np.ndarray:
    """Inverse of pack_canonical: bool m x d."""
    return np.unpackbits(np.asarray(packed, dtype=np.uint8), axis=1, count=d,
                         bitorder="little").astype(bool)


def _check_tiles(m: int, d: int) -> None:
    if m % TILE_ROWS or d % TILE_COLS:
        raise ValueError(f"device order needs m % {TILE_ROWS} == 0 and d % {TILE_COLS} == 0, got {m}x{d}")


def pack_device(neg: np.ndarray) -> np.ndarray:
    """Device tile order: uint32 array of m d / 32 words (see module docstring)."""
    neg = np.asarray(neg, dtype=bool)
    m, d = neg.shape
    _check_tiles(m, d)
    RT, G = m // TILE_ROWS, d // TILE_COLS
    weights = (np.uint64(1) << np.arange(32, dtype=np.uint64))
    out = np.empty((RT, G * TILE_WORDS), dtype=np.uint32)
    for rt in range(RT):
        # neg[rt*128 + rr, g*256 + 32 t + 4 (4 h + pp) + q] -> axes (rr, g, t, h, pp, q)
        a = neg[rt * TILE_ROWS:(rt + 1) * TILE_ROWS].reshape(TILE_ROWS, G, 8, 2, 4, 4)
        # word (g, h, rr, pp) holds the bits indexed 8 q + t
        a = a.transpose(1, 3, 0, 4, 5, 2).reshape(G, 2, TILE_ROWS, 4, 32)
        out[rt] = (a.astype(np.uint64) * weights).sum(axis=-1).astype(np.uint32).reshape(-1)
    return out.reshape(-1)


def unpack_device(words: np.ndarray, m: int, d: int) -> np.ndarray:
    """Inverse of pack_device: bool m x d."""
    _check_tiles(m, d)
    RT, G = m // TILE_ROWS, d // TILE_COLS
    w_all = np.asarray(words, dtype=np.uint32).reshape(RT, G, 2, TILE_ROWS, 4)
    out = np.empty((m, d), dtype=bool)
    shifts = np.arange(32, dtype=np.uint32)
    for rt in range(RT):
        w = w_all[rt][..., None]                                  # (g, h, rr, pp, 1)
        bits = ((w >> shifts) & 1).astype(bool)                   # (g, h, rr, pp, 32): index 8q+t
        bits = bits.reshape(G, 2, TILE_ROWS, 4, 4, 8)             # (g, h, rr, pp, q, t)
        a = bits.transpose(2, 0, 5, 1, 3, 4)                      # (rr, g, t, h, pp, q)
        out[rt * TILE_ROWS:(rt + 1) * TILE_ROWS] = a.reshape(TILE_ROWS, d)
    return out


def device_position(r: int, c: int, d: int):
    """(word index, bit index) of sign (r, c) in the device order, by direct arithmetic.

    A scalar restatement of the layout used by the brute-force test of pack_device.
    """
    rt, rr = divmod(r, TILE_ROWS)
    g, cl = divmod(c, TILE_COLS)
    t, rem = divmod(cl, 32)
    p, q = divmod(rem, 4)
    h, pp = divmod(p, 4)
    tile = rt * (d // TILE_COLS) + g
    return tile * TILE_WORDS + h * 512 + rr * 4 + pp, 8 * q + t


def make_record(neg: np.ndarray, U: np.ndarray, V: np.ndarray) -> np.ndarray:
    """The block record bytes (uint8): device-order sign words, then U, then V."""
    neg = np.asarray(neg, dtype=bool)
    m, d = neg.shape
    U = np.ascontiguousarray(U, dtype=np.float16)
    V = np.ascontiguousarray(V, dtype=np.float16)
    k = U.shape[1]
    if U.shape != (m, k) or V.shape != (d, k):
        raise ValueError("factor shapes do not match the sign matrix")
    words = pack_device(neg).astype("<u4")
    rec = np.concatenate([words.view(np.uint8), U.view(np.uint8).reshape(-1),
                          V.view(np.uint8).reshape(-1)])
    assert rec.size == block_bytes(m, d, k)
    return rec


def parse_record(rec: np.ndarray, m: int, d: int, k: int):
    """Split a record into (neg bool m x d, U fp16 m x k, V fp16 d x k)."""
    rec = np.asarray(rec, dtype=np.uint8)
    nsb = m * d // 8
    words = rec[:nsb].view("<u4")
    U = rec[nsb:nsb + 2 * m * k].view(np.float16).reshape(m, k)
    V = rec[nsb + 2 * m * k:nsb + 2 * k * (m + d)].view(np.float16).reshape(d, k)
    return unpack_device(words, m, d), U, V


def plain_block_bytes(m: int, d: int, kp: int) -> int:
    """Bytes of one vanilla-SVD ("w/o AVD") block record: 2 k' (m + d) (fp16 U, V)."""
    return 2 * kp * (m + d)


def make_plain_record(U: np.ndarray, V: np.ndarray) -> np.ndarray:
    """The "w/o AVD" record bytes (uint8): U (m x k' fp16 row-major), then V (d x k')."""
    U = np.ascontiguousarray(U, dtype=np.float16)
    V = np.ascontiguousarray(V, dtype=np.float16)
    if U.shape[1] != V.shape[1]:
        raise ValueError("U and V ranks differ")
    return np.concatenate([U.view(np.uint8).reshape(-1), V.view(np.uint8).reshape(-1)])

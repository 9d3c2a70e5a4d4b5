"""Packer / unpacker of libtq's packed code layout, written from the layout statement in
include/tq.h (test-side only; shares nothing with the library).

Record of one vector: P planes over d_pad = 32*ceil(d/32) positions, 4 quarters of
P*d_pad/32 bytes; quarter q holds positions [q*d_pad/4, (q+1)*d_pad/4); plane p sits at
offset p*d_pad/32 inside the quarter; bit b of that chunk (LSB first) is position
q*d_pad/4 + b.  Planes 0..k-1 hold the index bits, plane k (prod mode) the QJL signs.
"""
import numpy as np


def geometry(d: int, k: int, prod: bool):
    d_pad = 32 * ((d + 31) // 32)
    planes = k + (1 if prod else 0)
    return d_pad, planes, planes * d_pad // 8


def _bit_positions(d: int, planes: int):
    """byte offset and bit for every (plane, position) -> arrays [planes, d_pad]."""
    d_pad = 32 * ((d + 31) // 32)
    quarter, chunk = d_pad // 4, d_pad // 32
    i = np.arange(d_pad)
    q, b = i // quarter, i % quarter
    byte = np.empty((planes, d_pad), dtype=np.int64)
    for p in range(planes):
        byte[p] = q * planes * chunk + p * chunk + b // 8
    return byte, np.broadcast_to(b % 8, (planes, d_pad))


def pack(idx: np.ndarray, signs, d: int, k: int) -> np.ndarray:
    prod = signs is not None
    d_pad, planes, nbytes = geometry(d, k, prod)
    n = idx.shape[0]
    out = np.zeros((n, nbytes), dtype=np.uint8)
    byte, bit = _bit_positions(d, planes)
    for p in range(planes):
        vals = ((idx >> p) & 1) if p < k else signs
        vals = np.asarray(vals, dtype=np.uint8)
        for i in range(d):
            np.bitwise_or.at(out, (slice(None), byte[p, i]), (vals[:, i] << bit[p, i]).astype(np.uint8))
    return out


def unpack(codes: np.ndarray, d: int, k: int, prod: bool):
    """-> idx [n, d] int64, signs [n, d] uint8 (or None), and the padding bits (must be 0)."""
    d_pad, planes, nbytes = geometry(d, k, prod)
    codes = np.asarray(codes, dtype=np.uint8).reshape(-1, nbytes)
    byte, bit = _bit_positions(d, planes)
    bits = (codes[:, byte] >> bit) & 1            # [n, planes, d_pad]
    idx = np.zeros((codes.shape[0], d), dtype=np.int64)
    for p in range(k):
        idx |= bits[:, p, :d].astype(np.int64) << p
    signs = bits[:, k, :d].astype(np.uint8) if prod else None
    return idx, signs, bits[:, :, d:]

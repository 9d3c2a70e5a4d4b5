"""Packer / unpacker of libtq's packed code layout, written from the layout statement in
include/tq.h (test-side only; shares nothing with the library).

Every coordinate carries a P-bit code (P = k index bits, plus the QJL sign in prod mode).
The index enters the code in sign-magnitude form: with K = 2^k levels, bit k-1 is the
"negative half" flag n = [idx < K/2] and the low k-1 bits are the magnitude rank
m = n ? K/2-1-idx : idx-K/2.  In prod mode the QJL sign bit [S r >= 0] sits above the
index, as code bit k.  The top code bit (bit P-1) is the "top" bit of the layout.

A record is d_pad/32 groups (d_pad = 32*ceil(d/32)), each P little-endian 32-bit words.
Inside a group, coordinate e = 8s + j (slice s, j = 4h + i) stores code bit b in
  P = 1: top bit            -> word 0, bit E = 8i + 7 - (2s + h)
  P = 2: bit 0              -> word 0, bit 4j + s;         top -> word 1, bit E
  P = 3: bits 0, 1          -> word s&1, bit 4j + 2(s>>1) + b;  top -> word 2, bit E
  P = 4: bits 0..2          -> word s, bit 4j + b;         top -> word s, bit 8i+7 (h=0) or 8i+3 (h=1)
  P = 5: bits 0..3 as P = 4 (bit 3 in the P = 4 top slot);  top (bit 4) -> word 4, bit E
"""
import numpy as np


def geometry(d: int, k: int, prod: bool):
    d_pad = 32 * ((d + 31) // 32)
    planes = k + (1 if prod else 0)
    return d_pad, planes, planes * d_pad // 8


def _pos(P: int, e: int, b: int):
    """(word, bit) of code bit b of group coordinate e."""
    s, j = divmod(e, 8)
    h, i = divmod(j, 4)
    E = 8 * i + 7 - (2 * s + h)
    top = b == P - 1
    if P == 1:
        return 0, E
    if P == 2:
        return (1, E) if top else (0, 4 * j + s)
    if P == 3:
        return (2, E) if top else (s & 1, 4 * j + 2 * (s >> 1) + b)
    if P == 5 and top:
        return 4, E
    if b == 3:
        return s, (8 * i + 7) if h == 0 else (8 * i + 3)
    return s, 4 * j + b


def _bit_positions(d: int, P: int):
    """byte offset and bit of every (code bit, coordinate) -> arrays [P, d_pad]."""
    d_pad = 32 * ((d + 31) // 32)
    byte = np.empty((P, d_pad), dtype=np.int64)
    bit = np.empty((P, d_pad), dtype=np.int64)
    for x in range(d_pad):
        g, e = divmod(x, 32)
        for b in range(P):
            w, pos = _pos(P, e, b)
            byte[b, x] = g * 4 * P + 4 * w + pos // 8
            bit[b, x] = pos % 8
    return byte, bit


def _to_sign_magnitude(idx, k):
    K = 1 << k
    if k == 1:
        return (idx == 0).astype(np.int64)
    neg = idx < K // 2
    mag = np.where(neg, K // 2 - 1 - idx, idx - K // 2)
    return (neg.astype(np.int64) << (k - 1)) | mag


def _from_sign_magnitude(code, k):
    K = 1 << k
    if k == 1:
        return np.where(code & 1, 0, 1).astype(np.int64)
    neg = (code >> (k - 1)) & 1
    mag = code & ((1 << (k - 1)) - 1)
    return np.where(neg == 1, K // 2 - 1 - mag, K // 2 + mag).astype(np.int64)


def pack(idx: np.ndarray, signs, d: int, k: int) -> np.ndarray:
    prod = signs is not None
    d_pad, P, nbytes = geometry(d, k, prod)
    idx = np.asarray(idx, dtype=np.int64)
    n = idx.shape[0]
    code = _to_sign_magnitude(idx, k)
    if prod:
        code = code | (np.asarray(signs, dtype=np.int64) << k)
    out = np.zeros((n, nbytes), dtype=np.uint8)
    byte, bit = _bit_positions(d, P)
    for b in range(P):
        vals = ((code >> b) & 1).astype(np.uint8)
        for x in range(d):
            out[:, byte[b, x]] |= (vals[:, x] << bit[b, x]).astype(np.uint8)
    return out


def unpack(codes: np.ndarray, d: int, k: int, prod: bool):
    """-> idx [n, d] int64, signs [n, d] uint8 (or None), and the padding bits (must be 0)."""
    d_pad, P, nbytes = geometry(d, k, prod)
    codes = np.asarray(codes, dtype=np.uint8).reshape(-1, nbytes)
    byte, bit = _bit_positions(d, P)
    bits = (codes[:, byte] >> bit) & 1            # [n, P, d_pad]
    code = np.zeros((codes.shape[0], d), dtype=np.int64)
    for b in range(P):
        code |= bits[:, b, :d].astype(np.int64) << b
    idx = _from_sign_magnitude(code & ((1 << k) - 1), k)
    signs = ((code >> k) & 1).astype(np.uint8) if prod else None
    return idx, signs, bits[:, :, d:]

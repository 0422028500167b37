"""Counter-based random numbers for attention dropout, and the keep mask.

TEST INFRASTRUCTURE ONLY (see ``oracle/attention.py``): the library draws
the same numbers with its own device code; the two share nothing but the
published definition below.

Philox4x32-10 is restated from its published definition (J. K. Salmon,
M. A. Moraes, R. O. Dror, D. E. Shaw, "Parallel Random Numbers: As Easy as
1, 2, 3", SC'11): a 128-bit counter (four 32-bit
words c0..c3) and a 64-bit key (k0, k1) go through ten rounds.  One round
multiplies c0 by 0xD2511F53 and c2 by 0xCD9E8D57 into 64-bit products and
returns (hi(c2·M1) ^ c1 ^ k0, lo(c2·M1), hi(c0·M0) ^ c3 ^ k1, lo(c0·M0));
between rounds the key is bumped by the Weyl constants (0x9E3779B9,
0xBB67AE85) modulo 2^32.

The dropout mask (the 51CTO notes, section "算法的改进", mention dropout
steps in the V1 algorithm but fix no generator, so this layout is a reading):

* the [Nq, Nk] score matrix of head index bh = b·H + h is cut into 4×4
  blocks; block (i // 4, j // 4) takes counter (j // 4, i // 4, bh, offset)
  and key (seed mod 2^32, seed div 2^32);
* output word i % 4 belongs to query row i, and byte j % 4 of that word
  (least significant first) to key column j;
* the weight P_ij is kept iff that byte is below the threshold T =
  round((1 − p) · 256) for the dropout probability p (taken as float32), so
  a weight is kept with probability T / 256 and kept weights are scaled by
  256 / T.
"""
from __future__ import annotations

import numpy as np

M0 = 0xD2511F53
M1 = 0xCD9E8D57
W0 = 0x9E3779B9
W1 = 0xBB67AE85
_MASK32 = 0xFFFFFFFF


def philox4x32_10(ctr, key) -> np.ndarray:
    """Philox4x32-10 of counters ``ctr`` [..., 4] under keys ``key`` [..., 2]
    (both broadcast, any integer type holding 32-bit values); uint32 [..., 4]."""
    ctr = np.asarray(ctr, dtype=np.uint64) & _MASK32
    key = np.asarray(key, dtype=np.uint64) & _MASK32
    shape = np.broadcast_shapes(ctr.shape[:-1], key.shape[:-1])
    c0, c1, c2, c3 = (np.broadcast_to(ctr[..., n], shape).copy() for n in range(4))
    k0 = np.broadcast_to(key[..., 0], shape).copy()
    k1 = np.broadcast_to(key[..., 1], shape).copy()
    for rnd in range(10):
        if rnd > 0:
            k0 = (k0 + W0) & _MASK32
            k1 = (k1 + W1) & _MASK32
        p0 = c0 * np.uint64(M0)  # < 2^64: exact in uint64
        p1 = c2 * np.uint64(M1)
        hi0, lo0 = p0 >> np.uint64(32), p0 & _MASK32
        hi1, lo1 = p1 >> np.uint64(32), p1 & _MASK32
        c0, c1, c2, c3 = hi1 ^ c1 ^ k0, lo1, hi0 ^ c3 ^ k1, lo0
    return np.stack([c0, c1, c2, c3], axis=-1).astype(np.uint32)


def dropout_threshold(p: float) -> int:
    """T = round((1 − p) · 256) with p rounded to float32 first (the C ABI
    passes p as a float); valid dropout needs 0 <= p < 1 and T >= 1."""
    p32 = float(np.float32(p))
    if not (0.0 <= p32 < 1.0):
        raise ValueError("dropout probability must be in [0, 1)")
    t = int(np.rint((1.0 - p32) * 256.0))
    if t < 1:
        raise ValueError("dropout probability too close to 1 (keeps nothing)")
    return t


def keep_mask(bh: int, rows, cols, p: float, seed: int, offset: int) -> np.ndarray:
    """Boolean [len(rows), len(cols)] keep mask of head index ``bh`` at the
    given query rows and key columns (absolute indices)."""
    t = dropout_threshold(p)
    rows = np.asarray(rows, dtype=np.int64)
    cols = np.asarray(cols, dtype=np.int64)
    rb, cb = rows // 4, cols // 4
    urb, rinv = np.unique(rb, return_inverse=True)
    ucb, cinv = np.unique(cb, return_inverse=True)
    ctr = np.empty((len(urb), len(ucb), 4), dtype=np.uint64)
    ctr[..., 0] = ucb[None, :]
    ctr[..., 1] = urb[:, None]
    ctr[..., 2] = bh
    ctr[..., 3] = offset & _MASK32
    key = np.array([seed & _MASK32, (seed >> 32) & _MASK32], dtype=np.uint64)
    words = philox4x32_10(ctr, key)  # [rows blocks, col blocks, 4]
    w = words[rinv[:, None], cinv[None, :], (rows % 4)[:, None]].astype(np.uint64)
    byte = (w >> (8 * (cols % 4))[None, :].astype(np.uint64)) & np.uint64(0xFF)
    return byte < np.uint64(t)


def keep_scale(p: float) -> float:
    """256 / T: the factor that keeps E[dropped weights] equal to the weights."""
    return 256.0 / dropout_threshold(p)

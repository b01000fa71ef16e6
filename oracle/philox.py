"""Philox4x32-10 counter-based generator and the dropout keep-mask it defines.

TEST INFRASTRUCTURE ONLY. This module belongs to the float64 oracle: only the
test suite, the smoke check and the benchmark's CPU-baseline leg may import it.
The CUDA path implements the same published generator independently.

The generator is Philox4x32 with 10 rounds as defined by Salmon, Moraes, Dror
and Shaw, "Parallel Random Numbers: As Easy as 1, 2, 3" (SC'11), section 4.
Each round multiplies two counter words by fixed odd constants, exchanges the
words and folds the high product halves into the other two words together with
the key; the key is advanced by the Weyl increments between rounds.

Why a counter-based generator: "A different dropout mask changes the reverse
result" (alphabetamath.cc, example and its verification steps 1.1-2.1) shows
that the reverse pass must use the very realisation xi of the forward pass.
A generator addressed by (seed, b, h, i, j) lets both passes evaluate the same
xi_ij without storing a mask.

Counter convention used by this library (the pages leave it open):
    counter = (j >> 2, i, h, b)   with h the query head
    key     = (seed mod 2**32, seed >> 32)
    xi_ij   = 1  iff  word[j & 3] >= floor(rho * 2**32)
so the keep decision is an integer comparison and is bit-exact everywhere.
"""
from __future__ import annotations

import numpy as np

# Multipliers and key increments of Philox4x32 (Salmon et al., SC'11).
_MUL0 = np.uint64(0xD2511F53)
_MUL1 = np.uint64(0xCD9E8D57)
_WEYL0 = np.uint64(0x9E3779B9)
_WEYL1 = np.uint64(0xBB67AE85)
_LO32 = np.uint64(0xFFFFFFFF)
_SH32 = np.uint64(32)


def philox4x32(counter: np.ndarray, key: np.ndarray, rounds: int = 10) -> np.ndarray:
    """Evaluate Philox4x32-R elementwise.

    counter: uint32-valued array [..., 4]; key: uint32-valued array [..., 2]
    (broadcastable). Returns uint32 [..., 4].
    """
    c = np.asarray(counter, dtype=np.uint64)
    k = np.asarray(key, dtype=np.uint64)
    c0, c1, c2, c3 = c[..., 0], c[..., 1], c[..., 2], c[..., 3]
    k0, k1 = k[..., 0], k[..., 1]
    for r in range(rounds):
        if r:
            k0 = (k0 + _WEYL0) & _LO32
            k1 = (k1 + _WEYL1) & _LO32
        p0 = _MUL0 * c0  # < 2**64, exact in uint64
        p1 = _MUL1 * c2
        c0, c1, c2, c3 = (
            ((p1 >> _SH32) ^ c1 ^ k0) & _LO32,
            p1 & _LO32,
            ((p0 >> _SH32) ^ c3 ^ k1) & _LO32,
            p0 & _LO32,
        )
    return np.stack([c0, c1, c2, c3], axis=-1).astype(np.uint32)


def keep_threshold(rho: float) -> int:
    """Integer threshold: a 32-bit word w keeps its pair iff w >= threshold."""
    if not (0.0 <= rho < 1.0):
        raise ValueError("dropout rate must lie in [0, 1)")
    return min(int(np.floor(rho * 4294967296.0)), 0xFFFFFFFF)


def dropout_keep(seed: int, rho: float, batch: int, heads: int,
                 t_q: int, t_k: int) -> np.ndarray:
    """xi as a bool array [batch, heads, t_q, t_k] (True = kept)."""
    thr = np.uint32(keep_threshold(rho))
    key = np.array([seed & 0xFFFFFFFF, (seed >> 32) & 0xFFFFFFFF], dtype=np.uint64)
    n_groups = (t_k + 3) // 4
    out = np.empty((batch, heads, t_q, n_groups * 4), dtype=bool)
    jg = np.arange(n_groups, dtype=np.uint64)
    ii = np.arange(t_q, dtype=np.uint64)
    for b in range(batch):
        for h in range(heads):
            ctr = np.empty((t_q, n_groups, 4), dtype=np.uint64)
            ctr[..., 0] = jg[None, :]
            ctr[..., 1] = ii[:, None]
            ctr[..., 2] = h
            ctr[..., 3] = b
            words = philox4x32(ctr, key)  # [t_q, n_groups, 4]
            out[b, h] = (words >= thr).reshape(t_q, n_groups * 4)
    return out[..., :t_k]

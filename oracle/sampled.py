"""The oracle's definitions evaluated on chosen query rows or key columns.

TEST INFRASTRUCTURE ONLY (see the package docstring). For problems too large
to evaluate whole in float64, these functions compute exactly the quantities
of attention.forward / attention.backward, but only for the query rows or
key columns asked for. Each output row i depends only on row i's scores, and
each dK_j / dV_j is a plain sum over the query rows that allow key j, so
restricting the set of rows or columns changes nothing in the arithmetic of
an output element.
"""
from __future__ import annotations

import numpy as np

from .philox import keep_threshold, philox4x32

NEG_INF = -np.inf


def allowed_at(rows: np.ndarray, cols: np.ndarray, *, causal: bool = False, window_left: int = 0,
               block_mask: np.ndarray | None = None, block_q: int = 1, block_k: int = 1) -> np.ndarray:
    """A_i restricted to `cols`, for each i in `rows`: bool [len(rows), len(cols)]
    (block_mask here is one [nb_q, nb_k] grid)."""
    i = np.asarray(rows, np.int64)[:, None]
    j = np.asarray(cols, np.int64)[None, :]
    allow = np.ones((i.shape[0], j.shape[1]), dtype=bool)
    if causal:
        allow &= j <= i
    if window_left > 0:
        allow &= j > i - window_left
    if block_mask is not None:
        allow &= np.asarray(block_mask)[i // block_q, j // block_k] != 0
    return allow


def keep_at(seed: int, rho: float, b: int, h: int, rows, cols) -> np.ndarray:
    """xi for the pairs rows x cols of (b, h): counter (j >> 2, i, h, b),
    word j & 3, kept iff word >= floor(rho 2^32) (the philox module's
    convention)."""
    rows = np.asarray(rows, np.uint64)
    cols = np.asarray(cols, np.uint64)
    thr = np.uint32(keep_threshold(rho))
    key = np.array([seed & 0xFFFFFFFF, (seed >> 32) & 0xFFFFFFFF], dtype=np.uint64)
    ctr = np.empty((rows.size, cols.size, 4), dtype=np.uint64)
    ctr[..., 0] = (cols >> np.uint64(2))[None, :]
    ctr[..., 1] = rows[:, None]
    ctr[..., 2] = h
    ctr[..., 3] = b
    words = philox4x32(ctr, key)
    sel = (cols & np.uint64(3)).astype(np.int64)
    w = np.take_along_axis(words, np.broadcast_to(sel[None, :, None], (rows.size, cols.size, 1)), axis=2)[..., 0]
    return w >= thr


def keep_range(seed: int, rho: float, b: int, h: int, rows, c0: int, c1: int) -> np.ndarray:
    """xi for rows x the contiguous key range [c0, c1) of (b, h), c0 a
    multiple of 4: the same values as keep_at, but each generator call's four
    words serve the four keys j = 4 (j >> 2) + 0..3 that share its counter,
    so every call is made once instead of once per key."""
    if c0 % 4:
        raise ValueError("c0 must be a multiple of 4")
    rows = np.asarray(rows, np.uint64)
    nblk = (c1 - c0 + 3) // 4
    thr = np.uint32(keep_threshold(rho))
    key = np.array([seed & 0xFFFFFFFF, (seed >> 32) & 0xFFFFFFFF], dtype=np.uint64)
    ctr = np.empty((rows.size, nblk, 4), dtype=np.uint64)
    ctr[..., 0] = np.arange(c0 // 4, c0 // 4 + nblk, dtype=np.uint64)[None, :]
    ctr[..., 1] = rows[:, None]
    ctr[..., 2] = h
    ctr[..., 3] = b
    words = philox4x32(ctr, key)  # [rows, nblk, 4]: word w is key 4 * block + w
    return (words >= thr).reshape(rows.size, nblk * 4)[:, :c1 - c0]


def row_softmax(s: np.ndarray, allow: np.ndarray, z: float):
    """p, p_sink, LSE of each row (sink-inclusive LSE; empty rows: p = 0,
    LSE = -inf or z)."""
    sm = np.where(allow, s, NEG_INF)
    m = np.maximum(sm.max(axis=-1), z)
    finite = np.isfinite(m)
    shift = np.where(finite, m, 0.0)
    e = np.where(allow, np.exp(sm - shift[:, None]), 0.0)
    e_sink = np.exp(z - shift) if np.isfinite(z) else np.zeros_like(shift)
    total = e.sum(axis=-1) + e_sink
    safe = np.where(finite, total, 1.0)
    p = np.where(finite[:, None], e / safe[:, None], 0.0)
    return p, np.where(finite, e_sink / safe, 0.0), np.where(finite, shift + np.log(safe), NEG_INF)


def rows_forward_backward(q_h, k_kv, v_kv, g_h, rows, allow_rows, scale, z=NEG_INF, keep_rows=None,
                          rho=0.0):
    """Y_i, LSE_i, delta_i and dQ_i for the query rows `rows` of one (b, h).

    q_h, g_h: [T, d] and [T, dv] of that query head; k_kv, v_kv: [Tk, d], [Tk, dv];
    allow_rows: bool [len(rows), Tk]; keep_rows: bool [len(rows), Tk] or None.
    """
    q = np.asarray(q_h, np.float64)[rows]
    g = np.asarray(g_h, np.float64)[rows]
    k = np.asarray(k_kv, np.float64)
    v = np.asarray(v_kv, np.float64)
    s = scale * (q @ k.T)
    p, _, lse = row_softmax(s, allow_rows, z)
    drop = keep_rows / (1.0 - rho) if keep_rows is not None else 1.0
    y = (p * drop) @ v
    delta = np.sum(g * y, axis=-1)
    dp = (g @ v.T) * drop
    gamma = p * (dp - delta[:, None])
    dq = scale * (gamma @ k)
    return y, lse, delta, dq


def cols_backward(q_group, g_group, k_kv, v_kv, cols, allow_fn, lse_group, delta_group, scale, keep_fn=None,
                  rho=0.0):
    """dK_j and dV_j for the key columns `cols` of one K/V head.

    q_group, g_group: lists over the query heads of the group of [T, d] / [T, dv];
    allow_fn(hh, rows, cols) -> bool; keep_fn(hh, rows, cols) -> bool or None;
    lse_group, delta_group: lists of [T] (LSE_i and delta_i of every row).
    Each dK_j = c sum_h sum_i gamma_ij Q_hi and dV_j = sum_h sum_i p~_ij G_hi.
    """
    k = np.asarray(k_kv, np.float64)[cols]
    v = np.asarray(v_kv, np.float64)[cols]
    dk = np.zeros_like(k)
    dv = np.zeros_like(v)
    for hh, (qh, gh) in enumerate(zip(q_group, g_group)):
        T = qh.shape[0]
        rows = np.arange(T)
        allow = allow_fn(hh, rows, cols)
        use = allow.any(axis=1)
        rows = rows[use]
        if rows.size == 0:
            continue
        allow = allow[use]
        q = np.asarray(qh, np.float64)[rows]
        g = np.asarray(gh, np.float64)[rows]
        lse = np.asarray(lse_group[hh], np.float64)[rows]
        delta = np.asarray(delta_group[hh], np.float64)[rows]
        s = scale * (q @ k.T)
        p = np.where(allow & np.isfinite(lse)[:, None], np.exp(s - np.where(np.isfinite(lse), lse, 0.0)[:, None]),
                     0.0)
        drop = keep_fn(hh, rows, cols) / (1.0 - rho) if keep_fn is not None else 1.0
        dp = (g @ v.T) * drop
        gamma = p * (dp - delta[:, None])
        dk += scale * (gamma.T @ q)
        dv += (p * drop).T @ g
    return dk, dv

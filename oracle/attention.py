"""Float64 CPU oracle for exact masked softmax attention and its analytic VJP.

TEST INFRASTRUCTURE ONLY. Only the test suite, the smoke check and the
benchmark's CPU-baseline leg may import this package. It shares no code with
the CUDA library and imports nothing from it; both sides receive the same
seeded inputs from a separate generator module.

What it computes
----------------
The dense masked attention row map that "Tiled attention and its recomputed
reverse pass are exact" (alphabetamath.cc) proves the tiled algorithm reaches:
for every query row i with allowed key set A_i,

    s_ij = c * <Q_i, K_j>                      (proof, step 5.1)
    p_ij = exp(s_ij) / (exp(z) + sum_{l in A_i} exp(s_il))
    Y_i  = sum_{j in A_i} p~_ij V_j

with the optional per-head sink logit z of "DeepSeek Sparse Attention Forward
and Backward" (icavan.github.io, section 2.2; z = -inf disables it) and the
optional inverted dropout p~_ij = p_ij * xi_ij / (1 - rho) of "A different
dropout mask changes the reverse result" (alphabetamath.cc, example).

The reverse pass follows the same proof (steps 4.1-6.1) and the DSA note
(sections 3.1-3.5):

    delta_i = sum_a G_ia Y_ia
    dp_ij   = xi_ij / (1 - rho) * <G_i, V_j>
    gamma_ij = p_ij (dp_ij - delta_i)
    dQ_i = c sum_j gamma_ij K_j,   dK_j = c sum_i gamma_ij Q_i,
    dV_j = sum_i p~_ij G_i,        dz = -sum_i p_sink,i delta_i

With rho = 0 and no sink this is exactly the proof's gamma_ij = p_ij(G_i.V_j -
delta_i). With dropout it is the plain chain rule through p~ (delta still
equals sum_j p_ij dp_ij because Y is built from p~). Shared K/V heads add the
pullbacks of every query head that reads them ("Accumulate attention without
keeping the full grid", intale.github.io, section "Reconstruct probabilities
when a gradient needs them", last paragraph; proof step 6.1 for rows).

Everything is evaluated directly from these definitions: one score matrix per
(batch, head), no blocking, no fusion. A second entry point, tiled_forward,
runs the running-summary recurrence itself, in the order and notation of
"Accumulate attention without keeping the full grid", section "Rescale earlier
mass before adding a new tile", so that the recurrence can be pinned to the
trace cards that page prints.
"""
from __future__ import annotations

from dataclasses import dataclass, field

import numpy as np

NEG_INF = -np.inf


# ---------------------------------------------------------------------------
# Allowed sets A_i
# ---------------------------------------------------------------------------

def allowed_dense(t_q: int, t_k: int, *, causal: bool = False, window_left: int = 0,
                  block_mask: np.ndarray | None = None, block_q: int = 1,
                  block_k: int = 1, query_offset: int = 0,
                  lengths: np.ndarray | None = None,
                  starts: np.ndarray | None = None) -> np.ndarray:
    """Boolean A as [.., t_q, t_k]: the intersection of the enabled sets.

    causal: j <= i + query_offset ("Accumulate attention without keeping the
    full grid", section "Rescale earlier mass ...", causal eligibility
    lower <= key <= query).
    window_left = W > 0: j > i + query_offset - W (a local window of W keys
    ending at the query, section "Change attention evaluation inside the
    existing model": the causal range intersected with a local window).
    block_mask [.., ceil(t_q/block_q), ceil(t_k/block_k)]: key j is allowed
    for query i iff block_mask[i // block_q, j // block_k] != 0.
    Leading dimensions of block_mask (batch, head) are kept in the result.

    The row-interval layouts of the same page (section "Change attention
    evaluation inside the existing model": the causal range intersected with
    active lengths and packed-segment boundaries; the per-row lower bound
    `starts` of section "Rescale earlier mass ..."):
    lengths [B] (needs t_q == t_k): batch row b has L_b active cells; query
    rows i >= L_b and keys j >= L_b are outside every set (L_b is clamped to
    [0, t_k]). starts [B, t_q]: key j is allowed for query i of batch row b
    only if j >= starts[b, i] (a packed segment's first cell). Either one
    adds a batch axis: the result is [B, 1 or H, t_q, t_k].
    """
    i = np.arange(t_q)[:, None] + query_offset
    j = np.arange(t_k)[None, :]
    allow = np.ones((t_q, t_k), dtype=bool)
    if causal:
        allow &= j <= i
    if window_left > 0:
        allow &= j > i - window_left
    if block_mask is not None:
        bm = np.asarray(block_mask) != 0
        rows = np.arange(t_q) // block_q
        cols = np.arange(t_k) // block_k
        allow = allow & bm[..., rows[:, None], cols[None, :]]
    if lengths is not None or starts is not None:
        n_b = len(lengths) if lengths is not None else np.asarray(starts).shape[0]
        extra = np.ones((n_b, 1, t_q, t_k), dtype=bool)
        if lengths is not None:
            if t_q != t_k:
                raise ValueError("lengths need t_q == t_k")
            L = np.clip(np.asarray(lengths, dtype=np.int64), 0, t_k)[:, None, None, None]
            extra &= (np.arange(t_q)[:, None] < L) & (np.arange(t_k)[None, :] < L)
        if starts is not None:
            st = np.asarray(starts, dtype=np.int64)[:, None, :, None]
            extra &= j >= st
        if allow.ndim == 2:
            allow = allow[None, None]
        elif allow.ndim == 3:
            allow = allow[:, None]
        allow = allow & extra
    return allow


# ---------------------------------------------------------------------------
# Dense masked attention and its VJP
# ---------------------------------------------------------------------------

@dataclass
class ForwardResult:
    y: np.ndarray       # [B, Hq, Tq, dv]
    lse: np.ndarray     # [B, Hq, Tq]  natural-log, sink-inclusive
    p_sink: np.ndarray  # [B, Hq, Tq]


@dataclass
class BackwardResult:
    dq: np.ndarray
    dk: np.ndarray
    dv: np.ndarray
    dsink: np.ndarray | None = None
    delta: np.ndarray | None = field(default=None, repr=False)


def _row_softmax(s: np.ndarray, allow: np.ndarray, z: float):
    """p_ij, p_sink,i and LSE_i for one (batch, head) score matrix.

    LSE_i = ln(exp(z) + sum_{j in A_i} exp(s_ij)), the sink-inclusive
    convention of the DSA note, section 7.1; evaluated with the row maximum
    M_i = max(z, max_j s_ij) as the shift. Rows with A_i empty and no sink get
    p = 0 and LSE = -inf ("Accumulate attention without keeping the full
    grid": inactive rows remain zero and undergo no division).
    """
    sm = np.where(allow, s, NEG_INF)
    m = np.maximum(sm.max(axis=-1, initial=NEG_INF), z)  # a row of no columns is empty too
    finite = np.isfinite(m)
    shift = np.where(finite, m, 0.0)
    e = np.where(allow, np.exp(sm - shift[:, None]), 0.0)
    z = np.broadcast_to(np.asarray(z, dtype=np.float64), shift.shape)   # one z per row
    has_z = np.isfinite(z)
    e_sink = np.where(has_z, np.exp(np.where(has_z, z, 0.0) - shift), 0.0)
    total = e.sum(axis=-1) + e_sink
    safe = np.where(finite, total, 1.0)
    p = np.where(finite[:, None], e / safe[:, None], 0.0)
    p_sink = np.where(finite, e_sink / safe, 0.0)
    lse = np.where(finite, shift + np.log(safe), NEG_INF)
    return p, p_sink, lse


def _bcast_allowed(allowed: np.ndarray, B: int, H: int, Tq: int, Tk: int) -> np.ndarray:
    return np.broadcast_to(np.asarray(allowed, dtype=bool), (B, H, Tq, Tk))


def forward(q, k, v, allowed, scale: float, sink=None, keep=None,
            rho: float = 0.0) -> ForwardResult:
    """Dense masked attention.

    q [B,Hq,Tq,d], k [B,Hkv,Tk,d], v [B,Hkv,Tk,dv] (float64),
    allowed bool broadcastable to [B,Hq,Tq,Tk], sink [Hq] or None,
    keep bool [B,Hq,Tq,Tk] (the dropout realisation xi) or None.
    Query head h reads K/V head h // (Hq // Hkv) (adjacent grouping:
    "Accumulate attention without keeping the full grid", section "Change
    attention evaluation inside the existing model").
    """
    q, k, v = (np.asarray(x, dtype=np.float64) for x in (q, k, v))
    B, Hq, Tq, _ = q.shape
    Hkv, Tk, dv = k.shape[1], k.shape[2], v.shape[3]
    if Hq % Hkv:
        raise ValueError("Hq must be a multiple of Hkv")
    g = Hq // Hkv
    allow = _bcast_allowed(allowed, B, Hq, Tq, Tk)
    inv_keep = 1.0 / (1.0 - rho)
    y = np.zeros((B, Hq, Tq, dv))
    lse = np.full((B, Hq, Tq), NEG_INF)
    p_sink = np.zeros((B, Hq, Tq))
    for b in range(B):
        for h in range(Hq):
            kv = h // g
            s = scale * (q[b, h] @ k[b, kv].T)
            z = NEG_INF if sink is None else float(sink[h])
            p, ps, l = _row_softmax(s, allow[b, h], z)
            if keep is not None:
                p = p * (keep[b, h] * inv_keep)
            y[b, h] = p @ v[b, kv]
            lse[b, h] = l
            p_sink[b, h] = ps
    return ForwardResult(y, lse, p_sink)


def backward(q, k, v, g_out, allowed, scale: float, sink=None, keep=None,
             rho: float = 0.0, y=None) -> BackwardResult:
    """Analytic VJP of forward() for upstream gradient g_out [B,Hq,Tq,dv].

    Probabilities are recomputed from the scores (no saved P), as in the
    proof's step 7.1; delta uses the oracle's own float64 Y unless y is given.
    """
    q, k, v, g_out = (np.asarray(x, dtype=np.float64) for x in (q, k, v, g_out))
    B, Hq, Tq, d = q.shape
    Hkv, Tk = k.shape[1], k.shape[2]
    gq = Hq // Hkv
    allow = _bcast_allowed(allowed, B, Hq, Tq, Tk)
    if y is None:
        y = forward(q, k, v, allowed, scale, sink, keep, rho).y
    inv_keep = 1.0 / (1.0 - rho)
    dq = np.zeros_like(q)
    dk = np.zeros_like(k)
    dvv = np.zeros_like(v)
    dsink = np.zeros(Hq) if sink is not None else None
    delta_all = np.zeros((B, Hq, Tq))
    for b in range(B):
        for h in range(Hq):
            kv = h // gq
            s = scale * (q[b, h] @ k[b, kv].T)
            z = NEG_INF if sink is None else float(sink[h])
            p, ps, _ = _row_softmax(s, allow[b, h], z)
            drop = keep[b, h] * inv_keep if keep is not None else 1.0
            delta = np.sum(g_out[b, h] * y[b, h], axis=-1)          # delta_i
            dp = (g_out[b, h] @ v[b, kv].T) * drop                  # dp_ij
            gamma = p * (dp - delta[:, None])                       # gamma_ij
            dq[b, h] = scale * (gamma @ k[b, kv])
            dk[b, kv] += scale * (gamma.T @ q[b, h])
            dvv[b, kv] += (p * drop).T @ g_out[b, h]
            if dsink is not None:
                dsink[h] += -np.sum(ps * delta)
            delta_all[b, h] = delta
    return BackwardResult(dq, dk, dvv, dsink, delta_all)


# ---------------------------------------------------------------------------
# Shared-KV top-k sparse attention (DSA note, sections 1-3 and 5)
# ---------------------------------------------------------------------------

def topk_allowed(idx: np.ndarray, length: np.ndarray, t_kv: int) -> np.ndarray:
    """The top-k allowed sets as a dense boolean [Tq, Tkv] (distinct lists)."""
    t_q = idx.shape[0]
    allow = np.zeros((t_q, t_kv), dtype=bool)
    for t in range(t_q):
        allow[t, idx[t, :length[t]]] = True
    return allow


def topk_forward(q, kv, idx, length, dv: int, scale: float, sink=None):
    """Shared-KV top-k attention, one token at a time.

    q [Tq,H,Dqk], kv [Tkv,Dqk] with K = kv and V = kv[:, :dv] (section 1, tied
    layout), idx int [Tq,T] of selected KV rows, length [Tq] valid entries.
    Each listed position counts once (a sum over list positions).
    Returns O [Tq,H,dv], LSE [Tq,H] (sink-inclusive, section 7.1), p_sink.
    """
    q = np.asarray(q, dtype=np.float64)
    kv = np.asarray(kv, dtype=np.float64)
    t_q, H, _ = q.shape
    o = np.zeros((t_q, H, dv))
    lse = np.full((t_q, H), NEG_INF)
    p_sink = np.zeros((t_q, H))
    z = np.full(H, NEG_INF) if sink is None else np.asarray(sink, dtype=np.float64)
    for t in range(t_q):
        # All heads of one token at once: the matrix form of the DSA note, section 5.
        sel = np.asarray(idx[t, :length[t]], dtype=np.int64)
        ksel = kv[sel]                       # [L, Dqk]
        vsel = kv[sel, :dv]                  # [L, dv]
        s = scale * (q[t] @ ksel.T)          # [H, L]
        p, ps, l = _row_softmax(s, np.ones(s.shape, bool), z)
        o[t] = p @ vsel
        lse[t] = l
        p_sink[t] = ps
    return o, lse, p_sink


def topk_backward(q, kv, idx, length, dv: int, scale: float, d_o, sink=None,
                  o=None):
    """VJP of topk_forward: dQ [Tq,H,Dqk], dKV [Tkv,Dqk], dSink [H] or None.

    Per token (DSA note, sections 3.1-3.5): dP = dO V_sel^T, D = <dO, O>,
    G = c P (dP - D), dQ = G K_sel, dK_sel = G^T Q, dV_sel = P^T dO, and the
    tied row gradient dKV_sel[:, :dv] = dK_sel[:, :dv] + dV_sel,
    dKV_sel[:, dv:] = dK_sel[:, dv:], summed into the global rows.
    """
    q = np.asarray(q, dtype=np.float64)
    kv = np.asarray(kv, dtype=np.float64)
    d_o = np.asarray(d_o, dtype=np.float64)
    if o is None:
        o = topk_forward(q, kv, idx, length, dv, scale, sink)[0]
    t_q, H, _ = q.shape
    dq = np.zeros_like(q)
    dkv = np.zeros_like(kv)
    dsink = np.zeros(H) if sink is not None else None
    z = np.full(H, NEG_INF) if sink is None else np.asarray(sink, dtype=np.float64)
    for t in range(t_q):
        sel = np.asarray(idx[t, :length[t]], dtype=np.int64)
        ksel = kv[sel]
        vsel = kv[sel, :dv]
        s = scale * (q[t] @ ksel.T)                          # [H, L]
        p, ps, _ = _row_softmax(s, np.ones(s.shape, bool), z)
        dP = d_o[t] @ vsel.T                                 # [H, L]
        D = np.sum(d_o[t] * o[t], axis=-1)                   # [H]
        gam = scale * p * (dP - D[:, None])                  # G = c dS
        dq[t] = gam @ ksel
        contrib = gam.T @ q[t]                               # dK_sel [L, Dqk]
        contrib[:, :dv] += p.T @ d_o[t]                      # + dV_sel
        np.add.at(dkv, sel, contrib)
        if dsink is not None:
            dsink += -ps * D
    return dq, dkv, dsink


def topk_dsink(q, kv, idx, length, dv: int, scale: float, d_o, sink):
    """dz_h = -sum_t p_sink[t, h] D[t, h] with D = <dO, O> (DSA note,
    section 3.5), from the forward pass alone."""
    o, _, p_sink = topk_forward(q, kv, idx, length, dv, scale, sink)
    D = np.sum(np.asarray(d_o, dtype=np.float64) * o, axis=-1)     # [Tq, H]
    return -np.sum(p_sink * D, axis=0)


# ---------------------------------------------------------------------------
# The running-summary recurrence itself
# ---------------------------------------------------------------------------

@dataclass
class TileCard:
    """State of the traced row after one key tile has contributed."""
    key_start: int
    key_end: int
    m: float
    alpha: float
    ell: float
    u: np.ndarray


def tiled_forward(q, k, v, allowed, scale: float, tile_q: int, tile_k: int,
                  key_tile_order=None, trace_row: int | None = None):
    """One (batch, head) slice through the tiled recurrence.

    "Accumulate attention without keeping the full grid", section "Rescale
    earlier mass before adding a new tile": each row starts from m = -inf,
    ell = 0, u = 0 (the state "bottom" of the exactness proof, step 1.1); for
    each key tile with a nonempty eligible set J,
        a = max_{j in J} s_j,  m' = max(m, a),  alpha = exp(m - m'),
        p_j = exp(s_j - m'),  ell' = alpha ell + sum p_j,
        u' = alpha u + sum p_j v_j,
    with alpha = 0 for the first contributing tile; a tile with J empty
    leaves (m, ell, u) untouched. After the last tile o = u / ell.

    q [n,d], k [n_k,d], v [n_k,dv], allowed bool [n,n_k].
    key_tile_order: permutation of the key-tile indices (default ascending)
    to exercise merge-order independence.
    Returns (y [n,dv], m [n], ell [n], cards for trace_row).
    """
    q, k, v = (np.asarray(x, dtype=np.float64) for x in (q, k, v))
    n, n_k, dv = q.shape[0], k.shape[0], v.shape[1]
    allowed = np.asarray(allowed, dtype=bool)
    m = np.full(n, NEG_INF)
    ell = np.zeros(n)
    u = np.zeros((n, dv))
    n_kt = (n_k + tile_k - 1) // tile_k
    order = list(range(n_kt)) if key_tile_order is None else list(key_tile_order)
    cards: list[TileCard] = []
    for q0 in range(0, n, tile_q):
        q1 = min(q0 + tile_q, n)
        for kt in order:
            k0, k1 = kt * tile_k, min((kt + 1) * tile_k, n_k)
            s_tile = scale * (q[q0:q1] @ k[k0:k1].T)
            for r in range(q0, q1):
                J = allowed[r, k0:k1]
                if not J.any():
                    continue
                s = s_tile[r - q0]
                a = s[J].max()
                m_new = max(m[r], a)
                alpha = 0.0 if ell[r] == 0.0 else np.exp(m[r] - m_new)
                p = np.where(J, np.exp(np.where(J, s, m_new) - m_new), 0.0)
                ell[r] = alpha * ell[r] + p.sum()
                u[r] = alpha * u[r] + p @ v[k0:k1]
                m[r] = m_new
                if trace_row == r:
                    cards.append(TileCard(k0, k1, float(m_new), float(alpha),
                                          float(ell[r]), u[r].copy()))
    y = np.zeros((n, dv))
    nz = ell > 0
    y[nz] = u[nz] / ell[nz, None]
    return y, m, ell, cards


# ---------------------------------------------------------------------------
# Block summaries and their merge ("Tiled attention and its recomputed reverse
# pass are exact", proof step 1.1; "Two merge orders give the same attention
# summary", alphabetamath.cc examples)
# ---------------------------------------------------------------------------

def block_summary(s_row: np.ndarray, v: np.ndarray, J: np.ndarray):
    """Sigma_i(I) = (m, ell, z) over the allowed keys J of one block, or None
    (the state bottom) when J is empty."""
    J = np.asarray(J, dtype=bool)
    if not J.any():
        return None
    m = float(np.max(s_row[J]))
    w = np.exp(s_row[J] - m)
    return m, float(w.sum()), w @ np.asarray(v)[J]


def merge_summaries(a, b):
    """Merge two summaries of disjoint key sets (None is the empty state)."""
    if a is None:
        return b
    if b is None:
        return a
    m = max(a[0], b[0])
    ea, eb = np.exp(a[0] - m), np.exp(b[0] - m)
    return m, ea * a[1] + eb * b[1], ea * np.asarray(a[2]) + eb * np.asarray(b[2])


# ---------------------------------------------------------------------------
# LSE conventions (DSA note, sections 7.1-7.3)
# ---------------------------------------------------------------------------

def _log_sum_exp_allowed(s: np.ndarray, allow: np.ndarray) -> np.ndarray:
    """ln sum_{j allowed} exp(s_j) along the last axis; -inf for an empty row."""
    sm = np.where(allow, s, NEG_INF)
    m = sm.max(axis=-1, initial=NEG_INF)
    shift = np.where(np.isfinite(m), m, 0.0)
    tot = np.where(allow, np.exp(sm - shift[..., None]), 0.0).sum(axis=-1)
    with np.errstate(divide="ignore"):
        return np.where(tot > 0, shift + np.log(np.where(tot > 0, tot, 1.0)), NEG_INF)


def kv_only_lse(q, k, allowed, scale: float) -> np.ndarray:
    """LSE_kv = ln sum_{j in A_i} exp(s_ij), the sink left out (DSA note,
    section 7.2). q [B,Hq,Tq,d], k [B,Hkv,Tk,d]; returns [B,Hq,Tq]."""
    q, k = np.asarray(q, dtype=np.float64), np.asarray(k, dtype=np.float64)
    B, Hq, Tq, _ = q.shape
    Hkv, Tk = k.shape[1], k.shape[2]
    allow = _bcast_allowed(allowed, B, Hq, Tq, Tk)
    out = np.empty((B, Hq, Tq))
    for b in range(B):
        for h in range(Hq):
            out[b, h] = _log_sum_exp_allowed(scale * (q[b, h] @ k[b, h // (Hq // Hkv)].T), allow[b, h])
    return out


def topk_kv_only_lse(q, kv, idx, length, scale: float) -> np.ndarray:
    """LSE_kv of the shared-KV top-k layout: [Tq, H], each listed position
    counted once, -inf for an empty list."""
    q, kv = np.asarray(q, dtype=np.float64), np.asarray(kv, dtype=np.float64)
    out = np.empty(q.shape[:2])
    for t in range(q.shape[0]):
        sel = np.asarray(idx[t, :length[t]], dtype=np.int64)
        s = scale * (q[t] @ kv[sel].T)
        out[t] = _log_sum_exp_allowed(s, np.ones(s.shape, bool))
    return out


def combine_lse(lse_kv: np.ndarray, z) -> np.ndarray:
    """LSE_total = logaddexp(LSE_kv, z), the first step of a backward pass
    that was handed a KV-only LSE while a sink is enabled (section 7.2)."""
    return np.logaddexp(np.asarray(lse_kv, dtype=np.float64), z)


def scaled_lse(lse: np.ndarray) -> np.ndarray:
    """The base-2 stored form of section 7.3: scaled_LSE = -log2 Z for
    LSE = ln Z (an empty row, LSE = -inf, gives +inf)."""
    return -np.asarray(lse, dtype=np.float64) / np.log(2.0)

"""Pins for the float64 oracle: worked examples printed on the pages, closed
forms, finite differences, invariants and published generator vectors.

Each pin is chosen so that a plausible slip in the oracle (a dropped term, a
wrong sign, a transposed operand, a wrong group map, a mis-indexed counter)
fails at least one test. None of these tests uses the CUDA library.
"""
import json
import math
import os

import numpy as np
import pytest

import oracle
from oracle import attention as A
from oracle import philox as P

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def _golden(name):
    with open(os.path.join(GOLDEN, name)) as f:
        return json.load(f)


def _as4(x):
    return np.asarray(x, dtype=np.float64)[None, None]


# ---------------------------------------------------------------------------
# Worked examples of the pages
# ---------------------------------------------------------------------------

def test_one_key_example():
    ex = _golden("worked_examples.json")["one_key"]
    q, k, v, g = (_as4(ex[n]) for n in ("q", "k", "v", "g"))
    allow = np.array(ex["allowed"], bool)
    fw = A.forward(q, k, v, allow, ex["scale"])
    assert np.allclose(fw.y[0, 0], ex["y"], atol=0)
    bw = A.backward(q, k, v, g, allow, ex["scale"])
    assert np.allclose(bw.dq[0, 0], ex["dq"], atol=1e-15)
    assert np.allclose(bw.dk[0, 0], ex["dk"], atol=1e-15)
    assert np.allclose(bw.dv[0, 0], ex["dv"], atol=1e-15)
    assert np.allclose(bw.delta[0, 0], ex["delta"])
    s = A.block_summary(np.array([6.0]), np.array([[7.0]]), np.array([True]))
    assert s[0] == ex["summary"][0] and s[1] == ex["summary"][1]
    assert np.allclose(s[2], [ex["summary"][2]])
    y, _, _, _ = A.tiled_forward(q[0, 0], k[0, 0], v[0, 0], allow, 1.0, 1, 1)
    assert np.allclose(y, ex["y"])


def test_empty_first_block_example():
    ex = _golden("worked_examples.json")["empty_first_block"]
    q, k, v = (np.array(ex[n], float) for n in ("q", "k", "v"))
    allow = np.array(ex["allowed"], bool)
    fw = A.forward(q[None, None], k[None, None], v[None, None], allow, 1.0)
    assert np.allclose(fw.y[0, 0], ex["y"])
    y, m, ell, cards = A.tiled_forward(q, k, v, allow, 1.0, 1, ex["block"], trace_row=1)
    assert np.allclose(y, ex["y"])
    # Row 2 (index 1): summary (0,1,3) after block 1, (0,2,8) after block 2.
    got = [(c.m, c.ell, float(c.u[0])) for c in cards]
    assert got == [tuple(map(float, s)) for s in ex["row2_summaries"]]
    # Row 1 (index 0) skipped its empty first block: only one card.
    _, _, _, cards0 = A.tiled_forward(q, k, v, allow, 1.0, 1, 1, trace_row=0)
    assert len(cards0) == 1 and cards0[0].key_start == 1 and cards0[0].alpha == 0.0


def test_merge_order_example():
    ex = _golden("worked_examples.json")["merge_orders"]
    q, k, v = (np.array(ex[n], float) for n in ("q", "k", "v"))
    s = (q @ k.T)[0]
    s1 = A.block_summary(s, v, np.array([True, False]))
    s2 = A.block_summary(s, v, np.array([False, True]))
    assert np.allclose([s1[0], s1[1], s1[2][0]], ex["summary_block1"])
    assert np.allclose([s2[0], s2[1], s2[2][0]], ex["summary_block2"])
    for a, b in ((s1, s2), (s2, s1)):
        m = A.merge_summaries(a, b)
        assert np.allclose([m[0], m[1], m[2][0]], ex["merged"], rtol=1e-15)
        assert math.isclose(m[2][0] / m[1], 2.0, rel_tol=1e-15)
    assert A.merge_summaries(None, s1) is s1 and A.merge_summaries(s2, None) is s2
    allow = np.array(ex["allowed"], bool)
    for order in ([0, 1], [1, 0]):
        y, *_ = A.tiled_forward(q, k, v, allow, 1.0, 1, 1, key_tile_order=order)
        assert np.allclose(y, ex["y"], rtol=1e-15)


def test_dropout_replay_example():
    ex = _golden("worked_examples.json")["dropout_replay"]
    q, k, v, g = (np.array(ex[n], float)[None, None] for n in ("q", "k", "v", "g"))
    allow = np.ones((2, 2), bool)
    rho = ex["rho"]
    for xi, dv_expect in ((ex["xi_row1"], ex["dv"]), (ex["xi_row1_alt"], ex["dv_alt"])):
        keep = np.ones((1, 1, 2, 2), bool)
        keep[0, 0, 0] = np.array(xi, bool)
        fw = A.forward(q, k, v, allow, 1.0, keep=keep, rho=rho)
        bw = A.backward(q, k, v, g, allow, 1.0, keep=keep, rho=rho)
        assert np.allclose(bw.dv[0, 0], dv_expect)
        if xi == ex["xi_row1"]:
            assert np.allclose(fw.y[0, 0, 0], ex["y_row1"])


def test_sink_example_dense_and_topk():
    ex = _golden("worked_examples.json")["sink"]
    p1, p2 = ex["p"]
    z = math.log(ex["p_sink"])
    # Dense realisation: d = dv = 1, c = 1, Q = [1], K = (ln p1, ln p2) so
    # that Z = exp(z) + p1 + p2 = 1 and the printed probabilities appear.
    q = np.array([[1.0]])[None, None]
    k = np.array([[math.log(p1)], [math.log(p2)]])[None, None]
    v = np.array([[ex["v"][0]], [ex["v"][1]]])[None, None]
    g = np.array([[ex["g"]]], float)[None, None]
    sink = np.array([z])
    allow = np.ones((1, 2), bool)
    fw = A.forward(q, k, v, allow, 1.0, sink=sink)
    assert math.isclose(fw.y[0, 0, 0, 0], ex["o"], rel_tol=1e-14)
    assert math.isclose(fw.p_sink[0, 0, 0], ex["p_sink"], rel_tol=1e-14)
    assert abs(fw.lse[0, 0, 0]) < 1e-15                       # ln Z = ln 1
    bw = A.backward(q, k, v, g, allow, 1.0, sink=sink)
    assert np.allclose(bw.dk[0, 0, :, 0], ex["dS"], atol=1e-14)   # dK_j = c gamma_j Q
    assert math.isclose(bw.dsink[0], ex["dz"], rel_tol=1e-13)
    assert np.allclose(bw.dv[0, 0, :, 0], ex["p"], atol=1e-15)
    dq_expect = ex["dS"][0] * math.log(p1) + ex["dS"][1] * math.log(p2)
    assert math.isclose(bw.dq[0, 0, 0, 0], dq_expect, rel_tol=1e-13)
    # Softmax shift invariance: the three logit gradients sum to zero.
    assert abs(sum(ex["dS"]) + ex["dz"]) < 1e-15
    assert abs(bw.dk[0, 0, :, 0].sum() + bw.dsink[0]) < 1e-14
    # Tied top-k realisation: KV rows (v_j, ln p_j), Q = (0, 1), Dv = 1.
    kv = np.array([[ex["v"][0], math.log(p1)], [ex["v"][1], math.log(p2)]])
    qt = np.array([[[0.0, 1.0]]])
    idx = np.array([[0, 1]], np.int32)
    ln = np.array([2], np.int32)
    o, lse, ps = A.topk_forward(qt, kv, idx, ln, 1, 1.0, sink)
    assert math.isclose(o[0, 0, 0], ex["o"], rel_tol=1e-14)
    dq, dkv, dsink = A.topk_backward(qt, kv, idx, ln, 1, 1.0,
                                     np.array([[[ex["g"]]]], float), sink)
    assert np.allclose(dkv[:, 1], ex["dS"], atol=1e-14)
    assert np.allclose(dkv[:, 0], ex["p"], atol=1e-14)          # 0 * G + p g
    assert math.isclose(dsink[0], ex["dz"], rel_tol=1e-13)
    assert np.allclose(dq[0, 0], ex["dS"][0] * kv[0] + ex["dS"][1] * kv[1], atol=1e-14)


def test_two_tile_trace_cards():
    gd = _golden("two_tile_trace.json")
    inp = gd["inputs"]
    q, k, v = (np.array(inp[n], float) for n in ("q", "k", "v"))
    allow = A.allowed_dense(4, 4, causal=True)
    y, m, ell, cards = A.tiled_forward(q, k, v, allow, inp["scale"], inp["tile_q"],
                                       inp["tile_k"], trace_row=inp["trace_row"])
    assert len(cards) == 2
    for card, want in zip(cards, gd["cards"]):
        assert (card.key_start, card.key_end) == (want["key_start"], want["key_end"])
        assert card.m == want["m"]
        assert math.isclose(card.alpha, want["alpha"], rel_tol=1e-15, abs_tol=0)
        assert math.isclose(card.ell, want["ell"], rel_tol=1e-15)
        assert np.allclose(card.u, want["u"], rtol=1e-15, atol=0)
    assert np.allclose(y[3], gd["tiled_output_row3"], rtol=1e-15, atol=0)
    fw = A.forward(q[None, None], k[None, None], v[None, None], allow, 1.0)
    assert np.allclose(fw.y[0, 0, 3], gd["dense_output_row3"], rtol=1e-15, atol=0)
    err = np.abs(fw.y[0, 0] - y).max()
    assert err <= gd["published_tolerance"]


def test_two_tile_example_gradients_by_finite_differences():
    gd = _golden("two_tile_trace.json")
    inp = gd["inputs"]
    q, k, v = (np.array(inp[n], float)[None, None] for n in ("q", "k", "v"))
    g = np.array(gd["gradient_upstream_seed"], float).reshape(1, 1, 4, 2)
    allow = A.allowed_dense(4, 4, causal=True)
    _check_fd(q, k, v, g, allow, 1.0)


# ---------------------------------------------------------------------------
# Finite differences (the page's small-kernel test design: every coordinate,
# central differences with step 1e-6 and absolute tolerance 4e-6)
# ---------------------------------------------------------------------------

def _loss(q, k, v, g, allow, scale, sink=None, keep=None, rho=0.0):
    return float(np.sum(g * A.forward(q, k, v, allow, scale, sink, keep, rho).y))


def _check_fd(q, k, v, g, allow, scale, sink=None, keep=None, rho=0.0,
              step=1e-6, tol=4e-6):
    bw = A.backward(q, k, v, g, allow, scale, sink, keep, rho)
    pairs = [(q, bw.dq), (k, bw.dk), (v, bw.dv)]
    if sink is not None:
        pairs.append((sink, bw.dsink))
    for x, grad in pairs:
        flat = x.reshape(-1)
        for idx in range(flat.size):
            old = flat[idx]
            flat[idx] = old + step
            up = _loss(q, k, v, g, allow, scale, sink, keep, rho)
            flat[idx] = old - step
            dn = _loss(q, k, v, g, allow, scale, sink, keep, rho)
            flat[idx] = old
            fd = (up - dn) / (2 * step)
            assert abs(fd - grad.reshape(-1)[idx]) <= tol, (idx, fd, grad.reshape(-1)[idx])


@pytest.mark.parametrize("variant", ["mha_causal", "gqa_window", "mqa_block", "sink",
                                     "dropout", "large_equal_scores"])
def test_finite_differences(variant):
    rng = np.random.default_rng(sum(map(ord, variant)))
    B, Hq, Hkv, T, d, dv = 1, 2, 2, 7, 3, 2
    scale = 1 / math.sqrt(d)
    sink = keep = None
    rho = 0.0
    kw = {}
    if variant == "mha_causal":
        kw = dict(causal=True)
    elif variant == "gqa_window":
        B, Hq, Hkv = 2, 4, 2
        kw = dict(causal=True, window_left=3)
    elif variant == "mqa_block":
        B, Hq, Hkv = 2, 3, 1
        bm = rng.random((2, 4, 4)) < 0.5
        bm[:, np.arange(4), np.arange(4)] = True
        kw = dict(causal=True, block_mask=bm[:, None], block_q=2, block_k=2)
    elif variant == "sink":
        kw = dict(causal=True)
        sink = rng.standard_normal(Hq)
    elif variant == "dropout":
        rho = 0.3
        kw = dict(causal=True)
        keep = rng.random((B, Hq, T, T)) >= rho
    elif variant == "large_equal_scores":
        kw = dict(causal=True)
    q = rng.standard_normal((B, Hq, T, d))
    k = rng.standard_normal((B, Hkv, T, d))
    v = rng.standard_normal((B, Hkv, T, dv))
    g = rng.standard_normal((B, Hq, T, dv))
    if variant == "large_equal_scores":
        q *= 0.0
        q += 3.0
        k[:] = 4.0          # every score equal and large (tied maxima)
        k[..., 0, :] += 1e-3
    allow = A.allowed_dense(T, T, **kw)
    _check_fd(q, k, v, g, allow, scale, sink, keep, rho)


# ---------------------------------------------------------------------------
# Tiled recurrence equals the dense definition; invariants
# ---------------------------------------------------------------------------

@pytest.mark.parametrize("seed", range(6))
def test_tiled_recurrence_matches_dense(seed):
    rng = np.random.default_rng(100 + seed)
    n, d, dv = int(rng.integers(5, 40)), int(rng.integers(1, 6)), int(rng.integers(1, 5))
    tq, tk = int(rng.integers(1, 9)), int(rng.integers(1, 9))
    q, k, v = rng.standard_normal((n, d)), rng.standard_normal((n, d)), rng.standard_normal((n, dv))
    bm = rng.random(((n + 2) // 3, (n + 2) // 3)) < 0.4
    np.fill_diagonal(bm, True)
    allow = A.allowed_dense(n, n, causal=True, window_left=int(rng.integers(0, n)),
                            block_mask=bm, block_q=3, block_k=3)
    y_dense = A.forward(q[None, None], k[None, None], v[None, None], allow, 0.7).y[0, 0]
    n_kt = (n + tk - 1) // tk
    for order in (None, list(rng.permutation(n_kt))):
        y, m, ell, _ = A.tiled_forward(q, k, v, allow, 0.7, tq, tk, key_tile_order=order)
        assert np.abs(y - y_dense).max() <= 1e-12
        assert np.all(ell[allow.any(1)] > 0)                # ell_i > 0 when A_i nonempty
        assert np.all(np.isfinite(m[allow.any(1)]))


def test_invariants_probability_mass_and_identities():
    rng = np.random.default_rng(7)
    B, Hq, Hkv, T, d, dv = 2, 4, 2, 33, 8, 5
    q = rng.standard_normal((B, Hq, T, d))
    k = rng.standard_normal((B, Hkv, T, d))
    v = rng.standard_normal((B, Hkv, T, dv))
    g = rng.standard_normal((B, Hq, T, dv))
    sink = rng.standard_normal(Hq)
    rho = 0.25
    keep = rng.random((B, Hq, T, T)) >= rho
    allow = A.allowed_dense(T, T, causal=True, window_left=9)
    c = 0.3
    fw = A.forward(q, k, v, allow, c, sink=sink, keep=keep, rho=rho)
    bw = A.backward(q, k, v, g, allow, c, sink=sink, keep=keep, rho=rho)
    # sum_j p_ij + p_sink,i = 1, from the saved LSE.
    for b in range(B):
        for h in range(Hq):
            s = c * q[b, h] @ k[b, h // 2].T
            p = np.where(allow, np.exp(s - fw.lse[b, h][:, None]), 0)
            mass = p.sum(1) + np.exp(sink[h] - fw.lse[b, h])
            assert np.allclose(mass, 1.0, atol=1e-13)
    # sum_i Q_i.dQ_i = sum_j K_j.dK_j (both equal sum gamma_ij s_ij / c * c).
    assert math.isclose(np.sum(q * bw.dq), np.sum(k * bw.dk), rel_tol=1e-10)
    # sum_j V_j.dV_j = sum_i G_i.Y_i.
    assert math.isclose(np.sum(v * bw.dv), np.sum(g * fw.y), rel_tol=1e-10)
    # Shift invariance per row: sum_j gamma_ij - p_sink delta = 0, summed over rows
    # and heads it is sum over h of (sum_j dS) + dsink_h.


def test_empty_rows_are_zero_and_lse_conventions():
    q = np.ones((1, 1, 3, 2))
    k = np.ones((1, 1, 3, 2))
    v = np.arange(6, dtype=float).reshape(1, 1, 3, 2)
    allow = np.array([[0, 0, 0], [1, 0, 0], [1, 1, 0]], bool)
    fw = A.forward(q, k, v, allow, 1.0)
    assert np.all(fw.y[0, 0, 0] == 0) and fw.lse[0, 0, 0] == -np.inf
    sink = np.array([0.5])
    fw2 = A.forward(q, k, v, allow, 1.0, sink=sink)
    assert fw2.lse[0, 0, 0] == 0.5 and fw2.p_sink[0, 0, 0] == 1.0
    bw = A.backward(q, k, v, np.ones((1, 1, 3, 2)), allow, 1.0, sink=sink)
    assert np.all(bw.dq[0, 0, 0] == 0)


# ---------------------------------------------------------------------------
# Top-k reduces to the dense definition with the selected allowed sets
# ---------------------------------------------------------------------------

def test_topk_equals_dense_with_selected_sets():
    rng = np.random.default_rng(11)
    Tq, Tkv, H, Dqk, Dv, topk = 5, 12, 3, 6, 4, 6
    q = rng.standard_normal((Tq, H, Dqk))
    kv = rng.standard_normal((Tkv, Dqk))
    d_o = rng.standard_normal((Tq, H, Dv))
    sink = rng.standard_normal(H)
    from exact_tiled_attention_softmax_b200.workloads import topk_lists
    idx, ln = topk_lists(Tq, Tkv, topk, 2, topk, 3)
    c = 0.4
    o, lse, ps = A.topk_forward(q, kv, idx, ln, Dv, c, sink)
    dq, dkv, dsink = A.topk_backward(q, kv, idx, ln, Dv, c, d_o, sink)
    allow = A.topk_allowed(idx, ln, Tkv)
    qd = q.transpose(1, 0, 2)[None]                     # [1,H,Tq,Dqk]
    kd = kv[None, None]
    vd = kv[None, None, :, :Dv]
    fw = A.forward(qd, kd, vd, allow, c, sink=sink)
    bw = A.backward(qd, kd, vd, d_o.transpose(1, 0, 2)[None], allow, c, sink=sink)
    assert np.allclose(o, fw.y[0].transpose(1, 0, 2), atol=1e-13)
    assert np.allclose(lse, fw.lse[0].T, atol=1e-13)
    assert np.allclose(dq, bw.dq[0].transpose(1, 0, 2), atol=1e-12)
    dkv_dense = bw.dk[0, 0].copy()
    dkv_dense[:, :Dv] += bw.dv[0, 0]
    assert np.allclose(dkv, dkv_dense, atol=1e-12)
    assert np.allclose(dsink, bw.dsink, atol=1e-12)
    assert np.allclose(A.topk_dsink(q, kv, idx, ln, Dv, c, d_o, sink), bw.dsink, atol=1e-12)


def test_topk_lists_are_causal_and_distinct():
    from exact_tiled_attention_softmax_b200.workloads import topk_lists
    idx, ln = topk_lists(64, 256, 128, 40, 128, 9)
    for t in range(64):
        sel = idx[t, :ln[t]]
        assert len(set(sel.tolist())) == ln[t]
        assert sel.min() >= 0 and sel.max() <= 256 - 64 + t
        assert np.all(idx[t, ln[t]:] == -1)


# ---------------------------------------------------------------------------
# Philox and the dropout mask
# ---------------------------------------------------------------------------

def test_philox_known_answers():
    kat = _golden("philox4x32_10_kat.json")
    for vec in kat["vectors"]:
        ctr = np.array([int(x, 16) for x in vec["counter"]], dtype=np.uint64)
        key = np.array([int(x, 16) for x in vec["key"]], dtype=np.uint64)
        out = P.philox4x32(ctr, key)
        assert [int(x) for x in out] == [int(x, 16) for x in vec["out"]]


def test_dropout_mask_counter_layout_and_rate():
    seed, rho = 0x123456789ABCDEF, 0.1
    keep = P.dropout_keep(seed, rho, 2, 3, 9, 11)
    thr = P.keep_threshold(rho)
    # Element (b=1, h=2, i=5, j=7): counter (7>>2, 5, 2, 1), word 7&3.
    w = P.philox4x32(np.array([1, 5, 2, 1], np.uint64),
                     np.array([seed & 0xFFFFFFFF, seed >> 32], np.uint64))
    assert keep[1, 2, 5, 7] == (int(w[3]) >= thr)
    assert np.array_equal(keep, P.dropout_keep(seed, rho, 2, 3, 9, 11))  # replay
    big = P.dropout_keep(99, rho, 1, 2, 300, 300)
    n = big.size
    rate = big.mean()
    sigma = math.sqrt(rho * (1 - rho) / n)
    assert abs(rate - (1 - rho)) < 6 * sigma
    assert P.keep_threshold(0.0) == 0
    with pytest.raises(ValueError):
        P.keep_threshold(1.0)


def test_dropout_replay_seed_search():
    """A seed whose realisation for query row 0 is xi = (1, 0) exists and
    reproduces the replay example through the generated mask."""
    ex = _golden("worked_examples.json")["dropout_replay"]
    seed = find_replay_seed()
    keep = P.dropout_keep(seed, 0.5, 1, 1, 2, 2)
    assert keep[0, 0, 0].tolist() == [True, False]
    q, k, v, g = (np.array(ex[n], float)[None, None] for n in ("q", "k", "v", "g"))
    bw = A.backward(q, k, v, g, np.ones((2, 2), bool), 1.0, keep=keep, rho=0.5)
    assert np.allclose(bw.dv[0, 0], ex["dv"])


def find_replay_seed():
    for seed in range(1, 1000):
        if P.dropout_keep(seed, 0.5, 1, 1, 2, 2)[0, 0, 0].tolist() == [True, False]:
            return seed
    raise AssertionError("no seed found")


def test_oracle_detects_planted_mistakes():
    """Mutation check: flipping the sign of delta or transposing the value
    gradient makes the finite-difference pin fail."""
    rng = np.random.default_rng(5)
    q = rng.standard_normal((1, 1, 4, 2))
    k = rng.standard_normal((1, 1, 4, 2))
    v = rng.standard_normal((1, 1, 4, 3))
    g = rng.standard_normal((1, 1, 4, 3))
    allow = A.allowed_dense(4, 4, causal=True)
    good = A.backward(q, k, v, g, allow, 0.5)
    orig = A.backward

    def bad_backward(*a, **kw):
        r = orig(*a, **kw)
        r.dq = -r.dq
        return r
    A.backward = bad_backward
    try:
        with pytest.raises(AssertionError):
            _check_fd(q, k, v, g, allow, 0.5)
    finally:
        A.backward = orig
    assert np.abs(good.dq).max() > 1e-3


# ---------------------------------------------------------------------------
# Row/column-restricted evaluation equals the full definition
# ---------------------------------------------------------------------------

def test_sampled_rows_and_columns_match_full_oracle():
    from oracle import sampled as S
    rng = np.random.default_rng(17)
    B, Hq, Hkv, T, d, dv = 1, 4, 2, 37, 6, 5
    q = rng.standard_normal((B, Hq, T, d))
    k = rng.standard_normal((B, Hkv, T, d))
    v = rng.standard_normal((B, Hkv, T, dv))
    g = rng.standard_normal((B, Hq, T, dv))
    sink = rng.standard_normal(Hq)
    rho, seed, c = 0.2, 77, 0.45
    bm = rng.random((5, 5)) < 0.6
    np.fill_diagonal(bm, True)
    kw = dict(causal=True, window_left=11, block_mask=bm, block_q=8, block_k=8)
    allow = A.allowed_dense(T, T, **kw)
    keep = P.dropout_keep(seed, rho, B, Hq, T, T)
    fw = A.forward(q, k, v, allow, c, sink=sink, keep=keep, rho=rho)
    bw = A.backward(q, k, v, g, allow, c, sink=sink, keep=keep, rho=rho)
    rows = np.array([0, 3, 17, 36])
    cols = np.array([1, 20, 36])
    gq = Hq // Hkv
    for h in range(Hq):
        ar = S.allowed_at(rows, np.arange(T), **kw)
        assert np.array_equal(ar, allow[rows])
        kr = S.keep_at(seed, rho, 0, h, rows, np.arange(T))
        assert np.array_equal(kr, keep[0, h][rows])
        y, lse, delta, dq = S.rows_forward_backward(q[0, h], k[0, h // gq], v[0, h // gq], g[0, h], rows, ar, c,
                                                    z=sink[h], keep_rows=kr, rho=rho)
        assert np.allclose(y, fw.y[0, h][rows], atol=1e-13)
        assert np.allclose(lse, fw.lse[0, h][rows], atol=1e-13)
        assert np.allclose(dq, bw.dq[0, h][rows], atol=1e-12)
        assert np.allclose(delta, bw.delta[0, h][rows], atol=1e-12)
    for kvh in range(Hkv):
        heads = [kvh * gq + hh for hh in range(gq)]
        dk, dvv = S.cols_backward(
            [q[0, h] for h in heads], [g[0, h] for h in heads], k[0, kvh], v[0, kvh], cols,
            lambda hh, r, cc: S.allowed_at(r, cc, **kw),
            [fw.lse[0, h] for h in heads], [bw.delta[0, h] for h in heads], c,
            keep_fn=lambda hh, r, cc, hs=heads: S.keep_at(seed, rho, 0, hs[hh], r, cc), rho=rho)
        assert np.allclose(dk, bw.dk[0, kvh][cols], atol=1e-12)
        assert np.allclose(dvv, bw.dv[0, kvh][cols], atol=1e-12)


def test_keep_range_equals_the_full_mask():
    """The block-wise keep evaluator gives the full mask's values on every
    row and contiguous key range it is asked for (ranges starting on a
    4-key block, ending anywhere)."""
    from oracle import sampled as S
    seed, rho, B, Hq, T = (1 << 40) + 123, 0.3, 2, 3, 45
    keep = P.dropout_keep(seed, rho, B, Hq, T, T)
    rows = np.array([0, 5, 44])
    for b, h, c0, c1 in ((0, 0, 0, 45), (1, 2, 8, 9), (1, 1, 4, 43), (0, 2, 40, 45)):
        got = S.keep_range(seed, rho, b, h, rows, c0, c1)
        assert np.array_equal(got, keep[b, h][rows][:, c0:c1])
        assert np.array_equal(got, S.keep_at(seed, rho, b, h, rows, np.arange(c0, c1)))
    with pytest.raises(ValueError):
        S.keep_range(seed, rho, 0, 0, rows, 2, 10)


def test_topk_empty_list_gives_zero_output_and_sink_lse():
    """An empty selection is an empty allowed set: Y = 0 and LSE = z with a
    sink, -inf without one; the other tokens are unaffected."""
    rng = np.random.default_rng(9)
    q = rng.standard_normal((2, 3, 8))
    kv = rng.standard_normal((10, 8))
    idx = np.array([[1, 4, 7], [0, 0, 0]], dtype=np.int32)
    ln = np.array([3, 0], dtype=np.int32)
    z = np.array([0.5, -1.0, 2.0])
    o, lse, ps = oracle.topk_forward(q, kv, idx, ln, 4, 0.3, z)
    assert np.all(o[1] == 0.0) and np.allclose(lse[1], z) and np.allclose(ps[1], 1.0)
    o2, lse2, _ = oracle.topk_forward(q, kv, idx, ln, 4, 0.3, None)
    assert np.all(o2[1] == 0.0) and np.all(np.isneginf(lse2[1]))
    o1, lse1, _ = oracle.topk_forward(q[:1], kv, idx[:1], ln[:1], 4, 0.3, z)
    assert np.allclose(o1[0], o[0]) and np.allclose(lse1[0], lse[0])


# ---------------------------------------------------------------------------
# Row-interval layouts: a query block against a longer key range, packed
# segments (per-row lower bound) and active lengths
# ---------------------------------------------------------------------------

def _rand(rng, *shape):
    return rng.standard_normal(shape)


def test_query_block_equals_trailing_rows_of_full_causal():
    """Bottom-right alignment: the last Tq query rows of causal attention over
    Tk cells, evaluated as a separate Tq-row block, give the same rows, LSE
    and (with the upstream gradient zero on the other rows) the same K/V
    gradients as the full Tk x Tk causal problem."""
    rng = np.random.default_rng(301)
    B, Hq, Hkv, Tk, Tq, d, dv = 2, 4, 2, 23, 9, 5, 3
    q, k, v = _rand(rng, B, Hq, Tk, d), _rand(rng, B, Hkv, Tk, d), _rand(rng, B, Hkv, Tk, dv)
    g = _rand(rng, B, Hq, Tk, dv)
    g[:, :, :Tk - Tq] = 0.0
    sink = _rand(rng, Hq)
    full_allow = A.allowed_dense(Tk, Tk, causal=True, window_left=6)
    blk_allow = A.allowed_dense(Tq, Tk, causal=True, window_left=6, query_offset=Tk - Tq)
    fw_full = A.forward(q, k, v, full_allow, 0.4, sink=sink)
    fw_blk = A.forward(q[:, :, Tk - Tq:], k, v, blk_allow, 0.4, sink=sink)
    np.testing.assert_allclose(fw_blk.y, fw_full.y[:, :, Tk - Tq:], rtol=0, atol=1e-13)
    np.testing.assert_allclose(fw_blk.lse, fw_full.lse[:, :, Tk - Tq:], rtol=0, atol=1e-13)
    bw_full = A.backward(q, k, v, g, full_allow, 0.4, sink=sink)
    bw_blk = A.backward(q[:, :, Tk - Tq:], k, v, g[:, :, Tk - Tq:], blk_allow, 0.4, sink=sink)
    np.testing.assert_allclose(bw_blk.dq, bw_full.dq[:, :, Tk - Tq:], rtol=0, atol=1e-12)
    np.testing.assert_allclose(bw_blk.dk, bw_full.dk, rtol=0, atol=1e-12)
    np.testing.assert_allclose(bw_blk.dv, bw_full.dv, rtol=0, atol=1e-12)
    np.testing.assert_allclose(bw_blk.dsink, bw_full.dsink, rtol=0, atol=1e-12)
    # Tq > Tk: the first Tq - Tk rows sit before the first key and are empty.
    long_allow = A.allowed_dense(7, 4, causal=True, query_offset=4 - 7)
    assert not long_allow[:3].any() and long_allow[3:].sum() == 10


def test_packed_segments_equal_separate_sequences():
    """Causal attention over packed segments (starts = each row's segment
    start) equals causal attention over each segment on its own: outputs,
    LSE, all three gradients, and a sink gradient that is the sum over the
    segments."""
    rng = np.random.default_rng(302)
    B, Hq, Hkv, T, d, dv = 2, 4, 2, 41, 6, 5
    bounds = [[0, 13, 29, 41], [0, 41]]
    starts = np.zeros((B, T), dtype=np.int32)
    for b, bd in enumerate(bounds):
        for s0, s1 in zip(bd[:-1], bd[1:]):
            starts[b, s0:s1] = s0
    q, k, v = _rand(rng, B, Hq, T, d), _rand(rng, B, Hkv, T, d), _rand(rng, B, Hkv, T, dv)
    g = _rand(rng, B, Hq, T, dv)
    sink = _rand(rng, Hq)
    allow = A.allowed_dense(T, T, causal=True, starts=starts)
    assert allow.shape == (B, 1, T, T)
    fw = A.forward(q, k, v, allow, 0.3, sink=sink)
    bw = A.backward(q, k, v, g, allow, 0.3, sink=sink)
    dsink = np.zeros(Hq)
    for b, bd in enumerate(bounds):
        for s0, s1 in zip(bd[:-1], bd[1:]):
            sl = slice(s0, s1)
            one = A.allowed_dense(s1 - s0, s1 - s0, causal=True)
            f1 = A.forward(q[b:b + 1, :, sl], k[b:b + 1, :, sl], v[b:b + 1, :, sl], one, 0.3, sink=sink)
            b1 = A.backward(q[b:b + 1, :, sl], k[b:b + 1, :, sl], v[b:b + 1, :, sl], g[b:b + 1, :, sl], one,
                            0.3, sink=sink)
            np.testing.assert_allclose(fw.y[b:b + 1, :, sl], f1.y, rtol=0, atol=1e-13)
            np.testing.assert_allclose(fw.lse[b:b + 1, :, sl], f1.lse, rtol=0, atol=1e-13)
            for name in ("dq", "dk", "dv"):
                np.testing.assert_allclose(getattr(bw, name)[b:b + 1, :, sl], getattr(b1, name), rtol=0, atol=1e-12)
            dsink += b1.dsink
    np.testing.assert_allclose(bw.dsink, dsink, rtol=0, atol=1e-12)


@pytest.mark.parametrize("causal", [True, False])
def test_lengths_equal_truncated_sequences(causal):
    """Active lengths: rows and keys past L_b take no part. The active block
    equals the attention of the truncated sequence, padding rows are empty
    (Y = 0, LSE = -inf) and padding K/V rows get zero gradients."""
    rng = np.random.default_rng(303 + causal)
    B, Hq, Hkv, T, d, dv = 3, 2, 1, 19, 4, 3
    lengths = np.array([19, 7, 0], dtype=np.int32)
    q, k, v = _rand(rng, B, Hq, T, d), _rand(rng, B, Hkv, T, d), _rand(rng, B, Hkv, T, dv)
    g = _rand(rng, B, Hq, T, dv)
    allow = A.allowed_dense(T, T, causal=causal, lengths=lengths)
    fw = A.forward(q, k, v, allow, 0.5)
    bw = A.backward(q, k, v, g, allow, 0.5)
    for b, L in enumerate(lengths):
        assert np.all(fw.y[b, :, L:] == 0) and np.all(fw.lse[b, :, L:] == -np.inf)
        assert np.all(bw.dq[b, :, L:] == 0) and np.all(bw.dk[b, :, L:] == 0) and np.all(bw.dv[b, :, L:] == 0)
        if L == 0:
            continue
        one = A.allowed_dense(L, L, causal=causal)
        f1 = A.forward(q[b:b + 1, :, :L], k[b:b + 1, :, :L], v[b:b + 1, :, :L], one, 0.5)
        b1 = A.backward(q[b:b + 1, :, :L], k[b:b + 1, :, :L], v[b:b + 1, :, :L], g[b:b + 1, :, :L], one, 0.5)
        np.testing.assert_allclose(fw.y[b:b + 1, :, :L], f1.y, rtol=0, atol=1e-13)
        np.testing.assert_allclose(fw.lse[b:b + 1, :, :L], f1.lse, rtol=0, atol=1e-13)
        for name in ("dq", "dk", "dv"):
            np.testing.assert_allclose(getattr(bw, name)[b:b + 1, :, :L], getattr(b1, name), rtol=0, atol=1e-12)
    with pytest.raises(ValueError):
        A.allowed_dense(4, 6, lengths=np.array([3]))


# ---------------------------------------------------------------------------
# LSE conventions: sink-inclusive, KV-only, base-2 scaled
# ---------------------------------------------------------------------------

def test_lse_conventions_on_the_sink_example():
    """The DSA note's sink example has Z = exp(z) + p1 + p2 = 1 (scores
    ln p1, ln p2): LSE_total = 0, LSE_kv = ln(p1 + p2) = ln(1 - p_sink),
    their logaddexp with z gives back 0, and scaled_LSE = -log2 Z = 0."""
    ex = _golden("worked_examples.json")["sink"]
    p1, p2 = ex["p"]
    z = math.log(ex["p_sink"])
    q = np.array([[1.0]])[None, None]
    k = np.array([[math.log(p1)], [math.log(p2)]])[None, None]
    allow = np.ones((1, 2), bool)
    lkv = A.kv_only_lse(q, k, allow, 1.0)[0, 0, 0]
    assert math.isclose(lkv, math.log(p1 + p2), rel_tol=1e-14)
    assert math.isclose(lkv, math.log(1.0 - ex["p_sink"]), rel_tol=1e-12)
    assert abs(A.combine_lse(lkv, z)) < 1e-15
    assert A.scaled_lse(0.0) == 0.0
    assert math.isclose(A.scaled_lse(math.log(8.0)), -3.0, rel_tol=1e-15)
    assert A.scaled_lse(-np.inf) == np.inf
    kv = np.array([[0.0, math.log(p1)], [0.0, math.log(p2)]])
    lt = A.topk_kv_only_lse(np.array([[[0.0, 1.0]]]), kv, np.array([[0, 1]]), np.array([2]), 1.0)
    assert math.isclose(lt[0, 0], math.log(p1 + p2), rel_tol=1e-14)


def test_kv_only_lse_combines_to_the_sink_inclusive_lse():
    """logaddexp(LSE_kv, z) equals the forward's sink-inclusive LSE (two
    separate evaluations); without a sink the two conventions coincide; an
    empty allowed set gives LSE_kv = -inf and LSE_total = z."""
    rng = np.random.default_rng(311)
    B, Hq, Hkv, T, d = 2, 4, 2, 17, 6
    q, k, v = rng.standard_normal((B, Hq, T, d)), rng.standard_normal((B, Hkv, T, d)), \
        rng.standard_normal((B, Hkv, T, 3))
    allow = A.allowed_dense(T, T, causal=True, window_left=5)
    allow = allow & (rng.random((B, Hq, T, T)) < 0.7)
    allow[0, 0, 3] = False                          # one empty row
    sink = rng.standard_normal(Hq) * 2
    lkv = A.kv_only_lse(q, k, allow, 0.7)
    fw = A.forward(q, k, v, allow, 0.7, sink=sink)
    np.testing.assert_allclose(A.combine_lse(lkv, sink[None, :, None]), fw.lse, rtol=0, atol=1e-13)
    assert lkv[0, 0, 3] == -np.inf and fw.lse[0, 0, 3] == sink[0]
    fw0 = A.forward(q, k, v, allow, 0.7)
    np.testing.assert_array_equal(np.isfinite(lkv), np.isfinite(fw0.lse))
    fin = np.isfinite(lkv)
    np.testing.assert_allclose(lkv[fin], fw0.lse[fin], rtol=0, atol=1e-13)
    # Top-k layout: the same identity token by token.
    Tkv, H = 40, 3
    qt, kvt = rng.standard_normal((5, H, d)), rng.standard_normal((Tkv, d))
    idx = np.stack([rng.permutation(Tkv)[:8] for _ in range(5)]).astype(np.int32)
    ln = np.array([8, 3, 0, 5, 1], np.int32)
    zt = rng.standard_normal(H)
    lt = A.topk_kv_only_lse(qt, kvt, idx, ln, 0.5)
    _, lse_t, _ = A.topk_forward(qt, kvt, idx, ln, 2, 0.5, zt)
    np.testing.assert_allclose(A.combine_lse(lt, zt[None, :]), lse_t, rtol=0, atol=1e-13)
    assert np.all(lt[2] == -np.inf)

"""Full-size parity for the five workloads, in the launch configuration the
benchmark times, against the float64 oracle.

causal_2k            every head, every element.
window_block_8k      4 sampled heads (0, 9, 18, 31), every element of those heads.
gqa_dropout_16k      K/V group (b=0, kv=0): every row of its 4 query heads
                     (Y, LSE, dQ) and dK/dV on keys 0-255 (every row sees them),
                     8064-8319 and the last 256; group (b=1, kv=7): Y/LSE/dQ on
                     128 sampled rows, dK/dV on the last 256 keys.
topk_shared_kv       O/LSE/dQ on 256 sampled tokens; dKV on the last 256 KV
                     rows (selectable only by the last 256 tokens); dSink over
                     all tokens.
Plus, for every workload, exact identities over all outputs:
  sum Q.dQ = sum K.dK  and  sum V.dV = sum G.Y  (dense),
  sum KV.dKV = sum Q.dQ + sum G.O  (tied top-k).
"""
import math

import numpy as np
import pytest

torch = pytest.importorskip("torch")

pytestmark = pytest.mark.gpu

import exact_tiled_attention_softmax_b200 as eta  # noqa: E402
from exact_tiled_attention_softmax_b200 import workloads as W  # noqa: E402
import oracle  # noqa: E402
from oracle import sampled as S  # noqa: E402
from tests.parity_util import BF16_GRAD_REL, BF16_O_ABS, o_excess, rel_fro  # noqa: E402


@pytest.fixture(scope="module", autouse=True)
def _cuda():
    if not torch.cuda.is_available():
        pytest.skip("no GPU")
    eta.load_library()


def _dev(x, dt=torch.bfloat16):
    return torch.from_numpy(np.ascontiguousarray(x)).cuda().to(dt)


def _np(t):
    return t.float().cpu().numpy().astype(np.float64)


def _run_dense(case):
    q, k, v, g = W.dense_inputs(case)
    bm = W.block_mask(case)
    allowed = eta.AllowedSet(causal=case.causal, window_left=case.window_left,
                             block_mask=_dev(bm, torch.uint8) if bm is not None else None,
                             block_q=case.block_size or 128, block_k=case.block_size or 128,
                             dropout_p=case.dropout_p, dropout_seed=case.dropout_seed)
    tq, tk, tv, tg = (_dev(x) for x in (q, k, v, g))
    o, lse = eta.attn_fwd(tq, tk, tv, allowed, case.scale)
    dq, dk, dv, _ = eta.attn_bwd(tq, tk, tv, o, tg, lse, allowed, case.scale)
    torch.cuda.synchronize()
    return (q, k, v, g, bm), (o, lse, dq, dk, dv), (tq, tk, tv, tg)


def _identities(tensors, outs):
    tq, tk, tv, tg = tensors
    o, lse, dq, dk, dv = outs
    f = lambda a, b: float((a.double() * b.double()).sum())
    mag = lambda a, b: float((a.double().abs() * b.double().abs()).sum())
    lhs, rhs = f(tq, dq), f(tk, dk)
    assert abs(lhs - rhs) <= 1e-2 * (mag(tq, dq) + mag(tk, dk)), (lhs, rhs)
    lhs, rhs = f(tv, dv), f(tg, o)
    assert abs(lhs - rhs) <= 1e-2 * (mag(tv, dv) + mag(tg, o)), (lhs, rhs)


def test_causal_2k_all_heads():
    case = W.WORKLOADS["causal_2k"]
    (q, k, v, g, _), outs, tensors = _run_dense(case)
    o, lse, dq, dk, dv = outs
    allow = oracle.allowed_dense(case.T, case.T, causal=True)
    fw = oracle.forward(q, k, v, allow, case.scale)
    bw = oracle.backward(q, k, v, g, allow, case.scale, y=fw.y)
    assert np.abs(_np(o) - fw.y).max() <= BF16_O_ABS
    assert np.abs(_np(lse) - fw.lse).max() <= 1e-3
    for name, got, want in (("dQ", dq, bw.dq), ("dK", dk, bw.dk), ("dV", dv, bw.dv)):
        assert rel_fro(_np(got), want) <= BF16_GRAD_REL, name
    _identities(tensors, outs)


def _head_full(q, k, v, g, b, h, kvh, case, bm, chunk=1024):
    """Every output of one (b, h) whose K/V head is not shared: row passes in
    chunks, then every key column from the oracle's own LSE and delta."""
    T = case.T
    kw = dict(causal=case.causal, window_left=case.window_left, block_mask=bm,
              block_q=case.block_size or 1, block_k=case.block_size or 1)
    y = np.zeros((T, case.dv))
    lse = np.zeros(T)
    delta = np.zeros(T)
    dq = np.zeros((T, case.d))
    cols = np.arange(T)
    for r0 in range(0, T, chunk):
        rows = np.arange(r0, min(r0 + chunk, T))
        ar = S.allowed_at(rows, cols, **kw)
        y[rows], lse[rows], delta[rows], dq[rows] = S.rows_forward_backward(
            q[b, h], k[b, kvh], v[b, kvh], g[b, h], rows, ar, case.scale)
    dk = np.zeros((T, case.d))
    dv = np.zeros((T, case.dv))
    for c0 in range(0, T, chunk):
        cc = np.arange(c0, min(c0 + chunk, T))
        dk[cc], dv[cc] = S.cols_backward([q[b, h]], [g[b, h]], k[b, kvh], v[b, kvh], cc,
                                         lambda hh, r, c: S.allowed_at(r, c, **kw), [lse], [delta], case.scale)
    return y, lse, dq, dk, dv


def test_window_block_8k_sampled_heads():
    case = W.WORKLOADS["window_block_8k"]
    (q, k, v, g, bm), outs, tensors = _run_dense(case)
    o, lse, dq, dk, dv = outs
    for h in (0, 9, 18, 31):
        y_r, lse_r, dq_r, dk_r, dv_r = _head_full(q, k, v, g, 0, h, h, case, bm)
        assert np.abs(_np(o[0, h]) - y_r).max() <= BF16_O_ABS, h
        assert np.abs(_np(lse[0, h]) - lse_r).max() <= 1e-3, h
        assert rel_fro(_np(dq[0, h]), dq_r) <= BF16_GRAD_REL, h
        assert rel_fro(_np(dk[0, h]), dk_r) <= BF16_GRAD_REL, h
        assert rel_fro(_np(dv[0, h]), dv_r) <= BF16_GRAD_REL, h
    _identities(tensors, outs)


def _dropout_head_rows(q, k, v, g, case, b, h, kvh, chunk=256, threads=16):
    """Y, LSE, delta and dQ of every row of one causal dropout head, from the
    oracle's row evaluator over chunks of rows (each chunk against the keys
    it can see). NumPy releases the GIL in its array kernels, so chunks run
    on a thread pool."""
    from concurrent.futures import ThreadPoolExecutor
    T, rho, seed = case.T, case.dropout_p, case.dropout_seed
    kk = k[b, kvh].astype(np.float64)
    vv = v[b, kvh].astype(np.float64)

    def one(r0):
        r1 = min(r0 + chunk, T)
        rows = np.arange(r0, r1)
        ar = S.allowed_at(rows, np.arange(r1), causal=True)
        kr = S.keep_range(seed, rho, b, h, rows, 0, r1)
        return S.rows_forward_backward(q[b, h], kk[:r1], vv[:r1], g[b, h], rows, ar, case.scale,
                                       keep_rows=kr, rho=rho)

    with ThreadPoolExecutor(threads) as ex:
        parts = list(ex.map(one, range(0, T, chunk)))
    return tuple(np.concatenate([p[i] for p in parts]) for i in range(4))


def test_gqa_dropout_16k_whole_group_and_first_key_tiles():
    """One K/V group (b=0, kv=0: 4 query heads) in full: Y, LSE and dQ of every
    row of every head, and dK/dV on the first two key tiles (keys 0-255, the
    longest accumulation of the key-centric reverse: every one of the
    16384 rows of the 4 heads sees them, with dropout replayed throughout), on
    a middle band across a tile edge (keys 8064-8319) and on the last 256
    keys, from the oracle's own LSE and delta of every row."""
    case = W.WORKLOADS["gqa_dropout_16k"]
    (q, k, v, g, _), outs, tensors = _run_dense(case)
    o, lse, dq, dk, dv = outs
    T, group, rho, seed = case.T, case.Hq // case.Hkv, case.dropout_p, case.dropout_seed
    b, kvh = 0, 0
    heads = [kvh * group + hh for hh in range(group)]
    lse_g, delta_g = [], []
    for h in heads:
        y_r, lse_r, delta_r, dq_r = _dropout_head_rows(q, k, v, g, case, b, h, kvh)
        assert o_excess(_np(o[b, h]), y_r) <= BF16_O_ABS, h
        assert np.abs(_np(lse[b, h]) - lse_r).max() <= 1e-3, h
        assert rel_fro(_np(dq[b, h]), dq_r) <= BF16_GRAD_REL, h
        lse_g.append(lse_r)
        delta_g.append(delta_r)
    for c0, c1 in ((0, 256), (8064, 8320), (T - 256, T)):
        cols = np.arange(c0, c1)
        dk_r, dv_r = S.cols_backward(
            [q[b, h] for h in heads], [g[b, h] for h in heads], k[b, kvh], v[b, kvh], cols,
            lambda hh, r, c: S.allowed_at(r, c, causal=True), lse_g, delta_g, case.scale,
            keep_fn=lambda hh, r, c: S.keep_range(seed, rho, b, heads[hh], r, int(c[0]), int(c[-1]) + 1), rho=rho)
        assert rel_fro(_np(dk[b, kvh])[cols], dk_r) <= BF16_GRAD_REL, (c0, c1)
        assert rel_fro(_np(dv[b, kvh])[cols], dv_r) <= BF16_GRAD_REL, (c0, c1)
    _identities(tensors, outs)
    # A second group on sampled rows and its last 256 keys (whose allowed
    # query rows are the last 256 rows).
    rng = np.random.default_rng(5)
    rows = np.unique(np.concatenate([[0, 1, 127, 128, T - 1], rng.integers(0, T, 123)]))
    tail = np.arange(T - 256, T)
    cols = np.arange(T)
    b, kvh = 1, 7
    heads = [kvh * group + hh for hh in range(group)]
    lse_g, delta_g = [], []
    for h in heads:
        ar = S.allowed_at(rows, cols, causal=True)
        kr = S.keep_range(seed, rho, b, h, rows, 0, T)
        y_r, lse_r, _, dq_r = S.rows_forward_backward(q[b, h], k[b, kvh], v[b, kvh], g[b, h], rows, ar,
                                                      case.scale, keep_rows=kr, rho=rho)
        assert o_excess(_np(o[b, h])[rows], y_r) <= BF16_O_ABS, h
        assert np.abs(_np(lse[b, h])[rows] - lse_r).max() <= 1e-3, h
        assert rel_fro(_np(dq[b, h])[rows], dq_r) <= BF16_GRAD_REL, h
        at = S.allowed_at(tail, cols, causal=True)
        kt = S.keep_range(seed, rho, b, h, tail, 0, T)
        _, l_t, d_t, _ = S.rows_forward_backward(q[b, h], k[b, kvh], v[b, kvh], g[b, h], tail, at, case.scale,
                                                 keep_rows=kt, rho=rho)
        lf = np.full(T, np.nan)
        df = np.full(T, np.nan)
        lf[tail], df[tail] = l_t, d_t
        lse_g.append(lf)
        delta_g.append(df)
    dk_r, dv_r = S.cols_backward(
        [q[b, h] for h in heads], [g[b, h] for h in heads], k[b, kvh], v[b, kvh], tail,
        lambda hh, r, c: S.allowed_at(r, c, causal=True), lse_g, delta_g, case.scale,
        keep_fn=lambda hh, r, c: S.keep_range(seed, rho, b, heads[hh], r, int(c[0]), int(c[-1]) + 1), rho=rho)
    assert rel_fro(_np(dk[b, kvh])[tail], dk_r) <= BF16_GRAD_REL
    assert rel_fro(_np(dv[b, kvh])[tail], dv_r) <= BF16_GRAD_REL


def test_topk_shared_kv_sampled():
    case = W.TOPK_WORKLOADS["topk_shared_kv"]
    q, kv, g, idx, ln, sink = W.topk_inputs(case)
    Dv = case.Dv
    tq, tkv, tg = _dev(q), _dev(kv), _dev(g)
    allowed = eta.AllowedSet(topk_idxs=_dev(idx, torch.int32), topk_length=_dev(ln, torch.int32),
                             sink=_dev(sink, torch.float32))
    o, lse = eta.attn_fwd(tq, tkv, tkv[:, :Dv], allowed, case.scale)
    dq, dkv, _, ds = eta.attn_bwd(tq, tkv, tkv[:, :Dv], o, tg, lse, allowed, case.scale)
    torch.cuda.synchronize()
    sink64 = sink.astype(np.float64)
    rng = np.random.default_rng(6)
    tok = np.unique(np.concatenate([[0, case.Tq - 1], rng.integers(0, case.Tq, 254)]))
    o_r, lse_r, _ = oracle.topk_forward(q[tok], kv, idx[tok], ln[tok], Dv, case.scale, sink64)
    dq_r, _, _ = oracle.topk_backward(q[tok], kv, idx[tok], ln[tok], Dv, case.scale, g[tok], sink64, o=o_r)
    assert np.abs(_np(o)[tok] - o_r).max() <= BF16_O_ABS
    assert np.abs(_np(lse)[tok] - lse_r).max() <= 1e-3
    assert rel_fro(_np(dq)[tok], dq_r) <= BF16_GRAD_REL
    # The deterministic reverse (fixed-point dKV in two column passes) on the
    # same inputs.
    al_det = eta.AllowedSet(topk_idxs=_dev(idx, torch.int32), topk_length=_dev(ln, torch.int32),
                            sink=_dev(sink, torch.float32), deterministic=True)
    dq_d, dkv_d, _, _ = eta.attn_bwd(tq, tkv, tkv[:, :Dv], o, tg, lse, al_det, case.scale)
    torch.cuda.synchronize()
    assert torch.equal(dq_d, dq)  # dQ is summed by one CTA per token in both modes
    # KV rows >= Tkv - 256 can only be listed by the last 256 tokens.
    last = np.arange(case.Tq - 256, case.Tq)
    _, dkv_r, _ = oracle.topk_backward(q[last], kv, idx[last], ln[last], Dv, case.scale, g[last], sink64)
    rows = np.arange(case.Tkv - 256, case.Tkv)
    assert rel_fro(_np(dkv)[rows], dkv_r[rows]) <= BF16_GRAD_REL
    assert rel_fro(_np(dkv_d)[rows], dkv_r[rows]) <= BF16_GRAD_REL
    # Rows listed by about 200 tokens each (the longest sums, spread over
    # both column passes of the fixed-point form): every token that lists
    # one of them enters the oracle, so these rows of its dKV are exact.
    rows2 = np.array([0, 1, 12345, 28000])
    lists = np.array([np.isin(idx[t, :ln[t]], rows2).any() for t in range(case.Tq)])
    tk = np.nonzero(lists)[0]
    _, dkv_r2, _ = oracle.topk_backward(q[tk], kv, idx[tk], ln[tk], Dv, case.scale, g[tk], sink64)
    assert rel_fro(_np(dkv)[rows2], dkv_r2[rows2]) <= BF16_GRAD_REL
    assert rel_fro(_np(dkv_d)[rows2], dkv_r2[rows2]) <= BF16_GRAD_REL
    # dSink needs every token.
    ds_r = oracle.topk_dsink(q, kv, idx, ln, Dv, case.scale, g, sink64)
    assert np.abs(ds.cpu().numpy() - ds_r).max() <= 2e-2 * max(1.0, np.abs(ds_r).max())
    # Tied identity over every output.
    f = lambda a, b: float((a.double() * b.double()).sum())
    lhs, rhs = f(tkv, dkv), f(tq, dq) + f(tg, o)
    mag = float((tkv.double().abs() * dkv.double().abs()).sum())
    assert abs(lhs - rhs) <= 1e-2 * mag + 1e-6, (lhs, rhs)

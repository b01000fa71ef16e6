"""GPU parity: the CUDA library against the float64 oracle, element by element,
on seeded inputs that span several kernel tiles and a ragged tail, plus the
pages' worked examples run through the C ABI."""
import json
import math
import os

import numpy as np
import pytest

torch = pytest.importorskip("torch")

pytestmark = pytest.mark.gpu

import exact_tiled_attention_softmax_b200 as eta  # noqa: E402
from exact_tiled_attention_softmax_b200 import workloads as W  # noqa: E402
import oracle  # noqa: E402
from oracle import philox as P  # noqa: E402
from tests.parity_util import check_close, to_dev, to_np  # noqa: E402

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")
TORCH_DTYPE = {"bf16": torch.bfloat16, "f16": torch.float16, "f32": torch.float32}


@pytest.fixture(scope="module", autouse=True)
def _cuda():
    if not torch.cuda.is_available():
        pytest.skip("no GPU")
    eta.load_library()


def _dense_case(B, Hq, Hkv, T, d, dv, dtype, seed, *, causal=True, window=0, block=0, p_keep=0.5,
                dropout=0.0, sink=False, scale=None):
    rng = np.random.default_rng(seed)
    f = lambda s: W.round_to_storage(rng.standard_normal(s, dtype=np.float32), dtype)  # noqa: E731
    q, k, v, g = f((B, Hq, T, d)), f((B, Hkv, T, d)), f((B, Hkv, T, dv)), f((B, Hq, T, dv))
    bm = None
    if block:
        nb = (T + block - 1) // block
        bm = (rng.random((B, Hq, nb, nb)) < p_keep).astype(np.uint8)
        for i in range(nb):
            bm[:, :, i, i] = 1
    sk = rng.standard_normal(Hq).astype(np.float32) if sink else None
    scale = scale if scale is not None else 1 / math.sqrt(d)
    return dict(q=q, k=k, v=v, g=g, bm=bm, sink=sk, scale=scale, causal=causal, window=window,
                block=block, dropout=dropout, seed=seed, dtype=dtype)


def _run_gpu(c):
    tdt = TORCH_DTYPE[c["dtype"]]
    q, k, v, g = (to_dev(c[n], tdt) for n in ("q", "k", "v", "g"))
    allowed = eta.AllowedSet(
        causal=c["causal"], window_left=c["window"],
        block_mask=to_dev(c["bm"], torch.uint8) if c["bm"] is not None else None,
        block_q=c["block"] or 128, block_k=c["block"] or 128,
        sink=to_dev(c["sink"], torch.float32) if c["sink"] is not None else None,
        dropout_p=c["dropout"], dropout_seed=c["seed"])
    wf = torch.empty(eta.attn_fwd_workspace_size(q, k, v, allowed), dtype=torch.uint8, device="cuda")
    wb = torch.empty(eta.attn_bwd_workspace_size(q, k, v, allowed), dtype=torch.uint8, device="cuda")
    o, lse = eta.attn_fwd(q, k, v, allowed, c["scale"], workspace=wf)
    assert eta.attn_get_status(wf) == 0, "device status after attn_fwd"
    dq, dk, dv, dsink = eta.attn_bwd(q, k, v, o, g, lse, allowed, c["scale"], workspace=wb)
    assert eta.attn_get_status(wb) == 0, "device status after attn_bwd"
    torch.cuda.synchronize()
    return dict(o=o, lse=lse, dq=dq, dk=dk, dv=dv, dsink=dsink, inputs=(q, k, v, g), allowed=allowed)


def _run_oracle(c):
    B, Hq, T = c["q"].shape[:3]
    allow = oracle.allowed_dense(T, T, causal=c["causal"], window_left=c["window"],
                                 block_mask=c["bm"], block_q=c["block"] or 1, block_k=c["block"] or 1)
    keep = P.dropout_keep(c["seed"], c["dropout"], B, Hq, T, T) if c["dropout"] else None
    q, k, v, g = (c[n].astype(np.float64) for n in ("q", "k", "v", "g"))
    sink = c["sink"].astype(np.float64) if c["sink"] is not None else None
    fw = oracle.forward(q, k, v, allow, c["scale"], sink=sink, keep=keep, rho=c["dropout"])
    bw = oracle.backward(q, k, v, g, allow, c["scale"], sink=sink, keep=keep, rho=c["dropout"], y=fw.y)
    return fw, bw


def _compare(c, gpu, fw, bw):
    fp32 = c["dtype"] == "f32"
    check_close("O", to_np(gpu["o"]), fw.y, fp32=fp32, grad=False, storage=c["dtype"])
    lse_g, lse_o = to_np(gpu["lse"]), fw.lse
    fin = np.isfinite(lse_o)
    assert np.array_equal(np.isfinite(lse_g), fin)
    assert np.abs(lse_g[fin] - lse_o[fin]).max(initial=0) <= (1e-5 if fp32 else 1e-3)
    check_close("dQ", to_np(gpu["dq"]), bw.dq, fp32=fp32, grad=True)
    check_close("dK", to_np(gpu["dk"]), bw.dk, fp32=fp32, grad=True)
    check_close("dV", to_np(gpu["dv"]), bw.dv, fp32=fp32, grad=True)
    if bw.dsink is not None:
        err = np.abs(to_np(gpu["dsink"]) - bw.dsink).max()
        assert err <= (1e-5 if fp32 else 2e-2 * max(1.0, np.abs(bw.dsink).max())), err


def test_tiny_causal_fp32_full():
    """B=1 H=1 T=64 d=dv=16 fp32, c=1/4, causal: every element <= 1e-5."""
    case = W.WORKLOADS["tiny_causal_fp32"]
    q, k, v, g = W.dense_inputs(case)
    c = dict(q=q, k=k, v=v, g=g, bm=None, sink=None, scale=case.scale, causal=True, window=0, block=0,
             dropout=0.0, seed=case.seed, dtype="f32")
    gpu = _run_gpu(c)
    fw, bw = _run_oracle(c)
    _compare(c, gpu, fw, bw)


@pytest.mark.parametrize("kind", ["causal", "window_block", "gqa_dropout", "sink", "noncausal_mqa"])
@pytest.mark.parametrize("dtype", ["bf16", "f32", "f16"])
def test_small_dense_cases(kind, dtype):
    """Multi-tile shapes with a ragged tail (T=300) for every allowed-set kind."""
    if kind == "causal":
        c = _dense_case(2, 4, 4, 300, 128, 128, dtype, 11)
    elif kind == "window_block":
        c = _dense_case(1, 3, 3, 300, 128, 128, dtype, 12, window=100, block=64)
    elif kind == "gqa_dropout":
        c = _dense_case(2, 4, 2, 300, 128, 128, dtype, 13, dropout=0.1)
    elif kind == "sink":
        c = _dense_case(1, 4, 2, 300, 128, 128, dtype, 14, sink=True)
    else:
        c = _dense_case(1, 4, 1, 200, 64, 96, dtype, 15, causal=False)
    gpu = _run_gpu(c)
    fw, bw = _run_oracle(c)
    _compare(c, gpu, fw, bw)


def test_backward_is_deterministic():
    c = _dense_case(1, 4, 2, 300, 128, 128, "bf16", 21, dropout=0.1, sink=True)
    a = _run_gpu(c)
    q, k, v, g = a["inputs"]
    for _ in range(2):
        dq, dk, dv, ds = eta.attn_bwd(q, k, v, a["o"], g, a["lse"], a["allowed"], c["scale"])
        torch.cuda.synchronize()
        assert torch.equal(dk, a["dk"]) and torch.equal(dv, a["dv"]) and torch.equal(ds, a["dsink"])


def _golden(name):
    with open(os.path.join(GOLDEN, name)) as f:
        return json.load(f)


def _f32(x):
    return torch.tensor(np.asarray(x, np.float32)).cuda()


def test_worked_examples_on_gpu():
    ex = _golden("worked_examples.json")
    # One key: Y=[7], dQ=dK=0, dV=[4].
    e = ex["one_key"]
    q, k, v, g = (_f32(e[n])[None, None] for n in ("q", "k", "v", "g"))
    o, lse = eta.attn_fwd(q, k, v, None, 1.0)
    dq, dk, dv, _ = eta.attn_bwd(q, k, v, o, g, lse, None, 1.0)
    assert abs(o.item() - 7) <= 1e-6 and abs(dq.item()) <= 1e-6 and abs(dk.item()) <= 1e-6
    assert abs(dv.item() - 4) <= 1e-6
    # Empty first block for row 1: A_1={2}, A_2={1,2} as a block mask of size 1.
    e = ex["empty_first_block"]
    q, k, v = (_f32(e[n])[None, None] for n in ("q", "k", "v"))
    bm = torch.tensor(e["allowed"], dtype=torch.uint8).cuda()
    al = eta.AllowedSet(block_mask=bm, block_q=1, block_k=1)
    o, _ = eta.attn_fwd(q, k, v, al, 1.0)
    assert torch.allclose(o.flatten().cpu(), torch.tensor([5.0, 4.0]), atol=1e-6)
    # Merge orders: permuting keys (a different tile order) leaves Y = 2.
    e = ex["merge_orders"]
    q, k, v = (_f32(e[n])[None, None] for n in ("q", "k", "v"))
    o1, _ = eta.attn_fwd(q, k, v, None, 1.0)
    o2, _ = eta.attn_fwd(q, k.flip(2), v.flip(2), None, 1.0)
    assert torch.allclose(o1.flatten().cpu(), torch.tensor([2.0, 2.0]), atol=1e-6)
    assert torch.allclose(o1, o2, atol=1e-6)
    # Two-tile trace: the traced row's output.
    gd = _golden("two_tile_trace.json")
    inp = gd["inputs"]
    q, k, v = (_f32(inp[n])[None, None] for n in ("q", "k", "v"))
    o, _ = eta.attn_fwd(q, k, v, eta.AllowedSet(causal=True), 1.0)
    assert np.allclose(o[0, 0, 3].cpu().numpy(), gd["tiled_output_row3"], rtol=1e-6)
    # Sink: o = 0.7, dS = (0.65, -0.51), dz = -0.14 (dense realisation).
    e = ex["sink"]
    # The dense layout has as many query rows as keys: a second query row with
    # zero upstream gradient contributes nothing to any gradient.
    q = _f32([[1.0], [0.3]])[None, None]
    k = _f32([[math.log(e["p"][0])], [math.log(e["p"][1])]])[None, None]
    v = _f32([[e["v"][0]], [e["v"][1]]])[None, None]
    g = _f32([[e["g"]], [0.0]])[None, None]
    al = eta.AllowedSet(sink=_f32([math.log(e["p_sink"])]))
    o, lse = eta.attn_fwd(q, k, v, al, 1.0)
    dq, dk, dv, ds = eta.attn_bwd(q, k, v, o, g, lse, al, 1.0)
    assert abs(o[0, 0, 0, 0].item() - e["o"]) <= 1e-6
    assert abs(lse[0, 0, 0].item()) <= 1e-6
    assert np.allclose(dk.flatten().cpu().numpy(), e["dS"], atol=1e-6)
    assert np.allclose(dv.flatten().cpu().numpy(), e["p"], atol=1e-6)
    assert abs(ds.item() - e["dz"]) <= 1e-6


def test_dropout_replay_example_on_gpu():
    """The replay example through the in-kernel generator: a seed whose
    realisation for query row 0 is xi = (1, 0) gives Y_1 = 2 and dV = (1, 0)."""
    e = _golden("worked_examples.json")["dropout_replay"]
    seed = next(s for s in range(1, 1000)
                if P.dropout_keep(s, 0.5, 1, 1, 2, 2)[0, 0, 0].tolist() == [True, False])
    q, k, v, g = (_f32(e[n])[None, None] for n in ("q", "k", "v", "g"))
    al = eta.AllowedSet(dropout_p=0.5, dropout_seed=seed)
    o, lse = eta.attn_fwd(q, k, v, al, 1.0)
    dq, dk, dv, _ = eta.attn_bwd(q, k, v, o, g, lse, al, 1.0)
    assert abs(o[0, 0, 0, 0].item() - 2.0) <= 1e-6
    assert np.allclose(dv.flatten().cpu().numpy(), np.ravel(e["dv"]), atol=1e-6)


def _topk_small(dtype, seed, Tq=40, Tkv=300, H=8, Dqk=96, Dv=64, topk=128, lo=20, hi=128, sink=True):
    rng = np.random.default_rng(seed)
    f = lambda s: W.round_to_storage(rng.standard_normal(s, dtype=np.float32), dtype)  # noqa: E731
    q, kv, g = f((Tq, H, Dqk)), f((Tkv, Dqk)), f((Tq, H, Dv))
    idx, ln = W.topk_lists(Tq, Tkv, topk, lo, hi, seed + 1)
    sk = rng.standard_normal(H).astype(np.float32) if sink else None
    return q, kv, g, idx, ln, sk


@pytest.mark.parametrize("dtype", ["bf16", "f32", "f16"])
def test_small_topk(dtype):
    q, kv, g, idx, ln, sk = _topk_small(dtype, 31)
    Dv = g.shape[-1]
    scale = 1 / math.sqrt(q.shape[-1])
    tdt = TORCH_DTYPE[dtype]
    qd, kvd, gd = to_dev(q, tdt), to_dev(kv, tdt), to_dev(g, tdt)
    al = eta.AllowedSet(topk_idxs=to_dev(idx, torch.int32), topk_length=to_dev(ln, torch.int32),
                        sink=to_dev(sk, torch.float32))
    o, lse = eta.attn_fwd(qd, kvd, kvd[:, :Dv], al, scale)
    dq, dkv, _, ds = eta.attn_bwd(qd, kvd, kvd[:, :Dv], o, gd, lse, al, scale)
    torch.cuda.synchronize()
    o_ref, lse_ref, _ = oracle.topk_forward(q, kv, idx, ln, Dv, scale, sk.astype(np.float64))
    dq_ref, dkv_ref, ds_ref = oracle.topk_backward(q, kv, idx, ln, Dv, scale, g, sk.astype(np.float64),
                                                   o=o_ref)
    fp32 = dtype == "f32"
    check_close("O", to_np(o), o_ref, fp32=fp32, grad=False, storage=dtype)
    check_close("dQ", to_np(dq), dq_ref, fp32=fp32, grad=True)
    check_close("dKV", to_np(dkv), dkv_ref, fp32=fp32, grad=True)
    assert np.abs(to_np(lse) - lse_ref).max() <= (1e-5 if fp32 else 1e-3)
    assert np.abs(to_np(ds) - ds_ref).max() <= (1e-5 if fp32 else 2e-2)
    # dKV and dSink are bitwise reproducible.
    dq2, dkv2, _, ds2 = eta.attn_bwd(qd, kvd, kvd[:, :Dv], o, gd, lse, al, scale)
    torch.cuda.synchronize()
    assert torch.equal(dkv2, dkv) and torch.equal(ds2, ds)


def test_topk_bad_index_sets_status_and_returns():
    q, kv, g, idx, ln, sk = _topk_small("bf16", 41, Tq=8, Tkv=64, H=4, Dqk=64, Dv=32, topk=16, lo=4, hi=16)
    idx[3, 0] = 10_000  # out of range, inside the valid length
    qd, kvd = to_dev(q, torch.bfloat16), to_dev(kv, torch.bfloat16)
    al = eta.AllowedSet(topk_idxs=to_dev(idx, torch.int32), topk_length=to_dev(ln, torch.int32))
    ws = torch.empty(eta.attn_fwd_workspace_size(qd, kvd, kvd[:, :32], al), dtype=torch.uint8, device="cuda")
    eta.attn_fwd(qd, kvd, kvd[:, :32], al, 0.125, workspace=ws)
    assert eta.attn_get_status(ws) & eta.ATTN_DEVERR_TOPK_INDEX
    assert eta.attn_get_status(ws) == 0  # read clears


def _qk_case(B, Hq, Hkv, Tq, Tk, d, dv, dtype, seed, *, causal=True, window=0, block=0, dropout=0.0, sink=False):
    rng = np.random.default_rng(seed)
    f = lambda s: W.round_to_storage(rng.standard_normal(s, dtype=np.float32), dtype)  # noqa: E731
    q, g = f((B, Hq, Tq, d)), f((B, Hq, Tq, dv))
    k, v = f((B, Hkv, Tk, d)), f((B, Hkv, Tk, dv))
    bm = None
    if block:
        bm = (rng.random((B, Hq, (Tq + block - 1) // block, (Tk + block - 1) // block)) < 0.6).astype(np.uint8)
    sk = rng.standard_normal(Hq).astype(np.float32) if sink else None
    return dict(q=q, k=k, v=v, g=g, bm=bm, sink=sk, scale=1 / math.sqrt(d), causal=causal, window=window,
                block=block, dropout=dropout, seed=seed, dtype=dtype)


@pytest.mark.parametrize("kind", ["causal_short_q", "causal_long_q", "window_block", "gqa_dropout_sink"])
@pytest.mark.parametrize("dtype", ["bf16", "f32"])
def test_query_block_against_longer_or_shorter_keys(kind, dtype):
    """Tq != Tk with bottom-right alignment: query row i sits at key position
    i + Tk - Tq (rows with no key position left get the empty-set result)."""
    if kind == "causal_short_q":
        c = _qk_case(2, 4, 2, 200, 330, 128, 128, dtype, 21)
    elif kind == "causal_long_q":
        c = _qk_case(1, 4, 4, 300, 130, 128, 128, dtype, 22)
    elif kind == "window_block":
        c = _qk_case(1, 3, 3, 130, 400, 128, 128, dtype, 23, window=100, block=64)
    else:
        c = _qk_case(2, 4, 2, 150, 290, 128, 128, dtype, 24, dropout=0.1, sink=True)
    gpu = _run_gpu(c)
    B, Hq, Tq = c["q"].shape[:3]
    Tk = c["k"].shape[2]
    allow = oracle.allowed_dense(Tq, Tk, causal=c["causal"], window_left=c["window"], block_mask=c["bm"],
                                 block_q=c["block"] or 1, block_k=c["block"] or 1, query_offset=Tk - Tq)
    keep = P.dropout_keep(c["seed"], c["dropout"], B, Hq, Tq, Tk) if c["dropout"] else None
    q, k, v, g = (c[n].astype(np.float64) for n in ("q", "k", "v", "g"))
    sink = c["sink"].astype(np.float64) if c["sink"] is not None else None
    fw = oracle.forward(q, k, v, allow, c["scale"], sink=sink, keep=keep, rho=c["dropout"])
    bw = oracle.backward(q, k, v, g, allow, c["scale"], sink=sink, keep=keep, rho=c["dropout"], y=fw.y)
    _compare(c, gpu, fw, bw)


def _segment_starts(bounds_per_batch, T):
    st = np.zeros((len(bounds_per_batch), T), dtype=np.int32)
    for b, bd in enumerate(bounds_per_batch):
        for s0, s1 in zip(bd[:-1], bd[1:]):
            st[b, s0:s1] = s0
    return st


def _run_layout_case(c, lengths=None, starts=None):
    tdt = TORCH_DTYPE[c["dtype"]]
    q, k, v, g = (to_dev(c[n], tdt) for n in ("q", "k", "v", "g"))
    allowed = eta.AllowedSet(
        causal=c["causal"], window_left=c["window"],
        block_mask=to_dev(c["bm"], torch.uint8) if c["bm"] is not None else None,
        block_q=c["block"] or 128, block_k=c["block"] or 128,
        sink=to_dev(c["sink"], torch.float32) if c["sink"] is not None else None,
        dropout_p=c["dropout"], dropout_seed=c["seed"],
        lengths=to_dev(lengths, torch.int32) if lengths is not None else None,
        starts=to_dev(starts, torch.int32) if starts is not None else None)
    wf = torch.empty(eta.attn_fwd_workspace_size(q, k, v, allowed), dtype=torch.uint8, device="cuda")
    wb = torch.empty(eta.attn_bwd_workspace_size(q, k, v, allowed), dtype=torch.uint8, device="cuda")
    o, lse = eta.attn_fwd(q, k, v, allowed, c["scale"], workspace=wf)
    assert eta.attn_get_status(wf) == 0
    dq, dk, dv, dsink = eta.attn_bwd(q, k, v, o, g, lse, allowed, c["scale"], workspace=wb)
    assert eta.attn_get_status(wb) == 0
    torch.cuda.synchronize()
    gpu = dict(o=o, lse=lse, dq=dq, dk=dk, dv=dv, dsink=dsink)
    B, Hq, Tq = c["q"].shape[:3]
    Tk = c["k"].shape[2]
    allow = oracle.allowed_dense(Tq, Tk, causal=c["causal"], window_left=c["window"], block_mask=c["bm"],
                                 block_q=c["block"] or 1, block_k=c["block"] or 1, query_offset=Tk - Tq,
                                 lengths=lengths, starts=starts)
    keep = P.dropout_keep(c["seed"], c["dropout"], B, Hq, Tq, Tk) if c["dropout"] else None
    qq, kk, vv, gg = (c[n].astype(np.float64) for n in ("q", "k", "v", "g"))
    sink = c["sink"].astype(np.float64) if c["sink"] is not None else None
    fw = oracle.forward(qq, kk, vv, allow, c["scale"], sink=sink, keep=keep, rho=c["dropout"])
    bw = oracle.backward(qq, kk, vv, gg, allow, c["scale"], sink=sink, keep=keep, rho=c["dropout"], y=fw.y)
    _compare(c, gpu, fw, bw)
    return gpu


@pytest.mark.parametrize("dtype", ["bf16", "f32"])
def test_packed_segments(dtype):
    """Causal attention inside packed segments (starts = the segment's first
    cell), with GQA and a sink; boundaries fall inside and on tile edges."""
    T = 600
    c = _qk_case(2, 4, 2, T, T, 128, 128, dtype, 31, sink=True)
    st = _segment_starts([[0, 70, 200, 256, 431, 600], [0, 128, 600]], T)
    _run_layout_case(c, starts=st)


@pytest.mark.parametrize("causal", [True, False])
@pytest.mark.parametrize("dtype", ["bf16", "f32"])
def test_active_lengths(dtype, causal):
    """Active lengths per batch row (a full row, one ending inside a 64-row
    slice and a 128-key tile, one empty) with dropout: padding rows are
    empty, padding keys take no part."""
    T = 300
    c = _qk_case(3, 4, 2, T, T, 128, 128, dtype, 32, causal=causal, dropout=0.1)
    gpu = _run_layout_case(c, lengths=np.array([300, 131, 0], dtype=np.int32))
    o = to_np(gpu["o"])
    assert np.all(o[1, :, 131:] == 0) and np.all(o[2] == 0)
    assert np.all(to_np(gpu["dk"])[1, :, 131:] == 0) and np.all(to_np(gpu["dv"])[2] == 0)


@pytest.mark.parametrize("dtype", ["bf16", "f32"])
def test_starts_with_window_block_and_longer_keys(dtype):
    """Per-row lower bounds of arbitrary shape (not segments) together with a
    window, a block mask and Tq < Tk."""
    Tq, Tk = 200, 420
    c = _qk_case(2, 2, 2, Tq, Tk, 128, 128, dtype, 33, window=300, block=64)
    rng = np.random.default_rng(34)
    pos = np.arange(Tq) + Tk - Tq
    st = (pos[None, :] - rng.integers(0, 260, size=(2, Tq))).clip(0).astype(np.int32)
    _run_layout_case(c, starts=st)


def test_lengths_need_equal_query_and_key_counts():
    q = torch.zeros(1, 1, 8, 128, dtype=torch.bfloat16, device="cuda")
    k = torch.zeros(1, 1, 16, 128, dtype=torch.bfloat16, device="cuda")
    al = eta.AllowedSet(causal=True, lengths=torch.tensor([8], dtype=torch.int32, device="cuda"))
    with pytest.raises(eta.AttnError):
        eta.attn_fwd(q, k, k, al)

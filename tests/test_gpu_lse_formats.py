"""GPU parity of the LSE formats ("DeepSeek Sparse Attention Forward and
Backward", section 7): the forward writes the sink-inclusive or the KV-only
LSE, in natural log or as -log2 Z; the reverse pass, handed the same format,
must give the same gradients as with the default one. Dense tensor-core and
fp32 row paths, and the top-k tensor-core and row paths."""
import math

import numpy as np
import pytest

torch = pytest.importorskip("torch")

pytestmark = pytest.mark.gpu

import exact_tiled_attention_softmax_b200 as eta  # noqa: E402
from exact_tiled_attention_softmax_b200 import workloads as W  # noqa: E402
import oracle  # noqa: E402
from tests.parity_util import BF16_GRAD_REL, check_close, rel_fro, to_dev, to_np  # noqa: E402

FORMATS = [(False, False), (True, False), (False, True), (True, True)]


@pytest.fixture(scope="module", autouse=True)
def _cuda():
    if not torch.cuda.is_available():
        pytest.skip("no GPU")
    eta.load_library()


def _expected_lse(lse_total, lse_kv, kv_only, neg_log2):
    v = lse_kv if kv_only else lse_total
    return oracle.scaled_lse(v) if neg_log2 else v


def _check_lse(got, want, fp32):
    fin = np.isfinite(want)
    assert np.array_equal(np.isfinite(got), fin)
    assert np.array_equal(np.sign(got[~fin]), np.sign(want[~fin]))
    # bf16 inputs: the scores carry the bf16 rounding of Q and K only, the
    # LSE itself is fp32; 1e-3 absolute covers both natural and base-2 forms.
    assert np.abs(got[fin] - want[fin]).max(initial=0) <= (1e-5 if fp32 else 1e-3)


@pytest.mark.parametrize("kv_only,neg_log2", FORMATS)
@pytest.mark.parametrize("dtype", ["bf16", "f32"])
def test_dense_lse_formats(dtype, kv_only, neg_log2):
    rng = np.random.default_rng(41)
    B, Hq, Hkv, T, d = 2, 4, 2, 300, 128
    f = (lambda s: W.round_to_bf16(rng.standard_normal(s, dtype=np.float32))) if dtype == "bf16" else \
        (lambda s: rng.standard_normal(s, dtype=np.float32))
    q, k, v, g = f((B, Hq, T, d)), f((B, Hkv, T, d)), f((B, Hkv, T, d)), f((B, Hq, T, d))
    sink = (rng.standard_normal(Hq) * 2).astype(np.float32)
    lengths = np.array([300, 200], dtype=np.int32)    # padding rows: empty allowed sets
    scale = 1 / math.sqrt(d)
    tdt = torch.bfloat16 if dtype == "bf16" else torch.float32
    qd, kd, vd, gd = (to_dev(x, tdt) for x in (q, k, v, g))
    al = eta.AllowedSet(causal=True, sink=to_dev(sink, torch.float32), lengths=to_dev(lengths, torch.int32),
                        lse_kv_only=kv_only, lse_neg_log2=neg_log2)
    o, lse = eta.attn_fwd(qd, kd, vd, al, scale)
    dq, dk, dv, ds = eta.attn_bwd(qd, kd, vd, o, gd, lse, al, scale)
    torch.cuda.synchronize()
    allow = oracle.allowed_dense(T, T, causal=True, lengths=lengths)
    q64, k64, v64, g64 = (x.astype(np.float64) for x in (q, k, v, g))
    fw = oracle.forward(q64, k64, v64, allow, scale, sink=sink.astype(np.float64))
    bw = oracle.backward(q64, k64, v64, g64, allow, scale, sink=sink.astype(np.float64), y=fw.y)
    lkv = oracle.kv_only_lse(q64, k64, allow, scale)
    fp32 = dtype == "f32"
    _check_lse(to_np(lse), _expected_lse(fw.lse, lkv, kv_only, neg_log2), fp32)
    check_close("O", to_np(o), fw.y, fp32=fp32, grad=False)
    check_close("dQ", to_np(dq), bw.dq, fp32=fp32, grad=True)
    check_close("dK", to_np(dk), bw.dk, fp32=fp32, grad=True)
    check_close("dV", to_np(dv), bw.dv, fp32=fp32, grad=True)
    err = np.abs(to_np(ds) - bw.dsink).max()
    assert err <= (1e-5 if fp32 else 2e-2 * max(1.0, np.abs(bw.dsink).max())), err


def _topk_case(seed, Tq, Tkv, H, Dqk, topk, lo, hi, dtype):
    rng = np.random.default_rng(seed)
    f = (lambda s: W.round_to_bf16(rng.standard_normal(s, dtype=np.float32))) if dtype == "bf16" else \
        (lambda s: rng.standard_normal(s, dtype=np.float32))
    q, kv = f((Tq, H, Dqk)), f((Tkv, Dqk))
    idx, ln = W.topk_lists(Tq, Tkv, topk, lo, hi, seed + 1)
    ln[3] = 0
    sink = (rng.standard_normal(H) * 2).astype(np.float32)
    return q, kv, idx, ln, sink


@pytest.mark.parametrize("kv_only,neg_log2", FORMATS)
@pytest.mark.parametrize("path", ["tensor_core", "rows_f32"])
def test_topk_lse_formats(path, kv_only, neg_log2):
    if path == "tensor_core":
        H, Dqk, Dv, dtype = 64, 576, 512, "bf16"
        q, kv, idx, ln, sink = _topk_case(51, 16, 600, H, Dqk, 256, 1, 256, dtype)
    else:
        H, Dqk, Dv, dtype = 4, 96, 64, "f32"
        q, kv, idx, ln, sink = _topk_case(52, 20, 300, H, Dqk, 64, 1, 64, dtype)
    rng = np.random.default_rng(53)
    g = rng.standard_normal((q.shape[0], H, Dv), dtype=np.float32)
    if dtype == "bf16":
        g = W.round_to_bf16(g)
    scale = 1 / math.sqrt(Dqk)
    tdt = torch.bfloat16 if dtype == "bf16" else torch.float32
    qd, kvd, gd = to_dev(q, tdt), to_dev(kv, tdt), to_dev(g, tdt)
    al = eta.AllowedSet(topk_idxs=to_dev(idx, torch.int32), topk_length=to_dev(ln, torch.int32),
                        sink=to_dev(sink, torch.float32), lse_kv_only=kv_only, lse_neg_log2=neg_log2)
    o, lse = eta.attn_fwd(qd, kvd, kvd[:, :Dv], al, scale)
    dq, dkv, _, ds = eta.attn_bwd(qd, kvd, kvd[:, :Dv], o, gd, lse, al, scale)
    torch.cuda.synchronize()
    s64 = sink.astype(np.float64)
    o_ref, lse_ref, _ = oracle.topk_forward(q, kv, idx, ln, Dv, scale, s64)
    lkv = oracle.topk_kv_only_lse(q, kv, idx, ln, scale)
    fp32 = dtype == "f32"
    _check_lse(to_np(lse), _expected_lse(lse_ref, lkv, kv_only, neg_log2), fp32)
    dq_ref, dkv_ref, ds_ref = oracle.topk_backward(q, kv, idx, ln, Dv, scale, g, s64, o=o_ref)
    if fp32:
        check_close("dQ", to_np(dq), dq_ref, fp32=True, grad=True)
        check_close("dKV", to_np(dkv), dkv_ref, fp32=True, grad=True)
    else:
        assert rel_fro(to_np(dq), dq_ref) <= BF16_GRAD_REL
        assert rel_fro(to_np(dkv), dkv_ref) <= BF16_GRAD_REL
    assert np.abs(to_np(ds) - ds_ref).max() <= (1e-5 if fp32 else 2e-2 * max(1.0, np.abs(ds_ref).max()))


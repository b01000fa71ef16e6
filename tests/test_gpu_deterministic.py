"""The deterministic reverse pass (ATTN_BWD_DETERMINISTIC): dQ from the
query-centric pass matches the float64 oracle on every allowed-set kind, and
repeated calls return bitwise identical dQ, dK, dV and dSink."""
import math

import numpy as np
import pytest

torch = pytest.importorskip("torch")

pytestmark = pytest.mark.gpu

import exact_tiled_attention_softmax_b200 as eta  # noqa: E402
import oracle  # noqa: E402
from oracle import philox as P  # noqa: E402
from tests.parity_util import check_close, to_dev, to_np  # noqa: E402
from tests.test_gpu_parity import TORCH_DTYPE, _qk_case, _segment_starts  # noqa: E402


@pytest.fixture(scope="module", autouse=True)
def _cuda():
    if not torch.cuda.is_available():
        pytest.skip("no GPU")
    eta.load_library()


def _allowed(c, **extra):
    return eta.AllowedSet(
        causal=c["causal"], window_left=c["window"],
        block_mask=to_dev(c["bm"], torch.uint8) if c["bm"] is not None else None,
        block_q=c["block"] or 128, block_k=c["block"] or 128,
        sink=to_dev(c["sink"], torch.float32) if c["sink"] is not None else None,
        dropout_p=c["dropout"], dropout_seed=c["seed"], **extra)


CASES = {
    "causal": dict(args=(2, 4, 2, 300, 300), kw=dict()),
    "window_block": dict(args=(1, 3, 3, 300, 300), kw=dict(window=100, block=64)),
    "gqa_dropout_sink": dict(args=(2, 4, 2, 260, 260), kw=dict(dropout=0.1, sink=True)),
    "noncausal_longer_keys": dict(args=(1, 2, 1, 150, 330), kw=dict(causal=False)),
    "causal_shorter_keys": dict(args=(1, 2, 2, 300, 130), kw=dict()),
    "packed_segments": dict(args=(2, 2, 2, 384, 384), kw=dict()),
}


@pytest.mark.parametrize("kind", list(CASES))
@pytest.mark.parametrize("dtype", ["bf16", "f16"])
def test_deterministic_dq_matches_oracle_and_repeats(kind, dtype):
    spec = CASES[kind]
    B, Hq, Hkv, Tq, Tk = spec["args"]
    c = _qk_case(B, Hq, Hkv, Tq, Tk, 128, 128, dtype, 61, **spec["kw"])
    extra = {}
    starts = None
    if kind == "packed_segments":
        starts = _segment_starts([[0, 70, 200, 384], [0, 128, 300, 384]], Tq)
        extra["starts"] = to_dev(starts, torch.int32)
    tdt = TORCH_DTYPE[dtype]
    q, k, v, g = (to_dev(c[n], tdt) for n in ("q", "k", "v", "g"))
    al = _allowed(c, deterministic=True, **extra)
    wf = torch.empty(eta.attn_fwd_workspace_size(q, k, v, al), dtype=torch.uint8, device="cuda")
    o, lse = eta.attn_fwd(q, k, v, al, c["scale"], workspace=wf)
    assert eta.attn_get_status(wf) == 0
    wb = torch.empty(eta.attn_bwd_workspace_size(q, k, v, al), dtype=torch.uint8, device="cuda")
    first = eta.attn_bwd(q, k, v, o, g, lse, al, c["scale"], workspace=wb)
    assert eta.attn_get_status(wb) == 0
    for _ in range(2):
        again = eta.attn_bwd(q, k, v, o, g, lse, al, c["scale"], workspace=wb)
        torch.cuda.synchronize()
        for x, y in zip(first, again):
            if x is not None:
                assert torch.equal(x, y)
    dq, dk, dv, ds = first
    allow = oracle.allowed_dense(Tq, Tk, causal=c["causal"], window_left=c["window"], block_mask=c["bm"],
                                 block_q=c["block"] or 1, block_k=c["block"] or 1, query_offset=Tk - Tq,
                                 starts=starts)
    keep = P.dropout_keep(c["seed"], c["dropout"], B, Hq, Tq, Tk) if c["dropout"] else None
    q64, k64, v64, g64 = (c[n].astype(np.float64) for n in ("q", "k", "v", "g"))
    sink = c["sink"].astype(np.float64) if c["sink"] is not None else None
    fw = oracle.forward(q64, k64, v64, allow, c["scale"], sink=sink, keep=keep, rho=c["dropout"])
    bw = oracle.backward(q64, k64, v64, g64, allow, c["scale"], sink=sink, keep=keep, rho=c["dropout"], y=fw.y)
    check_close("dQ", to_np(dq), bw.dq, fp32=False, grad=True)
    check_close("dK", to_np(dk), bw.dk, fp32=False, grad=True)
    check_close("dV", to_np(dv), bw.dv, fp32=False, grad=True)
    # The two reverse modes agree to rounding: same dK and dV kernels, dQ
    # summed in another order.
    al2 = _allowed(c, **extra)
    dq2, dk2, dv2, _ = eta.attn_bwd(q, k, v, o, g, lse, al2, c["scale"])
    torch.cuda.synchronize()
    assert torch.equal(dk2, dk) and torch.equal(dv2, dv)
    rel = float((dq2.float() - dq.float()).norm() / max(dq.float().norm(), 1e-30))
    assert rel <= 1e-2, rel


def test_deterministic_flag_on_the_row_paths_is_accepted():
    """fp32 and top-k calls are deterministic already; the flag is accepted."""
    rng = np.random.default_rng(62)
    q = torch.from_numpy(rng.standard_normal((1, 2, 70, 64), dtype=np.float32)).cuda()
    k = torch.from_numpy(rng.standard_normal((1, 2, 70, 64), dtype=np.float32)).cuda()
    g = torch.from_numpy(rng.standard_normal((1, 2, 70, 64), dtype=np.float32)).cuda()
    al = eta.AllowedSet(causal=True, deterministic=True)
    o, lse = eta.attn_fwd(q, k, k, al, 0.125)
    a = eta.attn_bwd(q, k, k, o, g, lse, al, 0.125)
    b = eta.attn_bwd(q, k, k, o, g, lse, al, 0.125)
    torch.cuda.synchronize()
    assert all(torch.equal(x, y) for x, y in zip(a[:3], b[:3]))
    assert math.isfinite(float(a[0].abs().sum()))

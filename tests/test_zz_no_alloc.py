"""The allocation-free reverse pass (attn_bwd_noalloc), called through the C
ABI, against the regular attn_bwd on the same inputs, two calls in a row.

attn_bwd_noalloc serves callers that cannot allocate device memory (a host
framework that owns the device memory budget, a plugin that may not allocate
behind it, a loop where an allocation's implicit synchronisation is not
allowed). Its scratch is a fixed 64 MiB array inside the library, shared by
every call and keeping the previous call's contents, so every case below runs
twice with the outputs refilled with garbage in between, and covers each part
of the scratch a pass uses: the dense dQ accumulator, the deterministic dQ
pass (which leaves that accumulator unread), the converted copy of an LSE in
another format, and the top-k dKV accumulator (fp32, or fixed point in the
deterministic mode) with its G/P rows. The computation is the regular one,
so everything the regular pass makes reproducible (dK, dV, dSink, dQ in the
deterministic and top-k paths, and the deterministic top-k dKV) must be
bitwise equal; the dense dQ and the default top-k dKV, summed with
floating-point atomics, are held to the parity tolerance.

This file is named so that pytest collects it last."""
import math
import subprocess
import sys
import os

import numpy as np
import pytest

torch = pytest.importorskip("torch")

pytestmark = pytest.mark.gpu

import exact_tiled_attention_softmax_b200 as eta  # noqa: E402
from exact_tiled_attention_softmax_b200 import workloads as W  # noqa: E402
from tests.parity_util import BF16_GRAD_REL, rel_fro  # noqa: E402

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module", autouse=True)
def _cuda():
    if not torch.cuda.is_available():
        pytest.skip("no GPU")
    eta.load_library()


def _bf16(rng, shape):
    return torch.from_numpy(W.round_to_bf16(rng.standard_normal(shape, dtype=np.float32))).cuda().bfloat16()


def _dense_case(kind):
    rng = np.random.default_rng({"causal_gqa": 90, "window_sink": 91, "deterministic": 92, "lse_formats": 93}[kind])
    B, Hq, Hkv, T, d = 2, 4, 2, 300, 128
    q, k, v, g = (_bf16(rng, s) for s in ((B, Hq, T, d), (B, Hkv, T, d), (B, Hkv, T, d), (B, Hq, T, d)))
    sink = torch.tensor([0.3, -0.2, 1.0, 0.0], device="cuda")
    allowed = {
        "causal_gqa": lambda: eta.AllowedSet(causal=True),
        "window_sink": lambda: eta.AllowedSet(causal=True, window_left=100, sink=sink),
        "deterministic": lambda: eta.AllowedSet(causal=True, sink=sink, deterministic=True, dropout_p=0.1,
                                                dropout_seed=7),
        "lse_formats": lambda: eta.AllowedSet(causal=True, sink=sink, lse_kv_only=True, lse_neg_log2=True),
    }[kind]()
    return (q, k, v, g), allowed, 1 / math.sqrt(d)


def _check(kind, got, ref, bitwise_dq):
    names = ("dq", "dk", "dv", "dsink")
    for name, a, b in zip(names, got, ref):
        if a is None:
            assert b is None, name
            continue
        if name == "dq" and not bitwise_dq:
            err = rel_fro(a.float().cpu().numpy(), b.float().cpu().numpy())
            assert err <= BF16_GRAD_REL, (kind, name, err)
        else:
            assert torch.equal(a, b), (kind, name)


@pytest.mark.parametrize("kind", ["causal_gqa", "window_sink", "deterministic", "lse_formats"])
def test_noalloc_dense_matches_regular_backward_twice(kind):
    (q, k, v, g), allowed, scale = _dense_case(kind)
    o, lse = eta.attn_fwd(q, k, v, allowed, scale)
    ref = eta.attn_bwd(q, k, v, o, g, lse, allowed, scale)
    outs = [torch.empty_like(q), torch.empty_like(k), torch.empty_like(v)]
    ds = torch.empty(4, device="cuda") if allowed.sink is not None else None
    for _ in range(2):  # the array keeps the previous call's contents
        for t in outs:
            t.fill_(7.0)
        if ds is not None:
            ds.fill_(7.0)
        eta.attn_bwd_noalloc(q, k, v, o, g, lse, allowed, scale, dq=outs[0], dk=outs[1], dv=outs[2], dsink=ds)
        assert eta.attn_get_status(None) == 0  # the array's own status word, read through the C ABI
        _check(kind, (*outs, ds), ref, bitwise_dq=(kind == "deterministic"))


@pytest.mark.parametrize("deterministic", [False, True])
def test_noalloc_topk_matches_regular_backward_twice(deterministic):
    """The tied top-k layout on the tensor-core path (64 heads, Dqk = 576,
    Dv = 512) with a sink: dQ and dSink bitwise equal to attn_bwd, and dKV
    too with the fixed-point reductions (deterministic); the fp32 reductions'
    dKV within the bf16 gradient bound."""
    rng = np.random.default_rng(94)
    Tq, Tkv, H, Dqk, Dv = 64, 700, 64, 576, 512
    q, kv, g = _bf16(rng, (Tq, H, Dqk)), _bf16(rng, (Tkv, Dqk)), _bf16(rng, (Tq, H, Dv))
    idx, ln = W.topk_lists(Tq, Tkv, 256, 1, 256, 95)
    sink = torch.from_numpy(rng.standard_normal(H).astype(np.float32)).cuda()
    allowed = eta.AllowedSet(topk_idxs=torch.from_numpy(idx).cuda(), topk_length=torch.from_numpy(ln).cuda(),
                             sink=sink, deterministic=deterministic)
    scale = 1 / math.sqrt(Dqk)
    v = kv[:, :Dv]
    o, lse = eta.attn_fwd(q, kv, v, allowed, scale)
    ref = eta.attn_bwd(q, kv, v, o, g, lse, allowed, scale)
    dq, dkv, ds = torch.empty_like(q), torch.empty_like(kv), torch.empty(H, device="cuda")
    for _ in range(2):
        for t in (dq, dkv, ds):
            t.fill_(7.0)
        eta.attn_bwd_noalloc(q, kv, v, o, g, lse, allowed, scale, dq=dq, dk=dkv, dsink=ds)
        assert eta.attn_get_status(None) == 0
        assert torch.equal(dq, ref[0]) and torch.equal(ds, ref[3])
        if deterministic:
            assert torch.equal(dkv, ref[1])
        else:
            err = rel_fro(dkv.float().cpu().numpy(), ref[1].float().cpu().numpy())
            assert err <= BF16_GRAD_REL, err


def test_noalloc_rejects_problems_beyond_its_scratch():
    # B*Hq*T = 2^17 rows needs > 64 MiB (an fp32 dQ accumulator alone is 64 MiB).
    q = torch.empty(1, 16, 8192, 128, dtype=torch.bfloat16, device="cuda")
    k = torch.empty(1, 16, 8192, 128, dtype=torch.bfloat16, device="cuda")
    lse = torch.empty(1, 16, 8192, device="cuda")
    with pytest.raises(eta.AttnError) as ei:
        eta.attn_bwd_noalloc(q, k, k, q, q, lse, eta.AllowedSet(causal=True), 0.1,
                             dq=torch.empty_like(q), dk=torch.empty_like(k), dv=torch.empty_like(k))
    assert ei.value.code == eta.ATTN_ERR_WORKSPACE


_FIRST_CALL_IN_CAPTURE = r"""
import torch, exact_tiled_attention_softmax_b200 as eta
eta.load_library()
q = torch.randn(1, 1, 64, 128, device="cuda").bfloat16()
al = eta.AllowedSet(causal=True)
o, lse = eta.attn_fwd(q, q, q, al, 0.1)
outs = [torch.empty_like(q) for _ in range(3)]
s = torch.cuda.Stream()
torch.cuda.synchronize()
g = torch.cuda.CUDAGraph()
code = None
with torch.cuda.graph(g, stream=s):
    try:
        eta.attn_bwd_noalloc(q, q, q, o, q, lse, al, 0.1, dq=outs[0], dk=outs[1], dv=outs[2], stream=s)
    except eta.AttnError as e:
        code = e.code
assert code == eta.ATTN_ERR_UNSUPPORTED, code
# Outside the capture the same call sets the array up and runs.
eta.attn_bwd_noalloc(q, q, q, o, q, lse, al, 0.1, dq=outs[0], dk=outs[1], dv=outs[2])
assert eta.attn_get_status(None) == 0
print("ok")
"""


def test_noalloc_first_call_inside_a_capture_is_refused():
    """In a fresh process, a first call made while its stream is being
    captured cannot look up the array (that lookup is not a stream operation
    and may load device code): it returns ATTN_ERR_UNSUPPORTED and enqueues
    nothing; the next call, outside the capture, runs."""
    r = subprocess.run([sys.executable, "-c", _FIRST_CALL_IN_CAPTURE], cwd=ROOT, capture_output=True, text=True,
                       timeout=300)
    assert r.returncode == 0 and r.stdout.strip().endswith("ok"), r.stdout[-2000:] + r.stderr[-2000:]

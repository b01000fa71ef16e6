"""The allocation-free reverse pass (attn_bwd_noalloc), called through the C
ABI, against the regular attn_bwd on the same inputs, two calls in a row.

attn_bwd_noalloc serves callers that cannot allocate device memory (a host
framework that owns the device memory budget, a plugin that may not allocate
behind it, a loop where an allocation's implicit synchronisation is not
allowed). Its scratch is a fixed 64 MiB array inside the library. This file
is named so that pytest collects it last."""
import math

import numpy as np
import pytest

torch = pytest.importorskip("torch")

pytestmark = pytest.mark.gpu

import exact_tiled_attention_softmax_b200 as eta  # noqa: E402
from exact_tiled_attention_softmax_b200 import workloads as W  # noqa: E402
from tests.parity_util import BF16_GRAD_REL, rel_fro  # noqa: E402


@pytest.fixture(scope="module", autouse=True)
def _cuda():
    if not torch.cuda.is_available():
        pytest.skip("no GPU")
    eta.load_library()


def _inputs(B, Hq, Hkv, T, d, seed):
    rng = np.random.default_rng(seed)
    f = lambda s: torch.from_numpy(W.round_to_bf16(rng.standard_normal(s, dtype=np.float32))).cuda().bfloat16()
    return f((B, Hq, T, d)), f((B, Hkv, T, d)), f((B, Hkv, T, d)), f((B, Hq, T, d))


@pytest.mark.parametrize("kind", ["causal_gqa", "window_sink"])
def test_noalloc_matches_regular_backward_twice(kind):
    q, k, v, g = _inputs(2, 4, 2, 300, 128, 90 if kind == "causal_gqa" else 91)
    if kind == "causal_gqa":
        allowed = eta.AllowedSet(causal=True)
    else:
        allowed = eta.AllowedSet(causal=True, window_left=100,
                                 sink=torch.tensor([0.3, -0.2, 1.0, 0.0], device="cuda"))
    scale = 1 / math.sqrt(128)
    o, lse = eta.attn_fwd(q, k, v, allowed, scale)
    ref = eta.attn_bwd(q, k, v, o, g, lse, allowed, scale)
    outs = [torch.empty_like(q), torch.empty_like(k), torch.empty_like(v)]
    ds = torch.empty(4, device="cuda") if allowed.sink is not None else None
    for _ in range(2):  # the array keeps the previous call's contents
        for t in outs:
            t.fill_(7.0)
        eta.attn_bwd_noalloc(q, k, v, o, g, lse, allowed, scale, dq=outs[0], dk=outs[1], dv=outs[2], dsink=ds)
        torch.cuda.synchronize()
        for name, got, want in zip(("dq", "dk", "dv"), outs, ref[:3]):
            err = rel_fro(got.float().cpu().numpy(), want.float().cpu().numpy())
            assert err <= BF16_GRAD_REL, (name, err)
        if ds is not None:
            assert torch.allclose(ds, ref[3], rtol=1e-5, atol=1e-5)


def test_noalloc_rejects_problems_beyond_its_scratch():
    # B*Hq*T = 2^17 rows needs > 64 MiB (an fp32 dQ accumulator alone is 64 MiB).
    q = torch.empty(1, 16, 8192, 128, dtype=torch.bfloat16, device="cuda")
    k = torch.empty(1, 16, 8192, 128, dtype=torch.bfloat16, device="cuda")
    lse = torch.empty(1, 16, 8192, device="cuda")
    with pytest.raises(eta.AttnError) as ei:
        eta.attn_bwd_noalloc(q, k, k, q, q, lse, eta.AllowedSet(causal=True), 0.1,
                             dq=torch.empty_like(q), dk=torch.empty_like(k), dv=torch.empty_like(k))
    assert ei.value.code == eta.ATTN_ERR_WORKSPACE

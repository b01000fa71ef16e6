"""The autograd node over the C ABI: gradients equal the direct attn_bwd
outputs bit for bit, reach a sink tensor, and the tied top-k layout returns
dKV once to a KV leaf that K and V were sliced from."""
import math

import numpy as np
import pytest

torch = pytest.importorskip("torch")

pytestmark = pytest.mark.gpu

import exact_tiled_attention_softmax_b200 as eta  # noqa: E402
from exact_tiled_attention_softmax_b200 import workloads as W  # noqa: E402
from tests.parity_util import to_dev  # noqa: E402


@pytest.fixture(scope="module", autouse=True)
def _cuda():
    if not torch.cuda.is_available():
        pytest.skip("no GPU")
    eta.load_library()


def test_dense_autograd_matches_direct_calls():
    rng = np.random.default_rng(81)
    f = lambda s: to_dev(W.round_to_bf16(rng.standard_normal(s, dtype=np.float32)), torch.bfloat16)  # noqa: E731
    q, k, v, g = f((1, 4, 200, 128)), f((1, 2, 200, 128)), f((1, 2, 200, 128)), f((1, 4, 200, 128))
    sink = torch.from_numpy(rng.standard_normal(4).astype(np.float32)).cuda()
    al = eta.AllowedSet(causal=True, window_left=90)
    scale = 1 / math.sqrt(128)
    qa, ka, va, sa = (x.clone().requires_grad_(True) for x in (q, k, v, sink))
    o, lse = eta.attention(qa, ka, va, al, scale, sink=sa)
    o.backward(g)
    al_s = eta.AllowedSet(causal=True, window_left=90, sink=sink)
    o_d, lse_d = eta.attn_fwd(q, k, v, al_s, scale)
    dq, dk, dv, ds = eta.attn_bwd(q, k, v, o_d, g, lse_d, al_s, scale)
    torch.cuda.synchronize()
    assert torch.equal(o.detach(), o_d) and torch.equal(lse, lse_d)
    assert torch.equal(qa.grad, dq) and torch.equal(ka.grad, dk) and torch.equal(va.grad, dv)
    assert torch.equal(sa.grad, ds)
    assert not lse.requires_grad


def test_topk_autograd_returns_tied_dkv_once():
    rng = np.random.default_rng(82)
    Tq, Tkv, H, Dqk, Dv = 16, 300, 4, 96, 64
    q = to_dev(W.round_to_bf16(rng.standard_normal((Tq, H, Dqk), dtype=np.float32)), torch.bfloat16)
    kv = to_dev(W.round_to_bf16(rng.standard_normal((Tkv, Dqk), dtype=np.float32)), torch.bfloat16)
    g = to_dev(W.round_to_bf16(rng.standard_normal((Tq, H, Dv), dtype=np.float32)), torch.bfloat16)
    idx, ln = W.topk_lists(Tq, Tkv, 64, 8, 64, 83)
    al = eta.AllowedSet(topk_idxs=to_dev(idx, torch.int32), topk_length=to_dev(ln, torch.int32))
    kv_leaf = kv.clone().requires_grad_(True)
    q_leaf = q.clone().requires_grad_(True)
    o, _ = eta.attention(q_leaf, kv_leaf, kv_leaf[:, :Dv], al, 1 / math.sqrt(Dqk))
    o.backward(g)
    o_d, lse_d = eta.attn_fwd(q, kv, kv[:, :Dv], al, 1 / math.sqrt(Dqk))
    dq, dkv, _, _ = eta.attn_bwd(q, kv, kv[:, :Dv], o_d, g, lse_d, al, 1 / math.sqrt(Dqk))
    torch.cuda.synchronize()
    assert torch.equal(q_leaf.grad, dq)
    assert torch.equal(kv_leaf.grad, dkv)

"""Checks that stand in for a memory checker, plus the device-side contract
checks of the top-k path.

1. Guard bytes. Every output (and the workspace) is carved out of a larger
   buffer filled with a canary byte: guard regions before and after it, and,
   for row-strided outputs, a gap after every row. After attn_fwd and
   attn_bwd every byte that is not an element of an output must still hold
   the canary, on the dense tensor-core path (default and deterministic
   reverse), the top-k tensor-core path and the row-wise kernels, at ragged
   sizes.
2. The top-k lists' causality (DSA note, section 1: each token's list holds
   only indices up to its own position, Tkv - Tq + t). With the debug flag an
   index past that position sets ATTN_DEVERR_TOPK_CAUSAL and is still used
   (the result equals the oracle on the given lists); without it nothing is
   reported.
3. The fixed-point dKV sum (the row kernels, and the tensor-core path with
   ATTN_BWD_DETERMINISTIC). Planted contributions below the per-addend clamp
   (2^30) whose sum over the tokens that list one KV row exceeds the 32.32
   range (2^31) set ATTN_DEVERR_OVERFLOW; nothing faults.
"""
import math

import numpy as np
import pytest

torch = pytest.importorskip("torch")

pytestmark = pytest.mark.gpu

import exact_tiled_attention_softmax_b200 as eta  # noqa: E402
from exact_tiled_attention_softmax_b200 import workloads as W  # noqa: E402
import oracle  # noqa: E402
from tests.parity_util import BF16_GRAD_REL, BF16_O_ABS, o_excess, rel_fro, to_np  # noqa: E402

CANARY = 0xA5
GUARD = 4096  # bytes before and after each region (a multiple of 256)


@pytest.fixture(scope="module", autouse=True)
def _cuda():
    if not torch.cuda.is_available():
        pytest.skip("no GPU")
    eta.load_library()


class Guarded:
    """A tensor of `shape` and `dtype` inside a canary-filled byte buffer,
    with GUARD bytes on both sides and `pad` unused elements after every
    innermost row (so the row stride is shape[-1] + pad)."""

    def __init__(self, shape, dtype, pad=0):
        es = torch.empty(0, dtype=dtype).element_size()
        full = tuple(shape[:-1]) + (shape[-1] + pad,)
        n = int(np.prod(full)) * es
        self.buf = torch.full((GUARD + n + GUARD,), CANARY, dtype=torch.uint8, device="cuda")
        region = self.buf[GUARD:GUARD + n]
        self.t = region.view(dtype).view(full)[..., :shape[-1]]
        own = torch.zeros_like(self.buf, dtype=torch.bool)
        own[GUARD:GUARD + n].view(full[:-1] + (full[-1] * es,))[..., :shape[-1] * es] = True
        self.free = ~own

    def intact(self) -> bool:
        return bool((self.buf[self.free] == CANARY).all())


def _ws(nbytes):
    """A workspace with guard bytes on both sides (256-byte aligned start)."""
    g = Guarded((nbytes,), torch.uint8)
    return g, g.t


def _bf16(rng, shape):
    return torch.from_numpy(W.round_to_bf16(rng.standard_normal(shape, dtype=np.float32))).cuda().bfloat16()


@pytest.mark.parametrize("deterministic", [False, True])
def test_guard_bytes_dense_tensor_cores(deterministic):
    rng = np.random.default_rng(101)
    B, Hq, Hkv, T, d = 2, 4, 2, 300, 128
    q, k, v, g = (_bf16(rng, s) for s in ((B, Hq, T, d), (B, Hkv, T, d), (B, Hkv, T, d), (B, Hq, T, d)))
    sink = torch.tensor([0.3, -0.2, 1.0, 0.0], device="cuda")
    al = eta.AllowedSet(causal=True, window_left=170, sink=sink, dropout_p=0.1, dropout_seed=5,
                        deterministic=deterministic)
    scale = 1 / math.sqrt(d)
    o, lse = Guarded((B, Hq, T, d), torch.bfloat16, pad=8), Guarded((B, Hq, T), torch.float32, pad=5)
    gwf, wf = _ws(eta.attn_fwd_workspace_size(q, k, v, al))
    eta.attn_fwd(q, k, v, al, scale, out=o.t, lse=lse.t, workspace=wf)
    assert eta.attn_get_status(wf) == 0
    dq, dk, dv = (Guarded(x.shape, torch.bfloat16, pad=8) for x in (q, k, v))
    ds = Guarded((Hq,), torch.float32)
    gwb, wb = _ws(eta.attn_bwd_workspace_size(q, k, v, al))
    eta.attn_bwd(q, k, v, o.t, g, lse.t, al, scale, dq=dq.t, dk=dk.t, dv=dv.t, dsink=ds.t, workspace=wb)
    assert eta.attn_get_status(wb) == 0
    torch.cuda.synchronize()
    for name, x in (("o", o), ("lse", lse), ("dq", dq), ("dk", dk), ("dv", dv), ("dsink", ds), ("fwd ws", gwf),
                    ("bwd ws", gwb)):
        assert x.intact(), name
    # The strided outputs hold the same values as contiguous ones.
    o2, lse2 = eta.attn_fwd(q, k, v, al, scale)
    dq2, dk2, dv2, ds2 = eta.attn_bwd(q, k, v, o2, g, lse2, al, scale)
    assert torch.equal(o.t, o2) and torch.equal(lse.t, lse2)
    assert torch.equal(dk.t, dk2) and torch.equal(dv.t, dv2) and torch.equal(ds.t, ds2)
    assert rel_fro(to_np(dq.t), to_np(dq2)) <= 1e-2


def _topk_case(seed, Tq, Tkv, H, Dqk, Dv, topk, dtype=torch.bfloat16):
    rng = np.random.default_rng(seed)
    rnd = (lambda s: _bf16(rng, s)) if dtype == torch.bfloat16 else \
        (lambda s: torch.from_numpy(rng.standard_normal(s, dtype=np.float32)).cuda())
    q, kv, g = rnd((Tq, H, Dqk)), rnd((Tkv, Dqk)), rnd((Tq, H, Dv))
    idx, ln = W.topk_lists(Tq, Tkv, topk, 1, topk, seed + 1)
    sink = torch.from_numpy(rng.standard_normal(H).astype(np.float32)).cuda()
    return q, kv, g, idx, ln, sink


@pytest.mark.parametrize("path", ["tensor_cores", "rows"])
def test_guard_bytes_topk(path):
    if path == "tensor_cores":
        Tq, Tkv, H, Dqk, Dv, dt, pad = 40, 700, 64, 576, 512, torch.bfloat16, 8
    else:
        Tq, Tkv, H, Dqk, Dv, dt, pad = 37, 300, 6, 96, 64, torch.float32, 3
    q, kv, g, idx, ln, sink = _topk_case(102, Tq, Tkv, H, Dqk, Dv, 200, dt)
    al = eta.AllowedSet(topk_idxs=torch.from_numpy(idx).cuda(), topk_length=torch.from_numpy(ln).cuda(), sink=sink)
    scale = 1 / math.sqrt(Dqk)
    v = kv[:, :Dv]
    o, lse = Guarded((Tq, H, Dv), dt, pad=pad), Guarded((Tq, H), torch.float32, pad=3)
    gwf, wf = _ws(eta.attn_fwd_workspace_size(q, kv, v, al))
    eta.attn_fwd(q, kv, v, al, scale, out=o.t, lse=lse.t, workspace=wf)
    assert eta.attn_get_status(wf) == 0
    dq, dkv, ds = Guarded((Tq, H, Dqk), dt, pad=pad), Guarded((Tkv, Dqk), dt, pad=pad), Guarded((H,), torch.float32)
    gwb, wb = _ws(eta.attn_bwd_workspace_size(q, kv, v, al))
    eta.attn_bwd(q, kv, v, o.t, g, lse.t, al, scale, dq=dq.t, dk=dkv.t, dsink=ds.t, workspace=wb)
    assert eta.attn_get_status(wb) == 0
    torch.cuda.synchronize()
    for name, x in (("o", o), ("lse", lse), ("dq", dq), ("dkv", dkv), ("dsink", ds), ("fwd ws", gwf),
                    ("bwd ws", gwb)):
        assert x.intact(), name


def test_guard_bytes_dense_rows():
    """fp32 and a head width without a tensor-core kernel: the row-wise kernels."""
    rng = np.random.default_rng(103)
    B, Hq, Hkv, T, d, dv = 1, 3, 1, 201, 64, 96
    f = lambda s: torch.from_numpy(rng.standard_normal(s, dtype=np.float32)).cuda()  # noqa: E731
    q, k, v, g = f((B, Hq, T, d)), f((B, Hkv, T, d)), f((B, Hkv, T, dv)), f((B, Hq, T, dv))
    al = eta.AllowedSet(causal=True, dropout_p=0.2, dropout_seed=9, sink=torch.tensor([0.1, 0.2, -0.3]).cuda())
    o, lse = Guarded((B, Hq, T, dv), torch.float32, pad=3), Guarded((B, Hq, T), torch.float32, pad=2)
    gwf, wf = _ws(eta.attn_fwd_workspace_size(q, k, v, al))
    eta.attn_fwd(q, k, v, al, 0.125, out=o.t, lse=lse.t, workspace=wf)
    dq, dk, dvv = Guarded((B, Hq, T, d), torch.float32, 3), Guarded((B, Hkv, T, d), torch.float32, 3), \
        Guarded((B, Hkv, T, dv), torch.float32, 3)
    ds = Guarded((Hq,), torch.float32)
    gwb, wb = _ws(eta.attn_bwd_workspace_size(q, k, v, al))
    eta.attn_bwd(q, k, v, o.t, g, lse.t, al, 0.125, dq=dq.t, dk=dk.t, dv=dvv.t, dsink=ds.t, workspace=wb)
    torch.cuda.synchronize()
    for name, x in (("o", o), ("lse", lse), ("dq", dq), ("dk", dk), ("dv", dvv), ("dsink", ds), ("fwd ws", gwf),
                    ("bwd ws", gwb)):
        assert x.intact(), name


def _non_causal_lists(idx, ln, Tq, Tkv):
    """Copies of the lists where token 3 and token Tq - 2 each list one index
    past their causal position (still inside [0, Tkv))."""
    idx, ln = idx.copy(), ln.copy()
    for t in (3, Tq - 2):
        pos = Tkv - Tq + t
        ln[t] = max(ln[t], 2)
        idx[t, 1] = min(pos + 1 + t % 5, Tkv - 1)
        assert idx[t, 1] > pos and idx[t, 1] not in idx[t, :1]
    return idx, ln


@pytest.mark.parametrize("path", ["tensor_cores", "rows"])
def test_topk_causal_debug_check(path):
    if path == "tensor_cores":
        Tq, Tkv, H, Dqk, Dv, dt = 24, 300, 64, 576, 512, torch.bfloat16
    else:
        Tq, Tkv, H, Dqk, Dv, dt = 24, 300, 4, 96, 64, torch.float32
    q, kv, g, idx, ln, sink = _topk_case(104, Tq, Tkv, H, Dqk, Dv, 64, dt)
    idx, ln = _non_causal_lists(idx, ln, Tq, Tkv)
    scale = 1 / math.sqrt(Dqk)
    v = kv[:, :Dv]
    for check in (False, True):
        al = eta.AllowedSet(topk_idxs=torch.from_numpy(idx).cuda(), topk_length=torch.from_numpy(ln).cuda(),
                            sink=sink, topk_check_causal=check)
        wf = torch.empty(eta.attn_fwd_workspace_size(q, kv, v, al), dtype=torch.uint8, device="cuda")
        wb = torch.empty(eta.attn_bwd_workspace_size(q, kv, v, al), dtype=torch.uint8, device="cuda")
        o, lse = eta.attn_fwd(q, kv, v, al, scale, workspace=wf)
        bits_f = eta.attn_get_status(wf)
        dq, dkv, _, ds = eta.attn_bwd(q, kv, v, o, g, lse, al, scale, workspace=wb)
        bits_b = eta.attn_get_status(wb)
        expect = eta.ATTN_DEVERR_TOPK_CAUSAL if check else 0
        assert bits_f == expect and bits_b == expect, (bits_f, bits_b)
    # The flagged entries are used: the result is the oracle's on the given lists.
    q64 = q.float().cpu().numpy()
    kv64 = kv.float().cpu().numpy()
    g64 = g.float().cpu().numpy()
    s64 = sink.cpu().numpy().astype(np.float64)
    o_r, lse_r, _ = oracle.topk_forward(q64, kv64, idx, ln, Dv, scale, s64)
    dq_r, dkv_r, _ = oracle.topk_backward(q64, kv64, idx, ln, Dv, scale, g64, s64, o=o_r)
    fp32 = dt == torch.float32
    if fp32:
        assert np.abs(to_np(o) - o_r).max() <= 1e-5
    else:
        assert o_excess(to_np(o), o_r) <= BF16_O_ABS
    assert rel_fro(to_np(dq), dq_r) <= (1e-5 if fp32 else BF16_GRAD_REL)
    assert rel_fro(to_np(dkv), dkv_r) <= (1e-5 if fp32 else BF16_GRAD_REL)


@pytest.mark.parametrize("path", ["tensor_cores", "rows"])
def test_fixed_point_sum_overflow_is_flagged(path):
    """Every token lists KV row 0 alone (no sink): P = 1, so the row's
    contribution per token is the sum over heads of that token's upstream
    gradient, 64 (or 4) x 2^23 = 5.4e8 (3.4e7) per element: under the 2^30
    clamp, but 300 tokens push the sum past 2^31 (the 32.32 range). The
    overflow bit comes from the bound on the sum; a small case with the same
    lists stays clean."""
    if path == "tensor_cores":
        H, Dqk, Dv, dt = 64, 576, 512, torch.bfloat16
    else:
        H, Dqk, Dv, dt = 4, 96, 64, torch.float32
    Tq, Tkv = 300, 600
    rng = np.random.default_rng(105)
    q = torch.from_numpy(rng.standard_normal((Tq, H, Dqk), dtype=np.float32)).cuda().to(dt)
    kv = torch.from_numpy(rng.standard_normal((Tkv, Dqk), dtype=np.float32)).cuda().to(dt)
    idx = np.full((Tq, 4), -1, np.int32)
    idx[:, 0] = 0
    ln = np.ones(Tq, np.int32)
    al = eta.AllowedSet(topk_idxs=torch.from_numpy(idx).cuda(), topk_length=torch.from_numpy(ln).cuda(),
                        deterministic=True)
    v = kv[:, :Dv]
    o, lse = eta.attn_fwd(q, kv, v, al, 1 / 24)
    for big, expect in ((2.0 ** 23, eta.ATTN_DEVERR_OVERFLOW), (1.0, 0)):
        g = torch.full((Tq, H, Dv), big, device="cuda", dtype=dt)
        wb = torch.empty(eta.attn_bwd_workspace_size(q, kv, v, al), dtype=torch.uint8, device="cuda")
        eta.attn_bwd(q, kv, v, o, g, lse, al, 1 / 24, workspace=wb)
        assert eta.attn_get_status(wb) == expect, big

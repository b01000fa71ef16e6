"""GPU parity of the tensor-core top-k forward (64 heads, Dqk = 576, Dv = 512,
bf16: the shape the DSA note's kernel targets) against the float64 oracle.

Cases span several 64-key tiles with ragged last tiles, an empty list, the
sink, the lazy running-max move (later tiles with much larger scores), and a
listed index outside [0, Tkv) that must be skipped and flagged."""
import math

import numpy as np
import pytest

torch = pytest.importorskip("torch")

pytestmark = pytest.mark.gpu

import exact_tiled_attention_softmax_b200 as eta  # noqa: E402
from exact_tiled_attention_softmax_b200 import workloads as W  # noqa: E402
import oracle  # noqa: E402
from tests.parity_util import BF16_O_ABS, o_excess, to_dev, to_np  # noqa: E402

H, DQK, DV = 64, 576, 512


@pytest.fixture(scope="module", autouse=True)
def _cuda():
    if not torch.cuda.is_available():
        pytest.skip("no GPU")
    eta.load_library()


def _case(seed, Tq=24, Tkv=700, topk=256, lo=1, hi=256, sink=True, grow=False):
    rng = np.random.default_rng(seed)
    q = W.round_to_bf16(rng.standard_normal((Tq, H, DQK), dtype=np.float32))
    kv = W.round_to_bf16(rng.standard_normal((Tkv, DQK), dtype=np.float32))
    idx, ln = W.topk_lists(Tq, Tkv, topk, lo, hi, seed + 1)
    if grow:
        # The last 64 columns (they enter the scores only, never V) of the
        # rows in the upper half of the index range are 16x larger (exact in
        # bf16) and every list is sorted: later tiles raise the running max
        # by far more than 2^8 while O stays of unit scale.
        kv[Tkv // 2:, DV:] *= 16.0
        for t in range(Tq):
            idx[t, :ln[t]] = np.sort(idx[t, :ln[t]])
    sk = rng.standard_normal(H).astype(np.float32) if sink else None
    return q, kv, idx, ln, sk


def _run(q, kv, idx, ln, sk, scale):
    qd, kvd = to_dev(q, torch.bfloat16), to_dev(kv, torch.bfloat16)
    al = eta.AllowedSet(topk_idxs=to_dev(idx, torch.int32), topk_length=to_dev(ln, torch.int32),
                        sink=to_dev(sk, torch.float32) if sk is not None else None)
    ws = torch.empty(eta.attn_fwd_workspace_size(qd, kvd, kvd[:, :DV], al), dtype=torch.uint8, device="cuda")
    o, lse = eta.attn_fwd(qd, kvd, kvd[:, :DV], al, scale, workspace=ws)
    status = eta.attn_get_status(ws)
    torch.cuda.synchronize()
    return to_np(o), to_np(lse), status


def _check(o, lse, o_ref, lse_ref, storage="bf16", p_abs=None):
    # Element by element: |O - O_ref| <= 1e-2 + ulp(O_ref)/2 in the storage
    # type (+ the P operand's rounding bound where p_abs is given).
    err = o_excess(o, o_ref, storage, p_abs)
    assert err <= BF16_O_ABS, err
    fin = np.isfinite(lse_ref)
    assert np.array_equal(np.isfinite(lse), fin)
    assert np.abs(lse[fin] - lse_ref[fin]).max(initial=0) <= 1e-3


@pytest.mark.parametrize("sink", [True, False])
def test_topk_tc_ragged_tiles(sink):
    q, kv, idx, ln, sk = _case(71, sink=sink)
    ln[5] = 0        # empty list: O = 0, LSE = z or -inf
    ln[6] = 64       # exactly one tile
    ln[7] = 65       # one key into the second tile
    scale = 1 / math.sqrt(DQK)
    o, lse, status = _run(q, kv, idx, ln, sk, scale)
    assert status == 0
    o_ref, lse_ref, _ = oracle.topk_forward(q, kv, idx, ln, DV, scale,
                                            sk.astype(np.float64) if sk is not None else None)
    _check(o, lse, o_ref, lse_ref)


def test_topk_tc_running_max_moves():
    q, kv, idx, ln, sk = _case(72, grow=True, lo=128, hi=256)
    scale = 1 / math.sqrt(DQK)
    o, lse, status = _run(q, kv, idx, ln, sk, scale)
    assert status == 0
    o_ref, lse_ref, _ = oracle.topk_forward(q, kv, idx, ln, DV, scale, sk.astype(np.float64))
    # These rows are nearly one-hot on keys whose |V| reaches 4 and more: the
    # bf16 rounding of the dominant P entry (up to 2^-8 relative) alone moves
    # O by up to ~0.017, so the bound adds 2^-8 sum_j p_j |V_j| per element,
    # from the oracle's dense form with |V| (the same p, since p does not
    # depend on V).
    q64 = q.astype(np.float64).transpose(1, 0, 2)[None]
    kv64 = kv.astype(np.float64)
    p_abs = oracle.forward(q64, kv64[None, None], np.abs(kv64[:, :DV])[None, None],
                           oracle.topk_allowed(idx, ln, kv.shape[0]), scale,
                           sink=sk.astype(np.float64)).y[0].transpose(1, 0, 2)
    _check(o, lse, o_ref, lse_ref, p_abs=p_abs)


def test_topk_tc_bad_index_skipped_and_flagged():
    q, kv, idx, ln, sk = _case(73, lo=100, hi=200)
    bad_t = 3
    idx[bad_t, 10] = kv.shape[0] + 5   # outside [0, Tkv), inside the valid length
    scale = 1 / math.sqrt(DQK)
    o, lse, status = _run(q, kv, idx, ln, sk, scale)
    assert status & eta.ATTN_DEVERR_TOPK_INDEX
    # The reference drops the bad entry (the list shifts left by one).
    idx_ref, ln_ref = idx.copy(), ln.copy()
    idx_ref[bad_t, 10:-1] = idx[bad_t, 11:]
    ln_ref[bad_t] -= 1
    o_ref, lse_ref, _ = oracle.topk_forward(q, kv, idx_ref, ln_ref, DV, scale, sk.astype(np.float64))
    _check(o, lse, o_ref, lse_ref)


@pytest.mark.parametrize("deterministic", [False, True])
def test_topk_tc_backward_matches_oracle_and_is_reproducible(deterministic):
    """dQ, dKV and dSink against the oracle with the fp32 dKV reductions
    (default) and the 32.32 fixed-point ones (deterministic); dQ and dSink
    repeat bit for bit in both modes, dKV in the deterministic one."""
    from tests.parity_util import BF16_GRAD_REL, rel_fro
    q, kv, idx, ln, sk = _case(74)
    ln[5] = 0
    ln[6] = 64
    ln[7] = 65
    rng = np.random.default_rng(75)
    g = W.round_to_bf16(rng.standard_normal((q.shape[0], H, DV), dtype=np.float32))
    scale = 1 / math.sqrt(DQK)
    qd, kvd, gd = to_dev(q, torch.bfloat16), to_dev(kv, torch.bfloat16), to_dev(g, torch.bfloat16)
    al = eta.AllowedSet(topk_idxs=to_dev(idx, torch.int32), topk_length=to_dev(ln, torch.int32),
                        sink=to_dev(sk, torch.float32), deterministic=deterministic)
    o, lse = eta.attn_fwd(qd, kvd, kvd[:, :DV], al, scale)
    ws = torch.empty(eta.attn_bwd_workspace_size(qd, kvd, kvd[:, :DV], al), dtype=torch.uint8, device="cuda")
    dq, dkv, _, ds = eta.attn_bwd(qd, kvd, kvd[:, :DV], o, gd, lse, al, scale, workspace=ws)
    assert eta.attn_get_status(ws) == 0
    sink64 = sk.astype(np.float64)
    o_ref, _, _ = oracle.topk_forward(q, kv, idx, ln, DV, scale, sink64)
    dq_ref, dkv_ref, ds_ref = oracle.topk_backward(q, kv, idx, ln, DV, scale, g, sink64, o=o_ref)
    assert rel_fro(to_np(dq), dq_ref) <= BF16_GRAD_REL
    assert rel_fro(to_np(dkv), dkv_ref) <= BF16_GRAD_REL
    assert np.abs(to_np(ds) - ds_ref).max() <= 2e-2 * max(1.0, np.abs(ds_ref).max())
    assert np.all(to_np(dq)[5] == 0.0)  # the empty list's token
    dq2, dkv2, _, ds2 = eta.attn_bwd(qd, kvd, kvd[:, :DV], o, gd, lse, al, scale, workspace=ws)
    torch.cuda.synchronize()
    assert torch.equal(dq2, dq) and torch.equal(ds2, ds)
    if deterministic:
        assert torch.equal(dkv2, dkv)
    else:
        assert rel_fro(to_np(dkv2), to_np(dkv).astype(np.float64)) <= 1e-2


@pytest.mark.parametrize("deterministic", [False, True])
def test_topk_tc_fp16_storage(deterministic):
    """fp16 storage (the DSA note's storage table allows BF16 or FP16): the
    same kernels with fp16 operands, forward and reverse against the oracle
    on the fp16-rounded inputs, with either dKV reduction."""
    from tests.parity_util import BF16_GRAD_REL, rel_fro
    rng = np.random.default_rng(76)
    Tq, Tkv = 24, 700
    q = W.round_to_fp16(rng.standard_normal((Tq, H, DQK), dtype=np.float32))
    kv = W.round_to_fp16(rng.standard_normal((Tkv, DQK), dtype=np.float32))
    g = W.round_to_fp16(rng.standard_normal((Tq, H, DV), dtype=np.float32))
    idx, ln = W.topk_lists(Tq, Tkv, 256, 128, 256, 77)   # every list holds >= 128 entries
    ln[5] = 0
    ln[6] = 64
    ln[7] = 65
    sk = rng.standard_normal(H).astype(np.float32)
    scale = 1 / math.sqrt(DQK)
    qd, kvd, gd = to_dev(q, torch.float16), to_dev(kv, torch.float16), to_dev(g, torch.float16)
    al = eta.AllowedSet(topk_idxs=to_dev(idx, torch.int32), topk_length=to_dev(ln, torch.int32),
                        sink=to_dev(sk, torch.float32), deterministic=deterministic)
    wf = torch.empty(eta.attn_fwd_workspace_size(qd, kvd, kvd[:, :DV], al), dtype=torch.uint8, device="cuda")
    o, lse = eta.attn_fwd(qd, kvd, kvd[:, :DV], al, scale, workspace=wf)
    assert eta.attn_get_status(wf) == 0
    ws = torch.empty(eta.attn_bwd_workspace_size(qd, kvd, kvd[:, :DV], al), dtype=torch.uint8, device="cuda")
    dq, dkv, _, ds = eta.attn_bwd(qd, kvd, kvd[:, :DV], o, gd, lse, al, scale, workspace=ws)
    assert eta.attn_get_status(ws) == 0
    sink64 = sk.astype(np.float64)
    o_ref, lse_ref, _ = oracle.topk_forward(q, kv, idx, ln, DV, scale, sink64)
    _check(to_np(o), to_np(lse), o_ref, lse_ref, storage="f16")
    dq_ref, dkv_ref, ds_ref = oracle.topk_backward(q, kv, idx, ln, DV, scale, g, sink64, o=o_ref)
    assert rel_fro(to_np(dq), dq_ref) <= BF16_GRAD_REL
    assert rel_fro(to_np(dkv), dkv_ref) <= BF16_GRAD_REL
    assert np.abs(to_np(ds) - ds_ref).max() <= 2e-2 * max(1.0, np.abs(ds_ref).max())

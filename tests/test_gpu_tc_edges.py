"""Edge cases forced through the dense tensor-core path (bf16 or fp16 storage,
d = dv = 128, the shapes the tcgen05 kernels take).

1. The pages' worked examples, zero-padded from their one- or two-wide heads
   to d = dv = 128. Zero columns add nothing to any score and give zero
   output and gradient columns, so the padded problem has the examples'
   results in its first columns. Where the examples' values are exact in
   bf16 the results are checked exactly; where they are not (ln 2, ln 0.3),
   against the oracle on the rounded inputs and against the printed values
   within the bf16 bound:
   - one key: Y = 7, dQ = dK = 0, dV = 4 ("Exact tiled attention and
     memory-aware differentiation - Examples", example "One-key tiled
     attention");
   - an empty first key block for row 1, A_1 = {2}, A_2 = {1, 2}: Y = (5, 4)
     (same page, example "An empty first masked key block");
   - two merge orders give the same result, Y = 2 (same page);
   - the two-tile trace's last row (3.4927, 34.927) ("Accumulate attention
     without keeping the full grid", trace cards);
   - the sink example: o = 0.7, dS = (0.65, -0.51), dz = -0.14 ("DeepSeek
     Sparse Attention Forward and Backward", section 4);
   - dropout replay: xi = (1, 0) gives Y_1 = 2 and dV = (1, 0) ("A different
     dropout mask changes the reverse result").
2. The lazy running maximum of the forward kernel: later key tiles score far
   higher than earlier ones (by more than the 2^8 move threshold from one
   tile to the next on some rows, less on others, and falling on others), so
   the maximum moves and the O accumulator is rescaled in TMEM.
"""
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
from tests.parity_util import BF16_GRAD_REL, BF16_O_ABS, o_excess, rel_fro, to_np  # noqa: E402

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")
D = 128


@pytest.fixture(scope="module", autouse=True)
def _cuda():
    if not torch.cuda.is_available():
        pytest.skip("no GPU")
    eta.load_library()


def _golden(name):
    with open(os.path.join(GOLDEN, name)) as f:
        return json.load(f)


def _pad(x):
    """[T, w] values -> [T, 128] float32 with zero columns after the first w."""
    x = np.asarray(x, np.float32)
    out = np.zeros((x.shape[0], D), np.float32)
    out[:, :x.shape[1]] = x
    return out


def _bf16(x):
    """Padded [T, 128] values as a [1, 1, T, 128] bf16 device tensor (exact
    when the values are bf16-representable) and the same rounded values."""
    r = W.round_to_bf16(_pad(x))
    return torch.from_numpy(r).cuda().bfloat16()[None, None], r


def _run(qx, kx, vx, gx, allowed, scale=1.0):
    q, qr = _bf16(qx)
    k, kr = _bf16(kx)
    v, vr = _bf16(vx)
    g, gr = _bf16(gx)
    wf = torch.empty(eta.attn_fwd_workspace_size(q, k, v, allowed), dtype=torch.uint8, device="cuda")
    wb = torch.empty(eta.attn_bwd_workspace_size(q, k, v, allowed), dtype=torch.uint8, device="cuda")
    o, lse = eta.attn_fwd(q, k, v, allowed, scale, workspace=wf)
    assert eta.attn_get_status(wf) == 0
    dq, dk, dv, ds = eta.attn_bwd(q, k, v, o, g, lse, allowed, scale, workspace=wb)
    assert eta.attn_get_status(wb) == 0
    torch.cuda.synchronize()
    res = dict(o=to_np(o)[0, 0], lse=to_np(lse)[0, 0], dq=to_np(dq)[0, 0], dk=to_np(dk)[0, 0],
               dv=to_np(dv)[0, 0], ds=None if ds is None else ds.cpu().numpy().astype(np.float64))
    return res, (qr, kr, vr, gr)


def _oracle(rounded, allow, scale=1.0, sink=None, keep=None, rho=0.0):
    q, k, v, g = (x.astype(np.float64)[None, None] for x in rounded)
    fw = oracle.forward(q, k, v, allow, scale, sink=sink, keep=keep, rho=rho)
    bw = oracle.backward(q, k, v, g, allow, scale, sink=sink, keep=keep, rho=rho, y=fw.y)
    return fw, bw


def test_one_key_example_exact():
    e = _golden("worked_examples.json")["one_key"]
    r, _ = _run(e["q"], e["k"], e["v"], e["g"], None)
    want_y = _pad(e["y"])[0]
    assert np.array_equal(r["o"][0], want_y)
    assert np.all(r["dq"] == 0) and np.all(r["dk"] == 0)
    assert np.array_equal(r["dv"][0], _pad(e["dv"])[0])
    assert abs(r["lse"][0] - 6.0) <= 1e-5  # s = 2 * 3, one key


def test_empty_first_block_example_exact():
    e = _golden("worked_examples.json")["empty_first_block"]
    bm = torch.tensor(e["allowed"], dtype=torch.uint8, device="cuda")
    al = eta.AllowedSet(block_mask=bm, block_q=1, block_k=1)
    r, _ = _run(e["q"], e["k"], e["v"], np.zeros((2, 1)), al)
    assert np.array_equal(r["o"][:, 0], np.array([5.0, 4.0]))
    assert np.all(r["o"][:, 1:] == 0)
    assert abs(r["lse"][0]) <= 1e-6 and abs(r["lse"][1] - math.log(2)) <= 1e-5


def test_merge_orders_example():
    e = _golden("worked_examples.json")["merge_orders"]
    g = np.array([[1.0], [-0.5]])
    r1, rounded = _run(e["q"], e["k"], e["v"], g, None)
    # The keys in the other order (a different tile order): same rows of Y.
    r2, _ = _run(e["q"], np.flip(np.asarray(e["k"]), 0), np.flip(np.asarray(e["v"]), 0), g, None)
    fw, bw = _oracle(rounded, np.ones((2, 2), bool))
    for r in (r1, r2):
        assert o_excess(r["o"], fw.y[0, 0]) <= BF16_O_ABS
        assert np.abs(r["o"][:, 0] - 2.0).max() <= BF16_O_ABS  # the printed Y (with ln 2 rounded to bf16)
    for n in ("dq", "dk", "dv"):
        assert rel_fro(r1[n], getattr(bw, n)[0, 0]) <= BF16_GRAD_REL, n


def test_two_tile_trace_example():
    gd = _golden("two_tile_trace.json")
    inp = gd["inputs"]
    g = np.asarray(gd["gradient_upstream_seed"], np.float64).reshape(4, 2)
    r, rounded = _run(inp["q"], inp["k"], inp["v"], g, eta.AllowedSet(causal=True))
    fw, bw = _oracle(rounded, oracle.allowed_dense(4, 4, causal=True))
    want = np.asarray(gd["tiled_output_row3"])
    assert o_excess(r["o"][3, :2], want) <= BF16_O_ABS
    assert o_excess(r["o"], fw.y[0, 0]) <= BF16_O_ABS
    for n in ("dq", "dk", "dv"):
        assert rel_fro(r[n], getattr(bw, n)[0, 0]) <= BF16_GRAD_REL, n


def test_sink_example():
    e = _golden("worked_examples.json")["sink"]
    # Dense realisation (scale 1): row 0 scores ln p_j against z = ln p_sink;
    # a second row with zero upstream gradient adds nothing to any gradient.
    qx = [[1.0], [0.3]]
    kx = [[math.log(e["p"][0])], [math.log(e["p"][1])]]
    vx = [[e["v"][0]], [e["v"][1]]]
    gx = [[e["g"]], [0.0]]
    z = np.array([math.log(e["p_sink"])], np.float32)
    al = eta.AllowedSet(sink=torch.from_numpy(z).cuda())
    r, rounded = _run(qx, kx, vx, gx, al)
    fw, bw = _oracle(rounded, np.ones((2, 2), bool), sink=z.astype(np.float64))
    assert o_excess(r["o"], fw.y[0, 0]) <= BF16_O_ABS
    assert abs(r["ds"][0] - bw.dsink[0]) <= 1e-3
    for n in ("dq", "dk", "dv"):
        assert rel_fro(r[n], getattr(bw, n)[0, 0]) <= BF16_GRAD_REL, n
    # The printed values hold up to the bf16 rounding of ln 0.5 and ln 0.3.
    assert abs(r["o"][0, 0] - e["o"]) <= BF16_O_ABS
    assert np.abs(r["dk"][:, 0] - np.asarray(e["dS"])).max() <= 2e-2
    assert abs(r["ds"][0] - e["dz"]) <= 1e-2


def test_dropout_replay_example_exact():
    e = _golden("worked_examples.json")["dropout_replay"]
    seed = next(s for s in range(1, 1000)
                if P.dropout_keep(s, 0.5, 1, 1, 2, 2)[0, 0, 0].tolist() == [True, False])
    al = eta.AllowedSet(dropout_p=0.5, dropout_seed=seed)
    r, rounded = _run(e["q"], e["k"], e["v"], e["g"], al)
    assert r["o"][0, 0] == 2.0
    assert np.array_equal(r["dv"][:, 0], np.ravel(e["dv"]))
    keep = P.dropout_keep(seed, 0.5, 1, 1, 2, 2)
    fw, bw = _oracle(rounded, np.ones((2, 2), bool), keep=keep, rho=0.5)
    assert o_excess(r["o"], fw.y[0, 0]) <= BF16_O_ABS
    assert np.array_equal(r["dv"], bw.dv[0, 0])


def _growing_scores(dtype, seed, B, H, T, step):
    """Q, K, V, G whose scores rise from one 128-key tile to the next: every
    key of tile t carries t * step along the first coordinate, and query row i
    carries gamma_i in {-4, -2, 0, 2, 4} there, so row i's scores rise by about
    c * gamma_i * step per tile (c = 1/sqrt(128))."""
    rng = np.random.default_rng(seed)
    q = rng.standard_normal((B, H, T, D), dtype=np.float32)
    k = rng.standard_normal((B, H, T, D), dtype=np.float32)
    v = rng.standard_normal((B, H, T, D), dtype=np.float32)
    g = rng.standard_normal((B, H, T, D), dtype=np.float32)
    gamma = rng.choice(np.array([-4.0, -2.0, 0.0, 2.0, 4.0], np.float32), size=(B, H, T))
    q[..., 0] += gamma
    k[..., 0] += (np.arange(T) // 128).astype(np.float32) * step
    return tuple(W.round_to_storage(x, dtype) for x in (q, k, v, g))


@pytest.mark.parametrize("causal", [False, True])
@pytest.mark.parametrize("dtype", ["bf16", "f16"])
def test_running_max_moves_on_tensor_cores(dtype, causal):
    """With step 24 a row with gamma = 4 gains 4 * 24 / sqrt(128) = 8.5 natural
    units (12.2 in base 2, above the 2^8 threshold) per key tile, gamma = 2
    gains 6.1 in base 2 per tile (the maximum moves every second tile), and
    rows with gamma <= 0 keep their first maximum. T = 600: five key tiles,
    the last one ragged."""
    B, H, T = 1, 2, 600
    q, k, v, g = _growing_scores(dtype, 81 + causal, B, H, T, 24.0)
    tdt = torch.bfloat16 if dtype == "bf16" else torch.float16
    dev = lambda x: torch.from_numpy(x).cuda().to(tdt)  # noqa: E731
    tq, tk, tv, tg = dev(q), dev(k), dev(v), dev(g)
    al = eta.AllowedSet(causal=causal)
    scale = 1 / math.sqrt(D)
    wf = torch.empty(eta.attn_fwd_workspace_size(tq, tk, tv, al), dtype=torch.uint8, device="cuda")
    o, lse = eta.attn_fwd(tq, tk, tv, al, scale, workspace=wf)
    assert eta.attn_get_status(wf) == 0
    dq, dk, dv, _ = eta.attn_bwd(tq, tk, tv, o, tg, lse, al, scale)
    torch.cuda.synchronize()
    allow = oracle.allowed_dense(T, T, causal=causal)
    q64, k64, v64, g64 = (x.astype(np.float64) for x in (q, k, v, g))
    fw = oracle.forward(q64, k64, v64, allow, scale)
    bw = oracle.backward(q64, k64, v64, g64, allow, scale, y=fw.y)
    # The forced case: the largest score of a row lies many tiles after its
    # first key tile, far above the first tile's maximum.
    s_max_last = (scale * np.einsum("bhid,bhjd->bhij", q64[..., -128:, :], k64[..., 512:, :])).max()
    s_max_first = (scale * np.einsum("bhid,bhjd->bhij", q64[..., -128:, :], k64[..., :128, :])).max()
    assert s_max_last - s_max_first > 20.0
    assert o_excess(to_np(o), fw.y, dtype) <= BF16_O_ABS
    assert np.abs(to_np(lse) - fw.lse).max() <= 1e-3
    for name, got, want in (("dQ", dq, bw.dq), ("dK", dk, bw.dk), ("dV", dv, bw.dv)):
        assert rel_fro(to_np(got), want) <= BF16_GRAD_REL, name

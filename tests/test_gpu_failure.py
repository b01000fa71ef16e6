"""Failure detection on the device without a fault: a bounded pipeline wait
that nothing completes runs out, sets the timeout bit in the status word and
returns; the host reads the bit, and the same context then runs attention
that matches the oracle."""
import math
import time

import numpy as np
import pytest

torch = pytest.importorskip("torch")

pytestmark = pytest.mark.gpu

import exact_tiled_attention_softmax_b200 as eta  # noqa: E402
import oracle  # noqa: E402
from exact_tiled_attention_softmax_b200 import workloads as W  # noqa: E402
from tests.parity_util import to_dev  # noqa: E402


@pytest.fixture(scope="module", autouse=True)
def _cuda():
    if not torch.cuda.is_available():
        pytest.skip("no GPU")
    eta.load_library()


def test_bounded_wait_reports_timeout_and_context_stays_usable():
    ws = torch.zeros(256, dtype=torch.uint8, device="cuda")
    torch.cuda.synchronize()
    t0 = time.perf_counter()
    eta.attn_selftest_wait_timeout(ws)
    bits = eta.attn_get_status(ws)
    waited = time.perf_counter() - t0
    assert bits == eta.ATTN_DEVERR_TIMEOUT
    assert 1.9 < waited < 60.0  # the wait's limit is 2 s
    assert eta.attn_get_status(ws) == 0  # reading cleared the word

    # The context is intact: a causal bf16 case on the tensor-core path.
    rng = np.random.default_rng(91)
    shp = (1, 2, 300, 128)
    qn, kn, vn = (W.round_to_bf16(rng.standard_normal(shp, dtype=np.float32)) for _ in range(3))
    q, k, v = (to_dev(x, torch.bfloat16) for x in (qn, kn, vn))
    scale = 1 / math.sqrt(128)
    o, lse = eta.attn_fwd(q, k, v, eta.AllowedSet(causal=True), scale)
    torch.cuda.synchronize()
    ref = oracle.forward(qn.astype(np.float64), kn.astype(np.float64), vn.astype(np.float64),
                         oracle.allowed_dense(300, 300, causal=True), scale)
    assert np.abs(o.float().cpu().numpy() - ref.y).max() <= 1e-2
    assert np.abs(lse.cpu().numpy() - ref.lse).max() <= 1e-3

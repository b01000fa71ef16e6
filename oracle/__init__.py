"""Float64 CPU oracle for exact tiled masked softmax attention.

TEST INFRASTRUCTURE ONLY. The test suite, the smoke check and the benchmark's
CPU-baseline leg are the only code allowed to import this package. The CUDA
library never imports, links or executes anything here, and this package
imports nothing from the library: both sides receive the same seeded inputs
from the library's input-generator module, which holds no attention
arithmetic.

Modules
-------
attention  dense masked attention, its analytic VJP, the shared-KV top-k
           variant, the running-summary recurrence with trace cards, and the
           block-summary merge, and the LSE conventions (sink-inclusive,
           KV-only with its logaddexp combination, base-2 scaled form).
philox     Philox4x32-10 (Salmon et al., SC'11) and the dropout keep-mask
           convention built on it.
"""
from .attention import (  # noqa: F401
    BackwardResult, ForwardResult, TileCard, allowed_dense, backward,
    block_summary, combine_lse, forward, kv_only_lse, merge_summaries,
    scaled_lse, tiled_forward, topk_allowed, topk_backward, topk_dsink,
    topk_forward, topk_kv_only_lse,
)
from .philox import dropout_keep, keep_threshold, philox4x32  # noqa: F401

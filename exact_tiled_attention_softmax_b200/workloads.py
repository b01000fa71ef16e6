"""Seeded synthetic inputs shared by the CUDA path, its tests and the oracle.

This module holds no attention arithmetic: it only draws random tensors,
masks and index lists with NumPy's PCG64 generator and rounds them to the
storage dtype. Both the library's callers and the float64 oracle consume
exactly these arrays, so a parity test compares the two implementations on
identical values.

Workloads (sizes named by what they are):
  tiny_causal_fp32   B=1 H=1 T=64 d=dv=16, fp32, c=1/4, causal
  causal_2k          B=4 H=16 T=2048 d=dv=128, bf16, causal
  window_block_8k    B=1 H=32 T=8192 d=dv=128, bf16, sliding window 1024
                     intersected with a 64x64 Bernoulli(0.5) grid of 128x128
                     blocks whose diagonal is kept
  gqa_dropout_16k    B=2 Hq=32 Hkv=8 T=16384 d=dv=128, bf16, causal,
                     dropout rho=0.1
  topk_shared_kv     Tq=4096 Tkv=32768 H=64 Dqk=576 Dv=512, bf16, top-k lists
                     of distinct indices <= the causal position with lengths
                     uniform in [1024, 2048], per-head sink ~ N(0,1)
  causal_8k          B=1 H=32 T=8192 d=dv=128, bf16, causal (throughput case)
"""
from __future__ import annotations

import math
from dataclasses import dataclass

import numpy as np


def round_to_fp16(x: np.ndarray) -> np.ndarray:
    """Round float32 values to the nearest IEEE half (ties to even), returned
    as float32."""
    return np.ascontiguousarray(x, dtype=np.float32).astype(np.float16).astype(np.float32)


def round_to_storage(x: np.ndarray, dtype: str) -> np.ndarray:
    """Inputs as the library will store them: "bf16", "f16" or "f32"."""
    if dtype == "bf16":
        return round_to_bf16(x)
    if dtype == "f16":
        return round_to_fp16(x)
    return np.ascontiguousarray(x, dtype=np.float32)


def round_to_bf16(x: np.ndarray) -> np.ndarray:
    """Round float32 values to the nearest bfloat16 (ties to even), returned
    as float32 so that both sides can read them."""
    x = np.ascontiguousarray(x, dtype=np.float32)
    bits = x.view(np.uint32).astype(np.uint64)
    lsb = (bits >> np.uint64(16)) & np.uint64(1)
    rounded = (bits + np.uint64(0x7FFF) + lsb) & np.uint64(0xFFFF0000)
    return rounded.astype(np.uint32).view(np.float32)


@dataclass
class DenseCase:
    """A dense-layout problem: Q [B,Hq,T,d], K [B,Hkv,T,d], V [B,Hkv,T,dv]."""
    name: str
    B: int
    Hq: int
    Hkv: int
    T: int
    d: int
    dv: int
    dtype: str                 # "f32" or "bf16"
    scale: float
    causal: bool = True
    window_left: int = 0
    block_size: int = 0        # 0 = no explicit block mask
    block_p_keep: float = 0.5
    dropout_p: float = 0.0
    seed: int = 0
    mask_seed: int = 0
    dropout_seed: int = 0
    with_sink: bool = False

    @property
    def flops_per_pair(self) -> int:
        """fwd 2d + 2dv, bwd 6d + 4dv (S, PV; S again, dP, dV, dQ, dK)."""
        return 2 * self.d + 2 * self.dv + 6 * self.d + 4 * self.dv


@dataclass
class TopkCase:
    name: str
    Tq: int
    Tkv: int
    H: int
    Dqk: int
    Dv: int
    topk: int
    len_lo: int
    len_hi: int
    scale: float
    seed: int = 0
    idx_seed: int = 0
    with_sink: bool = True

    @property
    def flops_per_pair(self) -> int:
        return 2 * self.Dqk + 2 * self.Dv + 6 * self.Dqk + 4 * self.Dv


WORKLOADS = {
    "tiny_causal_fp32": DenseCase("tiny_causal_fp32", 1, 1, 1, 64, 16, 16, "f32",
                                  0.25, causal=True, seed=1001),
    "causal_2k": DenseCase("causal_2k", 4, 16, 16, 2048, 128, 128, "bf16",
                           1 / math.sqrt(128), causal=True, seed=1002),
    "window_block_8k": DenseCase("window_block_8k", 1, 32, 32, 8192, 128, 128,
                                 "bf16", 1 / math.sqrt(128), causal=True,
                                 window_left=1024, block_size=128,
                                 block_p_keep=0.5, seed=1003, mask_seed=2003),
    "gqa_dropout_16k": DenseCase("gqa_dropout_16k", 2, 32, 8, 16384, 128, 128,
                                 "bf16", 1 / math.sqrt(128), causal=True,
                                 dropout_p=0.1, seed=1004, dropout_seed=1004),
    "causal_8k": DenseCase("causal_8k", 1, 32, 32, 8192, 128, 128, "bf16",
                           1 / math.sqrt(128), causal=True, seed=1006),
}

TOPK_WORKLOADS = {
    "topk_shared_kv": TopkCase("topk_shared_kv", 4096, 32768, 64, 576, 512, 2048,
                               1024, 2048, 1 / 24, seed=1005, idx_seed=2005),
}


def _normal(rng: np.random.Generator, shape, dtype: str) -> np.ndarray:
    x = rng.standard_normal(size=shape, dtype=np.float32)
    return round_to_bf16(x) if dtype == "bf16" else x


def dense_inputs(case: DenseCase):
    """Q, K, V, dO as float32 arrays holding exactly representable values of
    the case's storage dtype (standard normal draws)."""
    rng = np.random.default_rng(case.seed)
    q = _normal(rng, (case.B, case.Hq, case.T, case.d), case.dtype)
    k = _normal(rng, (case.B, case.Hkv, case.T, case.d), case.dtype)
    v = _normal(rng, (case.B, case.Hkv, case.T, case.dv), case.dtype)
    do = _normal(rng, (case.B, case.Hq, case.T, case.dv), case.dtype)
    return q, k, v, do


def sink_values(n_heads: int, seed: int) -> np.ndarray:
    return np.random.default_rng(seed + 7).standard_normal(n_heads).astype(np.float32)


def block_mask(case: DenseCase) -> np.ndarray | None:
    """uint8 [nb, nb] Bernoulli(p_keep) grid with its diagonal set, shared by
    every batch row and head; None when the case has no explicit block mask."""
    if not case.block_size:
        return None
    nb = (case.T + case.block_size - 1) // case.block_size
    rng = np.random.default_rng(case.mask_seed)
    bm = (rng.random((nb, nb)) < case.block_p_keep).astype(np.uint8)
    np.fill_diagonal(bm, 1)
    return bm


def topk_inputs(case: TopkCase):
    """Q [Tq,H,Dqk], KV [Tkv,Dqk], dO [Tq,H,Dv] (bf16 values as float32),
    idx int32 [Tq,topk] (distinct indices <= Tkv-Tq+t, -1 padded),
    length int32 [Tq] uniform in [len_lo, len_hi], sink float32 [H]."""
    rng = np.random.default_rng(case.seed)
    q = _normal(rng, (case.Tq, case.H, case.Dqk), "bf16")
    kv = _normal(rng, (case.Tkv, case.Dqk), "bf16")
    do = _normal(rng, (case.Tq, case.H, case.Dv), "bf16")
    idx, length = topk_lists(case.Tq, case.Tkv, case.topk, case.len_lo,
                             case.len_hi, case.idx_seed)
    sink = sink_values(case.H, case.seed) if case.with_sink else None
    return q, kv, do, idx, length, sink


def topk_lists(t_q: int, t_kv: int, topk: int, len_lo: int, len_hi: int, seed: int):
    """Distinct uniform indices from [0, t_kv - t_q + t] for query token t."""
    rng = np.random.default_rng(seed)
    idx = np.full((t_q, topk), -1, dtype=np.int32)
    length = np.empty(t_q, dtype=np.int32)
    for t in range(t_q):
        pos = t_kv - t_q + t
        n = min(int(rng.integers(len_lo, len_hi + 1)), pos + 1, topk)
        idx[t, :n] = rng.choice(pos + 1, size=n, replace=False)
        length[t] = n
    return idx, length

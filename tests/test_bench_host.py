"""bench.py's host-side accounting on CPU: the allowed-pair count that the
TFLOP/s figures divide by (checked against the oracle's allowed sets on small
shapes and against the causal closed form at the headline size), the
whole-job throughput arithmetic, and the rule that a recorded DRAM traffic
figure is reported only for the kernel source it was captured from."""
import dataclasses
import json
import os
import sys

import numpy as np
import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)

import bench  # noqa: E402
import oracle  # noqa: E402
from exact_tiled_attention_softmax_b200 import workloads as W  # noqa: E402


@pytest.mark.parametrize("kind", ["causal", "window", "window_block", "noncausal"])
def test_allowed_pairs_equal_the_oracle_sets(kind):
    base = W.WORKLOADS["window_block_8k"]
    case = dataclasses.replace(base, B=2, Hq=3, Hkv=3, T=300, block_size=0, window_left=0, causal=True)
    if kind == "window":
        case = dataclasses.replace(case, window_left=70)
    elif kind == "window_block":
        case = dataclasses.replace(case, window_left=90, block_size=64)
    elif kind == "noncausal":
        case = dataclasses.replace(case, causal=False)
    bm = W.block_mask(case)
    allow = oracle.allowed_dense(case.T, case.T, causal=case.causal, window_left=case.window_left,
                                 block_mask=bm, block_q=case.block_size or 1, block_k=case.block_size or 1)
    expect = int(np.broadcast_to(allow, (case.B, case.Hq, case.T, case.T)).sum())
    assert bench.allowed_pairs(case) == expect


def test_headline_pairs_and_throughput_arithmetic():
    case = W.WORKLOADS["causal_8k"]
    assert bench.allowed_pairs(case) == case.B * case.Hq * case.T * (case.T + 1) // 2
    # 2 ranks x 10 steps x 1.5 TFLOP over a 30 ms slowest-rank time
    assert abs(bench.whole_job_tflops(2, 1.5e12, 10, 30.0) - 1000.0) < 1e-9
    assert bench.max_over_ranks(12.5, 1) == 12.5


def test_recorded_traffic_only_for_the_captured_source(tmp_path, monkeypatch):
    rec = json.load(open(os.path.join(ROOT, "profiles", "dram_traffic.json")))
    entry = rec["bwd_kernel"]["causal_8k"]
    got = bench.recorded_traffic("bwd_kernel", "causal_8k")
    import hashlib
    digest = hashlib.sha256(open(os.path.join(ROOT, entry["source"]), "rb").read()).hexdigest()
    if digest == entry["source_sha256"]:
        assert got == entry["dram_bytes_read"] + entry["dram_bytes_write"]
    else:
        assert got is None
    # A copy of the tree whose kernel source differs reports no traffic.
    (tmp_path / "profiles").mkdir()
    bad = dict(rec)
    bad["bwd_kernel"] = {"causal_8k": dict(entry, source_sha256="0" * 64)}
    (tmp_path / "profiles" / "dram_traffic.json").write_text(json.dumps(bad))
    src = tmp_path / entry["source"]
    src.parent.mkdir(parents=True)
    src.write_text("// not the captured kernel\n")
    monkeypatch.setattr(bench, "ROOT", str(tmp_path))
    assert bench.recorded_traffic("bwd_kernel", "causal_8k") is None


def test_deterministic_reverse_has_no_borrowed_traffic():
    # The deterministic reverse launches the key-centric bwd_kernel without its
    # dQ product; the capture of the fused instantiation must not stand in for it.
    rec = json.load(open(os.path.join(ROOT, "profiles", "dram_traffic.json")))
    if "causal_8k_deterministic" not in rec.get("bwd_kernel", {}):
        assert bench.recorded_traffic("bwd_kernel", "causal_8k_deterministic") is None


def test_conventional_count_is_the_dense_half_for_causal_only():
    for name in ("causal_8k", "causal_2k", "gqa_dropout_16k"):
        case = W.WORKLOADS[name]
        conv = bench.conventional_flops(case)
        alg = bench.allowed_pairs(case) * (8 * case.d + 6 * case.dv)
        # T^2/2 pairs per head against the algorithmic T(T+1)/2
        assert conv * (case.T + 1) == alg * case.T
    assert bench.conventional_flops(W.WORKLOADS["window_block_8k"]) is None
    r = bench.conventional_rate({"conventional_flops_per_step": 900}, 830.0, 1000.0)
    assert abs(r["tflops"] - 747.0) < 1e-9 and r["flops_per_step"] == 900
    assert bench.conventional_rate({}, 830.0, 1000.0) is None


def test_topk_gather_rate():
    got = bench.topk_gather_rate({"gathered_bytes_per_pass": 7_000_000_000}, 3.5)
    assert abs(got["fwd_gbs"] - 2000.0) < 1e-9
    assert bench.topk_gather_rate({}, 3.5) is None


def test_both_arms_name_the_workload_alike():
    case = W.WORKLOADS["causal_8k"]
    cfg = bench.dense_config(case)
    assert {"workload", "B", "Hq", "Hkv", "T", "d", "dv", "mask"} <= set(cfg)
    assert cfg["workload"] == "causal_8k" and cfg["mask"] == "causal"
    assert cfg["conventional_flops_per_step"] == bench.conventional_flops(case)
    assert "reverse" in bench.dense_config(case, deterministic=True)
    # 1.924 TFLOP at 0.0192 TFLOP/s is about 100 s per full step
    flops = bench.allowed_pairs(case) * case.flops_per_pair
    assert abs(bench.reference_ms_per_step(flops, flops / 1e14) - 1e5) < 1e-6
    assert bench.reference_ms_per_step(flops, 0.0) is None


def test_reference_arm_runs_on_rank_zero_only(capsys):
    import argparse
    args = argparse.Namespace(steps=1, warmup=0)
    # Any rank but 0 leaves at once, with nothing printed and no oracle work.
    assert bench.run_reference(args, W.WORKLOADS["causal_8k"], rank=1, world=2) is None
    assert capsys.readouterr().out == ""

"""Throughput of exact tiled masked softmax attention, forward + reverse, on B200.

Default workload (causal_8k): B=1, H=32, T=8192, d=dv=128, bf16, causal.
One step = attn_fwd + attn_bwd over one batch already resident in HBM.
value = algorithmic TFLOP/s over all ranks: allowed pairs x (2d + 2dv + 6d + 4dv)
(= 1792 flops per pair at d = dv = 128), divided by the max over ranks of the
summed CUDA-event step times. L2 is flushed (a 256 MB write) before every
step, outside the timed events.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--workload NAME]
    python bench.py --impl reference ...   # the float64 CPU oracle on a sample

Multi-GPU runs are independent replicas (the dense path has no exchange
step): each rank runs the same workload; torch.distributed is used only for
the barrier and the max-over-ranks of the device time.
"""
from __future__ import annotations

import argparse
import json
import math
import os
import statistics
import subprocess
import sys
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

from exact_tiled_attention_softmax_b200 import workloads as W  # noqa: E402

METRIC = "attention fwd+bwd TFLOP/s (bf16) and % of B200 dense BF16 tensor peak"
UNIT = "TFLOP/s"
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}


def load_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            return json.load(f), "measured"
    except OSError:
        return FALLBACK_PEAKS, "fallback"


def allowed_pairs(case: W.DenseCase) -> int:
    """Sum over (b, h, i) of |A_i|: causal / window in closed form, a block
    mask counted block pair by block pair."""
    T = case.T
    i = np.arange(T, dtype=np.int64)
    lo = np.zeros(T, np.int64) if not case.window_left else np.maximum(0, i - case.window_left + 1)
    hi = i if case.causal else np.full(T, T - 1, np.int64)
    if not case.block_size:
        return int(case.B * case.Hq * np.sum(hi - lo + 1))
    bm = W.block_mask(case)
    bs = case.block_size
    total = 0
    for kb in range(bm.shape[1]):
        c0, c1 = kb * bs, min(T, (kb + 1) * bs) - 1
        rows = np.nonzero(np.repeat(bm[:, kb], bs)[:T])[0]
        cnt = np.minimum(hi[rows], c1) - np.maximum(lo[rows], c0) + 1
        total += int(np.sum(np.maximum(cnt, 0)))
    return int(case.B * case.Hq * total)


def conventional_flops(case: W.DenseCase):
    """The FlashAttention-style count for a purely causal dense workload: the
    dense count B Hq T^2 (8d + 6dv) halved, i.e. T^2/2 pairs per head where
    the algorithmic count has T(T+1)/2. None for other allowed sets, where
    that convention has no agreed meaning."""
    if not case.causal or case.window_left or case.block_size:
        return None
    return case.B * case.Hq * case.T * case.T * (8 * case.d + 6 * case.dv) // 2


def conventional_rate(config: dict, value: float, flops_step: float):
    """`value` (algorithmic TFLOP/s) restated under the conventional count
    recorded in `config`, or None when the workload has none."""
    conv = config.get("conventional_flops_per_step")
    if not conv:
        return None
    return {"flops_per_step": conv, "tflops": value * conv / flops_step,
            "rule": "dense count halved for causal (T^2/2 pairs per head, not T(T+1)/2)"}


def topk_gather_rate(config: dict, fwd_kernel_ms: float):
    """Bytes of listed KV rows the top-k forward gathers (every listed row of
    Dqk 16-bit values, once per query token) and their rate over the forward
    kernel's time; None for dense workloads."""
    nbytes = config.get("gathered_bytes_per_pass")
    if not nbytes:
        return None
    return {"bytes_per_pass": nbytes, "fwd_gbs": nbytes / (fwd_kernel_ms / 1e3) / 1e9}


def fp32_alu_peak_tflops(sm_mhz: float) -> float:
    """Dense fp32 FFMA rate: 148 SMs x 128 lanes x 2 flops x clock."""
    return 148 * 128 * 2 * sm_mhz * 1e6 / 1e12


class ClockSampler:
    """nvidia-smi clocks and throttle reasons, sampled every 20 ms; summary()
    keeps the samples whose timestamps fall inside the timed window."""

    FIELDS = ("timestamp,index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index: int):
        self.gpu = gpu_index
        self.proc = None
        self.lines = []
        self.window = None

    def start(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--id={self.gpu}", f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits",
                 "-lms", "20"], stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
        except OSError:
            self.proc = None
        return self

    def stop(self):
        if self.proc is not None:
            self.proc.terminate()
            try:
                out, _ = self.proc.communicate(timeout=5)
            except subprocess.TimeoutExpired:
                self.proc.kill()
                out, _ = self.proc.communicate()
            self.lines = [ln for ln in out.splitlines() if ln.strip()]

    @staticmethod
    def _epoch(stamp: str):
        import datetime
        for fmt in ("%Y/%m/%d %H:%M:%S.%f", "%Y/%m/%d %H:%M:%S"):
            try:
                return datetime.datetime.strptime(stamp, fmt).timestamp()
            except ValueError:
                continue
        return None

    def summary(self):
        rows = [[c.strip() for c in ln.split(",")] for ln in self.lines]
        rows = [r for r in rows if len(r) >= 10]
        inside = rows
        where = "all samples"
        if self.window and rows:
            t0, t1 = self.window
            sel = [r for r in rows if (lambda e: e is not None and t0 - 0.05 <= e <= t1 + 0.05)(self._epoch(r[0]))]
            if sel:
                inside, where = sel, "timed window"
        if not inside:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["unsampled"], "samples": 0}
        num = lambda x: x.replace(".", "", 1).isdigit()
        sm = [float(r[2]) for r in inside if num(r[2])]
        mx = [float(r[3]) for r in inside if num(r[3])]
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        reasons = sorted({names[k] for r in inside for k in range(4) if r[6 + k].lower() == "active"})
        return {"sm_mhz": statistics.median(sm) if sm else None, "sm_max_mhz": max(mx) if mx else None,
                "reasons": reasons, "samples": len(inside), "sampled": where}


def recorded_traffic(kernel: str, workload: str):
    """DRAM bytes (read + write) per launch of `kernel` from the ncu capture
    recorded in profiles/dram_traffic.json, or None when the kernel source
    has changed since that capture (its SHA-256 no longer matches)."""
    import hashlib
    try:
        with open(os.path.join(ROOT, "profiles", "dram_traffic.json")) as f:
            rec = json.load(f)[kernel][workload]
        with open(os.path.join(ROOT, rec["source"]), "rb") as f:
            digest = hashlib.sha256(f.read()).hexdigest()
    except (OSError, KeyError, ValueError):
        return None
    if digest != rec["source_sha256"]:
        return None
    return rec["dram_bytes_read"] + rec["dram_bytes_write"]


def cpu_baseline(case: W.DenseCase, budget_s: float = 12.0):
    """The float64 oracle, as it stands, on a bounded sample of the workload:
    whole (b, h) slices of the same shape, one after another, until the time
    budget is spent; scaled to TFLOP/s by the algorithmic flops of the slices
    it finished."""
    import oracle
    rng = np.random.default_rng(case.seed)
    T, d = case.T, case.d
    allow = oracle.allowed_dense(T, T, causal=case.causal, window_left=case.window_left)
    per_head_pairs = int(allow.sum())
    q = W.round_to_bf16(rng.standard_normal((1, 1, T, d), dtype=np.float32)).astype(np.float64)
    k = W.round_to_bf16(rng.standard_normal((1, 1, T, d), dtype=np.float32)).astype(np.float64)
    v = W.round_to_bf16(rng.standard_normal((1, 1, T, d), dtype=np.float32)).astype(np.float64)
    g = W.round_to_bf16(rng.standard_normal((1, 1, T, d), dtype=np.float32)).astype(np.float64)
    done, t0 = 0, time.perf_counter()
    while True:
        fw = oracle.forward(q, k, v, allow, case.scale)
        oracle.backward(q, k, v, g, allow, case.scale, y=fw.y)
        done += 1
        el = time.perf_counter() - t0
        if el >= budget_s:
            break
    flops = done * per_head_pairs * case.flops_per_pair
    return {"value": flops / el / 1e12, "unit": UNIT, "cores": os.cpu_count(), "kind": "oracle",
            "sample": f"{done} (b,h) slice(s) of B=1 H=1 T={T} d={d} causal fwd+bwd in float64 NumPy, "
                      f"{el:.1f} s; oracle BLAS threads = all host cores"}


def reference_ms_per_step(flops_step: float, tflops: float):
    """Time one full step would take at the rate the sampled slices ran."""
    return flops_step / (tflops * 1e12) * 1e3 if tflops > 0 else None


def run_reference(args, case, rank, world):
    """--impl reference: the oracle is the reference arm (rank 0 only)."""
    if rank != 0:
        return
    vals = []
    for _ in range(max(args.warmup, 0)):
        cpu_baseline(case, budget_s=1.0)
    for _ in range(args.steps):
        vals.append(cpu_baseline(case, budget_s=max(2.0, 60.0 / max(args.steps, 1)))["value"])
    v = statistics.median(vals)
    cb = cpu_baseline(case, budget_s=1.0)
    cb["value"] = v
    pairs = allowed_pairs(case)
    config = dense_config(case)
    config.update({"allowed_pairs": pairs, "flops_per_pair": case.flops_per_pair})
    line = {"metric": METRIC, "value": v, "unit": UNIT, "impl": "reference", "n_gpus": world,
            "steps": args.steps, "warmup": args.warmup,
            "ms_per_step": reference_ms_per_step(pairs * case.flops_per_pair, v),
            "ms_per_step_basis": "the full workload's flops at the sampled slices' rate",
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
            "data": "synthetic", "config": config,
            "cpu_baseline": cb,
            "e2e": {"value": v, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)


def max_over_ranks(ms: float, world: int, device=None) -> float:
    """The slowest rank's time: every rank contributes its device-timed total
    and all of them receive the maximum (one all-reduce, identical on every
    rank). Replicas run independent problems, so the whole job ends when the
    slowest one does."""
    if world <= 1:
        return ms
    import torch
    import torch.distributed as dist
    t = torch.tensor([float(ms)], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def whole_job_tflops(world: int, flops_per_rank_step: float, steps: int, max_ms: float) -> float:
    """Whole-job throughput: the work every rank did over the slowest rank's time."""
    return world * flops_per_rank_step * steps / (max_ms / 1e3) / 1e12


class Problem:
    """One workload on the device: the fwd and bwd calls through the public
    binding, their inputs (for the end-to-end copies) and outputs, and the
    algorithmic work per step."""

    def __init__(self, name, pairs, fwd_fpp, bwd_fpp, inputs, outputs, fwd, bwd, config, bound, launches):
        self.name, self.pairs, self.fwd_fpp, self.bwd_fpp = name, pairs, fwd_fpp, bwd_fpp
        self.inputs, self.outputs, self.fwd, self.bwd = inputs, outputs, fwd, bwd
        self.config, self.bound, self.launches = config, bound, launches


def dense_config(case: W.DenseCase, deterministic: bool = False) -> dict:
    """The `config` object both arms print for a dense workload."""
    mask = "causal" + (f" & window {case.window_left}" if case.window_left else "") + \
        (f" & {case.block_size}-blocks p={case.block_p_keep}" if case.block_size else "") + \
        (f", dropout {case.dropout_p}" if case.dropout_p else "")
    config = {"workload": case.name, "B": case.B, "Hq": case.Hq, "Hkv": case.Hkv, "T": case.T, "d": case.d,
              "dv": case.dv, "mask": mask}
    if deterministic:
        config["reverse"] = "deterministic (dQ from the query-centric pass)"
    if conventional_flops(case):
        config["conventional_flops_per_step"] = conventional_flops(case)
    return config


def dense_problem(case: W.DenseCase, dev, torch, eta, deterministic: bool = False) -> Problem:
    q, k, v, g = W.dense_inputs(case)
    tq, tk, tv, tg = (torch.from_numpy(x).to(dev).to(torch.bfloat16) for x in (q, k, v, g))
    bm = W.block_mask(case)
    allowed = eta.AllowedSet(causal=case.causal, window_left=case.window_left,
                             block_mask=torch.from_numpy(bm).to(dev) if bm is not None else None,
                             block_q=case.block_size or 128, block_k=case.block_size or 128,
                             dropout_p=case.dropout_p, dropout_seed=case.dropout_seed,
                             deterministic=deterministic)
    o = torch.empty_like(tq)
    lse = torch.empty(tq.shape[:-1], dtype=torch.float32, device=dev)
    dq, dk, dv = torch.empty_like(tq), torch.empty_like(tk), torch.empty_like(tv)
    ws_f = torch.empty(eta.attn_fwd_workspace_size(tq, tk, tv, allowed), dtype=torch.uint8, device=dev)
    ws_b = torch.empty(eta.attn_bwd_workspace_size(tq, tk, tv, allowed), dtype=torch.uint8, device=dev)
    config = dense_config(case, deterministic)
    return Problem(case.name, allowed_pairs(case), 2 * case.d + 2 * case.dv, 6 * case.d + 4 * case.dv,
                   [tq, tk, tv, tg], [dq, dk, dv],
                   lambda: eta.attn_fwd(tq, tk, tv, allowed, case.scale, out=o, lse=lse, workspace=ws_f),
                   lambda: eta.attn_bwd(tq, tk, tv, o, tg, lse, allowed, case.scale, dq=dq, dk=dk, dv=dv,
                                        workspace=ws_b),
                   config, "tensor",
                   # fwd_kernel; prepare, bwd_kernel, dq_finish (or the query-centric dQ kernel);
                   # plus a tile-class pass per call
                   # when a block mask is present
                   4 + (2 if bm is not None else 0))


def topk_problem(case: W.TopkCase, dev, torch, eta, deterministic: bool = False) -> Problem:
    q, kv, g, idx, ln, sink = W.topk_inputs(case)
    tq, tkv, tg = (torch.from_numpy(x).to(dev).to(torch.bfloat16) for x in (q, kv, g))
    allowed = eta.AllowedSet(topk_idxs=torch.from_numpy(idx).to(dev), topk_length=torch.from_numpy(ln).to(dev),
                             sink=torch.from_numpy(sink).to(dev), deterministic=deterministic)
    tv = tkv[:, :case.Dv]
    o = torch.empty((case.Tq, case.H, case.Dv), dtype=torch.bfloat16, device=dev)
    lse = torch.empty((case.Tq, case.H), dtype=torch.float32, device=dev)
    dq = torch.empty_like(tq)
    dkv = torch.empty_like(tkv)
    dsink = torch.empty(case.H, dtype=torch.float32, device=dev)
    ws_f = torch.empty(eta.attn_fwd_workspace_size(tq, tkv, tv, allowed), dtype=torch.uint8, device=dev)
    ws_b = torch.empty(eta.attn_bwd_workspace_size(tq, tkv, tv, allowed), dtype=torch.uint8, device=dev)
    config = {"workload": case.name, "Tq": case.Tq, "Tkv": case.Tkv, "H": case.H, "Dqk": case.Dqk, "Dv": case.Dv,
              "mask": f"top-k lists, lengths U[{case.len_lo},{case.len_hi}], sink",
              "gathered_bytes_per_pass": int(ln.astype(np.int64).sum()) * case.Dqk * 2,
              "reverse": ("deterministic (dKV summed in 32.32 fixed point)" if deterministic
                          else "dKV summed with fp32 atomics")}
    return Problem(case.name, case.H * int(ln.astype(np.int64).sum()), 2 * case.Dqk + 2 * case.Dv,
                   6 * case.Dqk + 4 * case.Dv, [tq, tkv, tg], [dq, dkv],
                   lambda: eta.attn_fwd(tq, tkv, tv, allowed, case.scale, out=o, lse=lse, workspace=ws_f),
                   lambda: eta.attn_bwd(tq, tkv, tv, o, tg, lse, allowed, case.scale, dq=dq, dk=dkv, dv=None,
                                        dsink=dsink, workspace=ws_b),
                   config, "tensor",
                   # forward; delta, dQ + G/P, dKV contributions, dKV cast, dSink
                   6)


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--sustained-steps", type=int, default=-1,
                    help="back-to-back steps after the timed ones, the last half reported as 'sustained' "
                         "(-1: about 0.6 s worth, 0: skip)")
    ap.add_argument("--workload", default="causal_8k",
                    choices=["causal_8k", "causal_2k", "window_block_8k", "gqa_dropout_16k", "topk_shared_kv"])
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--topk-tokens", type=int, default=0,
                    help="top-k workload with only this many query tokens (a smaller case for ncu)")
    ap.add_argument("--deterministic", action="store_true",
                    help="bitwise reproducible reverse pass (dense dQ from a query-centric pass; top-k dKV in fixed point)")
    args = ap.parse_args()

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if args.impl == "reference":
        if args.workload not in ("causal_8k", "causal_2k"):
            raise SystemExit("--impl reference times the oracle on the causal workloads")
        run_reference(args, W.WORKLOADS[args.workload], rank, world)
        return

    import torch
    import torch.distributed as dist

    import exact_tiled_attention_softmax_b200 as eta

    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    if world > 1:
        import datetime
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120), device_id=dev)
    eta.load_library()

    def make_problem():
        if args.workload in W.TOPK_WORKLOADS:
            case = W.TOPK_WORKLOADS[args.workload]
            if args.topk_tokens:  # the same lists and shapes for fewer query tokens (profiling captures)
                import dataclasses
                case = dataclasses.replace(case, Tq=args.topk_tokens)
            return topk_problem(case, dev, torch, eta, args.deterministic)
        return dense_problem(W.WORKLOADS[args.workload], dev, torch, eta, args.deterministic)

    prob = make_problem()
    flush = torch.empty(256 * 1024 * 1024, dtype=torch.uint8, device=dev)
    stream = torch.cuda.current_stream()

    def step():
        prob.fwd()
        prob.bwd()

    clk = ClockSampler(local).start()
    time.sleep(0.5)  # nvidia-smi needs a moment before its first sample
    for _ in range(max(args.warmup, 3)):
        step()
    torch.cuda.synchronize()

    n_ev = args.steps
    ev = [tuple(torch.cuda.Event(enable_timing=True) for _ in range(3)) for _ in range(n_ev)]
    # Events around the main kernel of each call, recorded by the library
    # itself on the launching stream.
    kev = [tuple(torch.cuda.Event(enable_timing=True) for _ in range(4)) for _ in range(n_ev)]
    for evs in kev:
        for e in evs:
            e.record(stream)
    torch.cuda.synchronize()
    if world > 1:
        dist.barrier()
    torch.cuda.synchronize()
    t_wall0 = time.time()
    for s in range(n_ev):
        flush.fill_(s & 0xFF)
        e0, e1, e2 = ev[s]
        k0, k1, k2, k3 = kev[s]
        e0.record(stream)
        eta.attn_set_kernel_events(k0, k1)
        prob.fwd()
        e1.record(stream)
        eta.attn_set_kernel_events(k2, k3)
        prob.bwd()
        e2.record(stream)
    torch.cuda.synchronize()
    t_wall1 = time.time()
    clk.stop()
    clk.window = (t_wall0, t_wall1)
    if world > 1:
        dist.barrier()
    t_fwd = [a.elapsed_time(b) for a, b, _ in ev]
    t_bwd = [b.elapsed_time(c) for _, b, c in ev]
    t_fwd_kernel = [k0.elapsed_time(k1) for k0, k1, _, _ in kev]
    t_bwd_kernel = [k2.elapsed_time(k3) for _, _, k2, k3 in kev]
    total_ms = max_over_ranks(sum(f + b for f, b in zip(t_fwd, t_bwd)), world, dev)
    ms_step = total_ms / n_ev
    pairs = prob.pairs
    flops_step = pairs * (prob.fwd_fpp + prob.bwd_fpp)
    value = whole_job_tflops(world, flops_step, n_ev, total_ms)

    # End to end through the public API, pipelined as an input loader would
    # run it: every step copies its inputs in from pinned host memory on one
    # stream while the previous step computes, and copies its gradients out
    # on a third stream. Two device copies of the problem alternate; a step
    # reuses one only after the step two back has finished computing and its
    # results have been read out.
    probs = [prob, make_problem()]
    hosts_in = [x.to("cpu").pin_memory() for x in prob.inputs]
    hosts_out = [torch.empty(x.shape, dtype=x.dtype, pin_memory=True) for x in prob.outputs]
    h2d = sum(x.numel() * x.element_size() for x in hosts_in)
    d2h = sum(x.numel() * x.element_size() for x in hosts_out)
    s_in, s_out = torch.cuda.Stream(device=dev), torch.cuda.Stream(device=dev)

    def pipelined(n_steps):
        ev = lambda: torch.cuda.Event(enable_timing=True)  # noqa: E731
        ev_in, ev_comp, ev_out = [], [], []
        start, end = ev(), ev()
        start.record(s_in)
        for s in range(n_steps):
            p = probs[s % 2]
            with torch.cuda.stream(s_in):
                if s >= 2:
                    s_in.wait_event(ev_comp[s - 2])  # its inputs are no longer read
                for d_, h_ in zip(p.inputs, hosts_in):
                    d_.copy_(h_, non_blocking=True)
                ev_in.append(ev())
                ev_in[-1].record(s_in)
            stream.wait_event(ev_in[s])
            if s >= 2:
                stream.wait_event(ev_out[s - 2])  # its outputs have been read out
            flush.fill_(s & 0xFF)
            p.fwd()
            p.bwd()
            ev_comp.append(ev())
            ev_comp[-1].record(stream)
            with torch.cuda.stream(s_out):
                s_out.wait_event(ev_comp[s])
                for h_, d_ in zip(hosts_out, p.outputs):
                    h_.copy_(d_, non_blocking=True)
                ev_out.append(ev())
                ev_out[-1].record(s_out)
        end.record(s_out)
        torch.cuda.synchronize()
        return start.elapsed_time(end)

    pipelined(3)  # warm-up
    e2e_ms = [pipelined(n_ev)]
    e2e_total = max_over_ranks(sum(e2e_ms), world, dev)
    e2e_value = whole_job_tflops(world, flops_step, n_ev, e2e_total)

    # Sustained load: the same step back to back for about half a second.
    # Under full load the B200 lowers its clock after some tens of
    # milliseconds (the power limit), faster than nvidia-smi's samples show;
    # the timed steps above fit inside that window at the default count. The
    # second half of this run is reported apart, against the sustained peak.
    sustained = None
    n_sus = args.sustained_steps if args.sustained_steps >= 0 else max(40, min(400, int(600.0 / max(ms_step, 1e-3))))
    if n_sus > 0:
        sev = [tuple(torch.cuda.Event(enable_timing=True) for _ in range(4)) for _ in range(n_sus)]
        torch.cuda.synchronize()
        for s_ in range(n_sus):
            e0, e1, k2, k3 = sev[s_]
            flush.fill_(s_ & 0xFF)
            e0.record(stream)
            prob.fwd()
            eta.attn_set_kernel_events(k2, k3)
            prob.bwd()
            e1.record(stream)
        torch.cuda.synchronize()
        half = sev[n_sus // 2:]
        sus_total = max_over_ranks(sum(a.elapsed_time(b) for a, b, _, _ in half), world, dev)
        sus_kernel = statistics.mean(k2.elapsed_time(k3) for _, _, k2, k3 in half)
        sus_achieved = pairs * (prob.bwd_fpp - (2 * prob.config["d"] if args.deterministic and "d" in prob.config
                                                else 0)) / (sus_kernel / 1e3) / 1e12
        sustained = {"steps": n_sus, "measured": f"last {len(half)} steps",
                     "ms_per_step": sus_total / len(half),
                     "value": whole_job_tflops(world, flops_step, len(half), sus_total),
                     "bwd_main_ms": sus_kernel,
                     "bwd_main_frac_of_sustained_peak": (sus_achieved / float(load_peaks()[0]["bf16_tflops_sustained"])
                                                         if prob.bound == "tensor" else None)}

    peaks, peak_src = load_peaks()
    bwd_flops, fwd_flops = pairs * prob.bwd_fpp, pairs * prob.fwd_fpp
    fwd_ms, bwd_ms = statistics.mean(t_fwd), statistics.mean(t_bwd)
    fwd_kernel_ms, bwd_kernel_ms = statistics.mean(t_fwd_kernel), statistics.mean(t_bwd_kernel)
    # The key-centric reverse kernel does all five products, or, in the
    # deterministic mode, all but dQ (4d + 4dv flops per pair; dQ comes from
    # the query-centric pass, timed inside bwd_ms).
    kernel_fpp = prob.bwd_fpp - (2 * prob.config["d"] if args.deterministic and "d" in prob.config else 0)
    kernel_flops = pairs * kernel_fpp
    achieved = kernel_flops / (bwd_kernel_ms / 1e3) / 1e12

    if rank == 0:
        clocks = clk.summary()
        if prob.bound == "tensor":
            peak = float(peaks["bf16_tflops"])
            kname = "bwd_kernel" if args.workload not in W.TOPK_WORKLOADS else \
                "top-k reverse kernels (dQ + G/P, dKV contributions)"
            if args.deterministic and args.workload not in W.TOPK_WORKLOADS:
                kname = "bwd_kernel (key-centric, without dQ)"
            src = f"{peak_src} bf16 burst (MEASURED_PEAKS.json)"
        else:
            peak = fp32_alu_peak_tflops(clocks.get("sm_max_mhz") or 1965.0)
            kname = "row-wise reverse kernels (CUDA cores, fp32 FFMA)"
            src = "derived: 148 SMs x 128 fp32 lanes x 2 flops x max SM clock"
        # The deterministic reverse runs another bwd_kernel instantiation (no
        # dQ product, no dQ accumulator traffic): its capture is keyed apart.
        traffic_key = prob.name + ("_deterministic" if args.deterministic else "")
        config = dict(prob.config)
        config.update({"allowed_pairs": pairs, "flops_per_pair": prob.fwd_fpp + prob.bwd_fpp,
                       "l2": "flushed (256 MB write) before every step", "parallelism": f"replicas x{world}"})
        line = {
            "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world, "steps": args.steps,
            "warmup": max(args.warmup, 3), "ms_per_step": ms_step, "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "bf16", "data": "synthetic",
            "config": config,
            "pct_of_peak": {"measured_bf16_burst": 100 * value / world / float(peaks["bf16_tflops"]),
                            "nvidia_dense_bf16_spec_2250": 100 * value / world / 2250.0},
            "conventional": conventional_rate(prob.config, value, flops_step),
            "gather": topk_gather_rate(prob.config, fwd_kernel_ms),
            "fwd_ms": fwd_ms, "bwd_ms": bwd_ms, "fwd_tflops": fwd_flops / (fwd_ms / 1e3) / 1e12,
            "bwd_tflops": bwd_flops / (bwd_ms / 1e3) / 1e12,
            "kernels": {"fwd_main": {"ms": fwd_kernel_ms, "tflops": fwd_flops / (fwd_kernel_ms / 1e3) / 1e12},
                        "bwd_main": {"ms": bwd_kernel_ms, "tflops": achieved}},
            "roofline": {"bound": prob.bound, "kernel": kname,
                         "achieved": achieved, "peak": peak, "unit": UNIT, "frac": achieved / peak,
                         "traffic": recorded_traffic("bwd_kernel", traffic_key) if prob.bound == "tensor" else None,
                         "work_per_launch": f"{kernel_flops:.4e} flops = {pairs} allowed pairs x {kernel_fpp}",
                         "peak_source": src},
            "clocks": clocks,
            "e2e": {"value": e2e_value, "unit": UNIT, "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h,
                    "schedule": "step s+1's inputs copied in and step s-1's gradients copied out "
                                "on their own streams while step s computes"},
            "gpu_launches": prob.launches * args.steps,
        }
        if sustained is not None:
            line["sustained"] = sustained
        if world == 1 and not args.no_cpu_baseline and args.workload == "causal_8k":
            case = W.WORKLOADS["causal_8k"]
            line["cpu_baseline"] = cpu_baseline(W.DenseCase(
                "causal_8k_slice", 1, 1, 1, case.T, case.d, case.dv, "bf16", case.scale, causal=True,
                seed=case.seed))
        print(json.dumps(line), flush=True)
    if world > 1:
        dist.barrier()
        dist.destroy_process_group()


if __name__ == "__main__":
    main()

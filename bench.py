#!/usr/bin/env python
"""Benchmark of the Orthrus dual-view decode step hot path on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]
                    [--workload qwen3_8b_step] [--order cold|interleaved] [--no-graph]
                    [--no-e2e] [--no-cpu-baseline] [--no-configs]

One step = block install + attention of the diffusion view over every layer,
block install + attention of the AR verification view over every layer, the
greedy consensus over the AR logits and the KV commit of the accepted prefix,
all through liborthrus's C ABI, replayed from CUDA graphs.  Inputs are seeded
synthetic tensors of the named Qwen3-shaped workload, resident in HBM before the
timed region; the 36-layer workload reads 2.4 GB of KV per step, far more than
the 126 MB L2, and the cold order re-reads each layer's cache only after every
other layer has streamed through.

Prints ONE JSON line (rank 0).  ``value`` is verified tokens/s over all ranks:
sum over ranks of (tokens committed per step x steps) / max-over-ranks time.
Multi-GPU runs are independent replicas (data parallel, no collective on the
data path; "scaling": "weak").  The line also carries a ``configs`` block: the
attention of both views, KV-read bandwidth and its fraction of the measured HBM
bandwidth, and verified tokens/s for every workload of the decode step (medians
of at least 50 L2-cold iterations each, with the fp64 oracle's time for the
same step on the host cores), and the rows beyond the step: the fused LM head,
the QKV projection, prefill and rejection verification.

``--impl reference`` times the fp64 CPU oracle on the host cores instead: each
step runs whole layer-view attentions (every output row) of the same workload,
as many as keep the whole run within a few minutes (all 72 of a step at the
default driver settings), plus the consensus when the step is complete.
"""
from __future__ import annotations

import argparse
import hashlib
import json
import os
import statistics
import subprocess
import sys
import threading
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = ("dual-view decode-step attn µs & KV-read GB/s vs 8 TB/s; verified tokens/s")
UNIT = "verified tokens/s"
FALLBACK_HBM_GBS = 6650.0
L2_FLUSH_BYTES = 256 << 20          # twice the 126 MB L2
CONFIG_ITERS = 60                   # per configuration of the configs block
REF_BUDGET_S = 150.0                # reference arm: timed CPU seconds per run

# DRAM traffic of one attn_tc_kernel launch on the headline workload, from the
# ncu capture summarised in profiles/ (bytes read + written), keyed by the hash
# of the kernel source it was taken on; reported as null once the source changes.
NCU_TRAFFIC = {("qwen3_8b_step", "5140e1e2a658290e"): 34.09e6}

# The workloads of the configs block: (label, workload, order).  The 36-layer
# step in its specified per-layer order (DIFF then AR per layer) is timed in
# full; the others are single attention layers.
CONFIG_SET = (("qwen3_1p7b_layer", "qwen3_1p7b_layer", "cold"),
              ("qwen3_8b_step_interleaved", "qwen3_8b_step", "interleaved"),
              ("qwen3_4b_ragged", "qwen3_4b_ragged", "cold"),
              ("qwen3_8b_long_k8", "qwen3_8b_long_k8", "cold"),
              ("qwen3_8b_long_k16", "qwen3_8b_long_k16", "cold"),
              ("qwen3_8b_long_k32", "qwen3_8b_long_k32", "cold"))


def parse():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=2000)
    ap.add_argument("--warmup", type=int, default=20)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--workload", default="qwen3_8b_step")
    ap.add_argument("--order", choices=["cold", "interleaved"], default="cold")
    ap.add_argument("--no-graph", action="store_true")
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-configs", action="store_true")
    ap.add_argument("--only", default=None,
                    help="time one entry of the configs block alone (a profiling aid) and print it")
    return ap.parse_args()


def measure_one(label, dev, stream, hbm, iters):
    """One entry of the configs block by its label."""
    from lossless_diffusion_speculative_b200 import workloads as wl
    for lab, name, order in CONFIG_SET:
        if lab == label:
            return measure_config(lab, wl.WORKLOADS[name], order, dev, stream, hbm, iters)
    if label == "qwen3_8b_step_fused_qkv":
        return measure_fused_step("qwen3_8b_step", dev, stream, hbm, iters)
    for name in LM_HEAD_SET:
        if label == "lm_head_consensus_" + name:
            return measure_lm_head(name, dev, stream, hbm, iters)
    for name in QKV_SET:
        if label == "qkv_projection_" + name:
            return measure_qkv(name, dev, stream, hbm, iters)
    for name, S in PREFILL_SET:
        if label == f"prefill_{name}_S{S}":
            return measure_prefill(name, S, dev, stream, tensor_peak()[0], iters)
    for name in REJECT_SET:
        if label == "rejection_verify_" + name:
            return measure_rejection(name, dev, stream, hbm, iters)
    raise SystemExit(f"--only: no configs entry named {label!r}")


def peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            d = json.load(f)
        return float(d["hbm_gbs"]), "measured"
    except Exception:
        return FALLBACK_HBM_GBS, "fallback"


def tensor_peak():
    """Measured dense bf16 TFLOP/s (burst: a kernel timed on its own)."""
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            return float(json.load(f)["bf16_tflops"]), "measured"
    except Exception:
        return 1590.0, "fallback"


def kernel_hash():
    p = os.path.join(ROOT, "lossless_diffusion_speculative_b200", "csrc", "attn_tc.cu")
    with open(p, "rb") as f:
        return hashlib.sha256(f.read()).hexdigest()[:16]


# ----------------------------------------------------------------------------- clocks
class ClockSampler:
    """nvidia-smi samples (100 ms) of SM clock, power, throttle reasons and GPU
    utilisation, from the first warm-up step to the end of the last GPU leg.
    Samples with the GPU at least half busy count as "under load"."""
    FIELDS = ("clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap,"
              "utilization.gpu")

    def __init__(self, gpu_id: str):
        self.gpu_id = gpu_id
        self.proc = None
        self.lines = []

    def start(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", self.gpu_id, f"--query-gpu={self.FIELDS}",
                 "--format=csv,noheader,nounits", "-lms", "100"],
                stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
            self.t = threading.Thread(target=self._read, daemon=True)
            self.t.start()
        except Exception:
            self.proc = None

    def _read(self):
        for line in self.proc.stdout:
            self.lines.append(line.strip())

    def stop(self):
        if self.proc is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"],
                    "samples": 0}
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except Exception:
            self.proc.kill()
        rows = []
        names = ("hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap")
        for ln in self.lines:
            parts = [x.strip() for x in ln.split(",")]
            if len(parts) < 9:
                continue
            try:
                sm, smax, pw = float(parts[0]), float(parts[1]), float(parts[2])
                util = float(parts[8])
            except ValueError:
                continue
            active = {n for n, v in zip(names, parts[4:8]) if v.lower() == "active"}
            rows.append((sm, smax, pw, active, util))
        if not rows:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": [], "samples": 0}
        load = [r for r in rows if r[4] >= 50.0] or rows
        reasons = sorted(set().union(*[r[3] for r in load]))
        return {"sm_mhz": statistics.median(r[0] for r in load), "sm_max_mhz": rows[-1][1],
                "reasons": reasons, "samples": len(rows), "samples_under_load": len(load),
                "power_w_max": max(r[2] for r in rows),
                "window": "first warm-up step to the end of the last GPU leg"}


# ----------------------------------------------------------------------------- CPU oracle
class OracleStep:
    """One decode step of the fp64 oracle: 2 x layers whole layer-view
    attentions (every output row, all host threads) and the consensus.

    The attention inputs of layer 0 (both views) stand in for every layer: the
    oracle's cost depends on the shapes only (its loops have no data-dependent
    trip counts), and regenerating 36 seeded caches per step would dominate the
    run with untimed input generation."""

    def __init__(self, w):
        from lossless_diffusion_speculative_b200 import workloads as wl
        self.w = w
        self.li = [wl.layer_inputs(w, 0, v, poison=False) for v in (0, 1)]
        self.ci = wl.consensus_inputs(w)
        self.n_views = 2 * w.layers

    def layer_view(self, j: int) -> None:
        import oracle
        li = self.li[j % 2]
        oracle.attention(j % 2, li.q, li.k_cache, li.v_cache, li.ctx_lens)

    def consensus(self) -> None:
        import oracle
        oracle.consensus(self.ci.logits, self.ci.proposed)

    def full_step(self) -> float:
        t0 = time.perf_counter()
        for j in range(self.n_views):
            self.layer_view(j)
        self.consensus()
        return time.perf_counter() - t0


def run_reference(args, w, rank, world):
    """Reference arm: the oracle as it stands, on the host cores, rank 0 only."""
    if rank != 0:
        return
    import oracle
    from lossless_diffusion_speculative_b200 import workloads as wl
    os_ = OracleStep(w)
    t0 = time.perf_counter()
    os_.layer_view(0)                                   # first call: sizes the sample
    t_lv = time.perf_counter() - t0
    per_step = int(min(os_.n_views, max(1, REF_BUDGET_S / max(1, args.steps) / t_lv)))
    full = per_step == os_.n_views
    for s in range(args.warmup):                        # untimed, one layer-view each
        os_.layer_view(s)
    times, lv_times = [], []
    for s in range(args.steps):
        t0 = time.perf_counter()
        for j in range(per_step):
            os_.layer_view(s * per_step + j)
        t1 = time.perf_counter()
        if full:
            os_.consensus()
        t2 = time.perf_counter()
        times.append(t2 - t0)
        lv_times.append((t1 - t0) / per_step)
    tokens = int(np.minimum(os_.ci.planted_accept + 1, w.K).sum())
    tokens_exp = wl.expected_tokens_per_step(w)
    if full:
        step_s = float(np.median(times))
        sample = (f"every step: all {os_.n_views} layer-view attentions (all rows) + the "
                  "consensus over the full vocabulary; median step time")
    else:
        t0 = time.perf_counter()
        os_.consensus()
        t_cons = time.perf_counter() - t0
        step_s = float(np.median(lv_times)) * os_.n_views + t_cons
        sample = (f"every step: {per_step} of {os_.n_views} layer-view attentions (all rows); "
                  "a full step = median layer-view time x "
                  f"{os_.n_views} + one consensus ({t_cons * 1e3:.0f} ms)")
    value = tokens / step_s
    line = {"impl": "reference", "metric": METRIC, "value": value, "unit": UNIT,
            "n_gpus": world, "steps": args.steps, "warmup": args.warmup,
            "ms_per_step": float(np.mean(times)) * 1e3,
            "ms_per_full_step": step_s * 1e3, "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "dtype": "f64", "data": "synthetic (seeded)",
            "config": config_of(w, args),
            "tokens_per_step": tokens, "tokens_per_step_expected": tokens_exp,
            "value_at_expected_tokens": tokens_exp / step_s,
            "cpu_baseline": {"value": value, "unit": UNIT, "cores": oracle.num_threads(),
                             "kind": "oracle", "sample": sample},
            "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0,
                    "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)


def config_of(w, args):
    ctx = w.ctx_lens()
    return {"workload": w.name, "B": w.B, "Hq": w.Hq, "Hkv": w.Hkv, "D": w.D,
            "layers": w.layers, "ctx": int(ctx[0]) if w.ctx_lo == w.ctx_hi else
            [int(ctx.min()), int(ctx.max())], "K": w.K, "vocab": w.vocab,
            "order": args.order, "graphs": not args.no_graph,
            "l2": ("inputs larger than L2: each step streams every layer's KV cache "
                   f"({w.kv_bytes_per_view_layer() * 2 * w.layers / 1e9:.2f} GB) through the "
                   "126 MB L2") if w.kv_bytes_per_view_layer() * w.layers > L2_FLUSH_BYTES // 2
            else "KV cache fits in L2: the configs block flushes L2 before every attention"}


# ----------------------------------------------------------------------------- configs block
def measure_config(label, w, order, dev, stream, hbm, iters, st=None, oracle_timing=False):
    """Median µs of each launch segment of one workload's step over `iters`
    replays, L2 flushed before every attention segment (outside the events).
    `st` reuses an existing DecodeStep of the same workload."""
    import torch
    from lossless_diffusion_speculative_b200.step import DecodeStep, layer_groups

    if st is None:
        st = DecodeStep(w, order=order, device=dev)
    graphs = st.capture(stream, order=order)
    flush = torch.empty(L2_FLUSH_BYTES, dtype=torch.uint8, device=dev)
    names = [n for n, _ in graphs[1:]]
    ev = [[(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
           for _ in names] for _ in range(iters)]
    with torch.cuda.stream(stream):
        for it in range(3 + iters):
            graphs[0][1].replay()
            for k, (name, g) in enumerate(graphs[1:]):
                if name.startswith("attn"):
                    flush.zero_()
                if it >= 3:
                    ev[it - 3][k][0].record()
                g.replay()
                if it >= 3:
                    ev[it - 3][k][1].record()
        torch.cuda.synchronize()
    if int(st.status.item()) != 0:
        raise RuntimeError(f"{label}: device status {int(st.status.item()):#x}")
    med = {n: float(np.median([ev[i][k][0].elapsed_time(ev[i][k][1]) for i in range(iters)]))
           * 1e3 for k, n in enumerate(names)}
    attn_us = sum(v for n, v in med.items() if n.startswith("attn"))
    step_us = sum(med.values())
    kv = st.kv_bytes_per_attn_call() * 2 * st.L
    gbs = kv / (attn_us * 1e-6) / 1e9
    tok, tok_e = st.tokens_per_step(), st.tokens_per_step_expected()
    calls = 2 * st.L
    out = {"workload": w.name, "order": order, "B": w.B, "K": w.K, "layers": st.L,
           "ctx": [int(w.ctx_lens().min()), int(w.ctx_lens().max())],
           "attn_us": attn_us, "attn_us_per_call": attn_us / calls,
           "kv_bytes_per_step": kv, "kv_read_gbs": gbs, "kv_read_frac_of_hbm": gbs / hbm,
           "kv_read_frac_of_8tbs": gbs / 8000.0, "step_us": step_us,
           "tokens_per_step": tok, "tokens_per_step_expected": tok_e,
           "verified_tokens_per_s": tok / (step_us * 1e-6),
           "verified_tokens_per_s_at_expected": tok_e / (step_us * 1e-6),
           "segments_us": med, "iters": iters,
           "timing": "median of per-segment CUDA events; L2 flushed before each attention segment"}
    del graphs, st
    if oracle_timing:
        out["oracle"] = oracle_step_time(w, tok, step_us)
    return out


def oracle_step_time(w, tok, step_us):
    """The fp64 oracle on the host cores for one step of workload w: one
    layer-view attention (DIFF, every row) timed and scaled to the step's 2 x
    layers views, plus one timed consensus.  The oracle's loops have no
    data-dependent trip counts, so zero-filled inputs of the workload's shapes
    and context lengths time exactly the work of seeded ones, without the
    seconds of generating them (the arrays are written first, so no page is
    first touched inside the timed region)."""
    import oracle
    q = np.full((w.B, w.K, w.Hq, w.D), 0.01, np.float32)
    kc = np.full((w.B, w.Hkv, w.S_max, w.D), 0.01, np.float32)
    ctx = np.asarray(w.ctx_lens(), np.int32)
    logits = np.full((w.B, w.K, w.vocab), 0.5, np.float32)
    prop = np.zeros((w.B, w.K), np.int32)
    t0 = time.perf_counter()
    oracle.attention(oracle.DIFF, q, kc, kc, ctx)
    t1 = time.perf_counter()
    oracle.consensus(logits, prop)
    t2 = time.perf_counter()
    ms = ((t1 - t0) * 2 * w.layers + (t2 - t1)) * 1e3
    return {"ms_per_step": ms, "cores": oracle.num_threads(), "kind": "oracle",
            "sample": f"one layer-view (all rows) x {2 * w.layers} views + one consensus",
            "verified_tokens_per_s": tok / (ms * 1e-3), "gpu_step_speedup": ms * 1e3 / step_us}


# ----------------------------------------------------------------------------- fused layer step
def measure_fused_step(name, dev, stream, hbm, iters, st=None):
    """The decode step with each layer's QKV projection fused with the cache
    tail write (orthrus_qkv_project) ahead of its attention, per view, then
    consensus and commit: the fused step's median µs, and the projections
    alone (same launches, no attention) for their weight-read bandwidth."""
    import torch
    from lossless_diffusion_speculative_b200 import workloads as wl
    from lossless_diffusion_speculative_b200.step import DecodeStep, layer_groups

    w = wl.WORKLOADS[name]
    if st is None:
        st = DecodeStep(w, order="fused", device=dev, project=True)
    else:
        st.enable_projection()
    out = {"workload": name, "layers": st.L, "B": w.B, "K": w.K, "hidden": w.hidden}
    for order in ("fused", "project_only"):
        graphs = st.capture(stream, order=order)
        names = [n for n, _ in graphs[1:]]
        ev = [[(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
               for _ in names] for _ in range(iters)]
        with torch.cuda.stream(stream):
            for it in range(3 + iters):
                graphs[0][1].replay()
                for k, (_, g) in enumerate(graphs[1:]):
                    if it >= 3:
                        ev[it - 3][k][0].record()
                    g.replay()
                    if it >= 3:
                        ev[it - 3][k][1].record()
            torch.cuda.synchronize()
        if int(st.status.item()) != 0:
            raise RuntimeError(f"fused step {name}: device status {int(st.status.item()):#x}")
        med = {n: float(np.median([ev[i][k][0].elapsed_time(ev[i][k][1]) for i in range(iters)])) * 1e3
               for k, n in enumerate(names)}
        out["segments_us_" + order] = med
        del graphs
    fused = out["segments_us_fused"]
    proj = out["segments_us_project_only"]
    step_us = sum(fused.values())
    proj_us = sum(proj.values())
    calls = 2 * st.L
    wbytes = sum(t.numel() * t.element_size() for t in st.w_qkv[0])
    out.update({"step_us": step_us, "project_us_per_call": proj_us / calls,
                "project_weight_bytes": wbytes,
                "project_weight_read_gbs": wbytes / (proj_us / calls * 1e-6) / 1e9,
                "project_frac_of_hbm": wbytes / (proj_us / calls * 1e-6) / 1e9 / hbm,
                "attn_us_in_step_est": step_us - fused.get("consensus_commit", 0.0) - proj_us,
                "verified_tokens_per_s": st.tokens_per_step() / (step_us * 1e-6),
                "verified_tokens_per_s_at_expected": st.tokens_per_step_expected() / (step_us * 1e-6),
                "timing": "median of per-segment CUDA events over graph replays (inputs larger than L2)"})
    return out


# ----------------------------------------------------------------------------- QKV projection
QKV_SET = ("qwen3_1p7b_layer", "qwen3_8b_step", "qwen3_4b_ragged")


def measure_qkv(name, dev, stream, hbm, iters):
    """orthrus_qkv_project for one layer and one view of the workload (its
    width, heads and batch; the block's key and value rows written into a
    cache of context 8192): median µs per call with L2 flushed before each,
    and the weight-read bandwidth (the stacked [Hq + 2 Hkv] * D x hidden bf16
    weights are the algorithmic traffic; the block's hidden states and outputs
    are < 2 % of it at B * K = 32)."""
    import torch
    from lossless_diffusion_speculative_b200 import binding as ob
    from lossless_diffusion_speculative_b200 import workloads as wl

    w = wl.WORKLOADS[name]
    B, K, hidden, Hq, Hkv, D = w.B, w.K, w.hidden, w.Hq, w.Hkv, w.D
    g = torch.Generator(device=dev)
    g.manual_seed(1000 * w.cid + 93)
    x = torch.randn((B, K, hidden), generator=g, device=dev).to(torch.bfloat16)
    wts = [(torch.randn((n * D, hidden), generator=g, device=dev) / hidden ** 0.5).to(torch.bfloat16)
           for n in (Hq, Hkv, Hkv)]
    ctx = 8192
    kc = torch.zeros((B, Hkv, ctx + 2 * K, D), dtype=torch.bfloat16, device=dev)
    vc = torch.zeros_like(kc)
    ctx_lens = torch.full((B,), ctx, dtype=torch.int32, device=dev)
    q = torch.empty((B, K, Hq, D), dtype=torch.bfloat16, device=dev)
    ws = torch.zeros(ob.orthrus_qkv_workspace_size(B, K, hidden, Hq, Hkv, D), dtype=torch.uint8, device=dev)
    status = torch.zeros(1, dtype=torch.int32, device=dev)
    flush = torch.empty(L2_FLUSH_BYTES, dtype=torch.uint8, device=dev)
    ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
          for _ in range(iters)]
    with torch.cuda.stream(stream):
        for it in range(3 + iters):
            flush.zero_()
            if it >= 3:
                ev[it - 3][0].record()
            ob.orthrus_qkv_project(x, *wts, ctx_lens, q, kc, vc, ws, status=status, stream=stream)
            if it >= 3:
                ev[it - 3][1].record()
        torch.cuda.synchronize()
    if int(status.item()) != 0:
        raise RuntimeError(f"qkv projection: device status {int(status.item()):#x}")
    us = float(np.median([e0.elapsed_time(e1) for e0, e1 in ev])) * 1e3
    wb = sum(t.numel() * 2 for t in wts)
    gbs = wb / (us * 1e-6) / 1e9
    return {"workload": name, "B": B, "K": K, "hidden": hidden, "Hq": Hq, "Hkv": Hkv, "D": D,
            "us_per_call": us, "weight_bytes": wb, "weight_read_gbs": gbs, "frac_of_hbm": gbs / hbm,
            "iters": iters, "kernel": "qkv_proj_kernel (tcgen05 skinny GEMM, split-K, cache-row store)",
            "timing": "median of CUDA events per call; L2 flushed before each call"}


# ----------------------------------------------------------------------------- prefill
PREFILL_SET = (("qwen3_8b_step", 4096), ("qwen3_8b_step", 16384))


def measure_prefill(name, S, dev, stream, tf_peak, iters):
    """orthrus_prefill_attn over one layer of an S-token prompt of the
    workload's attention shape (batch 1): median µs, and the tensor throughput
    on the causal attention's algorithmic flops, 4 * Hq * D * S (S + 1) / 2
    (Q K^T and P V; the kernel's second P V term, which keeps the bf16
    probabilities exact to 2^-14, is not counted)."""
    import torch
    from lossless_diffusion_speculative_b200 import binding as ob
    from lossless_diffusion_speculative_b200 import workloads as wl

    w = wl.WORKLOADS[name]
    Hq, Hkv, D = w.Hq, w.Hkv, w.D
    g = torch.Generator(device=dev)
    g.manual_seed(1000 * w.cid + 94 + S)
    sc = 1.0 / D ** 0.5
    q = (torch.randn((1, S, Hq, D), generator=g, device=dev) * sc).to(torch.bfloat16)
    kc = (torch.randn((1, Hkv, S + 64, D), generator=g, device=dev) * sc).to(torch.bfloat16)
    vc = (torch.randn((1, Hkv, S + 64, D), generator=g, device=dev) * sc).to(torch.bfloat16)
    out = torch.empty((1, S, Hq, D), dtype=torch.float32, device=dev)
    ws = torch.zeros(ob.orthrus_prefill_workspace_size(1, S, Hq, Hkv, D), dtype=torch.uint8, device=dev)
    status = torch.zeros(1, dtype=torch.int32, device=dev)
    flush = torch.empty(L2_FLUSH_BYTES, dtype=torch.uint8, device=dev)
    ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
          for _ in range(iters)]
    with torch.cuda.stream(stream):
        for it in range(3 + iters):
            flush.zero_()
            if it >= 3:
                ev[it - 3][0].record()
            ob.orthrus_prefill_attn(q, kc, vc, out, ws, status=status, stream=stream)
            if it >= 3:
                ev[it - 3][1].record()
        torch.cuda.synchronize()
    if int(status.item()) != 0:
        raise RuntimeError(f"prefill: device status {int(status.item()):#x}")
    us = float(np.median([e0.elapsed_time(e1) for e0, e1 in ev])) * 1e3
    flops = 4.0 * Hq * D * S * (S + 1) / 2
    tf = flops / (us * 1e-6) / 1e12
    return {"workload": name, "S": S, "Hq": Hq, "Hkv": Hkv, "D": D, "us_per_layer": us,
            "tflops": tf, "frac_of_tensor_peak": tf / tf_peak, "iters": iters,
            "kernel": "attn_tc_kernel (prompt chunks as AR-view blocks)",
            "timing": "median of CUDA events per call; L2 flushed before each call"}


# ----------------------------------------------------------------------------- fused LM head
LM_HEAD_SET = ("qwen3_1p7b_layer", "qwen3_8b_step", "qwen3_4b_ragged", "qwen3_8b_long_k32")


def measure_lm_head(name, dev, stream, hbm, iters):
    """orthrus_lm_head_consensus on the workload's Qwen3 width and vocabulary:
    median µs per call over `iters` calls with L2 flushed before each, and the
    weight-read bandwidth (the [V, Hd] bf16 weight is the algorithmic traffic;
    hidden states, proposals and outputs are < 0.5 %).  Inputs are drawn on the
    device from a seeded torch generator (random N(0, 1/Hd) weights, N(0, 1)
    hidden states, one planted argmax per token row, proposals matching the
    plant on the workload's planted acceptance length)."""
    import torch
    from lossless_diffusion_speculative_b200 import binding as ob
    from lossless_diffusion_speculative_b200 import workloads as wl

    w = wl.WORKLOADS[name]
    B, K, V, Hd = w.B, w.K, w.vocab, w.hidden
    g = torch.Generator(device=dev)
    g.manual_seed(1000 * w.cid + 97)
    W = (torch.randn((V, Hd), generator=g, device=dev) * (1.0 / Hd ** 0.5)).to(torch.bfloat16)
    h = torch.randn((B * K, Hd), generator=g, device=dev).to(torch.bfloat16)
    r = torch.randperm(V, generator=g, device=dev)[:B * K]
    hf = h.float()
    W[r] = (12.0 * hf / (hf * hf).sum(dim=1, keepdim=True)).to(torch.bfloat16)
    a = torch.from_numpy(wl.planted_accept_lengths(w)).to(dev)
    prop = torch.randint(0, V, (B, K), generator=g, device=dev, dtype=torch.int32)
    rr = r.view(B, K).to(torch.int32)
    slot = torch.arange(K, device=dev)[None, :]
    prop = torch.where(slot < a[:, None], rr, prop)
    prop = torch.where(slot == a[:, None], (rr + 1) % V, prop).contiguous()
    h = h.view(B, K, Hd).contiguous()
    acc = torch.empty(B, dtype=torch.int32, device=dev)
    nxt = torch.empty(B, dtype=torch.int32, device=dev)
    ws = torch.zeros(ob.orthrus_lm_head_workspace_size(B, K), dtype=torch.uint8, device=dev)
    status = torch.zeros(1, dtype=torch.int32, device=dev)
    flush = torch.empty(L2_FLUSH_BYTES, dtype=torch.uint8, device=dev)
    ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
          for _ in range(iters)]
    with torch.cuda.stream(stream):
        for it in range(3 + iters):
            flush.zero_()
            if it >= 3:
                ev[it - 3][0].record()
            ob.orthrus_lm_head_consensus(h, W, prop, acc, nxt, ws, status=status, stream=stream)
            if it >= 3:
                ev[it - 3][1].record()
        torch.cuda.synchronize()
    exp_a = torch.clamp(a, max=K).to(torch.int32)
    if int(status.item()) != 0 or not torch.equal(acc, exp_a):
        raise RuntimeError(f"lm_head {name}: status {int(status.item()):#x}, accepted {acc.tolist()}")
    us = float(np.median([e0.elapsed_time(e1) for e0, e1 in ev])) * 1e3
    wbytes = V * Hd * 2
    gbs = wbytes / (us * 1e-6) / 1e9
    flops = 2.0 * B * K * Hd * V
    out = {"workload": name, "B": B, "K": K, "V": V, "Hd": Hd, "us_per_call": us,
           "weight_bytes": wbytes, "weight_read_gbs": gbs, "frac_of_hbm": gbs / hbm,
           "tflops": flops / (us * 1e-6) / 1e12, "iters": iters,
           "kernel": "lm_head_kernel (tcgen05 swap-AB GEMM, argmax epilogue, last-CTA consensus)",
           "timing": "median of CUDA events per call; L2 flushed before each call"}
    del W, h, flush
    return out


# ----------------------------------------------------------------------------- rejection sampling
REJECT_SET = ("qwen3_8b_step", "qwen3_4b_ragged", "qwen3_8b_long_k32")


def measure_rejection(name, dev, stream, hbm, iters):
    """orthrus_rejection_verify (temperature 1) on the workload's [B, K, V]
    logits of both views: median µs per call, L2 flushed before each call.
    Algorithmic bytes: both views' logits once (2 x B x K x V x 4) plus the
    rejected row of both views once more per sequence (2 x B x V x 4).  Inputs
    drawn on the device: AR logits N(0, 2), draft logits = AR + N(0, 1),
    proposals = the draft's argmax, uniform draws."""
    import torch
    from lossless_diffusion_speculative_b200 import binding as ob
    from lossless_diffusion_speculative_b200 import workloads as wl

    w = wl.WORKLOADS[name]
    B, K, V = w.B, w.K, w.vocab
    g = torch.Generator(device=dev)
    g.manual_seed(1000 * w.cid + 96)
    ar = torch.randn((B, K, V), generator=g, device=dev) * 2.0
    dr = ar + torch.randn((B, K, V), generator=g, device=dev)
    prop = dr.argmax(dim=2).to(torch.int32).contiguous()
    ua = torch.rand((B, K), generator=g, device=dev)
    ur = torch.rand((B,), generator=g, device=dev)
    acc = torch.empty(B, dtype=torch.int32, device=dev)
    nxt = torch.empty(B, dtype=torch.int32, device=dev)
    ws = torch.zeros(ob.orthrus_rejection_workspace_size(B, K, V), dtype=torch.uint8, device=dev)
    flush = torch.empty(L2_FLUSH_BYTES, dtype=torch.uint8, device=dev)
    ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
          for _ in range(iters)]
    with torch.cuda.stream(stream):
        for it in range(3 + iters):
            flush.zero_()
            if it >= 3:
                ev[it - 3][0].record()
            ob.orthrus_rejection_verify(ar, dr, prop, ua, ur, 1.0, acc, nxt, ws, stream=stream)
            if it >= 3:
                ev[it - 3][1].record()
        torch.cuda.synchronize()
    us = float(np.median([e0.elapsed_time(e1) for e0, e1 in ev])) * 1e3
    nbytes = 2 * B * K * V * 4 + 2 * B * V * 4
    gbs = nbytes / (us * 1e-6) / 1e9
    out = {"workload": name, "B": B, "K": K, "V": V, "us_per_call": us, "bytes": nbytes,
           "read_gbs": gbs, "frac_of_hbm": gbs / hbm, "mean_accepted": float(acc.float().mean()),
           "iters": iters, "kernel": "rs_stats_kernel + rs_resid_kernel",
           "timing": "median of CUDA events per call; L2 flushed before each call"}
    del ar, dr, flush
    return out


# ----------------------------------------------------------------------------- main
def main():
    args = parse()
    import torch
    import torch.distributed as dist
    from lossless_diffusion_speculative_b200 import workloads as wl

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    w = wl.WORKLOADS[args.workload]

    if args.impl == "reference":
        run_reference(args, w, rank, world)
        return

    from datetime import timedelta
    from lossless_diffusion_speculative_b200.replicas import max_over_ranks, replica_throughput
    from lossless_diffusion_speculative_b200.step import DecodeStep, layer_groups

    torch.cuda.set_device(local)
    if args.only:
        dev = torch.device("cuda", local)
        r = measure_one(args.only, dev, torch.cuda.Stream(device=dev), peaks()[0], args.steps)
        print(json.dumps({"only": args.only, **r}), flush=True)
        return
    if world > 1:
        dist.init_process_group("nccl", timeout=timedelta(seconds=120),
                                device_id=torch.device("cuda", local))
    dev = torch.device("cuda", local)
    hbm, hbm_src = peaks()
    st = DecodeStep(w, order=args.order, device=dev)
    stream = torch.cuda.Stream(device=dev)
    graphs = None if args.no_graph else st.capture(stream)
    whole = None if args.no_graph else st.capture_whole(stream)
    segs = [n for n, _ in st.segments()]
    uuid = str(torch.cuda.get_device_properties(dev).uuid)
    sampler = ClockSampler(uuid if uuid.startswith("GPU-") else f"GPU-{uuid}")

    def one_step(evs=None):
        if graphs is None:
            st.reset()
            for i, (_, fn) in enumerate(st.segments()):
                if evs is not None:
                    evs[i].record()
                fn()
            if evs is not None:
                evs[-1].record()
        else:
            graphs[0][1].replay()
            for i, (_, g) in enumerate(graphs[1:]):
                if evs is not None:
                    evs[i].record()
                g.replay()
            if evs is not None:
                evs[-1].record()

    def barrier():
        if world > 1:
            dist.barrier()

    with torch.cuda.stream(stream):
        sampler.start()
        for _ in range(args.warmup):
            one_step()
        torch.cuda.synchronize()
        res = st.result()
        if int(st.status.item()) != 0:
            raise RuntimeError(f"device status {int(st.status.item()):#x}")
        nseg = len(segs)
        # the headline: K steps, each one replay of the whole step's graph
        # (an event between steps gives the per-step median)
        step_ev = [torch.cuda.Event(enable_timing=True) for _ in range(args.steps + 1)]
        barrier()
        torch.cuda.synchronize()
        step_ev[0].record()
        for s in range(args.steps):
            if whole is not None:
                whole.replay()
            else:
                one_step()
            step_ev[s + 1].record()
        torch.cuda.synchronize()
        barrier()
        elapsed_ms = step_ev[0].elapsed_time(step_ev[-1])
        step_ms = np.array([step_ev[s].elapsed_time(step_ev[s + 1]) for s in range(args.steps)])
        # the breakdown: K more steps replayed segment by segment, with events
        # between the segments (attention time for the roofline)
        ev = [[torch.cuda.Event(enable_timing=True) for _ in range(nseg + 1)]
              for _ in range(args.steps)]
        barrier()
        torch.cuda.synchronize()
        for s in range(args.steps):
            one_step(ev[s])
        torch.cuda.synchronize()
        barrier()
        seg_ms = np.zeros((args.steps, nseg))
        for s in range(args.steps):
            for i in range(nseg):
                seg_ms[s, i] = ev[s][i].elapsed_time(ev[s][i + 1])

        # ---- end to end: host inputs in (pinned), result out, every step
        e2e = None
        if not args.no_e2e:
            host = {n: torch.empty(t.shape, dtype=t.dtype, pin_memory=True)
                    for n, t in (("q", st.q_all), ("kb", st.kb_all), ("vb", st.vb_all),
                                 ("logits", st.logits), ("proposed", st.proposed))}
            for n, t in (("q", st.q_all), ("kb", st.kb_all), ("vb", st.vb_all),
                         ("logits", st.logits), ("proposed", st.proposed)):
                host[n].copy_(t)
            dst = {"q": st.q_all, "kb": st.kb_all, "vb": st.vb_all, "logits": st.logits,
                   "proposed": st.proposed}
            out_acc = torch.empty(w.B, dtype=torch.int32, pin_memory=True)
            out_nxt = torch.empty(w.B, dtype=torch.int32, pin_memory=True)
            h2d = sum(t.numel() * t.element_size() for t in host.values())
            d2h = 2 * w.B * 4
            e_steps = max(1, min(args.steps, 500))

            # The copies of a step go out on their own stream in the order the
            # step consumes them (per group of layers: block K/V and queries of
            # the DIFF view, then the same of the AR view, then logits and
            # proposals); the step runs as graphs of those layer groups and each
            # waits only for what it reads.  A step's copies start once the
            # previous step is done with the buffers.
            cs = torch.cuda.Stream(device=dev)
            # diffusion-view layer groups of 1, 2, 4, 8 and the rest: a layer's
            # copies take about half its compute, so each group's inputs land
            # while the groups before it run and only the first group's copy is
            # exposed; the AR view's inputs arrive during the diffusion view,
            # so it runs as one group
            chunk = {"diff": (1, 2, 4, 8, 21), "ar": 64}
            egraphs = None if graphs is None else st.capture(stream, chunk=chunk)
            chunks, needs = [], {}
            if args.order == "cold":
                for view, vn in ((0, "diff"), (1, "ar")):
                    for layers in layer_groups(st.L, chunk[vn]):
                        c = layers.start
                        sl = (view, slice(c, layers.stop))
                        needs[f"write_block_{vn}_{c}"] = needs[f"attn_{vn}_{c}"] = len(chunks)
                        chunks.append([("kb", sl), ("vb", sl), ("q", sl)])
            else:
                needs["attn_interleaved"] = len(chunks)
                chunks.append([("kb", None), ("vb", None), ("q", None)])
            needs["consensus_commit"] = len(chunks)
            chunks.append([("logits", None), ("proposed", None)])
            ready = [torch.cuda.Event() for _ in chunks]
            done = torch.cuda.Event()

            # The whole end-to-end step as one CUDA graph: the copy stream
            # forks from the step, each group's copies then an event, the
            # step's segments each after its group's event, the result read
            # back, the copy stream joined (one launch per step)
            whole_e2e = None
            if graphs is not None:
                try:
                    seg_fns = st.segments(chunk)
                    fork, join = torch.cuda.Event(), torch.cuda.Event()
                    for _, fn in seg_fns:
                        fn()
                    torch.cuda.synchronize()
                    whole_e2e = torch.cuda.CUDAGraph()
                    with torch.cuda.graph(whole_e2e, stream=stream):
                        fork.record(stream)
                        cs.wait_event(fork)
                        with torch.cuda.stream(cs):
                            for ev_i, ch in zip(ready, chunks):
                                for n, v in ch:
                                    d_t, h_t = (dst[n], host[n]) if v is None else (dst[n][v], host[n][v])
                                    d_t.copy_(h_t, non_blocking=True)
                                ev_i.record(cs)
                            join.record(cs)
                        st.reset()
                        for name, fn in seg_fns:
                            stream.wait_event(ready[needs[name]])
                            fn()
                        out_acc.copy_(st.accepted, non_blocking=True)
                        out_nxt.copy_(st.next_token, non_blocking=True)
                        stream.wait_event(join)
                    torch.cuda.synchronize()
                except Exception as exc:                  # (fall back to per-segment graphs)
                    print(f"bench: whole-step end-to-end graph not captured ({exc}); "
                          "per-segment graphs instead", file=sys.stderr)
                    whole_e2e = None
                    torch.cuda.synchronize()

            def e2e_step():
                if whole_e2e is not None:
                    whole_e2e.replay()
                    return
                if graphs is None:
                    for n in host:
                        dst[n].copy_(host[n], non_blocking=True)
                    one_step()
                else:
                    cs.wait_event(done)
                    with torch.cuda.stream(cs):
                        for ev_i, ch in zip(ready, chunks):
                            for n, v in ch:
                                d_t, h_t = (dst[n], host[n]) if v is None else (dst[n][v], host[n][v])
                                d_t.copy_(h_t, non_blocking=True)
                            ev_i.record(cs)
                    egraphs[0][1].replay()
                    for name, g in egraphs[1:]:
                        stream.wait_event(ready[needs[name]])
                        g.replay()
                out_acc.copy_(st.accepted, non_blocking=True)
                out_nxt.copy_(st.next_token, non_blocking=True)
                done.record(stream)

            done.record(stream)
            for _ in range(3):
                e2e_step()
            torch.cuda.synchronize()
            barrier()
            a0 = torch.cuda.Event(enable_timing=True)
            a1 = torch.cuda.Event(enable_timing=True)
            a0.record()
            done.record(stream)
            for _ in range(e_steps):
                e2e_step()
            a1.record()
            torch.cuda.synchronize()
            barrier()
            e2e_ms = a0.elapsed_time(a1)
            assert int(out_acc[0]) == int(res.accepted[0])
            e2e = (e2e_ms, e_steps, h2d, d2h)
            egraphs = whole_e2e = None

        # ---- every workload of the decode step, one at a time (rank 0 only)
        configs = None
        if rank == 0 and world == 1 and not args.no_configs:
            configs = {}
            for label, name, order in CONFIG_SET:
                configs[label] = measure_config(label, wl.WORKLOADS[name], order, dev, stream,
                                                hbm, CONFIG_ITERS,
                                                st=st if name == w.name else None,
                                                oracle_timing=not args.no_cpu_baseline and name != w.name)
                torch.cuda.empty_cache()
            configs["qwen3_8b_step_fused_qkv"] = measure_fused_step(
                "qwen3_8b_step", dev, stream, hbm, CONFIG_ITERS // 2,
                st=st if w.name == "qwen3_8b_step" else None)
            torch.cuda.empty_cache()
            for name in LM_HEAD_SET:
                configs["lm_head_consensus_" + name] = measure_lm_head(name, dev, stream, hbm,
                                                                       CONFIG_ITERS)
                torch.cuda.empty_cache()
            for name in QKV_SET:
                configs["qkv_projection_" + name] = measure_qkv(name, dev, stream, hbm, CONFIG_ITERS)
                torch.cuda.empty_cache()
            tfp, _ = tensor_peak()
            for name, S in PREFILL_SET:
                configs[f"prefill_{name}_S{S}"] = measure_prefill(name, S, dev, stream, tfp, CONFIG_ITERS // 3)
                torch.cuda.empty_cache()
            for name in REJECT_SET:
                configs["rejection_verify_" + name] = measure_rejection(name, dev, stream, hbm,
                                                                        CONFIG_ITERS)
                torch.cuda.empty_cache()
        torch.cuda.synchronize()
        clocks = sampler.stop()

    # ---- max over ranks (independent replicas: no data-path collective)
    elapsed_ms, e2e_ms_max = max_over_ranks([elapsed_ms, e2e[0] if e2e else 0.0], device=dev)

    tokens = st.tokens_per_step()
    tokens_exp = st.tokens_per_step_expected()
    ms_per_step = elapsed_ms / args.steps
    value = replica_throughput(tokens, args.steps, world, elapsed_ms)
    kv_step = st.kv_bytes_per_attn_call() * 2 * st.L
    if args.order == "cold":
        attn_ms_steps = seg_ms[:, segs.index("attn_diff")] + seg_ms[:, segs.index("attn_ar")]
    else:
        attn_ms_steps = seg_ms[:, segs.index("attn_interleaved")]
    attn_ms = float(np.mean(attn_ms_steps))
    attn_ms_med = float(np.median(attn_ms_steps))
    per_call_s = attn_ms / 1e3 / (2 * st.L)
    achieved = st.kv_bytes_per_attn_call() / per_call_s / 1e9
    traffic = NCU_TRAFFIC.get((w.name, kernel_hash()))
    per_call = 1 if st.tc_path else 2             # tcgen05: one launch; CUDA-core: + combine
    launches_per_step = (2 + 2 * st.L * per_call + 2 + 1) if args.order == "cold" else \
        (2 * st.L + 2 * st.L * per_call + 2 + 1)

    if rank == 0:
        line = {
            "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms_per_step,
            "ms_per_step_median": float(np.median(step_ms)),
            "timing": ("each step one replay of the whole step's CUDA graph (CUDA events between "
                       "steps); the segment breakdown and attention time from K further steps "
                       "replayed segment by segment"),
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
            "dtype": "bf16", "data": "synthetic (seeded Qwen3-shaped tensors; planted acceptance)",
            "config": config_of(w, args),
            "tokens_per_step": tokens,
            "tokens_per_step_expected": tokens_exp,
            "value_at_expected_tokens": replica_throughput(tokens_exp, args.steps, world,
                                                           elapsed_ms),
            "attn_us_per_step": attn_ms * 1e3,
            "attn_us_per_step_median": attn_ms_med * 1e3,
            "kv_read_gbs": kv_step / (attn_ms / 1e3) / 1e9,
            "kv_read_frac_of_hbm": kv_step / (attn_ms / 1e3) / 1e9 / hbm,
            "kv_read_frac_of_8tbs": kv_step / (attn_ms / 1e3) / 1e9 / 8000.0,
            "segments_us": {n: float(v * 1e3) for n, v in zip(segs, seg_ms.mean(axis=0))},
            "attn_path": "tcgen05" if st.tc_path else "cuda-core",
            "roofline": {"bound": "hbm", "achieved": achieved, "peak": hbm, "unit": "GB/s",
                         "frac": achieved / hbm, "traffic": traffic,
                         "kernel": ("orthrus_attn (attn_tc_kernel, split merge in-kernel)" if st.tc_path
                                    else "orthrus_attn (attn_simt_kernel + attn_combine_kernel)"),
                         "peak_source": f"{hbm_src} hbm_gbs",
                         "bytes_per_launch": st.kv_bytes_per_attn_call()},
            "gpu_launches": launches_per_step * args.steps,
            "clocks": clocks,
        }
        if e2e:
            line["e2e"] = {"value": replica_throughput(tokens, e2e[1], world, e2e_ms_max), "unit": UNIT,
                           "h2d_bytes_per_step": e2e[2], "d2h_bytes_per_step": e2e[3],
                           "steps": e2e[1]}
        if configs:
            line["configs"] = configs
        if world == 1 and not args.no_cpu_baseline:
            os_ = OracleStep(w)
            step_s = os_.full_step()
            import oracle
            line["cpu_baseline"] = {"value": tokens / step_s, "unit": UNIT,
                                    "cores": oracle.num_threads(), "kind": "oracle",
                                    "sample": f"one full decode step: all {os_.n_views} "
                                              "layer-view attentions (all rows) + the consensus",
                                    "ms_per_step": step_s * 1e3}
        print(json.dumps(line), flush=True)
    st.graphs = None
    graphs = None
    if world > 1:
        dist.barrier()
        dist.destroy_process_group()


if __name__ == "__main__":
    main()

"""Benchmark of the TokenGate pruned-prefill hot path on B200.

One step = one pass of the whole path over one synthetic 128k-token request
(hidden 2048, gate MLP 2048->256->1, question 512 tokens, budget K = 8192):
    tg_gate_score (131072 tokens) -> tg_select_topk -> tg_gather (8704 rows)
    -> 27 x tg_gated_attention (S = 8704, Hq 16, Hkv 8, D 128, independent Q/K/V per layer).

Prints one JSON line.  ``value`` is the gated-attention algorithmic TFLOP/s of the
whole step (27 layers of 4*D*Hq*S*(S+1)/2 flops divided by the full step time, the
gate/top-K/gather time included); the gate+top-K+gather path is reported beside
it in GB/s against HBM.  Inputs are resident in HBM before timing starts; the
per-step working set (512 MiB residual + 1.9 GB of Q/K/V) is larger than L2.
``roofline`` is the attention kernel against the measured burst bf16 peak (the timed
region is a fraction of a second); ``in_run_peaks`` re-measures a cuBLAS bf16 GEMM and
an HBM copy in the same process with their clocks, so the kernel's fraction can also be
read at the clock it ran at.
``attention.context`` compares, outside the timed step, the kernel with and without
the key bias and the library's causal attention on the same layers.
``next_rows`` gives the device time of the calls around the path on the same
workload, outside the timed step: the pruned layer's projections, the whole pruned
layer chain (QKV + norm + rotary -> gated attention -> o_proj + residual), the attention
backward, random-K and a 4-budget sweep.

``--sweep`` instead prints one JSON line per (workload, budget) of every named
workload: the 16k budgets, the 32k budgets and its full-context pass, the 128k budgets
and the ragged 4-request batch through the packed (varlen) calls; each line carries
the attention TFLOP/s against the bf16 peaks, the select path's GB/s against HBM and
the oracle timed on the host cores on a bounded row sample.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl {tokengate,reference}] [--sweep]
"""
from __future__ import annotations

import argparse
import json
import math
import os
import statistics
import subprocess
import sys
import threading
import time

import numpy as np
import torch

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

WORKLOAD = "qwen3_1p7b_n128k"
METRIC = "gated-attn TFLOP/s & % bf16 peak; gate+topK+gather GB/s & % HBM, N=128k"
DATASHEET_HBM_GBS = 8000.0
NOMINAL_BF16_TFLOPS = 2250.0

# DRAM traffic (dram__bytes_read.sum and dram__bytes_write.sum) of one attention launch
# at S = 8704, from one ncu capture of the kernel (its summary is kept with the
# profiles).  It is reported only while the kernel sources are the ones that capture
# measured.
ATTENTION_TRAFFIC = {"sources_sha1": "d0c1fe096e48f54362f073462bcaa26f7d08a5f7",
                     "read": 71617024, "write": 9345280}


def attention_sources_sha1() -> str:
    import hashlib
    h = hashlib.sha1()
    for f in ("attention.cu", "ptx.cuh"):
        with open(os.path.join(ROOT, "learned_token_pruning_mlp_b200", "csrc", f), "rb") as fh:
            h.update(fh.read())
    return h.hexdigest()


def attention_traffic():
    """(read, write) DRAM bytes of one launch from the ncu record, or None once the kernel changed."""
    if attention_sources_sha1() != ATTENTION_TRAFFIC["sources_sha1"]:
        return None
    return ATTENTION_TRAFFIC["read"], ATTENTION_TRAFFIC["write"]


def attention_bytes(S: int, hq: int, hkv: int, d: int):
    """Algorithmic HBM bytes of one gated-attention launch: (read, write).  Q, K, V, the
    key scores and the gains are read once; O is written once."""
    read = (hq + 2 * hkv) * d * 2 * S + 4 * S + 4 * hq
    write = hq * d * 2 * S
    return read, write


def attention_flops(S: int, hq: int, d: int) -> int:
    """Algorithmic flops of one causal gated-attention layer: QK^T and PV over the visible pairs."""
    return 4 * d * hq * S * (S + 1) // 2


def select_path_bytes(n: int, d: int, h: int, S: int) -> int:
    """Algorithmic HBM bytes of gate + top-K + gather: each input read once, each output written once."""
    gate = n * d * 2 + h * d * 2 + 3 * h * 2 + 2 + n * 4
    topk = n * 4 + n * 1 + S * 4 + 4
    gather = S * 4 + 2 * S * d * 2 + S * 4 + S * 4
    return gate + topk + gather


def load_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as f:
            j = json.load(f)
        return {"hbm_gbs": j["hbm_gbs"], "bf16_tflops": j["bf16_tflops"],
                "bf16_tflops_sustained": j.get("bf16_tflops_sustained", j["bf16_tflops"]), "source": "measured"}
    return {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0, "source": "fallback"}


class ClockSampler:
    """Samples nvidia-smi clocks and throttle reasons while the timed region runs."""

    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, index: int):
        self.index = index
        self.proc = None
        self.lines = []
        self.thread = None

    def start(self):
        try:
            self.proc = subprocess.Popen(["nvidia-smi", f"--id={self.index}", f"--query-gpu={self.FIELDS}",
                                          "--format=csv,noheader,nounits", "-lms", "50"],
                                         stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
        except (OSError, ValueError):
            self.proc = None
            return
        self.thread = threading.Thread(target=self._read, daemon=True)
        self.thread.start()

    def _read(self):
        for line in self.proc.stdout:
            self.lines.append(line.strip())

    def stop(self):
        if self.proc is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"]}
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except subprocess.TimeoutExpired:
            self.proc.kill()
        if self.thread:
            self.thread.join(timeout=2)
        sm, mx, reasons = [], [], set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for ln in self.lines:
            parts = [p.strip() for p in ln.split(",")]
            if len(parts) < 9:
                continue
            try:
                sm.append(float(parts[1]))
                mx.append(float(parts[2]))
            except ValueError:
                continue
            for nm, v in zip(names, parts[5:9]):
                if v.lower() == "active":
                    reasons.add(nm)
        return {"sm_mhz": statistics.median(sm) if sm else None, "sm_max_mhz": max(mx) if mx else None,
                "reasons": sorted(reasons), "samples": len(sm)}


def dist_setup(n_gpus: int):
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world > 1:
        import datetime
        torch.cuda.set_device(local)
        torch.distributed.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                             device_id=torch.device("cuda", local))
    return world, rank, local


def barrier(world):
    if world > 1:
        torch.distributed.barrier()


def max_over_ranks(x: float, world: int) -> float:
    """The slowest rank's value (timing is reported as the max over ranks)."""
    if world == 1:
        return x
    dev = "cuda" if torch.distributed.get_backend() == "nccl" else "cpu"
    t = torch.tensor([x], dtype=torch.float64, device=dev)
    torch.distributed.all_reduce(t, op=torch.distributed.ReduceOp.MAX)
    return float(t.item())


def replica_throughput(units_per_rank: float, ms_per_step_max: float, world: int) -> float:
    """Whole-job throughput of ``world`` independent replicas: every rank's units over the
    slowest rank's step time (replicas only: no data-path exchange between ranks)."""
    return world * units_per_rank / (ms_per_step_max * 1e-3)


def workload_config(world: int, K: int, S: int, L: int, n: int) -> dict:
    return {"workload": f"{WORKLOAD}: N={n} (question 512), d=2048, gate 2048->256->1, K={K}, "
                        f"S={S}, {L} gated layers Hq=16 Hkv=8 D=128",
            "global_batch": world, "seq_len": n, "kept": S, "parallelism": f"replicas x{world}",
            "l2": "inputs larger than L2 (512 MiB residual + 1.9 GB Q/K/V per step)"}


# ----------------------------------------------------------------------------- tokengate arm
def make_inputs(w, K):
    from learned_token_pruning_mlp_b200 import workloads as W
    hidden, W1, b1, W2, b2 = W.gate_inputs(w)
    mask = W.doc_mask(w)
    sel = W.selection_scores(w)
    q = w.segments[0].q
    S = K + q
    gain, tau = W.attention_params(w)
    layers = [W.attention_inputs(w, S, layer=l) for l in range(w.layers)]
    return dict(hidden=hidden, W1=W1, b1=b1, W2=W2, b2=b2, mask=mask, sel=sel, gain=gain, tau=tau, layers=layers, S=S)


def run_tokengate(args, world, rank, local):
    import learned_token_pruning_mlp_b200 as tg
    from learned_token_pruning_mlp_b200 import build as tgbuild
    from learned_token_pruning_mlp_b200 import workloads as W
    tgbuild.build()
    dev = torch.device("cuda", local)
    torch.cuda.set_device(dev)
    w = W.get(WORKLOAD)
    K = args.budget
    host = make_inputs(w, K)
    S = host["S"]
    n, d, h = w.n, w.d, w.h
    L = w.layers

    # device-resident copies
    dv = {k: host[k].to(dev) for k in ("hidden", "W1", "b1", "W2", "b2", "mask", "sel", "gain")}
    layers = [tuple(t.to(dev) for t in lay) for lay in host["layers"]]
    scores = torch.empty(n, dtype=torch.float32, device=dev)
    kept = torch.empty(n, dtype=torch.int32, device=dev)
    n_kept = torch.empty(1, dtype=torch.int32, device=dev)
    hidden_k = torch.empty(S, d, dtype=torch.bfloat16, device=dev)
    s_k = torch.empty(S, dtype=torch.float32, device=dev)
    outs = [torch.empty(S, w.hq, w.head_dim, dtype=torch.bfloat16, device=dev) for _ in range(L)]
    stream = torch.cuda.current_stream(dev)
    tau = host["tau"]

    def step(ev=None):
        if ev is not None:
            ev[0].record(stream)
        tg.tg_gate_score(dv["hidden"], dv["W1"], dv["b1"], dv["W2"], dv["b2"], scores=scores)
        tg.tg_select_topk(dv["sel"], dv["mask"], K, kept_idx=kept, n_kept=n_kept)
        tg.tg_gather(dv["hidden"], kept, n_rows=S, n_kept=n_kept, hidden_k=hidden_k, scores=dv["sel"], s_k=s_k)
        if ev is not None:
            ev[1].record(stream)
        for l in range(L):
            Q, Kc, V = layers[l]
            tg.tg_gated_attention(Q, Kc, V, s_k, dv["gain"], tau, O=outs[l])
        if ev is not None:
            ev[2].record(stream)

    for _ in range(args.warmup):
        step()
    torch.cuda.synchronize()
    bits = tg.tg_get_device_error()
    if bits:
        raise RuntimeError(f"device status bits {bits} after warm-up")
    if int(n_kept.item()) != S:
        raise RuntimeError(f"kept {int(n_kept.item())} tokens, expected {S}")

    evs = [[torch.cuda.Event(enable_timing=True) for _ in range(3)] for _ in range(args.steps)]
    start, stop = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    sampler = ClockSampler(local)
    barrier(world)
    torch.cuda.synchronize()
    sampler.start()
    time.sleep(0.3)
    start.record(stream)
    for i in range(args.steps):
        step(evs[i])
    stop.record(stream)
    torch.cuda.synchronize()
    clocks = sampler.stop()
    barrier(world)
    total_ms = start.elapsed_time(stop)
    sel_ms = [e[0].elapsed_time(e[1]) for e in evs]
    att_ms = [e[1].elapsed_time(e[2]) for e in evs]
    ms_per_step = max_over_ranks(total_ms / args.steps, world)
    bits = tg.tg_get_device_error()
    if bits:
        raise RuntimeError(f"device status bits {bits} after timing")

    flops_layer = attention_flops(S, w.hq, w.head_dim)
    flops_step = flops_layer * L
    sel_bytes = select_path_bytes(n, d, h, S)
    peaks = load_peaks()
    value = replica_throughput(flops_step, ms_per_step, world) / 1e12
    att_launch_ms = statistics.mean(att_ms) / L
    att_tflops = flops_layer / (att_launch_ms * 1e-3) / 1e12
    sel_mean = statistics.mean(sel_ms)
    sel_gbs = sel_bytes / (sel_mean * 1e-3) / 1e9

    # The select path alone, back to back (gate -> top-K -> gather, repeated), so that
    # its launches overlap as they do inside a pipeline instead of being cut by events.
    # Two forms: the workload's fixed selector scores (as in the step), and the chain on
    # the gate's own output (top-K reading the scores the gate just wrote).
    sel_iters = max(10, args.steps)

    def select_only(own_scores: bool):
        tg.tg_gate_score(dv["hidden"], dv["W1"], dv["b1"], dv["W2"], dv["b2"], scores=scores)
        src = scores if own_scores else dv["sel"]
        tg.tg_select_topk(src, dv["mask"], K, kept_idx=kept, n_kept=n_kept)
        tg.tg_gather(dv["hidden"], kept, n_rows=S, n_kept=n_kept, hidden_k=hidden_k, scores=src, s_k=s_k)

    def time_select(own_scores: bool) -> float:
        for _ in range(3):
            select_only(own_scores)
        barrier(world)
        torch.cuda.synchronize()
        s0, s1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        s0.record(stream)
        for _ in range(sel_iters):
            select_only(own_scores)
        s1.record(stream)
        torch.cuda.synchronize()
        return max_over_ranks(s0.elapsed_time(s1) / sel_iters * 1e3, world)

    # The select path's marginal cost inside the step: the same steps with the 27
    # attention layers alone, timed the same way; the difference is what gate -> top-K
    # -> gather add to a step once their launches overlap their neighbours' (the
    # event-bracketed in-step figure above cuts that overlap at both ends).
    def attention_only():
        for l in range(L):
            Q, Kc, V = layers[l]
            tg.tg_gated_attention(Q, Kc, V, s_k, dv["gain"], tau, O=outs[l])

    for _ in range(3):
        attention_only()
    barrier(world)
    torch.cuda.synchronize()
    a0, a1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    a0.record(stream)
    for _ in range(args.steps):
        attention_only()
    a1.record(stream)
    torch.cuda.synchronize()
    attn_only_ms = max_over_ranks(a0.elapsed_time(a1) / args.steps, world)
    marginal_us = (ms_per_step - attn_only_ms) * 1e3

    sel_b2b_us = time_select(False)
    sel_b2b_gbs = sel_bytes / (sel_b2b_us * 1e-6) / 1e9
    own_us = time_select(True)
    own_gbs = sel_bytes / (own_us * 1e-6) / 1e9
    if tg.tg_get_device_error() & ~tg.TG_DEVERR_K_GT_NDOC:
        raise RuntimeError("device status bits set by the select-path timings")

    # end to end through the public calls with host buffers: H2D of the step's inputs
    # from pinned memory and D2H of its results inside the timed region
    e2e = run_e2e(tg, host, dev, w, K, S, tau, world, args)
    next_rows = time_next_rows(tg, dev, w, host, dv, kept, S)
    attn_ctx = attention_context(tg, dev, w, layers, s_k, dv["gain"], tau, S)
    in_run = measure_in_run_peaks(dev, local)

    a_read, a_write = attention_bytes(S, w.hq, w.hkv, w.head_dim)
    traffic = attention_traffic()
    burst = peaks["bf16_tflops"]
    roofline = {"bound": "tensor", "achieved": round(att_tflops, 1), "peak": burst, "unit": "TFLOP/s",
                "frac": round(att_tflops / burst, 4),
                "traffic": (traffic[0] + traffic[1]) if traffic else None,
                "traffic_detail": {
                    "dram_read_bytes": traffic[0] if traffic else None,
                    "dram_write_bytes": traffic[1] if traffic else None,
                    "algorithmic_read_bytes": a_read, "algorithmic_write_bytes": a_write,
                    "note": "one ncu capture of one launch; O's lines still dirty in L2 when the kernel ends are "
                            "written back after it and are not counted in its write bytes"},
                "kernel": "gated_attention_kernel<128>",
                "peak_source": f"{peaks['source']} bf16 burst (MEASURED_PEAKS.json; the timed region lasts "
                               f"{total_ms / 1e3:.2f} s)"}
    if in_run.get("bf16_gemm_tflops") and clocks.get("sm_mhz") and in_run.get("gemm_sm_mhz"):
        # both sides at the clock they ran at: TFLOP/s per GHz of the median sampled SM clock
        att_per_ghz = att_tflops / (clocks["sm_mhz"] / 1e3)
        gemm_per_ghz = in_run["bf16_gemm_tflops"] / (in_run["gemm_sm_mhz"] / 1e3)
        roofline["clock_consistent"] = {
            "attention_tflops_per_ghz": round(att_per_ghz, 1), "gemm_tflops_per_ghz": round(gemm_per_ghz, 1),
            "frac": round(att_per_ghz / gemm_per_ghz, 4),
            "frac_of_in_run_gemm": round(att_tflops / in_run["bf16_gemm_tflops"], 4)}

    out = {
        "metric": METRIC, "value": round(value, 2), "unit": "TFLOP/s", "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": round(ms_per_step, 4), "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "bf16", "data": "synthetic",
        "config": workload_config(world, K, S, L, n),
        "attention": {"ms_per_layer": round(att_launch_ms, 4), "tflops": round(att_tflops, 1),
                      "frac_of_bf16_peak": round(att_tflops / burst, 4),
                      "frac_of_bf16_sustained": round(att_tflops / peaks["bf16_tflops_sustained"], 4),
                      "frac_of_nominal_2250": round(att_tflops / NOMINAL_BF16_TFLOPS, 4), "context": attn_ctx},
        "select_path": {"us": round(sel_b2b_us, 2), "bytes": sel_bytes, "gbs": round(sel_b2b_gbs, 1),
                        "frac_of_hbm": round(sel_b2b_gbs / peaks["hbm_gbs"], 4),
                        "frac_of_datasheet_8tbs": round(sel_b2b_gbs / DATASHEET_HBM_GBS, 4),
                        "timing": f"{sel_iters} back-to-back gate->top-K->gather passes",
                        "in_step_us": round(sel_mean * 1e3, 2),
                        "in_step_gbs": round(sel_gbs, 1),
                        "in_step_frac_of_hbm": round(sel_gbs / peaks["hbm_gbs"], 4),
                        "in_step_timing": "CUDA events around gate -> top-K -> gather in every timed step (the "
                                          "events stop the launches overlapping the neighbouring kernels)",
                        "in_step_marginal_us": round(marginal_us, 2),
                        "in_step_marginal_timing": f"step time minus the same {args.steps} steps of the "
                                                   f"{L} attention layers alone ({attn_only_ms:.4f} ms per step): "
                                                   f"what the select path adds to a step once its kernels "
                                                   f"overlap the compute-bound attention's first and last "
                                                   f"waves (not a bandwidth figure)",
                        "gate_scores_chain": {
                            "us": round(own_us, 2), "gbs": round(own_gbs, 1),
                            "frac_of_hbm": round(own_gbs / peaks["hbm_gbs"], 4),
                            "timing": f"{sel_iters} back-to-back passes, top-K and gather reading the gate's "
                                      f"own scores"}},
        "roofline": roofline,
        "in_run_peaks": in_run,
        "e2e": e2e,
        "next_rows": next_rows,
        "gpu_launches": args.steps * (3 + L),
        "clocks": clocks,
    }
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        out["cpu_baseline"] = cpu_baseline(host["layers"][0], host["gain"], host["tau"], w, S,
                                           budget_s=args.cpu_seconds)
    return out


def measure_in_run_peaks(dev, local, gemm_n: int = 8192, gemm_reps: int = 200, copy_gib: float = 1.0,
                         copy_reps: int = 20) -> dict:
    """The roofline denominators re-measured in this process, with the SM clock sampled
    while they run: a cuBLAS bf16 GEMM (gemm_n^3, back to back for a fraction of a second,
    like the timed step) and an HBM copy (read + write bytes).  Context for the kernel's
    fraction at the clock it ran at; the reported ``roofline.peak`` stays the measured
    MEASURED_PEAKS.json figure."""
    try:
        stream = torch.cuda.current_stream(dev)
        a = torch.randn(gemm_n, gemm_n, device=dev).to(torch.bfloat16)
        b = torch.randn(gemm_n, gemm_n, device=dev).to(torch.bfloat16)
        c = torch.empty(gemm_n, gemm_n, device=dev, dtype=torch.bfloat16)
        for _ in range(5):
            torch.matmul(a, b, out=c)
        torch.cuda.synchronize()
        evs = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(gemm_reps)]
        sampler = ClockSampler(local)
        sampler.start()
        time.sleep(0.2)
        for e0, e1 in evs:
            e0.record(stream)
            torch.matmul(a, b, out=c)
            e1.record(stream)
        torch.cuda.synchronize()
        gclk = sampler.stop()
        times = sorted(e0.elapsed_time(e1) for e0, e1 in evs)
        flops = 2.0 * gemm_n ** 3
        best = flops / (times[0] * 1e-3) / 1e12
        med = flops / (times[len(times) // 2] * 1e-3) / 1e12
        del a, b, c
        n_el = int(copy_gib * (1 << 30)) // 2
        x = torch.empty(n_el, dtype=torch.bfloat16, device=dev).normal_()
        y = torch.empty_like(x)
        for _ in range(3):
            y.copy_(x)
        torch.cuda.synchronize()
        cev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(copy_reps)]
        for e0, e1 in cev:
            e0.record(stream)
            y.copy_(x)
            e1.record(stream)
        torch.cuda.synchronize()
        ct = min(e0.elapsed_time(e1) for e0, e1 in cev)
        del x, y
        return {"bf16_gemm_tflops": round(best, 1), "bf16_gemm_tflops_median": round(med, 1),
                "gemm_sm_mhz": gclk.get("sm_mhz"), "gemm_clock_reasons": gclk.get("reasons"),
                "hbm_copy_gbs": round(2 * n_el * 2 / (ct * 1e-3) / 1e9, 1),
                "how": f"torch.matmul bf16 {gemm_n}^3 x {gemm_reps} back to back (best / median launch); "
                       f"copy of {copy_gib:g} GiB bf16, best of {copy_reps} (read + write bytes)"}
    except Exception as exc:  # context only: report why it is missing
        return {"unavailable": f"{type(exc).__name__}: {exc}"[:200]}


def attention_context(tg, dev, w, layers, s_k, gain, tau, S):
    """Per-layer time of the attention over the step's 27 layers (inputs larger than L2):
    the gated kernel, the same kernel without the key bias (plain causal attention), and,
    as context only, the library's causal attention (torch scaled_dot_product_attention)
    without and with an additive bias mask.  Outside the timed step."""
    stream = torch.cuda.current_stream(dev)
    L = len(layers)
    outs = [torch.empty(S, w.hq, w.head_dim, dtype=torch.bfloat16, device=dev) for _ in range(2)]

    def per_layer_us(fn, n_layers):
        for i in range(min(3, n_layers)):
            fn(i)
        torch.cuda.synchronize()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        for i in range(n_layers):
            fn(i)
        e1.record(stream)
        torch.cuda.synchronize()
        return e0.elapsed_time(e1) / n_layers * 1e3

    gated = per_layer_us(lambda i: tg.tg_gated_attention(*layers[i], s_k, gain, tau, O=outs[i & 1]), L)
    plain = per_layer_us(lambda i: tg.tg_gated_attention(*layers[i], None, None, tau, O=outs[i & 1]), L)
    out = {"gated_us_per_layer": round(gated, 2), "no_bias_us_per_layer": round(plain, 2),
           "bias_overhead": round(gated / plain, 4)}
    try:
        import torch.nn.functional as F
        n_lib = min(L, 6)
        lib_layers = [tuple(t.transpose(0, 1).unsqueeze(0).contiguous() for t in layers[i]) for i in range(n_lib)]
        scale = tau / math.sqrt(w.head_dim)
        sdpa = per_layer_us(lambda i: F.scaled_dot_product_attention(
            *lib_layers[i % n_lib], is_causal=True, scale=scale, enable_gqa=True), n_lib * 2)
        # an additive mask: causal -inf plus the bias of head 0 on every head (one mask)
        bias = (gain[0] * s_k).to(torch.bfloat16)
        mask = torch.full((S, S), float("-inf"), device=dev, dtype=torch.bfloat16).triu(1) + bias[None, :]
        sdpa_b = per_layer_us(lambda i: F.scaled_dot_product_attention(
            *lib_layers[i % n_lib], attn_mask=mask[None, None], scale=scale, enable_gqa=True), n_lib * 2)
        out.update({"library_sdpa_causal_us_per_layer": round(sdpa, 2),
                    "library_sdpa_bias_mask_us_per_layer": round(sdpa_b, 2),
                    "library": f"torch {torch.__version__} scaled_dot_product_attention, bf16, GQA"})
        del lib_layers, mask
    except Exception as exc:  # context only: report why it is missing
        out["library"] = f"unavailable: {type(exc).__name__}: {exc}"[:200]
    return out


def time_next_rows(tg, dev, w, host, dv, kept, S, reps=5):
    """Device time of the calls around the hot path on the same workload, outside the timed
    step: the pruned layer's projections, the attention backward (training forward + backward),
    random-K and a 4-budget sweep.  CUDA events on the launching stream, after one warm-up."""
    from learned_token_pruning_mlp_b200 import workloads as W
    peaks = load_peaks()
    stream = torch.cuda.current_stream(dev)
    Wq, Wo, qn, kn = (t.to(dev) for t in W.layer_weights(w))
    Q, Kc, V = host["layers"][0]
    Q, Kc, V = Q.to(dev), Kc.to(dev), V.to(dev)
    s_k = torch.randn(S, generator=torch.Generator().manual_seed(5)).to(dev)
    gain, tau = host["gain"].to(dev), host["tau"]
    hk = torch.randn(S, w.d, generator=torch.Generator().manual_seed(6)).to(torch.bfloat16).to(dev)
    pos = kept[:S].contiguous()
    q_o = torch.empty_like(Q)
    k_o, v_o = torch.empty_like(Kc), torch.empty_like(V)
    y = torch.empty(S, w.d, dtype=torch.bfloat16, device=dev)
    dO = torch.randn(S, w.hq, w.head_dim, generator=torch.Generator().manual_seed(7)).to(torch.bfloat16).to(dev)
    O, lse, O32 = tg.tg_gated_attention_train(Q, Kc, V, s_k, gain, tau)
    ds = torch.empty(S, device=dev)
    dg = torch.empty(w.hq, device=dev)
    dt = torch.empty(1, device=dev)
    ws = torch.empty(tg.tg_gated_attention_backward_workspace(S, w.hq), dtype=torch.uint8, device=dev)
    kr = torch.empty(w.n, dtype=torch.int32, device=dev)
    nkr = torch.empty(1, dtype=torch.int32, device=dev)
    ks = torch.tensor([2048, 4096, 8192, 16384], dtype=torch.int32, device=dev)
    ksw = torch.empty(4 * w.n, dtype=torch.int32, device=dev)
    nksw = torch.empty(4, dtype=torch.int32, device=dev)
    K = S - w.segments[0].q
    D, hq, hkv, d = w.head_dim, w.hq, w.hkv, w.d
    calls = {
        "qkv_rope": (lambda: tg.tg_qkv_rope(hk, Wq, pos, w.rope_base, hq, hkv, D, qn, kn, w.norm_eps,
                                            Q=q_o, Kc=k_o, V=v_o), 2 * S * (hq + 2 * hkv) * D * d, "tensor"),
        "o_proj_residual": (lambda: tg.tg_linear(O.view(S, hq * D), Wo, hk, y=y), 2 * S * d * hq * D, "tensor"),
        "attention_train_forward": (lambda: tg.tg_gated_attention_train(Q, Kc, V, s_k, gain, tau, O=O, lse=lse,
                                                                         O32=O32), attention_flops(S, hq, D), "tensor"),
        "attention_backward": (lambda: tg.tg_gated_attention_backward(Q, Kc, V, s_k, gain, tau, O, dO, lse, O32, ds,
                                                                      dg, dt, workspace=ws),
                               attention_flops(S, hq, D), "tensor"),
        "random_k": (lambda: tg.tg_select_random_k(dv["mask"], K, 42, kept_idx=kr, n_kept=nkr), w.n + S * 4, "latency"),
        "budget_sweep_4": (lambda: tg.tg_select_topk_sweep(dv["sel"], dv["mask"], ks, kept_idx=ksw, n_kept=nksw,
                                                           stride=w.n), w.n * 5, "latency"),
    }
    out = {}
    for name, (fn, work, bound) in calls.items():
        fn()
        torch.cuda.synchronize()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        for _ in range(reps):
            fn()
        e1.record(stream)
        torch.cuda.synchronize()
        us = e0.elapsed_time(e1) / reps * 1e3
        row = {"us": round(us, 2), "reps": reps}
        if bound == "tensor":
            tf = work / (us * 1e-6) / 1e12
            row.update({"tflops": round(tf, 1), "frac_of_bf16_peak": round(tf / peaks["bf16_tflops"], 4)})
        out[name] = row

    # The whole pruned layer above the gate, the workload's layers chained: x -> QKV +
    # per-head norm + rotary at the kept positions -> gated attention -> o_proj + residual
    # -> the next layer's x (synthetic weights per layer; the layer's MLP and norms are
    # outside the path).
    Ws = [tuple(t.to(dev) for t in W.layer_weights(w, l)) for l in range(w.layers)]
    bufs = [torch.empty_like(hk), torch.empty_like(hk)]
    O_c = torch.empty_like(Q)

    def chain():
        x = hk
        for l, (Wq_l, Wo_l, qn_l, kn_l) in enumerate(Ws):
            tg.tg_qkv_rope(x, Wq_l, pos, w.rope_base, hq, hkv, D, qn_l, kn_l, w.norm_eps, Q=q_o, Kc=k_o, V=v_o)
            tg.tg_gated_attention(q_o, k_o, v_o, s_k, gain, tau, O=O_c)
            y_l = bufs[l & 1]
            tg.tg_linear(O_c.view(S, hq * D), Wo_l, x, y=y_l)
            x = y_l

    chain()
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    chain()
    e1.record(stream)
    torch.cuda.synchronize()
    per_layer_us = e0.elapsed_time(e1) / len(Ws) * 1e3
    layer_flops = 2 * S * (hq + 2 * hkv) * D * d + attention_flops(S, hq, D) + 2 * S * d * hq * D
    tf = layer_flops / (per_layer_us * 1e-6) / 1e12
    out["pruned_layer_chain"] = {"layers": len(Ws), "us_per_layer": round(per_layer_us, 2),
                                 "flops_per_layer": layer_flops, "tflops": round(tf, 1),
                                 "frac_of_bf16_peak": round(tf / peaks["bf16_tflops"], 4),
                                 "calls": "tg_qkv_rope -> tg_gated_attention -> tg_linear (+ residual) per layer"}
    del Ws, bufs
    bits = tg.tg_get_device_error()
    if bits:
        raise RuntimeError(f"device status bits {bits} after the next-row timings")
    return out


def run_e2e(tg, host, dev, w, K, S, tau, world, args):
    pin = lambda t: t.pin_memory()
    h_in = {k: pin(host[k]) for k in ("hidden", "W1", "b1", "W2", "b2", "mask", "sel", "gain")}
    h_layers = [tuple(pin(t) for t in lay) for lay in host["layers"]]
    L = w.layers
    d_in = {k: torch.empty_like(v, device=dev) for k, v in h_in.items()}
    d_layers = [tuple(torch.empty_like(t, device=dev) for t in lay) for lay in h_layers]
    scores = torch.empty(w.n, dtype=torch.float32, device=dev)
    kept = torch.empty(w.n, dtype=torch.int32, device=dev)
    n_kept = torch.empty(1, dtype=torch.int32, device=dev)
    hidden_k = torch.empty(S, w.d, dtype=torch.bfloat16, device=dev)
    s_k = torch.empty(S, dtype=torch.float32, device=dev)
    outs = [torch.empty(S, w.hq, w.head_dim, dtype=torch.bfloat16, device=dev) for _ in range(L)]
    h_kept = torch.empty(S, dtype=torch.int32).pin_memory()
    h_outs = [torch.empty(S, w.hq, w.head_dim, dtype=torch.bfloat16).pin_memory() for _ in range(L)]
    h2d = sum(v.numel() * v.element_size() for v in h_in.values()) + \
        sum(t.numel() * t.element_size() for lay in h_layers for t in lay)
    d2h = h_kept.numel() * 4 + sum(o.numel() * o.element_size() for o in h_outs)

    comp = torch.cuda.current_stream(dev)
    h2d_stream, d2h_stream = torch.cuda.Stream(dev), torch.cuda.Stream(dev)

    def step():
        # Host-to-device copies on their own stream (the select path's inputs, then each
        # layer's Q/K/V in order), device-to-host reads of each result on another, so the
        # copies overlap the kernels; a step starts after the previous one has finished
        # (its device buffers are reused) and ends when its results are on the host.
        h2d_stream.wait_stream(comp)
        layer_ready = []
        with torch.cuda.stream(h2d_stream):
            for k in h_in:
                d_in[k].copy_(h_in[k], non_blocking=True)
            inputs_ready = torch.cuda.Event()
            inputs_ready.record(h2d_stream)
            for l in range(L):
                for a, b in zip(d_layers[l], h_layers[l]):
                    a.copy_(b, non_blocking=True)
                e = torch.cuda.Event()
                e.record(h2d_stream)
                layer_ready.append(e)
        comp.wait_event(inputs_ready)
        tg.tg_gate_score(d_in["hidden"], d_in["W1"], d_in["b1"], d_in["W2"], d_in["b2"], scores=scores)
        tg.tg_select_topk(d_in["sel"], d_in["mask"], K, kept_idx=kept, n_kept=n_kept)
        tg.tg_gather(d_in["hidden"], kept, n_rows=S, n_kept=n_kept, hidden_k=hidden_k, scores=d_in["sel"], s_k=s_k)
        sel_done = torch.cuda.Event()
        sel_done.record(comp)
        d2h_stream.wait_event(sel_done)
        with torch.cuda.stream(d2h_stream):
            h_kept.copy_(kept[:S], non_blocking=True)
        for l in range(L):
            comp.wait_event(layer_ready[l])
            Q, Kc, V = d_layers[l]
            tg.tg_gated_attention(Q, Kc, V, s_k, d_in["gain"], tau, O=outs[l])
            done = torch.cuda.Event()
            done.record(comp)
            d2h_stream.wait_event(done)
            with torch.cuda.stream(d2h_stream):
                h_outs[l].copy_(outs[l], non_blocking=True)
        comp.wait_stream(d2h_stream)

    steps = max(1, min(args.steps, 3))
    step()
    torch.cuda.synchronize()
    barrier(world)
    t0 = torch.cuda.Event(enable_timing=True)
    t1 = torch.cuda.Event(enable_timing=True)
    t0.record(comp)
    for _ in range(steps):
        step()
    t1.record(comp)
    torch.cuda.synchronize()
    ms = max_over_ranks(t0.elapsed_time(t1) / steps, world)
    flops = attention_flops(S, w.hq, w.head_dim) * L
    del d_in, d_layers, outs
    return {"value": round(world * flops / (ms * 1e-3) / 1e12, 3), "unit": "TFLOP/s", "ms_per_step": round(ms, 3),
            "h2d_bytes_per_step": int(h2d), "d2h_bytes_per_step": int(d2h), "steps": steps}


# ----------------------------------------------------------------------------- sweep
# Every named workload and budget: the 16k budgets, the 32k budgets and its full-context
# pass (K = N - 512, every document token kept), the 128k budgets, and the ragged batch.
SWEEP = [("qwen3_1p7b_n16k", 1024), ("qwen3_1p7b_n16k", 2048), ("qwen3_1p7b_n16k", 4096),
         ("qwen3_1p7b_n32k", 2048), ("qwen3_1p7b_n32k", 4096), ("qwen3_1p7b_n32k", 8192),
         ("qwen3_1p7b_n32k", 32256),
         ("qwen3_1p7b_n128k", 4096), ("qwen3_1p7b_n128k", 8192), ("qwen3_1p7b_n128k", 16384),
         ("ragged_4req", None)]


def run_sweep(args, local):
    """One JSON line per (workload, budget); see the module docstring."""
    import learned_token_pruning_mlp_b200 as tg
    from learned_token_pruning_mlp_b200 import build as tgbuild
    from learned_token_pruning_mlp_b200 import workloads as W
    tgbuild.build()
    dev = torch.device("cuda", local)
    torch.cuda.set_device(dev)
    peaks = load_peaks()
    flush = torch.empty(256 << 20, dtype=torch.uint8, device=dev)  # 256 MiB > the 126 MB L2
    only = set(args.sweep_only.split(",")) if args.sweep_only else None
    gate_cache = {}
    for name, K in SWEEP:
        if only and name not in only:
            continue
        w0 = W.get(name)
        if name not in gate_cache:
            gate_cache.clear()
            gate_cache[name] = (W.gate_inputs(w0), W.doc_mask(w0), W.selection_scores(w0))
        (hidden, W1, b1, W2, b2), mask, sel = gate_cache[name]
        line = sweep_line(tg, W, dev, local, w0, K, hidden, W1, b1, W2, b2, mask, sel, flush, peaks, args)
        print(json.dumps(line), flush=True)
        torch.cuda.empty_cache()


def sweep_line(tg, W, dev, local, w0, K, hidden, W1, b1, W2, b2, mask, sel, flush, peaks, args):
    stream = torch.cuda.current_stream(dev)
    varlen = w0.varlen
    w = w0 if varlen else w0.with_budget(K)
    segs = list(w.segments)
    kept_counts = [min(sg.k, sg.n - sg.q) + sg.q for sg in segs]
    S = sum(kept_counts)
    L = w.layers
    gain, tau = W.attention_params(w)
    layers_h = [W.attention_inputs(w, S, layer=l) for l in range(L)]
    n, d, h = w.n, w.d, w.h
    dv = {k: t.to(dev) for k, t in (("hidden", hidden), ("W1", W1), ("b1", b1), ("W2", W2), ("b2", b2),
                                     ("mask", mask), ("gain", gain))}
    dsel = sel.to(dev) if sel is not None else None
    layers = [tuple(t.to(dev) for t in lay) for lay in layers_h]
    scores = torch.empty(n, dtype=torch.float32, device=dev)
    kept = torch.empty(n, dtype=torch.int32, device=dev)
    n_kept = torch.empty(1, dtype=torch.int32, device=dev)
    hidden_k = torch.empty(S, d, dtype=torch.bfloat16, device=dev)
    s_k = torch.empty(S, dtype=torch.float32, device=dev)
    outs = [torch.empty(S, w.hq, w.head_dim, dtype=torch.bfloat16, device=dev) for _ in range(L)]
    if varlen:
        cu = w.cu_seqlens().to(dev)
        ks = torch.tensor([sg.k for sg in segs], dtype=torch.int32, device=dev)
        cu_kept = torch.empty(len(segs) + 1, dtype=torch.int32, device=dev)
        max_len = max(sg.n for sg in segs)
        max_kept = max(kept_counts)
        cu_kept_host = np.concatenate([[0], np.cumsum(kept_counts)]).astype(np.int32)

    def step(ev=None):
        if ev is not None:
            ev[0].record(stream)
        tg.tg_gate_score(dv["hidden"], dv["W1"], dv["b1"], dv["W2"], dv["b2"], scores=scores)
        src = dsel if dsel is not None else scores
        if varlen:
            tg.tg_select_topk_varlen(src, dv["mask"], cu, ks, max_len, kept_idx=kept, cu_kept=cu_kept)
            tg.tg_gather(dv["hidden"], kept, n_rows=S, hidden_k=hidden_k, scores=src, s_k=s_k)
        else:
            tg.tg_select_topk(src, dv["mask"], K, kept_idx=kept, n_kept=n_kept)
            tg.tg_gather(dv["hidden"], kept, n_rows=S, n_kept=n_kept, hidden_k=hidden_k, scores=src, s_k=s_k)
        if ev is not None:
            ev[1].record(stream)
        for l in range(L):
            Q, Kc, V = layers[l]
            if varlen:
                tg.tg_gated_attention_varlen(Q, Kc, V, s_k, dv["gain"], tau, cu_kept, max_kept, O=outs[l])
            else:
                tg.tg_gated_attention(Q, Kc, V, s_k, dv["gain"], tau, O=outs[l])
        if ev is not None:
            ev[2].record(stream)

    for _ in range(args.warmup):
        flush.zero_()
        step()
    torch.cuda.synchronize()
    bits = tg.tg_get_device_error()
    if bits & ~tg.TG_DEVERR_K_GT_NDOC:
        raise RuntimeError(f"{w.name} K={K}: device status bits {bits} after warm-up")
    if varlen:
        if not np.array_equal(cu_kept.cpu().numpy(), cu_kept_host):
            raise RuntimeError(f"{w.name}: kept counts differ from the budgets")
    elif int(n_kept.item()) != S:
        raise RuntimeError(f"{w.name} K={K}: kept {int(n_kept.item())} tokens, expected {S}")

    steps = args.sweep_steps
    evs = [[torch.cuda.Event(enable_timing=True) for _ in range(3)] for _ in range(steps)]
    sampler = ClockSampler(local)
    torch.cuda.synchronize()
    sampler.start()
    time.sleep(0.2)
    for i in range(steps):
        flush.zero_()  # L2 flushed before every step, outside the timed events
        step(evs[i])
    torch.cuda.synchronize()
    clocks = sampler.stop()
    if tg.tg_get_device_error() & ~tg.TG_DEVERR_K_GT_NDOC:
        raise RuntimeError(f"{w.name} K={K}: device status bits set during timing")
    sel_ms = statistics.mean(e[0].elapsed_time(e[1]) for e in evs)
    att_ms = statistics.mean(e[1].elapsed_time(e[2]) for e in evs)
    step_ms = statistics.mean(e[0].elapsed_time(e[2]) for e in evs)

    if varlen:
        flops_layer = sum(attention_flops(c, w.hq, w.head_dim) for c in kept_counts)
    else:
        flops_layer = attention_flops(S, w.hq, w.head_dim)
    att_us = att_ms / L * 1e3
    att_tf = flops_layer / (att_us * 1e-6) / 1e12
    sel_bytes = select_path_bytes(n, d, h, S)
    sel_gbs = sel_bytes / (sel_ms * 1e-3) / 1e9
    burst = peaks["bf16_tflops"]
    desc = (f"{w.name}: " + (", ".join(f"N={sg.n} (question {sg.q}, K={sg.k})" for sg in segs) if varlen else
                             f"N={n} (question {segs[0].q}), K={K}") +
            f", d={d}, gate {d}->{h}->1, S={S}, {L} gated layer{'s' if L > 1 else ''} Hq={w.hq} Hkv={w.hkv} "
            f"D={w.head_dim}" + (" (packed varlen calls)" if varlen else "") +
            (" (full context: every document token kept)" if not varlen and K >= segs[0].n - segs[0].q else ""))
    out = {"sweep": True, "metric": METRIC, "value": round(flops_layer * L / (step_ms * 1e-3) / 1e12, 2),
           "unit": "TFLOP/s", "n_gpus": 1, "steps": steps, "warmup": args.warmup, "ms_per_step": round(step_ms, 4),
           "higher_is_better": True, "dtype": "bf16", "data": "synthetic",
           "config": {"workload": desc, "global_batch": len(segs), "seq_len": n, "kept": S, "budget": K,
                      "l2": "flushed before every step (256 MiB write outside the timed events)"},
           "attention": {"us_per_layer": round(att_us, 2), "flops_per_layer": flops_layer, "tflops": round(att_tf, 1),
                         "frac_of_bf16_peak": round(att_tf / burst, 4),
                         "frac_of_bf16_sustained": round(att_tf / peaks["bf16_tflops_sustained"], 4),
                         "frac_of_nominal_2250": round(att_tf / NOMINAL_BF16_TFLOPS, 4)},
           "select_path": {"us": round(sel_ms * 1e3, 2), "bytes": sel_bytes, "gbs": round(sel_gbs, 1),
                           "frac_of_hbm": round(sel_gbs / peaks["hbm_gbs"], 4),
                           "frac_of_datasheet_8tbs": round(sel_gbs / DATASHEET_HBM_GBS, 4),
                           "scores": "fixed selector scores (mixture)" if sel is not None else "the gate's own output",
                           "timing": "in-step events, L2 cold"},
           "clocks": clocks}
    if not args.no_cpu_baseline:
        if varlen:
            b = int(np.argmax(kept_counts))
            lo, hi = int(cu_kept_host[b]), int(cu_kept_host[b + 1])
            lay = tuple(t[lo:hi].contiguous() for t in layers_h[0])
            cb = cpu_baseline(lay, gain, tau, w, hi - lo, budget_s=args.sweep_cpu_seconds, one_core=False)
            cb["sample"] += f" (request {b}, the longest)"
        else:
            cb = cpu_baseline(layers_h[0], gain, tau, w, S, budget_s=args.sweep_cpu_seconds,
                              one_core=(w.name == "qwen3_1p7b_n16k"))
        out["cpu_baseline"] = cb
    del layers, outs, dv
    return out


# ----------------------------------------------------------------------------- oracle (CPU) arm
def cpu_baseline(layer, gain, tau, w, S, budget_s: float = 10.0, steps: int = 1, one_core: bool = True):
    """Time the fp64 CPU oracle on a bounded row sample of one attention layer
    (``layer`` = its Q, K, V on the host); report TFLOP/s."""
    import oracle
    Q, K, V = layer
    s = torch.zeros(S)  # the key bias does not change the amount of work
    # calibrate: rows near the end of the sequence cost ~S*4*D*Hq flops each
    probe = np.arange(max(0, S - 4), S, dtype=np.int64)
    t0 = time.perf_counter()
    oracle.gated_attention(Q, K, V, s, gain, tau, rows=probe)
    dt = max(time.perf_counter() - t0, 1e-6)
    per_row = dt / len(probe)
    n_rows = int(max(min(4, S), min(S, budget_s / per_row)))
    rows = np.arange(S - n_rows, S, dtype=np.int64)
    flops = sum(4 * w.head_dim * w.hq * (int(r) + 1) for r in rows)
    times = []
    for _ in range(steps):
        t0 = time.perf_counter()
        oracle.gated_attention(Q, K, V, s, gain, tau, rows=rows)
        times.append(time.perf_counter() - t0)
    el = min(times)
    full = attention_flops(S, w.hq, w.head_dim)
    cores = oracle.num_threads()
    out = {"value": round(flops / el / 1e12, 6), "unit": "TFLOP/s", "cores": cores,
           "kind": "oracle",
           "sample": f"fp64 C oracle, gated attention layer 0, last {n_rows} of {S} query rows x {w.hq} heads "
                     f"(the longest causal rows), {flops:.3e} flops in {el:.2f} s",
           "rows_per_s": round(n_rows / el, 2),
           "extrapolated_full_layer_s": round(full / (flops / el), 2),
           "affinity_cores": len(os.sched_getaffinity(0)), "cpu_model": host_cpu_model()}
    if one_core:
        # the same oracle on one core, on the last few rows (a few seconds)
        oracle.set_num_threads(1)
        try:
            n1 = int(max(min(2, S), min(n_rows, budget_s / 4 / (per_row * cores))))
            rows1 = np.arange(S - n1, S, dtype=np.int64)
            flops1 = sum(4 * w.head_dim * w.hq * (int(r) + 1) for r in rows1)
            t0 = time.perf_counter()
            oracle.gated_attention(Q, K, V, s, gain, tau, rows=rows1)
            el1 = time.perf_counter() - t0
        finally:
            oracle.set_num_threads(cores)
        out["one_core"] = {"value": round(flops1 / el1 / 1e12, 6), "unit": "TFLOP/s",
                           "sample": f"last {n1} query rows x {w.hq} heads, {flops1:.3e} flops in {el1:.2f} s"}
    return out


def host_cpu_model() -> str:
    """The host CPU's model name (Linux /proc/cpuinfo), for the oracle's timing record."""
    try:
        with open("/proc/cpuinfo") as fh:
            for line in fh:
                if line.startswith("model name"):
                    return line.split(":", 1)[1].strip()
    except OSError:
        pass
    return "unknown"


def run_reference(args, world, rank):
    """The slow oracle on the host cores, on the same workload (bounded sample per step)."""
    if rank != 0:
        return None
    from learned_token_pruning_mlp_b200 import workloads as W
    import oracle
    w = W.get(WORKLOAD)
    K = args.budget
    q = w.segments[0].q
    S = K + q
    Q, Kc, V = W.attention_inputs(w, S, layer=0)
    gain, tau = W.attention_params(w)
    s = W.random_scores(S, 0)
    n_rows = max(2, int(args.ref_rows))
    rows = np.arange(S - n_rows, S, dtype=np.int64)
    flops = sum(4 * w.head_dim * w.hq * (int(r) + 1) for r in rows)
    for _ in range(args.warmup):
        oracle.gated_attention(Q, Kc, V, s, gain, tau, rows=rows[:2])
    t0 = time.perf_counter()
    for _ in range(args.steps):
        oracle.gated_attention(Q, Kc, V, s, gain, tau, rows=rows)
    el = (time.perf_counter() - t0) / args.steps
    val = flops / el / 1e12
    sample = (f"fp64 C oracle, gated attention layer 0 of {WORKLOAD} (S={S}), last {n_rows} query rows x "
              f"{w.hq} heads per step ({flops:.3e} flops)")
    return {"impl": "reference", "metric": METRIC, "value": round(val, 6), "unit": "TFLOP/s", "n_gpus": world,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": round(el * 1e3, 3), "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
            "config": workload_config(world, K, S, w.layers, w.n),
            "cpu_baseline": {"value": round(val, 6), "unit": "TFLOP/s", "cores": oracle.num_threads(),
                             "kind": "oracle", "sample": sample,
                             "affinity_cores": len(os.sched_getaffinity(0)), "cpu_model": host_cpu_model()},
            "e2e": {"value": round(val, 6), "unit": "TFLOP/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=30)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--impl", choices=["tokengate", "reference"], default="tokengate")
    ap.add_argument("--budget", type=int, default=8192)
    ap.add_argument("--cpu-seconds", type=float, default=10.0)
    ap.add_argument("--ref-rows", type=int, default=48)
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--sweep", action="store_true", help="one JSON line per (workload, budget)")
    ap.add_argument("--sweep-only", default="", help="comma-separated workload names for --sweep")
    ap.add_argument("--sweep-steps", type=int, default=10)
    ap.add_argument("--sweep-cpu-seconds", type=float, default=3.0)
    args = ap.parse_args()
    if args.warmup < 3:
        ap.error("--warmup must be at least 3")
    if args.sweep:
        if int(os.environ.get("WORLD_SIZE", "1")) > 1 or args.impl != "tokengate":
            ap.error("--sweep runs the product arm on one GPU")
        run_sweep(args, int(os.environ.get("LOCAL_RANK", "0")))
        return

    if args.impl == "reference":
        world = int(os.environ.get("WORLD_SIZE", "1"))
        rank = int(os.environ.get("RANK", "0"))
        out = run_reference(args, world, rank)
        if out is not None:
            print(json.dumps(out), flush=True)
        return

    world, rank, local = dist_setup(args.gpus)
    try:
        out = run_tokengate(args, world, rank, local)
        if rank == 0:
            print(json.dumps(out), flush=True)
    finally:
        if world > 1:
            torch.distributed.destroy_process_group()


if __name__ == "__main__":
    main()

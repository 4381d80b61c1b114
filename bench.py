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
``attention.context`` compares, outside the timed step, the kernel with and without
the key bias and the library's causal attention on the same layers.
``next_rows`` gives the device time of the calls around the path on the same
workload, outside the timed step: the pruned layer's projections, the attention
backward, random-K and a 4-budget sweep.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl {tokengate,reference}]
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

# DRAM traffic (dram__bytes_read.sum + dram__bytes_write.sum) of one attention launch at
# S = 8704, from one ncu capture of the kernel (its summary is kept with the profiles).
# It is reported only while the kernel sources are the ones that capture measured.
ATTENTION_TRAFFIC = {"sources_sha1": "743548f20766cd6c49c4c9f7fb5019e1ff6048a2", "bytes_per_launch": 72093184 + 9845248}


def attention_traffic():
    import hashlib
    h = hashlib.sha1()
    for f in ("attention.cu", "ptx.cuh"):
        with open(os.path.join(ROOT, "learned_token_pruning_mlp_b200", "csrc", f), "rb") as fh:
            h.update(fh.read())
    return ATTENTION_TRAFFIC["bytes_per_launch"] if h.hexdigest() == ATTENTION_TRAFFIC["sources_sha1"] else None


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
    sel_iters = max(10, args.steps)

    def select_only():
        tg.tg_gate_score(dv["hidden"], dv["W1"], dv["b1"], dv["W2"], dv["b2"], scores=scores)
        tg.tg_select_topk(dv["sel"], dv["mask"], K, kept_idx=kept, n_kept=n_kept)
        tg.tg_gather(dv["hidden"], kept, n_rows=S, n_kept=n_kept, hidden_k=hidden_k, scores=dv["sel"], s_k=s_k)

    for _ in range(3):
        select_only()
    barrier(world)
    torch.cuda.synchronize()
    s0, s1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    s0.record(stream)
    for _ in range(sel_iters):
        select_only()
    s1.record(stream)
    torch.cuda.synchronize()
    sel_b2b_us = max_over_ranks(s0.elapsed_time(s1) / sel_iters * 1e3, world)
    sel_b2b_gbs = sel_bytes / (sel_b2b_us * 1e-6) / 1e9

    # end to end through the public calls with host buffers: H2D of the step's inputs
    # from pinned memory and D2H of its results inside the timed region
    e2e = run_e2e(tg, host, dev, w, K, S, tau, world, args)
    next_rows = time_next_rows(tg, dev, w, host, dv, kept, S)
    attn_ctx = attention_context(tg, dev, w, layers, s_k, dv["gain"], tau, S)

    out = {
        "metric": METRIC, "value": round(value, 2), "unit": "TFLOP/s", "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": round(ms_per_step, 4), "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "bf16", "data": "synthetic",
        "config": workload_config(world, K, S, L, n),
        "attention": {"ms_per_layer": round(att_launch_ms, 4), "tflops": round(att_tflops, 1),
                      "frac_of_bf16_peak": round(att_tflops / peaks["bf16_tflops"], 4),
                      "frac_of_bf16_sustained": round(att_tflops / peaks["bf16_tflops_sustained"], 4),
                      "frac_of_nominal_2250": round(att_tflops / 2250.0, 4), "context": attn_ctx},
        "select_path": {"us": round(sel_b2b_us, 2), "bytes": sel_bytes, "gbs": round(sel_b2b_gbs, 1),
                        "frac_of_hbm": round(sel_b2b_gbs / peaks["hbm_gbs"], 4),
                        "frac_of_datasheet_8tbs": round(sel_b2b_gbs / DATASHEET_HBM_GBS, 4),
                        "timing": f"{sel_iters} back-to-back gate->top-K->gather passes",
                        "in_step_us": round(sel_mean * 1e3, 2),
                        "in_step_gbs": round(sel_gbs, 1),
                        "in_step_frac_of_hbm": round(sel_gbs / peaks["hbm_gbs"], 4)},
        "roofline": {"bound": "tensor", "achieved": round(att_tflops, 1), "peak": peaks["bf16_tflops_sustained"],
                     "unit": "TFLOP/s", "frac": round(att_tflops / peaks["bf16_tflops_sustained"], 4),
                     "traffic": attention_traffic(), "kernel": "gated_attention_kernel<128>",
                     "peak_source": f"{peaks['source']} bf16 sustained (kernel timed inside a long step)"},
        "e2e": e2e,
        "next_rows": next_rows,
        "gpu_launches": args.steps * (3 + L),
        "clocks": clocks,
    }
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        out["cpu_baseline"] = cpu_baseline(host, w, S, budget_s=args.cpu_seconds)
    return out


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


# ----------------------------------------------------------------------------- oracle (CPU) arm
def cpu_baseline(host, w, S, budget_s: float = 10.0, steps: int = 1):
    """Time the fp64 CPU oracle on a bounded row sample of layer 0's attention; report TFLOP/s."""
    import oracle
    gain, tau = host["gain"], host["tau"]
    Q, K, V = host["layers"][0]
    s = torch.zeros(S)  # the key bias does not change the amount of work
    # calibrate: rows near the end of the sequence cost ~S*4*D*Hq flops each
    probe = np.arange(S - 4, S, dtype=np.int64)
    t0 = time.perf_counter()
    oracle.gated_attention(Q, K, V, s, gain, tau, rows=probe)
    dt = max(time.perf_counter() - t0, 1e-6)
    per_row = dt / len(probe)
    n_rows = int(max(4, min(S, budget_s / per_row)))
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
    # the same oracle on one core, on the last few rows (a few seconds)
    oracle.set_num_threads(1)
    try:
        n1 = int(max(2, min(n_rows, budget_s / 4 / (per_row * cores))))
        rows1 = np.arange(S - n1, S, dtype=np.int64)
        flops1 = sum(4 * w.head_dim * w.hq * (int(r) + 1) for r in rows1)
        t0 = time.perf_counter()
        oracle.gated_attention(Q, K, V, s, gain, tau, rows=rows1)
        el1 = time.perf_counter() - t0
    finally:
        oracle.set_num_threads(cores)
    return {"value": round(flops / el / 1e12, 6), "unit": "TFLOP/s", "cores": cores,
            "kind": "oracle",
            "sample": f"fp64 C oracle, gated attention layer 0, last {n_rows} of {S} query rows x {w.hq} heads "
                      f"(the longest causal rows), {flops:.3e} flops in {el:.2f} s",
            "rows_per_s": round(n_rows / el, 2),
            "extrapolated_full_layer_s": round(full / (flops / el), 2),
            "affinity_cores": len(os.sched_getaffinity(0)), "cpu_model": host_cpu_model(),
            "one_core": {"value": round(flops1 / el1 / 1e12, 6), "unit": "TFLOP/s",
                         "sample": f"last {n1} query rows x {w.hq} heads, {flops1:.3e} flops in {el1:.2f} s"}}


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
    args = ap.parse_args()
    if args.warmup < 3:
        ap.error("--warmup must be at least 3")

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

"""Run one TokenGate call repeatedly on seeded inputs (for profilers and quick timing).

    python -m learned_token_pruning_mlp_b200.runone attention --S 8704 --repeat 3
    python -m learned_token_pruning_mlp_b200.runone gate --n 131072
    python -m learned_token_pruning_mlp_b200.runone topk --n 131072 --k 8192
    python -m learned_token_pruning_mlp_b200.runone randomk --n 131072 --k 8192
    python -m learned_token_pruning_mlp_b200.runone sweep --n 131072 --k 8192   # budgets k/4, k/2, k, 2k
    python -m learned_token_pruning_mlp_b200.runone gather --n 131072 --rows 8704
    python -m learned_token_pruning_mlp_b200.runone qkv --S 8704        # QKV + norm + rotary
    python -m learned_token_pruning_mlp_b200.runone oproj --S 8704      # output projection + residual
    python -m learned_token_pruning_mlp_b200.runone attnbwd --S 8704    # backward w.r.t. s, gain, tau
    python -m learned_token_pruning_mlp_b200.runone fused --graph       # gate -> top-K -> gather, one call
    python -m learned_token_pruning_mlp_b200.runone chain --graph       # the same as three calls

Each call is timed with CUDA events on the launching stream (after one warm-up
call) and the mean per-call time is printed.  Shapes default to the 128k-context
Qwen3-1.7B-like workload (d 2048, h 256, Hq 16, Hkv 8, D 128).
"""
from __future__ import annotations

import argparse
import math

import torch

from . import _lib as tg
from . import build as tgbuild
from . import workloads as W


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("call", choices=["gate", "topk", "randomk", "sweep", "gather", "attention", "qkv", "oproj", "attnbwd", "fused", "chain"])
    ap.add_argument("--n", type=int, default=131072)
    ap.add_argument("--d", type=int, default=2048)
    ap.add_argument("--h", type=int, default=256)
    ap.add_argument("--k", type=int, default=8192)
    ap.add_argument("--rows", type=int, default=8704)
    ap.add_argument("--S", type=int, default=8704)
    ap.add_argument("--hq", type=int, default=16)
    ap.add_argument("--hkv", type=int, default=8)
    ap.add_argument("--D", type=int, default=128)
    ap.add_argument("--tau", type=float, default=1.1)
    ap.add_argument("--repeat", type=int, default=3)
    ap.add_argument("--graph", action="store_true", help="time a CUDA-graph replay of the calls")
    a = ap.parse_args()
    tgbuild.build()
    dev = torch.device("cuda:0")
    g = torch.Generator(device="cpu").manual_seed(0)

    if a.call == "gate":
        hidden = torch.randn(a.n, a.d, generator=g).to(torch.bfloat16).to(dev)
        W1 = (torch.randn(a.h, a.d, generator=g) / math.sqrt(a.d)).to(torch.bfloat16).to(dev)
        b1 = torch.zeros(a.h, dtype=torch.bfloat16, device=dev)
        W2 = (torch.randn(a.h, generator=g) / math.sqrt(a.h)).to(torch.bfloat16).to(dev)
        b2 = torch.zeros(1, dtype=torch.bfloat16, device=dev)
        out = torch.empty(a.n, dtype=torch.float32, device=dev)
        fn = lambda: tg.tg_gate_score(hidden, W1, b1, W2, b2, scores=out)
    elif a.call == "topk":
        s = W.mixture_scores(a.n, 3).to(dev)
        m = torch.ones(a.n, dtype=torch.uint8, device=dev)
        m[-512:] = 0
        kept = torch.empty(a.n, dtype=torch.int32, device=dev)
        nk = torch.empty(1, dtype=torch.int32, device=dev)
        fn = lambda: tg.tg_select_topk(s, m, a.k, kept_idx=kept, n_kept=nk)
    elif a.call == "randomk":
        m = torch.ones(a.n, dtype=torch.uint8, device=dev)
        m[-512:] = 0
        kept = torch.empty(a.n, dtype=torch.int32, device=dev)
        nk = torch.empty(1, dtype=torch.int32, device=dev)
        fn = lambda: tg.tg_select_random_k(m, a.k, 42, kept_idx=kept, n_kept=nk)
    elif a.call == "sweep":
        s = W.mixture_scores(a.n, 3).to(dev)
        m = torch.ones(a.n, dtype=torch.uint8, device=dev)
        m[-512:] = 0
        ks = torch.tensor([a.k // 4, a.k // 2, a.k, 2 * a.k], dtype=torch.int32, device=dev)
        kept = torch.empty(4 * a.n, dtype=torch.int32, device=dev)
        nk = torch.empty(4, dtype=torch.int32, device=dev)
        fn = lambda: tg.tg_select_topk_sweep(s, m, ks, kept_idx=kept, n_kept=nk, stride=a.n)
    elif a.call == "gather":
        hidden = torch.randn(a.n, a.d, generator=g).to(torch.bfloat16).to(dev)
        sc = torch.randn(a.n, generator=g).to(dev)
        idx = torch.sort(torch.randperm(a.n, generator=g)[:a.rows]).values.to(torch.int32).to(dev)
        hk = torch.empty(a.rows, a.d, dtype=torch.bfloat16, device=dev)
        sk = torch.empty(a.rows, dtype=torch.float32, device=dev)
        fn = lambda: tg.tg_gather(hidden, idx, hidden_k=hk, scores=sc, s_k=sk)
    elif a.call == "qkv":
        x = torch.randn(a.S, a.d, generator=g).to(torch.bfloat16).to(dev)
        Wq = (torch.randn((a.hq + 2 * a.hkv) * a.D, a.d, generator=g) / math.sqrt(a.d)).to(torch.bfloat16).to(dev)
        qn = torch.ones(a.D, dtype=torch.bfloat16, device=dev)
        pos = torch.sort(torch.randperm(a.n, generator=g)[:a.S]).values.to(torch.int32).to(dev)
        Q = torch.empty(a.S, a.hq, a.D, dtype=torch.bfloat16, device=dev)
        K = torch.empty(a.S, a.hkv, a.D, dtype=torch.bfloat16, device=dev)
        V = torch.empty_like(K)
        fn = lambda: tg.tg_qkv_rope(x, Wq, pos, 1e6, a.hq, a.hkv, a.D, qn, qn, 1e-6, Q=Q, Kc=K, V=V)
    elif a.call == "oproj":
        x = torch.randn(a.S, a.hq * a.D, generator=g).to(torch.bfloat16).to(dev)
        Wo = (torch.randn(a.d, a.hq * a.D, generator=g) / math.sqrt(a.hq * a.D)).to(torch.bfloat16).to(dev)
        res = torch.randn(a.S, a.d, generator=g).to(torch.bfloat16).to(dev)
        y = torch.empty(a.S, a.d, dtype=torch.bfloat16, device=dev)
        fn = lambda: tg.tg_linear(x, Wo, res, y=y)
    elif a.call in ("fused", "chain"):
        hidden = torch.randn(a.n, a.d, generator=g).to(torch.bfloat16).to(dev)
        W1 = (torch.randn(a.h, a.d, generator=g) / math.sqrt(a.d)).to(torch.bfloat16).to(dev)
        b1 = torch.zeros(a.h, dtype=torch.bfloat16, device=dev)
        W2 = (torch.randn(a.h, generator=g) / math.sqrt(a.h)).to(torch.bfloat16).to(dev)
        b2 = torch.zeros(1, dtype=torch.bfloat16, device=dev)
        m = torch.ones(a.n, dtype=torch.uint8, device=dev)
        m[-512:] = 0
        S = a.k + 512
        sc = torch.empty(a.n, dtype=torch.float32, device=dev)
        kept = torch.empty(a.n, dtype=torch.int32, device=dev)
        nk = torch.empty(1, dtype=torch.int32, device=dev)
        hk = torch.empty(S, a.d, dtype=torch.bfloat16, device=dev)
        sk = torch.empty(S, dtype=torch.float32, device=dev)
        ws = torch.empty(tg.tg_select_fused_workspace(a.n), dtype=torch.uint8, device=dev)
        if a.call == "fused":
            fn = lambda: tg.tg_select_fused(hidden, W1, b1, W2, b2, m, a.k, n_rows=S, scores=sc, kept_idx=kept,
                                            n_kept=nk, hidden_k=hk, s_k=sk, workspace=ws)
        else:
            def fn():
                tg.tg_gate_score(hidden, W1, b1, W2, b2, scores=sc)
                tg.tg_select_topk(sc, m, a.k, kept_idx=kept, n_kept=nk)
                tg.tg_gather(hidden, kept, n_rows=S, n_kept=nk, hidden_k=hk, scores=sc, s_k=sk)
    elif a.call == "attnbwd":
        Q = torch.randn(a.S, a.hq, a.D, generator=g).to(torch.bfloat16).to(dev)
        K = torch.randn(a.S, a.hkv, a.D, generator=g).to(torch.bfloat16).to(dev)
        V = torch.randn(a.S, a.hkv, a.D, generator=g).to(torch.bfloat16).to(dev)
        dO = torch.randn(a.S, a.hq, a.D, generator=g).to(torch.bfloat16).to(dev)
        s = torch.randn(a.S, generator=g).to(dev)
        gain = (0.5 + torch.rand(a.hq, generator=g)).to(dev)
        O, lse, O32 = tg.tg_gated_attention_train(Q, K, V, s, gain, a.tau)
        ds = torch.empty(a.S, device=dev)
        dg = torch.empty(a.hq, device=dev)
        dt = torch.empty(1, device=dev)
        ws = torch.empty(tg.tg_gated_attention_backward_workspace(a.S, a.hq), dtype=torch.uint8, device=dev)
        fn = lambda: tg.tg_gated_attention_backward(Q, K, V, s, gain, a.tau, O, dO, lse, O32, ds, dg, dt, workspace=ws)
    else:
        Q = torch.randn(a.S, a.hq, a.D, generator=g).to(torch.bfloat16).to(dev)
        K = torch.randn(a.S, a.hkv, a.D, generator=g).to(torch.bfloat16).to(dev)
        V = torch.randn(a.S, a.hkv, a.D, generator=g).to(torch.bfloat16).to(dev)
        s = torch.randn(a.S, generator=g).to(dev)
        gain = (0.5 + torch.rand(a.hq, generator=g)).to(dev)
        O = torch.empty_like(Q)
        fn = lambda: tg.tg_gated_attention(Q, K, V, s, gain, a.tau, O=O)

    fn()
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    if a.graph:
        # replay the calls from a CUDA graph so host-side call overhead does not leave the
        # GPU idle between launches of a short kernel
        stream = torch.cuda.Stream()
        graph = torch.cuda.CUDAGraph()
        with torch.cuda.stream(stream):
            with torch.cuda.graph(graph, stream=stream):
                for _ in range(a.repeat):
                    fn()
        graph.replay()
        torch.cuda.synchronize()
        e0.record()
        graph.replay()
        e1.record()
    else:
        e0.record()
        for _ in range(a.repeat):
            fn()
        e1.record()
    torch.cuda.synchronize()
    ms = e0.elapsed_time(e1) / a.repeat
    bits = tg.tg_get_device_error()
    extra = ""
    if a.call in ("attention", "attnbwd"):
        fl = 4 * a.D * a.hq * a.S * (a.S + 1) / 2
        extra = f" {fl / ms / 1e9:.1f} TFLOP/s"
    elif a.call in ("fused", "chain"):
        S = a.k + 512
        by = a.n * a.d * 2 + a.h * a.d * 2 + a.n * 4 + a.n * 4 + a.n + S * 4 + 2 * S * a.d * 2 + 2 * S * 4
        extra = f" {by / ms / 1e6:.1f} GB/s algorithmic"
    elif a.call in ("qkv", "oproj"):
        n_out = (a.hq + 2 * a.hkv) * a.D if a.call == "qkv" else a.d
        k_in = a.d if a.call == "qkv" else a.hq * a.D
        extra = f" {2 * a.S * n_out * k_in / ms / 1e9:.1f} TFLOP/s"
    print(f"{a.call}: {ms * 1e3:.1f} us per call{extra} (status bits {bits})")
    if bits:
        raise SystemExit(1)


if __name__ == "__main__":
    main()

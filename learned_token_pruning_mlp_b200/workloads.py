"""Seeded synthetic inputs for the TokenGate pruned-prefill hot path.

This module only draws random tensors with the shapes, value distributions and
structure of the workloads the TokenGate article describes (Qwen3-1.7B-shaped
layers, batch 1, contexts 16k-128k, a question at the end of the prompt that is
never pruned).  It holds none of the method's arithmetic: no gate, no selection,
no attention.  Both the CUDA path (through the tests and the bench) and the CPU
oracle are fed from here, so the two sides always see identical bytes.

Every tensor comes from its own ``torch.Generator`` seeded from
(workload seed, tag), so drawing one input never shifts another.
All tensors are created on the CPU; callers move them to the device.
"""
from __future__ import annotations

import dataclasses
import math
from typing import Optional, Sequence

import torch

# Tags that separate the random streams of one workload.
_TAG = {
    "hidden": 1, "needles": 2, "w1": 3, "b1": 4, "w2": 5, "b2": 6,
    "gain": 7, "q": 8, "k": 9, "v": 10, "mix_base": 11, "mix_pick": 12,
    "mix_tail": 13, "ties": 14, "sel": 15, "wqkv": 16, "wo": 17, "qn": 18, "kn": 19,
}


def _gen(seed: int, tag: str, sub: int = 0) -> torch.Generator:
    g = torch.Generator(device="cpu")
    g.manual_seed((seed * 1_000_003 + _TAG[tag] * 7_919 + sub * 104_729) & 0x7FFF_FFFF_FFFF)
    return g


@dataclasses.dataclass(frozen=True)
class Segment:
    """One request of a packed batch: ``n`` prompt tokens, the last ``q`` of them the question."""
    n: int
    q: int
    k: int  # kept document-token budget

    @property
    def n_doc(self) -> int:
        return self.n - self.q


@dataclasses.dataclass(frozen=True)
class Workload:
    name: str
    segments: Sequence[Segment]       # one entry for a single sequence
    d: int                            # hidden width of the residual
    h: int                            # gate MLP width
    hq: int                           # query heads above the gate
    hkv: int                          # key/value heads above the gate
    head_dim: int                     # D
    seed: int
    budgets: Sequence[int] = ()       # budget sweep (single-sequence workloads)
    layers: int = 1                   # gated-attention layers above the gate
    needle_frac: float = 0.0          # share of document positions scaled x4
    score_mixture: bool = False       # selection scores drawn from N(0,1)+2% N(4,1)
    tau: float = 1.1
    rope_base: float = 1e6            # Qwen3's rotary base
    norm_eps: float = 1e-6            # Qwen3's RMS-norm epsilon

    @property
    def n(self) -> int:
        return sum(s.n for s in self.segments)

    @property
    def varlen(self) -> bool:
        return len(self.segments) > 1

    def cu_seqlens(self) -> torch.Tensor:
        out = [0]
        for s in self.segments:
            out.append(out[-1] + s.n)
        return torch.tensor(out, dtype=torch.int32)

    def with_budget(self, k: int) -> "Workload":
        assert not self.varlen
        s = self.segments[0]
        return dataclasses.replace(self, segments=(Segment(s.n, s.q, k),))


def _single(name, n, q, k, **kw) -> Workload:
    return Workload(name=name, segments=(Segment(n, q, k),), **kw)


# The named workloads.  Shapes follow the article's dense Qwen3-1.7B setting
# (hidden 2048, 16 query heads, 8 KV heads, head dim 128) at batch 1.
WORKLOADS = {
    # Tiny case that the oracle finishes in milliseconds.
    "tiny_n512": _single("tiny_n512", 512, 64, 128, d=256, h=64, hq=4, hkv=2,
                         head_dim=64, seed=0, budgets=(128,)),
    # One gated layer at 16k with 1% "needle" residuals.
    "qwen3_1p7b_n16k": _single("qwen3_1p7b_n16k", 16384, 512, 2048, d=2048, h=256,
                               hq=16, hkv=8, head_dim=128, seed=1,
                               budgets=(1024, 2048, 4096), needle_frac=0.01),
    # 32k, plus a full-context budget (every document token kept).
    "qwen3_1p7b_n32k": _single("qwen3_1p7b_n32k", 32768, 512, 4096, d=2048, h=256,
                               hq=16, hkv=8, head_dim=128, seed=1,
                               budgets=(2048, 4096, 8192, 32256)),
    # 128k long-context sweep: gate at layer 1, 27 gated layers above it.
    "qwen3_1p7b_n128k": _single("qwen3_1p7b_n128k", 131072, 512, 8192, d=2048, h=256,
                                hq=16, hkv=8, head_dim=128, seed=3,
                                budgets=(4096, 8192, 16384), layers=27,
                                score_mixture=True),
    # Ragged batch of four packed requests, budget N/8 each.
    "ragged_4req": Workload(name="ragged_4req",
                            segments=(Segment(8192, 128, 1024), Segment(24576, 256, 3072),
                                      Segment(49152, 512, 6144), Segment(65536, 1024, 8192)),
                            d=2048, h=256, hq=16, hkv=8, head_dim=128, seed=4),
}


def get(name: str) -> Workload:
    return WORKLOADS[name]


def _randn_bf16(shape, g, scale: float = 1.0) -> torch.Tensor:
    x = torch.randn(shape, generator=g, dtype=torch.float32)
    if scale != 1.0:
        x = x * scale
    return x.to(torch.bfloat16)


def doc_mask(w: Workload) -> torch.Tensor:
    """uint8[n]: 1 for document tokens, 0 for question tokens (question at the end of each request)."""
    parts = []
    for s in w.segments:
        m = torch.ones(s.n, dtype=torch.uint8)
        if s.q:
            m[s.n - s.q:] = 0
        parts.append(m)
    return torch.cat(parts)


def gate_inputs(w: Workload):
    """Residual stream at the gate layer plus gate weights, all bf16.

    hidden ~ N(0,1) (a chosen share of document rows scaled by 4 as needles);
    W1 [h,d], b1 [h] ~ N(0, 1/d); W2 [h], b2 [1] ~ N(0, 1/h).
    """
    hidden = torch.randn((w.n, w.d), generator=_gen(w.seed, "hidden"), dtype=torch.float32)
    if w.needle_frac > 0:
        mask = doc_mask(w).bool()
        doc_pos = torch.nonzero(mask).flatten()
        n_needles = max(1, int(round(w.needle_frac * doc_pos.numel())))
        pick = torch.randperm(doc_pos.numel(), generator=_gen(w.seed, "needles"))[:n_needles]
        hidden[doc_pos[pick]] *= 4.0
    hidden = hidden.to(torch.bfloat16)
    W1 = _randn_bf16((w.h, w.d), _gen(w.seed, "w1"), 1.0 / math.sqrt(w.d))
    b1 = _randn_bf16((w.h,), _gen(w.seed, "b1"), 1.0 / math.sqrt(w.d))
    W2 = _randn_bf16((w.h,), _gen(w.seed, "w2"), 1.0 / math.sqrt(w.h))
    b2 = _randn_bf16((1,), _gen(w.seed, "b2"), 1.0 / math.sqrt(w.h))
    return hidden, W1, b1, W2, b2


def mixture_scores(n: int, seed: int, tail_frac: float = 0.02) -> torch.Tensor:
    """fp32[n] drawn from N(0,1) with a ``tail_frac`` share replaced by N(4,1)."""
    base = torch.randn(n, generator=_gen(seed, "mix_base"), dtype=torch.float32)
    pick = torch.rand(n, generator=_gen(seed, "mix_pick")) < tail_frac
    tail = torch.randn(n, generator=_gen(seed, "mix_tail"), dtype=torch.float32) + 4.0
    return torch.where(pick, tail, base)


def selection_scores(w: Workload) -> Optional[torch.Tensor]:
    """Scores the selector consumes when the workload fixes their distribution, else None
    (the selector then consumes the gate's own output)."""
    if w.score_mixture:
        return mixture_scores(w.n, w.seed)
    return None


def tie_scores(n: int, seed: int, levels: int = 16) -> torch.Tensor:
    """fp32[n] quantised to ``levels`` distinct values: a tie-heavy selector input."""
    g = _gen(seed, "ties")
    return (torch.randint(0, levels, (n,), generator=g).to(torch.float32) - levels / 2) * 0.25


def attention_params(w: Workload):
    """Per-head gain ~ U(0.5, 1.5) (fp32[hq]) and the temperature."""
    gain = 0.5 + torch.rand(w.hq, generator=_gen(w.seed, "gain"), dtype=torch.float32)
    return gain, float(w.tau)


def attention_inputs(w: Workload, S: int, layer: int = 0):
    """Independent Q [S,hq,D], K and V [S,hkv,D] (bf16, N(0,1)) for one gated layer."""
    Q = _randn_bf16((S, w.hq, w.head_dim), _gen(w.seed, "q", layer))
    K = _randn_bf16((S, w.hkv, w.head_dim), _gen(w.seed, "k", layer))
    V = _randn_bf16((S, w.hkv, w.head_dim), _gen(w.seed, "v", layer))
    return Q, K, V


def random_scores(n: int, seed: int) -> torch.Tensor:
    """fp32[n] ~ N(0,1): a generic key-bias vector for attention-only cases."""
    return torch.randn(n, generator=_gen(seed, "sel"), dtype=torch.float32)


def layer_weights(w: Workload, layer: int = 0):
    """Synthetic weights of one pruned attention layer, all bf16:
    W_qkv [(hq + 2 hkv) D, d] ~ N(0, 1/d) (Q rows, then K rows, then V rows),
    W_o [d, hq D] ~ N(0, 1/(hq D)), per-head norm weights q_norm, k_norm [D] ~ 1 + N(0, 0.1^2)."""
    D = w.head_dim
    W_qkv = _randn_bf16(((w.hq + 2 * w.hkv) * D, w.d), _gen(w.seed, "wqkv", layer), 1.0 / math.sqrt(w.d))
    W_o = _randn_bf16((w.d, w.hq * D), _gen(w.seed, "wo", layer), 1.0 / math.sqrt(w.hq * D))
    q_norm = (1.0 + 0.1 * torch.randn(D, generator=_gen(w.seed, "qn", layer))).to(torch.bfloat16)
    k_norm = (1.0 + 0.1 * torch.randn(D, generator=_gen(w.seed, "kn", layer))).to(torch.bfloat16)
    return W_qkv, W_o, q_norm, k_norm

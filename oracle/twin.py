"""numpy fp64 twin of the C oracle, for small sizes only.

TEST INFRASTRUCTURE ONLY.  Written separately from ``oracle.c`` (vectorised
numpy instead of scalar loops) so the two can check each other.

Definitions follow the MarkTechPost TokenGate article: "How does TokenGate
learned token pruning work?" (gate MLP on the residual, top-K over the
document, question never pruned, pruned forward on the kept tokens) and
"What is token-gated attention?" (gate score as a logit bias with per-head gain
and a temperature).
"""
from __future__ import annotations

import numpy as np
import torch


def _f64(t) -> np.ndarray:
    if isinstance(t, torch.Tensor):
        return t.detach().cpu().to(torch.float64).numpy()
    return np.asarray(t, dtype=np.float64)


def gate_score(hidden, W1, b1, W2, b2) -> np.ndarray:
    x, w1, c1, w2, c2 = (_f64(t) for t in (hidden, W1, b1, W2, b2))
    z = x @ w1.T + c1[None, :]
    a = z / (1.0 + np.exp(-z))
    return a @ w2 + c2[0]


def select_topk(scores, doc_mask, k: int) -> np.ndarray:
    s = np.asarray(scores.detach().cpu().numpy() if isinstance(scores, torch.Tensor) else scores,
                   dtype=np.float32)
    m = np.asarray(doc_mask.detach().cpu().numpy() if isinstance(doc_mask, torch.Tensor) else doc_mask)
    doc = np.nonzero(m != 0)[0]
    sd = s[doc].astype(np.float64)
    nan = np.isnan(sd)
    neg = np.where(nan, 0.0, -sd)
    order = np.lexsort((doc, neg, nan))        # primary: not-NaN first; then score desc; then index
    take = doc[order[:max(0, min(int(k), len(doc)))]]
    keep = np.zeros(len(s), dtype=bool)
    keep[take] = True
    keep[m == 0] = True
    return np.nonzero(keep)[0].astype(np.int32)


def gated_attention(Q, K, V, s, gain, tau: float) -> np.ndarray:
    q, kk, v = _f64(Q), _f64(K), _f64(V)
    sv, gv = _f64(s), _f64(gain)
    S, Hq, D = q.shape
    Hkv = kk.shape[1]
    rep = Hq // Hkv
    out = np.empty((S, Hq, D))
    causal = np.tril(np.ones((S, S), dtype=bool))
    for h in range(Hq):
        g = h // rep
        L = tau * (q[:, h, :] @ kk[:, g, :].T) / np.sqrt(D) + gv[h] * sv[None, :]
        L = np.where(causal, L, -np.inf)
        L = L - L.max(axis=1, keepdims=True)
        P = np.exp(L)
        P /= P.sum(axis=1, keepdims=True)
        out[:, h, :] = P @ v[:, g, :]
    return out

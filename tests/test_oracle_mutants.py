"""The pins catch plausible mistakes.

Each test plants one mistake in a CPU copy of a definition (never in the CUDA
path) and checks that the pin used for the real oracle rejects it: a dropped
bias term, a transposed GQA head index, a wrong tie-break, a divided
temperature, a missing causal mask, a wrong activation.
"""
import math

import numpy as np
import torch
import torch.nn.functional as F

import oracle
from oracle import twin
from test_oracle_pins import _attn_case, _brute_topk, _load_topk_golden, _sdpa_reference, _rand_bf16, _gate_torch


def _attn_variant(Q, K, V, s, gain, tau, *, bias=True, head_map="group", causal=True, tau_mode="mul"):
    q, kk, v = Q.double().numpy(), K.double().numpy(), V.double().numpy()
    sv, gv = np.asarray(s, np.float64), np.asarray(gain, np.float64)
    S, Hq, D = q.shape
    Hkv = kk.shape[1]
    out = np.empty((S, Hq, D))
    for h in range(Hq):
        g = h // (Hq // Hkv) if head_map == "group" else h % Hkv
        t = tau if tau_mode == "mul" else 1.0 / tau
        L = t * (q[:, h] @ kk[:, g].T) / math.sqrt(D)
        if bias:
            L = L + gv[h] * sv[None, :]
        if causal:
            L = np.where(np.tril(np.ones((S, S), bool)), L, -np.inf)
        L -= L.max(1, keepdims=True)
        P = np.exp(L)
        P /= P.sum(1, keepdims=True)
        out[:, h] = P @ v[:, g]
    return out


def _rejected(got, ref):
    return not np.allclose(got, ref, rtol=1e-9, atol=1e-10)


def test_attention_pin_rejects_planted_mistakes():
    Q, K, V, s, gain = _attn_case(40, 8, 2, 16, 123)
    tau = 1.1
    ref = _sdpa_reference(Q, K, V, torch.as_tensor(s), torch.as_tensor(gain), tau)
    assert not _rejected(_attn_variant(Q, K, V, s, gain, tau), ref)            # the unmutated copy passes
    assert _rejected(_attn_variant(Q, K, V, s, gain, tau, bias=False), ref)
    assert _rejected(_attn_variant(Q, K, V, s, gain, tau, head_map="mod"), ref)
    assert _rejected(_attn_variant(Q, K, V, s, gain, tau, causal=False), ref)
    assert _rejected(_attn_variant(Q, K, V, s, gain, tau, tau_mode="div"), ref)


def test_topk_pins_reject_wrong_tie_break_and_nan_order():
    g, s, m = _load_topk_golden()

    def ties_to_higher(scores, mask, k):
        doc = np.nonzero(mask)[0]
        key = np.where(np.isnan(scores[doc]), -np.inf, scores[doc])
        order = np.lexsort((-doc, -key))
        keep = np.zeros(len(scores), bool)
        keep[doc[order[:k]]] = True
        keep[mask == 0] = True
        return np.nonzero(keep)[0]

    def nan_on_top(scores, mask, k):
        doc = np.nonzero(mask)[0]
        key = np.where(np.isnan(scores[doc]), np.inf, scores[doc])
        order = np.lexsort((doc, -key))
        keep = np.zeros(len(scores), bool)
        keep[doc[order[:k]]] = True
        keep[mask == 0] = True
        return np.nonzero(keep)[0]

    for mutant in (ties_to_higher, nan_on_top):
        bad = [c for c in g["cases"] if mutant(s, m, c["k"]).tolist() != c["kept"]]
        assert bad, mutant.__name__


def test_gate_pin_rejects_wrong_activation_and_transposed_weight():
    n, d, h = 30, 16, 16
    hidden = _rand_bf16((n, d), 1)
    W1 = _rand_bf16((h, d), 2, 0.3)
    b1 = _rand_bf16((h,), 3)
    W2 = _rand_bf16((h,), 4)
    b2 = _rand_bf16((1,), 5)
    ref = _gate_torch(hidden, W1, b1, W2, b2)
    x = hidden.double().numpy()
    w1 = W1.double().numpy()
    z = x @ w1.T + b1.double().numpy()
    relu = np.maximum(z, 0) @ W2.double().numpy() + float(b2[0])
    zt = x @ w1 + b1.double().numpy()                         # W1 used transposed (h == d here)
    transposed = (zt / (1 + np.exp(-zt))) @ W2.double().numpy() + float(b2[0])
    no_b1 = (x @ w1.T / (1 + np.exp(-(x @ w1.T)))) @ W2.double().numpy() + float(b2[0])
    for bad in (relu, transposed, no_b1):
        assert _rejected(bad, ref)
    np.testing.assert_allclose(twin.gate_score(hidden, W1, b1, W2, b2), ref, rtol=1e-12, atol=1e-12)

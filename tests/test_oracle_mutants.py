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


def _qkv_rope_variant(x, Wt, positions, base, Hq, Hkv, D, q_norm=None, k_norm=None, eps=1e-6, *,
                      pairs="half", sign=1.0, expo=2.0, norm_scope="head", use_rows=False):
    """A numpy copy of the projection + per-head norm + rotary definition with one planted mistake."""
    y = x.double().numpy() @ Wt.double().numpy().T
    S = y.shape[0]
    pos = np.arange(S) if use_rows else np.asarray(positions, np.float64)
    out = []
    for lo, H, w in ((0, Hq, q_norm), (Hq * D, Hkv, k_norm)):
        u = y[:, lo:lo + H * D].reshape(S, H, D).copy()
        if w is not None:
            wv = w.double().numpy()
            if norm_scope == "head":
                ms = np.mean(u ** 2, axis=-1, keepdims=True)
            else:
                ms = np.mean(u.reshape(S, -1) ** 2, axis=-1)[:, None, None]
            u = u / np.sqrt(ms + eps) * wv
        j = np.arange(D // 2)
        phi = pos[:, None] * base ** (-expo * j / D)
        c, s = np.cos(phi)[:, None, :], np.sin(phi)[:, None, :]
        if pairs == "half":
            a, b = u[..., :D // 2], u[..., D // 2:]
        else:
            a, b = u[..., 0::2], u[..., 1::2]
        ra, rb = a * c - sign * b * s, b * c + sign * a * s
        r = np.empty_like(u)
        if pairs == "half":
            r[..., :D // 2], r[..., D // 2:] = ra, rb
        else:
            r[..., 0::2], r[..., 1::2] = ra, rb
        out.append(r)
    v = y[:, (Hq + Hkv) * D:].reshape(S, Hkv, D)
    return out[0], out[1], v


def test_projection_pins_reject_planted_mistakes():
    from test_oracle_pins import _load_rope_golden, _rope_golden_case, _proj_case
    g = _load_rope_golden()

    def golden_ok(**mut):
        fn = lambda *a, **k: _qkv_rope_variant(*a, **k, **mut)  # noqa: E731
        for c in g["cases"]:
            Q, K, V = _rope_golden_case(fn, g, c)
            if not np.allclose(Q[0, 0], c["q"], rtol=0, atol=g["tol"]):
                return False
        return True

    assert golden_ok()                         # the unmutated copy passes
    assert not golden_ok(pairs="interleaved")  # (2j, 2j+1) pairs instead of (j, j + D/2)
    assert not golden_ok(sign=-1.0)            # rotation the wrong way
    assert not golden_ok(expo=1.0)             # base^(-j/D) instead of base^(-2j/D)

    # norm over all heads of a row instead of per head: the per-head unit-RMS pin fails
    Hq, Hkv, D = 4, 2, 32
    x, Wq, _, _ = _proj_case(8, Hq, Hkv, D, 64, 51)
    ones = _bf16_ones(D)
    pos = np.arange(8) * 3
    Q, _, _ = _qkv_rope_variant(x, Wq, pos, 1e6, Hq, Hkv, D, ones, ones, 0.0)
    assert np.allclose(np.mean(Q ** 2, axis=-1), 1.0, rtol=1e-12)
    Qm, _, _ = _qkv_rope_variant(x, Wq, pos, 1e6, Hq, Hkv, D, ones, ones, 0.0, norm_scope="row")
    assert not np.allclose(np.mean(Qm ** 2, axis=-1), 1.0, rtol=1e-6)

    # compacted row numbers as positions: pruning no longer commutes with the projection
    x, Wq, qn, kn = _proj_case(64, 2, 1, 32, 64, 61)
    kept = np.sort(np.random.default_rng(1).choice(64, 20, replace=False))
    full = _qkv_rope_variant(x, Wq, np.arange(64), 1e6, 2, 1, 32, qn, kn)
    sub = x[torch.as_tensor(kept)]
    assert np.allclose(full[0][kept], _qkv_rope_variant(sub, Wq, kept, 1e6, 2, 1, 32, qn, kn)[0])
    assert not np.allclose(full[0][kept], _qkv_rope_variant(sub, Wq, kept, 1e6, 2, 1, 32, qn, kn, use_rows=True)[0])


def _bf16_ones(D):
    return torch.ones(D, dtype=torch.bfloat16)


def _backward_variant(Q, K, V, dO, s, gain, tau, *, delta=True, gain_in_ds=True, sqrt_d=True, causal=True):
    """A numpy copy of the score / gain / temperature backward with one planted mistake."""
    q, kk, v, do = (t.double().numpy() for t in (Q, K, V, dO))
    sv, gv = np.asarray(s, np.float64), np.asarray(gain, np.float64)
    S, Hq, D = q.shape
    Hkv = kk.shape[1]
    ds, dg, dt = np.zeros(S), np.zeros(Hq), 0.0
    for h in range(Hq):
        g = h // (Hq // Hkv)
        qk = q[:, h] @ kk[:, g].T / math.sqrt(D)
        L = tau * qk + gv[h] * sv[None, :]
        if causal:
            L = np.where(np.tril(np.ones((S, S), bool)), L, -np.inf)
        P = np.exp(L - L.max(1, keepdims=True))
        P /= P.sum(1, keepdims=True)
        dP = do[:, h] @ v[:, g].T
        dl = P * (dP - ((P * dP).sum(1, keepdims=True) if delta else 0.0))
        ds += (gv[h] if gain_in_ds else 1.0) * dl.sum(0)
        dg[h] = (dl * sv[None, :]).sum()
        dt += (dl * (qk if sqrt_d else qk * math.sqrt(D))).sum()
    return ds, dg, dt


def test_backward_pins_reject_planted_mistakes():
    from test_oracle_pins import _bwd_case, _autograd_backward
    Q, K, V, dO, s, gain = _bwd_case(24, 4, 2, 16, 0)
    tau = 1.1
    ref = _autograd_backward(Q, K, V, dO, s, gain, tau)

    def passes(**mut):
        got = _backward_variant(Q, K, V, dO, s, gain, tau, **mut)
        return all(np.allclose(a, b, rtol=1e-9, atol=1e-12) for a, b in zip(got, ref))

    assert passes()                        # the unmutated copy passes
    assert not passes(delta=False)         # softmax Jacobian without the Delta term
    assert not passes(gain_in_ds=False)    # score gradient without the head's gain
    assert not passes(sqrt_d=False)        # temperature gradient without 1/sqrt(D)
    assert not passes(causal=False)        # keys after the query counted


def _spread_variant(Q, K, V, s, gain, tau, *, mode="ok"):
    """A CPU copy of the spread (sum_j w_j |V_j - O|) with one planted mistake."""
    q, kk, v = Q.double().numpy(), K.double().numpy(), V.double().numpy()
    sv, gv = np.asarray(s, np.float64), np.asarray(gain, np.float64)
    S, Hq, D = q.shape
    Hkv = kk.shape[1]
    out = np.empty((S, Hq, D))
    for h in range(Hq):
        g = h // (Hq // Hkv)
        L = tau * (q[:, h] @ kk[:, g].T) / math.sqrt(D) + gv[h] * sv[None, :]
        L = np.where(np.tril(np.ones((S, S), bool)), L, -np.inf)
        P = np.exp(L - L.max(1, keepdims=True))
        if mode != "unnormalised":
            P /= P.sum(1, keepdims=True)
        O = P @ v[:, g] if mode != "unnormalised" else (P @ v[:, g]) / P.sum(1, keepdims=True)
        for c in range(D):
            dev = v[None, :, g, c] - O[:, None, c]
            if mode == "no_abs":
                out[:, h, c] = (P * dev).sum(1)
            elif mode == "abs_v":
                out[:, h, c] = (P * np.abs(v[None, :, g, c])).sum(1)
            else:
                out[:, h, c] = (P * np.abs(dev)).sum(1)
    return out


def test_spread_pins_reject_planted_mistakes():
    """The two-key identity and row 0 (the spread pins) reject a spread without the
    absolute value, one of |V| instead of |V - O|, and one with unnormalised weights."""
    Q, K, V, s, gain = _attn_case(12, 2, 1, 8, 77)
    o = oracle.gated_attention(Q, K, V, s, gain, 1.1)
    v = V.double().numpy()

    def pins_hold(sp):
        if not np.allclose(sp[0], 0.0, atol=1e-12):
            return False
        for h in range(2):
            a, b = v[0, 0], v[1, 0]
            want = 2 * np.abs(o[1, h] - b) * np.abs(a - o[1, h]) / np.abs(a - b)
            if not np.allclose(sp[1, h], want, rtol=1e-9, atol=1e-12):
                return False
        return True

    assert pins_hold(_spread_variant(Q, K, V, s, gain, 1.1))
    assert pins_hold(oracle.gated_attention(Q, K, V, s, gain, 1.1, return_spread=True)[1])
    for mode in ("no_abs", "abs_v", "unnormalised"):
        assert not pins_hold(_spread_variant(Q, K, V, s, gain, 1.1, mode=mode)), mode

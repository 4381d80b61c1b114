"""Pins of the fp64 CPU oracle against things other than itself.

Each test ties an oracle function to a library routine (torch fp64), a brute
force, a hand-worked example under tests/golden/, or an invariant the TokenGate
article fixes (question never pruned, |kept| = K + question length, pruned keys
never influence an output).  None of them retypes the oracle's own formula.
"""
import json
import math
import os

import numpy as np
import pytest
import torch
import torch.nn.functional as F

import oracle
from oracle import twin
from learned_token_pruning_mlp_b200 import workloads as W

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def _bf16(a):
    return torch.as_tensor(np.asarray(a, dtype=np.float32)).to(torch.bfloat16)


def _rand_bf16(shape, seed, scale=1.0):
    g = torch.Generator().manual_seed(seed)
    return (torch.randn(shape, generator=g) * scale).to(torch.bfloat16)


# ============================================================================ gate
def _gate_torch(hidden, W1, b1, W2, b2):
    x = hidden.to(torch.float64)
    z = F.linear(x, W1.to(torch.float64), b1.to(torch.float64))
    return F.linear(F.silu(z), W2.to(torch.float64)[None, :], b2.to(torch.float64)).squeeze(-1).numpy()


@pytest.mark.parametrize("n,d,h,seed", [(64, 32, 8, 0), (300, 256, 64, 1), (129, 72, 24, 2)])
def test_gate_matches_torch_linear_silu(n, d, h, seed):
    hidden = _rand_bf16((n, d), seed)
    W1 = _rand_bf16((h, d), seed + 10, 1 / math.sqrt(d))
    b1 = _rand_bf16((h,), seed + 11, 1 / math.sqrt(d))
    W2 = _rand_bf16((h,), seed + 12, 1 / math.sqrt(h))
    b2 = _rand_bf16((1,), seed + 13, 1 / math.sqrt(h))
    ref = _gate_torch(hidden, W1, b1, W2, b2)
    got = oracle.gate_score(hidden, W1, b1, W2, b2)
    np.testing.assert_allclose(got, ref, rtol=1e-12, atol=1e-12)


def test_gate_matches_twin_on_tiny_workload():
    w = W.get("tiny_n512")
    args = W.gate_inputs(w)
    np.testing.assert_allclose(oracle.gate_score(*args), twin.gate_score(*args), rtol=1e-12, atol=1e-12)


def test_gate_zero_w1_gives_constant_library_value():
    n, d, h = 17, 16, 8
    hidden = _rand_bf16((n, d), 3)
    W1 = torch.zeros((h, d), dtype=torch.bfloat16)
    b1 = _rand_bf16((h,), 4)
    W2 = _rand_bf16((h,), 5)
    b2 = _rand_bf16((1,), 6)
    expect = float((F.silu(b1.double()) * W2.double()).sum() + b2.double()[0])
    got = oracle.gate_score(hidden, W1, b1, W2, b2)
    np.testing.assert_allclose(got, np.full(n, expect), rtol=1e-13, atol=1e-13)


def test_gate_invariances():
    n, d, h = 40, 24, 12
    hidden = _rand_bf16((n, d), 7)
    W1 = _rand_bf16((h, d), 8, 0.3)
    b1 = _rand_bf16((h,), 9)
    W2 = _rand_bf16((h,), 10)
    b2 = _rand_bf16((1,), 11)
    base = oracle.gate_score(hidden, W1, b1, W2, b2)
    # permuting the hidden units changes nothing
    p = torch.randperm(h, generator=torch.Generator().manual_seed(0))
    np.testing.assert_allclose(oracle.gate_score(hidden, W1[p], b1[p], W2[p], b2), base, rtol=1e-12, atol=1e-12)
    # each token is scored from its own residual only
    t = torch.randperm(n, generator=torch.Generator().manual_seed(1))
    np.testing.assert_allclose(oracle.gate_score(hidden[t], W1, b1, W2, b2), base[t.numpy()], rtol=0, atol=0)
    # b2 enters additively
    b2s = (b2.float() + 2.0).to(torch.bfloat16)
    delta = float(b2s[0]) - float(b2[0])
    np.testing.assert_allclose(oracle.gate_score(hidden, W1, b1, W2, b2s) - delta, base, rtol=1e-12, atol=1e-12)
    # the output layer is linear in W2
    np.testing.assert_allclose(oracle.gate_score(hidden, W1, b1, W2 * 2, b2) - float(b2[0]),
                               2 * (base - float(b2[0])), rtol=1e-12, atol=1e-12)


def test_gate_one_hot_rows_reduce_to_elementwise_silu():
    # W1 = identity (h = d), b1 = 0, W2 = e_j: the score is silu(x_j) + b2 (torch.nn.functional.silu)
    d = 8
    hidden = _rand_bf16((10, d), 12, 3.0)
    W1 = torch.eye(d, dtype=torch.bfloat16)
    b1 = torch.zeros(d, dtype=torch.bfloat16)
    b2 = torch.zeros(1, dtype=torch.bfloat16)
    for j in range(d):
        W2 = torch.zeros(d, dtype=torch.bfloat16)
        W2[j] = 1
        got = oracle.gate_score(hidden, W1, b1, W2, b2)
        np.testing.assert_allclose(got, F.silu(hidden[:, j].double()).numpy(), rtol=1e-14, atol=1e-300)


# ============================================================================ top-K
def _brute_topk(scores, mask, k):
    """O(n^2) rank counting: document token i is kept iff fewer than k document tokens
    precede it in (score desc with NaN last, index asc)."""
    s = [float(x) for x in scores]
    n = len(s)
    keep = []
    for i in range(n):
        if not mask[i]:
            keep.append(i)
            continue
        rank = 0
        for j in range(n):
            if j == i or not mask[j]:
                continue
            ni, nj = math.isnan(s[i]), math.isnan(s[j])
            if ni and not nj:
                rank += 1
            elif ni == nj and not ni and s[j] > s[i]:
                rank += 1
            elif (ni == nj) and (ni or s[j] == s[i]) and j < i:
                rank += 1
        if rank < k:
            keep.append(i)
    return np.asarray(keep, dtype=np.int32)


def _load_topk_golden():
    with open(os.path.join(GOLDEN, "topk_worked.json")) as f:
        g = json.load(f)
    s = np.asarray([float(x) for x in g["scores"]], dtype=np.float32)
    return g, s, np.asarray(g["doc_mask"], dtype=np.uint8)


def test_topk_hand_worked_fixture():
    g, s, m = _load_topk_golden()
    for case in g["cases"]:
        assert oracle.select_topk(s, m, case["k"]).tolist() == case["kept"], case
        assert twin.select_topk(s, m, case["k"]).tolist() == case["kept"], case


@pytest.mark.parametrize("seed", range(12))
def test_topk_matches_brute_force(seed):
    rng = np.random.default_rng(seed)
    n = int(rng.integers(1, 48))
    kind = seed % 4
    if kind == 0:
        s = rng.standard_normal(n).astype(np.float32)
    elif kind == 1:
        s = (rng.integers(0, 3, n) - 1).astype(np.float32)          # heavy ties
    elif kind == 2:
        s = rng.standard_normal(n).astype(np.float32)
        s[rng.random(n) < 0.3] = np.nan
        s[rng.random(n) < 0.2] = -0.0
        s[rng.random(n) < 0.1] = -np.inf
    else:
        s = np.zeros(n, dtype=np.float32)                          # all equal
    m = (rng.random(n) < 0.7).astype(np.uint8)
    n_doc = int(m.sum())
    for k in range(0, n_doc + 3):
        ref = _brute_topk(s, m, k)
        got = oracle.select_topk(s, m, k)
        assert got.tolist() == ref.tolist(), (seed, k)
        assert twin.select_topk(s, m, k).tolist() == ref.tolist(), (seed, k)


def test_topk_invariants_on_mixture_scores():
    n, q = 4096, 96
    s = W.mixture_scores(n, seed=5).numpy()
    m = np.ones(n, dtype=np.uint8)
    m[-q:] = 0
    for k in (0, 1, 100, 1000, n - q, n):
        kept = oracle.select_topk(s, m, k)
        kk = min(k, n - q)
        assert len(kept) == kk + q                                   # |kept| = K + question length
        assert set(range(n - q, n)) <= set(kept.tolist())            # question never pruned
        assert np.all(np.diff(kept) > 0)                             # strictly ascending
        doc_kept = np.asarray([i for i in kept if m[i]], dtype=np.int64)
        pruned = np.setdiff1d(np.nonzero(m)[0], doc_kept)
        if len(doc_kept) and len(pruned):
            assert s[doc_kept].min() >= s[pruned].max()


def test_topk_all_equal_keeps_lowest_indices():
    n = 300
    s = np.full(n, 1.5, dtype=np.float32)
    m = np.ones(n, dtype=np.uint8)
    m[::7] = 0
    doc = np.nonzero(m)[0]
    kept = oracle.select_topk(s, m, 50)
    expect = np.union1d(doc[:50], np.nonzero(m == 0)[0])
    assert kept.tolist() == expect.tolist()


def test_topk_interleaved_question_tokens_kept():
    rng = np.random.default_rng(3)
    n = 200
    s = rng.standard_normal(n).astype(np.float32)
    m = (rng.random(n) < 0.5).astype(np.uint8)
    for k in (0, 5, 50):
        kept = oracle.select_topk(s, m, k)
        assert set(np.nonzero(m == 0)[0].tolist()) <= set(kept.tolist())
        assert kept.tolist() == _brute_topk(s, m, k).tolist()


def test_topk_varlen_is_per_request():
    cu = [0, 50, 50, 170, 171]
    rng = np.random.default_rng(9)
    n = cu[-1]
    s = rng.standard_normal(n).astype(np.float32)
    m = (rng.random(n) < 0.8).astype(np.uint8)
    ks = [10, 3, 200, 0]
    kept, cu_kept = oracle.select_topk_varlen(s, m, cu, ks)
    for b in range(4):
        lo, hi = cu[b], cu[b + 1]
        seg = kept[cu_kept[b]:cu_kept[b + 1]]
        assert seg.tolist() == (_brute_topk(s[lo:hi], m[lo:hi], ks[b]) + lo).tolist()


# ============================================================================ gather
def test_gather_matches_fancy_indexing():
    hidden = _rand_bf16((100, 40), 21)
    scores = torch.randn(100, generator=torch.Generator().manual_seed(2))
    kept = np.asarray([0, 3, 4, 50, 99], dtype=np.int32)
    hk, sk = oracle.gather(hidden, kept, scores)
    assert np.array_equal(hk, hidden.view(torch.int16).numpy().view(np.uint16)[kept])
    assert np.array_equal(sk, scores.numpy()[kept])


# ============================================================================ attention
def _sdpa_reference(Q, K, V, s, gain, tau):
    """torch scaled_dot_product_attention in fp64 with GQA expanded and the gate score
    as an additive float mask; causal handled through the mask."""
    S, Hq, D = Q.shape
    Hkv = K.shape[1]
    rep = Hq // Hkv
    q = Q.double().permute(1, 0, 2)
    k = K.double().repeat_interleave(rep, dim=1).permute(1, 0, 2)
    v = V.double().repeat_interleave(rep, dim=1).permute(1, 0, 2)
    causal = torch.ones(S, S, dtype=torch.bool).tril()
    bias = gain.double()[:, None, None] * s.double()[None, None, :]
    bias = bias.masked_fill(~causal[None], float("-inf"))
    o = F.scaled_dot_product_attention(q, k, v, attn_mask=bias, scale=tau / math.sqrt(D))
    return o.permute(1, 0, 2).numpy()


def _attn_case(S, Hq, Hkv, D, seed):
    Q = _rand_bf16((S, Hq, D), seed)
    K = _rand_bf16((S, Hkv, D), seed + 1)
    V = _rand_bf16((S, Hkv, D), seed + 2)
    s = torch.randn(S, generator=torch.Generator().manual_seed(seed + 3))
    gain = 0.5 + torch.rand(Hq, generator=torch.Generator().manual_seed(seed + 4))
    return Q, K, V, s, gain


def test_attention_plain_causal_when_gain_zero_tau_one():
    # every document token kept, gain 0 and tau 1: ordinary causal attention
    Q, K, V, s, _ = _attn_case(70, 4, 2, 32, 30)
    gain = torch.zeros(4)
    S, Hq, D = Q.shape
    q = Q.double().permute(1, 0, 2)
    k = K.double().repeat_interleave(2, dim=1).permute(1, 0, 2)
    v = V.double().repeat_interleave(2, dim=1).permute(1, 0, 2)
    ref = F.scaled_dot_product_attention(q, k, v, is_causal=True).permute(1, 0, 2).numpy()
    got = oracle.gated_attention(Q, K, V, s, gain, 1.0)
    np.testing.assert_allclose(got, ref, rtol=1e-11, atol=1e-12)


@pytest.mark.parametrize("S,Hq,Hkv,D,tau", [(33, 4, 2, 16, 1.1), (64, 4, 4, 64, 0.7), (17, 8, 2, 8, 2.0)])
def test_attention_matches_torch_sdpa_with_bias(S, Hq, Hkv, D, tau):
    Q, K, V, s, gain = _attn_case(S, Hq, Hkv, D, 40 + S)
    ref = _sdpa_reference(Q, K, V, s, gain, tau)
    got = oracle.gated_attention(Q, K, V, s, gain, tau)
    np.testing.assert_allclose(got, ref, rtol=1e-11, atol=1e-12)
    np.testing.assert_allclose(twin.gated_attention(Q, K, V, s, gain, tau), got, rtol=1e-11, atol=1e-12)


def test_attention_hand_worked_fixture():
    with open(os.path.join(GOLDEN, "attention_worked.json")) as f:
        g = json.load(f)
    for ex in g["examples"]:
        Q = _bf16(ex["Q"])[:, None, :]
        K = _bf16(ex["K"])[:, None, :]
        V = _bf16(ex["V"])[:, None, :]
        s = np.asarray(ex["s"], dtype=np.float32)
        gain = np.asarray([ex["gain"]], dtype=np.float32)
        got = oracle.gated_attention(Q, K, V, s, gain, ex["tau"])[:, 0, :]
        np.testing.assert_allclose(got, np.asarray(ex["O"]), rtol=0, atol=max(ex["tol"], 1e-15), err_msg=ex["name"])


def test_attention_row_zero_is_v0_and_shift_invariance():
    Q, K, V, s, gain = _attn_case(50, 4, 2, 32, 60)
    o = oracle.gated_attention(Q, K, V, s, gain, 1.1)
    rep = 2
    for h in range(4):
        assert np.array_equal(o[0, h], V[0, h // rep].double().numpy())
    # adding the same constant to every key score leaves each softmax row unchanged
    # (scores on a 2^-10 grid so that the fp32 shift is exact)
    s = torch.round(s * 1024) / 1024
    o = oracle.gated_attention(Q, K, V, s, gain, 1.1)
    o2 = oracle.gated_attention(Q, K, V, s + 3.25, gain, 1.1)
    np.testing.assert_allclose(o2, o, rtol=1e-12, atol=1e-13)


def test_attention_temperature_scales_the_dot_product():
    Q, K, V, s, gain = _attn_case(40, 4, 2, 16, 70)
    a = oracle.gated_attention(Q, K, V, s, gain, 2.0)
    b = oracle.gated_attention((Q.float() * 2).to(torch.bfloat16), K, V, s, gain, 1.0)
    np.testing.assert_allclose(a, b, rtol=1e-12, atol=1e-13)


def test_attention_gqa_equals_duplicated_kv_heads():
    Q, K, V, s, gain = _attn_case(45, 8, 2, 16, 80)
    a = oracle.gated_attention(Q, K, V, s, gain, 1.1)
    b = oracle.gated_attention(Q, K.repeat_interleave(4, dim=1), V.repeat_interleave(4, dim=1), s, gain, 1.1)
    np.testing.assert_allclose(a, b, rtol=0, atol=0)


def test_attention_rows_inside_visible_value_hull():
    Q, K, V, s, gain = _attn_case(64, 4, 2, 32, 90)
    o = oracle.gated_attention(Q, K, V, s, gain, 1.1)
    v = V.double().numpy()
    for i in range(64):
        for h in range(4):
            vis = v[: i + 1, h // 2, :]
            assert np.all(o[i, h] <= vis.max(axis=0) + 1e-12)
            assert np.all(o[i, h] >= vis.min(axis=0) - 1e-12)


def test_attention_sampled_rows_equal_full_rows():
    Q, K, V, s, gain = _attn_case(300, 4, 2, 16, 95)
    full = oracle.gated_attention(Q, K, V, s, gain, 1.1)
    rows = oracle.sampled_rows(300, seed=1, head=10, tail=10, rand=20)
    np.testing.assert_array_equal(oracle.gated_attention(Q, K, V, s, gain, 1.1, rows=rows), full[rows])


def test_attention_varlen_is_block_diagonal():
    Q, K, V, s, gain = _attn_case(90, 4, 2, 16, 97)
    cu = [0, 30, 31, 90]
    o = oracle.gated_attention_varlen(Q, K, V, s, gain, 1.1, cu)
    for b in range(3):
        lo, hi = cu[b], cu[b + 1]
        np.testing.assert_array_equal(o[lo:hi], oracle.gated_attention(Q[lo:hi], K[lo:hi], V[lo:hi], s[lo:hi], gain, 1.1))


# ------------------------------------------------------------ spread (tolerance sizing)
def test_attention_spread_hand_worked():
    """spread[i,c] = sum_j w_ij |V_jc - O_ic| by hand on the fixture's cases.  'uniform':
    row 1 averages V0 = (1, 2) and V1 = (3, -2): O = (2, 0), spread = (1, 2); row 2 averages
    three rows: O = (1, 2), spread = ((0 + 2 + 2) / 3, (0 + 4 + 4) / 3).  'ln3_bias': row 1
    weights 1/4, 3/4: O = (2.5, -1), spread = 2 (1/4)(3/4) |V0 - V1| = (0.75, 1.5); row 2
    weights 0.2, 0.6, 0.2: O = (1.8, 0.4), spread = (0.16 + 0.72 + 0.56, 0.32 + 1.44 + 1.12)."""
    with open(os.path.join(GOLDEN, "attention_worked.json")) as f:
        ex = {e["name"]: e for e in json.load(f)["examples"]}
    expected = {"uniform": [[0.0, 0.0], [1.0, 2.0], [4.0 / 3.0, 8.0 / 3.0]],
                "ln3_bias": [[0.0, 0.0], [0.75, 1.5], [1.44, 2.88]]}
    for name, want in expected.items():
        e = ex[name]
        Q, K, V = (_bf16(e[k])[:, None, :] for k in ("Q", "K", "V"))
        o, sp = oracle.gated_attention(Q, K, V, np.asarray(e["s"], np.float32), np.asarray([e["gain"]], np.float32),
                                       e["tau"], return_spread=True)
        np.testing.assert_allclose(o[:, 0, :], np.asarray(e["O"]), rtol=0, atol=max(e["tol"], 1e-15))
        np.testing.assert_allclose(sp[:, 0, :], np.asarray(want), rtol=0, atol=max(4 * e["tol"], 1e-14), err_msg=name)


def test_attention_spread_invariants():
    """Row 0 sees one key (spread 0); with two visible keys the weights follow from O
    itself (w0 = (O - V1) / (V0 - V1)), so spread = 2 |O - V1| |V0 - O| / |V0 - V1|; the
    spread does not move when V is shifted and scales with V; constant V rows give 0; it
    never exceeds the largest deviation of a visible V row; O is unchanged by asking."""
    Q, K, V, s, gain = _attn_case(60, 4, 2, 16, 131)
    # V on a 1/8 grid in [-4, 4) so that V + 2 and 2 V are exact in bf16
    g = torch.Generator().manual_seed(7)
    V = (torch.randint(-32, 32, V.shape, generator=g).float() / 8).to(torch.bfloat16)
    o, sp = oracle.gated_attention(Q, K, V, s, gain, 1.1, return_spread=True)
    np.testing.assert_array_equal(o, oracle.gated_attention(Q, K, V, s, gain, 1.1))
    assert np.all(sp >= 0)
    np.testing.assert_allclose(sp[0], 0.0, atol=1e-15)
    v = V.double().numpy()
    for h in range(4):
        a, b = v[0, h // 2], v[1, h // 2]
        ok = np.abs(a - b) > 0
        want = 2 * np.abs(o[1, h] - b) * np.abs(a - o[1, h]) / np.where(ok, np.abs(a - b), 1.0)
        np.testing.assert_allclose(sp[1, h][ok], want[ok], rtol=1e-9, atol=1e-12)
        np.testing.assert_allclose(sp[1, h][~ok], 0.0, atol=1e-12)
        for i in (5, 33, 59):
            dev = np.abs(v[: i + 1, h // 2] - o[i, h]).max(axis=0)
            assert np.all(sp[i, h] <= dev + 1e-12)
    _, sp_shift = oracle.gated_attention(Q, K, (V.float() + 2).to(torch.bfloat16), s, gain, 1.1, return_spread=True)
    np.testing.assert_allclose(sp_shift, sp, rtol=1e-9, atol=1e-12)
    _, sp_scale = oracle.gated_attention(Q, K, (V.float() * 2).to(torch.bfloat16), s, gain, 1.1, return_spread=True)
    np.testing.assert_allclose(sp_scale, 2 * sp, rtol=1e-9, atol=1e-12)
    Vc = torch.full_like(V, 1.5)
    _, sp_const = oracle.gated_attention(Q, K, Vc, s, gain, 1.1, return_spread=True)
    np.testing.assert_allclose(sp_const, 0.0, atol=1e-12)
    # rows, varlen and the full run agree
    rows = np.array([0, 7, 59])
    o_r, sp_r = oracle.gated_attention(Q, K, V, s, gain, 1.1, rows=rows, return_spread=True)
    np.testing.assert_array_equal(sp_r, sp[rows])
    _, sp_v = oracle.gated_attention_varlen(Q, K, V, s, gain, 1.1, [0, 60], return_spread=True)
    np.testing.assert_array_equal(sp_v, sp)


# ============================================================================ pipeline
def test_pruned_tokens_never_influence_outputs():
    """Layers above the gate see only kept tokens and keep no KV for pruned ones: poisoning
    every pruned position of the full-length inputs with NaN leaves the outputs bitwise equal
    and NaN-free."""
    w = W.get("tiny_n512")
    hidden, W1, b1, W2, b2 = W.gate_inputs(w)
    mask = W.doc_mask(w)
    scores = oracle.gate_score(hidden, W1, b1, W2, b2).astype(np.float32)
    kept = oracle.select_topk(scores, mask, 128)
    assert len(kept) == 128 + 64
    N = w.n
    Qf, Kf, Vf = W.attention_inputs(w, N)
    gain, tau = W.attention_params(w)
    pruned = np.setdiff1d(np.arange(N), kept)

    def run(Qf, Kf, Vf, sc, hid):
        hk, sk = oracle.gather(hid, kept, sc)
        o = oracle.gated_attention(Qf[kept], Kf[kept], Vf[kept], sk, gain, tau)
        return hk, sk, o

    clean = run(Qf, Kf, Vf, scores, hidden)
    Qp, Kp, Vp, hp = Qf.clone(), Kf.clone(), Vf.clone(), hidden.clone()
    sp = scores.copy()
    nan = float("nan")
    Qp[pruned] = nan
    Kp[pruned] = nan
    Vp[pruned] = nan
    hp[pruned] = nan
    sp[pruned] = nan
    poisoned = run(Qp, Kp, Vp, sp, hp)
    for a, b in zip(clean, poisoned):
        assert np.array_equal(a, b)
        assert not np.isnan(np.asarray(b, dtype=np.float64)).any()


# ============================================================================ random-K and sweep
def test_splitmix64_matches_published_outputs():
    with open(os.path.join(GOLDEN, "splitmix64_vectors.json")) as f:
        g = json.load(f)
    got = [oracle.splitmix64(g["seed"], i) for i in range(len(g["outputs"]))]
    assert got == [int(v) for v in g["outputs"]]


def test_random_k_is_top_k_of_the_random_keys():
    rng = np.random.default_rng(4)
    for n in (1, 37, 500):
        m = (rng.random(n) < 0.75).astype(np.uint8)
        for seed in (0, 7, 2**63 + 5):
            keys = np.asarray([oracle.splitmix64(seed, i) >> 33 for i in range(n)], dtype=np.float64)
            for k in (0, 1, int(m.sum()) // 2, int(m.sum()), int(m.sum()) + 3):
                got = oracle.select_random_k(m, k, seed)
                assert got.tolist() == _brute_topk(keys, m, k).tolist()


def test_random_k_is_roughly_uniform():
    # every document position is kept with probability k / n_doc over seeds
    n, k, trials = 64, 16, 400
    m = np.ones(n, dtype=np.uint8)
    hits = np.zeros(n)
    for seed in range(trials):
        hits[oracle.select_random_k(m, k, seed)] += 1
    freq = hits / trials
    assert abs(freq.mean() - k / n) < 1e-12
    assert np.all(np.abs(freq - k / n) < 0.12)


def test_sweep_is_nested_and_matches_single_budgets():
    s = W.mixture_scores(3000, 9).numpy()
    m = np.ones(3000, dtype=np.uint8)
    m[-100:] = 0
    ks = [0, 10, 500, 2900, 5000]
    sets = oracle.select_topk_sweep(s, m, ks)
    for k, kept in zip(ks, sets):
        assert kept.tolist() == oracle.select_topk(s, m, k).tolist()
    for a, b in zip(sets, sets[1:]):
        assert set(a.tolist()) <= set(b.tolist())


# ============================================================================ projections
def test_linear_matches_torch_fp64_with_and_without_residual():
    x = _rand_bf16((37, 72), 11)
    Wt = _rand_bf16((96, 72), 12, 0.1)
    res = _rand_bf16((37, 96), 13)
    ref = F.linear(x.double(), Wt.double()).numpy()
    assert np.allclose(oracle.linear(x, Wt), ref, rtol=1e-13, atol=1e-13)
    assert np.allclose(oracle.linear(x, Wt, res), ref + res.double().numpy(), rtol=1e-13, atol=1e-13)
    rows = [36, 0, 5]
    assert np.array_equal(oracle.linear(x, Wt, res, rows=rows), oracle.linear(x, Wt, res)[rows])


def test_qkv_at_position_zero_without_norm_is_the_plain_projection():
    Hq, Hkv, D, d = 4, 2, 16, 48
    x = _rand_bf16((9, d), 21)
    Wq = _rand_bf16(((Hq + 2 * Hkv) * D, d), 22, 0.2)
    Q, K, V = oracle.qkv_rope(x, Wq, np.zeros(9, np.int32), 1e6, Hq, Hkv, D)
    y = F.linear(x.double(), Wq.double()).numpy()
    assert np.allclose(Q.reshape(9, -1), y[:, :Hq * D], rtol=1e-13, atol=1e-13)
    assert np.allclose(K.reshape(9, -1), y[:, Hq * D:(Hq + Hkv) * D], rtol=1e-13, atol=1e-13)
    assert np.allclose(V.reshape(9, -1), y[:, (Hq + Hkv) * D:], rtol=1e-13, atol=1e-13)


def _load_rope_golden():
    with open(os.path.join(GOLDEN, "rope_worked.json")) as f:
        return json.load(f)


def _rope_golden_case(fn, g, c):
    """Run ``fn`` (an oracle-shaped qkv_rope) on one fixture case: W_qkv = three 4x4 identities."""
    D = g["D"]
    Wt = _bf16(np.vstack([np.eye(D)] * 3))
    x = _bf16(np.asarray(c["x"], np.float32)[None, :])
    w = _bf16(np.ones(D, np.float32)) if c["norm"] else None
    return fn(x, Wt, np.asarray([c["pos"]], np.int32), g["base"], 1, 1, D, q_norm=w, k_norm=w, eps=c["eps"])


def test_rope_hand_worked_fixture():
    g = _load_rope_golden()
    for c in g["cases"]:
        Q, K, V = _rope_golden_case(oracle.qkv_rope, g, c)
        assert np.allclose(Q[0, 0], c["q"], rtol=0, atol=g["tol"]), c["name"]
        assert np.allclose(K[0, 0], c["q"], rtol=0, atol=g["tol"]), c["name"]
        assert np.allclose(V[0, 0], c["v"], rtol=0, atol=g["tol"]), c["name"]


def _proj_case(S, Hq, Hkv, D, d, seed):
    x = _rand_bf16((S, d), seed)
    Wq = _rand_bf16(((Hq + 2 * Hkv) * D, d), seed + 1, d ** -0.5)
    qn = (1.0 + 0.25 * _rand_bf16((D,), seed + 2).float()).bfloat16()
    kn = (1.0 + 0.25 * _rand_bf16((D,), seed + 3).float()).bfloat16()
    return x, Wq, qn, kn


@pytest.mark.parametrize("shift", [1000, 1 << 20])
def test_rope_scores_depend_only_on_relative_position(shift):
    """(R_p q) . (R_p' k) = q . R_(p'-p) k: shifting every position leaves every q.k unchanged."""
    Hq, Hkv, D = 2, 1, 32
    x, Wq, qn, kn = _proj_case(12, Hq, Hkv, D, 64, 31)
    pos = np.sort(np.random.default_rng(0).choice(5000, 12, replace=False)).astype(np.int32)
    Q0, K0, _ = oracle.qkv_rope(x, Wq, pos, 1e4, Hq, Hkv, D, qn, kn)
    Q1, K1, _ = oracle.qkv_rope(x, Wq, pos + shift, 1e4, Hq, Hkv, D, qn, kn)
    for h in range(Hq):
        a, b = Q0[:, h] @ K0[:, 0].T, Q1[:, h] @ K1[:, 0].T
        assert np.allclose(a, b, rtol=1e-9, atol=1e-9 * np.abs(a).max())
    assert not np.allclose(Q0, Q1)  # the rotation itself did move


def test_rope_preserves_head_norms_and_leaves_v_alone():
    Hq, Hkv, D = 4, 2, 64
    x, Wq, _, _ = _proj_case(10, Hq, Hkv, D, 64, 41)
    pos = np.arange(10, dtype=np.int32) * 7919
    Q0, K0, V0 = oracle.qkv_rope(x, Wq, np.zeros(10, np.int32), 1e6, Hq, Hkv, D)
    Q1, K1, V1 = oracle.qkv_rope(x, Wq, pos, 1e6, Hq, Hkv, D)
    assert np.allclose(np.linalg.norm(Q0, axis=-1), np.linalg.norm(Q1, axis=-1), rtol=1e-12)
    assert np.allclose(np.linalg.norm(K0, axis=-1), np.linalg.norm(K1, axis=-1), rtol=1e-12)
    half = D // 2  # each (j, j + D/2) pair keeps its own length
    pair0 = Q0[..., :half] ** 2 + Q0[..., half:] ** 2
    pair1 = Q1[..., :half] ** 2 + Q1[..., half:] ** 2
    assert np.allclose(pair0, pair1, rtol=1e-10, atol=1e-12)
    assert np.array_equal(V0, V1)


def test_head_norm_is_per_head_and_scale_free():
    Hq, Hkv, D = 4, 2, 32
    x, Wq, _, _ = _proj_case(8, Hq, Hkv, D, 64, 51)
    ones = _bf16(np.ones(D, np.float32))
    pos = np.arange(8, dtype=np.int32) * 3
    Q, K, _ = oracle.qkv_rope(x, Wq, pos, 1e6, Hq, Hkv, D, ones, ones, eps=0.0)
    assert np.allclose(np.mean(Q ** 2, axis=-1), 1.0, rtol=1e-12)   # every head has unit RMS
    assert np.allclose(np.mean(K ** 2, axis=-1), 1.0, rtol=1e-12)
    Q4, K4, V4 = oracle.qkv_rope((x.float() * 4).bfloat16(), Wq, pos, 1e6, Hq, Hkv, D, ones, ones, eps=0.0)
    assert np.allclose(Q4, Q, rtol=1e-12, atol=1e-12) and np.allclose(K4, K, rtol=1e-12, atol=1e-12)
    _, _, V = oracle.qkv_rope(x, Wq, pos, 1e6, Hq, Hkv, D, ones, ones, eps=0.0)
    assert np.allclose(V4, 4 * V, rtol=1e-12)


def test_pruning_commutes_with_projection_at_original_positions():
    """Projecting the kept rows at their original positions equals projecting the whole
    prompt at positions 0..n-1 and keeping those rows."""
    Hq, Hkv, D = 2, 1, 32
    x, Wq, qn, kn = _proj_case(64, Hq, Hkv, D, 64, 61)
    kept = np.sort(np.random.default_rng(1).choice(64, 20, replace=False)).astype(np.int32)
    full = oracle.qkv_rope(x, Wq, np.arange(64, dtype=np.int32), 1e6, Hq, Hkv, D, qn, kn)
    pruned = oracle.qkv_rope(x[torch.as_tensor(kept, dtype=torch.long)], Wq, kept, 1e6, Hq, Hkv, D, qn, kn)
    for a, b in zip(full, pruned):
        assert np.array_equal(a[kept], b)
    rows = oracle.qkv_rope(x, Wq, np.arange(64, dtype=np.int32), 1e6, Hq, Hkv, D, qn, kn, rows=kept)
    for a, b in zip(full, rows):
        assert np.array_equal(a[kept], b)


# ============================================================================ attention backward
def _bwd_case(S, Hq, Hkv, D, seed, quant=False):
    g = torch.Generator().manual_seed(seed)
    Q = torch.randn(S, Hq, D, generator=g).to(torch.bfloat16)
    K = torch.randn(S, Hkv, D, generator=g).to(torch.bfloat16)
    V = torch.randn(S, Hkv, D, generator=g).to(torch.bfloat16)
    dO = torch.randn(S, Hq, D, generator=g).to(torch.bfloat16)
    s = torch.randn(S, generator=g)
    gain = 0.5 + torch.rand(Hq, generator=g)
    if quant:  # on a 2^-8 grid, so s +- 2^-10 and gain +- 2^-10 stay exact in fp32
        s = torch.round(s * 256) / 256
        gain = torch.round(gain * 256) / 256
    return Q, K, V, dO, s, gain


def _autograd_backward(Q, K, V, dO, s, gain, tau):
    """Independent fp64 torch forward (explicit softmax over masked logits) and torch.autograd."""
    q, k, v, do = (t.double() for t in (Q, K, V, dO))
    S, Hq, D = q.shape
    Hkv = k.shape[1]
    sv = s.double().clone().requires_grad_(True)
    gv = gain.double().clone().requires_grad_(True)
    tv = torch.tensor(float(tau), dtype=torch.float64, requires_grad=True)
    kk = k.repeat_interleave(Hq // Hkv, dim=1)
    vv = v.repeat_interleave(Hq // Hkv, dim=1)
    logits = tv * torch.einsum("ihd,jhd->hij", q, kk) / math.sqrt(D) + gv[:, None, None] * sv[None, None, :]
    mask = torch.tril(torch.ones(S, S, dtype=torch.bool))
    logits = logits.masked_fill(~mask, float("-inf"))
    out = torch.einsum("hij,jhd->ihd", torch.softmax(logits, dim=-1), vv)
    (out * do).sum().backward()
    return sv.grad.numpy(), gv.grad.numpy(), float(tv.grad)


@pytest.mark.parametrize("S,Hq,Hkv,D,tau,seed", [(24, 4, 2, 16, 1.1, 0), (40, 2, 1, 8, -0.7, 1), (17, 2, 2, 32, 0.0, 2)])
def test_backward_matches_torch_autograd(S, Hq, Hkv, D, tau, seed):
    Q, K, V, dO, s, gain = _bwd_case(S, Hq, Hkv, D, seed)
    ds, dg, dt = oracle.gated_attention_backward(Q, K, V, s, gain, tau, dO)
    rs, rg, rt = _autograd_backward(Q, K, V, dO, s, gain, tau)
    assert np.allclose(ds, rs, rtol=1e-10, atol=1e-12)
    assert np.allclose(dg, rg, rtol=1e-10, atol=1e-12)
    assert math.isclose(dt, rt, rel_tol=1e-10, abs_tol=1e-12)


def _loss(Q, K, V, dO, s, gain, tau):
    """sum(dO * O) with O from the (separately pinned) forward oracle."""
    return float(np.sum(dO.double().numpy() * oracle.gated_attention(Q, K, V, s, gain, tau)))


def test_backward_matches_central_differences_of_the_forward():
    Q, K, V, dO, s, gain = _bwd_case(16, 2, 1, 8, 5, quant=True)
    tau = 0.9
    ds, dg, dt = oracle.gated_attention_backward(Q, K, V, s, gain, tau, dO)
    eps = 2.0 ** -10
    for j in (0, 3, 9, 15):
        e = torch.zeros_like(s)
        e[j] = eps
        fd = (_loss(Q, K, V, dO, s + e, gain, tau) - _loss(Q, K, V, dO, s - e, gain, tau)) / (2 * eps)
        assert math.isclose(ds[j], fd, rel_tol=1e-4, abs_tol=1e-6), (j, ds[j], fd)
    for h in range(2):
        e = torch.zeros_like(gain)
        e[h] = eps
        fd = (_loss(Q, K, V, dO, s, gain + e, tau) - _loss(Q, K, V, dO, s, gain - e, tau)) / (2 * eps)
        assert math.isclose(dg[h], fd, rel_tol=1e-4, abs_tol=1e-6), (h, dg[h], fd)
    fd = (_loss(Q, K, V, dO, s, gain, tau + eps) - _loss(Q, K, V, dO, s, gain, tau - eps)) / (2 * eps)
    assert math.isclose(dt, fd, rel_tol=1e-4, abs_tol=1e-6), (dt, fd)


def test_backward_hand_worked_fixture():
    with open(os.path.join(GOLDEN, "attention_backward_worked.json")) as f:
        c = json.load(f)
    S, Hq, Hkv, D = c["S"], c["Hq"], c["Hkv"], c["D"]
    Q = _bf16(np.asarray(c["q"], np.float32).reshape(S, Hq, D))
    K = _bf16(np.asarray(c["k"], np.float32).reshape(S, Hkv, D))
    V = _bf16(np.asarray(c["v"], np.float32).reshape(S, Hkv, D))
    dO = _bf16(np.asarray(c["dO"], np.float32).reshape(S, Hq, D))
    ds, dg, dt = oracle.gated_attention_backward(Q, K, V, np.asarray(c["s"], np.float32),
                                                 np.asarray(c["gain"], np.float32), c["tau"], dO)
    assert np.allclose(ds, c["ds"], rtol=0, atol=c["tol"])
    assert np.allclose(dg, c["dgain"], rtol=0, atol=c["tol"])
    assert abs(dt - c["dtau"]) <= c["tol"]


def test_backward_invariants():
    Q, K, V, dO, s, gain = _bwd_case(30, 4, 2, 16, 7)
    ds, dg, dt = oracle.gated_attention_backward(Q, K, V, s, gain, 1.3, dO)
    # a constant added to every score leaves each softmax row unchanged
    assert abs(ds.sum()) <= 1e-12 * np.abs(ds).sum()
    # no gain: the scores do not reach the logits
    ds0, _, _ = oracle.gated_attention_backward(Q, K, V, s, torch.zeros_like(gain), 1.3, dO)
    assert np.all(ds0 == 0.0)
    # no upstream gradient
    z = oracle.gated_attention_backward(Q, K, V, s, gain, 1.3, torch.zeros_like(dO))
    assert np.all(z[0] == 0) and np.all(z[1] == 0) and z[2] == 0
    # the last token's score only reaches the last row
    dsl, _, _ = oracle.gated_attention_backward(Q[-1:], K[-1:], V[-1:], s[-1:], gain, 1.3, dO[-1:])
    assert dsl[0] == 0.0  # one key: softmax is constant


def test_lse_matches_torch_logsumexp():
    Q, K, _, _, s, gain = _bwd_case(33, 4, 2, 16, 9)
    tau = 1.2
    q, k = Q.double(), K.double().repeat_interleave(2, dim=1)
    logits = tau * torch.einsum("ihd,jhd->hij", q, k) / 4.0 + gain.double()[:, None, None] * s.double()[None, None, :]
    logits = logits.masked_fill(~torch.tril(torch.ones(33, 33, dtype=torch.bool)), float("-inf"))
    ref = torch.logsumexp(logits, dim=-1).T.numpy()
    assert np.allclose(oracle.gated_attention_lse(Q, K, s, gain, tau), ref, rtol=1e-12, atol=1e-12)
    rows = [32, 0, 7]
    assert np.allclose(oracle.gated_attention_lse(Q, K, s, gain, tau, rows=rows), ref[rows], rtol=1e-12, atol=1e-12)


def test_oracle_results_do_not_depend_on_thread_count():
    # the timed CPU baseline also runs the oracle on one core; every row is computed by
    # one thread in a fixed order, so the count cannot change a single bit
    g = torch.Generator().manual_seed(12)
    S, Hq, Hkv, D = 70, 4, 2, 16
    Q = torch.randn(S, Hq, D, generator=g).to(torch.bfloat16)
    K = torch.randn(S, Hkv, D, generator=g).to(torch.bfloat16)
    V = torch.randn(S, Hkv, D, generator=g).to(torch.bfloat16)
    s = torch.randn(S, generator=g)
    gain = 0.5 + torch.rand(Hq, generator=g)
    many = oracle.num_threads()
    ref = oracle.gated_attention(Q, K, V, s, gain, 1.1)
    oracle.set_num_threads(1)
    try:
        assert oracle.num_threads() == 1
        one = oracle.gated_attention(Q, K, V, s, gain, 1.1)
    finally:
        oracle.set_num_threads(many)
    assert oracle.num_threads() == many
    assert np.array_equal(one, ref)

"""The seeded synthetic inputs follow their stated recipe (host only): shapes, the question
at the end of every request, the needle share, the score mixture, the weight scales, the
tie-heavy arrays, and bitwise repeatability."""
import math

import numpy as np
import torch

from learned_token_pruning_mlp_b200 import workloads as W


def test_every_workload_has_consistent_shapes():
    for name, w in W.WORKLOADS.items():
        assert w.n == sum(s.n for s in w.segments)
        assert w.hq % w.hkv == 0 and w.head_dim in (64, 128)
        for s in w.segments:
            assert 0 <= s.q < s.n and 0 < s.k <= s.n - s.q


def test_question_tokens_sit_at_the_end_of_every_request():
    w = W.get("ragged_4req")
    m = W.doc_mask(w).numpy()
    off = 0
    for s in w.segments:
        seg = m[off:off + s.n]
        assert seg[:s.n - s.q].all() and not seg[s.n - s.q:].any()
        off += s.n


def test_gate_inputs_shapes_scales_and_repeatability():
    w = W.get("tiny_n512")
    a = W.gate_inputs(w)
    b = W.gate_inputs(w)
    for x, y in zip(a, b):
        assert x.dtype == torch.bfloat16 and torch.equal(x, y)
    hidden, W1, b1, W2, b2 = a
    assert hidden.shape == (w.n, w.d) and W1.shape == (w.h, w.d) and b1.shape == (w.h,)
    assert W2.shape == (w.h,) and b2.shape == (1,)
    assert abs(W1.float().std().item() - 1 / math.sqrt(w.d)) < 0.1 / math.sqrt(w.d)
    assert abs(hidden.float().std().item() - 1.0) < 0.05


def test_needles_scale_one_percent_of_document_rows():
    w = W.get("qwen3_1p7b_n16k")
    hidden = W.gate_inputs(w)[0].float()
    doc = W.doc_mask(w).bool()
    norms = hidden.pow(2).mean(dim=1).sqrt()
    loud = norms > 2.5  # N(0,1) rows have rms ~1, needles ~4
    assert not loud[~doc].any()
    n_doc = int(doc.sum())
    assert int(loud.sum()) == max(1, round(0.01 * n_doc))


def test_selection_scores_mix_two_percent_of_a_shifted_normal():
    w = W.get("qwen3_1p7b_n128k")
    s = W.selection_scores(w).numpy()
    assert s.shape == (w.n,) and s.dtype == np.float32
    frac_high = float(np.mean(s > 2.5))
    # N(0,1) alone puts 0.62 % above 2.5; 2 % of N(4,1) adds ~1.87 %
    assert 0.022 < frac_high < 0.027
    assert W.selection_scores(W.get("qwen3_1p7b_n16k")) is None


def test_tie_scores_take_exactly_the_stated_levels():
    t = W.tie_scores(4096, 3, levels=16).numpy()
    assert len(np.unique(t)) == 16
    assert np.array_equal(t, W.tie_scores(4096, 3, levels=16).numpy())


def test_attention_inputs_differ_by_layer_and_repeat_by_seed():
    w = W.get("tiny_n512")
    q0, k0, v0 = W.attention_inputs(w, 100, layer=0)
    q1, _, _ = W.attention_inputs(w, 100, layer=1)
    assert q0.shape == (100, w.hq, w.head_dim) and k0.shape == (100, w.hkv, w.head_dim)
    assert not torch.equal(q0, q1)
    assert torch.equal(q0, W.attention_inputs(w, 100, layer=0)[0])
    gain, tau = W.attention_params(w)
    assert gain.shape == (w.hq,) and bool(((gain >= 0.5) & (gain < 1.5)).all()) and tau == w.tau

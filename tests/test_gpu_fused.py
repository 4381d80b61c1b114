"""The fused gate -> top-K -> gather call (the gate's epilogue histograms the selector's
first radix digit) against the three separate calls and the fp64 oracle.

  * the fused call's scores, kept indices, count, gathered rows and scores equal those
    of tg_gate_score -> tg_select_topk -> tg_gather on the same inputs, bitwise (the
    same kernels compute them; only the first radix pass takes another route);
  * the per-CTA histograms in the workspace add up to the histogram of the top byte of
    every document token's selection key, counted here from the returned scores;
  * scores against the oracle gate within the gate tolerance, and the kept set against
    the oracle's selection on the oracle's own scores: identical except for document
    tokens whose oracle score lies within that tolerance of the K-th score (where both
    selections are correct), checked to be exactly such tokens.
"""
import math

import numpy as np
import pytest
import torch

import oracle
import learned_token_pruning_mlp_b200 as tg
from learned_token_pruning_mlp_b200 import workloads as W
from test_gpu_parity import assert_gate_close

pytestmark = pytest.mark.gpu
DEV = "cuda:0"


@pytest.fixture(scope="module", autouse=True)
def _gpu():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from learned_token_pruning_mlp_b200 import build
    build.build()
    tg.tg_get_device_error()
    yield


def _key_top_bytes(scores, mask):
    """Top byte of the selection order key of each document token (numbers only)."""
    b = scores.astype(np.float32).view(np.uint32).copy()
    b[b == 0x80000000] = 0
    key = np.where(b & 0x80000000, ~b, b | 0x80000000).astype(np.uint32)
    isnan = np.isnan(scores)
    key[isnan] = 1
    return (key[mask != 0] >> 24).astype(np.int64)


def _run_both(w, K):
    hidden, W1, b1, W2, b2 = (t.to(DEV) for t in W.gate_inputs(w))
    mask = W.doc_mask(w).to(DEV)
    n = w.n
    S = min(K, int(mask.sum().item())) + int((mask == 0).sum().item())
    ws = torch.empty(tg.tg_select_fused_workspace(n), dtype=torch.uint8, device=DEV)
    f_scores, f_kept, f_nk, f_hk, f_sk = tg.tg_select_fused(hidden, W1, b1, W2, b2, mask, K, n_rows=S,
                                                            workspace=ws)
    scores = tg.tg_gate_score(hidden, W1, b1, W2, b2)
    kept, nk = tg.tg_select_topk(scores, mask, K)
    hk, sk = tg.tg_gather(hidden, kept, n_rows=S, n_kept=nk, scores=scores)
    torch.cuda.synchronize()
    return dict(f=(f_scores, f_kept, f_nk, f_hk, f_sk), u=(scores, kept, nk, hk, sk), ws=ws, S=S, mask=mask)


@pytest.mark.parametrize("name,K", [("tiny_n512", 128), ("tiny_n512", 0), ("tiny_n512", 1000),
                                    ("qwen3_1p7b_n16k", 2048), ("qwen3_1p7b_n128k", 8192),
                                    ("qwen3_1p7b_n128k", 16384), ("ragged_4req", 20000)])
def test_fused_equals_separate_calls(name, K):
    w = W.get(name)
    r = _run_both(w, K)
    f_scores, f_kept, f_nk, f_hk, f_sk = r["f"]
    scores, kept, nk, hk, sk = r["u"]
    S = r["S"]
    assert torch.equal(f_scores, scores)
    assert int(f_nk.item()) == int(nk.item()) == S
    assert torch.equal(f_kept[:S], kept[:S])
    assert torch.equal(f_hk[:S], hk[:S]) and torch.equal(f_sk[:S], sk[:S])
    # the epilogue's histograms add up to the histogram of the document keys' top byte
    parts = r["ws"].view(torch.int32).view(-1, 256).cpu().numpy().astype(np.int64)
    ref = np.bincount(_key_top_bytes(scores.cpu().numpy(), r["mask"].cpu().numpy()), minlength=256)
    assert np.array_equal(parts.sum(0), ref)
    bits = tg.tg_get_device_error()
    assert bits & ~tg.TG_DEVERR_K_GT_NDOC == 0


@pytest.mark.parametrize("name,K", [("tiny_n512", 128), ("qwen3_1p7b_n16k", 2048)])
def test_fused_against_oracle(name, K):
    w = W.get(name)
    hidden, W1, b1, W2, b2 = W.gate_inputs(w)
    mask = W.doc_mask(w)
    n = w.n
    f_scores, f_kept, f_nk, _, _ = tg.tg_select_fused(*(t.to(DEV) for t in (hidden, W1, b1, W2, b2)), mask.to(DEV),
                                                      K, n_rows=0)
    torch.cuda.synchronize()
    ref = np.empty(n)
    for i in range(0, n, 16384):
        ref[i:i + 16384] = oracle.gate_score(hidden[i:i + 16384], W1, b1, W2, b2)
    assert_gate_close(f_scores.cpu().numpy(), ref)
    ref_kept = oracle.select_topk(ref.astype(np.float32), mask, K)
    got = f_kept[:int(f_nk.item())].cpu().numpy()
    assert len(got) == len(ref_kept)
    diff = np.setxor1d(got, ref_kept)
    if len(diff):
        m = mask.numpy() != 0
        doc_scores = np.sort(ref[m])[::-1]
        kth = doc_scores[min(K, len(doc_scores)) - 1]
        rms = math.sqrt(float(np.mean(ref ** 2)))
        tol = 2e-3 * (abs(kth) + rms)  # twice the per-score gate tolerance: both sides may move
        assert np.all(m[diff]) and np.all(np.abs(ref[diff] - kth) <= tol), "selection differs beyond near-ties"

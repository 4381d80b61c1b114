"""Full-size parity of the named workloads, in the launch configuration the bench times.

For every workload and budget the whole path runs on the GPU through the C ABI and
is checked against the fp64 oracle:
  * gate scores on a seeded row sample (first 128, last 128, 256 random rows);
  * top-K bit-exact, both sides reading the same fp32 array: the oracle's own gate
    scores rounded to fp32 (or the workload's fixed selector scores);
  * gather bit-exact, both sides gathering with the oracle's kept indices;
  * gated attention on a row sample (all heads) over the rows the oracle kept;
  * the all-GPU chain (GPU scores -> GPU top-K -> GPU gather) for the properties the
    article fixes: |kept| = K + question length, every question token kept, ascending.
Tolerances are the ones of the parity tests (test_gpu_parity.py).
"""
import numpy as np
import pytest
import torch

import oracle
import learned_token_pruning_mlp_b200 as tg
from learned_token_pruning_mlp_b200 import workloads as W
from test_gpu_parity import assert_gate_close, check_attention

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


_CACHE = {}


def _inputs(name):
    if name not in _CACHE:
        _CACHE.clear()
        w = W.get(name)
        _CACHE[name] = (w, W.gate_inputs(w), W.doc_mask(w), W.selection_scores(w))
    return _CACHE[name]


def _check_structure(kept, mask, k):
    mask = np.asarray(mask)
    n_doc = int(mask.sum())
    q = len(mask) - n_doc
    assert len(kept) == min(k, n_doc) + q
    assert np.all(np.diff(kept) > 0)
    assert set(np.nonzero(mask == 0)[0].tolist()) <= set(kept.tolist())


CASES = [("qwen3_1p7b_n16k", 1024), ("qwen3_1p7b_n16k", 2048), ("qwen3_1p7b_n16k", 4096),
         ("qwen3_1p7b_n32k", 2048), ("qwen3_1p7b_n32k", 4096), ("qwen3_1p7b_n32k", 8192),
         ("qwen3_1p7b_n32k", 32256),
         ("qwen3_1p7b_n128k", 4096), ("qwen3_1p7b_n128k", 8192), ("qwen3_1p7b_n128k", 16384)]


@pytest.mark.parametrize("name,K", CASES)
def test_full_size_path(name, K):
    w0, (hidden, W1, b1, W2, b2), mask, sel = _inputs(name)
    w = w0.with_budget(K)
    n = w.n
    d_hidden = hidden.to(DEV)
    d_w = [t.to(DEV) for t in (W1, b1, W2, b2)]
    d_mask = mask.to(DEV)

    # gate: sampled rows against the oracle
    scores = tg.tg_gate_score(d_hidden, *d_w)
    rows = oracle.sampled_rows(n, seed=K)
    assert_gate_close(scores.cpu().numpy()[rows], oracle.gate_score(hidden[rows], W1, b1, W2, b2))

    # all-GPU chain: structural properties
    gpu_sel = sel.to(DEV) if sel is not None else scores
    kept_g, nk_g = tg.tg_select_topk(gpu_sel, d_mask, K)
    S = int(nk_g.item())
    _check_structure(kept_g[:S].cpu().numpy(), mask.numpy(), K)

    # top-K on a shared fp32 array the oracle produced (or the workload's fixed scores)
    if sel is not None:
        shared = sel.numpy()
    else:
        shared = np.empty(n, dtype=np.float32)
        chunk = 16384
        for i in range(0, n, chunk):  # the oracle gate over every token, in row blocks
            shared[i:i + chunk] = oracle.gate_score(hidden[i:i + chunk], W1, b1, W2, b2).astype(np.float32)
    ref_kept = oracle.select_topk(shared, mask, K)
    kept, nk = tg.tg_select_topk(torch.as_tensor(shared).to(DEV), d_mask, K)
    assert int(nk.item()) == len(ref_kept)
    assert np.array_equal(kept[:len(ref_kept)].cpu().numpy(), ref_kept)

    # gather with the oracle's kept indices
    S = len(ref_kept)
    d_kept = torch.as_tensor(ref_kept).to(DEV)
    hk, sk = tg.tg_gather(d_hidden, d_kept, scores=torch.as_tensor(shared).to(DEV))
    ref_hk, ref_sk = oracle.gather(hidden, ref_kept, shared)
    assert np.array_equal(hk.cpu().view(torch.int16).numpy().view(np.uint16), ref_hk)
    assert np.array_equal(sk.cpu().numpy(), ref_sk)

    # gated attention over the kept tokens (layer 0 of the workload), sampled rows
    Q, Kc, V = W.attention_inputs(w, S, layer=0)
    gain, tau = W.attention_params(w)
    O = tg.tg_gated_attention(Q.to(DEV), Kc.to(DEV), V.to(DEV), torch.as_tensor(ref_sk).to(DEV), gain.to(DEV), tau)
    arows = oracle.sampled_rows(S, seed=S, head=64, tail=64, rand=128)
    check_attention(O.float().cpu().numpy()[arows], Q, Kc, V, ref_sk, gain, tau, rows=arows)
    bits = tg.tg_get_device_error()
    assert bits & ~tg.TG_DEVERR_K_GT_NDOC == 0


def test_full_size_ragged_batch():
    """Four packed requests (8k, 24k, 48k, 64k tokens; questions 128..1024; K = N/8)."""
    w, (hidden, W1, b1, W2, b2), mask, _ = _inputs("ragged_4req")
    n = w.n
    cu = w.cu_seqlens()
    ks = torch.tensor([s.k for s in w.segments], dtype=torch.int32)
    d_hidden = hidden.to(DEV)
    scores = tg.tg_gate_score(d_hidden, *(t.to(DEV) for t in (W1, b1, W2, b2)))
    rows = oracle.sampled_rows(n, seed=4)
    assert_gate_close(scores.cpu().numpy()[rows], oracle.gate_score(hidden[rows], W1, b1, W2, b2))

    shared = np.empty(n, dtype=np.float32)
    for i in range(0, n, 16384):
        shared[i:i + 16384] = oracle.gate_score(hidden[i:i + 16384], W1, b1, W2, b2).astype(np.float32)
    ref_kept, ref_cu = oracle.select_topk_varlen(shared, mask, cu.numpy(), ks.numpy())
    max_len = max(s.n for s in w.segments)
    kept, cu_kept = tg.tg_select_topk_varlen(torch.as_tensor(shared).to(DEV), mask.to(DEV), cu.to(DEV), ks.to(DEV),
                                             max_len)
    assert np.array_equal(cu_kept.cpu().numpy(), ref_cu)
    assert np.array_equal(kept[:ref_cu[-1]].cpu().numpy(), ref_kept)

    S = int(ref_cu[-1])
    hk, sk = tg.tg_gather(d_hidden, torch.as_tensor(ref_kept).to(DEV), scores=torch.as_tensor(shared).to(DEV))
    ref_hk, ref_sk = oracle.gather(hidden, ref_kept, shared)
    assert np.array_equal(hk.cpu().view(torch.int16).numpy().view(np.uint16), ref_hk)

    Q, Kc, V = W.attention_inputs(w, S, layer=0)
    gain, tau = W.attention_params(w)
    max_kept = int(np.max(np.diff(ref_cu)))
    O = tg.tg_gated_attention_varlen(Q.to(DEV), Kc.to(DEV), V.to(DEV), torch.as_tensor(ref_sk).to(DEV), gain.to(DEV),
                                     tau, torch.as_tensor(ref_cu).to(DEV), max_kept)
    # sampled rows from every request: first, last and random rows of each
    rng = np.random.default_rng(0)
    arows = []
    for b in range(len(ref_cu) - 1):
        lo, hi = int(ref_cu[b]), int(ref_cu[b + 1])
        arows += list(range(lo, min(lo + 32, hi))) + list(range(max(lo, hi - 32), hi))
        arows += list(rng.choice(np.arange(lo, hi), size=min(32, hi - lo), replace=False))
    arows = np.unique(np.asarray(arows, dtype=np.int64))
    check_attention(O.float().cpu().numpy()[arows], Q, Kc, V, ref_sk, gain, tau, rows=arows, cu=ref_cu)
    assert tg.tg_get_device_error() == 0

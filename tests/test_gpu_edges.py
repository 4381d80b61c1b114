"""Empty and degenerate inputs of the calls around the hot path, on the GPU through the
C ABI: nothing to compute must still leave every output defined (counts 0, gradients 0)
and touch nothing it does not own."""
import pytest
import torch

import learned_token_pruning_mlp_b200 as tg
from learned_token_pruning_mlp_b200 import workloads as W

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


def test_projections_with_no_rows():
    x = torch.empty(0, 64, dtype=torch.bfloat16, device=DEV)
    Wt = torch.randn(96, 64, device=DEV).to(torch.bfloat16)
    y = tg.tg_linear(x, Wt)
    assert y.shape == (0, 96)
    Wq = torch.randn((4 + 2 * 2) * 64, 64, device=DEV).to(torch.bfloat16)
    Q, K, V = tg.tg_qkv_rope(x, Wq, torch.empty(0, dtype=torch.int32, device=DEV), 1e6, 4, 2, 64)
    assert Q.shape == (0, 4, 64) and K.shape == (0, 2, 64)
    torch.cuda.synchronize()
    assert tg.tg_get_device_error() == 0


def test_backward_with_no_tokens_writes_zero_gradients():
    Hq, Hkv, D = 4, 2, 64
    e = lambda *shape: torch.empty(*shape, dtype=torch.bfloat16, device=DEV)  # noqa: E731
    Q, K, V, dO = e(0, Hq, D), e(0, Hkv, D), e(0, Hkv, D), e(0, Hq, D)
    s = torch.empty(0, device=DEV)
    gain = torch.ones(Hq, device=DEV)
    dg = torch.full((Hq,), 5.0, device=DEV)
    dt = torch.full((1,), 5.0, device=DEV)
    ds, dg, dt = tg.tg_gated_attention_backward(Q, K, V, s, gain, 1.1, Q, dO, torch.empty(0, Hq, device=DEV),
                                                dgain=dg, dtau=dt)
    torch.cuda.synchronize()
    assert ds.numel() == 0 and torch.all(dg == 0) and float(dt.item()) == 0.0
    dg.fill_(5.0)
    dt.fill_(5.0)
    tg.tg_gated_attention_backward_noalloc(Q, K, V, s, gain, 1.1, Q, dO, torch.empty(0, Hq, device=DEV),
                                           dgain=dg, dtau=dt)
    torch.cuda.synchronize()
    assert torch.all(dg == 0) and float(dt.item()) == 0.0
    assert tg.tg_get_device_error() == 0


def test_train_forward_with_no_tokens():
    Hq, Hkv, D = 4, 2, 64
    e = lambda *shape: torch.empty(*shape, dtype=torch.bfloat16, device=DEV)  # noqa: E731
    O, lse, O32 = tg.tg_gated_attention_train(e(0, Hq, D), e(0, Hkv, D), e(0, Hkv, D), torch.empty(0, device=DEV),
                                              torch.ones(Hq, device=DEV), 1.1)
    torch.cuda.synchronize()
    assert O.numel() == 0 and lse.numel() == 0
    assert tg.tg_get_device_error() == 0


def test_fused_select_with_no_tokens_and_with_only_question_tokens():
    w = W.get("tiny_n512")
    _, W1, b1, W2, b2 = (t.to(DEV) for t in W.gate_inputs(w))
    hidden = torch.empty(0, w.d, dtype=torch.bfloat16, device=DEV)
    kept = torch.full((4,), -7, dtype=torch.int32, device=DEV)
    nk = torch.full((1,), -7, dtype=torch.int32, device=DEV)
    tg.tg_select_fused(hidden, W1, b1, W2, b2, torch.empty(0, dtype=torch.uint8, device=DEV), 10, n_rows=0,
                       kept_idx=kept, n_kept=nk, cap=4)
    torch.cuda.synchronize()
    assert int(nk.item()) == 0
    # every token a question token: all are kept, none selected
    n = 300
    hidden = torch.randn(n, w.d, device=DEV).to(torch.bfloat16)
    mask = torch.zeros(n, dtype=torch.uint8, device=DEV)
    scores, kept, nk, hk, sk = tg.tg_select_fused(hidden, W1, b1, W2, b2, mask, 10, n_rows=n)
    torch.cuda.synchronize()
    assert int(nk.item()) == n
    assert torch.equal(kept[:n], torch.arange(n, dtype=torch.int32, device=DEV))
    assert torch.equal(hk[:n], hidden) and torch.equal(sk[:n], scores)
    assert tg.tg_get_device_error() & ~tg.TG_DEVERR_K_GT_NDOC == 0

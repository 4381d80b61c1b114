"""The allocation-free backward entry point (scratch in a fixed device array inside the
library) against the entry point with a caller workspace, on two calls in a row.

The two run the same kernels on the same inputs, so the results must agree bitwise,
also on the second call (the static scratch is reused, not re-initialised).  The file
is collected last so that it also runs after every other test has used the library;
it passes alone too.
"""
import pytest
import torch

import learned_token_pruning_mlp_b200 as tg

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


def _inputs(S, Hq, Hkv, D, seed):
    g = torch.Generator().manual_seed(seed)
    Q = torch.randn(S, Hq, D, generator=g).to(torch.bfloat16).to(DEV)
    K = torch.randn(S, Hkv, D, generator=g).to(torch.bfloat16).to(DEV)
    V = torch.randn(S, Hkv, D, generator=g).to(torch.bfloat16).to(DEV)
    dO = torch.randn(S, Hq, D, generator=g).to(torch.bfloat16).to(DEV)
    s = torch.randn(S, generator=g).to(DEV)
    gain = (0.5 + torch.rand(Hq, generator=g)).to(DEV)
    return Q, K, V, dO, s, gain


@pytest.mark.parametrize("S,Hq,Hkv,D", [(8704, 16, 8, 128), (300, 4, 2, 64)])
def test_noalloc_matches_workspace_entry_point_twice(S, Hq, Hkv, D):
    Q, K, V, dO, s, gain = _inputs(S, Hq, Hkv, D, S + Hq)
    O, lse, O32 = tg.tg_gated_attention_train(Q, K, V, s, gain, 1.1)
    for call in range(2):
        ref = tg.tg_gated_attention_backward(Q, K, V, s, gain, 1.1, O, dO, lse, O32)
        got = tg.tg_gated_attention_backward_noalloc(Q, K, V, s, gain, 1.1, O, dO, lse, O32)
        torch.cuda.synchronize()
        for a, b, name in zip(got, ref, ("ds", "dgain", "dtau")):
            assert torch.equal(a, b), f"call {call}: {name} differs"
    assert tg.tg_get_device_error() == 0


def test_noalloc_rejects_sizes_beyond_its_scratch():
    Q, K, V, dO, s, gain = _inputs(30000, 16, 8, 128, 1)
    O = torch.empty_like(Q)
    lse = torch.empty(30000, 16, device=DEV)
    with pytest.raises(tg.TokenGateError, match="static scratch"):
        tg.tg_gated_attention_backward_noalloc(Q, K, V, s, gain, 1.1, O, dO, lse)

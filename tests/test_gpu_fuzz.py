"""Seeded random cases of the hot-path calls against the fp64 oracle.

Each case draws its shapes and parameters from a fixed seed (so a failure reproduces):
attention on both kernels (random length, heads, head dimension, temperature sign and
size, gain and score scales, with or without scores), packed batches with random request
lengths (empty ones included) and slack in max_seqlen, the selector with random
budgets, masks and tie-heavy scores, the backward (fed the oracle's forward) and the gate
at random shapes.
"""
import numpy as np
import pytest
import torch

import oracle
import learned_token_pruning_mlp_b200 as tg
from test_gpu_attention_kernels import KERNELS, run
from test_gpu_parity import check_attention

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


def _draw_attention(seed):
    rng = np.random.default_rng(seed)
    S = int(rng.integers(1, 1200))
    Hkv = int(rng.choice([1, 2, 4]))
    Hq = Hkv * int(rng.choice([1, 2, 4]))
    D = int(rng.choice([64, 128]))
    tau = float(rng.choice([-1.0, 1.0]) * rng.uniform(0.05, 3.0))
    g = torch.Generator().manual_seed(seed)
    Q = torch.randn(S, Hq, D, generator=g).to(torch.bfloat16)
    K = torch.randn(S, Hkv, D, generator=g).to(torch.bfloat16)
    V = torch.randn(S, Hkv, D, generator=g).to(torch.bfloat16)
    s = torch.randn(S, generator=g) * float(rng.uniform(0.1, 6.0))
    gain = torch.rand(Hq, generator=g) * float(rng.uniform(0.2, 2.0)) - float(rng.uniform(0.0, 0.5))
    with_scores = bool(rng.random() < 0.8)
    return S, Q, K, V, (s if with_scores else None), (gain if with_scores else None), tau


@pytest.mark.parametrize("kernel", KERNELS)
@pytest.mark.parametrize("seed", range(100, 140))
def test_attention_random_cases(kernel, seed):
    S, Q, K, V, s, gain, tau = _draw_attention(seed)
    O = run(kernel, tg.tg_gated_attention, Q, K, V, s, gain, tau)
    if s is None:
        s, gain = np.zeros(S, np.float32), np.zeros(Q.shape[1], np.float32)
    check_attention(O.float().numpy(), Q, K, V, s, gain, tau, max_abs_below=2.0)


@pytest.mark.parametrize("kernel", KERNELS)
@pytest.mark.parametrize("seed", range(200, 220))
def test_attention_varlen_random_batches(kernel, seed):
    rng = np.random.default_rng(seed)
    B = int(rng.integers(1, 7))
    lens = [int(x) for x in rng.integers(0, 600, size=B)]
    if rng.random() < 0.3:
        lens[int(rng.integers(0, B))] = 0
    cu = np.concatenate([[0], np.cumsum(lens)]).astype(np.int32)
    total = int(cu[-1])
    if total == 0:
        lens[0] = 5
        cu = np.concatenate([[0], np.cumsum(lens)]).astype(np.int32)
        total = int(cu[-1])
    max_seqlen = max(lens) + int(rng.integers(0, 200))  # an upper bound, not the exact maximum
    max_seqlen = min(max_seqlen, total)
    g = torch.Generator().manual_seed(seed)
    Hq, Hkv, D = 4, 2, 128
    Q = torch.randn(total, Hq, D, generator=g).to(torch.bfloat16)
    K = torch.randn(total, Hkv, D, generator=g).to(torch.bfloat16)
    V = torch.randn(total, Hkv, D, generator=g).to(torch.bfloat16)
    s = torch.randn(total, generator=g) * 2.0
    gain = 0.5 + torch.rand(Hq, generator=g)
    O = run(kernel, tg.tg_gated_attention_varlen, Q, K, V, s, gain, 1.1, torch.as_tensor(cu).to(DEV), max_seqlen,
            max_seqlen=max_seqlen, B=B)
    # short requests give rows with few keys, near one V row and above 2 in magnitude (half
    # a bf16 ulp there is 2^-7): max-abs 1e-2 is required below 2, the per-element
    # rounding bound of every output
    check_attention(O.float().numpy(), Q, K, V, s, gain, 1.1, cu=cu, max_abs_below=2.0)


@pytest.mark.parametrize("seed", range(300, 340))
def test_topk_random_cases(seed):
    rng = np.random.default_rng(seed)
    n = int(rng.choice([int(rng.integers(1, 9000)), int(rng.integers(9000, 150000))]))
    kind = seed % 4
    if kind == 0:
        s = rng.standard_normal(n).astype(np.float32)
    elif kind == 1:
        s = rng.integers(0, 7, size=n).astype(np.float32)  # heavy ties
    elif kind == 2:
        s = (rng.standard_normal(n) * 1e-30).astype(np.float32)  # tiny magnitudes, -0.0 and +0.0
        s[rng.random(n) < 0.1] = -0.0
    else:
        s = rng.standard_normal(n).astype(np.float32)
        s[rng.random(n) < 0.05] = np.nan
        s[rng.random(n) < 0.02] = np.inf
    mask = (rng.random(n) < rng.uniform(0.5, 1.0)).astype(np.uint8)
    k = int(rng.integers(0, n + 2))
    ref = oracle.select_topk(s, mask, k)
    kept, n_kept = tg.tg_select_topk(torch.as_tensor(s).to(DEV), torch.as_tensor(mask).to(DEV), k)
    assert int(n_kept.item()) == len(ref)
    assert np.array_equal(kept[:len(ref)].cpu().numpy(), ref)
    assert tg.tg_get_device_error() & ~tg.TG_DEVERR_K_GT_NDOC == 0


@pytest.mark.parametrize("seed", range(400, 416))
def test_backward_random_cases(seed):
    """The backward fed the oracle's forward (kernel parity) at random shapes, temperatures
    (either sign), gains and score scales."""
    from test_gpu_backward import _gpu_backward_on_oracle_forward, assert_kernel_close
    rng = np.random.default_rng(seed)
    S = int(rng.integers(64, 900))
    Hkv = int(rng.choice([1, 2, 4]))
    Hq = Hkv * int(rng.choice([1, 2, 4]))
    D = int(rng.choice([64, 128]))
    tau = float(rng.choice([-1.0, 1.0]) * rng.uniform(0.2, 2.5))
    g = torch.Generator().manual_seed(seed)
    Q = torch.randn(S, Hq, D, generator=g).to(torch.bfloat16)
    K = torch.randn(S, Hkv, D, generator=g).to(torch.bfloat16)
    V = torch.randn(S, Hkv, D, generator=g).to(torch.bfloat16)
    dO = torch.randn(S, Hq, D, generator=g).to(torch.bfloat16)
    s = torch.randn(S, generator=g) * float(rng.uniform(0.2, 3.0))
    gain = 0.25 + torch.rand(Hq, generator=g) * float(rng.uniform(0.5, 1.5))
    got = _gpu_backward_on_oracle_forward(Q, K, V, dO, s, gain, tau)
    assert_kernel_close(got, oracle.gated_attention_backward(Q, K, V, s, gain, tau, dO))
    assert tg.tg_get_device_error() == 0


@pytest.mark.parametrize("seed", range(500, 510))
def test_gate_random_cases(seed):
    from test_gpu_parity import assert_gate_close
    rng = np.random.default_rng(seed)
    n = int(rng.integers(1, 5000))
    d = 8 * int(rng.integers(1, 300))
    h = 16 * int(rng.integers(1, 17))
    g = torch.Generator().manual_seed(seed)
    x = torch.randn(n, d, generator=g).to(torch.bfloat16)
    W1 = (torch.randn(h, d, generator=g) / d ** 0.5).to(torch.bfloat16)
    b1 = (torch.randn(h, generator=g) / d ** 0.5).to(torch.bfloat16)
    W2 = (torch.randn(h, generator=g) / h ** 0.5).to(torch.bfloat16)
    b2 = (torch.randn(1, generator=g) / h ** 0.5).to(torch.bfloat16)
    got = tg.tg_gate_score(*(t.to(DEV) for t in (x, W1, b1, W2, b2)))
    assert_gate_close(got.cpu().numpy(), oracle.gate_score(x, W1, b1, W2, b2))
    assert tg.tg_get_device_error() == 0

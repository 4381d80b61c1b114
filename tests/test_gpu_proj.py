"""Projections of a pruned layer (QKV with per-head norm and rotary embedding at the kept
tokens' positions; output projection with the residual add) vs the fp64 CPU oracle,
through the C ABI.

Tolerance, element-wise: |gpu - oracle| <= 2^-8 |oracle| + 1e-3 rms(oracle).
The GPU rounds its fp32 result to bf16 once; half a bf16 ulp is at most 2^-8 of the
value.  The 1e-3 rms term covers fp32 accumulation over K <= 2048 products (expected
near 1e-5 rms), the fp32 norm and the fp32 sin/cos of the fp64-reduced angle.
The layer chain (projection -> gated attention -> output projection) compares the
GPU chain with the oracle chain, which rounds its intermediates to bf16 as the
buffers between the GPU calls do; a one-ulp difference in an intermediate is allowed
to propagate: |gpu - oracle| <= 2^-7 |oracle| + 1e-2 rms(oracle).
"""
import math

import numpy as np
import pytest
import torch

import oracle
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


def assert_proj_close(got, ref, rtol=2.0 ** -8, rms_tol=1e-3):
    got = np.asarray(got, dtype=np.float64)
    assert np.isfinite(got).all(), "non-finite output"
    rms = math.sqrt(float(np.mean(ref ** 2)))
    bound = rtol * np.abs(ref) + rms_tol * rms
    err = np.abs(got - ref)
    bad = err > bound
    assert not bad.any(), f"{bad.sum()} of {ref.size} outside tolerance; worst {np.max(err / bound):.3f}x the bound"


def _rand(shape, seed, scale=1.0):
    g = torch.Generator().manual_seed(seed)
    return (torch.randn(shape, generator=g) * scale).to(torch.bfloat16)


def _positions(S, span, seed, offset=0):
    g = np.random.default_rng(seed)
    return (np.sort(g.choice(span, S, replace=False)) + offset).astype(np.int32)


# =============================================================================== output projection
@pytest.mark.parametrize("M,K,N,res", [(300, 136, 96, False), (300, 136, 96, True), (1, 8, 32, True),
                                       (1000, 520, 800, True), (257, 2048, 2048, False)])
def test_linear_matches_oracle(M, K, N, res):
    x = _rand((M, K), M + K)
    Wt = _rand((N, K), N, K ** -0.5)
    r = _rand((M, N), 7) if res else None
    y = tg.tg_linear(x.to(DEV), Wt.to(DEV), r.to(DEV) if res else None)
    assert_proj_close(y.float().cpu().numpy(), oracle.linear(x, Wt, r))
    assert tg.tg_get_device_error() == 0


def test_linear_writes_only_its_rows():
    M, K, N = 130, 64, 64
    x, Wt = _rand((M, K), 1), _rand((N, K), 2, 0.125)
    y = torch.full((M + 3, N), 7.0, dtype=torch.bfloat16, device=DEV)
    tg.tg_linear(x.to(DEV), Wt.to(DEV), y=y[:M])
    torch.cuda.synchronize()
    assert torch.all(y[M:] == 7.0)
    assert_proj_close(y[:M].float().cpu().numpy(), oracle.linear(x, Wt))


# =============================================================================== QKV + norm + rotary
@pytest.mark.parametrize("S,d,Hq,Hkv,D,norm,span,offset", [
    (300, 256, 4, 2, 64, False, 512, 0),
    (300, 256, 4, 2, 64, True, 512, 0),
    (700, 2048, 16, 8, 128, True, 131072, 0),
    (129, 520, 2, 1, 128, False, 4096, 0),
    (333, 2048, 16, 8, 128, True, 1 << 20, (1 << 31) - (1 << 20) - 1),  # positions up to 2^31 - 1
    (1, 64, 1, 1, 64, True, 1, 5),
])
def test_qkv_rope_matches_oracle(S, d, Hq, Hkv, D, norm, span, offset):
    x = _rand((S, d), S + d)
    Wq = _rand(((Hq + 2 * Hkv) * D, d), D + d, d ** -0.5)
    qn = (1.0 + 0.1 * _rand((D,), 3).float()).bfloat16() if norm else None
    kn = (1.0 + 0.1 * _rand((D,), 4).float()).bfloat16() if norm else None
    pos = _positions(S, span, S, offset)
    Q, K, V = tg.tg_qkv_rope(x.to(DEV), Wq.to(DEV), torch.as_tensor(pos).to(DEV), 1e6, Hq, Hkv, D,
                             qn.to(DEV) if norm else None, kn.to(DEV) if norm else None, 1e-6)
    rQ, rK, rV = oracle.qkv_rope(x, Wq, pos, 1e6, Hq, Hkv, D, qn, kn, 1e-6)
    assert_proj_close(Q.float().cpu().numpy(), rQ)
    assert_proj_close(K.float().cpu().numpy(), rK)
    assert_proj_close(V.float().cpu().numpy(), rV)
    assert tg.tg_get_device_error() == 0


def test_qkv_rope_small_base_and_zero_positions():
    """Base 10000 (every pair turns fast) and position 0 (no rotation) in one batch."""
    S, d, Hq, Hkv, D = 64, 128, 2, 2, 64
    x = _rand((S, d), 5)
    Wq = _rand(((Hq + 2 * Hkv) * D, d), 6, d ** -0.5)
    pos = np.arange(S, dtype=np.int32) * 977
    pos[::5] = 0
    Q, K, V = tg.tg_qkv_rope(x.to(DEV), Wq.to(DEV), torch.as_tensor(pos).to(DEV), 1e4, Hq, Hkv, D)
    rQ, rK, rV = oracle.qkv_rope(x, Wq, pos, 1e4, Hq, Hkv, D, eps=1e-6)
    for got, ref in ((Q, rQ), (K, rK), (V, rV)):
        assert_proj_close(got.float().cpu().numpy(), ref)


# =============================================================================== full size
def test_full_size_layer_projections_sampled_rows():
    """Qwen3-1.7B layer shapes at the 128k workload's kept count (8192 + 512 question rows):
    QKV [8704 x 2048] -> [4096] and the output projection [8704 x 2048] -> [2048] with the
    residual, in the launch configuration the bench times; sampled rows against the oracle."""
    w = W.get("qwen3_1p7b_n128k")
    S = 8704
    Wq, Wo, qn, kn = W.layer_weights(w)
    x = _rand((S, w.d), 11)
    pos = _positions(S, w.n, 12)
    Q, K, V = tg.tg_qkv_rope(x.to(DEV), Wq.to(DEV), torch.as_tensor(pos).to(DEV), w.rope_base, w.hq, w.hkv,
                             w.head_dim, qn.to(DEV), kn.to(DEV), w.norm_eps)
    rows = oracle.sampled_rows(S, seed=5, head=64, tail=64, rand=128)
    rQ, rK, rV = oracle.qkv_rope(x, Wq, pos, w.rope_base, w.hq, w.hkv, w.head_dim, qn, kn, w.norm_eps, rows=rows)
    assert_proj_close(Q.float().cpu().numpy()[rows], rQ)
    assert_proj_close(K.float().cpu().numpy()[rows], rK)
    assert_proj_close(V.float().cpu().numpy()[rows], rV)

    O = _rand((S, w.hq * w.head_dim), 13)
    y = tg.tg_linear(O.to(DEV), Wo.to(DEV), x.to(DEV))
    assert_proj_close(y.float().cpu().numpy()[rows], oracle.linear(O, Wo, x, rows=rows))
    assert tg.tg_get_device_error() == 0


# =============================================================================== a whole gated layer
@pytest.mark.parametrize("name,S", [("tiny_n512", 200), ("qwen3_1p7b_n16k", 1000)])
def test_gated_layer_chain(name, S):
    """hidden_k -> QKV + norm + rotary at the kept positions -> token-gated attention ->
    output projection + residual, all on the GPU, against the same chain on the oracle."""
    w = W.get(name)
    Wq, Wo, qn, kn = W.layer_weights(w)
    hidden, *_ = W.gate_inputs(w)
    kept = _positions(S, w.n, 21)
    hk, _ = oracle.gather(hidden, kept)
    hk = torch.from_numpy(hk.view(np.int16)).view(torch.bfloat16)
    s_k = W.random_scores(S, 22)
    gain, tau = W.attention_params(w)
    Hq, Hkv, D = w.hq, w.hkv, w.head_dim

    d_hk = hk.to(DEV)
    Q, K, V = tg.tg_qkv_rope(d_hk, Wq.to(DEV), torch.as_tensor(kept).to(DEV), w.rope_base, Hq, Hkv, D,
                             qn.to(DEV), kn.to(DEV), w.norm_eps)
    O = tg.tg_gated_attention(Q, K, V, s_k.to(DEV), gain.to(DEV), tau)
    y = tg.tg_linear(O.view(S, Hq * D), Wo.to(DEV), d_hk)

    rQ, rK, rV = oracle.qkv_rope(hk, Wq, kept, w.rope_base, Hq, Hkv, D, qn, kn, w.norm_eps)
    bf = lambda a: torch.as_tensor(a).to(torch.bfloat16)  # noqa: E731  the bf16 buffers between the calls
    rO = oracle.gated_attention(bf(rQ), bf(rK), bf(rV), s_k, gain, tau)
    ry = oracle.linear(bf(rO).reshape(S, Hq * D), Wo, hk)
    assert_proj_close(y.float().cpu().numpy(), ry, rtol=2.0 ** -7, rms_tol=1e-2)
    assert tg.tg_get_device_error() == 0

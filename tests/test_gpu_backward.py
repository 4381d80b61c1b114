"""Backward of token-gated attention (gradients w.r.t. key scores, gains and temperature)
and the forward's log-sum-exp, vs the fp64 CPU oracle, through the C ABI.

Two kinds of comparison, each with its own tolerance derived from the arithmetic.

Kernel parity: the GPU backward gets the oracle's own forward quantities (lse, and O
both as fp32 and rounded to bf16), so only its fp32 arithmetic remains: products of
bf16 values are exact, sums over <= 8704 terms in fp32, exp2 to ~2^-22 relative.
Expected errors are ~1e-5 of the outputs' scale; the bounds are
  * ds:    max |err| <= 2e-3 rms(ds),  mean |err| <= 2e-4 rms(ds);
  * dgain: max |err| <= 2e-3 rms(dgain);   dtau: |err| <= 2e-3 |dtau| + 1e-4.

Chained (GPU forward for training -> GPU backward): the backward then also carries the
forward's roundings: the lse built from bf16-rounded weights (2^-9 relative in the
row sum) and O (fp32 before rounding when kept, else bf16), which enter
Delta_i = dO_i . O_i.  Both move every dl_ij of a row with the same sign, so they do
not average out over rows.  Simulating exactly these roundings in fp64 gives at most
ds 1.7e-2 rms (max) and 2.8e-4 rms (mean), dgain 8.5e-3 of its rms and dtau 3.3e-2
relative (the last at tau = 2.5, where dtau is a small difference of large terms),
over S 256-700 and 2-16 heads with either O; at S = 8704 ds reaches 1.3e-2 rms with
the fp32 O but 9.2e-2 with the bf16 O at the first key (seen by every row), so the
full-length chained case keeps the fp32 O.  Bounds, with margin:
  * ds:    max |err| <= 3e-2 rms(ds),  mean |err| <= 1e-3 rms(ds);
  * dgain: max |err| <= 2e-2 rms(dgain);   dtau: |err| <= 5e-2 |dtau|;
  * lse:   |err| <= 4e-3 (the row sum's relative rounding, 2^-9, in log units).
The single-block chained cases (S = 2, 17) use small logits and drop the mean bound
(a mean over 2 keys is its max); the simulation gives at most ds 1.3e-2 rms, dgain
1.4e-2 rms and dtau 8.5e-3 there.
"""
import math

import numpy as np
import pytest
import torch

import oracle
import learned_token_pruning_mlp_b200 as tg
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


def _case(S, Hq, Hkv, D, seed, q_scale=1.0, s_scale=1.0):
    g = torch.Generator().manual_seed(seed)
    Q = (torch.randn(S, Hq, D, generator=g) * q_scale).to(torch.bfloat16)
    K = torch.randn(S, Hkv, D, generator=g).to(torch.bfloat16)
    V = torch.randn(S, Hkv, D, generator=g).to(torch.bfloat16)
    dO = torch.randn(S, Hq, D, generator=g).to(torch.bfloat16)
    s = torch.randn(S, generator=g) * s_scale
    gain = 0.5 + torch.rand(Hq, generator=g)
    return Q, K, V, dO, s, gain


def _gpu_backward(Q, K, V, dO, s, gain, tau, keep_fp32=True):
    """GPU forward for training, then the GPU backward (the chained path)."""
    d = [t.to(DEV) for t in (Q, K, V, dO, s, gain)]
    O, lse, O32 = tg.tg_gated_attention_train(d[0], d[1], d[2], d[4], d[5], tau, keep_fp32=keep_fp32)
    ds, dg, dt = tg.tg_gated_attention_backward(d[0], d[1], d[2], d[4], d[5], tau, O, d[3], lse, O32=O32)
    torch.cuda.synchronize()
    return O, lse, ds.cpu().numpy().astype(np.float64), dg.cpu().numpy().astype(np.float64), float(dt.item())


def _gpu_backward_on_oracle_forward(Q, K, V, dO, s, gain, tau):
    """The GPU backward fed with the oracle's forward (lse, fp32 O, bf16 O)."""
    O_ref = oracle.gated_attention(Q, K, V, s, gain, tau)
    lse_ref = oracle.gated_attention_lse(Q, K, s, gain, tau)
    O32 = torch.as_tensor(O_ref, dtype=torch.float32)
    d = [t.to(DEV) for t in (Q, K, V, dO, s, gain)]
    ds, dg, dt = tg.tg_gated_attention_backward(
        d[0], d[1], d[2], d[4], d[5], tau, O32.to(torch.bfloat16).to(DEV), d[3],
        torch.as_tensor(lse_ref, dtype=torch.float32).to(DEV), O32=O32.to(DEV))
    torch.cuda.synchronize()
    return ds.cpu().numpy().astype(np.float64), dg.cpu().numpy().astype(np.float64), float(dt.item())


def assert_grads_close(got, ref, mean_tol=1e-3, ds_tol=3e-2, dg_tol=2e-2, dt_tol=5e-2, dt_abs=0.0):
    ds, dg, dt = got
    rds, rdg, rdt = ref
    assert np.isfinite(ds).all() and np.isfinite(dg).all() and math.isfinite(dt)
    rms = math.sqrt(float(np.mean(rds ** 2)))
    e = np.abs(ds - rds)
    assert e.max() <= ds_tol * rms, f"ds max-err {e.max() / rms:.2e} rms"
    if mean_tol is not None:
        assert e.mean() <= mean_tol * rms, f"ds mean-err {e.mean() / rms:.2e} rms"
    grms = math.sqrt(float(np.mean(rdg ** 2)))
    assert np.max(np.abs(dg - rdg)) <= dg_tol * grms, f"dgain err {np.max(np.abs(dg - rdg)) / grms:.2e} rms"
    assert abs(dt - rdt) <= dt_tol * abs(rdt) + dt_abs, f"dtau {dt} vs {rdt}"


def assert_kernel_close(got, ref):
    assert_grads_close(got, ref, mean_tol=2e-4, ds_tol=2e-3, dg_tol=2e-3, dt_tol=2e-3, dt_abs=1e-4)


KERNEL_CASES = [(300, 4, 2, 64, 1.1), (700, 16, 8, 128, 1.1), (129, 2, 1, 128, 1.1), (1000, 16, 8, 128, -0.7),
                (256, 4, 4, 64, 2.5), (385, 8, 2, 128, 1.1), (200, 4, 2, 64, 0.0), (17, 2, 1, 64, 1.1),
                (2, 2, 1, 128, 1.1)]


@pytest.mark.parametrize("S,Hq,Hkv,D,tau", KERNEL_CASES)
def test_backward_kernel_matches_oracle(S, Hq, Hkv, D, tau):
    Q, K, V, dO, s, gain = _case(S, Hq, Hkv, D, S + Hq + 1000)
    got = _gpu_backward_on_oracle_forward(Q, K, V, dO, s, gain, tau)
    assert_kernel_close(got, oracle.gated_attention_backward(Q, K, V, s, gain, tau, dO))
    assert tg.tg_get_device_error() == 0


def test_backward_kernel_full_length_two_heads():
    """S = 8704 (the 128k workload's kept count) in the kernel configuration of the
    full-size run, two heads so the fp64 oracle finishes in seconds."""
    Q, K, V, dO, s, gain = _case(8704, 2, 1, 128, 12)
    got = _gpu_backward_on_oracle_forward(Q, K, V, dO, s, gain, 1.1)
    assert_kernel_close(got, oracle.gated_attention_backward(Q, K, V, s, gain, 1.1, dO))


@pytest.mark.parametrize("S,Hq,Hkv,D,tau", [(300, 4, 2, 64, 1.1), (700, 16, 8, 128, 1.1), (129, 2, 1, 128, 1.1),
                                            (1000, 16, 8, 128, -0.7), (256, 4, 4, 64, 2.5), (385, 8, 2, 128, 1.1)])
def test_backward_chained_matches_oracle(S, Hq, Hkv, D, tau):
    Q, K, V, dO, s, gain = _case(S, Hq, Hkv, D, S + Hq)
    _, _, ds, dg, dt = _gpu_backward(Q, K, V, dO, s, gain, tau)
    assert_grads_close((ds, dg, dt), oracle.gated_attention_backward(Q, K, V, s, gain, tau, dO))
    assert tg.tg_get_device_error() == 0


def test_backward_from_bf16_output():
    """Without the fp32 output the backward forms dO . O from the bf16 O (the same bounds
    hold at this length; the error grows with the number of rows a key is seen by)."""
    Q, K, V, dO, s, gain = _case(700, 16, 8, 128, 21)
    _, _, ds, dg, dt = _gpu_backward(Q, K, V, dO, s, gain, 1.1, keep_fp32=False)
    assert_grads_close((ds, dg, dt), oracle.gated_attention_backward(Q, K, V, s, gain, 1.1, dO))


def test_backward_zero_temperature():
    """tau = 0: logits are the biases alone; dtau still follows from q.k."""
    Q, K, V, dO, s, gain = _case(200, 4, 2, 64, 3)
    _, _, ds, dg, dt = _gpu_backward(Q, K, V, dO, s, gain, 0.0)
    assert_grads_close((ds, dg, dt), oracle.gated_attention_backward(Q, K, V, s, gain, 0.0, dO))


def test_backward_tiny_and_single_token():
    """One partial key block (1, 2 and 17 tokens).  With a handful of rows the rounding of
    O in Delta is not averaged out, and a row whose softmax is nearly one-hot has a tiny true
    gradient; small logits keep every row's weights spread, which is what these sizes test
    (masking of the padding keys and queries), not conditioning."""
    for S in (1, 2, 17):
        Q, K, V, dO, s, gain = _case(S, 2, 1, 64, 40 + S, q_scale=0.3, s_scale=0.3)
        _, _, ds, dg, dt = _gpu_backward(Q, K, V, dO, s, gain, 1.1)
        rds, rdg, rdt = oracle.gated_attention_backward(Q, K, V, s, gain, 1.1, dO)
        if S == 1:
            # one key: the softmax is constant and every gradient is zero; the GPU's dP (tensor
            # core) and Delta (prep kernel) sum the same 64 products in different fp32 orders
            assert np.all(np.abs(ds) <= 1e-4) and np.all(np.abs(dg) <= 1e-4) and abs(dt) <= 1e-4
        else:
            # a mean over 2 or 17 keys is no better than the max: only the max bounds apply
            assert_grads_close((ds, dg, dt), (rds, rdg, rdt), mean_tol=None)


def test_lse_matches_oracle_and_forward_unchanged():
    Q, K, V, dO, s, gain = _case(700, 16, 8, 128, 9)
    d = [t.to(DEV) for t in (Q, K, V, s, gain)]
    O, lse, O32 = tg.tg_gated_attention_train(d[0], d[1], d[2], d[3], d[4], 1.1)
    O2 = tg.tg_gated_attention(d[0], d[1], d[2], d[3], d[4], 1.1)
    torch.cuda.synchronize()
    assert torch.equal(O, O2)                      # the extra outputs do not change O
    assert torch.equal(O32.to(torch.bfloat16), O)  # O is the bf16 rounding of O32
    ref = oracle.gated_attention_lse(Q, K, s, gain, 1.1)
    assert np.max(np.abs(lse.cpu().numpy() - ref)) <= 4e-3
    # both outputs of the training forward within the forward's rounding budget (the fp32
    # output without the bf16 output rounding)
    check_attention(O.float().cpu().numpy(), Q, K, V, s, gain, 1.1)
    check_attention(O32.cpu().numpy(), Q, K, V, s, gain, 1.1, fp32_out=True)


def test_train_forward_varied_shapes_within_budget():
    for S, Hq, Hkv, D, tau in ((1000, 4, 2, 64, -0.7), (257, 8, 2, 128, 2.5)):
        Q, K, V, dO, s, gain = _case(S, Hq, Hkv, D, S + D)
        d = [t.to(DEV) for t in (Q, K, V, s, gain)]
        O, lse, O32 = tg.tg_gated_attention_train(d[0], d[1], d[2], d[3], d[4], tau)
        check_attention(O.float().cpu().numpy(), Q, K, V, s, gain, tau)
        check_attention(O32.cpu().numpy(), Q, K, V, s, gain, tau, fp32_out=True)
    assert tg.tg_get_device_error() == 0


def test_backward_is_deterministic_and_overwrites_outputs():
    Q, K, V, dO, s, gain = _case(500, 8, 4, 128, 11)
    d = [t.to(DEV) for t in (Q, K, V, dO, s, gain)]
    O, lse, O32 = tg.tg_gated_attention_train(d[0], d[1], d[2], d[4], d[5], 1.1)
    outs = []
    for fill in (0.0, 123.0):
        ds = torch.full((500,), fill, device=DEV)
        dg = torch.full((8,), fill, device=DEV)
        dt = torch.full((1,), fill, device=DEV)
        ws = torch.full((tg.tg_gated_attention_backward_workspace(500, 8),), 0xAB, dtype=torch.uint8, device=DEV)
        tg.tg_gated_attention_backward(d[0], d[1], d[2], d[4], d[5], 1.1, O, d[3], lse, O32, ds, dg, dt, workspace=ws)
        outs.append((ds.clone(), dg.clone(), dt.clone()))
    torch.cuda.synchronize()
    for a, b in zip(*outs):
        assert torch.equal(a, b)


def test_backward_chained_full_length_two_heads():
    """The chained path at S = 8704 with the fp32 O kept."""
    Q, K, V, dO, s, gain = _case(8704, 2, 1, 128, 12)
    _, _, ds, dg, dt = _gpu_backward(Q, K, V, dO, s, gain, 1.1)
    assert_grads_close((ds, dg, dt), oracle.gated_attention_backward(Q, K, V, s, gain, 1.1, dO))


def test_backward_full_size_invariant():
    """S = 8704, 16 heads: a constant added to every score leaves each softmax row unchanged,
    so sum_j ds_j = 0 up to rounding."""
    Q, K, V, dO, s, gain = _case(8704, 16, 8, 128, 13)
    _, _, ds, dg, dt = _gpu_backward(Q, K, V, dO, s, gain, 1.1)
    assert np.isfinite(ds).all() and np.isfinite(dg).all() and math.isfinite(dt)
    assert abs(ds.sum()) <= 1e-3 * np.abs(ds).sum()
    assert tg.tg_get_device_error() == 0
